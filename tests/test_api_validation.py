"""The Python API refuses malformed tensor arguments before any pointer
reaches the library: wrong dtypes, layouts or sizes (which would let a kernel
read or write past a buffer) and host tensors (which a kernel cannot
address). Runs on the CPU: every refusal happens before a CUDA call."""

import pytest
import torch


@pytest.fixture(scope="module")
def K():
    import kv_cache_vector_turboquant_b200 as K

    return K


@pytest.fixture(scope="module")
def tq(K):
    return K.TurboQuant(128, 4)


def _raises(fn, text):
    with pytest.raises(ValueError, match=text):
        fn()


def test_codec_calls_refuse_host_tensors(tq):
    x = torch.zeros(4, 128, dtype=torch.float16)
    _raises(lambda: tq.encode(x), "CUDA")
    _raises(lambda: tq.encode_os(x), "CUDA")
    _raises(lambda: tq.decode(torch.zeros(4, 64, dtype=torch.uint8), torch.zeros(4)), "CUDA")
    _raises(lambda: tq.decode_os(torch.zeros(4, 64, dtype=torch.uint8), torch.zeros(4, dtype=torch.int32)), "CUDA")


def test_codec_calls_check_dtypes_and_sizes(tq):
    _raises(lambda: tq.encode_os(torch.zeros(4, 128, dtype=torch.float32)), "dtype")
    _raises(lambda: tq.encode_os(torch.zeros(4, 64, dtype=torch.float16)), "head_dim")
    _raises(lambda: tq.decode_os(torch.zeros(4, 64, dtype=torch.uint8), torch.zeros(3, dtype=torch.int32)),
            "elements")
    _raises(lambda: tq.decode_os(torch.zeros(4, 64, dtype=torch.uint8), torch.zeros(4, dtype=torch.float32)),
            "dtype")
    _raises(lambda: tq.decode_os(torch.zeros(4, 32, dtype=torch.uint8), torch.zeros(4, dtype=torch.int32)),
            "head_dim")


def test_append_checks_cache_shapes_then_device(tq):
    n_seq, s_max, h = 3, 8, 2
    x = torch.zeros(n_seq, h, 128, dtype=torch.float16)
    cache = torch.zeros(n_seq, s_max, h, 64, dtype=torch.uint8)
    cn = torch.zeros(n_seq, s_max, h, dtype=torch.float32)
    slot = torch.zeros(n_seq, dtype=torch.int32)
    _raises(lambda: tq.encode_append(x, cache[..., :32].contiguous(), cn, slot), "shape")
    _raises(lambda: tq.encode_append(x, cache, cn[:, :4].contiguous(), slot), "shape")
    _raises(lambda: tq.encode_append(x, cache, cn, slot[:2]), "elements")
    _raises(lambda: tq.encode_append(x, cache, cn, slot.long()), "dtype")
    _raises(lambda: tq.encode_append(x, cache, cn, slot), "CUDA")
    _raises(lambda: tq.encode_append_kv(x, x, cache, cn, cache, cn, slot), "CUDA")
    _raises(lambda: tq.encode_append_kv(x, x[:2], cache, cn, cache, cn, slot), "n_seq")


def test_slots_check_pool_and_mapping(tq):
    x = torch.zeros(5, 2, 128, dtype=torch.float16)
    pool = torch.zeros(4, 16, 2, 64, dtype=torch.uint8)
    pn = torch.zeros(4, 16, 2, dtype=torch.float32)
    m = torch.zeros(5, dtype=torch.int32)
    _raises(lambda: tq.encode_slots(x, pool, pn[:2].contiguous(), m), "elements")
    _raises(lambda: tq.encode_slots(x, pool, pn, m[:4]), "elements")
    _raises(lambda: tq.encode_slots(x, pool, pn, m), "CUDA")


def test_attention_checks_every_operand(K):
    kc, vc = K.TurboQuant(128, 4), K.TurboQuant(128, 2)
    B, S, hkv, hq = 2, 32, 2, 8
    q = torch.zeros(B, hq, 128, dtype=torch.float16)
    kp = torch.zeros(B, S, hkv, 64, dtype=torch.uint8)
    vp = torch.zeros(B, S, hkv, 32, dtype=torch.uint8)
    kn = torch.zeros(B, S, hkv, dtype=torch.float32)
    vn = torch.zeros(B, S, hkv, dtype=torch.float32)
    pos = torch.full((B,), S, dtype=torch.int32)
    _raises(lambda: K.attend_decode(q, kc, vc, vp, kn, vp, vn, pos), "k_packed: shape")  # V's row size as K's
    _raises(lambda: K.attend_decode(q, kc, vc, kp, kn, vp, vn[:, :16].contiguous(), pos), "v_norms: shape")
    _raises(lambda: K.attend_decode(q, kc, vc, kp, kn, vp, vn, pos.long()), "positions: dtype")
    _raises(lambda: K.attend_decode(q, kc, vc, kp, kn, vp, vn, pos, out=torch.zeros(B, hq, 64,
                                                                                    dtype=torch.float16)), "out")
    _raises(lambda: K.attend_decode(q, kc, vc, kp, kn, vp, vn, pos), "CUDA")
    # paged: pools of 16-position blocks and [B, max_blocks] tables
    kpool, vpool = kp.reshape(B * S // 16, 16, hkv, 64), vp.reshape(B * S // 16, 16, hkv, 32)
    knp, vnp = kn.reshape(B * S // 16, 16, hkv), vn.reshape(B * S // 16, 16, hkv)
    bt = torch.zeros(B, S // 16, dtype=torch.int32)
    _raises(lambda: K.attend_decode_paged(q, kc, vc, kpool, knp, vpool, vnp, bt.long(), pos), "block_tables")
    _raises(lambda: K.attend_decode_paged(q, kc, vc, kpool, knp, vpool, vnp, bt, pos[:1]), "context_lens")
    _raises(lambda: K.attend_decode_paged(q, kc, vc, kpool, knp, vpool, vnp, bt, pos), "CUDA")
    _raises(lambda: K.TQPagedAttention(kc, hq, v_tq=vc)(q, kpool, knp, vpool, vnp, bt, pos), "CUDA")
