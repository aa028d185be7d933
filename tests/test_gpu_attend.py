"""Fused decode-step attention over packed caches vs the oracle's
decode-then-attend in fp64 (needs a B200)."""

import numpy as np
import pytest
import torch

import oracle as O
from parity import ATTN_RTOL, attn_row_error

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K(cuda_device):
    import kv_cache_vector_turboquant_b200 as K

    return K


@pytest.fixture(scope="module")
def W():
    import tq_workloads as W

    return W


def _make_cache(K, W, B, S, hkv, d, kb, vb, seed):
    kc, vc = K.TurboQuant(d, kb), K.TurboQuant(d, vb)
    k = W.randn_f16((B, S, hkv, d), seed, "cuda")
    v = W.randn_f16((B, S, hkv, d), seed + 1, "cuda")
    kp, kn = kc.encode(k)
    vp, vn = vc.encode(v)
    return kc, vc, kp, kn, vp, vn


def _oracle(q, kp, kn, vp, vn, pos, kb, vb, batches=None):
    qn = q.cpu().numpy()
    if batches is None:
        batches = range(q.shape[0])
    out = {}
    for b in batches:
        o = O.attend_decode(qn[b:b + 1], kp[b:b + 1].cpu().numpy(), kn[b:b + 1].cpu().numpy(),
                            vp[b:b + 1].cpu().numpy(), vn[b:b + 1].cpu().numpy(), [int(pos[b])], kb, vb)
        out[b] = o[0]
    return out


CASES = [
    # d, kb, vb, B, S, hq, hkv, positions
    (128, 4, 2, 3, 200, 8, 2, [200, 1, 77]),
    (128, 3, 3, 2, 97, 32, 8, [97, 33]),
    (64, 4, 4, 2, 64, 4, 4, [64, 31]),
    (64, 2, 3, 2, 130, 16, 2, [5, 130]),
    (256, 4, 2, 2, 70, 8, 1, [70, 64]),
    (256, 2, 4, 1, 40, 16, 2, [40]),
    (128, 2, 2, 2, 50, 16, 16, [50, 17]),  # two groups of 8 kv heads
    (128, 4, 3, 1, 1000, 4, 1, [999]),
    # 4-bit K / 2-bit V with 4, 8 or 16 kv heads: the fast kernel (tensor-map
    # tiles, one CTA per SM, two warp groups or two column tiles per head)
    (128, 4, 2, 3, 200, 32, 8, [200, 1, 77]),
    (128, 4, 2, 2, 333, 32, 4, [333, 160]),  # 8 query heads per kv head
    (128, 4, 2, 2, 150, 16, 16, [150, 33]),  # two groups of 8 kv heads
    (256, 4, 2, 2, 300, 16, 8, [300, 257]),
    (256, 4, 2, 1, 129, 64, 8, [129]),
]


@pytest.mark.parametrize("d,kb,vb,B,S,hq,hkv,pos", CASES)
def test_attention_matches_oracle(K, W, d, kb, vb, B, S, hq, hkv, pos):
    kc, vc, kp, kn, vp, vn = _make_cache(K, W, B, S, hkv, d, kb, vb, seed=d + kb * 10 + vb + S)
    q = W.randn_f16((B, hq, d), 99 + B, "cuda", scale=1.0 / np.sqrt(d))
    positions = torch.tensor(pos, dtype=torch.int32, device="cuda")
    o = K.attend_decode(q, kc, vc, kp, kn, vp, vn, positions)
    torch.cuda.synchronize()
    ref = _oracle(q, kp, kn, vp, vn, pos, kb, vb)
    on = o.cpu().numpy().astype(np.float64)
    for b, r in ref.items():
        err = attn_row_error(on[b], r)
        assert err.max() <= ATTN_RTOL, (b, err.max())
    assert K.tq_device_error() == (K.TQ_OK, 0)


def test_sharp_attention(K, W):
    """Large query norms: softmax concentrated on a few positions."""
    d, kb, vb, B, S, hq, hkv = 128, 4, 2, 2, 300, 8, 2
    kc, vc, kp, kn, vp, vn = _make_cache(K, W, B, S, hkv, d, kb, vb, seed=5)
    q = W.randn_f16((B, hq, d), 6, "cuda", scale=3.0)
    pos = [300, 150]
    o = K.attend_decode(q, kc, vc, kp, kn, vp, vn, torch.tensor(pos, dtype=torch.int32, device="cuda"))
    ref = _oracle(q, kp, kn, vp, vn, pos, kb, vb)
    for b, r in ref.items():
        assert attn_row_error(o[b].cpu().numpy(), r).max() <= ATTN_RTOL


def test_single_position_returns_decoded_value(K, W):
    d, B, S, hq, hkv = 128, 2, 64, 8, 2
    kc, vc, kp, kn, vp, vn = _make_cache(K, W, B, S, hkv, d, 4, 2, seed=8)
    q = W.randn_f16((B, hq, d), 9, "cuda")
    o = K.attend_decode(q, kc, vc, kp, kn, vp, vn, torch.ones(B, dtype=torch.int32, device="cuda"))
    V = O.decode_f64(vp[:, 0].cpu().numpy(), vn[:, 0].cpu().numpy(), 2, 42, d)  # [B, hkv, d]
    on = o.cpu().numpy().astype(np.float64)
    for b in range(B):
        for h in range(hq):
            ref = V[b, h // (hq // hkv)]
            assert np.abs(on[b, h] - ref).max() <= 1e-3 * np.abs(ref).max()


def test_positions_edge_cases(K, W):
    d, B, S, hq, hkv = 128, 3, 96, 8, 2
    kc, vc, kp, kn, vp, vn = _make_cache(K, W, B, S, hkv, d, 4, 2, seed=10)
    q = W.randn_f16((B, hq, d), 11, "cuda")
    K.tq_device_error()
    pos = torch.tensor([0, S + 50, S], dtype=torch.int32, device="cuda")
    o = K.attend_decode(q, kc, vc, kp, kn, vp, vn, pos)
    st, bits = K.tq_device_error()
    assert st == K.TQ_ERR_DEVICE and bits & K.TQ_DEVERR_POS_RANGE
    assert torch.all(o[0] == 0)  # empty context -> zero row
    ref = _oracle(q, kp, kn, vp, vn, [0, S, S], 4, 2, batches=[1, 2])
    for b, r in ref.items():  # a position past the cache is clamped to S
        assert attn_row_error(o[b].cpu().numpy(), r).max() <= ATTN_RTOL


def test_decode_step_workload_sampled(K, W):
    """The benchmarked decode step: q [16,32,128], K (4 bits) / V (2 bits)
    caches of 32768 positions x 8 kv heads, encoded on the GPU; all 32 heads
    of all 16 sequences against the oracle."""
    q, k, v = W.decode_step()
    kc, vc = K.TurboQuant(128, 4), K.TurboQuant(128, 2)
    kp, kn = kc.encode(k)
    vp, vn = vc.encode(v)
    del k, v
    pos = torch.full((16,), 32768, dtype=torch.int32, device="cuda")
    o = K.attend_decode(q, kc, vc, kp, kn, vp, vn, pos)
    torch.cuda.synchronize()
    ref = _oracle(q, kp, kn, vp, vn, pos.cpu().numpy(), 4, 2)
    assert len(ref) == 16
    for b, r in ref.items():
        err = attn_row_error(o[b].cpu().numpy(), r)
        assert err.max() <= ATTN_RTOL, (b, err.max())
    assert K.tq_device_error() == (K.TQ_OK, 0)


@pytest.mark.parametrize("hkv,hq", [(8, 32), (4, 32)])
def test_many_tiles_per_split(K, W, hkv, hq):
    """Splits of 15+ tiles of 32 positions, so every stage of the fast
    kernel's pipeline is refilled several times; ragged positions."""
    d, B, S = 128, 16, 4096
    kc, vc, kp, kn, vp, vn = _make_cache(K, W, B, S, hkv, d, 4, 2, seed=40 + hkv)
    q = W.randn_f16((B, hq, d), 41, "cuda", scale=1.0 / np.sqrt(d))
    rng = np.random.default_rng(42)
    pos = rng.integers(1, S + 1, size=B)
    pos[0], pos[5] = S, 4000
    positions = torch.tensor(pos, dtype=torch.int32, device="cuda")
    o = K.attend_decode(q, kc, vc, kp, kn, vp, vn, positions)
    torch.cuda.synchronize()
    ref = _oracle(q, kp, kn, vp, vn, pos, 4, 2, batches=[0, 5, 9, 15])
    for b, r in ref.items():
        err = attn_row_error(o[b].cpu().numpy(), r)
        assert err.max() <= ATTN_RTOL, (b, err.max())
    assert K.tq_device_error() == (K.TQ_OK, 0)


PAGED_CASES = [
    # d, kb, vb, B, S (multiple of 16), hq, hkv, context lengths
    (128, 4, 2, 3, 256, 32, 8, [256, 1, 77]),   # fast kernel
    (256, 4, 2, 2, 160, 16, 8, [160, 129]),     # fast kernel, head_dim 256
    (128, 4, 2, 2, 96, 32, 4, [96, 40]),        # fast kernel, 8 query heads per kv head
    (128, 3, 3, 2, 112, 32, 8, [112, 33]),      # generic kernel
    (64, 2, 4, 2, 64, 8, 2, [17, 64]),          # generic kernel, head_dim 64
]


def _to_pages(t, perm):
    """[B, S, ...] contiguous cache -> pool [B*S/16, 16, ...] with logical block
    j of sequence b stored at physical block perm[b * S/16 + j]."""
    B, S = t.shape[0], t.shape[1]
    blocks = t.reshape(B * S // 16, 16, *t.shape[2:])
    pool = torch.empty_like(blocks)
    pool[perm] = blocks
    return pool


@pytest.mark.parametrize("d,kb,vb,B,S,hq,hkv,lens", PAGED_CASES)
def test_paged_attention_matches_contiguous_and_oracle(K, W, d, kb, vb, B, S, hq, hkv, lens):
    """Paged caches with the blocks scattered by a random permutation: output
    bit-identical to tq_attend_decode on the contiguous cache (same tiles, same
    arithmetic) and within the tolerance of the oracle's paged attention."""
    kc, vc, kp, kn, vp, vn = _make_cache(K, W, B, S, hkv, d, kb, vb, seed=3 * d + kb + vb + S)
    q = W.randn_f16((B, hq, d), 7 + B, "cuda", scale=1.0 / np.sqrt(d))
    lens_t = torch.tensor(lens, dtype=torch.int32, device="cuda")
    nb = S // 16
    perm = torch.randperm(B * nb, generator=torch.Generator().manual_seed(d + S)).cuda()
    kpool, vpool = _to_pages(kp, perm), _to_pages(vp, perm)
    knpool, vnpool = _to_pages(kn, perm), _to_pages(vn, perm)
    bt = perm.reshape(B, nb).to(torch.int32)
    # table entries past each context are never read: fill them with garbage
    for b, n in enumerate(lens):
        bt[b, (n + 15) // 16:] = -12345
    o_paged = K.attend_decode_paged(q, kc, vc, kpool, knpool, vpool, vnpool, bt, lens_t)
    o_contig = K.attend_decode(q, kc, vc, kp, kn, vp, vn, lens_t)
    # the pages' class form of the same call
    o_class = K.TQPagedAttention(kc, hq, v_tq=vc).forward(q, kpool, knpool, vpool, vnpool, bt, lens_t)
    torch.cuda.synchronize()
    assert torch.equal(o_paged, o_contig)
    assert torch.equal(o_class, o_paged)
    assert K.tq_device_error() == (K.TQ_OK, 0)
    ref = O.attend_decode_paged(q.cpu().numpy(), kpool.cpu().numpy(), knpool.cpu().numpy(), vpool.cpu().numpy(),
                                vnpool.cpu().numpy(), bt.cpu().numpy(), lens, kb, vb)
    err = attn_row_error(o_paged.cpu().numpy().astype(np.float64), ref)
    assert err.max() <= ATTN_RTOL, err.max()


def test_paged_attention_out_of_range_block_is_clamped_and_flagged(K, W):
    d, B, S, hq, hkv = 128, 1, 64, 32, 8
    kc, vc, kp, kn, vp, vn = _make_cache(K, W, B, S, hkv, d, 4, 2, seed=5)
    q = W.randn_f16((B, hq, d), 8, "cuda", scale=1.0 / np.sqrt(d))
    bt = torch.tensor([[0, 1, 99, 3]], dtype=torch.int32, device="cuda")  # block 99 of 4
    lens = torch.tensor([64], dtype=torch.int32, device="cuda")
    o = K.attend_decode_paged(q, kc, vc, kp.reshape(4, 16, hkv, -1), kn.reshape(4, 16, hkv),
                              vp.reshape(4, 16, hkv, -1), vn.reshape(4, 16, hkv), bt, lens)
    torch.cuda.synchronize()
    st, bits = K.tq_device_error()
    assert st == K.TQ_ERR_DEVICE and bits == K.TQ_DEVERR_BLOCK_RANGE
    assert torch.isfinite(o.float()).all()
