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
    from kv_cache_vector_turboquant_b200 import workloads as W

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
    of two sequences against the oracle."""
    q, k, v = W.decode_step()
    kc, vc = K.TurboQuant(128, 4), K.TurboQuant(128, 2)
    kp, kn = kc.encode(k)
    vp, vn = vc.encode(v)
    del k, v
    pos = torch.full((16,), 32768, dtype=torch.int32, device="cuda")
    o = K.attend_decode(q, kc, vc, kp, kn, vp, vn, pos)
    torch.cuda.synchronize()
    ref = _oracle(q, kp, kn, vp, vn, pos.cpu().numpy(), 4, 2, batches=[0, 15])
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
