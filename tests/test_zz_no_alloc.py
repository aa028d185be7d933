"""tq_attend_decode_static: the attention entry point that allocates nothing.

Callers such as a plugin inside a framework that owns all device memory, or a
decode loop that must not call cudaMalloc, use this entry point: its split-S
scratch is the library's own fixed device array instead of a caller-supplied
workspace. These tests call it through the C ABI twice in a row, with
different queries, and compare each result with the workspace-taking entry
point on the same inputs: the kernels, split geometry and scratch layout are
the same, so the outputs must be bit-identical. One case takes the generic
partial kernel, the other the fast 4-bit-K / 2-bit-V kernel of the
benchmarked decode step. The file is named so that pytest collects it last.
"""

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K(cuda_device):
    import kv_cache_vector_turboquant_b200 as K

    return K


# (B, S, hq, hkv, d, K bits, V bits, positions): hkv = 2 is not a multiple of
# the fast kernel's kv-head groups (generic kernel); hkv = 8 with 4-bit keys
# and 2-bit values is the fast kernel's case
CASES = {
    "generic": (4, 777, 8, 2, 128, 4, 2, [777, 1, 400, 129]),
    "fast": (3, 1000, 32, 8, 128, 4, 2, [1000, 33, 517]),
}


@pytest.mark.parametrize("case", sorted(CASES))
def test_static_scratch_matches_workspace_entry_point(K, case):
    import tq_workloads as W

    B, S, hq, hkv, d, kb, vb, lens = CASES[case]
    kc, vc = K.TurboQuant(d, kb), K.TurboQuant(d, vb)
    kp, kn = kc.encode(W.randn_f16((B, S, hkv, d), 31, "cuda"))
    vp, vn = vc.encode(W.randn_f16((B, S, hkv, d), 32, "cuda"))
    pos = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ws_bytes = K.tq_attend_workspace_bytes(B, hq, d, S)
    assert 0 < ws_bytes <= K.TQ_ATTEND_STATIC_SCRATCH_BYTES
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device="cuda")
    for call, seed in enumerate((33, 34)):  # two calls in a row, different queries
        q = W.randn_f16((B, hq, d), seed, "cuda", scale=d ** -0.5)
        ref = torch.empty_like(q)
        K.tq_attend_decode(kc.ctx, vc.ctx, q, B, hq, hkv, kp, kn, vp, vn, S, pos, ref, ws, ws_bytes)
        out = torch.full_like(q, float("nan"))
        K.tq_attend_decode_static(kc.ctx, vc.ctx, q, B, hq, hkv, kp, kn, vp, vn, S, pos, out)
        torch.cuda.synchronize()
        assert torch.isfinite(out).all(), call
        assert torch.equal(out, ref), (call, (out.float() - ref.float()).abs().max().item())
    assert K.tq_device_error() == (K.TQ_OK, 0)


def test_static_scratch_rejects_oversized_calls(K):
    """A batch whose split-S scratch exceeds the fixed array by a few bytes is
    rejected on the host and nothing is launched. The buffers are real and of
    the sizes the call describes, with every sequence empty, so that even a
    launch would read and write inside them."""
    B, S, hq, hkv, d = 109, 32, 148, 37, 128
    need = K.tq_attend_workspace_bytes(B, hq, d, S)
    assert K.TQ_ATTEND_STATIC_SCRATCH_BYTES < need <= K.TQ_ATTEND_STATIC_SCRATCH_BYTES + 64
    kc, vc = K.TurboQuant(d, 4), K.TurboQuant(d, 2)
    q = torch.zeros(B, hq, d, dtype=torch.float16, device="cuda")
    out = torch.zeros_like(q)
    kp = torch.zeros(B, S, hkv, kc.packed_bytes, dtype=torch.uint8, device="cuda")
    vp = torch.zeros(B, S, hkv, vc.packed_bytes, dtype=torch.uint8, device="cuda")
    kn = torch.zeros(B, S, hkv, dtype=torch.float32, device="cuda")
    vn = torch.zeros_like(kn)
    pos = torch.zeros(B, dtype=torch.int32, device="cuda")
    torch.cuda.synchronize()
    st = K._binding._lib.tq_attend_decode_static(kc.ctx.handle, vc.ctx.handle, q.data_ptr(), B, hq, hkv,
                                                 kp.data_ptr(), kn.data_ptr(), vp.data_ptr(), vn.data_ptr(), S,
                                                 pos.data_ptr(), out.data_ptr(), None)
    assert st == K.TQ_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert K.tq_device_error() == (K.TQ_OK, 0)
    assert np.all(out.cpu().numpy() == 0)
