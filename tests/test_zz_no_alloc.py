"""tq_attend_decode_static: the attention entry point that allocates nothing.

Callers such as a plugin inside a framework that owns all device memory, or a
decode loop that must not call cudaMalloc, use this entry point: its split-S
scratch is the library's own fixed device array instead of a caller-supplied
workspace. These tests call it through the C ABI twice in a row, with
different queries, and compare each result with the workspace-taking entry
point on the same inputs. The file is named so that pytest collects it last.
"""

import numpy as np
import pytest
import torch

from parity import ATTN_RTOL, attn_row_error

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K(cuda_device):
    import kv_cache_vector_turboquant_b200 as K

    return K


def test_static_scratch_matches_workspace_entry_point(K):
    from kv_cache_vector_turboquant_b200 import workloads as W

    B, S, hq, hkv, d = 4, 777, 8, 2, 128
    kc, vc = K.TurboQuant(d, 4), K.TurboQuant(d, 2)
    kp, kn = kc.encode(W.randn_f16((B, S, hkv, d), 31, "cuda"))
    vp, vn = vc.encode(W.randn_f16((B, S, hkv, d), 32, "cuda"))
    pos = torch.tensor([S, 1, 400, 129], dtype=torch.int32, device="cuda")
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
        o, r = out.cpu().numpy().astype(np.float64), ref.cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(o)), call
        err = max(attn_row_error(o[b], r[b]).max() for b in range(B))
        assert err <= ATTN_RTOL, (call, err)
    assert K.tq_device_error() == (K.TQ_OK, 0)


def test_static_scratch_rejects_oversized_calls(K):
    # a batch whose split-S scratch exceeds the fixed array: rejected on the
    # host, nothing launched (the pointers are never dereferenced)
    kc, vc = K.TurboQuant(128, 4), K.TurboQuant(128, 2)
    B, hq, S = 256, 64, 1 << 20
    assert K.tq_attend_workspace_bytes(B, hq, 128, S) > K.TQ_ATTEND_STATIC_SCRATCH_BYTES
    A = 0x100000
    st = K._binding._lib.tq_attend_decode_static(kc.ctx.handle, vc.ctx.handle, A, B, hq, 8, A, A, A, A, S, A, A,
                                                 None)
    assert st == K.TQ_ERR_WORKSPACE
