"""Bulk encode and decode (the tensor-core kernels) against the fp64 oracle
over seven input distributions that stress different parts of the exactness
argument: heavy tails, per-channel scales spanning decades, outlier channels,
elements spread over 2^28 in magnitude (the tensor core's addend cut),
sparse rows, and rows dominated by a common offset (needs a B200)."""

import zlib

import numpy as np
import pytest
import torch

import oracle as O
from parity import assert_decode_ulp, assert_norms, code_mismatches

pytestmark = pytest.mark.gpu

N, SAMPLE = 131072, 16384


@pytest.fixture(scope="module")
def K(cuda_device):
    import kv_cache_vector_turboquant_b200 as K

    return K


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_stress_distributions_match_oracle(K, d, bits):
    import tq_workloads as W

    tq = K.TurboQuant(d, bits)
    for kind in W.STRESS_KINDS:
        seed = zlib.crc32(f"{kind}/{d}/{bits}".encode()) & 0xFFFF
        x = W.stress_rows(kind, N, d, seed)
        packed, norms = tq.encode(x)  # a bulk call: the tensor-core kernel
        dec = tq.decode(packed, norms)
        torch.cuda.synchronize()
        rows = torch.randperm(N, generator=torch.Generator().manual_seed(seed))[:SAMPLE].sort().values.cuda()
        det = O.encode_detail(x[rows].cpu().numpy(), bits, 42)
        gp, gn = packed[rows].cpu().numpy(), norms[rows].cpu().numpy()
        assert code_mismatches(gp, det, bits, d) == 0, kind
        assert_norms(gn, det)
        ref = O.decode(gp, gn, bits, 42, d)
        fin = np.isfinite(ref).all(axis=1)
        assert_decode_ulp(dec[rows].cpu().numpy()[fin], ref[fin])
    assert K.tq_device_error() == (K.TQ_OK, 0)
