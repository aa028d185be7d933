"""The tensor-core encode kernel against the fp64 oracle (needs a B200).

tq_encode runs this kernel from 128 x SM-count vectors on; the test hook
tq_test_encode_path runs it (path 2) or the CUDA-core kernel (path 1) at any
size, so ragged and small cases reach it too.
"""

import math

import numpy as np
import pytest
import torch

import oracle as O
from parity import assert_decode_ulp, assert_norms, code_mismatches

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K(cuda_device):
    import kv_cache_vector_turboquant_b200 as K

    return K


@pytest.fixture(scope="module")
def W():
    import tq_workloads as W

    return W


def _enc_path(K, tq, x, path):
    n = x.shape[0]
    packed = torch.zeros(n, tq.packed_bytes, dtype=torch.uint8, device="cuda")
    norms = torch.zeros(n, dtype=torch.float32, device="cuda")
    assert K._binding.tq_test_encode_path(tq.ctx, x, n, packed, norms, path) == K.TQ_OK
    torch.cuda.synchronize()
    return packed, norms


def _parity(K, x_cpu, d, bits, max_boundary_frac=1e-6):
    tq = K.TurboQuant(d, bits)
    packed, norms = _enc_path(K, tq, x_cpu.cuda(), 2)
    det = O.encode_detail(x_cpu.numpy(), bits, 42)
    gp, gn = packed.cpu().numpy(), norms.cpu().numpy()
    n_mis = code_mismatches(gp, det, bits, d, max_boundary_frac)
    assert_norms(gn, det)
    assert K.tq_device_error() == (K.TQ_OK, 0)
    # decode of the kernel's own bytes vs the oracle decode of the same bytes
    xd = tq.decode(packed, norms)
    torch.cuda.synchronize()
    assert_decode_ulp(xd.cpu().numpy(), O.decode(gp, gn, bits, 42, d))
    return n_mis, gp, gn


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("n", [1, 127, 128, 129, 4103])
def test_tc_ragged_sizes(K, W, d, bits, n):
    """Partial tiles (the tensor copies fill missing rows with zeros, which
    are not stored), one tile, a tile and one row, 33 tiles."""
    x = W.single_tensor(n=n, d=d, seed=2000 + n + d + bits, outlier_frac=0.05)
    n_mis, _, _ = _parity(K, x, d, bits)
    assert n_mis == 0


@pytest.mark.parametrize("d,per_cta", [(64, 13), (128, 9), (256, 5)])
def test_tc_many_tiles_per_cta(K, W, d, per_cta):
    """Enough tiles that every CTA cycles its stage ring, its tensor-memory
    accumulators and all three epilogue warpgroups several times, with a
    ragged last tile; every row against the oracle, and the same codes as the
    CUDA-core kernel."""
    n = 148 * 128 * per_cta + 77
    x = W.single_tensor(n=n, d=d, seed=31 + d, outlier_frac=0.02)
    n_mis, gp, gn = _parity(K, x, d, 4)
    assert n_mis == 0
    tq = K.TurboQuant(d, 4)
    p1, n1 = _enc_path(K, tq, x.cuda(), 1)
    assert np.array_equal(p1.cpu().numpy(), gp)
    np.testing.assert_allclose(n1.cpu().numpy(), gn, rtol=2e-6)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_tc_degenerate_vectors(K, W, d, bits):
    """Zero, constant, spike, fp16-max, subnormal and alternating rows; exact
    ties at a boundary occur (z = 0 exactly), so only the band rule applies."""
    x = W.edge_vectors(d)
    _parity(K, x, d, bits, max_boundary_frac=None)
    tq = K.TurboQuant(d, bits)
    packed, norms = _enc_path(K, tq, x[:1].cuda(), 2)
    idx = O.unpack_codes(packed.cpu().numpy(), bits, d)
    assert norms.item() == 0.0 and np.all(idx == (1 << bits) // 2)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_tc_signed_hadamard_rows_rotate_to_spikes(K, d):
    """x = D r_k rotates to z = sqrt(d) e_k: code L-1 at k, 2^(b-1) elsewhere
    (the exact zeros of the other coordinates go up)."""
    import scipy.linalg

    s = O.sign_vector(42, d)
    R = scipy.linalg.hadamard(d)
    ks = list(range(0, d, max(1, d // 16)))
    rows = np.stack([s * R[k] for k in ks]).astype(np.float16)
    for bits in (2, 3, 4):
        tq = K.TurboQuant(d, bits)
        packed, norms = _enc_path(K, tq, torch.from_numpy(rows).cuda(), 2)
        idx = O.unpack_codes(packed.cpu().numpy(), bits, d)
        for r, k in enumerate(ks):
            want = np.full(d, (1 << bits) // 2)
            want[k] = (1 << bits) - 1
            assert np.array_equal(idx[r], want)
        assert np.allclose(norms.cpu().numpy(), math.sqrt(d), rtol=1e-6)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_tc_block_spikes_with_fine_residue(K, d):
    """The tensor core cuts each addend of a 16-term sum at 2^(E-25) below the
    largest exponent E. Rows with one large entry per 16-coordinate block and
    fifteen small entries full of low-order bits lose the most there, and
    their rotated values crowd the boundary at z = 0 (the large entries
    cancel in most coordinates); every code must still be the oracle's."""
    g = np.random.default_rng(d)
    n = 4096
    x = (g.standard_normal((n, d)) * 2.0 ** -6).astype(np.float64)
    pos = g.integers(0, 16, size=(n, d // 16))
    big = 512.0 * (1.0 + g.integers(0, 4, size=(n, d // 16)))
    sgn = np.where(g.integers(0, 2, size=(n, d // 16)) == 1, 1.0, -1.0)
    for b in range(d // 16):
        x[np.arange(n), 16 * b + pos[:, b]] = sgn[:, b] * big[:, b]
    x16 = torch.from_numpy(x.astype(np.float16))
    for bits in (2, 4):
        _parity(K, x16, d, bits, max_boundary_frac=None)


@pytest.mark.parametrize("d,bits", [(64, 4), (128, 2), (128, 3), (128, 4), (256, 4)])
def test_tc_output_rows_at_16_but_not_32_byte_alignment(K, W, d, bits):
    """Rows whose size is a multiple of 32 bytes are written with 32-byte
    stores only from a 32-byte aligned base; a base that is 16-byte aligned
    (all the API asks) but not 32 takes the 16-byte stores, same bytes."""
    n = 148 * 128 + 9
    x = W.single_tensor(n=n, d=d, seed=31 + d + bits).cuda()
    tq = K.TurboQuant(d, bits)
    ref, ref_n = _enc_path(K, tq, x, 2)
    P = tq.packed_bytes
    buf = torch.zeros(n * P + 64, dtype=torch.uint8, device="cuda")
    off = 16 if buf.data_ptr() % 32 == 0 else 0
    assert (buf.data_ptr() + off) % 32 == 16
    packed = buf[off:off + n * P].view(n, P)
    norms = torch.zeros(n, dtype=torch.float32, device="cuda")
    assert K._binding.tq_test_encode_path(tq.ctx, x, n, packed, norms, 2) == K.TQ_OK
    torch.cuda.synchronize()
    assert torch.equal(packed, ref) and torch.equal(norms, ref_n)
    assert int(buf[:off].sum()) == 0 and int(buf[off + n * P:].sum()) == 0  # nothing outside the rows
    assert K.tq_device_error() == (K.TQ_OK, 0)


def test_tc_bulk_encode_uses_the_tensor_core_kernel(K, W):
    """tq_encode of a bulk launch gives exactly the tensor-core kernel's
    output (codes and norms), and the CUDA-core kernel's codes."""
    n = 148 * 128 * 2 + 5
    x = W.single_tensor(n=n, d=128, seed=9).cuda()
    tq = K.TurboQuant(128, 3)
    p, nr = tq.encode(x)
    torch.cuda.synchronize()
    p2, n2 = _enc_path(K, tq, x, 2)
    p1, _ = _enc_path(K, tq, x, 1)
    assert torch.equal(p, p2) and torch.equal(nr, n2)
    assert torch.equal(p, p1)


def test_tensor_core_check_passes_and_a_failed_check_routes_bulk_launches_to_cuda_cores(K, W):
    """The run-time check of the MMA rounding passes on this GPU. When it is
    made to report a mismatch (host-side switch of the test hook), bulk
    tq_encode and tq_decode give exactly the CUDA-core kernels' outputs; once
    reset, the check passes again and bulk launches return to the tensor-core
    kernels."""
    assert K.tq_tensor_core_check() is True
    n = 148 * 128 * 2 + 5
    x = W.single_tensor(n=n, d=128, seed=19, outlier_frac=0.05).cuda()
    tq = K.TurboQuant(128, 4)
    p1, n1 = _enc_path(K, tq, x, 1)
    p2, n2 = _enc_path(K, tq, x, 2)
    d1 = torch.empty_like(x)
    assert K._binding.tq_test_decode_path(tq.ctx, p1, n1, n, d1, 1) == K.TQ_OK
    try:
        assert K._binding.tq_test_reset_tensor_core_check(True) == K.TQ_OK
        p, nr = tq.encode(x)  # bulk: runs the check, which reports a mismatch
        dec = tq.decode(p, nr)
        torch.cuda.synchronize()
        assert K.tq_tensor_core_check() is False
        assert torch.equal(p, p1) and torch.equal(nr, n1) and torch.equal(dec, d1)
    finally:
        assert K._binding.tq_test_reset_tensor_core_check(False) == K.TQ_OK
    p, nr = tq.encode(x)
    torch.cuda.synchronize()
    assert K.tq_tensor_core_check() is True
    assert torch.equal(p, p2) and torch.equal(nr, n2)
    assert K.tq_device_error() == (K.TQ_OK, 0)


def test_tc_bounded_wait_times_out_and_context_survives(K, W):
    """The tensor-core kernel with its tile copies withheld: the MMA warp's and
    the epilogue's bounded waits run out, TQ_DEVERR_TIMEOUT is recorded, the
    tensor memory is freed, nothing is written, and the next call works."""
    tq = K.TurboQuant(128, 4)
    x = W.single_tensor(n=1000).cuda()
    p = torch.zeros(1000, 64, dtype=torch.uint8, device="cuda")
    nrm = torch.zeros(1000, dtype=torch.float32, device="cuda")
    K.tq_device_error()
    assert K._binding.tq_test_encode_path(tq.ctx, x, 1000, p, nrm, 3) == K.TQ_OK
    st, bits = K.tq_device_error()
    assert st == K.TQ_ERR_TIMEOUT and bits & K.TQ_DEVERR_TIMEOUT
    assert torch.all(p == 0) and torch.all(nrm == 0)
    p2, n2 = _enc_path(K, tq, x, 2)
    assert K.tq_device_error() == (K.TQ_OK, 0)
    det = O.encode_detail(x.cpu().numpy(), 4, 42)
    assert code_mismatches(p2.cpu().numpy(), det, 4, 128) == 0


# ---------------------------------------------------------------- the tensor core's arithmetic
# The tensor-core encode kernel's exactness argument assumes, for one
# kind::f16 MMA with f32 accumulation and K = 16: products exact, each
# addend's magnitude cut to a multiple of 2^(E-25) (E the exponent of the
# largest addend), the sum rounded toward zero to f32. These tests pin that on
# the GPU the library runs on.


def _umma(K, a, b):
    at = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float16)).cuda()
    bt = torch.from_numpy(np.ascontiguousarray(b, dtype=np.float16)).cuda()
    d = torch.zeros(128, 16, dtype=torch.float32, device="cuda")
    assert K._binding.tq_test_umma_block(at, bt, d) == K.TQ_OK
    torch.cuda.synchronize()
    assert K.tq_device_error() == (K.TQ_OK, 0)
    return d.cpu().numpy().astype(np.float64)


def _round_toward_zero_f32(x):
    from fractions import Fraction

    x = Fraction(x)
    if x == 0:
        return 0.0
    s, m = (1, x) if x > 0 else (-1, -x)
    e = m.numerator.bit_length() - m.denominator.bit_length()
    if Fraction(2) ** e > m:
        e -= 1
    ulp = Fraction(2) ** (e - 23)
    return s * float((m // ulp) * ulp)


def test_tensor_core_cuts_addends_at_2_pow_minus_25_and_rounds_toward_zero(K):
    """Rows 1 (or -1) plus fifteen terms +-2^-t, t = 0 ... 39: the small terms
    count in full for t <= 25 and vanish beyond; the sum is rounded toward zero."""
    from fractions import Fraction

    a = np.zeros((128, 16))
    b = np.zeros((16, 16))
    for r in range(128):
        e = r % 25
        a[r, 0] = -1.0 if (r // 25) % 2 else 1.0
        a[r, 1:] = (-1.0 if (r // 50) % 2 else 1.0) * 2.0 ** -e
    for n in range(16):
        b[n, 0] = 1.0
        b[n, 1:] = 2.0 ** -n
    got = _umma(K, a, b)
    for r in range(128):
        for n in range(16):
            t = r % 25 + n
            small = Fraction(a[r, 1]) * Fraction(b[n, 1])
            kept = Fraction(a[r, 0]) + (15 * small if t <= 25 else 0)
            assert got[r, n] == _round_toward_zero_f32(kept), (r, n, t, got[r, n])


@pytest.mark.parametrize("cls", ["normal", "outliers", "log-uniform", "one-large", "cancelling"])
def test_tensor_core_error_within_the_bound_the_encode_kernel_uses(K, cls):
    """+-1-weighted 16-term sums (the 16-point Hadamard blocks) of five input
    classes: |S' - S| <= 15 * 2^(E-25) + 2^-23 |S| for every output."""
    import math

    g = np.random.default_rng(sum(map(ord, cls)))
    worst = 0.0
    for rep in range(8):
        if cls == "normal":
            a = g.standard_normal((128, 16))
        elif cls == "outliers":
            a = g.standard_normal((128, 16)) * np.where(g.random((128, 16)) < 0.06, 20.0, 1.0)
        elif cls == "log-uniform":
            a = np.where(g.random((128, 16)) < 0.5, -1.0, 1.0) * 2.0 ** (-24 + 39 * g.random((128, 16)))
        elif cls == "one-large":
            a = g.standard_normal((128, 16)) * 2.0 ** -8
            a[np.arange(128), g.integers(0, 16, 128)] = 1024.0 * (1 + g.random(128))
        else:
            x = (g.standard_normal((128, 8)) * 100).astype(np.float16).astype(np.float64)
            a = np.empty((128, 16))
            a[:, 0::2] = x
            a[:, 1::2] = -x + g.standard_normal((128, 8)) * 0.01
        a = a.astype(np.float16).astype(np.float64)
        b = np.where(g.random((16, 16)) < 0.5, -1.0, 1.0)
        got = _umma(K, a, b)
        for r in range(128):
            for n in range(16):
                p = a[r] * b[n]  # exact products
                s = math.fsum(p)
                mx = np.max(np.abs(p))
                if mx == 0:
                    assert got[r, n] == 0.0
                    continue
                e = math.floor(math.log2(mx))
                # fifteen cut addends, then rounding toward zero of the cut sum
                bound = 15 * 2.0 ** (e - 25) * (1 + 2.0 ** -23) + 2.0 ** -23 * abs(s)
                err = abs(got[r, n] - s)
                assert err <= bound, (cls, r, n, err, bound)
                worst = max(worst, err / bound)
    assert worst <= 1.0


def test_tc_matches_cuda_core_kernel_on_random_sizes(K, W):
    """40 seeded random (d, bits, n), n up to 200k (uneven tile counts per
    CTA, every ragged tail): the two encode kernels give identical codes and
    norms within 4e-6."""
    g = np.random.default_rng(2024)
    for t in range(40):
        d = int(g.choice([64, 128, 256]))
        bits = int(g.integers(2, 5))
        n = int(g.integers(1, 200_000))
        x = W.randn_f16((n, d), 9000 + t, "cuda")
        tq = K.TurboQuant(d, bits, seed=int(g.integers(0, 2**31)))
        p2, n2 = _enc_path(K, tq, x, 2)
        p1, n1 = _enc_path(K, tq, x, 1)
        assert torch.equal(p1, p2), (d, bits, n)
        torch.testing.assert_close(n2, n1, rtol=2e-6, atol=0)
        del x, p1, p2, n1, n2
    assert K.tq_device_error() == (K.TQ_OK, 0)
