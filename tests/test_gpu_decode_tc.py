"""The tensor-core decode kernel (needs a B200).

tq_decode runs it for head_dim 64 and 128 from 128 x SM-count vectors on; the
test hook tq_test_decode_path runs it (path 2) or the CUDA-core kernel
(path 1) at any size. Both compute H_pm c exactly and round only the product
by N / d and the fp16 conversion, so their outputs are bit-identical; the
oracle bounds both to 1 fp16 ulp.
"""

import numpy as np
import pytest
import torch

import oracle as O
from parity import assert_decode_ulp, os_decode_ok

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K(cuda_device):
    import kv_cache_vector_turboquant_b200 as K

    return K


@pytest.fixture(scope="module")
def W():
    import tq_workloads as W

    return W


def _dec_path(K, tq, packed, norms, path):
    n = norms.numel()
    x = torch.full((n, tq.head_dim), 7.0, dtype=torch.float16, device="cuda")
    assert K._binding.tq_test_decode_path(tq.ctx, packed, norms, n, x, path) == K.TQ_OK
    torch.cuda.synchronize()
    return x


def _random_codes(tq, n, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    packed = torch.randint(0, 256, (n, tq.packed_bytes), generator=g, device="cuda", dtype=torch.int32).to(torch.uint8)
    norms = torch.rand(n, generator=g, device="cuda") * 30.0
    if n > 3:
        norms[0] = 0.0
        norms[1] = 1.0e-30
        norms[2] = 6.0e4
    return packed, norms


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("n", [1, 127, 128, 129, 4103])
def test_tc_decode_ragged_sizes(K, d, bits, n):
    """Random bytes and norms (zero, tiny and large among them): partial
    tiles (read with plain loads, stores clipped), one tile, 33 tiles."""
    tq = K.TurboQuant(d, bits, seed=5 + bits)
    packed, norms = _random_codes(tq, n, 100 * d + 10 * bits + n)
    x2 = _dec_path(K, tq, packed, norms, 2)
    x1 = _dec_path(K, tq, packed, norms, 1)
    assert torch.equal(x1, x2)
    ref = O.decode(packed.cpu().numpy(), norms.cpu().numpy(), bits, 5 + bits, d)
    assert_decode_ulp(x2.cpu().numpy(), ref)
    assert K.tq_device_error() == (K.TQ_OK, 0)


@pytest.mark.parametrize("d,per_cta", [(64, 13), (128, 9)])
def test_tc_decode_many_tiles_per_cta(K, W, d, per_cta):
    """Every CTA cycles its stage ring, both tensor-memory slots and both
    epilogue warpgroups several times; the layer's own codes."""
    n = 148 * 128 * per_cta + 77
    x = W.single_tensor(n=n, d=d, seed=77 + d, outlier_frac=0.02).cuda()
    for bits in (2, 3, 4):
        tq = K.TurboQuant(d, bits)
        packed, norms = tq.encode(x)
        x2 = _dec_path(K, tq, packed, norms, 2)
        x1 = _dec_path(K, tq, packed, norms, 1)
        assert torch.equal(x1, x2), bits
        rows = torch.randperm(n, generator=torch.Generator().manual_seed(bits))[:2048].sort().values.cuda()
        ref = O.decode(packed[rows].cpu().numpy(), norms[rows].cpu().numpy(), bits, 42, d)
        assert_decode_ulp(x2[rows].cpu().numpy(), ref)
    assert K.tq_device_error() == (K.TQ_OK, 0)


def test_tc_decode_bulk_call_uses_it_and_head_dim_256_does_not(K, W):
    n = 148 * 128 * 2 + 3
    tq = K.TurboQuant(128, 4)
    packed, norms = _random_codes(tq, n, 11)
    xb = tq.decode(packed, norms)
    torch.cuda.synchronize()
    assert torch.equal(xb, _dec_path(K, tq, packed, norms, 2))
    t256 = K.TurboQuant(256, 4)
    p256, n256 = _random_codes(t256, 300, 12)
    x = torch.empty(300, 256, dtype=torch.float16, device="cuda")
    assert K._binding.tq_test_decode_path(t256.ctx, p256, n256, 300, x, 2) == K.TQ_ERR_UNSUPPORTED


def test_tc_decode_matches_cuda_core_kernel_on_random_sizes(K, W):
    """30 seeded random (d, bits, n, seed), n up to 300k (uneven tile counts
    per CTA, every ragged tail), the layer's own codes: the two decode
    kernels give identical fp16 rows."""
    g = np.random.default_rng(2027)
    for t in range(30):
        d = int(g.choice([64, 128]))
        bits = int(g.integers(2, 5))
        n = int(g.integers(1, 300_000))
        x = W.single_tensor(n=n, d=d, seed=500 + t, outlier_frac=0.02).cuda()
        tq = K.TurboQuant(d, bits, seed=int(g.integers(0, 2**31)))
        packed, norms = tq.encode(x)
        x2 = _dec_path(K, tq, packed, norms, 2)
        x1 = _dec_path(K, tq, packed, norms, 1)
        assert torch.equal(x1, x2), (d, bits, n)
        del x, packed, norms, x1, x2
    assert K.tq_device_error() == (K.TQ_OK, 0)


def _os_side(n, seed):
    """Side words fp16 offset | fp16 scale << 16, with a zero scale, a tiny
    and a large one, and a negative offset among them."""
    g = torch.Generator().manual_seed(seed)
    mu = (torch.rand(n, generator=g) * 4.0 - 2.0).to(torch.float16)
    sc = (torch.rand(n, generator=g) * 30.0).to(torch.float16)
    if n > 3:
        sc[0], sc[1], sc[2] = 0.0, 6.0e-8, 6.0e4
        mu[3] = -1.5
    bits = mu.view(torch.int16).to(torch.int32) & 0xFFFF
    bits |= (sc.view(torch.int16).to(torch.int32) & 0xFFFF) << 16
    return bits.cuda()


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("n", [1, 129, 148 * 128 * 3 + 77])
def test_tc_decode_offset_variant_matches_cuda_core_kernel(K, d, bits, n):
    """The offset + fp16-scale variant on the tensor cores (path 4) against
    the CUDA-core offset decode (path 3): the sign in f32 and the offset added
    before the rounding in both, so the outputs are bit-identical; the oracle
    bounds them to 1 fp16 ulp."""
    tq = K.TurboQuant(d, bits, seed=9 + bits)
    packed, _ = _random_codes(tq, n, 300 * d + 10 * bits + n)
    side = _os_side(n, 7 * d + bits + n)
    x4 = torch.full((n, d), 7.0, dtype=torch.float16, device="cuda")
    x3 = torch.full((n, d), 7.0, dtype=torch.float16, device="cuda")
    assert K._binding.tq_test_decode_path(tq.ctx, packed, side, n, x4, 4) == K.TQ_OK
    assert K._binding.tq_test_decode_path(tq.ctx, packed, side, n, x3, 3) == K.TQ_OK
    torch.cuda.synchronize()
    assert torch.equal(x3, x4)
    sw = side.cpu().numpy().astype(np.uint32)
    exact = O.decode_os_f64(packed.cpu().numpy(), sw, bits, 9 + bits, d)
    mu16 = (sw & 0xFFFF).astype(np.uint16).view(np.float16)
    assert np.all(os_decode_ok(x4.cpu().numpy(), exact, mu16))
    # a bulk tq_decode_os call takes the tensor-core kernel: same bytes
    if n >= 128 * 148:
        assert torch.equal(tq.decode_os(packed, side), x4)
    assert K.tq_device_error() == (K.TQ_OK, 0)
