"""CUDA encode / decode / append against the fp64 oracle (needs a B200)."""

import math

import numpy as np
import pytest
import torch

import oracle as O
from parity import assert_decode_ulp, assert_norms, code_mismatches, os_decode_ok

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def K(cuda_device):
    import kv_cache_vector_turboquant_b200 as K

    return K


@pytest.fixture(scope="module")
def W():
    import tq_workloads as W

    return W


def _encode(tq, x):
    packed, norms = tq.encode(x)
    torch.cuda.synchronize()
    return packed, norms


def _full_parity(K, x16_cpu, d, bits, seed=42, max_boundary_frac=1e-6):
    """Encode on the GPU, compare codes / norms / decode with the oracle."""
    tq = K.TurboQuant(d, bits, seed)
    x = x16_cpu.to("cuda")
    packed, norms = _encode(tq, x)
    xn = x16_cpu.numpy()
    det = O.encode_detail(xn, bits, seed)
    gp, gn = packed.cpu().numpy(), norms.cpu().numpy()
    n_mis = code_mismatches(gp, det, bits, d, max_boundary_frac)
    assert_norms(gn, det)
    # decode of the GPU's own bytes vs the oracle decode of the same bytes
    xd = tq.decode(packed, norms)
    torch.cuda.synchronize()
    ref = O.decode(gp, gn, bits, seed, d)
    assert_decode_ulp(xd.cpu().numpy().reshape(ref.shape), ref)
    st, bits_w = K.tq_device_error()
    assert st == K.TQ_OK and bits_w == 0
    return n_mis, gp, det


def test_single_tensor_workload(K, W):
    """4096 x 128 fp16 with 1% outlier vectors, 4 bits, seed 42: every code,
    norm and decoded value."""
    x = W.single_tensor()
    n_mis, gp, det = _full_parity(K, x, 128, 4)
    assert n_mis == 0
    assert gp.shape == (4096, 64)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("n", [1, 31, 33, 1000, 4103])
def test_ragged_sizes(K, W, d, bits, n):
    x = W.single_tensor(n=n, d=d, seed=1000 + n + d + bits, outlier_frac=0.05)
    n_mis, _, _ = _full_parity(K, x, d, bits)
    assert n_mis == 0


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_degenerate_vectors(K, W, d, bits):
    """Zero, constant, spike, extreme-magnitude and alternating rows. Exact ties
    at a boundary occur here (e.g. z = 0 exactly), so only the boundary-band
    rule applies, without the fraction bound."""
    x = W.edge_vectors(d)
    _full_parity(K, x, d, bits, max_boundary_frac=None)
    # the zero vector: norm 0, every code 2^(b-1), decodes to exact zeros
    tq = K.TurboQuant(d, bits)
    packed, norms = _encode(tq, x[:1].cuda())
    idx = O.unpack_codes(packed.cpu().numpy(), bits, d)
    assert norms.item() == 0.0 and np.all(idx == (1 << bits) // 2)
    assert torch.all(tq.decode(packed, norms) == 0)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_signed_hadamard_rows_rotate_to_spikes(K, d):
    """x = D r_k rotates to z = sqrt(d) e_k: code L-1 at k, 2^(b-1) elsewhere
    (exact ties at z = 0 go up)."""
    import scipy.linalg

    s = O.sign_vector(42, d)
    R = scipy.linalg.hadamard(d)
    rows = np.stack([s * R[k] for k in range(0, d, max(1, d // 16))]).astype(np.float16)
    for bits in (2, 3, 4):
        tq = K.TurboQuant(d, bits)
        packed, norms = _encode(tq, torch.from_numpy(rows).cuda())
        idx = O.unpack_codes(packed.cpu().numpy(), bits, d)
        for r, k in enumerate(range(0, d, max(1, d // 16))):
            want = np.full(d, (1 << bits) // 2)
            want[k] = (1 << bits) - 1
            assert np.array_equal(idx[r], want)
        assert np.allclose(norms.cpu().numpy(), math.sqrt(d), rtol=1e-7)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_llama_layer_full_size_sampled(K, W, bits):
    """Full [8, 8192, 8, 128] K and V layer on the GPU (the benchmarked
    launch); 65,536 sampled rows per tensor against the oracle, and the
    full-size distortion against the sphere-marginal value."""
    k, v = W.llama_layer(device="cuda")
    tq = K.TurboQuant(128, bits)
    g = torch.Generator().manual_seed(77 + bits)
    for x in (k, v):
        flat = x.reshape(-1, 128)
        packed, norms = tq.encode(flat)
        dec = tq.decode(packed, norms)
        torch.cuda.synchronize()
        rows = torch.randperm(flat.shape[0], generator=g)[:65536].sort().values
        xs = flat[rows.cuda()].cpu().numpy()
        det = O.encode_detail(xs, bits, 42)
        gp = packed[rows.cuda()].cpu().numpy()
        gn = norms[rows.cuda()].cpu().numpy()
        assert code_mismatches(gp, det, bits, 128) == 0
        assert_norms(gn, det)  # a bulk launch: the tensor-core kernel
        assert_decode_ulp(dec[rows.cuda()].cpu().numpy(), O.decode(gp, gn, bits, 42, 128))
        # whole-tensor property for the isotropic tensor (V: iid N(0,1), so the
        # unit direction is uniform on the sphere): the distortion equals the
        # sphere-marginal value. K's fixed outlier channels break isotropy.
        if x is v:
            u = flat.float() / flat.float().norm(dim=1, keepdim=True)
            uh = dec.float() / norms[:, None]
            mse = ((u - uh) ** 2).sum(dim=1).mean().item()
            want = O.sphere_marginal_mse(O.format_levels(bits), 128)
            assert abs(mse - want) / want < 0.01, (mse, want)
        del packed, norms, dec
    assert K.tq_device_error()[0] == K.TQ_OK


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_kv_in_one_buffer_equals_per_tensor_calls(K, W, bits):
    """The benchmarked step keeps the layer's K and V in one [2, n, 128]
    buffer and encodes (decodes) both with one call of 2n rows. Rows are
    independent, so codes, norms and decoded rows must be the bytes of one
    call per tensor; rows on both sides of the K/V seam and a random sample
    are also checked against the oracle."""
    k, v = W.llama_layer(device="cuda")
    n = k.numel() // 128
    kv = torch.stack([k.reshape(n, 128), v.reshape(n, 128)])
    del k, v
    tq = K.TurboQuant(128, bits)
    packed, norms = tq.encode(kv.reshape(2 * n, 128))
    dec = tq.decode(packed, norms)
    for t in range(2):
        p1, n1 = tq.encode(kv[t])
        d1 = tq.decode(p1, n1)
        torch.cuda.synchronize()
        assert torch.equal(packed[t * n:(t + 1) * n], p1)
        assert torch.equal(norms[t * n:(t + 1) * n], n1)
        assert torch.equal(dec[t * n:(t + 1) * n], d1)
        del p1, n1, d1
    g = torch.Generator().manual_seed(90 + bits)
    rows = torch.cat([torch.arange(n - 256, n + 256), torch.randint(0, 2 * n, (4096,), generator=g)]).unique()
    xs = kv.reshape(2 * n, 128)[rows.cuda()].cpu().numpy()
    det = O.encode_detail(xs, bits, 42)
    gp, gn = packed[rows.cuda()].cpu().numpy(), norms[rows.cuda()].cpu().numpy()
    assert code_mismatches(gp, det, bits, 128) == 0
    assert_norms(gn, det)
    assert_decode_ulp(dec[rows.cuda()].cpu().numpy(), O.decode(gp, gn, bits, 42, 128))
    assert K.tq_device_error()[0] == K.TQ_OK


@pytest.mark.parametrize("layer", [0, 41, 79])
def test_long_context_layer_sampled(K, W, layer):
    """Layers of the 80-layer long-context cache at 3 bits: K and V
    [1, 131072, 8, 128] with log-normal per-channel scales, encoded whole on
    the GPU; 4096 sampled rows per tensor against the oracle (codes, norms,
    decode of the same bytes)."""
    kx, vx = W.long_context_layer(layer)
    tq = K.TurboQuant(128, 3)
    g = torch.Generator().manual_seed(1000 + layer)
    for x in (kx, vx):
        flat = x.reshape(-1, 128)
        packed, norms = tq.encode(flat)
        dec = tq.decode(packed, norms)
        torch.cuda.synchronize()
        rows = torch.randperm(flat.shape[0], generator=g)[:4096].sort().values.cuda()
        xs = flat[rows].cpu().numpy()
        det = O.encode_detail(xs, 3, 42)
        gp, gn = packed[rows].cpu().numpy(), norms[rows].cpu().numpy()
        assert code_mismatches(gp, det, 3, 128) == 0
        assert_norms(gn, det)  # a bulk launch: the tensor-core kernel
        assert_decode_ulp(dec[rows].cpu().numpy(), O.decode(gp, gn, 3, 42, 128))
        del packed, norms, dec
    assert K.tq_device_error()[0] == K.TQ_OK


@pytest.mark.parametrize("d", [64, 256])
def test_append_replayed_from_cuda_graph(K, W, d):
    """The streaming append captured once in a CUDA graph (32 steps, K and V)
    and replayed writes the same bytes as the eager calls."""
    n_seq, h, s_max, steps, bits = 256, 8, 32, 32, 4
    tq = K.TurboQuant(d, bits)
    P = tq.packed_bytes
    toks = W.append_stream(run=7 + d, steps=steps, n_seq=n_seq, H=h, d=d)
    slots = torch.arange(steps, dtype=torch.int32, device="cuda")[:, None].expand(steps, n_seq).contiguous()
    caches = [(torch.zeros(n_seq, s_max, h, P, dtype=torch.uint8, device="cuda"),
               torch.zeros(n_seq, s_max, h, dtype=torch.float32, device="cuda")) for _ in range(2)]
    tq.encode_append(toks[0], caches[0][0], caches[0][1], slots[0])  # one eager call before capture
    torch.cuda.synchronize()
    caches[0][0].zero_()
    caches[0][1].zero_()
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(graph, stream=stream):
            for s in range(steps):
                tq.encode_append(toks[s], caches[1][0], caches[1][1], slots[s])
    torch.cuda.current_stream().wait_stream(stream)
    graph.replay()
    for s in range(steps):
        tq.encode_append(toks[s], caches[0][0], caches[0][1], slots[s])
    torch.cuda.synchronize()
    assert torch.equal(caches[0][0], caches[1][0])
    assert torch.equal(caches[0][1], caches[1][1])
    assert K.tq_device_error()[0] == K.TQ_OK
    del graph


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_append_kv_equals_two_appends(K, W, d, bits):
    """The key and value append of one launch writes exactly what two
    tq_encode_append calls write (ragged head count, a slot out of range
    skipped and flagged), and the same steps replayed from a CUDA graph give
    the same bytes again."""
    n_seq, h, s_max, steps = 37, 3, 8, 4
    tq = K.TurboQuant(d, bits)
    P = tq.packed_bytes
    ks = W.append_stream(run=50 + d + bits, steps=steps, n_seq=n_seq, H=h, d=d)
    vs = W.append_stream(run=60 + d + bits, steps=steps, n_seq=n_seq, H=h, d=d)
    g = torch.Generator().manual_seed(d * 10 + bits)
    slots = torch.randint(0, s_max, (steps, n_seq), generator=g, dtype=torch.int32).cuda()

    def caches():
        return [torch.full((n_seq, s_max, h, P), 0x3C, dtype=torch.uint8, device="cuda"),
                torch.full((n_seq, s_max, h), -3.0, dtype=torch.float32, device="cuda"),
                torch.full((n_seq, s_max, h, P), 0x5A, dtype=torch.uint8, device="cuda"),
                torch.full((n_seq, s_max, h), -5.0, dtype=torch.float32, device="cuda")]

    two, one, graphed = caches(), caches(), caches()
    for s in range(steps):
        tq.encode_append(ks[s], two[0], two[1], slots[s])
        tq.encode_append(vs[s], two[2], two[3], slots[s])
        tq.encode_append_kv(ks[s], vs[s], one[0], one[1], one[2], one[3], slots[s])
    torch.cuda.synchronize()
    assert K.tq_device_error() == (K.TQ_OK, 0)
    for a, b in zip(one, two):
        assert torch.equal(a, b)
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(graph, stream=stream):
            for s in range(steps):
                tq.encode_append_kv(ks[s], vs[s], graphed[0], graphed[1], graphed[2], graphed[3], slots[s])
    torch.cuda.current_stream().wait_stream(stream)
    graph.replay()
    torch.cuda.synchronize()
    for a, b in zip(graphed, two):
        assert torch.equal(a, b)
    del graph
    # a slot past the cache is skipped (both tensors) and flagged
    bad = slots[0].clone()
    bad[5] = s_max
    before = [t.clone() for t in one]
    tq.encode_append_kv(ks[0], vs[0], one[0], one[1], one[2], one[3], bad)
    torch.cuda.synchronize()
    st, bits_ = K.tq_device_error()
    assert st == K.TQ_ERR_DEVICE and bits_ == K.TQ_DEVERR_SLOT_RANGE
    for a, b in zip(one, before):
        assert torch.equal(a[5], b[5])


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_append_matches_bulk_encode(K, W, d, bits):
    """Streaming append of 6 steps x 256 sequences x 8 heads into a 16-slot
    cache: written slots are bit-identical to a bulk encode of the same rows,
    other slots untouched."""
    n_seq, h, s_max, steps = 256, 8, 16, 6
    tq = K.TurboQuant(d, bits)
    P = tq.packed_bytes
    toks = W.append_stream(run=bits + d, steps=steps, n_seq=n_seq, H=h, d=d)
    cache = torch.full((n_seq, s_max, h, P), 0xAB, dtype=torch.uint8, device="cuda")
    cnorm = torch.full((n_seq, s_max, h), -1.0, dtype=torch.float32, device="cuda")
    slots = torch.randint(0, s_max, (steps, n_seq), generator=torch.Generator().manual_seed(d + bits),
                          dtype=torch.int32)
    # distinct slots per sequence across steps so later steps do not overwrite
    slots = (torch.arange(steps, dtype=torch.int32)[:, None] * 2 + (slots % 2)) % s_max
    for s in range(steps):
        tq.encode_append(toks[s].contiguous(), cache, cnorm, slots[s].cuda())
    torch.cuda.synchronize()
    bp, bn = tq.encode(toks.reshape(-1, d).contiguous())
    bp = bp.reshape(steps, n_seq, h, P).cpu()
    bn = bn.reshape(steps, n_seq, h).cpu()
    cache, cnorm = cache.cpu(), cnorm.cpu()
    written = torch.zeros(n_seq, s_max, dtype=torch.bool)
    for s in range(steps):
        idx = torch.arange(n_seq)
        assert torch.equal(cache[idx, slots[s].long()], bp[s])
        assert torch.equal(cnorm[idx, slots[s].long()], bn[s])
        written[idx, slots[s].long()] = True
    assert torch.all(cache[~written] == 0xAB) and torch.all(cnorm[~written] == -1.0)
    # and the bulk encode itself matches the oracle on a sample
    xs = toks.reshape(-1, d)[:2048].cpu().numpy()
    det = O.encode_detail(xs, bits, 42)
    assert code_mismatches(bp.reshape(-1, P)[:2048].numpy(), det, bits, d) == 0


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_encode_slots_writes_bulk_codes_into_mapped_slots(K, W, d, bits):
    """Encode-on-write into a paged pool [num_blocks, 16, h, P]: token t lands
    in slot slot_mapping[t] with the oracle's codes and norms for its rows,
    bit-identical to a bulk encode of the same rows; padding tokens (slot -1)
    and every other slot are left untouched."""
    n_tok, h, num_blocks = 300, 8, 40
    tq = K.TurboQuant(d, bits)
    P = tq.packed_bytes
    x = W.append_stream(run=100 + d + bits, steps=1, n_seq=n_tok, H=h, d=d)[0].contiguous()
    g = torch.Generator().manual_seed(d * bits)
    slots = torch.randperm(num_blocks * 16, generator=g)[:n_tok].to(torch.int32)
    slots[::7] = -1  # padding tokens
    pool = torch.full((num_blocks, 16, h, P), 0x5A, dtype=torch.uint8, device="cuda")
    pnorm = torch.full((num_blocks, 16, h), -2.0, dtype=torch.float32, device="cuda")
    tq.encode_slots(x, pool, pnorm, slots.cuda())
    bp, bn = tq.encode(x.reshape(-1, d))
    torch.cuda.synchronize()
    assert K.tq_device_error() == (K.TQ_OK, 0)
    flat, fnorm = pool.reshape(-1, h, P).cpu(), pnorm.reshape(-1, h).cpu()
    bp, bn = bp.reshape(n_tok, h, P).cpu(), bn.reshape(n_tok, h).cpu()
    used = slots >= 0
    assert torch.equal(flat[slots[used].long()], bp[used])
    assert torch.equal(fnorm[slots[used].long()], bn[used])
    untouched = torch.ones(flat.shape[0], dtype=torch.bool)
    untouched[slots[used].long()] = False
    assert torch.all(flat[untouched] == 0x5A) and torch.all(fnorm[untouched] == -2.0)
    # the written slots against the fp64 oracle on the same fp16 rows
    rows = x.cpu()[used].reshape(-1, d).numpy()
    det = O.encode_detail(rows, bits, 42)
    got_p = flat[slots[used].long()].reshape(-1, P).numpy()
    got_n = fnorm[slots[used].long()].reshape(-1).numpy()
    assert code_mismatches(got_p, det, bits, d) == 0
    assert_norms(got_n, det)


def test_encode_slots_out_of_range_is_flagged(K, W):
    tq = K.TurboQuant(128, 4)
    x = W.append_stream(run=3, steps=1, n_seq=4, H=8, d=128)[0].contiguous()
    pool = torch.zeros(2, 16, 8, 64, dtype=torch.uint8, device="cuda")
    pnorm = torch.zeros(2, 16, 8, dtype=torch.float32, device="cuda")
    tq.encode_slots(x, pool, pnorm, torch.tensor([0, 31, 32, -1], dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    st, bits = K.tq_device_error()
    assert st == K.TQ_ERR_DEVICE and bits == K.TQ_DEVERR_SLOT_RANGE


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_offset_variant_matches_oracle(K, W, d, bits):
    """Offset + fp16-scale variant on rows with random offsets and outliers
    (ragged n): side data within one fp16 ulp of the oracle's (the GPU
    accumulates the mean in f32), codes bit-exact given the GPU's side data,
    decode of the same bytes within the fp16 rounding."""
    n = 3001
    g = torch.Generator().manual_seed(d * 7 + bits)
    x = torch.randn(n, d, generator=g) * torch.exp(torch.randn(n, 1, generator=g))
    x += torch.randn(n, 1, generator=g) * 3
    hit = torch.rand(n, d, generator=g) < 0.005
    x = torch.where(hit, x * 20, x).to(torch.float16)
    x[0] = 0.0
    x[1] = 2.5
    tq = K.TurboQuant(d, bits)
    packed, side = tq.encode_os(x.cuda())
    dec = tq.decode_os(packed, side)
    torch.cuda.synchronize()
    assert K.tq_device_error() == (K.TQ_OK, 0)
    xs = x.numpy()
    side_u = side.cpu().numpy().view(np.uint32)
    own = O.encode_os_detail(xs, bits, 42)
    gmu = (side_u & 0xFFFF).astype(np.uint16).view(np.float16)
    gn = (side_u >> 16).astype(np.uint16).view(np.float16)
    from parity import fp16_ulp_distance
    assert fp16_ulp_distance(gmu, own["mu16"]).max() <= 1
    assert fp16_ulp_distance(gn, own["n16"]).max() <= 1
    det = O.encode_os_detail(xs, bits, 42, side=side_u)
    gp = packed.cpu().numpy()
    assert code_mismatches(gp, det, bits, d) == 0
    exact = O.decode_os_f64(gp, side_u, bits, 42, d)
    assert np.all(os_decode_ok(dec.cpu().numpy(), exact, gmu))
    # the zero row decodes to zeros and the constant row to itself
    assert torch.all(dec[0] == 0) and torch.all(dec[1].cpu() == x[1])


def test_append_out_of_range_slot_is_skipped_and_flagged(K, W):
    tq = K.TurboQuant(128, 4)
    n_seq, h, s_max = 4, 8, 8
    x = W.append_stream(run=0, steps=1, n_seq=n_seq, H=h, d=128)[0].contiguous()
    cache = torch.zeros((n_seq, s_max, h, 64), dtype=torch.uint8, device="cuda")
    cn = torch.zeros((n_seq, s_max, h), dtype=torch.float32, device="cuda")
    slot = torch.tensor([0, -1, s_max, 3], dtype=torch.int32, device="cuda")
    K.tq_device_error()  # clear
    tq.encode_append(x, cache, cn, slot)
    st, bits = K.tq_device_error()
    assert st == K.TQ_ERR_DEVICE and bits & K.TQ_DEVERR_SLOT_RANGE
    assert torch.all(cache[1] == 0) and torch.all(cache[2] == 0)
    assert torch.any(cache[0, 0] != 0) and torch.any(cache[3, 3] != 0)


def test_non_default_stream(K, W):
    x = W.single_tensor(n=3000, seed=5).cuda()
    tq = K.TurboQuant(128, 3)
    ref_p, ref_n = _encode(tq, x)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        p, n = tq.encode(x, stream=s)
    s.synchronize()
    assert torch.equal(p, ref_p) and torch.equal(n, ref_n)


def test_bounded_wait_times_out_and_context_survives(K, W):
    """A kernel whose bulk copies never arrive: its bounded mbarrier wait runs
    out, it records TQ_DEVERR_TIMEOUT and returns; the host reads the status
    and the next call works."""
    tq = K.TurboQuant(128, 4)
    x = W.single_tensor(n=256).cuda()
    p = torch.zeros(256, 64, dtype=torch.uint8, device="cuda")
    nrm = torch.zeros(256, dtype=torch.float32, device="cuda")
    K.tq_device_error()
    assert K._binding.tq_test_encode_stalled(tq.ctx, x, 256, p, nrm) == K.TQ_OK
    st, bits = K.tq_device_error()
    assert st == K.TQ_ERR_TIMEOUT and bits & K.TQ_DEVERR_TIMEOUT
    assert torch.all(p == 0)
    # the context form of the query reports the same word
    assert K._binding.tq_test_encode_stalled(tq.ctx, x, 256, p, nrm) == K.TQ_OK
    torch.cuda.synchronize()
    assert K.tq_check_device_error(tq.ctx) == K.TQ_ERR_TIMEOUT
    assert K.tq_check_device_error(tq.ctx) == K.TQ_OK  # read and cleared
    # context usable afterwards, error word cleared
    p2, n2 = _encode(tq, x)
    assert K.tq_device_error() == (K.TQ_OK, 0)
    det = O.encode_detail(x.cpu().numpy(), 4, 42)
    assert code_mismatches(p2.cpu().numpy(), det, 4, 128) == 0


@pytest.mark.parametrize("d,bits", [(64, 3), (128, 2), (128, 4)])
def test_back_to_back_bulk_launches_see_each_others_outputs(K, W, d, bits):
    """The bulk kernels start while the previous kernel of the stream is
    finishing (programmatic dependent launch) and wait for it before
    touching global memory. A chain in which every launch consumes the
    previous one's output, issued with no synchronisation, gives the same
    bytes as the chain synchronised after every call."""
    n = 148 * 128 * 3 + 41
    x = W.single_tensor(n=n, d=d, seed=300 + d + bits).cuda()
    tq = K.TurboQuant(d, bits)

    def chain(sync):
        p1, n1 = tq.encode(x)
        if sync:
            torch.cuda.synchronize()
        y1 = tq.decode(p1, n1)  # reads the encode's codes and norms
        if sync:
            torch.cuda.synchronize()
        p2, n2 = tq.encode(y1)  # reads the decode's rows
        if sync:
            torch.cuda.synchronize()
        y2 = tq.decode(p2, n2)
        torch.cuda.synchronize()
        return p1, n1, y1, p2, n2, y2

    ref = chain(True)
    for _ in range(3):
        got = chain(False)
        for a, b in zip(got, ref):
            assert torch.equal(a, b)
    assert K.tq_device_error() == (K.TQ_OK, 0)


def test_bench_sustained_mode_reports_every_phase(K):
    """`bench.py --sustained` (its summary is committed under profiles/): one
    short run of every phase, each with a time, a clock and a power figure,
    and no device error."""
    import bench

    res = bench.run_sustained(seconds=0.2)
    names = [r["phase"] for r in res["sustained"]]
    assert names == [f"{k}_b{b}" for k in ("encode", "decode") for b in (2, 3, 4)] + ["codec_step", "attention_step"]
    for r in res["sustained"]:
        assert r["us"] > 0.0
        assert "sm_mhz" in r and "power_w" in r
    assert res["device_error"] == [K.TQ_OK, 0]


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_validate_and_benchmark_helpers(K, bits):
    """TurboQuant.validate / benchmark (the pages' helper methods): the
    reconstruction of N(0,1) vectors has the sphere-marginal distortion of
    the width (within 5 %), cosine close to 1, norms within 1e-6; benchmark
    returns positive times for both directions."""
    tq = K.TurboQuant(128, bits)
    v = tq.validate(num_vectors=20000)
    # ||x - x_hat||^2 / ||x||^2 is the squared error of the unit direction,
    # whose expectation is the sphere-marginal distortion of one coordinate
    want = O.sphere_marginal_mse(O.format_levels(bits), 128)
    assert abs(v["mse_relative"] - want) <= 0.05 * want, (v, want)
    assert v["cosine"] > 0.9 and v["max_norm_rel_err"] <= 1e-6
    b = tq.benchmark(num_vectors=32768, reps=3)
    assert b["encode_us"] > 0 and b["decode_us"] > 0
    assert K.tq_device_error() == (K.TQ_OK, 0)
