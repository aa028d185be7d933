"""Pins of the fp64 oracle against things other than itself.

Each test ties one step of the oracle to a closed form, a published value, a
library routine or brute force, so that a dropped term, a wrong sign or index or
a transposed operand anywhere in the oracle fails at least one of them.
"""

import math

import numpy as np
import pytest
import scipy.integrate
import scipy.linalg
import torch

import oracle as O
from conftest import golden_lines


# ---------------------------------------------------------------- Hadamard

@pytest.mark.parametrize("d", [1, 2, 4, 8, 16, 32, 64, 128, 256])
def test_hadamard_is_sylvester_and_orthonormal(d):
    H = O.hadamard(d)
    # library routine: scipy's Sylvester construction, natural order
    assert np.array_equal(O.hadamard_pm(d), scipy.linalg.hadamard(d).astype(np.float64))
    assert np.array_equal(H, scipy.linalg.hadamard(d).astype(np.float64) / math.sqrt(d))
    assert np.abs(H @ H - np.eye(d)).max() < 1e-12
    rng = np.random.default_rng(d)
    v = rng.standard_normal(d)
    assert abs(np.linalg.norm(H @ v) - np.linalg.norm(v)) < 1e-12 * np.linalg.norm(v)
    # a spike spreads to +-1/sqrt(d) exactly (up to the fp64 scaling)
    k = d // 3
    e = np.zeros(d)
    e[k] = 1.0
    assert np.allclose(np.abs(H @ e), 1.0 / math.sqrt(d), rtol=0, atol=1e-15)


# ---------------------------------------------------------------- codebook

def _max_table():
    rows = {}
    for ln in golden_lines("max1960_gaussian_quantizer.txt"):
        vals = ln.split()
        rows[int(vals[0])] = (float(vals[1]), [float(v) for v in vals[2:]])
    return rows


def test_lloyd_max_one_bit_closed_form():
    c = O.lloyd_max_levels(1)
    assert abs(c[1] - math.sqrt(2.0 / math.pi)) < 1e-12
    assert abs(c[0] + math.sqrt(2.0 / math.pi)) < 1e-12
    # MSE of the sign quantizer on N(0,1) is 1 - 2/pi
    assert abs(O.gaussian_cell_mse(c) - (1.0 - 2.0 / math.pi)) < 1e-12


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_lloyd_max_matches_published_table(bits):
    mse_pub, lv_pub = _max_table()[bits]
    c = O.lloyd_max_levels(bits)
    L = 1 << bits
    pos = c[L // 2:]
    # the table prints 4 significant digits
    for got, want in zip(pos, lv_pub):
        assert abs(got - want) <= 6e-4 * max(1.0, abs(want)), (bits, got, want)
    mse = O.gaussian_cell_mse(c)
    assert abs(mse - mse_pub) / mse_pub < 5e-4, (bits, mse, mse_pub)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_lloyd_max_centroid_and_symmetry(bits):
    c = O.lloyd_max_levels(bits)
    L = len(c)
    assert np.all(np.diff(c) > 0)
    assert np.abs(c + c[::-1]).max() < 1e-13
    t = [-np.inf] + list(0.5 * (c[1:] + c[:-1])) + [np.inf]
    pdf = lambda x: math.exp(-0.5 * x * x) / math.sqrt(2 * math.pi)  # noqa: E731
    for k in range(L):
        a, b = t[k], t[k + 1]
        m1, _ = scipy.integrate.quad(lambda x: x * pdf(x), a, b, epsabs=1e-15, epsrel=1e-13)
        m0, _ = scipy.integrate.quad(pdf, a, b, epsabs=1e-15, epsrel=1e-13)
        assert abs(m1 / m0 - c[k]) < 1e-10, (bits, k)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_cell_mse_closed_form_against_quadrature(bits):
    c = O.format_levels(bits)
    t = O.format_boundaries(c)
    edges = [-np.inf] + list(t) + [np.inf]
    pdf = lambda x: math.exp(-0.5 * x * x) / math.sqrt(2 * math.pi)  # noqa: E731
    total = 0.0
    for k in range(len(c)):
        v, _ = scipy.integrate.quad(lambda x: (x - c[k]) ** 2 * pdf(x), edges[k], edges[k + 1],
                                    epsabs=1e-15, epsrel=1e-13)
        total += v
    assert abs(total - O.gaussian_cell_mse(c, t)) < 1e-12


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_mse_within_27x_of_lower_bound(bits):
    # "aither-kvcache", section "Quantization Quality": within 2.7x of the
    # information-theoretic lower bound 4^-b.
    mse = O.gaussian_cell_mse(O.format_levels(bits), O.format_boundaries(O.format_levels(bits)))
    assert mse * 4 ** bits <= 2.7


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_format_levels_on_grid(bits):
    c = O.lloyd_max_levels(bits)
    f = O.format_levels(bits)
    g = f * 2 ** O.FORMAT_GRID_BITS
    assert np.array_equal(g, np.round(g))
    assert np.abs(f - c).max() <= 2.0 ** -(O.FORMAT_GRID_BITS + 1)
    t = O.format_boundaries(f)
    assert np.array_equal(t, (f[1:] + f[:-1]) / 2)
    # snapping changes the distortion by a negligible amount
    assert abs(O.gaussian_cell_mse(f, t) - O.gaussian_cell_mse(c)) < 1e-8
    # levels fit 16-bit integers on the grid
    assert np.abs(g).max() < 2 ** 16


# ---------------------------------------------------------------- signs

def test_splitmix64_published_vectors():
    for ln in golden_lines("splitmix64_vigna.txt"):
        vals = [int(v) for v in ln.split()]
        seed, want = vals[0], vals[1:]
        assert O.splitmix64(seed, len(want)) == want


def test_sign_vector_is_bit63():
    for ln in golden_lines("splitmix64_vigna.txt"):
        vals = [int(v) for v in ln.split()]
        seed, outs = vals[0], vals[1:]
        s = O.sign_vector(seed, len(outs))
        assert list(s) == [-1.0 if v >= 2 ** 63 else 1.0 for v in outs]
    s = O.sign_vector(42, 256)
    assert set(np.unique(s)) <= {-1.0, 1.0}
    assert 90 < (s > 0).sum() < 166  # a fair-coin sequence


# ---------------------------------------------------------------- quantizer

@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_quantize_is_nearest_level(bits):
    from fractions import Fraction

    c = O.format_levels(bits)
    t = O.format_boundaries(c)
    rng = np.random.default_rng(bits)
    z = np.concatenate([rng.standard_normal(20000) * 1.5, np.array([-30.0, 30.0])])
    brute = np.argmin(np.abs(z[:, None] - c[None, :]), axis=1)
    assert np.array_equal(O.quantize(z, t), brute)
    # one ulp either side of every boundary: brute force in exact rationals
    near = np.concatenate([np.nextafter(t, np.inf), np.nextafter(t, -np.inf)])
    cf = [Fraction(float(v)) for v in c]
    exact = [min(range(len(cf)), key=lambda k: abs(Fraction(float(v)) - cf[k])) for v in near]
    assert list(O.quantize(near, t)) == exact


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_quantize_ties_go_up(bits):
    c = O.format_levels(bits)
    t = O.format_boundaries(c)
    idx = O.quantize(t, t)
    assert np.array_equal(idx, np.arange(1, len(c)))
    assert O.quantize(np.array([0.0]), t)[0] == len(c) // 2


# ---------------------------------------------------------------- sizes

def test_bytes_per_vector_and_ratio():
    # "aither-kvcache", "Quick Start -- TurboQuant": [...,128] fp16 -> [...,64] uint8 + f32
    assert O.packed_bytes(128, 4) == 64
    for d in (64, 128, 256):
        for b in (2, 3, 4):
            assert O.compressed_bytes_per_vector(d, b) == d * b // 8 + 4
    # "aitherkvcache -- the crucible": 3.8-7.1x compression against FP16 at 2-4 bits
    ratios = {b: 2 * 128 / O.compressed_bytes_per_vector(128, b) for b in (2, 3, 4)}
    assert round(ratios[4], 1) == 3.8 and round(ratios[2], 1) == 7.1
    assert abs(ratios[3] - 256 / 52) < 1e-12


# ---------------------------------------------------------------- packing

def test_pack_golden_patterns():
    for ln in golden_lines("pack_patterns.txt"):
        b, codes, hexes = [p.strip() for p in ln.split("|")]
        bits = int(b)
        idx = np.array([[int(v) for v in codes.split()]])
        want = np.array([[int(h, 16) for h in hexes.split()]], dtype=np.uint8)
        assert np.array_equal(O.pack_codes(idx, bits), want)
        assert np.array_equal(O.unpack_codes(want, bits, idx.shape[1]), idx)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_pack_round_trip(bits):
    rng = np.random.default_rng(7 + bits)
    idx = rng.integers(0, 1 << bits, size=(50, 128))
    p = O.pack_codes(idx, bits)
    assert p.shape == (50, 128 * bits // 8)
    assert np.array_equal(O.unpack_codes(p, bits, 128), idx)


# ---------------------------------------------------------------- encode

@pytest.mark.parametrize("d", [8, 64, 128, 256])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_rotation_order_on_signed_hadamard_rows(d, bits):
    """x = D r_k (r_k a +-1 Hadamard row) rotates to z = sqrt(d) e_k.

    Holds only for sign flip first, then the natural-order Hadamard, then the
    sqrt(d) scale; a missing or misplaced sign flip, another Hadamard order or
    another scale moves z away from sqrt(d) e_k.
    """
    seed = 42
    s = O.sign_vector(seed, d)
    R = scipy.linalg.hadamard(d).astype(np.float64)
    for k in (0, 1, d // 2 + 3):
        x = (s * R[k]).astype(np.float16)[None, :]
        out = O.encode_detail(x, bits, seed)
        want = np.zeros(d)
        want[k] = math.sqrt(d)
        assert np.abs(out["z"][0] - want).max() < 1e-12
        assert out["idx"][0, k] == (1 << bits) - 1
        assert abs(out["norm64"][0] - math.sqrt(d)) < 1e-12


def test_exact_zero_coordinates_stay_zero():
    """A rotated coordinate that is exactly 0 in real arithmetic gives z == 0
    (and so the upper middle level), not a rounding residue of either sign."""
    d = 128
    s = O.sign_vector(42, d)
    R = scipy.linalg.hadamard(d).astype(np.float64)
    # x = D (r_1 + r_2): rotates to sqrt(d)/|x| (e_1 + e_2) * ..., every other coordinate exactly 0
    x = (s * (R[1] + R[2]) * 0.375).astype(np.float16)[None, :]
    out = O.encode_detail(x, 4, 42)
    zero = np.ones(d, dtype=bool)
    zero[[1, 2]] = False
    assert np.all(out["z"][0, zero] == 0.0)
    assert np.all(out["idx"][0, zero] == 8)


def test_norm_is_float32_of_fp64_norm():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((200, 128)).astype(np.float16)
    out = O.encode_detail(x, 4, 42)
    ref = np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=1))
    assert np.array_equal(out["norms"], ref.astype(np.float32))


def test_zero_vector_convention():
    x = np.zeros((2, 128), dtype=np.float16)
    out = O.encode_detail(x, 4, 42)
    assert np.all(out["idx"] == 8) and np.all(out["norms"] == 0)
    dec = O.decode(out["packed"], out["norms"], 4, 42, 128)
    assert np.all(dec == 0)


def test_encode_shapes_paged_block():
    # "aither-kvcache", section "Paged KV cache": [16, 8, 128] -> [16, 8, 64] + [16, 8]
    x = np.random.default_rng(0).standard_normal((16, 8, 128)).astype(np.float16)
    p, n = O.encode(x, 4, 42)
    assert p.shape == (16, 8, 64) and p.dtype == np.uint8
    assert n.shape == (16, 8) and n.dtype == np.float32


# ---------------------------------------------------------------- decode

@pytest.mark.parametrize("bits", [2, 3, 4])
def test_decode_error_equals_rotated_error(bits):
    """Parseval: the rotation is orthonormal, so the reconstruction error in
    the original domain equals the quantization error of z (scaled).  Fails for
    a decode that drops the sign flip, transposes or rescales the rotation."""
    d = 128
    rng = np.random.default_rng(11 + bits)
    x = rng.standard_normal((300, d)).astype(np.float16)
    enc = O.encode_detail(x, bits, 42)
    xh = O.decode_f64(enc["packed"], enc["norms"], bits, 42, d)
    nrm32 = enc["norms"].astype(np.float64)
    lv = O.format_levels(bits)
    q_err = ((enc["z"] - lv[enc["idx"]]) ** 2).sum(axis=1) / d
    target = x.astype(np.float64) * (nrm32 / enc["norm64"])[:, None]
    got = ((xh - target) ** 2).sum(axis=1)
    assert np.allclose(got, nrm32 ** 2 * q_err, rtol=1e-9, atol=1e-12)


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_encode_decode_mse_matches_sphere_marginal(bits):
    """For iid Gaussian input the rotated unit direction is uniform on the
    sphere whatever the signs are, so each z_i follows the sphere marginal; the
    mean per-coordinate distortion must match its numerical integral."""
    d = 128
    rng = np.random.default_rng(100 + bits)
    x = rng.standard_normal((12000, d)).astype(np.float16)
    enc = O.encode_detail(x, bits, 42)
    xh = O.decode_f64(enc["packed"], enc["norms"], bits, 42, d)
    u = x.astype(np.float64) / enc["norm64"][:, None]
    uh = xh / enc["norms"].astype(np.float64)[:, None]
    emp = ((u - uh) ** 2).sum(axis=1).mean()  # = mean over coords of (z - c)^2
    want = O.sphere_marginal_mse(O.format_levels(bits), d)
    assert abs(emp - want) / want < 0.02, (emp, want)
    # and the sphere marginal is close to the Gaussian one (O(1/d))
    g = O.gaussian_cell_mse(O.format_levels(bits))
    assert abs(want - g) / g < 0.1


# ---------------------------------------------------------------- attention

def _small_cache(rng, B, S, Hkv, d, kb, vb):
    k = rng.standard_normal((B, S, Hkv, d)).astype(np.float16)
    v = rng.standard_normal((B, S, Hkv, d)).astype(np.float16)
    kp, kn = O.encode(k, kb, 42)
    vp, vn = O.encode(v, vb, 42)
    return kp, kn, vp, vn


def test_attention_matches_library_sdpa():
    rng = np.random.default_rng(5)
    B, S, Hq, Hkv, d = 3, 37, 8, 2, 64
    kp, kn, vp, vn = _small_cache(rng, B, S, Hkv, d, 4, 2)
    q = (rng.standard_normal((B, Hq, d)) / math.sqrt(d)).astype(np.float16)
    pos = np.array([37, 1, 20])
    got = O.attend_decode(q, kp, kn, vp, vn, pos, 4, 2)
    K = torch.from_numpy(O.decode_f64(kp, kn, 4, 42, d))  # [B,S,Hkv,d]
    V = torch.from_numpy(O.decode_f64(vp, vn, 2, 42, d))
    for b in range(B):
        n = int(pos[b])
        kk = K[b, :n].permute(1, 0, 2).repeat_interleave(Hq // Hkv, dim=0)  # [Hq,n,d]
        vv = V[b, :n].permute(1, 0, 2).repeat_interleave(Hq // Hkv, dim=0)
        qq = torch.from_numpy(q[b].astype(np.float64))[:, None, :]
        ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv)[:, 0, :]
        assert np.abs(got[b] - ref.numpy()).max() < 1e-12


def test_attention_single_position_and_equal_keys():
    rng = np.random.default_rng(6)
    B, S, Hq, Hkv, d = 2, 9, 4, 1, 128
    kp, kn, vp, vn = _small_cache(rng, B, S, Hkv, d, 4, 2)
    q = rng.standard_normal((B, Hq, d)).astype(np.float16)
    o = O.attend_decode(q, kp, kn, vp, vn, np.array([1, 1]), 4, 2)
    V = O.decode_f64(vp, vn, 2, 42, d)
    for b in range(B):
        assert np.abs(o[b] - V[b, 0, 0][None, :]).max() < 1e-14
    # identical keys everywhere -> uniform weights -> mean of the values
    kp2 = np.repeat(kp[:, :1], S, axis=1)
    kn2 = np.repeat(kn[:, :1], S, axis=1)
    o2 = O.attend_decode(q, kp2, kn2, vp, vn, np.array([S, 5]), 4, 2)
    assert np.abs(o2[0] - V[0, :, 0].mean(axis=0)[None, :]).max() < 1e-12
    assert np.abs(o2[1] - V[1, :5, 0].mean(axis=0)[None, :]).max() < 1e-12


def test_paged_attention_matches_sdpa_on_gathered_rows():
    """Paged cache ("aither-kvcache", section "Paged KV cache"): the oracle's
    block-table gather against torch SDPA on rows picked by flat index
    block_tables[b, s // 16] * 16 + s % 16."""
    rng = np.random.default_rng(9)
    B, Hq, Hkv, d, blk, nblocks, maxb = 3, 8, 2, 64, 16, 11, 4
    pool_k = rng.standard_normal((nblocks * blk, Hkv, d)).astype(np.float16)
    pool_v = rng.standard_normal((nblocks * blk, Hkv, d)).astype(np.float16)
    kp, kn = O.encode(pool_k, 4, 42)
    vp, vn = O.encode(pool_v, 2, 42)
    kc, vc = kp.reshape(nblocks, blk, Hkv, -1), vp.reshape(nblocks, blk, Hkv, -1)
    knc, vnc = kn.reshape(nblocks, blk, Hkv), vn.reshape(nblocks, blk, Hkv)
    bt = np.stack([rng.permutation(nblocks)[:maxb] for _ in range(B)]).astype(np.int32)
    lens = np.array([64, 17, 5])
    q = (rng.standard_normal((B, Hq, d)) / math.sqrt(d)).astype(np.float16)
    got = O.attend_decode_paged(q, kc, knc, vc, vnc, bt, lens, 4, 2)
    K = torch.from_numpy(O.decode_f64(kp, kn, 4, 42, d))  # [rows, Hkv, d]
    V = torch.from_numpy(O.decode_f64(vp, vn, 2, 42, d))
    for b in range(B):
        s = np.arange(lens[b])
        rows = torch.from_numpy(bt[b, s // blk].astype(np.int64) * blk + s % blk)
        kk = K[rows].permute(1, 0, 2).repeat_interleave(Hq // Hkv, dim=0)
        vv = V[rows].permute(1, 0, 2).repeat_interleave(Hq // Hkv, dim=0)
        qq = torch.from_numpy(q[b].astype(np.float64))[:, None, :]
        ref = torch.nn.functional.scaled_dot_product_attention(qq, kk, vv)[:, 0, :]
        assert np.abs(got[b] - ref.numpy()).max() < 1e-12


def test_paged_attention_with_identity_table_is_contiguous_attention():
    rng = np.random.default_rng(10)
    B, S, Hq, Hkv, d = 2, 48, 4, 2, 64
    kp, kn, vp, vn = _small_cache(rng, B, S, Hkv, d, 3, 3)
    q = rng.standard_normal((B, Hq, d)).astype(np.float16)
    pos = np.array([48, 33])
    want = O.attend_decode(q, kp, kn, vp, vn, pos, 3, 3)
    nb = S // 16
    kc = kp.reshape(B * nb, 16, Hkv, -1)
    vc = vp.reshape(B * nb, 16, Hkv, -1)
    knc, vnc = kn.reshape(B * nb, 16, Hkv), vn.reshape(B * nb, 16, Hkv)
    bt = np.arange(B * nb, dtype=np.int32).reshape(B, nb)
    got = O.attend_decode_paged(q, kc, knc, vc, vnc, bt, pos, 3, 3)
    assert np.array_equal(got, want)


# ---------------------------------------------- offset + half-precision scale

def test_os_side_data_layout_and_constant_vectors():
    """Side data = fp16 bits of the offset | fp16 bits of the scale << 16:
    [1, 3, 1, 3, ...] has mean 2 and centred norm sqrt(64) = 8 (fp16 0x4000
    and 0x4800). A constant vector has scale 0, codes 2^(b-1) and decodes to
    itself exactly."""
    d = 64
    x = np.tile(np.array([1.0, 3.0], dtype=np.float16), d // 2)[None, :]
    det = O.encode_os_detail(x, 4, 42)
    assert int(det["side"][0]) == 0x4000 | (0x4800 << 16)
    c = np.full((3, 128), [[-2.5], [0.0], [1000.0]], dtype=np.float16)
    for bits in (2, 3, 4):
        p, sd = O.encode_os(c, bits, 7)
        assert np.all(O.unpack_codes(p, bits, 128) == 2 ** (bits - 1))
        assert np.array_equal(O.decode_os(p, sd, bits, 7, 128), c)


def test_os_codes_are_translation_invariant():
    """Adding a constant c to a zero-mean integer vector (every value, the
    mean c and the centred vector stay exact in fp16) leaves codes and scale
    unchanged and makes the offset c."""
    rng = np.random.default_rng(21)
    h = rng.integers(-40, 40, size=(50, 64)).astype(np.float16)
    x = np.concatenate([h, -h], axis=1)
    a = O.encode_os_detail(x, 3, 42)
    assert np.all(a["mu16"] == 0)
    for c in (4.0, -16.0, 100.0):
        b = O.encode_os_detail((x.astype(np.float64) + c).astype(np.float16), 3, 42)
        assert np.all(b["mu16"].astype(np.float64) == c)
        assert np.array_equal(a["idx"], b["idx"])
        assert np.array_equal(a["n16"], b["n16"])


def test_os_zero_mean_matches_turboquant_with_rounded_norm():
    """For vectors with an exactly zero mean the offset is 0 and the codes are
    the TurboQuant codes of the same vector with the norm rounded to fp16."""
    rng = np.random.default_rng(22)
    h = rng.standard_normal((200, 64)).astype(np.float16)
    x = np.concatenate([h, -h], axis=1)  # mean exactly 0
    os_ = O.encode_os_detail(x, 4, 42)
    tq = O.encode_detail(x, 4, 42)
    assert np.all(os_["mu16"] == 0)
    z = tq["z"] * (tq["norm64"] / os_["n16"].astype(np.float64))[:, None]
    assert np.array_equal(O.quantize(z, O.format_boundaries(O.format_levels(4))), os_["idx"])


@pytest.mark.parametrize("bits", [2, 3, 4])
def test_os_distortion_of_centred_gaussian_rows(bits):
    """Gaussian rows with a random offset: the per-coordinate distortion of the
    centred direction is the sphere-marginal value, as for TurboQuant (the fp16
    scale moves it by < 1e-3 relative)."""
    d = 128
    rng = np.random.default_rng(30 + bits)
    x = (rng.standard_normal((8000, d)) + rng.uniform(-3, 3, size=(8000, 1))).astype(np.float16)
    det = O.encode_os_detail(x, bits, 42)
    xh = O.decode_os_f64(det["packed"], det["side"], bits, 42, d)
    mu = det["mu16"].astype(np.float64)[:, None]
    y = x.astype(np.float64) - mu
    yh = xh - mu
    # ||y - yh||^2 / ||y||^2 = (n16 / ||y||)^2 * mean over coordinates of (z - c)^2
    emp = (((y - yh) ** 2).sum(axis=1) / (y * y).sum(axis=1)).mean()
    want = O.sphere_marginal_mse(O.format_levels(bits), d)
    assert abs(emp - want) / want < 0.02, (emp, want)
