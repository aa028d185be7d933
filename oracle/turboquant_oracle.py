"""Plain, slow, fp64 reference of the TurboQuant KV-cache codec.

TEST INFRASTRUCTURE ONLY -- never called by the library. Every routine below is
the plain definition of one step, written in fp64 with numpy (matrix products
and element-wise ops only; no fast transforms, no blocking, no fusion).

Sources (page title, then section):

* "aither-kvcache" (PyPI project page), section "Algorithm": normalise (extract
  the L2 norm, project to the unit sphere), rotate by a fixed data-oblivious
  random orthogonal matrix so each coordinate is ~N(0, 1/d), quantize each
  coordinate with a precomputed Lloyd-Max codebook, pack indices into uint8,
  store packed bytes plus a float32 norm; decoding reverses the steps.
* same page, sections "Quick Start -- TurboQuant" and "Paged KV cache":
  ``[..., 128] fp16 -> [..., 64] uint8 + [...] f32`` at 4 bits, arbitrary
  leading dimensions; constructor default ``seed=42`` ("API Reference").
* same page, section "Zero-buffer fused attention": rotate the query once,
  score in the rotated domain against codebook values, accumulate values in
  the rotated domain, rotate back once.
* "TurboQuant efficient inference" (qbc.network blog), section "What TurboQuant
  is": the rotation is a multiplier-free Walsh-Hadamard transform and the levels
  are the known optimal set for a bell curve (no calibration); section "2. A
  fused decode path": rotating only the query and folding the rotation onto the
  output equals the straightforward computation up to rounding.

Readings taken where the pages are silent:

* rotation = random +-1 sign flip D, then the orthonormal Walsh-Hadamard matrix
  H in natural (Sylvester) order, H[i, j] = (-1)^popcount(i & j) / sqrt(d);
  z = sqrt(d) * H D u.
* sign i is -1 iff bit 63 of the i-th splitmix64 output (seeded with ``seed``)
  is set (splitmix64: S. Vigna, public-domain reference generator).
  ``splitmix64`` and ``sign_vector`` are pinned to Vigna's published outputs,
  but the pages neither name their own generator nor print any sign or
  packed byte, so agreement with the pages' sign table is parity unpinned.
* the format codebook is the fp64 Lloyd-Max codebook for N(0, 1) snapped to the
  2^-14 grid; decision boundaries are the midpoints of the snapped levels;
  index = number of boundaries t with z >= t (ties go to the upper level).
* a zero vector has norm 0 and z := 0 (all indices 2^(b-1)).
* packing: little-endian bitstream, code i occupies stream bits [i*b, i*b+b),
  stream bit k is bit (k mod 8) of byte k // 8.
* attention: softmax scale 1/sqrt(d); query head h reads kv head
  h // (Hq / Hkv); ``positions[b]`` is the number of valid cache positions.
"""

from __future__ import annotations

import math

import numpy as np

__all__ = [
    "FORMAT_GRID_BITS",
    "lloyd_max_levels",
    "gaussian_cell_mse",
    "format_levels",
    "format_boundaries",
    "splitmix64",
    "sign_vector",
    "hadamard",
    "hadamard_pm",
    "packed_bytes",
    "compressed_bytes_per_vector",
    "pack_codes",
    "unpack_codes",
    "quantize",
    "encode",
    "encode_detail",
    "decode_f64",
    "decode",
    "attend_decode",
    "attend_decode_paged",
    "encode_os_detail",
    "encode_os",
    "decode_os_f64",
    "decode_os",
    "sphere_marginal_mse",
]

FORMAT_GRID_BITS = 14  # levels are stored on the 2^-14 grid (reading O7)


# --------------------------------------------------------------------------
# Codebook: Lloyd-Max quantizer for the standard normal density
# ("aither-kvcache", section "Algorithm", step 3; "TurboQuant efficient
# inference", section "What TurboQuant is": optimal levels for a bell curve,
# computed from the density, no calibration data).
# --------------------------------------------------------------------------

def _phi(x: float) -> float:
    """Standard normal density; 0 at +-inf."""
    if math.isinf(x):
        return 0.0
    return math.exp(-0.5 * x * x) / math.sqrt(2.0 * math.pi)


def _mass(a: float, b: float) -> float:
    """P(a <= X < b) for X ~ N(0,1), from erfc so the tails keep precision."""
    # Phi(x) = erfc(-x / sqrt 2) / 2; for a >= 0 use the upper-tail form.
    if a >= 0.0:
        return 0.5 * (math.erfc(a / math.sqrt(2.0)) - math.erfc(b / math.sqrt(2.0)))
    if b <= 0.0:
        return 0.5 * (math.erfc(-b / math.sqrt(2.0)) - math.erfc(-a / math.sqrt(2.0)))
    return 1.0 - 0.5 * math.erfc(-a / math.sqrt(2.0)) - 0.5 * math.erfc(b / math.sqrt(2.0))


def lloyd_max_levels(bits: int, tol: float = 1e-15, max_iter: int = 200000) -> np.ndarray:
    """Lloyd-Max levels for N(0,1) with 2^bits cells, ascending, fp64.

    Lloyd's iteration: boundaries are midpoints of neighbouring levels
    (t_0 = -inf, t_L = +inf) and each level moves to the conditional mean of
    its cell, E[X | t_k <= X < t_{k+1}] = (phi(t_k) - phi(t_{k+1})) / mass.
    Starts from a uniform spread and stops when no level moves by more than
    ``tol``.
    """
    L = 1 << bits
    c = [(-1.0 + (2.0 * k + 1.0) / L) * 2.0 for k in range(L)]
    for _ in range(max_iter):
        t = [-math.inf] + [0.5 * (c[k - 1] + c[k]) for k in range(1, L)] + [math.inf]
        new = [(_phi(t[k]) - _phi(t[k + 1])) / _mass(t[k], t[k + 1]) for k in range(L)]
        delta = max(abs(new[k] - c[k]) for k in range(L))
        c = new
        if delta < tol:
            break
    return np.array(c, dtype=np.float64)


def gaussian_cell_mse(levels: np.ndarray, boundaries: np.ndarray | None = None) -> float:
    """E[(X - Q(X))^2] for X ~ N(0,1), closed form per cell.

    Uses int_a^b x^2 phi = mass - [x phi]_a^b and int_a^b x phi = phi(a) - phi(b).
    ``boundaries`` default to the midpoints of ``levels``.
    """
    c = [float(v) for v in levels]
    L = len(c)
    if boundaries is None:
        inner = [0.5 * (c[k - 1] + c[k]) for k in range(1, L)]
    else:
        inner = [float(v) for v in boundaries]
    t = [-math.inf] + inner + [math.inf]
    total = 0.0
    for k in range(L):
        a, b = t[k], t[k + 1]
        m = _mass(a, b)
        xphi_a = 0.0 if math.isinf(a) else a * _phi(a)
        xphi_b = 0.0 if math.isinf(b) else b * _phi(b)
        second = m - (xphi_b - xphi_a)
        first = _phi(a) - _phi(b)
        total += second - 2.0 * c[k] * first + c[k] * c[k] * m
    return total


def format_levels(bits: int) -> np.ndarray:
    """Format levels: the Lloyd-Max levels rounded to the 2^-14 grid (fp64)."""
    scale = float(1 << FORMAT_GRID_BITS)
    return np.round(lloyd_max_levels(bits) * scale) / scale


def format_boundaries(levels: np.ndarray) -> np.ndarray:
    """Decision boundaries t_j = (c_{j-1} + c_j) / 2, j = 1 .. L-1."""
    return 0.5 * (levels[:-1] + levels[1:])


# --------------------------------------------------------------------------
# Random sign flip (the random part of the rotation)
# --------------------------------------------------------------------------

_MASK64 = (1 << 64) - 1


def splitmix64(seed: int, count: int) -> list[int]:
    """First ``count`` outputs of Vigna's splitmix64 seeded with ``seed``.

    state += 0x9E3779B97F4A7C15; z = state;
    z = (z ^ z >> 30) * 0xBF58476D1CE4E5B9; z = (z ^ z >> 27) * 0x94D049BB133111EB;
    output z ^ z >> 31 (all arithmetic mod 2^64).
    """
    state = seed & _MASK64
    out = []
    for _ in range(count):
        state = (state + 0x9E3779B97F4A7C15) & _MASK64
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
        out.append(z ^ (z >> 31))
    return out


def sign_vector(seed: int, d: int) -> np.ndarray:
    """s_i = -1 if bit 63 of the i-th splitmix64 output is set, else +1."""
    return np.array([-1.0 if (v >> 63) & 1 else 1.0 for v in splitmix64(seed, d)])


# --------------------------------------------------------------------------
# Orthonormal Walsh-Hadamard matrix ("TurboQuant efficient inference",
# section "What TurboQuant is"), dense, natural (Sylvester) order.
# --------------------------------------------------------------------------

def hadamard_pm(d: int) -> np.ndarray:
    """The unnormalised +-1 Walsh-Hadamard matrix, (-1)^popcount(i & j), entry by entry."""
    if d < 1 or d & (d - 1):
        raise ValueError("d must be a power of two")
    H = np.empty((d, d), dtype=np.float64)
    for i in range(d):
        for j in range(d):
            H[i, j] = -1.0 if bin(i & j).count("1") % 2 else 1.0
    return H


def hadamard(d: int) -> np.ndarray:
    """Orthonormal H[i, j] = (-1)^popcount(i & j) / sqrt(d)."""
    return hadamard_pm(d) / math.sqrt(d)


# --------------------------------------------------------------------------
# Sizes ("aither-kvcache", "Quick Start -- TurboQuant": 128 fp16 -> 64 uint8 + f32)
# --------------------------------------------------------------------------

def packed_bytes(d: int, bits: int) -> int:
    """Bytes of packed codes per vector: d * b / 8."""
    return d * bits // 8


def compressed_bytes_per_vector(d: int, bits: int) -> int:
    """Packed codes plus the float32 norm."""
    return packed_bytes(d, bits) + 4


# --------------------------------------------------------------------------
# Bit packing ("aither-kvcache", section "Algorithm", step 4)
# --------------------------------------------------------------------------

def pack_codes(idx: np.ndarray, bits: int) -> np.ndarray:
    """[n, d] integer codes -> [n, d*b/8] uint8 little-endian bitstream.

    Stream bit i*b + j is bit j of code i; stream bit k lives in bit (k mod 8)
    of byte k // 8.
    """
    idx = np.asarray(idx, dtype=np.int64)
    n, d = idx.shape
    if (d * bits) % 8:
        raise ValueError("d * bits must be a multiple of 8")
    stream = np.zeros((n, d * bits), dtype=np.uint8)
    for j in range(bits):
        stream[:, j::bits] = (idx >> j) & 1
    weights = (1 << np.arange(8)).astype(np.int64)
    return (stream.reshape(n, d * bits // 8, 8).astype(np.int64) @ weights).astype(np.uint8)


def unpack_codes(packed: np.ndarray, bits: int, d: int) -> np.ndarray:
    """Inverse of :func:`pack_codes`: [n, d*b/8] uint8 -> [n, d] int64 codes."""
    packed = np.asarray(packed, dtype=np.uint8)
    n = packed.shape[0]
    stream = ((packed[:, :, None] >> np.arange(8, dtype=np.uint8)) & 1).reshape(n, -1)
    idx = np.zeros((n, d), dtype=np.int64)
    for j in range(bits):
        idx |= stream[:, j::bits][:, :d].astype(np.int64) << j
    return idx


# --------------------------------------------------------------------------
# Quantizer ("aither-kvcache", section "Algorithm", step 3)
# --------------------------------------------------------------------------

def quantize(z: np.ndarray, boundaries: np.ndarray) -> np.ndarray:
    """Index of the nearest level: the number of boundaries t_j with z >= t_j."""
    z = np.asarray(z, dtype=np.float64)
    return (z[..., None] >= boundaries).sum(axis=-1).astype(np.int64)


# --------------------------------------------------------------------------
# Encode / decode ("aither-kvcache", section "Algorithm", steps 1-5 and
# "Decoding reverses steps 4-1")
# --------------------------------------------------------------------------

def _as_rows(x: np.ndarray, d: int) -> np.ndarray:
    x = np.asarray(x)
    if x.shape[-1] != d:
        raise ValueError("last dimension must be head_dim")
    return x.reshape(-1, d)


def encode_detail(x_f16: np.ndarray, bits: int, seed: int) -> dict:
    """Encode ``[..., d]`` fp16 rows; also return the intermediate values.

    Returns a dict with ``packed`` [n, d*b/8] uint8, ``norms`` [n] float32,
    ``idx`` [n, d] codes, ``z`` [n, d] scaled rotated coordinates (fp64) and
    ``norm64`` [n] (fp64 norm before the float32 rounding).
    """
    x16 = np.asarray(x_f16)
    if x16.dtype != np.float16:
        raise TypeError("input must be float16")
    d = x16.shape[-1]
    x = _as_rows(x16, d).astype(np.float64)  # fp16 -> fp64 is exact
    norm64 = np.sqrt((x * x).sum(axis=1))
    # steps 1-2: z = sqrt(d) * H D (x / N) with H orthonormal, written as
    # (H_pm D x) / N: H_pm D x is a sum of +-x_k, exact in fp64 for fp16 input
    # (multiples of 2^-24 below 2^23), so the only rounding is the final
    # division and a coordinate that is exactly 0 stays exactly 0.
    # (zero vector -> z = 0)
    s = sign_vector(seed, d)
    w = (x * s[None, :]) @ hadamard_pm(d).T
    safe = np.where(norm64 > 0.0, norm64, 1.0)
    z = np.where(norm64[:, None] > 0.0, w / safe[:, None], 0.0)
    # step 3: nearest level of the format codebook
    t = format_boundaries(format_levels(bits))
    idx = quantize(z, t)
    # steps 4-5: pack, store float32 norm
    return {
        "packed": pack_codes(idx, bits),
        "norms": norm64.astype(np.float32),
        "idx": idx,
        "z": z,
        "norm64": norm64,
    }


def encode(x_f16: np.ndarray, bits: int, seed: int = 42):
    """``[..., d]`` fp16 -> (``[..., d*b/8]`` uint8, ``[...]`` float32)."""
    x16 = np.asarray(x_f16)
    lead = x16.shape[:-1]
    out = encode_detail(x16, bits, seed)
    P = packed_bytes(x16.shape[-1], bits)
    return out["packed"].reshape(*lead, P), out["norms"].reshape(lead)


def decode_f64(packed: np.ndarray, norms: np.ndarray, bits: int, seed: int, d: int) -> np.ndarray:
    """Decoded rows in fp64 before the final fp16 rounding.

    x_hat = norm * D H (c[idx] / sqrt(d)), H symmetric orthonormal, D the signs.
    """
    packed = np.asarray(packed, dtype=np.uint8)
    P = packed_bytes(d, bits)
    lead = packed.shape[:-1]
    rows = packed.reshape(-1, P)
    nrm = np.asarray(norms, dtype=np.float32).reshape(-1).astype(np.float64)
    idx = unpack_codes(rows, bits, d)
    levels = format_levels(bits)
    y = levels[idx] / math.sqrt(d)
    H = hadamard(d)
    u = (y @ H) * sign_vector(seed, d)[None, :]
    return (u * nrm[:, None]).reshape(*lead, d)


def decode(packed: np.ndarray, norms: np.ndarray, bits: int, seed: int, d: int) -> np.ndarray:
    """Decode to fp16 (round to nearest even from fp64). A value beyond the
    fp16 range rounds to +-inf, which is what the cast gives; numpy's warning
    for that case is not raised."""
    with np.errstate(over="ignore"):
        return decode_f64(packed, norms, bits, seed, d).astype(np.float16)


# --------------------------------------------------------------------------
# Decode-step attention over a packed cache, done the straightforward way:
# decode K and V in fp64, then softmax attention ("aither-kvcache", section
# "Zero-buffer fused attention"; "TurboQuant efficient inference", section
# "2. A fused decode path" -- the fused form must equal this up to rounding).
# --------------------------------------------------------------------------

def attend_decode(q_f16, k_packed, k_norms, v_packed, v_norms, positions,
                  k_bits: int, v_bits: int, k_seed: int = 42, v_seed: int = 42) -> np.ndarray:
    """One decode step of attention over a contiguous packed cache, in fp64.

    q_f16: [B, Hq, d] fp16; k_packed: [B, S, Hkv, d*bk/8]; k_norms: [B, S, Hkv];
    v_packed / v_norms likewise; positions: [B] valid lengths (1..S).
    Returns o [B, Hq, d] fp64 with o = softmax(q k^T / sqrt(d)) v over the first
    positions[b] cache slots, query head h reading kv head h // (Hq / Hkv).
    """
    q = np.asarray(q_f16)
    if q.dtype != np.float16:
        raise TypeError("query must be float16")
    q = q.astype(np.float64)
    B, Hq, d = q.shape
    kp = np.asarray(k_packed)
    Hkv = kp.shape[2]
    if Hq % Hkv:
        raise ValueError("Hq must be a multiple of Hkv")
    group = Hq // Hkv
    out = np.zeros((B, Hq, d), dtype=np.float64)
    for b in range(B):
        n = int(positions[b])
        K = decode_f64(kp[b, :n], np.asarray(k_norms)[b, :n], k_bits, k_seed, d)  # [n, Hkv, d]
        V = decode_f64(np.asarray(v_packed)[b, :n], np.asarray(v_norms)[b, :n], v_bits, v_seed, d)
        for h in range(Hq):
            kv = h // group
            s = K[:, kv, :] @ q[b, h] / math.sqrt(d)
            p = np.exp(s - s.max())
            p /= p.sum()
            out[b, h] = p @ V[:, kv, :]
    return out


def attend_decode_paged(q_f16, k_cache, k_norms, v_cache, v_norms, block_tables, context_lens,
                        k_bits: int, v_bits: int, k_seed: int = 42, v_seed: int = 42,
                        block_size: int = 16) -> np.ndarray:
    """attend_decode over a paged cache ("aither-kvcache", section "Paged KV
    cache": blocks of 16 positions, a block table per sequence).

    k_cache: [num_blocks, block_size, Hkv, P]; k_norms: [num_blocks,
    block_size, Hkv]; v likewise; block_tables: [B, max_blocks], entry j of
    row b the block holding positions [block_size j, block_size (j + 1)) of
    sequence b; context_lens: [B]. Gathers each sequence's positions in order
    and applies attend_decode to them.
    """
    q = np.asarray(q_f16)
    B = q.shape[0]
    kc, vc = np.asarray(k_cache), np.asarray(v_cache)
    kn, vn = np.asarray(k_norms), np.asarray(v_norms)
    bt = np.asarray(block_tables)
    out = np.zeros(q.shape, dtype=np.float64)
    for b in range(B):
        n = int(context_lens[b])
        nb = -(-n // block_size)
        blocks = [int(bt[b, j]) for j in range(nb)]
        kb = np.concatenate([kc[j] for j in blocks], axis=0)[:n]
        vb = np.concatenate([vc[j] for j in blocks], axis=0)[:n]
        knb = np.concatenate([kn[j] for j in blocks], axis=0)[:n]
        vnb = np.concatenate([vn[j] for j in blocks], axis=0)[:n]
        out[b] = attend_decode(q[b:b + 1], kb[None], knb[None], vb[None], vnb[None], [n],
                               k_bits, v_bits, k_seed, v_seed)[0]
    return out


def _side_pack(mu16: np.ndarray, n16: np.ndarray) -> np.ndarray:
    return (mu16.astype(np.float16).view(np.uint16).astype(np.uint32)
            | (n16.astype(np.float16).view(np.uint16).astype(np.uint32) << 16))


def _side_unpack(side: np.ndarray):
    side = np.asarray(side, dtype=np.uint32).reshape(-1)
    mu16 = (side & 0xFFFF).astype(np.uint16).view(np.float16)
    n16 = (side >> 16).astype(np.uint16).view(np.float16)
    return mu16, n16


def encode_os_detail(x_f16: np.ndarray, bits: int, seed: int, side=None) -> dict:
    """The offset + half-precision scale variant ("TurboQuant efficient
    inference", section "1. The quantizer": remove a small per-vector offset,
    rotate, round each coordinate to a level, keep one scale alongside, codes
    packed two per byte at 4 bits, scales in half precision).

    Reading: offset mu16 = fp16(mean(x)); y = x - mu16; scale n16 =
    fp16(||y||); then the TurboQuant step on y with n16 in place of the norm:
    z = (H_pm D y) / n16, index_i = #{j : z_i >= t_j}. Side data per vector:
    uint32 = fp16 bits of mu16 | fp16 bits of n16 << 16.

    ``side``: optional [n] uint32 to use instead of computing mu16 and n16
    (to check codes given another implementation's side data).
    """
    x16 = np.asarray(x_f16)
    if x16.dtype != np.float16:
        raise TypeError("input must be float16")
    d = x16.shape[-1]
    x = _as_rows(x16, d).astype(np.float64)
    if side is None:
        mu16 = (x.sum(axis=1) / d).astype(np.float16)  # the fp16 sum is exact in fp64; /d exact
        y = x - mu16.astype(np.float64)[:, None]        # exact: both fp16
        nrm = np.sqrt((y * y).sum(axis=1))
        with np.errstate(over="ignore"):
            n16 = nrm.astype(np.float16)
    else:
        mu16, n16 = _side_unpack(side)
        y = x - mu16.astype(np.float64)[:, None]
        nrm = np.sqrt((y * y).sum(axis=1))
    nq = n16.astype(np.float64)
    s = sign_vector(seed, d)
    w = (y * s[None, :]) @ hadamard_pm(d).T  # sums of +-y_k: exact in fp64
    ok = (nq > 0.0) & np.isfinite(nq)
    z = np.where(ok[:, None], w / np.where(ok, nq, 1.0)[:, None], 0.0)
    idx = quantize(z, format_boundaries(format_levels(bits)))
    return {"packed": pack_codes(idx, bits), "side": _side_pack(mu16, n16), "idx": idx, "z": z,
            "mu16": mu16, "n16": n16, "norm64": nrm}


def encode_os(x_f16: np.ndarray, bits: int, seed: int = 42):
    """``[..., d]`` fp16 -> (``[..., d*b/8]`` uint8, ``[...]`` uint32 side data)."""
    x16 = np.asarray(x_f16)
    lead = x16.shape[:-1]
    out = encode_os_detail(x16, bits, seed)
    return out["packed"].reshape(*lead, packed_bytes(x16.shape[-1], bits)), out["side"].reshape(lead)


def decode_os_f64(packed: np.ndarray, side: np.ndarray, bits: int, seed: int, d: int) -> np.ndarray:
    """x_hat = mu16 + (n16 / d) D H_pm c[idx] in fp64, before the fp16 rounding."""
    pk = np.asarray(packed)
    lead = pk.shape[:-1]
    idx = unpack_codes(pk.reshape(-1, pk.shape[-1]), bits, d)
    c = format_levels(bits)[idx]
    mu16, n16 = _side_unpack(side)
    hc = c @ hadamard_pm(d).T * sign_vector(seed, d)[None, :]
    out = mu16.astype(np.float64)[:, None] + (n16.astype(np.float64) / d)[:, None] * hc
    return out.reshape(*lead, d)


def decode_os(packed: np.ndarray, side: np.ndarray, bits: int, seed: int, d: int) -> np.ndarray:
    return decode_os_f64(packed, side, bits, seed, d).astype(np.float16)


# --------------------------------------------------------------------------
# Statistics used as pins
# --------------------------------------------------------------------------

def sphere_marginal_mse(levels: np.ndarray, d: int) -> float:
    """E[(z - Q(z))^2] when z = sqrt(d) * (one coordinate of a uniform unit vector).

    The coordinate y of a uniform point on the unit sphere in R^d has density
    proportional to (1 - y^2)^((d - 3) / 2) on [-1, 1]; z = sqrt(d) y.
    Integrated numerically cell by cell.
    """
    from scipy import integrate, special

    levels = np.asarray(levels, dtype=np.float64)
    t = format_boundaries(levels)
    r = math.sqrt(d)
    # normalising constant of the density of z on [-r, r]
    log_norm = special.gammaln(d / 2.0) - special.gammaln((d - 1) / 2.0) - 0.5 * math.log(math.pi * d)

    def dens(z):
        v = 1.0 - z * z / d
        if v <= 0.0:
            return 0.0
        return math.exp(log_norm + 0.5 * (d - 3) * math.log(v))

    edges = [-r] + [float(v) for v in t] + [r]
    total = 0.0
    for k, c in enumerate(levels):
        a, b = max(edges[k], -r), min(edges[k + 1], r)
        if b <= a:
            continue
        val, _ = integrate.quad(lambda z: (z - c) ** 2 * dens(z), a, b, epsabs=1e-14, epsrel=1e-12, limit=200)
        total += val
    return total
