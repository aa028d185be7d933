"""Comparison rules between the CUDA path and the fp64 oracle.

* codes: bit-exact, except coordinates whose oracle value z lies within 1e-5
  of a decision boundary; those mismatches are counted and must stay below
  1e-6 of all coordinates (``max_boundary_frac``);
* norms: relative error <= 1e-6 (both encode kernels);
* decoded fp16: <= 1 fp16 ulp from the oracle's decode of the same bytes;
* attention: per output row, max |o - o_ref| / max |o_ref| <= 2e-3.
"""

from __future__ import annotations

import numpy as np

import oracle as O

BOUNDARY_BAND = 1e-5
NORM_RTOL = 1e-6
ATTN_RTOL = 2e-3


def code_mismatches(gpu_packed: np.ndarray, detail: dict, bits: int, d: int, max_boundary_frac=1e-6):
    """Return the number of code mismatches; assert each lies in the boundary band."""
    gi = O.unpack_codes(np.asarray(gpu_packed).reshape(-1, d * bits // 8), bits, d)
    oi = detail["idx"]
    mism = gi != oi
    n = int(mism.sum())
    if n:
        t = O.format_boundaries(O.format_levels(bits))
        z = detail["z"][mism]
        dist = np.min(np.abs(z[:, None] - t[None, :]), axis=1)
        assert np.all(dist < BOUNDARY_BAND), f"{n} mismatches, max boundary distance {dist.max():.3g}"
        # a mismatch may only move to the neighbouring level
        assert np.all(np.abs(gi[mism] - oi[mism]) == 1)
    if max_boundary_frac is not None:
        assert n <= max_boundary_frac * gi.size, f"{n} boundary mismatches of {gi.size}"
    return n


def assert_norms(gpu_norms: np.ndarray, detail: dict, rtol: float = NORM_RTOL):
    g = np.asarray(gpu_norms, dtype=np.float64).reshape(-1)
    ref = detail["norm64"]
    err = np.abs(g - ref)
    lim = rtol * np.abs(ref)
    assert np.all(err <= lim), f"norm rel err {np.max(err / np.maximum(np.abs(ref), 1e-300)):.3g}"


def _ordered(h: np.ndarray) -> np.ndarray:
    """fp16 bit patterns -> integers ordered like the values (+0 == -0)."""
    u = h.view(np.uint16).astype(np.int32)
    return np.where(u & 0x8000, -(u & 0x7FFF), u)


def fp16_ulp_distance(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    return np.abs(_ordered(np.asarray(a, dtype=np.float16)) - _ordered(np.asarray(b, dtype=np.float16)))


def assert_decode_ulp(gpu_x: np.ndarray, ref_x: np.ndarray, max_ulp: int = 1):
    dist = fp16_ulp_distance(gpu_x, ref_x)
    assert dist.max() <= max_ulp, f"max fp16 ulp distance {dist.max()}"


def attn_row_error(o: np.ndarray, ref: np.ndarray) -> np.ndarray:
    """Per (b, h) row: max_i |o_i - ref_i| / max_i |ref_i|."""
    o = np.asarray(o, dtype=np.float64)
    num = np.abs(o - ref).max(axis=-1)
    den = np.maximum(np.abs(ref).max(axis=-1), 1e-30)
    return num / den


def os_decode_ok(gpu16, exact, mu16):
    """fp16 decode of the offset variant against the fp64 value of the same
    bytes: within half an fp16 ulp of the exact value plus the two f32
    roundings (product, sum with the offset)."""
    g = np.asarray(gpu16, dtype=np.float64)
    a = np.abs(exact)
    ulp = np.where(a >= 2.0 ** -14, 2.0 ** (np.floor(np.log2(np.maximum(a, 2.0 ** -14))) - 10), 2.0 ** -24)
    mu = np.abs(mu16.astype(np.float64))[:, None]
    tol = 0.5 * ulp + 2.0 ** -22 * (mu + np.abs(exact - mu16.astype(np.float64)[:, None])) + 1e-30
    return np.abs(g - exact) <= tol
