"""Planted mistakes in the oracle must be caught by the pins.

Each case patches one step of the fp64 oracle (on the CPU, inside this test
process only) with a plausible mistake and checks that at least one pin from
``test_oracle_pins`` fails. This shows the pins constrain every step.
"""

import numpy as np
import pytest
import scipy.linalg

import oracle
import oracle.turboquant_oracle as T
import test_oracle_pins as P


class _Patch:
    """Patch a name in the oracle module and in the package that re-exports it."""

    def __init__(self, mp):
        self.mp = mp

    def setattr(self, _mod, name, value):
        self.mp.setattr(T, name, value)
        self.mp.setattr(oracle, name, value)


@pytest.fixture
def patch(monkeypatch):
    return _Patch(monkeypatch)


def _sequency_hadamard(d):
    # rows reordered by number of sign changes (Walsh order) instead of natural
    H = _natural(d)
    changes = [(np.diff(np.sign(H[i])) != 0).sum() for i in range(d)]
    return H[np.argsort(changes, kind="stable")]


def _natural(d):
    return scipy.linalg.hadamard(d).astype(np.float64) / np.sqrt(d)


def _fails(fn, *args):
    try:
        fn(*args)
    except AssertionError:
        return True
    return False


def test_constant_signs_are_caught(patch):
    patch.setattr(T, "sign_vector", lambda seed, d: np.ones(d))
    assert _fails(P.test_sign_vector_is_bit63)


def _encode_variant(order):
    def enc(x_f16, bits, seed):
        d = x_f16.shape[-1]
        x = np.asarray(x_f16).reshape(-1, d).astype(np.float64)
        nrm = np.sqrt((x * x).sum(axis=1))
        u = x / nrm[:, None]
        H = T.hadamard(d)
        s = T.sign_vector(seed, d)
        if order == "no-sign":
            y = u @ H.T
        else:  # Hadamard first, then the sign flip
            y = (u @ H.T) * s
        z = np.sqrt(d) * y
        idx = T.quantize(z, T.format_boundaries(T.format_levels(bits)))
        return {"packed": T.pack_codes(idx, bits), "norms": nrm.astype(np.float32),
                "idx": idx, "z": z, "norm64": nrm}
    return enc


def test_dropped_sign_flip_is_caught(patch):
    patch.setattr(T, "encode_detail", _encode_variant("no-sign"))
    assert _fails(P.test_rotation_order_on_signed_hadamard_rows, 128, 4)


def test_sign_after_hadamard_is_caught(patch):
    patch.setattr(T, "encode_detail", _encode_variant("sign-last"))
    assert _fails(P.test_rotation_order_on_signed_hadamard_rows, 128, 4)


def test_sequency_order_is_caught(patch):
    patch.setattr(T, "hadamard", _sequency_hadamard)
    assert _fails(P.test_hadamard_is_sylvester_and_orthonormal, 128)


def test_missing_sqrt_d_scale_is_caught(patch):
    orig = T.quantize
    patch.setattr(T, "quantize", lambda z, t: orig(np.asarray(z) / np.sqrt(128), t))
    assert _fails(P.test_encode_decode_mse_matches_sphere_marginal, 4)


def test_strict_tie_rule_is_caught(patch):
    patch.setattr(T, "quantize", lambda z, t: (np.asarray(z)[..., None] > t).sum(axis=-1))
    assert _fails(P.test_quantize_ties_go_up, 3)


def test_big_endian_bit_order_is_caught(patch):
    orig = T.pack_codes

    def msb_first(idx, bits):
        p = orig(idx, bits)
        rev = np.array([int(f"{v:08b}"[::-1], 2) for v in range(256)], dtype=np.uint8)
        return rev[p]

    patch.setattr(T, "pack_codes", msb_first)
    assert _fails(P.test_pack_golden_patterns)


def test_decode_without_signs_is_caught(patch):
    orig_sign = T.sign_vector
    orig_decode = T.decode_f64

    def dec(packed, norms, bits, seed, d):
        patch.setattr(T, "sign_vector", lambda s, dd: np.ones(dd))
        try:
            return orig_decode(packed, norms, bits, seed, d)
        finally:
            patch.setattr(T, "sign_vector", orig_sign)

    patch.setattr(T, "decode_f64", dec)
    assert _fails(P.test_decode_error_equals_rotated_error, 4)


def test_boundaries_not_midpoints_is_caught(patch):
    patch.setattr(T, "format_boundaries", lambda lv: 0.6 * lv[:-1] + 0.4 * lv[1:])
    assert _fails(P.test_quantize_is_nearest_level, 3)


def test_attention_scale_mistake_is_caught(patch):
    orig = T.attend_decode

    def wrong(q, *a, **k):
        return orig((np.asarray(q).astype(np.float32) * 2).astype(np.float16), *a, **k)

    patch.setattr(T, "attend_decode", wrong)
    assert _fails(P.test_attention_matches_library_sdpa)


def test_codebook_mistake_is_caught(patch):
    orig = T.lloyd_max_levels
    patch.setattr(T, "lloyd_max_levels", lambda b, **k: orig(b, max_iter=3))
    assert _fails(P.test_lloyd_max_matches_published_table, 4)
