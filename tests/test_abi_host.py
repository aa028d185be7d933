"""The C ABI without a GPU: exports, context tables, host-side validation.

No call here reaches a kernel launch: every call either touches host memory
only (tq_create, tq_get_tables) or fails host validation first.
"""

import ctypes
import os
import re

import numpy as np
import pytest

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def K():
    import kv_cache_vector_turboquant_b200 as K

    return K


@pytest.fixture(scope="module")
def lib(K):
    return ctypes.CDLL(K.LIB_PATH)


def _declared_symbols():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            text = open(os.path.join(ROOT, "include", f)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(tq_[a-z0-9_]+)\s*\(", text))
    return names


def test_library_exports_every_declared_symbol(lib, K):
    """libtq.so exports every call of include/tq.h and no test hook; the hooks
    of include/tq_test.h come from libtq_test.so."""
    names = _declared_symbols()
    assert {"tq_create", "tq_encode", "tq_decode", "tq_encode_append", "tq_attend_decode"} <= names
    hooks = {n for n in names if n.startswith("tq_test_")}
    assert {"tq_test_encode_path", "tq_test_umma_block", "tq_test_reset_tensor_core_check"} <= hooks
    test_lib = K._binding._test_lib()
    for n in sorted(names - hooks):
        assert hasattr(lib, n), n
    for n in sorted(hooks):
        assert hasattr(test_lib, n), n
        assert not hasattr(lib, n), f"{n} is a test hook but libtq.so exports it"


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_tables_match_oracle(K, d, bits):
    ctx = K.tq_create(d, bits, 42)
    assert (ctx.head_dim, ctx.bits, ctx.seed, ctx.packed_bytes) == (d, bits, 42, d * bits // 8)
    lv, bd, sb = K.tq_get_tables(ctx)
    assert np.array_equal(lv, O.format_levels(bits).astype(np.float32))
    assert np.array_equal(bd, O.format_boundaries(O.format_levels(bits)).astype(np.float32))
    # the f32 tables are exact copies of the fp64 grid values
    assert np.array_equal(lv.astype(np.float64), O.format_levels(bits))
    s = O.sign_vector(42, d)
    assert np.array_equal(sb, np.packbits((s < 0).astype(np.uint8), bitorder="little"))


def test_seed_changes_signs_only(K):
    a, b = K.tq_create(128, 4, 42), K.tq_create(128, 4, 7)
    la, _, sa = K.tq_get_tables(a)
    lb, _, sb = K.tq_get_tables(b)
    assert np.array_equal(la, lb) and not np.array_equal(sa, sb)
    s = O.sign_vector(7, 128)
    assert np.array_equal(sb, np.packbits((s < 0).astype(np.uint8), bitorder="little"))


def test_create_rejects_unsupported(K):
    for d, b in [(32, 4), (96, 4), (512, 4), (128, 1), (128, 5), (0, 4)]:
        with pytest.raises(K.TQError) as e:
            K.tq_create(d, b)
        assert e.value.status == K.TQ_ERR_UNSUPPORTED
    vp = ctypes.c_void_p
    assert K._binding._lib.tq_create(128, 4, 42, None) == K.TQ_ERR_INVALID_ARG


def test_status_strings(K):
    for s in range(9):
        assert K.tq_status_string(s).startswith("TQ_")
    assert K.tq_status_string(99) == "TQ_ERR_UNKNOWN"


def test_null_context_queries(lib):
    for fn in ("tq_head_dim", "tq_bits", "tq_packed_bytes"):
        f = getattr(lib, fn)
        f.argtypes = [ctypes.c_void_p]
        assert f(None) == 0
    # the context form of the device-error query validates before any CUDA call
    f = lib.tq_check_device_error
    f.argtypes = [ctypes.c_void_p]
    assert f(None) == 1  # TQ_ERR_INVALID_ARG


class _FakePtr:
    """Stands in for a tensor: only its address is read by the binding."""

    def __init__(self, addr):
        self.addr = addr

    def data_ptr(self):
        return self.addr


def _raw(K, name, *args):
    lib = K._binding._test_lib() if name.startswith("tq_test_") else K._binding._lib
    return getattr(lib, name)(*args)


def test_encode_decode_validation(K):
    ctx = K.tq_create(128, 4)
    h = ctx.handle
    A, B_, C = 0x10000, 0x20000, 0x30000
    # null context, negative n
    assert _raw(K, "tq_encode", None, A, 4, B_, C, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, "tq_encode", h, A, -1, B_, C, None) == K.TQ_ERR_INVALID_ARG
    # n == 0 is a no-op, even with null pointers
    assert _raw(K, "tq_encode", h, None, 0, None, None, None) == K.TQ_OK
    assert _raw(K, "tq_decode", h, None, None, 0, None, None) == K.TQ_OK
    # null pointers
    assert _raw(K, "tq_encode", h, None, 4, B_, C, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, "tq_decode", h, A, None, 4, C, None) == K.TQ_ERR_INVALID_ARG
    # misaligned pointers
    assert _raw(K, "tq_encode", h, A + 8, 4, B_, C, None) == K.TQ_ERR_ALIGNMENT
    assert _raw(K, "tq_encode", h, A, 4, B_ + 4, C, None) == K.TQ_ERR_ALIGNMENT
    assert _raw(K, "tq_encode", h, A, 4, B_, C + 2, None) == K.TQ_ERR_ALIGNMENT
    assert _raw(K, "tq_decode", h, A + 1, C, 4, B_, None) == K.TQ_ERR_ALIGNMENT
    assert _raw(K, "tq_decode", h, A, C, 4, B_ + 8, None) == K.TQ_ERR_ALIGNMENT


def test_encode_path_hook_validation(K):
    """The test hook that picks the encode kernel validates before launching."""
    ctx = K.tq_create(128, 4)
    h = ctx.handle
    A, B_, C = 0x10000, 0x20000, 0x30000
    for bad_path in (0, 4, -1):
        assert _raw(K, "tq_test_encode_path", h, A, 4, B_, C, bad_path, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, "tq_test_encode_path", None, A, 4, B_, C, 2, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, "tq_test_encode_path", h, A, 0, B_, C, 2, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, "tq_test_encode_path", h, A + 8, 4, B_, C, 2, None) == K.TQ_ERR_ALIGNMENT
    assert _raw(K, "tq_test_encode_path", h, A, 4, B_ + 4, C, 2, None) == K.TQ_ERR_ALIGNMENT


def test_decode_path_hook_validation(K):
    ctx = K.tq_create(128, 4)
    h = ctx.handle
    A, B_, C = 0x10000, 0x20000, 0x30000
    for bad_path in (0, 5, -1):
        assert _raw(K, "tq_test_decode_path", h, A, C, 4, B_, bad_path, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, "tq_test_decode_path", None, A, C, 4, B_, 2, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, "tq_test_decode_path", h, A, C, 0, B_, 2, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, "tq_test_decode_path", h, A + 8, C, 4, B_, 2, None) == K.TQ_ERR_ALIGNMENT
    assert _raw(K, "tq_test_decode_path", h, A, C + 2, 4, B_, 2, None) == K.TQ_ERR_ALIGNMENT


def test_umma_block_hook_validation(K):
    A, B_, C = 0x10000, 0x20000, 0x30000
    assert _raw(K, "tq_test_umma_block", None, B_, C, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, "tq_test_umma_block", A, None, C, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, "tq_test_umma_block", A, B_, None, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, "tq_test_umma_block", A + 1, B_, C, None) == K.TQ_ERR_ALIGNMENT
    assert _raw(K, "tq_test_umma_block", A, B_, C + 2, None) == K.TQ_ERR_ALIGNMENT


def test_append_validation(K):
    ctx = K.tq_create(128, 3)
    h = ctx.handle
    A, B_, C, S = 0x10000, 0x20000, 0x30000, 0x40000
    assert _raw(K, "tq_encode_append", h, A, 4, 0, B_, C, 16, S, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, "tq_encode_append", h, A, 4, 8, B_, C, 0, S, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, "tq_encode_append", h, A, -1, 8, B_, C, 16, S, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, "tq_encode_append", h, A, 0, 8, B_, C, 16, S, None) == K.TQ_OK
    assert _raw(K, "tq_encode_append", h, A, 4, 8, B_, C, 16, None, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, "tq_encode_append", h, A, 4, 8, B_, C, 16, S + 2, None) == K.TQ_ERR_ALIGNMENT


def test_append_kv_validation(K):
    ctx = K.tq_create(128, 3)
    h = ctx.handle
    A, A2, B_, C, B2, C2, S = 0x10000, 0x18000, 0x20000, 0x30000, 0x50000, 0x60000, 0x40000
    f = "tq_encode_append_kv"
    assert _raw(K, f, None, A, A2, 4, 8, B_, C, B2, C2, 16, S, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, f, h, A, A2, 4, 0, B_, C, B2, C2, 16, S, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, f, h, A, A2, 4, 8, B_, C, B2, C2, 0, S, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, f, h, A, A2, -1, 8, B_, C, B2, C2, 16, S, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, f, h, A, A2, 0, 8, B_, C, B2, C2, 16, S, None) == K.TQ_OK  # nothing to do
    assert _raw(K, f, h, A, None, 4, 8, B_, C, B2, C2, 16, S, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, f, h, A, A2, 4, 8, B_, C, None, C2, 16, S, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, f, h, A, A2, 4, 8, B_, C, B2, None, 16, S, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, f, h, A, A2, 4, 8, B_, C, B2, C2, 16, None, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, f, h, A, A2 + 8, 4, 8, B_, C, B2, C2, 16, S, None) == K.TQ_ERR_ALIGNMENT
    assert _raw(K, f, h, A, A2, 4, 8, B_, C, B2 + 4, C2, 16, S, None) == K.TQ_ERR_ALIGNMENT
    assert _raw(K, f, h, A, A2, 4, 8, B_, C, B2, C2 + 2, 16, S, None) == K.TQ_ERR_ALIGNMENT
    assert _raw(K, f, h, A, A2, 4, 8, B_, C, B2, C2, 16, S + 2, None) == K.TQ_ERR_ALIGNMENT


def test_attend_validation_and_workspace(K):
    k4, v2 = K.tq_create(128, 4), K.tq_create(128, 2)
    k64 = K.tq_create(64, 4)
    ws = K.tq_attend_workspace_bytes(16, 32, 128, 32768)
    assert ws > 0 and ws % 4 == 0
    # the workspace holds (max, sum, d accumulators) per (sequence, head, split)
    assert ws >= 16 * 32 * (128 + 2) * 4
    assert K.tq_attend_workspace_bytes(0, 32, 128, 10) == 0
    assert K.tq_attend_workspace_bytes(2, 8, 96, 10) == 0
    A = 0x100000
    args = lambda kc, vc, B, hq, hkv, s_max, ws_ptr, ws_b: (  # noqa: E731
        kc.handle, vc.handle, A, B, hq, hkv, A, A, A, A, s_max, A, A, ws_ptr, ws_b, None)
    need = K.tq_attend_workspace_bytes(2, 8, 128, 100)
    assert _raw(K, "tq_attend_decode", *args(k4, v2, 2, 8, 3, 100, A, need)) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, "tq_attend_decode", *args(k4, k64, 2, 8, 2, 100, A, need)) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, "tq_attend_decode", *args(k4, v2, 2, 8, 2, 0, A, need)) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, "tq_attend_decode", *args(k4, v2, 2, 8, 2, 100, A, need - 4)) == K.TQ_ERR_WORKSPACE
    assert _raw(K, "tq_attend_decode", *args(k4, v2, 2, 8, 2, 100, None, need)) == K.TQ_ERR_WORKSPACE
    assert _raw(K, "tq_attend_decode", *args(k4, v2, 2, 8, 2, 100, A + 4, need)) == K.TQ_ERR_ALIGNMENT
    assert _raw(K, "tq_attend_decode", *args(k4, v2, 0, 8, 2, 100, A, need)) == K.TQ_OK


def test_compression_ratio_matches_formula(K):
    for b, want in ((2, 256 / 36), (3, 256 / 52), (4, 256 / 68)):
        assert abs(K.TurboQuant(128, b).compression_ratio() - want) < 1e-12


def test_attend_paged_validation(K):
    """tq_attend_decode_paged: sizes, null pointers, workspace and alignment
    are checked on the host before anything is enqueued."""
    k4, v2 = K.tq_create(128, 4), K.tq_create(128, 2)
    k64 = K.tq_create(64, 4)
    A = 0x100000
    fn = "tq_attend_decode_paged"

    def args(kc=k4, vc=v2, B=2, hq=8, hkv=2, nblk=40, bt=A, maxb=8, lens=A, ws_ptr=A, ws_b=None):
        if ws_b is None:
            ws_b = K.tq_attend_workspace_bytes(B if B > 0 else 1, hq, 128, maxb * K.TQ_PAGE_BLOCK)
        return (kc.handle, vc.handle, A, B, hq, hkv, A, A, A, A, nblk, bt, maxb, lens, A, ws_ptr, ws_b, None)

    need = K.tq_attend_workspace_bytes(2, 8, 128, 8 * 16)
    assert _raw(K, fn, *args(hkv=3)) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, fn, *args(vc=k64)) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, fn, *args(nblk=0)) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, fn, *args(maxb=0)) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, fn, *args(bt=None)) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, fn, *args(lens=None)) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, fn, *args(bt=A + 2)) == K.TQ_ERR_ALIGNMENT
    assert _raw(K, fn, *args(ws_b=need - 4)) == K.TQ_ERR_WORKSPACE
    assert _raw(K, fn, *args(ws_ptr=None)) == K.TQ_ERR_WORKSPACE
    assert _raw(K, fn, *args(ws_ptr=A + 4)) == K.TQ_ERR_ALIGNMENT
    assert _raw(K, fn, *args(nblk=(1 << 26) + 1)) == K.TQ_ERR_UNSUPPORTED
    assert _raw(K, fn, *args(B=0)) == K.TQ_OK


def test_encode_slots_validation(K):
    ctx = K.tq_create(128, 4)
    h = ctx.handle
    A = 0x100000
    fn = "tq_encode_slots"
    assert _raw(K, fn, None, A, 4, 8, A, A, 64, A, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, fn, h, A, -1, 8, A, A, 64, A, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, fn, h, A, 4, 0, A, A, 64, A, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, fn, h, A, 4, 8, A, A, 0, A, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, fn, h, A, 4, 8, A, A, 64, None, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, fn, h, A + 8, 4, 8, A, A, 64, A, None) == K.TQ_ERR_ALIGNMENT
    assert _raw(K, fn, h, A, 4, 8, A, A + 2, 64, A, None) == K.TQ_ERR_ALIGNMENT
    assert _raw(K, fn, h, A, 0, 8, A, A, 64, A, None) == K.TQ_OK


def test_offset_variant_validation(K):
    ctx = K.tq_create(128, 4)
    h = ctx.handle
    A = 0x100000
    # tq_encode_os(ctx, x, n, packed, side, stream); tq_decode_os(ctx, packed, side, n, x, stream)
    assert _raw(K, "tq_encode_os", None, A, 4, A, A, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, "tq_encode_os", h, A, -1, A, A, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, "tq_encode_os", h, A, 0, A, A, None) == K.TQ_OK
    assert _raw(K, "tq_decode_os", None, A, A, 4, A, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, "tq_decode_os", h, A, A, -1, A, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, "tq_decode_os", h, A, A, 0, A, None) == K.TQ_OK
    assert _raw(K, "tq_encode_os", h, A, 4, A, None, None) == K.TQ_ERR_INVALID_ARG
    assert _raw(K, "tq_encode_os", h, A + 2, 4, A, A, None) == K.TQ_ERR_ALIGNMENT
    assert _raw(K, "tq_encode_os", h, A, 4, A, A + 2, None) == K.TQ_ERR_ALIGNMENT
    assert _raw(K, "tq_decode_os", h, A, A + 1, 4, A, None) == K.TQ_ERR_ALIGNMENT


@pytest.mark.parametrize("d,bits", [(64, 2), (128, 4), (256, 3)])
def test_memory_report_arithmetic(K, d, bits):
    """TurboQuant.memory_report: K and V of seq_len tokens x layers x kv
    heads, fp16 (2 d bytes per vector) against packed codes + f32 norm."""
    tq = K.TurboQuant(d, bits)
    r = tq.memory_report(4096, num_layers=32, num_kv_heads=8)
    vectors = 2 * 32 * 8 * 4096
    assert r["vectors"] == vectors
    assert r["fp16_bytes"] == vectors * 2 * d
    assert r["packed_bytes"] == vectors * (d * bits // 8 + 4)
    assert r["compression_ratio"] == pytest.approx(tq.compression_ratio())
