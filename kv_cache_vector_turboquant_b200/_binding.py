"""ctypes binding of libtq (include/tq.h): argument marshalling only.

Every function here converts torch tensors to device pointers and the current
CUDA stream to a handle, calls the C entry point of the same name and turns a
non-zero status into :class:`TQError`. All computation happens in the CUDA
kernels of ``libtq.so``; there is no fallback path. Importing this module
raises ``ImportError`` if the library has not been built
(``python kv_cache_vector_turboquant_b200/build.py``).
"""

from __future__ import annotations

import ctypes
import os

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtq.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(
        f"libtq.so not found at {_LIB_PATH}; build it with "
        "`python kv_cache_vector_turboquant_b200/build.py`"
    )
_lib = ctypes.CDLL(_LIB_PATH)

_c_int, _c_i64, _c_u64, _c_size, _vp = ctypes.c_int, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t, ctypes.c_void_p

_PROTOS = {
    "tq_status_string": (ctypes.c_char_p, [_c_int]),
    "tq_create": (_c_int, [_c_int, _c_int, _c_u64, ctypes.POINTER(_vp)]),
    "tq_destroy": (None, [_vp]),
    "tq_head_dim": (_c_int, [_vp]),
    "tq_bits": (_c_int, [_vp]),
    "tq_seed": (_c_u64, [_vp]),
    "tq_packed_bytes": (_c_size, [_vp]),
    "tq_get_tables": (_c_int, [_vp, _vp, _vp, _vp]),
    "tq_encode": (_c_int, [_vp, _vp, _c_i64, _vp, _vp, _vp]),
    "tq_decode": (_c_int, [_vp, _vp, _vp, _c_i64, _vp, _vp]),
    "tq_encode_append": (_c_int, [_vp, _vp, _c_int, _c_int, _vp, _vp, _c_i64, _vp, _vp]),
    "tq_encode_slots": (_c_int, [_vp, _vp, _c_i64, _c_int, _vp, _vp, _c_i64, _vp, _vp]),
    "tq_encode_append_kv": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _vp, _vp, _vp, _vp, _c_i64, _vp, _vp]),
    "tq_encode_os": (_c_int, [_vp, _vp, _c_i64, _vp, _vp, _vp]),
    "tq_decode_os": (_c_int, [_vp, _vp, _vp, _c_i64, _vp, _vp]),
    "tq_attend_workspace_bytes": (_c_size, [_c_int, _c_int, _c_int, _c_i64]),
    "tq_attend_decode": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _c_i64,
                                  _vp, _vp, _vp, _c_size, _vp]),
    "tq_attend_decode_static": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _c_i64,
                                         _vp, _vp, _vp]),
    "tq_attend_decode_paged": (_c_int, [_vp, _vp, _vp, _c_int, _c_int, _c_int, _vp, _vp, _vp, _vp, _c_i64, _vp,
                                        _c_int, _vp, _vp, _vp, _c_size, _vp]),
    "tq_device_error": (_c_int, [_vp, ctypes.POINTER(ctypes.c_uint32)]),
    "tq_check_device_error": (_c_int, [_vp]),
    "tq_tensor_core_check": (_c_int, [ctypes.POINTER(_c_int)]),
}
for _name, (_res, _args) in _PROTOS.items():
    _f = getattr(_lib, _name)
    _f.restype = _res
    _f.argtypes = _args

# Test hooks (include/tq_test.h) live in libtq_test.so, which is linked
# against libtq.so (the same loaded instance: same device error word) and is
# loaded only when a hook is first called.
_TEST_LIB_PATH = os.path.join(os.path.dirname(_LIB_PATH), "libtq_test.so")
_TEST_PROTOS = {
    "tq_test_reset_tensor_core_check": (_c_int, [_c_int]),
    "tq_test_encode_stalled": (_c_int, [_vp, _vp, _c_i64, _vp, _vp, _vp]),
    "tq_test_encode_path": (_c_int, [_vp, _vp, _c_i64, _vp, _vp, _c_int, _vp]),
    "tq_test_umma_block": (_c_int, [_vp, _vp, _vp, _vp]),
    "tq_test_decode_path": (_c_int, [_vp, _vp, _vp, _c_i64, _vp, _c_int, _vp]),
    "tq_test_attend_plan": (_c_int, [_c_int, _c_int, _c_int, _c_int, _c_int, _c_int, _vp]),
}
_test = None


def _test_lib():
    """libtq_test.so with its prototypes set (loaded on first use)."""
    global _test
    if _test is None:
        if not os.path.exists(_TEST_LIB_PATH):
            raise ImportError(f"libtq_test.so not found at {_TEST_LIB_PATH}; build it with "
                              "`python kv_cache_vector_turboquant_b200/build.py`")
        lib = ctypes.CDLL(_TEST_LIB_PATH)
        for name, (res, args) in _TEST_PROTOS.items():
            f = getattr(lib, name)
            f.restype = res
            f.argtypes = args
        _test = lib
    return _test

TQ_OK = 0
TQ_ERR_INVALID_ARG = 1
TQ_ERR_UNSUPPORTED = 2
TQ_ERR_ALIGNMENT = 3
TQ_ERR_WORKSPACE = 4
TQ_ERR_CUDA = 5
TQ_ERR_TIMEOUT = 6
TQ_ERR_NOMEM = 7
TQ_ERR_DEVICE = 8
TQ_DEVERR_TIMEOUT = 0x1
TQ_DEVERR_SLOT_RANGE = 0x2
TQ_DEVERR_POS_RANGE = 0x4
TQ_DEVERR_SMEM_LAYOUT = 0x8
TQ_DEVERR_BLOCK_RANGE = 0x10
TQ_PAGE_BLOCK = 16

LIB_PATH = _LIB_PATH


class TQError(RuntimeError):
    """A libtq call returned a non-zero status."""

    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {tq_status_string(status)}")


def tq_status_string(status: int) -> str:
    return _lib.tq_status_string(int(status)).decode()


def _check(status: int, what: str) -> None:
    if status != TQ_OK:
        raise TQError(status, what)


def _ptr(t) -> int | None:
    """Device (or host) address of a tensor, None for None."""
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream) -> int | None:
    import torch

    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


class Ctx:
    """Owns a ``tq_ctx*`` (host object); freed with the Python object."""

    def __init__(self, handle: int):
        self._h = ctypes.c_void_p(handle)

    @property
    def handle(self) -> ctypes.c_void_p:
        return self._h

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and h.value:
            _lib.tq_destroy(h)
            self._h = ctypes.c_void_p(0)

    @property
    def head_dim(self) -> int:
        return _lib.tq_head_dim(self._h)

    @property
    def bits(self) -> int:
        return _lib.tq_bits(self._h)

    @property
    def seed(self) -> int:
        return _lib.tq_seed(self._h)

    @property
    def packed_bytes(self) -> int:
        return _lib.tq_packed_bytes(self._h)


def tq_create(head_dim: int, bits: int, seed: int = 42) -> Ctx:
    out = ctypes.c_void_p(0)
    _check(_lib.tq_create(int(head_dim), int(bits), ctypes.c_uint64(seed & (2**64 - 1)), ctypes.byref(out)),
           "tq_create")
    return Ctx(out.value)


def tq_get_tables(ctx: Ctx):
    """(levels [2^b] f32, boundaries [2^b-1] f32, sign_bits [d/8] u8) as numpy arrays."""
    import numpy as np

    L = 1 << ctx.bits
    levels = np.zeros(L, dtype=np.float32)
    bounds = np.zeros(L - 1, dtype=np.float32)
    signs = np.zeros(ctx.head_dim // 8, dtype=np.uint8)
    _check(_lib.tq_get_tables(ctx.handle, levels.ctypes.data, bounds.ctypes.data, signs.ctypes.data),
           "tq_get_tables")
    return levels, bounds, signs


def tq_encode(ctx: Ctx, x, n: int, packed, norms, stream=None) -> None:
    _check(_lib.tq_encode(ctx.handle, _ptr(x), int(n), _ptr(packed), _ptr(norms), _stream(stream)), "tq_encode")


def tq_decode(ctx: Ctx, packed, norms, n: int, x, stream=None) -> None:
    _check(_lib.tq_decode(ctx.handle, _ptr(packed), _ptr(norms), int(n), _ptr(x), _stream(stream)), "tq_decode")


def tq_encode_append(ctx: Ctx, x, n_seq: int, h: int, cache_packed, cache_norms, s_max: int, slot,
                     stream=None) -> None:
    _check(_lib.tq_encode_append(ctx.handle, _ptr(x), int(n_seq), int(h), _ptr(cache_packed), _ptr(cache_norms),
                                 int(s_max), _ptr(slot), _stream(stream)), "tq_encode_append")


def tq_encode_append_kv(ctx: Ctx, k, v, n_seq: int, h: int, k_cache, k_norms, v_cache, v_norms, s_max: int, slot,
                        stream=None) -> None:
    _check(_lib.tq_encode_append_kv(ctx.handle, _ptr(k), _ptr(v), int(n_seq), int(h), _ptr(k_cache), _ptr(k_norms),
                                    _ptr(v_cache), _ptr(v_norms), int(s_max), _ptr(slot), _stream(stream)),
           "tq_encode_append_kv")


def tq_encode_os(ctx: Ctx, x, n: int, packed, side, stream=None) -> None:
    _check(_lib.tq_encode_os(ctx.handle, _ptr(x), int(n), _ptr(packed), _ptr(side), _stream(stream)), "tq_encode_os")


def tq_decode_os(ctx: Ctx, packed, side, n: int, x, stream=None) -> None:
    _check(_lib.tq_decode_os(ctx.handle, _ptr(packed), _ptr(side), int(n), _ptr(x), _stream(stream)), "tq_decode_os")


def tq_encode_slots(ctx: Ctx, x, n_tok: int, h: int, cache_packed, cache_norms, num_slots: int, slot_mapping,
                    stream=None) -> None:
    _check(_lib.tq_encode_slots(ctx.handle, _ptr(x), int(n_tok), int(h), _ptr(cache_packed), _ptr(cache_norms),
                                int(num_slots), _ptr(slot_mapping), _stream(stream)), "tq_encode_slots")


def tq_attend_workspace_bytes(B: int, hq: int, head_dim: int, s_max: int) -> int:
    return int(_lib.tq_attend_workspace_bytes(int(B), int(hq), int(head_dim), int(s_max)))


def tq_attend_decode(k: Ctx, v: Ctx, q, B: int, hq: int, hkv: int, k_packed, k_norms, v_packed, v_norms,
                     s_max: int, positions, out, workspace, ws_bytes: int, stream=None) -> None:
    _check(_lib.tq_attend_decode(k.handle, v.handle, _ptr(q), int(B), int(hq), int(hkv), _ptr(k_packed),
                                 _ptr(k_norms), _ptr(v_packed), _ptr(v_norms), int(s_max), _ptr(positions),
                                 _ptr(out), _ptr(workspace), int(ws_bytes), _stream(stream)), "tq_attend_decode")


def tq_attend_decode_paged(k: Ctx, v: Ctx, q, B: int, hq: int, hkv: int, k_cache, k_norms, v_cache, v_norms,
                           num_blocks: int, block_tables, max_blocks: int, context_lens, out, workspace,
                           ws_bytes: int, stream=None) -> None:
    _check(_lib.tq_attend_decode_paged(k.handle, v.handle, _ptr(q), int(B), int(hq), int(hkv), _ptr(k_cache),
                                       _ptr(k_norms), _ptr(v_cache), _ptr(v_norms), int(num_blocks),
                                       _ptr(block_tables), int(max_blocks), _ptr(context_lens), _ptr(out),
                                       _ptr(workspace), int(ws_bytes), _stream(stream)), "tq_attend_decode_paged")


def tq_attend_decode_static(k: Ctx, v: Ctx, q, B: int, hq: int, hkv: int, k_packed, k_norms, v_packed, v_norms,
                            s_max: int, positions, out, stream=None) -> None:
    """tq_attend_decode without a workspace argument: the library's own fixed
    device scratch is used, so the call allocates nothing."""
    _check(_lib.tq_attend_decode_static(k.handle, v.handle, _ptr(q), int(B), int(hq), int(hkv), _ptr(k_packed),
                                        _ptr(k_norms), _ptr(v_packed), _ptr(v_norms), int(s_max), _ptr(positions),
                                        _ptr(out), _stream(stream)), "tq_attend_decode_static")


TQ_ATTEND_STATIC_SCRATCH_BYTES = 8 << 20


def tq_device_error(stream=None) -> tuple[int, int]:
    """(status, error bits) of the current device; reads and clears the word."""
    bits = ctypes.c_uint32(0)
    st = _lib.tq_device_error(_stream(stream), ctypes.byref(bits))
    return st, bits.value


def tq_check_device_error(ctx) -> int:
    """Status of the current device's error word (read and cleared) for a
    caller that holds a context and has synchronised its streams."""
    return int(_lib.tq_check_device_error(ctx.handle if ctx is not None else None))


def tq_tensor_core_check() -> bool:
    """Run (once per device) the check of the tensor-core rounding that the
    bulk encode and decode kernels rely on; True if it passed."""
    passed = _c_int(0)
    _check(_lib.tq_tensor_core_check(ctypes.byref(passed)), "tq_tensor_core_check")
    return bool(passed.value)


def tq_test_attend_plan(d: int, hw: int, nt: int, paged: bool, reserved: int, max_dyn: int):
    """(status, plan) of the fast attention kernel's shared memory (host
    arithmetic); plan is a dict of the stage count, groups, regions and the
    per-stage buffer offsets."""
    out = (ctypes.c_int32 * 40)()
    st = _test_lib().tq_test_attend_plan(int(d), int(hw), int(nt), int(bool(paged)), int(reserved), int(max_dyn),
                                         ctypes.cast(out, _vp))
    v = list(out)
    plan = {"stages": v[0], "groups": v[1], "table_off": v[2], "table_bytes": v[3], "header_bytes": v[4],
            "k_bytes": v[5], "v_bytes": v[6], "norm_bytes": v[7],
            "k": v[8:16], "v": v[16:24], "kn": v[24:32], "vn": v[32:40]}
    return st, plan


def tq_test_reset_tensor_core_check(force_fail: bool = False) -> int:
    """Test hook: forget the current device's check result (force the next
    check to report a mismatch if `force_fail`); returns the status."""
    return _test_lib().tq_test_reset_tensor_core_check(int(bool(force_fail)))


def tq_test_encode_stalled(ctx: Ctx, x, n: int, packed, norms, stream=None) -> int:
    """Test hook: encode with the row copies withheld; returns the launch status."""
    return _test_lib().tq_test_encode_stalled(ctx.handle, _ptr(x), int(n), _ptr(packed), _ptr(norms), _stream(stream))


def tq_test_decode_path(ctx: Ctx, packed, norms, n: int, x, path: int, stream=None) -> int:
    """Test hook: decode through kernel `path` (1 CUDA cores, 2 tensor cores; 3 and 4 the same for the
    offset variant, `norms` then holding its int32 side words); returns the launch status."""
    return _test_lib().tq_test_decode_path(ctx.handle, _ptr(packed), _ptr(norms), int(n), _ptr(x), int(path), _stream(stream))


def tq_test_umma_block(a, b, d, stream=None) -> int:
    """Test hook: one tcgen05 MMA d[128,16] = a[128,16] @ b[16,16]^T (fp16 in, f32 out)."""
    return _test_lib().tq_test_umma_block(_ptr(a), _ptr(b), _ptr(d), _stream(stream))


def tq_test_encode_path(ctx: Ctx, x, n: int, packed, norms, path: int, stream=None) -> int:
    """Test hook: encode through kernel `path` (1 CUDA cores, 2 tensor cores, 3 tensor
    cores with the row copies withheld); returns the launch status."""
    return _test_lib().tq_test_encode_path(ctx.handle, _ptr(x), int(n), _ptr(packed), _ptr(norms), int(path),
                                    _stream(stream))
