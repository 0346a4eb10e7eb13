"""ctypes declarations of libtern.so's C ABI (include/tern.h). Argument marshalling only."""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
# TERN_LIBRARY=debug selects the TERN_DEBUG build (device-side bounds checks; build with --debug)
LIB_PATH = os.path.join(_HERE, "libtern_debug.so" if os.environ.get("TERN_LIBRARY") == "debug" else "libtern.so")

TERN_OK = 0
STATUS_NAMES = {
    0: "TERN_OK", 1: "TERN_ERR_NULL", 2: "TERN_ERR_SHAPE", 3: "TERN_ERR_ALIGN", 4: "TERN_ERR_BAD_TRIT",
    5: "TERN_ERR_BAD_CODE", 6: "TERN_ERR_RESIDUAL", 7: "TERN_ERR_WORKSPACE", 8: "TERN_ERR_CUDA",
    9: "TERN_ERR_TIMEOUT", 10: "TERN_ERR_ELEM", 11: "TERN_ERR_BOUNDS",
}
STATUS = {v: k for k, v in STATUS_NAMES.items()}

# every function the header declares, with (restype, argtypes)
_c = ctypes
EXPORTS = {
    "tern_pack_exec": (_c.c_int, [_c.c_void_p, _c.c_int64, _c.c_int64, _c.c_void_p, _c.c_void_p]),
    "tern_unpack_exec": (_c.c_int, [_c.c_void_p, _c.c_int64, _c.c_int64, _c.c_void_p, _c.c_void_p]),
    "tern_pack_store": (_c.c_int, [_c.c_void_p, _c.c_int64, _c.c_int64, _c.c_void_p, _c.c_void_p]),
    "tern_unpack_store": (_c.c_int, [_c.c_void_p, _c.c_int64, _c.c_int64, _c.c_void_p, _c.c_void_p]),
    "tern_weight_validate": (_c.c_int, [_c.c_void_p, _c.c_void_p]),
    "tern_decode_ranges": (_c.c_int, [_c.c_void_p, _c.c_int32, _c.c_int64, _c.c_void_p, _c.c_int32, _c.c_void_p,
                                     _c.c_void_p, _c.c_void_p]),
    "tern_residual_strip_counts": (_c.c_int, [_c.c_void_p, _c.c_int64, _c.c_int64, _c.c_void_p]),
    "tern_linear_workspace_bytes": (_c.c_size_t, [_c.c_void_p, _c.c_int64]),
    "tern_linear": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_int64, _c.c_void_p, _c.c_void_p, _c.c_size_t,
                               _c.c_void_p]),
    "tern_linear_with_prefetch": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_int64, _c.c_void_p, _c.c_void_p,
                                             _c.c_size_t, _c.c_void_p, _c.c_void_p]),
    "tern_linear_group": (_c.c_int, [_c.c_void_p, _c.c_int32, _c.c_void_p, _c.c_int64, _c.c_void_p, _c.c_void_p,
                                     _c.c_size_t, _c.c_void_p, _c.c_int32, _c.c_void_p]),
    "tern_fit": (_c.c_int, [_c.c_void_p, _c.c_int64, _c.c_int64, _c.c_void_p, _c.c_int64, _c.c_int32, _c.c_int32,
                            _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_void_p]),
    "tern_rotate": (_c.c_int, [_c.c_void_p, _c.c_int64, _c.c_int64, _c.c_void_p, _c.c_void_p, _c.c_void_p]),
    "tern_bits": (_c.c_int, [_c.c_int64, _c.c_int64, _c.c_int64, _c.c_int32, _c.c_void_p]),
    "tern_bits_offset": (_c.c_int, [_c.c_int64, _c.c_int64, _c.c_int64, _c.c_int32, _c.c_void_p]),
    "tern_bits_elem": (_c.c_int, [_c.c_int64, _c.c_int64, _c.c_int64, _c.c_int64, _c.c_int32, _c.c_int32,
                                  _c.c_void_p]),
    "tern_pack_elem": (_c.c_int, [_c.c_void_p, _c.c_int64, _c.c_int64, _c.c_void_p, _c.c_void_p, _c.c_void_p,
                                  _c.c_int64, _c.c_void_p, _c.c_void_p]),
    "tern_unpack_elem": (_c.c_int, [_c.c_void_p, _c.c_void_p, _c.c_void_p, _c.c_int64, _c.c_int64, _c.c_int64,
                                    _c.c_void_p, _c.c_void_p]),
    "tern_pack_residual": (_c.c_int, [_c.c_void_p, _c.c_int64, _c.c_int64, _c.c_void_p, _c.c_void_p, _c.c_void_p]),
    "tern_unpack_residual": (_c.c_int, [_c.c_void_p, _c.c_int64, _c.c_void_p, _c.c_int64, _c.c_void_p, _c.c_void_p,
                                        _c.c_void_p]),
    "tern_device_status": (_c.c_int, [_c.c_void_p]),
    "tern_selftest_timeout": (_c.c_int, [_c.c_int64, _c.c_void_p]),
    "tern_debug_build": (_c.c_int, []),
    "tern_status_string": (_c.c_char_p, [_c.c_int]),
    "tern_version": (_c.c_int, []),
}


class TernWeightC(ctypes.Structure):
    """struct tern_weight."""
    _fields_ = [
        ("N", ctypes.c_int64), ("K", ctypes.c_int64), ("group", ctypes.c_int32),
        ("plane1", ctypes.c_void_p), ("scale1", ctypes.c_void_p),
        ("r", ctypes.c_int64), ("res_rows", ctypes.c_void_p), ("res_slot", ctypes.c_void_p),
        ("plane2", ctypes.c_void_p), ("scale2", ctypes.c_void_p), ("flags", ctypes.c_uint32),
        ("mu", ctypes.c_void_p),
        ("ecount", ctypes.c_void_p), ("ebase", ctypes.c_void_p), ("eidx", ctypes.c_void_p),
        ("escale", ctypes.c_void_p), ("nnz2", ctypes.c_int64),
        ("res_per_strip", ctypes.c_void_p),
    ]


WEIGHT_STATIC = 1


class TernBitsReport(ctypes.Structure):
    """struct tern_bits_report."""
    _fields_ = [
        ("weights", ctypes.c_uint64), ("plane_trits", ctypes.c_uint64), ("store_bits", ctypes.c_uint64),
        ("exec_bits", ctypes.c_uint64), ("bpw_info", ctypes.c_double), ("bpw_store", ctypes.c_double),
        ("bpw_exec", ctypes.c_double),
    ]


_lib = None


def load() -> ctypes.CDLL:
    """The loaded libtern.so. Raises if it has not been built: there is no fallback path."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m ternary_weight_only_tern_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in EXPORTS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


class TernError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        self.name = STATUS_NAMES.get(status, str(status))
        msg = load().tern_status_string(status).decode()
        super().__init__(f"{fn}: {self.name} ({msg})")


def check(fn: str, status: int) -> None:
    if status != TERN_OK:
        raise TernError(fn, status)
