"""ctypes declarations of the C ABI in include/mac.h (libmac_b200.so)."""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmac_b200.so")

MAC_OK, MAC_ERR_ARG, MAC_ERR_SHAPE, MAC_ERR_CUDA, MAC_ERR_OOM, MAC_ERR_DEVICE = range(6)
MAC_DEV_BAD_SEQ_LEN, MAC_DEV_BAD_PAGE, MAC_DEV_TIMEOUT = 1, 2, 4

# Every symbol include/mac.h declares, with (restype, argtypes).
_P = C.c_void_p
SIGNATURES = {
    "mac_init_state": (C.c_int, [_P, C.POINTER(_P)]),
    "mac_destroy": (None, [_P]),
    "mac_reset_seq": (C.c_int, [_P, C.c_int, _P]),
    "mac_decode_step": (C.c_int, [_P] * 12),
    "mac_match": (C.c_int, [_P] * 10),
    "mac_attend": (C.c_int, [_P] * 7),
    "mac_append_kv": (C.c_int, [_P] * 8),
    "mac_decode_step_host": (C.c_int, [_P] * 14),
    "mac_get_status": (C.c_int, [_P, C.POINTER(C.c_int)]),
    "mac_state_bytes": (C.c_size_t, [_P]),
    "mac_export_state": (C.c_int, [_P, _P, C.c_size_t]),
    "mac_import_state": (C.c_int, [_P, _P, C.c_size_t]),
    "mac_set_min_keys_per_cta": (C.c_int, [_P, C.c_int]),
    "mac_set_piece_cost": (C.c_int, [_P, C.c_int]),
    "mac_set_whole_unit_keys": (C.c_int, [_P, C.c_int]),
    "mac_warm_start": (C.c_int, [_P, C.c_int, _P, _P, _P, _P, _P, _P, _P]),
    "mac_set_reproducible": (C.c_int, [_P, C.c_int]),
    "mac_set_one_launch": (C.c_int, [_P, C.c_int]),
    "mac_one_launch": (C.c_int, [_P]),
    "mac_set_trace": (C.c_int, [_P, C.c_int]),
    "mac_get_trace": (C.c_int, [_P, _P, C.c_size_t, _P]),
    "mac_attend_grid": (C.c_int, [_P]),
    "mac_error_string": (C.c_char_p, [C.c_int]),
    "mac_selftest_wait_timeout": (C.c_int, [_P, _P]),
    "mac_dense_decode_static": (C.c_int, [_P] * 9 + [C.c_int] * 4 + [C.c_double] + [C.c_int] * 4 + [_P]),
}


class MacConfig(C.Structure):
    _fields_ = [
        ("batch", C.c_int),
        ("num_q_heads", C.c_int),
        ("num_kv_heads", C.c_int),
        ("head_dim", C.c_int),
        ("window", C.c_int),
        ("band", C.c_int),
        ("tau", C.c_float),
        ("rope_theta", C.c_double),
        ("page_size", C.c_int),
        ("max_seq", C.c_int),
        ("max_pages_per_seq", C.c_int),
        ("num_pages", C.c_int),
        ("cut_mode", C.c_int),
        ("match_per_head", C.c_int),
        ("q_bf16", C.c_int),
        ("ring_bf16", C.c_int),
    ]


class MacError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__("%s failed: %s (code %d)" % (fn, msg, code))
        self.code = code


_lib = None


def load(path: str = LIB_PATH):
    """Load libmac_b200.so; raise if it is missing (there is no fallback path)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError("libmac_b200.so not built (python -m kv_cache_reuse_b200.build): %s" % path)
    lib = C.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def check(fn: str, rc: int) -> None:
    if rc != MAC_OK:
        raise MacError(fn, rc, load().mac_error_string(rc).decode())
