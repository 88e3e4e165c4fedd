"""ctypes binding of ``libh2o.so`` (declared in ``include/h2o.h``).

Argument marshalling only: every step of the H2O path runs in the library's
CUDA kernels. The functions keep the C names; ``H2OCache`` wraps a context
for use with torch tensors (device memory and streams come from torch).
Loading fails loudly if the library has not been built.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libh2o.so")

H2O_OK = 0
H2O_ERR_ARG = -1
H2O_ERR_ALIGN = -2
H2O_ERR_OOM = -3
H2O_ERR_CUDA = -4
H2O_ERR_TIMEOUT = -5
H2O_ERR_POISONED = -6
H2O_ERR_UNSUPPORTED = -7
H2O_POLICY_SUM = 0
H2O_POLICY_NORMALIZED = 1
H2O_POLICY_INSERT_ALWAYS = 2
H2O_BF16 = 0
H2O_FP32 = 1

STATUS_NAMES = {0: "H2O_OK", -1: "H2O_ERR_ARG", -2: "H2O_ERR_ALIGN", -3: "H2O_ERR_OOM",
                -4: "H2O_ERR_CUDA", -5: "H2O_ERR_TIMEOUT", -6: "H2O_ERR_POISONED",
                -7: "H2O_ERR_UNSUPPORTED"}

# (name, restype, argtypes) of every exported entry point.
_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
SIGNATURES = [
    ("h2o_create", _I, [_I, _I, _I, _I, _I, ctypes.POINTER(_P)]),
    ("h2o_create_ex", _I, [_I, _I, _I, _I, _I, _I, _I, ctypes.POINTER(_P)]),
    ("h2o_destroy", _I, [_P]),
    ("h2o_step", _I, [_P, _P, _P, _P, _P, _I, _P]),
    ("h2o_prefill", _I, [_P, _P, _P, _P, _P, _I, _I, _P]),
    ("h2o_step_host", _I, [_P, _P, _P, _P, _P, _I, _P]),
    ("h2o_backward", _I, [_P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P, _P]),
    ("h2o_step_host_async", _I, [_P, _P, _P, _P, _P, _I, _P]),
    ("h2o_host_sync", _I, [_P]),
    ("h2o_set_policy", _I, [_P, _I]),
    ("h2o_scores", _I, [_P, _P, _P]),
    ("h2o_positions", _I, [_P, _P, _P]),
    ("h2o_counters", _I, [_P, ctypes.POINTER(_I64), ctypes.POINTER(_I64)]),
    ("h2o_last_error", ctypes.c_char_p, [_P]),
    ("h2o_candidates", _I, [_P, _P, _P, _P, _P]),
    ("h2o_token_slots", _I, [_P, _P, _P]),
    ("h2o_lse", _I, [_P, _P, _P]),
    ("h2o_last_step_info", _I, [_P, ctypes.POINTER(_I), ctypes.POINTER(_I)]),
    ("h2o_get_state", _I, [_P, _P, _P, _P, _P, ctypes.POINTER(_I64), ctypes.POINTER(_I64), _P]),
    ("h2o_set_state", _I, [_P, _P, _P, _P, _P, _I64, _I64, _P]),
    ("h2o_reset", _I, [_P, _P]),
    ("h2o_sync_check", _I, [_P, _P]),
    ("h2o_selftest_wait", _I, [_P, _I, _P]),
    ("h2o_selftest_exp2", _I, [_P, _P, _P, _P, _I, _P]),
    ("h2o_version", ctypes.c_char_p, []),
    ("h2o_kernel_plan", _I, [_P, _I, ctypes.POINTER(ctypes.c_char_p), _I]),
    ("h2o_select_noalloc", _I, [_I, _I, _I, _I, _I64, _P, _P, _P, _P, _P, _P, _P]),
    ("h2o_profile_begin", _I, [_P, _I]),
    ("h2o_profile_end", _I, [_P, _I, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_double),
                             ctypes.POINTER(_I)]),
]

_lib = None


class H2OError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m h2o_kv_cache_step_b200.build` (no fallback exists)")
        L = ctypes.CDLL(LIB_PATH)
        for name, res, args in SIGNATURES:
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def check(rc: int, ctx=None) -> None:
    if rc != H2O_OK:
        msg = lib().h2o_last_error(ctx)
        raise H2OError(rc, msg.decode() if msg else "")
