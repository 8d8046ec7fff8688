"""ctypes loader for libfa_b200.so: argument and return types of every
``extern "C"`` entry point declared in include/fa.h.

There is no fallback: if the library is missing or fails to load, every call
raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfa_b200.so")
_LOCK = threading.Lock()
_LIB = None

c_void_p, c_int, c_float, c_size_t, c_uint = (ctypes.c_void_p, ctypes.c_int, ctypes.c_float,
                                              ctypes.c_size_t, ctypes.c_uint)
_P = c_void_p

SIGNATURES = {
    "fa_fwd": (c_int, [_P, _P, _P, _P, _P, c_int, c_int, c_int, c_int, c_float, c_int, _P]),
    "fa_bwd_workspace_size": (c_size_t, [c_int, c_int, c_int, c_int]),
    "fa_bwd": (c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, c_int, c_int, c_int, c_int, c_float,
                       c_int, _P, c_size_t, _P]),
    "fa_bwd_deterministic_workspace_size": (c_size_t, [c_int, c_int, c_int, c_int]),
    "fa_bwd_deterministic": (c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, c_int, c_int, c_int, c_int,
                                     c_float, c_int, _P, c_size_t, _P]),
    "fa_bwd_ex_workspace_size": (c_size_t, [c_int, c_int, c_int, c_int, c_int, c_int]),
    "fa_fwd_ex": (c_int, [_P, _P, _P, _P, _P, c_int, c_int, c_int, c_int, c_int, c_float, c_int, c_int,
                          _P, _P]),
    "fa_bwd_ex": (c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, c_int, c_int, c_int, c_int, c_int,
                          c_float, c_int, c_int, _P, c_int, _P, c_size_t, _P]),
    "fa_fwd_fp8_ex": (c_int, [_P, _P, _P, _P, _P, _P, _P, _P, c_int, c_int, c_int, c_int, c_int,
                              c_float, c_int, c_int, _P, _P]),
    "fa_bwd_noalloc": (c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, c_int, c_int, c_int, c_int,
                               c_float, c_int, _P]),
    "fa_quant_fp8": (c_int, [_P, _P, _P, c_int, c_int, c_int, c_int, _P, _P]),
    "fa_fwd_fp8": (c_int, [_P, _P, _P, _P, _P, _P, _P, _P, c_int, c_int, c_int, c_int, c_float,
                           c_int, _P]),
    "fa_selftest_wait_timeout": (c_int, [_P]),
    "fa_selftest_exp2": (c_int, [_P, _P, ctypes.c_longlong, c_int, _P]),
    "fa_set_tuning": (c_int, [c_int, c_int]),
    "fa_get_tuning": (c_int, [c_int, c_int]),
    "fa_get_status": (c_uint, []),
    "fa_clear_status": (None, []),
    "fa_status_string": (ctypes.c_char_p, [c_int]),
}

STATUS = {0: "FA_OK", 1: "FA_ERR_INVALID_ARG", 2: "FA_ERR_UNSUPPORTED", 3: "FA_ERR_MISALIGNED",
          4: "FA_ERR_WORKSPACE", 5: "FA_ERR_LAUNCH", 6: "FA_ERR_PIPELINE_TIMEOUT",
          7: "FA_ERR_NO_DEVICE", 8: "FA_ERR_SCRATCH_LIMIT"}


# fa_tune_knob values (include/fa.h)
(TUNE_FWD_POLY_PAIRS, TUNE_FWD_POLY_DEGREE, TUNE_BWD_POLY_GROUPS, TUNE_DQ_POLY_PAIRS, TUNE_FP8_POLY_PAIRS,
 TUNE_BWD_PAIR, TUNE_FWD_PERSISTENT, TUNE_FWD_CAUSAL_GROUP, TUNE_FWD_Q1, TUNE_BWD_CAUSAL_GROUP) = \
    1, 2, 3, 4, 5, 6, 8, 9, 10, 11


class FaError(RuntimeError):
    def __init__(self, fn: str, code: int):
        self.code = code
        super().__init__(f"{fn} returned {STATUS.get(code & 0xFF, code)} ({code})")


def library_path() -> str:
    return _PATH


def lib() -> ctypes.CDLL:
    """The loaded library (loaded once).  Raises if it has not been built."""
    global _LIB
    if _LIB is None:
        with _LOCK:
            if _LIB is None:
                if not os.path.exists(_PATH):
                    raise RuntimeError(
                        f"{_PATH} is missing: build it with `python -m exact_io_aware_42_b200.build`")
                h = ctypes.CDLL(_PATH)
                for name, (res, args) in SIGNATURES.items():
                    fn = getattr(h, name)
                    fn.restype = res
                    fn.argtypes = args
                _LIB = h
    return _LIB


def check(fn: str, code: int) -> None:
    if code != 0:
        raise FaError(fn, code)
