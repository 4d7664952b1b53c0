"""ctypes declarations of libthdcp's C ABI (include/thdcp.h).  Marshalling only."""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libthdcp.so")

THD_OK = 0
THD_DTYPE_BF16 = 0
THD_DTYPE_FP32 = 1
NOALLOC_MAX_ROWS_X_HEADS = 8388608
QT_FIELDS = 12
KSEG = 32
EN_FIELDS = 8

ERRORS = {
    -1: "INVALID_ARG", -2: "BAD_SEQLENS", -3: "NOT_DIVISIBLE", -4: "MISALIGNED",
    -5: "NOT_UPLOADED", -6: "CUDA", -7: "UNSUPPORTED", -8: "ALLOC", -9: "TOO_LARGE",
}

# Every entry point of include/thdcp.h: name -> (restype, argtypes)
_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_PI32 = ctypes.POINTER(ctypes.c_int32)
_F = ctypes.c_float
SIGNATURES = {
    "thd_cp_plan": (ctypes.c_int, [_PI32, _I32, _I32, ctypes.POINTER(_P)]),
    "thd_cp_plan_info": (ctypes.c_int, [_P, _P]),
    "thd_cp_plan_export": (ctypes.c_int, [_P, _PI32, _PI32, _PI32, _PI32, _PI32, _PI32, _PI32, _PI32, _PI32]),
    "thd_cp_plan_export_fwd": (ctypes.c_int, [_P, _PI32, _PI32, _PI32, _PI32, _PI32, _PI32, _PI32]),
    "thd_cp_plan_upload": (ctypes.c_int, [_P, _P]),
    "thd_cp_plan_update": (ctypes.c_int, [_P, _PI32, _I32, _I32, _P]),
    "thd_cp_plan_destroy": (None, [_P]),
    "thd_kv_gather": (ctypes.c_int, [_P, _P, _P, _P, _P, _I64, _I64, _P]),
    "thd_rows_to_global": (ctypes.c_int, [_P, _P, _P, _I64, _P]),
    "thd_cp_attn_fwd": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _F, _I32, _P]),
    "thd_cp_attn_fwd_fused_gather": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _F, _I32,
                                                    _P]),
    "thd_cu_seqlens_from_eod": (ctypes.c_int, [_P, ctypes.c_int64, _I32, _P, _I32, _P]),
    "thd_position_ids": (ctypes.c_int, [_P, _I32, _P]),
    "thd_rope_workspace": (ctypes.c_int, [ctypes.c_int64, _I32, _P]),
    "thd_rope_apply": (ctypes.c_int, [_P, _P, ctypes.c_int64, _I32, _I32, _I32, ctypes.c_double, _I32, _P,
                                      ctypes.c_size_t, _P]),
    "thd_cp_attn_fwd_mla": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _I32, _I32, _I32, _I32, _I32, _F, _I32,
                                           _P]),
    "thd_cp_attn_bwd_workspace": (ctypes.c_int, [_P, _I32, _I32, _I32, _I32, _I32, ctypes.POINTER(ctypes.c_size_t)]),
    "thd_cp_attn_bwd": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t,
                                       _I32, _I32, _I32, _I32, _F, _I32, _P]),
    "thd_cp_attn_bwd_noalloc": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                               _I32, _I32, _I32, _I32, _F, _I32, _P]),
    "thd_cp_device_status": (ctypes.c_int, [_P, _I32, _PI32]),
    "thd_cp_strerror": (ctypes.c_char_p, [ctypes.c_int]),
}


class PlanInfo(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int64), ("cp", ctypes.c_int32), ("n_docs", ctypes.c_int32),
                ("Tl", ctypes.c_int64), ("n_qtiles", ctypes.c_int64), ("n_entries", ctypes.c_int64),
                ("causal_pairs", ctypes.c_int64), ("n_kseg", ctypes.c_int64), ("n_fqtiles", ctypes.c_int64),
                ("n_fentries", ctypes.c_int64), ("n_fkseg", ctypes.c_int64)]


class ThdError(RuntimeError):
    def __init__(self, fn: str, code: int, text: str):
        super().__init__(f"{fn} failed: {ERRORS.get(code, code)} ({text})")
        self.code = code
        self.kind = ERRORS.get(code, str(code))


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library.  Raises if it has not been built: there is no fallback."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libthdcp.so is not built at {LIB_PATH}; run "
                              "`python -m context_packed_sequence_cp_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def check(fn: str, rc: int) -> None:
    if rc != THD_OK:
        raise ThdError(fn, rc, lib().thd_cp_strerror(rc).decode())
