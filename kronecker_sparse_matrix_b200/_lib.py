"""ctypes view of the C ABI declared in include/ks.h (libks_b200.so).

Loading fails loudly: if the shared library is missing or does not export
every entry point, importing the functions below raises instead of falling
back to anything else.
"""
from __future__ import annotations

import ctypes
import os
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libks_b200.so")

# ks_dtype
KS_F32, KS_TF32, KS_BF16 = 0, 1, 2
# ks_variant
KS_VARIANT_AUTO, KS_VARIANT_STREAM, KS_VARIANT_FMA, KS_VARIANT_TC = 0, 1, 2, 3
KS_CHAIN_UNFUSED = 1
ACTIVATIONS = {"none": 0, "relu": 1, "gelu_tanh": 2, "gelu_erf": 3}
VARIANTS = {"auto": 0, "stream": 1, "fma": 2, "tc": 3}
# ks_status
STATUS = {0: "KS_OK", 1: "KS_ERR_INVALID_ARG", 2: "KS_ERR_MISALIGNED", 3: "KS_ERR_UNSUPPORTED",
          4: "KS_ERR_ALLOC", 5: "KS_ERR_CUDA", 6: "KS_ERR_TIMEOUT"}

# Every function include/ks.h declares, with (restype, argtypes).
_i64 = ctypes.c_int64
_vp = ctypes.c_void_p
_int = ctypes.c_int


class KsPattern(ctypes.Structure):
    _fields_ = [("a", _i64), ("b", _i64), ("c", _i64), ("d", _i64)]


SIGNATURES = {
    "ks_matmul": (_int, [_vp, _vp, _i64, _i64, _i64, _i64, _i64, _vp, _int, _vp]),
    "ks_matmul_variant": (_int, [_vp, _vp, _i64, _i64, _i64, _i64, _i64, _vp, _int, _int, _vp]),
    "ks_matmul_host": (_int, [_vp, _vp, _i64, _i64, _i64, _i64, _i64, _vp, _int, _vp]),
    "ks_plan": (_int, [_i64, _i64, _i64, _i64, _i64, _int, ctypes.POINTER(_int)]),
    "ks_chain": (_int, [_vp, ctypes.POINTER(_vp), ctypes.POINTER(KsPattern), _int, _i64, _vp, _int, _vp]),
    "ks_matmul_ep": (_int, [_vp, _vp, _i64, _i64, _i64, _i64, _i64, _vp, _int, _vp, _int, _int, _vp]),
    "ks_chain_ep": (_int, [_vp, ctypes.POINTER(_vp), ctypes.POINTER(KsPattern), _int, _i64, _vp, _int, _int, _vp,
                           _int, _vp]),
    "ks_butterfly_factorize": (_int, [_vp, _int, ctypes.POINTER(_vp), _int, _vp]),
    "ks_matmul_dx": (_int, [_vp, _vp, _i64, _i64, _i64, _i64, _i64, _vp, _int, _vp]),
    "ks_matmul_dv": (_int, [_vp, _vp, _i64, _i64, _i64, _i64, _i64, _vp, _int, _vp]),
    "ks_chain_ex": (_int, [_vp, ctypes.POINTER(_vp), ctypes.POINTER(KsPattern), _int, _i64, _vp, _int, _int, _vp]),
    "ks_chain_noalloc": (_int, [_vp, ctypes.POINTER(_vp), ctypes.POINTER(KsPattern), _int, _i64, _vp, _int, _vp]),
    "ks_bias_grad": (_int, [_vp, _i64, _i64, _vp, _int, _vp]),
    "ks_workspace_info": (_int, [ctypes.POINTER(_i64), ctypes.POINTER(_i64)]),
    "ks_fma_rate_probe": (_int, [_vp, _int, _i64, _vp]),
    "ks_last_error": (ctypes.c_char_p, []),
    "ks_status_string": (ctypes.c_char_p, [_int]),
    "ks_sync_status": (_int, [_vp]),
    "ks_version": (_int, []),
}

_lock = threading.Lock()
_lib = None


class KsError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


def load() -> ctypes.CDLL:
    """Load libks_b200.so (build it with ``python -m kronecker_sparse_matrix_b200.build``)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"{LIB_PATH} is missing; build it with "
                                  "`python -m kronecker_sparse_matrix_b200.build`")
            lib = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)  # AttributeError if the symbol is not exported
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def check(status: int) -> None:
    if status != 0:
        msg = load().ks_last_error().decode(errors="replace")
        raise KsError(status, msg)
