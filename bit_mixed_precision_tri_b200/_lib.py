"""ctypes binding of libtri_b200.so: argument marshalling only.

Every computation happens inside the CUDA library; this module declares the
C signatures of include/tri.h and loads the in-tree shared library.  There is
no fallback: if the library is missing or fails to load, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import re

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB_PATH = os.path.join(PKG, "libtri_b200.so")
HEADER = os.path.join(ROOT, "include", "tri.h")

TRI_OK = 0
TRI_TQ1, TRI_TQ2 = 1, 2
PATH_AUTO, PATH_SIMT, PATH_MMA, PATH_TCGEN05, PATH_I8 = 0, 1, 2, 3, 4
STATUS_NAMES = {
    0: "TRI_OK", 1: "TRI_ERR_INVALID_ARG", 2: "TRI_ERR_SHAPE", 3: "TRI_ERR_ALIGNMENT",
    4: "TRI_ERR_NONFINITE", 5: "TRI_ERR_INVALID_CODE", 6: "TRI_ERR_CUDA",
    7: "TRI_ERR_NOT_IMPLEMENTED", 8: "TRI_ERR_WORKSPACE", 9: "TRI_ERR_NO_DEVICE",
    10: "TRI_ERR_SCRATCH_LIMIT",
}

_p = ctypes.c_void_p
_i64 = ctypes.c_int64
_i = ctypes.c_int
_sz = ctypes.c_size_t
_f = ctypes.c_float

SIGNATURES = {
    "tri_status_string": (ctypes.c_char_p, [_i]),
    "tri_version": (_i, []),
    "tri_last_cuda_error": (ctypes.c_char_p, []),
    "tri_absmean_workspace_bytes": (_sz, [_i64, _i64]),
    "tri_absmean": (_i, [_p, _i64, _i64, _f, _p, _p, _sz, _p]),
    "tri_ternarize": (_i, [_p, _i64, _i64, _f, _p, _p, _p, _sz, _p]),
    "tri_pack_tq2": (_i, [_p, _i64, _i64, _p, _i64, _p, _p, _p, _p]),
    "tri_pack_tq1": (_i, [_p, _i64, _i64, _p, _i64, _p, _p, _p, _p]),
    "tri_unpack": (_i, [_i, _p, _i64, _i64, _p, _p, _p]),
    "tri_gemm_workspace_bytes": (_sz, [_i, _i64, _i64, _i64]),
    "tri_gemm": (_i, [_i, _i, _p, _p, _p, _p, _i64, _i64, _i64, _p, _sz, _p]),
    "tri_gemm_tq2": (_i, [_p, _p, _p, _p, _i64, _i64, _i64, _p, _sz, _p]),
    "tri_gemm_tq1": (_i, [_p, _p, _p, _p, _i64, _i64, _i64, _p, _sz, _p]),
    "tri_gemm_auto_path": (_i, [_i, _i64, _i64, _i64]),
    "tri_gemm_swiglu_workspace_bytes": (_sz, [_i, _i64, _i64, _i64]),
    "tri_gemm_swiglu": (_i, [_i, _i, _p, _p, _p, _p, _i64, _i64, _i64, _p, _sz, _p]),
    "tri_gemm_tq2_noalloc": (_i, [_p, _p, _p, _p, _i64, _i64, _i64, _p]),
    "tri_gemm_tq2_noalloc_fits": (_i, [_i64, _i64, _i64]),
    "tri_wait_status": (_i, [_p, _i, _p]),
    "tri_selftest_wait_timeout": (_i, [_i, _p, _p]),
    "tri_rmsnorm": (_i, [_p, _p, _p, _p, _p, _i64, _i64, _f, _p]),
    "tri_rope_table": (_i, [_p, _i64, _i64, ctypes.c_double, _p]),
    "tri_qknorm_rope": (_i, [_p, _p, _p, _p, _p, _p, _p, _p, _i64, _i64, _i64, _i64, _f, _p]),
    "tri_attention_decode_workspace_bytes": (_sz, [_i64, _i64, _i64, _i64]),
    "tri_attention_decode": (_i, [_p, _p, _p, _p, _p, _i64, _i64, _i64, _i64, _i64, _p, _sz, _p]),
}


class TriError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)}")


def declared_symbols(header: str = HEADER) -> list:
    """Function names declared in include/tri.h."""
    with open(header) as f:
        text = f.read()
    return sorted(set(re.findall(r"TRI_API\s+[\w\s\*]+?\b(tri_\w+)\s*\(", text)))


_LIB = None


def lib() -> ctypes.CDLL:
    """The loaded CUDA library (raises if it was not built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m bit_mixed_precision_tri_b200.build`"
                " (there is no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def check(status: int, what: str) -> None:
    if status != TRI_OK:
        if status == 6:   # TRI_ERR_CUDA: add the runtime's message
            what = f"{what} ({lib().tri_last_cuda_error().decode()})"
        raise TriError(status, what)
