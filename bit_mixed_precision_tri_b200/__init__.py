"""B200 (sm_100a) ternary-weight linear layer: absmean ternarization, TQ2/TQ1
packing and an FP16 x packed-ternary GEMM, behind a C ABI (include/tri.h).

The torch-facing functions live in ``api``; they load ``libtri_b200.so``
(built in-tree by ``build.py``) on first use.
"""
from .api import (  # noqa: F401
    PATH_AUTO, PATH_I8, PATH_MMA, PATH_SIMT, PATH_TCGEN05, TernaryLinear, TriError, WaitGaveUp, Workspace,
    absmean,
    auto_path, gemm, gemm_swiglu, gemm_workspace_bytes, interleave_gate_up, pack, packed_row_bytes,
    selftest_wait_timeout, ternarize, unpack, wait_status,
)
