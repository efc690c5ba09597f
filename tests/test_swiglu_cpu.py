"""Host-side pieces of the fused gate/up (SwiGLU) call: the row interleave
of the packed weights and the workspace query, without a GPU."""
import torch

import bit_mixed_precision_tri_b200 as tri
from bit_mixed_precision_tri_b200 import _lib


def test_interleave_gate_up_layout():
    F, rb = 24, 64
    qg = torch.arange(F * rb, dtype=torch.int32).reshape(F, rb).to(torch.uint8)
    qu = (torch.arange(F * rb, dtype=torch.int32).reshape(F, rb) + 100).to(torch.uint8)
    dg = torch.arange(F * 4, dtype=torch.float32).reshape(F, 4).half()
    du = -dg
    q, d = tri.interleave_gate_up(qg, dg, qu, du)
    assert q.shape == (2 * F, rb) and d.shape == (2 * F, 4)
    for j in range(F // 8):
        for i in range(8):
            assert torch.equal(q[16 * j + i], qg[8 * j + i])
            assert torch.equal(q[16 * j + 8 + i], qu[8 * j + i])
            assert torch.equal(d[16 * j + 8 + i], du[8 * j + i])


def test_interleave_rejects_bad_shapes():
    q = torch.zeros(12, 64, dtype=torch.uint8)
    d = torch.zeros(12, 4, dtype=torch.float16)
    try:
        tri.interleave_gate_up(q, d, q, d)
        assert False, "F % 8 != 0 must be rejected"
    except ValueError:
        pass


def test_swiglu_workspace_query_no_gpu():
    L = _lib.lib()
    assert L.tri_gemm_swiglu_workspace_bytes(2, 4, 12, 256) == 0          # F % 8 != 0
    assert L.tri_gemm_swiglu_workspace_bytes(2, 4, 1024, 4096) >= 4 * 2048 * 2
    assert L.tri_gemm_swiglu_workspace_bytes(1, 16, 512, 1024) > 0
