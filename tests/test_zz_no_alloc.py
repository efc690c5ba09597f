"""The entry point for callers that cannot allocate device memory.

tri_gemm_tq2_noalloc runs the decode-regime GEMM with the library's static
scratch array instead of a caller workspace.  Callers such as a plugin whose
host framework owns every device allocation, or a real-time loop that keeps
a fixed memory footprint, cannot hand the library a cudaMalloc'd workspace.

Each output is checked against the FP64 CPU oracle at the GEMM tolerance
used by every other GEMM test, and against the workspace entry point
tri_gemm_tq2 on the same inputs, on two calls in a row (the second call finds
the first one's bytes in the shared array).

This file is named so that pytest collects it last: if it fails, a run that
stops at the first failure has already run every other test.  It must pass
both on its own in a fresh process and after the rest of the suite (the
static array then holds whatever earlier calls left in it).
"""
import numpy as np
import pytest
import torch

from bit_mixed_precision_tri_b200 import _lib, inputs
from oracle import tri_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _packed_case(M, N, K, seed):
    W = inputs.latent_weights(N, K, seed)
    trits, g = O.absmean_ternarize(W.numpy(), 1e-6)
    qs, d = O.pack_tq2(trits, np.array([g], np.float32))
    X = inputs.activations(M, K, seed + 1).numpy()
    y_ref = O.gemm_f64(X, trits, d)
    return (torch.from_numpy(X).to(DEV), torch.from_numpy(qs).to(DEV),
            torch.from_numpy(d).to(DEV), O.gemm_tolerance(X, d, y_ref), y_ref)


@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (5, 777, 2048), (16, 1000, 11008)])
def test_noalloc_matches_oracle_and_workspace_entry_point(M, N, K):
    L = _lib.lib()
    assert L.tri_gemm_tq2_noalloc_fits(M, N, K) == 1
    st = torch.cuda.current_stream().cuda_stream
    for call in range(2):                       # two calls in a row share the array
        Xd, qs, d, tol, y_ref = _packed_case(M, N, K, 40 + 10 * call + M)
        Y_static = torch.full((M, N), float("nan"), dtype=torch.float16, device=DEV)
        Y_ws = torch.empty(M, N, dtype=torch.float16, device=DEV)
        rc = L.tri_gemm_tq2_noalloc(Xd.data_ptr(), qs.data_ptr(), d.data_ptr(), Y_static.data_ptr(),
                                    M, N, K, st)
        assert rc == 0, _lib.STATUS_NAMES.get(rc, rc)
        wsb = L.tri_gemm_workspace_bytes(2, M, N, K)
        ws = torch.zeros(wsb, dtype=torch.uint8, device=DEV)
        rc = L.tri_gemm_tq2(Xd.data_ptr(), qs.data_ptr(), d.data_ptr(), Y_ws.data_ptr(), M, N, K,
                            ws.data_ptr(), wsb, st)
        assert rc == 0, _lib.STATUS_NAMES.get(rc, rc)
        torch.cuda.synchronize()
        a = Y_static.float().cpu().numpy().astype(np.float64)
        b = Y_ws.float().cpu().numpy().astype(np.float64)
        assert np.all(np.abs(a - y_ref) <= tol), f"call {call}: {float(np.max(np.abs(a - y_ref) - tol))}"
        assert np.all(np.abs(b - y_ref) <= tol)
        # the two entry points agree within the sum of their allowed errors
        assert np.all(np.abs(a - b) <= 2 * tol)


def test_noalloc_rejects_what_it_cannot_hold():
    L = _lib.lib()
    buf = torch.zeros(1 << 16, dtype=torch.uint8, device=DEV)
    p = buf.data_ptr()
    st = torch.cuda.current_stream().cuda_stream
    # batch above the decode regime
    assert L.tri_gemm_tq2_noalloc(p, p, p, p, 17, 256, 256, st) == 2
    # a reduction dimension whose prepared activations exceed the static array
    K = 1 << 20
    assert L.tri_gemm_tq2_noalloc_fits(16, 256, K) == 0
    assert L.tri_gemm_tq2_noalloc(p, p, p, p, 16, 256, K, st) == 10
    torch.cuda.synchronize()
