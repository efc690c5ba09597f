"""The device wait status word: bounded waits that run out are reported to the
host, the context stays usable, and healthy GEMM calls on every path leave the
word at zero.  The timeouts are made on purpose by the library's self-test
kernel, whose waits (an mbarrier phase nothing arrives on, a stamped word
nothing writes) cannot complete; nothing faults or traps."""
import time

import numpy as np
import pytest
import torch

import bit_mixed_precision_tri_b200 as tri
from bit_mixed_precision_tri_b200 import inputs
from oracle import tri_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _layer(M, N, K, seed):
    W = inputs.latent_weights(N, K, seed)
    trits, g = O.absmean_ternarize(W.numpy(), 1e-6)
    qs, d = O.pack("tq2", trits, np.array([g], np.float32))
    X = inputs.activations(M, K, seed + 100).numpy()
    return X, trits, d, torch.from_numpy(qs).to(DEV), torch.from_numpy(d).to(DEV)


def _assert_close(Y, X, trits, d):
    y_ref = O.gemm_f64(X, trits, d)
    err = np.abs(Y.float().cpu().numpy().astype(np.float64) - y_ref)
    assert not (err > O.gemm_tolerance(X, d, y_ref)).any()


@pytest.mark.parametrize("which,code", [(0, 90), (1, 91)])
def test_selftest_timeout_is_reported_and_cleared(which, code):
    torch.cuda.init()
    tri.wait_status(DEV, clear=True)
    t0 = time.perf_counter()
    tri.selftest_wait_timeout(which, DEV)
    got = tri.wait_status(DEV, clear=False)
    elapsed = time.perf_counter() - t0
    assert got == code
    assert elapsed < 10.0
    assert tri.wait_status(DEV, clear=True) == code      # sticky until cleared
    assert tri.wait_status(DEV) == 0


def test_first_code_sticks():
    tri.wait_status(DEV, clear=True)
    tri.selftest_wait_timeout(1, DEV)
    tri.selftest_wait_timeout(0, DEV)
    assert tri.wait_status(DEV, clear=True) == 91
    assert tri.wait_status(DEV) == 0


def test_context_usable_after_timeout():
    tri.wait_status(DEV, clear=True)
    tri.selftest_wait_timeout(0, DEV)
    assert tri.wait_status(DEV, clear=True) == 90
    X, trits, d, qs_t, d_t = _layer(4, 512, 1024, 7)
    Y = tri.gemm(torch.from_numpy(X).to(DEV), qs_t, d_t, 512, 1024, "tq2")
    _assert_close(Y, X, trits, d)
    assert tri.wait_status(DEV) == 0


@pytest.mark.parametrize("M,path", [(1, tri.PATH_I8), (2, tri.PATH_I8), (9, tri.PATH_I8),
                                    (4, tri.PATH_MMA), (16, tri.PATH_MMA),
                                    (64, tri.PATH_TCGEN05), (300, tri.PATH_TCGEN05)])
def test_healthy_calls_leave_status_zero(M, path):
    tri.wait_status(DEV, clear=True)
    N, K = 1024, 4096
    X, trits, d, qs_t, d_t = _layer(M, N, K, 11 + M)
    Xd = torch.from_numpy(X).to(DEV)
    for _ in range(3):
        Y = tri.gemm(Xd, qs_t, d_t, N, K, "tq2", path=path)
    assert tri.wait_status(DEV) == 0
    _assert_close(Y, X, trits, d)


@pytest.mark.parametrize("fmt", ["tq2", "tq1"])
def test_gemm_check_option(fmt):
    """gemm(check=True) returns normally after healthy calls, and raises
    WaitGaveUp when the word holds a code (here one left by the self-test
    kernel just before the call), clearing it."""
    tri.wait_status(DEV, clear=True)
    M, N, K = 1, 1024, 4096
    W = inputs.latent_weights(N, K, 3)
    trits, g = O.absmean_ternarize(W.numpy(), 1e-6)
    qs, d = O.pack(fmt, trits, np.array([g], np.float32))
    X = inputs.activations(M, K, 4).numpy()
    args = (torch.from_numpy(X).to(DEV), torch.from_numpy(qs).to(DEV), torch.from_numpy(d).to(DEV), N, K, fmt)
    Y = tri.gemm(*args, check=True)
    _assert_close(Y, X, trits, d)
    tri.selftest_wait_timeout(1, DEV)
    with pytest.raises(tri.WaitGaveUp) as e:
        tri.gemm(*args, check=True)
    assert e.value.code == 91
    assert tri.wait_status(DEV) == 0
    Y = tri.gemm_swiglu(torch.from_numpy(np.ascontiguousarray(X)).to(DEV), *tri.interleave_gate_up(
        args[1][:512], args[2][:512], args[1][512:], args[2][512:]), 512, K, fmt, check=True)
    assert Y.shape == (M, 512)
