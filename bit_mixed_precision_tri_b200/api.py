"""Torch-facing wrappers over the C ABI (include/tri.h).

PyTorch provides device memory and the current CUDA stream; every step of the
path runs in the library's CUDA kernels.  Functions raise ``TriError`` on a
non-OK status and never fall back to another implementation.
"""
from __future__ import annotations

import collections
import ctypes

import torch

from . import _lib
from ._lib import PATH_AUTO, PATH_I8, PATH_MMA, PATH_SIMT, PATH_TCGEN05, TRI_TQ1, TRI_TQ2, TriError  # noqa: F401

FORMATS = {"tq2": TRI_TQ2, "tq1": TRI_TQ1}


def _fmt(fmt) -> int:
    if isinstance(fmt, str):
        return FORMATS[fmt]
    return int(fmt)


def _ptr(t) -> int:
    return 0 if t is None else t.data_ptr()


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("tensors must live on a CUDA device")
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def packed_row_bytes(fmt, K: int) -> int:
    return K // 4 if _fmt(fmt) == TRI_TQ2 else (K // 256) * 52


# ------------------------------------------------------------------ a1, a2
def absmean(W: torch.Tensor, eps: float = 1e-6) -> torch.Tensor:
    """gamma = eps + mean|W| (exact sum), as a device float32 tensor of shape (1,)."""
    _require_cuda(W)
    N, K = W.shape
    L = _lib.lib()
    ws = torch.empty(L.tri_absmean_workspace_bytes(N, K), dtype=torch.uint8, device=W.device)
    g = torch.empty(1, dtype=torch.float32, device=W.device)
    _lib.check(L.tri_absmean(_ptr(W), N, K, eps, _ptr(g), _ptr(ws), ws.numel(), _stream(W.device)),
               "tri_absmean")
    return g


def ternarize(W: torch.Tensor, eps: float = 1e-6, check_finite: bool = True):
    """(trits int8[N][K], gamma float32[1]) by absmean ternarization.

    With ``check_finite`` the host waits for gamma and raises TriError
    (TRI_ERR_NONFINITE) when W held Inf or NaN.
    """
    _require_cuda(W)
    if W.dtype != torch.float32:
        raise ValueError("W must be float32")
    N, K = W.shape
    L = _lib.lib()
    ws = torch.empty(L.tri_absmean_workspace_bytes(N, K), dtype=torch.uint8, device=W.device)
    g = torch.empty(1, dtype=torch.float32, device=W.device)
    trits = torch.empty(N, K, dtype=torch.int8, device=W.device)
    _lib.check(L.tri_ternarize(_ptr(W), N, K, eps, _ptr(trits), _ptr(g), _ptr(ws), ws.numel(),
                               _stream(W.device)), "tri_ternarize")
    if check_finite and not torch.isfinite(g).item():
        raise TriError(4, "tri_ternarize: weights hold Inf or NaN")
    return trits, g


# ------------------------------------------------------------------ a3, a4
def pack(trits: torch.Tensor, scales: torch.Tensor, fmt="tq2", return_invalid: bool = False):
    """(qs uint8, d fp16[N][K/256]) in TQ2 or TQ1.  ``scales`` is float32 of
    one element (one scale for the matrix) or N*K/256 elements (per block)."""
    _require_cuda(trits, scales)
    N, K = trits.shape
    f = _fmt(fmt)
    qs = torch.empty(N, packed_row_bytes(f, K), dtype=torch.uint8, device=trits.device)
    d = torch.empty(N, K // 256, dtype=torch.float16, device=trits.device)
    inv = torch.zeros(1, dtype=torch.int32, device=trits.device)
    fn = _lib.lib().tri_pack_tq2 if f == TRI_TQ2 else _lib.lib().tri_pack_tq1
    _lib.check(fn(_ptr(trits), N, K, _ptr(scales), scales.numel(), _ptr(qs), _ptr(d), _ptr(inv),
                  _stream(trits.device)), "tri_pack")
    return (qs, d, inv) if return_invalid else (qs, d)


def unpack(qs: torch.Tensor, N: int, K: int, fmt="tq2", return_invalid: bool = False):
    """int8 trits[N][K] decoded from a packed plane."""
    _require_cuda(qs)
    trits = torch.empty(N, K, dtype=torch.int8, device=qs.device)
    inv = torch.zeros(1, dtype=torch.int32, device=qs.device)
    _lib.check(_lib.lib().tri_unpack(_fmt(fmt), _ptr(qs), N, K, _ptr(trits), _ptr(inv),
                                     _stream(qs.device)), "tri_unpack")
    return (trits, inv) if return_invalid else trits


# ------------------------------------------------------------------ a6
_WS_BYTES = {}


def gemm_workspace_bytes(fmt, M: int, N: int, K: int) -> int:
    key = (_fmt(fmt), M, N, K, torch.cuda.current_device() if torch.cuda.is_available() else -1)
    v = _WS_BYTES.get(key)
    if v is None:
        v = _WS_BYTES[key] = int(_lib.lib().tri_gemm_workspace_bytes(key[0], M, N, K))
    return v


def auto_path(fmt, M: int, N: int, K: int) -> int:
    return int(_lib.lib().tri_gemm_auto_path(_fmt(fmt), M, N, K))


class Workspace:
    """Device scratch for tri_gemm, grown on demand.  Its contents between
    calls do not matter; calls that share one must be ordered (one stream).
    A buffer that grows is allocated on the stream of the call that needs it,
    so the allocator frees the old one in that stream's order."""

    def __init__(self, device=None):
        self.device = torch.device(device or "cuda")
        self.buf = None

    def get(self, nbytes: int, stream=None) -> torch.Tensor:
        if self.buf is None or self.buf.numel() < nbytes:
            with torch.cuda.stream(stream):          # a no-op for stream=None
                self.buf = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=self.device)
        return self.buf


_default_ws = collections.OrderedDict()
_DEFAULT_WS_PER_DEVICE = 8


def _workspace_for(device, stream_handle: int) -> Workspace:
    """The default workspace of (device, stream): calls on different streams
    never share scratch, calls on one stream are ordered by it.  At most
    ``_DEFAULT_WS_PER_DEVICE`` streams per device keep one (least recently
    used dropped first), so short-lived streams do not pin device memory.  A
    dropped buffer is released through the caching allocator, which keeps it
    until the work already queued on its stream has used it (it was
    allocated on that stream)."""
    dev = torch.device(device)
    key = (dev, int(stream_handle))
    ws = _default_ws.get(key)
    if ws is None:
        ws = _default_ws[key] = Workspace(dev)
        mine = [k for k in _default_ws if k[0] == dev]
        for k in mine[:max(0, len(mine) - _DEFAULT_WS_PER_DEVICE)]:
            del _default_ws[k]
    else:
        _default_ws.move_to_end(key)
    return ws


class WaitGaveUp(RuntimeError):
    """A bounded wait inside a GEMM kernel ran out (code in ``.code``); the
    output of the call is unspecified."""

    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: a bounded wait in the kernel gave up (code {code})")


def _check_waits(device, stream_handle: int, what: str) -> None:
    """Synchronize `stream_handle`, read and clear the device's wait status
    word, raise WaitGaveUp when a wait gave up."""
    code = ctypes.c_uint32(0)
    with torch.cuda.device(device):
        st = _lib.lib().tri_wait_status(ctypes.byref(code), 1, stream_handle)
    if st:
        _lib.check(st, "tri_wait_status")
    if code.value:
        raise WaitGaveUp(int(code.value), what)


def gemm(X: torch.Tensor, qs: torch.Tensor, d: torch.Tensor, N: int, K: int, fmt="tq2",
         path: int = PATH_AUTO, out: torch.Tensor = None, workspace: Workspace = None,
         stream=None, check: bool = False) -> torch.Tensor:
    """Y = X (d * W_hat)^T in fp16 with fp32 accumulation.

    ``check=True`` (for debugging; it synchronizes the stream) reads the
    device's wait status word after the call and raises WaitGaveUp if a
    bounded wait inside the kernel ran out."""
    # the checks a decode step pays on every call, kept to attribute reads
    if not (X.is_cuda and qs.is_cuda and d.is_cuda):
        raise ValueError("tensors must live on a CUDA device")
    if not (X.is_contiguous() and qs.is_contiguous() and d.is_contiguous()):
        raise ValueError("tensors must be contiguous")
    if X.dtype != torch.float16:
        raise ValueError("X must be float16")
    M = X.shape[0]
    f = FORMATS[fmt] if isinstance(fmt, str) else int(fmt)
    if out is None:
        Y = torch.empty(M, N, dtype=torch.float16, device=X.device)
    else:
        if not (out.is_cuda and out.is_contiguous()):
            raise ValueError("out must be a contiguous CUDA tensor")
        Y = out
    s = stream.cuda_stream if stream is not None else _stream(X.device)
    ws = (workspace or _workspace_for(X.device, s)).get(gemm_workspace_bytes(f, M, N, K), stream)
    st = _lib.lib().tri_gemm(f, int(path), X.data_ptr(), qs.data_ptr(), d.data_ptr(), Y.data_ptr(),
                             M, N, K, ws.data_ptr(), ws.numel(), s)
    if st:
        _lib.check(st, "tri_gemm")
    if check:
        _check_waits(X.device, s, "tri_gemm")
    return Y


def interleave_gate_up(qs_gate: torch.Tensor, d_gate: torch.Tensor, qs_up: torch.Tensor,
                       d_up: torch.Tensor):
    """Packed weights of a gate and an up projection (F rows each, F % 8 == 0)
    as the 2F-row matrix that ``gemm_swiglu`` takes: rows interleaved in
    groups of eight (fused row 16j + i = gate row 8j + i, 16j + 8 + i = up row
    8j + i).  A one-time weight layout step (memory movement only)."""
    F = qs_gate.shape[0]
    if F % 8 or qs_up.shape != qs_gate.shape or d_up.shape != d_gate.shape:
        raise ValueError("gate and up must have the same shape, with a multiple of 8 rows")

    def inter(a, b):
        a = a.reshape(F // 8, 8, -1)
        b = b.reshape(F // 8, 8, -1)
        return torch.cat([a, b], dim=1).reshape(2 * F, -1).contiguous()

    return inter(qs_gate, qs_up), inter(d_gate, d_up)


def gemm_swiglu(X: torch.Tensor, qs: torch.Tensor, d: torch.Tensor, F: int, K: int, fmt="tq2",
                path: int = PATH_AUTO, out: torch.Tensor = None, workspace: Workspace = None,
                stream=None, check: bool = False) -> torch.Tensor:
    """Y = silu(X Wg^T) * (X Wu^T), fp16 [M][F], from the interleaved 2F-row
    packed weights of ``interleave_gate_up``; ``check`` as in ``gemm``."""
    if not (X.is_cuda and qs.is_cuda and d.is_cuda):
        raise ValueError("tensors must live on a CUDA device")
    if not (X.is_contiguous() and qs.is_contiguous() and d.is_contiguous()):
        raise ValueError("tensors must be contiguous")
    if X.dtype != torch.float16:
        raise ValueError("X must be float16")
    M = X.shape[0]
    f = FORMATS[fmt] if isinstance(fmt, str) else int(fmt)
    if out is None:
        Y = torch.empty(M, F, dtype=torch.float16, device=X.device)
    else:
        if not (out.is_cuda and out.is_contiguous()):
            raise ValueError("out must be a contiguous CUDA tensor")
        Y = out
    L = _lib.lib()
    s = stream.cuda_stream if stream is not None else _stream(X.device)
    ws = (workspace or _workspace_for(X.device, s)).get(
        max(int(L.tri_gemm_swiglu_workspace_bytes(f, M, F, K)), 256), stream)
    st = L.tri_gemm_swiglu(f, int(path), X.data_ptr(), qs.data_ptr(), d.data_ptr(), Y.data_ptr(),
                           M, F, K, ws.data_ptr(), ws.numel(), s)
    if st:
        _lib.check(st, "tri_gemm_swiglu")
    if check:
        _check_waits(X.device, s, "tri_gemm_swiglu")
    return Y


def wait_status(device=None, clear: bool = True) -> int:
    """Synchronize the device's current stream and return its wait status
    word: 0, or the code of the first bounded wait inside a GEMM kernel that
    gave up since the last clear (that call's output is then unspecified)."""
    dev = torch.device(device or "cuda")
    code = ctypes.c_uint32(0)
    with torch.cuda.device(dev):
        st = _lib.lib().tri_wait_status(ctypes.byref(code), int(clear), _stream(dev))
    if st:
        _lib.check(st, "tri_wait_status")
    return int(code.value)


def selftest_wait_timeout(which: int, device=None) -> None:
    """Enqueue a kernel whose bounded wait cannot complete (0: an mbarrier
    phase, 1: a stamped word), so that it records its code (90 or 91) in the
    wait status word; read it back with ``wait_status``."""
    dev = torch.device(device or "cuda")
    scratch = torch.empty(8, dtype=torch.uint8, device=dev)
    with torch.cuda.device(dev):
        st = _lib.lib().tri_selftest_wait_timeout(int(which), scratch.data_ptr(), _stream(dev))
    if st:
        _lib.check(st, "tri_selftest_wait_timeout")


class TernaryLinear:
    """A ternary linear layer: absmean-ternarized, packed weights and a GEMM.

    ``TernaryLinear.from_latent(W)`` ternarizes latent float32 weights on the
    GPU, packs them (TQ2 or TQ1) with d = fp16(gamma) in every block, and
    ``layer(X)`` computes X (gamma W_hat)^T.
    """

    def __init__(self, qs, d, N, K, fmt="tq2", gamma=None):
        self.qs, self.d, self.N, self.K, self.fmt, self.gamma = qs, d, N, K, fmt, gamma
        self.ws = Workspace(qs.device)

    @classmethod
    def from_latent(cls, W: torch.Tensor, fmt="tq2", eps: float = 1e-6):
        trits, g = ternarize(W, eps)
        qs, d = pack(trits, g, fmt)
        return cls(qs, d, W.shape[0], W.shape[1], fmt, g)

    def __call__(self, X: torch.Tensor, path: int = PATH_AUTO, out=None) -> torch.Tensor:
        return gemm(X, self.qs, self.d, self.N, self.K, self.fmt, path=path, out=out,
                    workspace=self.ws)
