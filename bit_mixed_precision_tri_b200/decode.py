"""One transformer-block decode step around the ternary linear layers.

"Scaling Laws and Efficient Inference for Ternary Language Models", section
"The model": the blocks follow LLaMA (SwiGLU MLP, rotary embeddings with
theta = 5e5, RMSNorm, QK-Norm, no biases); every linear layer is ternary.
This module marshals arguments for the library's decode-step entry points
(``tri_rmsnorm``, ``tri_rope_table``, ``tri_qknorm_rope``,
``tri_attention_decode``) and strings them together with the ternary GEMMs:
every step runs in the CUDA library.

Block (fp16 activations between steps, head dimension 128)::

    xn  = RMSNorm(x; g_attn)
    qkv = xn Wqkv^T                       (ternary, q / k / v rows fused)
    q, k, v = QK-Norm + RoPE(qkv, pos)    (k, v appended to the caches)
    a   = attention(q, K cache, V cache)  (grouped queries)
    h   = x + a Wo^T                      (ternary; the sum is fused into the norm kernel)
    hn  = RMSNorm(h; g_mlp)
    f   = SwiGLU(hn Wgate^T, hn Wup^T)    (ternary, fused gate / up)
    out = h + f Wdown^T                   (ternary)
"""
from __future__ import annotations

import torch

from . import _lib
from .api import PATH_AUTO, Workspace, _ptr, _require_cuda, _stream, gemm, gemm_swiglu, interleave_gate_up, pack

HEAD_DIM = 128
RMS_EPS = 1e-5
ROPE_THETA = 5.0e5


def _half(*ts):
    for t in ts:
        if t.dtype != torch.float16 or not t.is_contiguous():
            raise ValueError("activations, gains and caches must be contiguous float16 tensors")


def rmsnorm(x: torch.Tensor, g: torch.Tensor, r: torch.Tensor = None, eps: float = RMS_EPS,
            out: torch.Tensor = None, h_out: torch.Tensor = None):
    """y = RMSNorm(h) * g with h = x, or h = x + r (returned too) when r is given."""
    _require_cuda(x, g)
    _half(x, g)
    M, D = x.shape
    y = out if out is not None else torch.empty_like(x)
    h = None
    if r is not None:
        _half(r)
        h = h_out if h_out is not None else torch.empty_like(x)
    st = _lib.lib().tri_rmsnorm(_ptr(x), _ptr(r) if r is not None else None, _ptr(g),
                                _ptr(h) if h is not None else None, _ptr(y), M, D, eps, _stream(x.device))
    _lib.check(st, "tri_rmsnorm")
    return (y, h) if r is not None else y


def rope_table(Lmax: int, device, theta: float = ROPE_THETA) -> torch.Tensor:
    """(cos, sin) of p * theta^(-2i/128), float32 [Lmax][64][2]."""
    cs = torch.empty(Lmax, HEAD_DIM // 2, 2, dtype=torch.float32, device=device)
    st = _lib.lib().tri_rope_table(_ptr(cs), Lmax, HEAD_DIM, float(theta), _stream(cs.device))
    _lib.check(st, "tri_rope_table")
    return cs


def qknorm_rope(qkv: torch.Tensor, pos: torch.Tensor, gq: torch.Tensor, gk: torch.Tensor, cs: torch.Tensor,
                kcache: torch.Tensor, vcache: torch.Tensor, H: int, Hkv: int, eps: float = RMS_EPS,
                out: torch.Tensor = None) -> torch.Tensor:
    """Queries [M][H][128] normed and rotated; keys (normed, rotated) and
    values appended to the caches [M][Hkv][Lmax][128] at pos [M] (int32)."""
    _require_cuda(qkv, pos, gq, gk, cs, kcache, vcache)
    _half(qkv, gq, gk, kcache, vcache)
    if pos.dtype != torch.int32 or cs.dtype != torch.float32:
        raise ValueError("pos must be int32 and the RoPE table float32")
    M = qkv.shape[0]
    Lmax = kcache.shape[2]
    q = out if out is not None else torch.empty(M, H, HEAD_DIM, dtype=torch.float16, device=qkv.device)
    st = _lib.lib().tri_qknorm_rope(_ptr(qkv), _ptr(pos), _ptr(gq), _ptr(gk), _ptr(cs), _ptr(q), _ptr(kcache),
                                    _ptr(vcache), M, H, Hkv, Lmax, eps, _stream(qkv.device))
    _lib.check(st, "tri_qknorm_rope")
    return q


def attention_workspace_bytes(M: int, H: int, Hkv: int, max_len: int) -> int:
    return int(_lib.lib().tri_attention_decode_workspace_bytes(M, H, Hkv, max_len))


def attention_decode(q: torch.Tensor, kcache: torch.Tensor, vcache: torch.Tensor, pos: torch.Tensor,
                     max_len: int, workspace: Workspace = None, out: torch.Tensor = None) -> torch.Tensor:
    """softmax(K q / sqrt(128)) V over positions 0..pos[m]; [M][H * 128]."""
    _require_cuda(q, kcache, vcache, pos)
    _half(q, kcache, vcache)
    M, H, _ = q.shape
    Hkv, Lmax = kcache.shape[1], kcache.shape[2]
    y = out if out is not None else torch.empty(M, H * HEAD_DIM, dtype=torch.float16, device=q.device)
    L = _lib.lib()
    nbytes = int(L.tri_attention_decode_workspace_bytes(M, H, Hkv, max_len))
    ws = (workspace or Workspace(q.device)).get(max(nbytes, 256))
    st = L.tri_attention_decode(_ptr(q), _ptr(kcache), _ptr(vcache), _ptr(pos), _ptr(y), M, H, Hkv, Lmax, max_len,
                                _ptr(ws), ws.numel(), _stream(q.device))
    _lib.check(st, "tri_attention_decode")
    return y


class DecodeBlock:
    """One ternary transformer block with its KV caches, for decode steps of
    M sequences.  Weights are packed ternary planes (TQ2 or TQ1); gains fp16.

    ``weights``: dict of trits (int8, on any device) and float32 scales
    (one per matrix or one per 256-block) for "qkv" [(H + 2 Hkv) 128][D],
    "o" [D][H 128], "gate", "up" [F][D], "down" [D][F]; and fp16 gains
    "g_attn", "g_mlp" [D], "gq", "gk" [128]."""

    def __init__(self, weights: dict, D: int, H: int, Hkv: int, F: int, M: int, Lmax: int, device,
                 fmt: str = "tq2", eps: float = RMS_EPS, theta: float = ROPE_THETA):
        dev = torch.device(device)
        self.D, self.H, self.Hkv, self.F, self.M, self.Lmax, self.fmt, self.eps = D, H, Hkv, F, M, Lmax, fmt, eps
        self.dev = dev
        packed = {}
        for name in ("qkv", "o", "gate", "up", "down"):
            t, sc = weights[name]
            packed[name] = pack(t.to(dev), sc.to(dev), fmt)
        self.qkv = packed["qkv"]
        self.o = packed["o"]
        self.gu = interleave_gate_up(*packed["gate"], *packed["up"])
        self.down = packed["down"]
        self.g_attn, self.g_mlp = weights["g_attn"].to(dev), weights["g_mlp"].to(dev)
        self.gq, self.gk = weights["gq"].to(dev), weights["gk"].to(dev)
        self.kcache = torch.zeros(M, Hkv, Lmax, HEAD_DIM, dtype=torch.float16, device=dev)
        self.vcache = torch.zeros_like(self.kcache)
        self.cs = rope_table(Lmax, dev, theta)
        f16 = dict(dtype=torch.float16, device=dev)
        self.buf = {"xn": torch.empty(M, D, **f16), "qkv": torch.empty(M, (H + 2 * Hkv) * HEAD_DIM, **f16),
                    "q": torch.empty(M, H, HEAD_DIM, **f16), "attn": torch.empty(M, H * HEAD_DIM, **f16),
                    "o": torch.empty(M, D, **f16), "h": torch.empty(M, D, **f16), "hn": torch.empty(M, D, **f16),
                    "f": torch.empty(M, F, **f16), "down": torch.empty(M, D, **f16),
                    "out": torch.empty(M, D, **f16), "scratch": torch.empty(M, D, **f16)}
        self.ws = {k: Workspace(dev) for k in ("qkv", "o", "gu", "down", "attn")}

    @property
    def weight_bytes(self) -> int:
        n = 0
        for qs, d in (self.qkv, self.o, self.gu, self.down):
            n += qs.numel() * qs.element_size() + d.numel() * d.element_size()
        return n

    def step(self, x: torch.Tensor, pos: torch.Tensor, max_len: int, path: int = PATH_AUTO) -> torch.Tensor:
        """One decode step: x [M][D] fp16 (the new tokens' residual stream),
        pos [M] int32 device positions (< Lmax), max_len >= max(pos) + 1.
        Returns the block output [M][D] (a buffer reused by the next step)."""
        b, H, Hkv, D, F = self.buf, self.H, self.Hkv, self.D, self.F
        rmsnorm(x, self.g_attn, eps=self.eps, out=b["xn"])
        gemm(b["xn"], *self.qkv, (H + 2 * Hkv) * HEAD_DIM, D, self.fmt, path=path, out=b["qkv"],
             workspace=self.ws["qkv"])
        qknorm_rope(b["qkv"], pos, self.gq, self.gk, self.cs, self.kcache, self.vcache, H, Hkv, self.eps, out=b["q"])
        attention_decode(b["q"], self.kcache, self.vcache, pos, max_len, workspace=self.ws["attn"], out=b["attn"])
        gemm(b["attn"], *self.o, D, H * HEAD_DIM, self.fmt, path=path, out=b["o"], workspace=self.ws["o"])
        rmsnorm(x, self.g_mlp, r=b["o"], eps=self.eps, out=b["hn"], h_out=b["h"])
        gemm_swiglu(b["hn"], *self.gu, F, D, self.fmt, path=path, out=b["f"], workspace=self.ws["gu"])
        gemm(b["f"], *self.down, D, F, self.fmt, path=path, out=b["down"], workspace=self.ws["down"])
        # out = h + down; the norm it also produces is not used by a single block
        rmsnorm(b["h"], self.g_mlp, r=b["down"], eps=self.eps, out=b["scratch"], h_out=b["out"])
        return b["out"]
