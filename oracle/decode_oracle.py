"""CPU oracle for one transformer-block decode step -- TEST INFRASTRUCTURE ONLY.

The plain float64 statement of the synthetic decode step built around the
ternary linear layers: only the test suite, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline leg may import it; it imports nothing from the
product package.

Source: [TLS] "Scaling Laws and Efficient Inference for Ternary Language
Models", section "The model": the architecture follows LLaMA with SwiGLU
MLPs, rotary embeddings with theta = 5e5, RMSNorm, QK-Norm and no biases;
[SPC] "Spectra: ...", section "Architecture of TriLM and FloatLM":
RMSNorm, SwiGLU, rotary embeddings, multi-headed attention, no biases, and
activations kept in 16-bit floating point.  The pages name the parts and
give no formulas; the readings below are the plain LLaMA definitions.

Readings (D14-D20):

D14 RMSNorm(x) = x / sqrt(mean(x^2) + eps) * g over the feature axis, with a
    learned gain g and eps = 1e-5.
D15 QK-Norm = RMSNorm over each head's dh features of q and of k (one gain
    vector for q, one for k, shared by the heads), applied before RoPE.
D16 RoPE ("rotate half"): for i < dh/2 the pair (x_i, x_{i+dh/2}) is turned
    by the angle p * theta^(-2i/dh), p the token's position, theta = 5e5;
    angles and their cos / sin are exact (float64) here.
D17 Attention: scaled dot product, scale 1/sqrt(dh), softmax over the cached
    positions 0..p of the sequence (the new token's own key included); with
    fewer key/value heads than query heads (grouped queries), query head h
    reads key/value head h // (H / Hkv).
D18 Block: h = x + Wo attn(QKNormRoPE(Wqkv RMSNorm(x))), then
    out = h + Wdown SwiGLU(Wgate, Wup; RMSNorm(h)); every linear is a ternary
    layer (the GEMM of ``tri_oracle``).
D19 Storage points: activations are fp16 between steps (the pages keep
    activations in 16-bit floats); each step computes from the fp16 values
    it is given, in float64, and rounds once (to nearest even) where the
    product stores its result: xn, qkv, q and k (after norm and rotation),
    the attention output, the O product, h, hn, the SwiGLU output, the down
    product and out.  Residual sums are the exact sum rounded once.
D20 Caches: K and V of sequence m, head j, position p live at
    [m][j][p][0..dh) (fp16); the step writes the new token's k (normed and
    rotated) and v at p = pos[m].
"""
from __future__ import annotations

import numpy as np

from . import tri_oracle as T

RMS_EPS = 1e-5
ROPE_THETA = 5.0e5


def rn16(a) -> np.ndarray:
    """Round to fp16 (nearest even) and return as float64."""
    return np.asarray(a, dtype=np.float64).astype(np.float16).astype(np.float64)


def rmsnorm_f64(x, g, eps: float = RMS_EPS) -> np.ndarray:
    """D14: x / sqrt(mean(x^2) + eps) * g over the last axis."""
    x = np.asarray(x, dtype=np.float64)
    ms = np.mean(x * x, axis=-1, keepdims=True)
    return x / np.sqrt(ms + eps) * np.asarray(g, dtype=np.float64)


def residual_f16(x, r) -> np.ndarray:
    """D19: the exact sum of two fp16 tensors, rounded once to fp16."""
    return rn16(np.asarray(x, dtype=np.float64) + np.asarray(r, dtype=np.float64))


def rope_angles_f64(pos, dh: int, theta: float = ROPE_THETA) -> np.ndarray:
    """D16: angles [len(pos)][dh/2], p * theta^(-2i/dh)."""
    i = np.arange(dh // 2, dtype=np.float64)
    inv = theta ** (-2.0 * i / dh)
    return np.asarray(pos, dtype=np.float64)[:, None] * inv[None, :]


def rope_f64(x, pos, theta: float = ROPE_THETA) -> np.ndarray:
    """D16: rotate-half RoPE of x [n][..., dh] at positions pos [n]."""
    x = np.asarray(x, dtype=np.float64)
    dh = x.shape[-1]
    a = rope_angles_f64(pos, dh, theta)
    a = a.reshape((a.shape[0],) + (1,) * (x.ndim - 2) + (dh // 2,))
    c, s = np.cos(a), np.sin(a)
    x1, x2 = x[..., : dh // 2], x[..., dh // 2:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def qknorm_rope_f64(qkv, pos, gq, gk, H: int, Hkv: int, dh: int, eps: float = RMS_EPS,
                    theta: float = ROPE_THETA):
    """D15, D16, D19: from the fp16 QKV product [M][(H + 2 Hkv) dh] return
    (q [M][H][dh], k [M][Hkv][dh], v [M][Hkv][dh]) as stored: q and k normed
    per head, rotated and rounded to fp16; v as given."""
    qkv = np.asarray(qkv, dtype=np.float64)
    M = qkv.shape[0]
    q = qkv[:, : H * dh].reshape(M, H, dh)
    k = qkv[:, H * dh:(H + Hkv) * dh].reshape(M, Hkv, dh)
    v = qkv[:, (H + Hkv) * dh:(H + 2 * Hkv) * dh].reshape(M, Hkv, dh)
    qn = rope_f64(rmsnorm_f64(q, gq, eps), pos, theta)
    kn = rope_f64(rmsnorm_f64(k, gk, eps), pos, theta)
    return rn16(qn), rn16(kn), v.copy()


def attention_decode_f64(q, Kc, Vc, pos) -> np.ndarray:
    """D17: q [M][H][dh], caches [M][Hkv][Lmax][dh], sequence m attends to
    positions 0..pos[m]; returns [M][H * dh] in float64 (unrounded)."""
    q = np.asarray(q, dtype=np.float64)
    Kc = np.asarray(Kc, dtype=np.float64)
    Vc = np.asarray(Vc, dtype=np.float64)
    M, H, dh = q.shape
    Hkv = Kc.shape[1]
    G = H // Hkv
    out = np.zeros((M, H, dh))
    for m in range(M):
        L = int(pos[m]) + 1
        for h in range(H):
            j = h // G
            s = Kc[m, j, :L] @ q[m, h] / np.sqrt(dh)
            p = np.exp(s - s.max())
            out[m, h] = (p / p.sum()) @ Vc[m, j, :L]
    return out.reshape(M, H * dh)


def decode_block_f64(x, pos, Kc, Vc, w, H: int, Hkv: int, dh: int, eps: float = RMS_EPS,
                     theta: float = ROPE_THETA):
    """D18-D20: one decode step of one block for M sequences.

    x: fp16 values [M][D]; pos: [M] positions of the new tokens; Kc, Vc:
    caches (float64 copies, updated in place at pos[m]); w: dict of
    g_attn, g_mlp [D], gq, gk [dh] (fp16 values) and the ternary layers
    (trits, d) "qkv" [(H + 2 Hkv) dh x D], "o" [D x H dh], "gate", "up"
    [F x D], "down" [D x F].  Returns (out, intermediates)."""
    x = np.asarray(x, dtype=np.float64)
    xn = rn16(rmsnorm_f64(x, w["g_attn"], eps))
    qkv = rn16(T.gemm_f64(xn, *w["qkv"]))
    q, k, v = qknorm_rope_f64(qkv, pos, w["gq"], w["gk"], H, Hkv, dh, eps, theta)
    for m in range(x.shape[0]):
        Kc[m, :, int(pos[m])] = k[m]
        Vc[m, :, int(pos[m])] = v[m]
    a = rn16(attention_decode_f64(q, Kc, Vc, pos))
    o = rn16(T.gemm_f64(a, *w["o"]))
    h = residual_f16(x, o)
    hn = rn16(rmsnorm_f64(h, w["g_mlp"], eps))
    f = rn16(T.swiglu_f64(hn, *w["gate"], *w["up"])[0])
    dn = rn16(T.gemm_f64(f, *w["down"]))
    out = residual_f16(h, dn)
    return out, {"xn": xn, "qkv": qkv, "q": q, "k": k, "v": v, "attn": a, "o": o, "h": h, "hn": hn,
                 "f": f, "down": dn}
