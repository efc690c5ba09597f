"""CPU oracle for the ternary-weight linear layer -- TEST INFRASTRUCTURE ONLY.

This module is the plain, slow, obviously correct CPU statement of what the
hot path computes.  It exists to check the CUDA library, never to stand in for
it: only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg
of ``bench.py`` may import it.  It shares no code with the CUDA path (it
imports nothing from the product package) and works in float64 wherever the
method does arithmetic.

Sources (web pages, cited by title and section):

* [TLS] "Scaling Laws and Efficient Inference for Ternary Language Models"
  (Spectra-1.1 / TriTera project page): section "The model" (steps 1-3),
  section "Packing ternary weights" (subsections "2 bits per weight",
  "1.6 bits per weight", the worked example), section "Fast inference on
  CPUs" (256-weight blocks, one 16-bit scale, 66 bytes per block), section
  "TriRun: ternary inference on GPUs" (sixteen 2-bit weights per 32-bit word).
* [SPC] "Spectra: Surprising Effectiveness of Pretraining Ternary Language
  Models at Scale", section "Architecture of TriLM and FloatLM" (one scale
  per matrix, absolute-mean scale, round to nearest ternary state).

Readings of points the pages leave open:

R1  gamma is computed from the EXACT sum S = sum|W| (order independent):
    mean = RN64(RN64(S) / (N*K)), gamma = RN32(RN64(mean + eps)).
R2  W/gamma is an IEEE float32 division; clip to [-1, 1]; round half to even;
    a NaN quotient (non-finite W, or gamma = 0) gives trit 0.
R3  TQ2 byte i of a row holds trits 4i..4i+3, trit 4i+j in bits 2j..2j+1, so a
    little-endian 32-bit word holds sixteen trits, trit j at bits 2j.
    Storage is two planes: qs (64 B per 256-block) and d (one fp16 per block).
R4  TQ1 digit order: the first trit of a group is the most significant base-3
    digit (the worked example decodes to 2,0,1,1,2 in order only this way).
R5  TQ1 block layout: 52 bytes per 256-block; bytes 0..50 hold trits
    5g..5g+4, byte 51 holds trit 255 as its leading digit followed by four
    zero trits (digit 1).
R6  The fp16 block scale is d = fp16(gamma) (round to nearest even); the
    trits are decided with the float32 gamma, the product uses d.
R7  Invalid codes are counted, never trapped: a TQ2 field equal to 3, a TQ1
    byte outside the encoder's image, or a TQ1 block's last byte whose four
    padding digits are not the zero trit.

Parity pins for every function live in tests/test_oracle.py.
"""
from __future__ import annotations

import itertools
import math

import numpy as np

BLOCK = 256          # weights per block [TLS "Fast inference on CPUs"]
TQ2_BLOCK_BYTES = 64  # 256 trits * 2 bits
TQ1_BLOCK_BYTES = 52  # reading R5
TQ1_GROUPS = 51       # full five-trit groups per block (255 trits)


# --------------------------------------------------------------------------
# a1: absmean scale  [TLS "The model" step 1; SPC "Architecture"]
# --------------------------------------------------------------------------
def abs_sum_rn64(W: np.ndarray) -> float:
    """RN64(sum |W|): the exact sum of the absolute values, rounded once to
    the nearest double.

    math.fsum (Shewchuk's exact partials) returns the correctly rounded sum
    of its arguments; every float32 |w| is exactly a double, so this is the
    plain definition of reading R1 with no reduction order in it.  The values
    are fed in chunks only to bound memory; fsum sees one stream.
    """
    a = np.abs(np.ascontiguousarray(W, dtype=np.float32).reshape(-1))
    chunk = 1 << 22
    return math.fsum(itertools.chain.from_iterable(
        a[i:i + chunk].astype(np.float64).tolist() for i in range(0, a.size, chunk)))


def absmean_gamma(W: np.ndarray, eps: float) -> np.float32:
    """gamma = eps + mean|W| over the whole matrix, with readings R1.

    Returns NaN when W holds a non-finite value.
    """
    a = np.ascontiguousarray(W, dtype=np.float32)
    if a.size == 0 or not np.all(np.isfinite(a)):
        return np.float32(np.nan)
    s64 = abs_sum_rn64(a)                   # RN64(S)
    mean64 = s64 / float(a.size)            # IEEE double division
    g64 = mean64 + float(np.float32(eps))   # IEEE double addition
    return np.float32(g64)                  # round to nearest float32


# --------------------------------------------------------------------------
# a2: ternarize  [TLS "The model" step 2; SPC "Architecture"]
# --------------------------------------------------------------------------
def ternarize(W: np.ndarray, gamma) -> np.ndarray:
    """trits = round(clip(W / gamma, -1, 1)) in {-1, 0, 1}, reading R2."""
    a = np.ascontiguousarray(W, dtype=np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        x = a / np.float32(gamma)             # float32 / float32, IEEE RN
    x = np.where(np.isnan(x), np.float32(0.0), x)   # NaN quotient -> trit 0 (R2)
    x = np.clip(x, np.float32(-1.0), np.float32(1.0))
    return np.rint(x).astype(np.int8)         # rint: half to even


def absmean_ternarize(W: np.ndarray, eps: float = 1e-6):
    g = absmean_gamma(W, eps)
    return ternarize(W, g), g


# --------------------------------------------------------------------------
# block scales  [TLS "Fast inference on CPUs": one 16-bit scale per block]
# --------------------------------------------------------------------------
def block_scales_fp16(scales, N: int, K: int) -> np.ndarray:
    """fp16 scale plane d[N][K/256] from one scale or one per block (R6)."""
    s = np.asarray(scales, dtype=np.float32).reshape(-1)
    nb = K // BLOCK
    if s.size == 1:
        s = np.full(N * nb, s[0], dtype=np.float32)
    assert s.size == N * nb
    return s.astype(np.float16).reshape(N, nb)


# --------------------------------------------------------------------------
# a3: TQ2 pack / unpack  [TLS "2 bits per weight"; TriRun storage line]
# --------------------------------------------------------------------------
def invalid_trit_count(trits) -> int:
    """Number of input values outside {-1, 0, 1} (packed as 0, reading R7)."""
    t = np.asarray(trits, dtype=np.int64)
    return int(np.count_nonzero((t < -1) | (t > 1)))


def _valid_trits(trits) -> np.ndarray:
    t = np.asarray(trits, dtype=np.int64)
    return np.where((t < -1) | (t > 1), 0, t)


def pack_tq2(trits: np.ndarray, scales):
    """Return (qs uint8[N][K/4], d fp16[N][K/256]); reading R3."""
    t = _valid_trits(trits)
    N, K = t.shape
    assert K % BLOCK == 0
    dp = (t + 1).reshape(N, K // 4, 4)                 # d' = d + 1 in {0,1,2}
    qs = np.zeros((N, K // 4), dtype=np.int64)
    for j in range(4):
        qs += dp[:, :, j] << (2 * j)
    return qs.astype(np.uint8), block_scales_fp16(scales, N, K)


def unpack_tq2(qs: np.ndarray, N: int, K: int):
    """Return (trits int8[N][K], invalid_count): d' = (b >> 2j) & 3, t = d'-1."""
    b = np.asarray(qs, dtype=np.int64).reshape(N, K // 4)
    fields = np.stack([(b >> (2 * j)) & 3 for j in range(4)], axis=-1)
    invalid = int(np.count_nonzero(fields == 3))
    return (fields - 1).reshape(N, K).astype(np.int8), invalid


# --------------------------------------------------------------------------
# a4: TQ1 pack / unpack  [TLS "1.6 bits per weight"]
# --------------------------------------------------------------------------
def tq1_encode_digits(digits) -> int:
    """Five base-3 digits (first = most significant, R4) -> one byte.

    N5 is the base-3 number; the byte is floor((N5 * 2**8 + 242) / 243).
    """
    n5 = 0
    for dgt in digits:
        n5 = 3 * n5 + int(dgt)
    return (n5 * 256 + 242) // 243


def tq1_decode_inverse(byte: int):
    """Inverse-formula decoder: N5 = floor(243*b/256), digits by div/mod 3."""
    n5 = (243 * int(byte)) // 256
    out = []
    for p in (81, 27, 9, 3, 1):
        out.append(n5 // p)
        n5 %= p
    return out


def encode_kp(n: int, k: int, p: int) -> int:
    """General k-trits-in-p-bits rescale: floor((n * 2**p + 3**k - 1) / 3**k)."""
    return (n * (1 << p) + 3 ** k - 1) // 3 ** k


def pack_tq1(trits: np.ndarray, scales):
    """Return (qs uint8[N][(K/256)*52], d fp16[N][K/256]); readings R4, R5."""
    t = _valid_trits(trits)
    N, K = t.shape
    assert K % BLOCK == 0
    nb = K // BLOCK
    dp = (t + 1).reshape(N, nb, BLOCK)
    groups = dp[:, :, : 5 * TQ1_GROUPS].reshape(N, nb, TQ1_GROUPS, 5)
    last = np.concatenate(
        [dp[:, :, 5 * TQ1_GROUPS:], np.ones((N, nb, 4), dtype=np.int64)], axis=-1
    )[:, :, None, :]
    allg = np.concatenate([groups, last], axis=2)          # [N][nb][52][5]
    n5 = np.zeros(allg.shape[:3], dtype=np.int64)
    for j in range(5):
        n5 = 3 * n5 + allg[..., j]
    qs = (n5 * 256 + 242) // 243
    return qs.reshape(N, nb * TQ1_BLOCK_BYTES).astype(np.uint8), \
        block_scales_fp16(scales, N, K)


def unpack_tq1(qs: np.ndarray, N: int, K: int):
    """Return (trits int8[N][K], invalid_count) via the inverse formula."""
    nb = K // BLOCK
    b = np.asarray(qs, dtype=np.int64).reshape(N, nb, TQ1_BLOCK_BYTES)
    n5 = (243 * b) // 256
    digits = []
    rem = n5.copy()
    for p in (81, 27, 9, 3, 1):
        digits.append(rem // p)
        rem = rem % p
    dig = np.stack(digits, axis=-1)                          # [N][nb][52][5]
    reenc = (n5 * 256 + 242) // 243
    bad = reenc != b
    bad[:, :, -1] |= np.any(dig[:, :, -1, 1:] != 1, axis=-1)  # padding (R7)
    invalid = int(np.count_nonzero(bad))
    body = dig[:, :, :TQ1_GROUPS, :].reshape(N, nb, 5 * TQ1_GROUPS)
    lastt = dig[:, :, TQ1_GROUPS, 0:1]
    t = np.concatenate([body, lastt], axis=-1) - 1
    return t.reshape(N, K).astype(np.int8), invalid


def unpack(fmt: str, qs, N: int, K: int):
    return unpack_tq2(qs, N, K) if fmt == "tq2" else unpack_tq1(qs, N, K)


def pack(fmt: str, trits, scales):
    return pack_tq2(trits, scales) if fmt == "tq2" else pack_tq1(trits, scales)


# --------------------------------------------------------------------------
# a6: ternary GEMM  [TLS "The model" step 3; "TriRun" compute line]
# --------------------------------------------------------------------------
def gemm_f64(X: np.ndarray, trits: np.ndarray, d: np.ndarray,
             rows=None) -> np.ndarray:
    """Y[m][n] = sum_b d[n][b] * sum_{k in block b} X[m][k] * t[n][k], float64.

    X is (M, K) fp16, trits (N, K) int8, d (N, K/256) fp16.  ``rows``
    optionally restricts the output to the listed n (for sampled checks).
    The result is NOT rounded to fp16 (compare before rounding).
    """
    Xd = np.asarray(X, dtype=np.float64)
    M, K = Xd.shape
    t = np.asarray(trits)
    dd = np.asarray(d, dtype=np.float64)
    if rows is not None:
        t = t[np.asarray(rows)]
        dd = dd[np.asarray(rows)]
    Nr = t.shape[0]
    nb = K // BLOCK
    Y = np.zeros((M, Nr), dtype=np.float64)
    for b in range(nb):
        sl = slice(b * BLOCK, (b + 1) * BLOCK)
        part = Xd[:, sl] @ t[:, sl].astype(np.float64).T     # (M, Nr)
        Y += part * dd[:, b][None, :]
    return Y


def gemm_packed_f64(fmt: str, X, qs, d, N: int, K: int, rows=None):
    """Same as gemm_f64, unpacking the weights with this module's decoder."""
    if rows is not None:
        rows = np.asarray(rows)
        per_row = qs.reshape(N, -1)[rows]
        t, _ = unpack(fmt, per_row, len(rows), K)
        return gemm_f64(X, t, np.asarray(d).reshape(N, -1)[rows])
    t, _ = unpack(fmt, qs, N, K)
    return gemm_f64(X, t, d)


def gemm_tolerance(X, d, y_ref, rows=None) -> np.ndarray:
    """Allowed |y - y_ref|: 1e-3 * gamma_n * sum_k |x_mk| + 2**-10 * |y_ref|.

    With per-block scales gamma_n is max_b d[n][b] (the largest scale that
    multiplies any product of output n).
    """
    Xd = np.abs(np.asarray(X, dtype=np.float64)).sum(axis=1)       # (M,)
    dd = np.asarray(d, dtype=np.float64)
    if rows is not None:
        dd = dd[np.asarray(rows)]
    g = np.abs(dd).max(axis=1)                                       # (N,)
    return 1e-3 * Xd[:, None] * g[None, :] + 2.0 ** -10 * np.abs(y_ref)


# --------------------------------------------------------------------------
# a7 (next row): gated feed-forward unit  [TLS "The model": the MLP is a
# SwiGLU over two ternary projections]
# --------------------------------------------------------------------------
def silu_f64(g) -> np.ndarray:
    """silu(g) = g / (1 + e^-g) = g * sigmoid(g), float64, stable for large |g|."""
    g = np.asarray(g, dtype=np.float64)
    e = np.exp(-np.abs(g))
    sig = np.where(g >= 0, 1.0 / (1.0 + e), e / (1.0 + e))
    return g * sig


def swiglu_f64(X, trits_gate, d_gate, trits_up, d_up):
    """Y[m][f] = silu(G[m][f]) * U[m][f] with G, U the two ternary products
    (gemm_f64, not rounded).  Returns (Y, G, U)."""
    G = gemm_f64(X, trits_gate, d_gate)
    U = gemm_f64(X, trits_up, d_up)
    return silu_f64(G) * U, G, U


def swiglu_tolerance(X, d_gate, d_up, G, U) -> np.ndarray:
    """Allowed |y - y_ref| for the fused SwiGLU output.

    Each product may be off by its GEMM tolerance T (gemm_tolerance) and, on
    paths that store it, by fp16 rounding of the product (2^-11 relative);
    silu has slope at most 1.0999 (attained near g = 2.4), so
    |silu(g') u' - silu(g) u| <= 1.1 T_g (|u| + T_u) + |silu(g)| T_u, plus
    2^-10 |y| for the fp32 arithmetic and the fp16 rounding of y.
    """
    Tg = gemm_tolerance(X, d_gate, G)
    Tu = gemm_tolerance(X, d_up, U)
    Tg = Tg + 2.0 ** -11 * (np.abs(G) + Tg)
    Tu = Tu + 2.0 ** -11 * (np.abs(U) + Tu)
    Y = silu_f64(G) * U
    return 1.1 * Tg * (np.abs(U) + Tu) + np.abs(silu_f64(G)) * Tu + 2.0 ** -10 * np.abs(Y)


# --------------------------------------------------------------------------
# size identities  [TLS "2 bits per weight", "1.6 bits per weight",
# "Fast inference on CPUs"]
# --------------------------------------------------------------------------
def storage_bits_per_weight(fmt: str) -> float:
    """Stored bits per weight including the fp16 block scale."""
    per_block = (TQ2_BLOCK_BYTES if fmt == "tq2" else TQ1_BLOCK_BYTES) + 2
    return per_block * 8 / BLOCK


def packed_row_bytes(fmt: str, K: int) -> int:
    nb = K // BLOCK
    return nb * (TQ2_BLOCK_BYTES if fmt == "tq2" else TQ1_BLOCK_BYTES)
