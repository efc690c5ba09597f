"""GPU parity of the decode-step kernels (RMSNorm, RoPE table, QK-Norm + RoPE
with cache append, grouped-query attention) and of a whole ternary block's
decode step against the float64 oracle (oracle/decode_oracle.py), through the
C ABI.

Tolerances (each derived from where the product rounds):
* every kernel computes in fp32 from fp16 inputs and rounds once to fp16, so
  an output may differ from the oracle's correctly rounded value by one fp16
  step: |y - y_ref| <= 2^-10 |y_ref| + 2^-24 (RMSNorm, q, k);
* attention sums softmax-weighted values in fp32 over up to 2^16 positions
  (relative error well under 2^-16 of max|V|) before one fp16 rounding:
  |o - o_ref| <= 2^-10 |o_ref| + 2^-14 max|V|;
* the block chains nine rounding points; each may flip one fp16 step, and
  the ternary products damp an input step (|sum t x| << sum |x|), so the
  output stays within a few steps of the residual stream's magnitude:
  |out - out_ref| <= 2^-9 (|out_ref| + rms(out_ref)), and likewise the new
  cache entries."""
import numpy as np
import pytest
import torch

import bit_mixed_precision_tri_b200 as tri
from bit_mixed_precision_tri_b200 import decode as dec
from bit_mixed_precision_tri_b200 import inputs
from oracle import decode_oracle as D
from oracle import tri_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _h(a):
    return torch.from_numpy(np.asarray(a, dtype=np.float16)).to(DEV)


def _np(t):
    return t.float().cpu().numpy().astype(np.float64)


def _rng(seed):
    return np.random.default_rng(seed)


def _one_step_close(y, ref):
    assert np.all(np.abs(y - ref) <= 2.0 ** -10 * np.abs(ref) + 2.0 ** -24), np.max(np.abs(y - ref))


@pytest.mark.parametrize("M,Dm", [(1, 8), (3, 1024), (2, 8192), (5, 2056)])
@pytest.mark.parametrize("residual", [False, True])
def test_rmsnorm_vs_oracle(M, Dm, residual):
    rng = _rng(M * Dm + residual)
    x = D.rn16(rng.standard_normal((M, Dm)) * 3)
    r = D.rn16(rng.standard_normal((M, Dm)))
    g = D.rn16(rng.uniform(0.5, 1.5, Dm))
    if residual:
        y, h = dec.rmsnorm(_h(x), _h(g), r=_h(r))
        h_ref = D.residual_f16(x, r)
        assert np.array_equal(_np(h), h_ref)
        _one_step_close(_np(y), D.rmsnorm_f64(h_ref, g))
    else:
        y = dec.rmsnorm(_h(x), _h(g))
        _one_step_close(_np(y), D.rmsnorm_f64(x, g))


def test_rmsnorm_zero_row_and_tiny_values():
    x = np.zeros((2, 256))
    x[1, :] = 6e-8                                       # fp16 subnormal
    g = np.ones(256)
    y = _np(dec.rmsnorm(_h(x), _h(g)))
    _one_step_close(y, D.rmsnorm_f64(D.rn16(x), g))
    assert np.all(y[0] == 0)


def test_rope_table_vs_oracle():
    Lmax = 5000
    cs = dec.rope_table(Lmax, DEV).cpu().numpy().astype(np.float64)
    a = D.rope_angles_f64(np.arange(Lmax), 128)
    assert np.max(np.abs(cs[..., 0] - np.cos(a))) <= 2.0 ** -24
    assert np.max(np.abs(cs[..., 1] - np.sin(a))) <= 2.0 ** -24


def _qkv_case(M, H, Hkv, Lmax, seed):
    rng = _rng(seed)
    qkv = D.rn16(rng.standard_normal((M, (H + 2 * Hkv) * 128)) * 2)
    gq = D.rn16(rng.uniform(0.5, 1.5, 128))
    gk = D.rn16(rng.uniform(0.5, 1.5, 128))
    kc = D.rn16(rng.standard_normal((M, Hkv, Lmax, 128)))
    vc = D.rn16(rng.standard_normal((M, Hkv, Lmax, 128)))
    return qkv, gq, gk, kc, vc


@pytest.mark.parametrize("M,H,Hkv,Lmax,pos", [(1, 1, 1, 1, [0]), (3, 8, 2, 64, [0, 5, 63]),
                                               (2, 64, 8, 4096, [4095, 1234]), (4, 6, 3, 300, [7, 7, 299, 0])])
def test_qknorm_rope_vs_oracle(M, H, Hkv, Lmax, pos):
    qkv, gq, gk, kc, vc = _qkv_case(M, H, Hkv, Lmax, 10 + M + H)
    pos = np.array(pos)
    cs = dec.rope_table(Lmax, DEV)
    kct, vct = _h(kc), _h(vc)
    q = dec.qknorm_rope(_h(qkv), torch.from_numpy(pos.astype(np.int32)).to(DEV), _h(gq), _h(gk), cs, kct, vct, H, Hkv)
    q_ref, k_ref, v_ref = D.qknorm_rope_f64(qkv, pos, gq, gk, H, Hkv, 128)
    _one_step_close(_np(q), q_ref)
    kg, vg = _np(kct), _np(vct)
    for m in range(M):
        _one_step_close(kg[m, :, pos[m]], k_ref[m])
        assert np.array_equal(vg[m, :, pos[m]], v_ref[m])
        kg[m, :, pos[m]] = kc[m, :, pos[m]]
        vg[m, :, pos[m]] = vc[m, :, pos[m]]
    assert np.array_equal(kg, kc) and np.array_equal(vg, vc)    # nothing else written


def _attn_close(o, ref, Vc):
    tol = 2.0 ** -10 * np.abs(ref) + 2.0 ** -14 * np.max(np.abs(Vc))
    assert np.all(np.abs(o - ref) <= tol), np.max(np.abs(o - ref) - tol)


@pytest.mark.parametrize("M,H,Hkv,Lmax,pos,max_len", [
    (1, 8, 1, 1, [0], 1),                    # one position: the value itself
    (3, 16, 2, 2000, [0, 100, 1999], 2000),  # ragged lengths over several tiles and splits
    (2, 64, 8, 4096, [4095, 3000], 4096),    # 70B-like heads, full context
    (16, 64, 8, 1024, list(range(16)), 16),  # short contexts for a batch of 16
    (2, 4, 4, 700, [650, 63], 651),          # one query head per key/value head
])
def test_attention_vs_oracle(M, H, Hkv, Lmax, pos, max_len):
    rng = _rng(M * 1000 + H + Lmax)
    q = D.rn16(rng.standard_normal((M, H, 128)))
    Kc = D.rn16(rng.standard_normal((M, Hkv, Lmax, 128)))
    Vc = D.rn16(rng.standard_normal((M, Hkv, Lmax, 128)))
    pos = np.array(pos)
    o = dec.attention_decode(_h(q), _h(Kc), _h(Vc), torch.from_numpy(pos.astype(np.int32)).to(DEV), max_len)
    _attn_close(_np(o), D.attention_decode_f64(q, Kc, Vc, pos), Vc)


def test_attention_ignores_positions_past_pos_and_reads_its_group():
    M, H, Hkv, Lmax = 1, 8, 2, 256
    Kc = np.zeros((M, Hkv, Lmax, 128))
    Vc = np.zeros((M, Hkv, Lmax, 128))
    Vc[0, 0, :10] = 1.0
    Vc[0, 1, :10] = 2.0
    Vc[0, :, 10:] = 60000.0                                # beyond pos: must not count
    o = _np(dec.attention_decode(_h(np.ones((M, H, 128))), _h(Kc), _h(Vc),
                                 torch.tensor([9], dtype=torch.int32, device=DEV), 256)).reshape(H, 128)
    assert np.array_equal(o[:4], np.ones((4, 128))) and np.array_equal(o[4:], np.full((4, 128), 2.0))


# ---------------------------------------------------------------- whole block
def _block(Dm, F, H, Hkv, seed, fmt="tq2"):
    w = {}
    shapes = {"qkv": ((H + 2 * Hkv) * 128, Dm), "o": (Dm, H * 128), "gate": (F, Dm), "up": (F, Dm), "down": (Dm, F)}
    for i, (name, (n, k)) in enumerate(shapes.items()):
        t = inputs.random_trits(n, k, 0.31, seed + i).numpy()
        w[name] = (t, np.float32(0.0159))
    rng = _rng(seed)
    for name, n in (("g_attn", Dm), ("g_mlp", Dm), ("gq", 128), ("gk", 128)):
        w[name] = D.rn16(rng.uniform(0.5, 1.5, n))
    return w


def _run_block(Dm, F, H, Hkv, M, Lmax, pos, seed, fmt="tq2"):
    w = _block(Dm, F, H, Hkv, seed, fmt)
    rng = _rng(seed + 100)
    x = D.rn16(rng.standard_normal((M, Dm)))
    Kc = D.rn16(rng.standard_normal((M, Hkv, Lmax, 128)))
    Vc = D.rn16(rng.standard_normal((M, Hkv, Lmax, 128)))
    wt = {k: ((torch.from_numpy(v[0]), torch.tensor([float(v[1])], dtype=torch.float32)) if isinstance(v, tuple)
              else _h(v)) for k, v in w.items()}
    blk = dec.DecodeBlock(wt, Dm, H, Hkv, F, M, Lmax, DEV, fmt=fmt)
    blk.kcache.copy_(_h(Kc))
    blk.vcache.copy_(_h(Vc))
    pos = np.array(pos)
    out = _np(blk.step(_h(x), torch.from_numpy(pos.astype(np.int32)).to(DEV), int(pos.max()) + 1))
    wo = {k: ((v[0], O.block_scales_fp16(v[1], *v[0].shape)) if isinstance(v, tuple) else v) for k, v in w.items()}
    Kr, Vr = Kc.copy(), Vc.copy()
    ref, mid = D.decode_block_f64(x, pos, Kr, Vr, wo, H, Hkv, 128)
    tol = 2.0 ** -9 * (np.abs(ref) + np.sqrt(np.mean(ref ** 2)))
    assert np.all(np.abs(out - ref) <= tol), np.max(np.abs(out - ref) - tol)
    kg = _np(blk.kcache)
    for m in range(M):
        kref = mid["k"][m]
        ktol = 2.0 ** -9 * (np.abs(kref) + np.sqrt(np.mean(kref ** 2)))
        assert np.all(np.abs(kg[m, :, pos[m]] - kref) <= ktol)
    return blk


@pytest.mark.parametrize("fmt", ["tq2", "tq1"])
@pytest.mark.parametrize("M,pos", [(1, [0]), (2, [3, 40]), (5, [63, 0, 17, 17, 5])])
def test_decode_block_vs_oracle_small(fmt, M, pos):
    _run_block(512, 1024, 4, 2, M, 64, pos, 50 + M, fmt)


def test_decode_block_vs_oracle_70b_shapes():
    """One decode step of a block with the 70B-like shapes (D 8192, 64 query
    heads, 8 key/value heads, F 28672) for one sequence at position 1000."""
    _run_block(8192, 28672, 64, 8, 1, 1024, [1000], 70)


def test_decode_abi_rejects_bad_arguments():
    L = tri._lib.lib()
    x = torch.zeros(2, 64, dtype=torch.float16, device=DEV)
    g = torch.zeros(64, dtype=torch.float16, device=DEV)
    assert L.tri_rmsnorm(x.data_ptr(), None, g.data_ptr(), None, x.data_ptr(), 2, 12, 1e-5, None) == 2
    assert L.tri_rmsnorm(x.data_ptr(), x.data_ptr(), g.data_ptr(), None, x.data_ptr(), 2, 64, 1e-5, None) == 1
    assert L.tri_rmsnorm(x.data_ptr() + 2, None, g.data_ptr(), None, x.data_ptr(), 2, 64, 1e-5, None) == 3
    assert L.tri_rope_table(x.data_ptr(), 4, 64, 5e5, None) == 2
    assert L.tri_attention_decode_workspace_bytes(1, 16, 1, 10) == 0          # 16 query heads per group
    assert L.tri_attention_decode(x.data_ptr(), x.data_ptr(), x.data_ptr(), x.data_ptr(), x.data_ptr(),
                                  1, 8, 1, 16, 17, None, 0, None) == 2       # max_len > Lmax
