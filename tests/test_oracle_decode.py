"""Pins for the decode-step oracle (oracle/decode_oracle.py) against closed
forms, invariants and hand-computed values, so that a dropped term, a wrong
sign, index or pairing fails one of them.  CPU only."""
import math

import numpy as np
import pytest

from oracle import decode_oracle as D
from oracle import tri_oracle as T


# ---------------------------------------------------------------- RMSNorm (D14)
def test_rmsnorm_hand_example():
    y = D.rmsnorm_f64(np.array([[3.0, 4.0]]), np.array([1.0, 1.0]), eps=0.0)
    r = math.sqrt((9.0 + 16.0) / 2.0)
    assert np.allclose(y, [[3.0 / r, 4.0 / r]], rtol=0, atol=1e-15)


def test_rmsnorm_constant_vector_closed_form():
    c, eps = -0.25, 1e-5
    y = D.rmsnorm_f64(np.full((1, 64), c), np.full(64, 2.0), eps=eps)
    assert np.allclose(y, 2.0 * c / math.sqrt(c * c + eps), rtol=1e-15)


def test_rmsnorm_scale_invariance_and_unit_rms():
    x = np.random.default_rng(1).standard_normal((3, 128))
    g = np.ones(128)
    assert np.allclose(D.rmsnorm_f64(x, g, 0.0), D.rmsnorm_f64(7.5 * x, g, 0.0), rtol=1e-13)
    assert np.allclose(np.mean(D.rmsnorm_f64(x, g, 0.0) ** 2, axis=-1), 1.0, rtol=1e-13)


def test_rmsnorm_gain_is_per_feature():
    y = D.rmsnorm_f64(np.ones((1, 4)), np.array([1.0, 2.0, 3.0, 4.0]), eps=0.0)
    assert np.array_equal(y, [[1.0, 2.0, 3.0, 4.0]])


def test_residual_rounds_the_exact_sum_once():
    one = np.float16(1.0)
    # 1 + 2^-11 is a tie between 1 and 1 + 2^-10: even -> 1
    assert D.residual_f16(one, np.float16(2.0 ** -11)) == 1.0
    # 1 + 3 * 2^-12 is above the tie: 1 + 2^-10
    assert D.residual_f16(one, np.float16(3 * 2.0 ** -12)) == 1.0 + 2.0 ** -10


# ---------------------------------------------------------------- RoPE (D16)
def test_rope_position_zero_is_identity():
    x = np.random.default_rng(2).standard_normal((1, 3, 8))
    assert np.array_equal(D.rope_f64(x, np.array([0])), x)


def test_rope_hand_values():
    # dh = 2: one pair turned by p rad
    y = D.rope_f64(np.array([[1.0, 0.0]]), np.array([1]), theta=123.0)
    assert np.allclose(y, [[math.cos(1.0), math.sin(1.0)]], rtol=0, atol=1e-15)
    # dh = 4, theta = 16: pairs (x0, x2) at p, (x1, x3) at p / 4
    y = D.rope_f64(np.array([[1.0, 0.0, 0.0, 0.0]]), np.array([2]), theta=16.0)
    assert np.allclose(y, [[math.cos(2.0), 0.0, math.sin(2.0), 0.0]], atol=1e-15)
    y = D.rope_f64(np.array([[0.0, 1.0, 0.0, 0.0]]), np.array([2]), theta=16.0)
    assert np.allclose(y, [[0.0, math.cos(0.5), 0.0, math.sin(0.5)]], atol=1e-15)
    # the pages' theta: pair i = 1 of dh = 128 turns by p * 5e5^(-1/64)
    y = D.rope_f64(np.eye(128)[1][None, :], np.array([1000]))
    a = 1000 * 5.0e5 ** (-1.0 / 64)
    assert abs(y[0, 1] - math.cos(a)) < 1e-12 and abs(y[0, 65] - math.sin(a)) < 1e-12


def test_rope_keeps_pair_norms_and_depends_on_relative_position():
    rng = np.random.default_rng(3)
    q, k = rng.standard_normal((2, 1, 128))
    y = D.rope_f64(q[None], np.array([77]))[0]
    n0 = q[:, :64] ** 2 + q[:, 64:] ** 2
    assert np.allclose(y[:, :64] ** 2 + y[:, 64:] ** 2, n0, rtol=1e-12)
    d1 = np.sum(D.rope_f64(q[None], np.array([50]))[0] * D.rope_f64(k[None], np.array([20]))[0])
    d2 = np.sum(D.rope_f64(q[None], np.array([1030]))[0] * D.rope_f64(k[None], np.array([1000]))[0])
    assert abs(d1 - d2) < 1e-10


# ---------------------------------------------------------------- QK-Norm + RoPE (D15)
def test_qknorm_rope_hand_case():
    H, Hkv, dh = 1, 1, 4
    qkv = np.array([[2.0, 2.0, 2.0, 2.0, -1.0, -1.0, -1.0, -1.0, 0.5, 0.25, -0.5, 8.0]])
    q, k, v = D.qknorm_rope_f64(qkv, np.array([1]), np.ones(4), np.full(4, 0.5), H, Hkv, dh, eps=0.0,
                                theta=16.0)
    c1, s1, c4, s4 = math.cos(1.0), math.sin(1.0), math.cos(0.25), math.sin(0.25)
    # normed q = [1, 1, 1, 1]; pairs (0, 2) at angle 1, (1, 3) at angle 0.25
    assert np.array_equal(q[0, 0], D.rn16([c1 - s1, c4 - s4, s1 + c1, s4 + c4]))
    # normed k = -0.5 everywhere (gain 0.5)
    assert np.array_equal(k[0, 0], D.rn16(-0.5 * np.array([c1 - s1, c4 - s4, s1 + c1, s4 + c4])))
    assert np.array_equal(v[0, 0], [0.5, 0.25, -0.5, 8.0])


def test_qknorm_uses_each_heads_own_rms():
    H, Hkv, dh = 2, 1, 4
    qkv = np.concatenate([np.full(4, 3.0), np.full(4, 0.01), np.ones(4), np.ones(4)])[None]
    q, _, _ = D.qknorm_rope_f64(qkv, np.array([0]), np.ones(4), np.ones(4), H, Hkv, dh, eps=0.0)
    assert np.array_equal(q[0], np.ones((2, 4)))


# ---------------------------------------------------------------- attention (D17)
def test_attention_single_position_returns_v():
    M, H, Hkv, dh, Lmax = 1, 2, 1, 8, 4
    rng = np.random.default_rng(4)
    Kc, Vc = rng.standard_normal((2, M, Hkv, Lmax, dh))
    q = rng.standard_normal((M, H, dh))
    out = D.attention_decode_f64(q, Kc, Vc, np.array([0]))
    assert np.allclose(out.reshape(M, H, dh), Vc[:, [0, 0], 0], rtol=1e-15)


def test_attention_equal_keys_average_values_and_positions_past_pos_are_ignored():
    M, H, Hkv, dh, Lmax = 1, 1, 1, 8, 6
    rng = np.random.default_rng(5)
    Kc = np.tile(rng.standard_normal(dh), (M, Hkv, Lmax, 1))
    Vc = rng.standard_normal((M, Hkv, Lmax, dh))
    Vc[0, 0, 4:] = 1e6                                   # beyond pos: must not count
    out = D.attention_decode_f64(rng.standard_normal((M, H, dh)), Kc, Vc, np.array([3]))
    assert np.allclose(out[0], Vc[0, 0, :4].mean(axis=0), rtol=1e-13)


def test_attention_two_positions_logistic_weight_and_scale():
    dh = 16
    q = np.zeros((1, 1, dh)); q[0, 0, 0] = 2.0
    Kc = np.zeros((1, 1, 2, dh)); Kc[0, 0, 1, 0] = 3.0
    Vc = np.zeros((1, 1, 2, dh)); Vc[0, 0, 0, 1] = 1.0; Vc[0, 0, 1, 2] = 1.0
    out = D.attention_decode_f64(q, Kc, Vc, np.array([1]))[0]
    p1 = 1.0 / (1.0 + math.exp(-2.0 * 3.0 / math.sqrt(dh)))
    assert abs(out[2] - p1) < 1e-15 and abs(out[1] - (1 - p1)) < 1e-15


def test_attention_grouped_heads_read_their_group():
    M, H, Hkv, dh, Lmax = 1, 4, 2, 4, 1
    Kc = np.zeros((M, Hkv, Lmax, dh))
    Vc = np.zeros((M, Hkv, Lmax, dh))
    Vc[0, 0, 0] = 1.0
    Vc[0, 1, 0] = 2.0
    out = D.attention_decode_f64(np.ones((M, H, dh)), Kc, Vc, np.array([0])).reshape(H, dh)
    assert np.array_equal(out[:, 0], [1.0, 1.0, 2.0, 2.0])


# ---------------------------------------------------------------- block (D18-D20)
def _block_weights(D_, F, H, Hkv, dh, zero=(), seed=0):
    rng = np.random.default_rng(seed)
    shapes = {"qkv": ((H + 2 * Hkv) * dh, D_), "o": (D_, H * dh), "gate": (F, D_), "up": (F, D_),
              "down": (D_, F)}
    w = {}
    for name, (n, k) in shapes.items():
        t = np.zeros((n, k), np.int8) if name in zero else rng.integers(-1, 2, (n, k)).astype(np.int8)
        w[name] = (t, T.block_scales_fp16(np.float32(0.02), n, k))
    w["g_attn"] = D.rn16(rng.uniform(0.5, 1.5, D_))
    w["g_mlp"] = D.rn16(rng.uniform(0.5, 1.5, D_))
    w["gq"] = D.rn16(rng.uniform(0.5, 1.5, dh))
    w["gk"] = D.rn16(rng.uniform(0.5, 1.5, dh))
    return w


def test_block_with_zero_output_projections_returns_x_and_fills_the_cache():
    M, D_, F, H, Hkv, dh, Lmax = 2, 512, 512, 4, 2, 128, 8
    w = _block_weights(D_, F, H, Hkv, dh, zero=("o", "down"))
    x = D.rn16(np.random.default_rng(6).standard_normal((M, D_)))
    Kc = np.zeros((M, Hkv, Lmax, dh)); Vc = np.zeros((M, Hkv, Lmax, dh))
    pos = np.array([0, 5])
    out, mid = D.decode_block_f64(x, pos, Kc, Vc, w, H, Hkv, dh)
    assert np.array_equal(out, x)
    for m in range(M):
        assert np.array_equal(Kc[m, :, pos[m]], mid["k"][m])
        assert np.array_equal(Vc[m, :, pos[m]], mid["v"][m])
    # rotation keeps the normed key's pair norms: mean(k^2) = mean((gk * kn)^2) before rotation
    kraw = mid["qkv"][:, H * dh:(H + Hkv) * dh].reshape(M, Hkv, dh)
    ref = D.rmsnorm_f64(kraw, w["gk"])
    assert np.allclose(np.mean(mid["k"] ** 2, axis=-1), np.mean(ref ** 2, axis=-1), rtol=2e-3)


def test_block_with_all_zero_weights_is_the_identity():
    M, D_, F, H, Hkv, dh, Lmax = 1, 256, 256, 2, 1, 128, 4
    w = _block_weights(D_, F, H, Hkv, dh, zero=("qkv", "o", "gate", "up", "down"))
    x = D.rn16(np.random.default_rng(7).standard_normal((M, D_)))
    Kc = np.ones((M, Hkv, Lmax, dh)); Vc = np.ones((M, Hkv, Lmax, dh))
    out, mid = D.decode_block_f64(x, np.array([2]), Kc, Vc, w, H, Hkv, dh)
    assert np.array_equal(out, x)
    assert np.all(Kc[0, :, 2] == 0) and np.all(Vc[0, :, 2] == 0)
    assert np.all(Kc[0, :, :2] == 1)
