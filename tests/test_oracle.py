"""Pins for the CPU oracle: each check compares it with something other than
itself -- values printed on the pages, closed forms, independent library
routines, exact rational arithmetic (Fractions), brute force, and a second
decoder.

Pages: "Scaling Laws and Efficient Inference for Ternary Language Models"
(sections "The model", "Packing ternary weights", "Fast inference on CPUs",
"TriRun: ternary inference on GPUs") and "Spectra: Surprising Effectiveness of
Pretraining Ternary Language Models at Scale" (section "Architecture").
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

from oracle import tri_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _gold(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- a1 gamma
def _fraction_abs_sum(w):
    """Exact rational sum of |w| (Python Fractions), independent of math.fsum."""
    return sum((Fraction(abs(float(v))) for v in np.asarray(w, np.float32).reshape(-1)), Fraction(0))


@pytest.mark.parametrize("seed", range(6))
def test_abs_sum_is_the_correctly_rounded_exact_sum(seed):
    """RN64 of the exact sum: float(Fraction) rounds a rational correctly."""
    rng = np.random.default_rng(seed)
    n = 3000
    kind = seed % 3
    if kind == 0:
        w = rng.standard_normal(n) * 0.02
    elif kind == 1:   # very wide dynamic range, including denormals and zeros
        w = rng.standard_normal(n) * np.exp2(rng.integers(-149, 120, n).astype(np.float64))
        w[::17] = 0.0
    else:             # large and tiny values mixed: rounding depends on tiny ones
        w = np.where(rng.random(n) < 0.5, 1e30, 1e-30) * rng.standard_normal(n)
    w = w.astype(np.float32)
    assert O.abs_sum_rn64(w) == float(_fraction_abs_sum(w))


def test_abs_sum_denormal_and_powers():
    w = np.array([np.float32(2.0 ** -149), np.float32(2.0 ** -126), np.float32(-1.0),
                  np.float32(3.0), np.float32(2.0 ** 100)], dtype=np.float32)
    exact = Fraction(1, 1 << 149) + Fraction(1, 1 << 126) + 4 + (1 << 100)
    assert O.abs_sum_rn64(w) == float(exact) == 2.0 ** 100


def test_abs_sum_is_not_a_running_float_sum():
    """1 + 2^-53 + 2^-53: a left-to-right double sum loses both small terms
    (each addition is a tie, rounded to even), the exact sum is 1 + 2^-52."""
    w = np.array([1.0, 2.0 ** -53, -(2.0 ** -53)], dtype=np.float32)
    naive = 0.0
    for v in w.tolist():
        naive += abs(v)
    assert naive == 1.0
    assert O.abs_sum_rn64(w) == 1.0 + 2.0 ** -52
    # reversed order: a running sum would now be exact; the oracle is order-free
    assert O.abs_sum_rn64(w[::-1].copy()) == 1.0 + 2.0 ** -52
    # gamma from it: mean = (1 + 2^-52)/4 in double, then float32
    g = O.absmean_gamma(np.append(w, np.float32(0.0)), 0.0)
    assert g == np.float32((1.0 + 2.0 ** -52) / 4)


def test_gamma_hand_example():
    g = _gold("absmean_hand_example.json")
    W = np.array(g["W"], dtype=np.float32)
    gamma = O.absmean_gamma(W, g["eps"])
    # independent: exact rational mean of the float32 inputs, plus eps
    mean = sum(Fraction(float(abs(v))) for v in W) / len(W)
    assert abs(float(gamma) - float(mean + Fraction(float(np.float32(g["eps"]))))) < 1e-8
    assert abs(float(gamma) - g["gamma_approx"]) < g["gamma_abs_tol"] * 100
    assert O.ternarize(W, gamma).tolist() == g["trits"]


def test_gamma_and_zero_fraction_closed_form():
    """N(0, s) weights: mean|W| -> s*sqrt(2/pi); P(t = 0) = P(|z| < sqrt(2/pi)/2)."""
    rng = np.random.default_rng(7)
    s = 0.02
    W = (rng.standard_normal((1000, 1000)) * s).astype(np.float32)
    t, gamma = O.absmean_ternarize(W, 1e-6)
    expect_gamma = s * math.sqrt(2 / math.pi) + 1e-6
    assert abs(float(gamma) / expect_gamma - 1) < 3e-3
    p0 = math.erf(math.sqrt(2 / math.pi) / 2 / math.sqrt(2))
    assert abs(p0 - 0.3101) < 1e-3
    frac = float(np.mean(t == 0))
    assert abs(frac - p0) < 3e-3
    # +1 and -1 equally likely by symmetry
    assert abs(float(np.mean(t == 1)) - float(np.mean(t == -1))) < 3e-3


def test_gamma_nonfinite_is_nan():
    W = np.array([[0.1, np.inf]], dtype=np.float32)
    assert np.isnan(O.absmean_gamma(W, 1e-6))
    W = np.array([[0.1, np.nan]], dtype=np.float32)
    assert np.isnan(O.absmean_gamma(W, 1e-6))


# ---------------------------------------------------------------- a2 trits
def test_ternarize_tie_half_to_even():
    g = _gold("tie_case.json")
    W = np.array(g["W"], dtype=np.float32)
    gamma = O.absmean_gamma(W, g["eps"])
    assert float(gamma) == g["gamma"]
    assert O.ternarize(W, gamma).tolist() == g["trits_half_to_even"]


def test_ternarize_matches_scalar_python():
    """Elementwise pure-Python restatement: float32 quotient, clip, round()."""
    rng = np.random.default_rng(3)
    W = (rng.standard_normal(3000) * 0.02).astype(np.float32)
    W[:4] = [0.0, -0.0, 1e-30, -1e-30]
    gamma = O.absmean_gamma(W, 1e-6)
    got = O.ternarize(W, gamma)
    g = float(gamma)
    for w, t in zip(W.tolist(), got.tolist()):
        q = float(np.float32(w / g))   # double quotient of floats, rounded once to f32
        q = max(-1.0, min(1.0, q))
        assert round(q) == t           # Python round(): half to even


def test_ternarize_nan_quotient_is_zero_and_infinities_clip():
    """Reading R2 at its edges, by IEEE rules written out by hand:
    NaN / g is NaN -> 0; +-inf / g = +-inf -> clip -> +-1; with gamma = 0,
    0 / 0 is NaN -> 0 and w / 0 = +-inf -> +-1."""
    W = np.array([np.nan, np.inf, -np.inf, 0.3, -0.04, 0.0], dtype=np.float32)
    assert O.ternarize(W, np.float32(0.1)).tolist() == [0, 1, -1, 1, 0, 0]
    W = np.array([0.0, -0.0, 1e-30, -2.0], dtype=np.float32)
    assert O.ternarize(W, np.float32(0.0)).tolist() == [0, 0, 1, -1]
    # a NaN gamma (what absmean_gamma returns for non-finite W) zeroes every trit
    assert O.ternarize(np.array([1.0, -1.0, 0.5], np.float32), np.float32(np.nan)).tolist() == [0, 0, 0]


def test_invalid_trits_counted_and_packed_as_zero():
    """Reading R7 for packing: values outside {-1, 0, 1} are counted, packed
    as the zero weight (field value 1, i.e. d' = 0 + 1)."""
    t = np.zeros((2, 256), dtype=np.int8)
    t[0, :6] = [1, -1, 0, 2, -2, 127]
    t[1, 255] = -128
    assert O.invalid_trit_count(t) == 4
    assert O.invalid_trit_count(np.array([-1, 0, 1], np.int8)) == 0
    qs2, _ = O.pack_tq2(t, 1.0)
    # byte 0: fields 2,0,1,1 (t = 1,-1,0,0); byte 1: fields 1,1,1,1 (invalid -> 0, 127 -> 0, then zeros)
    assert int(qs2[0, 0]) == 2 | (0 << 2) | (1 << 4) | (1 << 6)
    assert int(qs2[0, 1]) == 0b01010101
    assert int(qs2[1, 63]) == 0b01010101
    qs1, _ = O.pack_tq1(t, 1.0)
    # first five-trit group of row 0: (1,-1,0,2->0,-2->0) -> digits 2,0,1,1,1 -> N5 = 162+0+9+3+1 = 175
    assert int(qs1[0, 0]) == (175 * 256 + 242) // 243
    # row 1, block's last byte: trit 255 (-128 -> 0) then four zero trits -> digits 1,1,1,1,1 -> N5 = 121
    assert int(qs1[1, 51]) == (121 * 256 + 242) // 243


# ---------------------------------------------------------------- a3 TQ2
def test_tq2_all_81_codes_round_trip():
    codes = list(itertools.product((-1, 0, 1), repeat=4))
    trits = np.zeros((1, 256), dtype=np.int8)
    seen = set()
    for c in codes:
        trits[0, :4] = c
        qs, d = O.pack_tq2(trits, 1.0)
        b = int(qs[0, 0])
        # page rule: d' = (b >> 2j) & 3 recovers d + 1
        assert [((b >> (2 * j)) & 3) - 1 for j in range(4)] == list(c)
        seen.add(b)
        back, bad = O.unpack_tq2(qs, 1, 256)
        assert back[0, :4].tolist() == list(c) and bad == 0
    assert len(seen) == 81
    assert all(((b >> (2 * j)) & 3) != 3 for b in seen for j in range(4))


def test_tq2_byte_example_and_word_layout():
    trits = np.zeros((1, 256), dtype=np.int8)
    trits[0, :4] = (-1, 0, 1, -1)                  # d' = 0, 1, 2, 0
    qs, _ = O.pack_tq2(trits, 1.0)
    assert int(qs[0, 0]) == 0b00_10_01_00
    # sixteen 2-bit weights per little-endian 32-bit word, weight j at bits 2j
    rng = np.random.default_rng(1)
    trits = rng.integers(-1, 2, (3, 512)).astype(np.int8)
    qs, _ = O.pack_tq2(trits, 1.0)
    words = qs.view("<u4")
    for r in range(3):
        for w in range(words.shape[1]):
            for j in range(16):
                assert ((int(words[r, w]) >> (2 * j)) & 3) - 1 == trits[r, 16 * w + j]


def test_tq2_invalid_field_counted():
    qs = np.full((2, 64), 0x55, dtype=np.uint8)    # all fields = 1 (zero trits)
    qs[0, 5] = 0b11_01_01_01                        # one field = 3
    qs[1, 9] = 0xFF                                 # four fields = 3
    t, bad = O.unpack_tq2(qs, 2, 256)
    assert bad == 5


def test_tq2_size_identity():
    N, K = 4, 1024
    qs, d = O.pack_tq2(np.zeros((N, K), np.int8), 0.5)
    assert qs.nbytes + d.nbytes == 66 * N * K // 256
    assert O.storage_bits_per_weight("tq2") == 2.0625
    assert abs(2 / math.log2(3) - 1 - 0.26) < 0.005        # "26% more bits"


# ---------------------------------------------------------------- a4 TQ1
def _mul_shift_decode(byte):
    """The page's SIMD decoder: multiply by 3, high byte = digit, low byte goes on."""
    out = []
    v = byte
    for _ in range(5):
        v = v * 3
        out.append(v >> 8)
        v &= 0xFF
    return out


def test_tq1_worked_example():
    g = _gold("tq1_worked_example.json")
    w = g["printed_on_page"]["weights"]
    trits = np.zeros((1, 256), np.int8)
    trits[0, :5] = w
    qs, _ = O.pack_tq1(trits, 1.0)
    assert int(qs[0, 0]) == g["derived_by_hand"]["byte"]
    digits = _mul_shift_decode(int(qs[0, 0]))
    assert digits == g["printed_on_page"]["decoded_digits_in_order"]
    assert [x - 1 for x in digits] == w
    assert O.tq1_decode_inverse(int(qs[0, 0])) == digits
    v = g["derived_by_hand"]["byte"]
    for prod, dig, rem in g["derived_by_hand"]["multiply_shift_trace"]:
        assert v * 3 == prod and (prod >> 8) == dig and (prod & 255) == rem
        v = rem


def test_tq1_all_243_patterns():
    """All 243 five-trit patterns: distinct bytes, and both decoders recover them."""
    seen = {}
    for digs in itertools.product(range(3), repeat=5):
        b = O.tq1_encode_digits(digs)
        assert 0 <= b <= 255
        assert _mul_shift_decode(b) == list(digs)
        assert O.tq1_decode_inverse(b) == list(digs)
        seen[b] = digs
    assert len(seen) == 243
    # the vectorised packer agrees with the scalar encoder, group by group
    trits = np.array([[d - 1 for d in digs] for digs in seen.values()], np.int8).reshape(-1)
    trits = np.concatenate([trits, np.zeros(255 * 5 - trits.size, np.int8)])  # 5 blocks of 255
    full = np.zeros((1, 5 * 256), np.int8)
    for blk in range(5):
        full[0, blk * 256: blk * 256 + 255] = trits[blk * 255:(blk + 1) * 255]
    qs, _ = O.pack_tq1(full, 1.0)
    back, bad = O.unpack_tq1(qs, 1, 5 * 256)
    assert bad == 0 and np.array_equal(back, full)


def test_tq1_decoders_agree_on_all_bytes_and_non_image():
    g = _gold("tq1_non_image_bytes.json")
    non_image = [b for b in range(256)
                 if all(((n * 256 + 242) // 243) != b for n in range(243))]
    assert non_image == g["non_image_bytes"]
    for b in range(256):
        assert _mul_shift_decode(b) == O.tq1_decode_inverse(b)
    qs = np.full((1, 52), O.tq1_encode_digits([1, 1, 1, 1, 1]), np.uint8)
    qs[0, 51] = O.tq1_encode_digits([1, 1, 1, 1, 1])
    for b in non_image:
        qs[0, 3] = b
        _, bad = O.unpack_tq1(qs, 1, 256)
        assert bad == 1
    qs[0, 3] = O.tq1_encode_digits([0, 1, 2, 1, 0])
    _, bad = O.unpack_tq1(qs, 1, 256)
    assert bad == 0
    qs[0, 51] = O.tq1_encode_digits([2, 0, 1, 1, 1])   # padding digit not the zero trit
    _, bad = O.unpack_tq1(qs, 1, 256)
    assert bad == 1


def test_tq1_block_layout_last_byte():
    trits = np.zeros((1, 512), np.int8)
    trits[0, 255] = -1
    trits[0, 511] = 1
    qs, _ = O.pack_tq1(trits, 1.0)
    assert qs.shape == (1, 104)
    assert int(qs[0, 51]) == O.tq1_encode_digits([0, 1, 1, 1, 1])
    assert int(qs[0, 103]) == O.tq1_encode_digits([2, 1, 1, 1, 1])
    back, bad = O.unpack_tq1(qs, 1, 512)
    assert bad == 0 and np.array_equal(back, trits)


def test_lossless_iff_rule():
    """k trits in p bits by rescaling is lossless iff 2^p > 3^k (brute force)."""
    for k in range(1, 7):
        for p in range(1, 12):
            codes = [O.encode_kp(n, k, p) for n in range(3 ** k)]
            injective = len(set(codes)) == 3 ** k and max(codes) < (1 << p)
            assert injective == ((1 << p) > 3 ** k), (k, p)
    assert O.encode_kp(176, 5, 8) == 186


def test_tq1_size_identities():
    assert 8 / 5 == 1.6
    assert abs(1.6 / math.log2(3) - 1 - 0.0095) < 0.0005   # "within 0.95%"
    assert O.storage_bits_per_weight("tq1") == 54 * 8 / 256
    qs, d = O.pack_tq1(np.zeros((3, 768), np.int8), 0.1)
    assert qs.nbytes == 3 * 3 * 52 and d.nbytes == 3 * 3 * 2


# ---------------------------------------------------------------- a6 GEMM
def _exact_gemm(X, trits, d):
    M, K = X.shape
    N = trits.shape[0]
    Y = [[Fraction(0)] * N for _ in range(M)]
    for m in range(M):
        for n in range(N):
            acc = Fraction(0)
            for b in range(K // 256):
                s = Fraction(0)
                for k in range(256 * b, 256 * b + 256):
                    t = int(trits[n, k])
                    if t:
                        s += t * Fraction(float(X[m, k]))
                acc += Fraction(float(d[n, b])) * s
            Y[m][n] = acc
    return Y


@pytest.mark.parametrize("M,N,K", [(1, 3, 256), (3, 5, 512), (2, 7, 768)])
def test_gemm_exact_rational_brute_force(M, N, K):
    rng = np.random.default_rng(M * 100 + N)
    X = rng.standard_normal((M, K)).astype(np.float16)
    trits = rng.integers(-1, 2, (N, K)).astype(np.int8)
    scales = rng.uniform(0.01, 0.05, (N, K // 256)).astype(np.float32)
    d = O.block_scales_fp16(scales, N, K)
    Y = O.gemm_f64(X, trits, d)
    E = _exact_gemm(X, trits, d)
    assert Y.shape == (M, N)
    for m in range(M):
        for n in range(N):
            assert abs(Y[m, n] - float(E[m][n])) <= 1e-12 * (1 + abs(float(E[m][n])))


def test_gemm_special_cases():
    rng = np.random.default_rng(11)
    M, N, K = 3, 4, 512
    X = rng.standard_normal((M, K)).astype(np.float16)
    d = O.block_scales_fp16(np.float32(0.0234), N, K)
    z = O.gemm_f64(X, np.zeros((N, K), np.int8), d)
    assert np.all(z == 0)
    ones = O.gemm_f64(X, np.ones((N, K), np.int8), d)
    rowsum = X.astype(np.float64).sum(axis=1) * float(d[0, 0])
    assert np.allclose(ones, rowsum[:, None], rtol=1e-13, atol=0)
    t = np.zeros((N, K), np.int8)
    t[2, 300] = -1
    single = O.gemm_f64(X, t, d)
    assert np.array_equal(single[:, 2], -float(d[2, 1]) * X[:, 300].astype(np.float64))
    assert np.all(single[:, [0, 1, 3]] == 0)


def test_gemm_packed_and_rows():
    rng = np.random.default_rng(5)
    M, N, K = 2, 9, 768
    X = rng.standard_normal((M, K)).astype(np.float16)
    trits = rng.integers(-1, 2, (N, K)).astype(np.int8)
    scales = rng.uniform(0.01, 0.05, (N, K // 256)).astype(np.float32)
    for fmt in ("tq2", "tq1"):
        qs, d = O.pack(fmt, trits, scales)
        full = O.gemm_packed_f64(fmt, X, qs, d, N, K)
        assert np.array_equal(full, O.gemm_f64(X, trits, d))
        rows = [0, 4, 8]
        part = O.gemm_packed_f64(fmt, X, qs, d, N, K, rows=rows)
        assert np.array_equal(part, full[:, rows])


def test_tolerance_formula_values():
    X = np.array([[1.0, -2.0] + [0.0] * 254], np.float16)
    d = np.array([[0.5]], np.float16)
    y = np.array([[4.0]])
    tol = O.gemm_tolerance(X, d, y)
    assert tol[0, 0] == 1e-3 * 3.0 * 0.5 + 4.0 / 1024


# ------------------------------------------------ planted mistakes are caught
def test_pins_catch_planted_mistakes():
    """Mutated copies of oracle steps (planted on the CPU) fail the pins above."""
    rng = np.random.default_rng(2)
    M, N, K = 2, 3, 512
    X = rng.standard_normal((M, K)).astype(np.float16)
    trits = rng.integers(-1, 2, (N, K)).astype(np.int8)
    d = O.block_scales_fp16(rng.uniform(0.01, 0.05, (N, K // 256)).astype(np.float32), N, K)
    E = np.array([[float(v) for v in row] for row in _exact_gemm(X, trits, d)])

    def wrong_block(Xa, t, dd):        # uses scale of block 0 everywhere
        return O.gemm_f64(Xa, t, np.repeat(dd[:, :1], dd.shape[1], axis=1))

    def transposed_sign(Xa, t, dd):    # sign flipped
        return -O.gemm_f64(Xa, t, dd)

    for bad in (wrong_block, transposed_sign):
        assert not np.allclose(bad(X, trits, d), E, rtol=1e-9)
    # LSB-first digit order would not reproduce the page's printed decode order
    digs = [2, 0, 1, 1, 2]
    lsd_first = O.tq1_encode_digits(list(reversed(digs)))
    assert _mul_shift_decode(lsd_first) != digs
    # a half-away-from-zero rounding fails the tie fixture
    g = _gold("tie_case.json")
    x = np.array(g["W"], np.float32)
    away = (np.sign(x) * np.floor(np.abs(np.clip(x, -1, 1)) + 0.5)).astype(np.int8)
    assert away.tolist() != g["trits_half_to_even"]


# ---------------------------------------------------------------- a7 SwiGLU
def test_silu_closed_forms():
    """silu(g) = g / (1 + e^-g): values fixed by the definition."""
    g = np.array([0.0, 1.0, -1.0, 2.0, 30.0, -40.0, -745.0])
    want = np.array([0.0, 1 / (1 + math.exp(-1)), -1 / (1 + math.exp(1)), 2 / (1 + math.exp(-2)),
                     30.0 / (1 + math.exp(-30)), -40.0 * math.exp(-40) / (1 + math.exp(-40)), -0.0])
    got = O.silu_f64(g)
    assert np.allclose(got, want, rtol=1e-15, atol=1e-300)
    assert abs(O.silu_f64(1.0) - 0.7310585786300049) < 1e-15     # sigmoid(1)
    assert np.all(np.isfinite(O.silu_f64(np.array([1e308, -1e308]))))


def test_swiglu_hand_example():
    """One row, one block: gate trits pick +x_0 - x_1, up trits sum x_0..x_3,
    so Y = silu(d_g (x0 - x1)) * d_u (x0 + x1 + x2 + x3)."""
    K = 256
    X = np.zeros((1, K), np.float16)
    X[0, :4] = [1.5, -0.5, 0.25, 2.0]
    tg = np.zeros((1, K), np.int8)
    tg[0, 0], tg[0, 1] = 1, -1
    tu = np.zeros((1, K), np.int8)
    tu[0, :4] = 1
    dg = np.array([[0.5]], np.float16)
    du = np.array([[0.25]], np.float16)
    Y, G, U = O.swiglu_f64(X, tg, dg, tu, du)
    g = 0.5 * (1.5 + 0.5)
    u = 0.25 * (1.5 - 0.5 + 0.25 + 2.0)
    assert G[0, 0] == g and U[0, 0] == u
    assert abs(Y[0, 0] - g / (1 + math.exp(-g)) * u) < 1e-15


def test_swiglu_zero_gate_and_tolerance_bounds():
    """An all-zero gate gives Y = 0 exactly; the tolerance is positive, and a
    planted error of 2x the tolerance in the gate product is rejected."""
    rng = np.random.default_rng(5)
    X = rng.standard_normal((3, 512)).astype(np.float16)
    tu = rng.integers(-1, 2, (16, 512)).astype(np.int8)
    du = np.full((16, 2), 0.03, np.float16)
    tg = np.zeros((16, 512), np.int8)
    Y, G, U = O.swiglu_f64(X, tg, du, tu, du)
    assert np.all(Y == 0.0)
    tg = rng.integers(-1, 2, (16, 512)).astype(np.int8)
    Y, G, U = O.swiglu_f64(X, tg, du, tu, du)
    tol = O.swiglu_tolerance(X, du, du, G, U)
    assert np.all(tol > 0)
    Tg = O.gemm_tolerance(X, du, G)
    bad = O.silu_f64(G + 4 * Tg + 1e-3) * U
    assert np.any(np.abs(bad - Y) > tol)
