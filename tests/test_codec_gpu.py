"""GPU parity of ternarization, packing and unpacking against the CPU oracle:
bit-exact gamma, trits, packed bytes, scales, decoded trits and invalid-code
counts, called through the C ABI."""
import numpy as np
import pytest
import torch

import bit_mixed_precision_tri_b200 as tri
from bit_mixed_precision_tri_b200 import inputs
from oracle import tri_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _gamma_bits(g):
    return np.float32(g).view(np.uint32)


@pytest.mark.parametrize("N,K,seed", [(256, 1024, 0), (1, 256, 1), (37, 768, 2), (300, 11008, 3),
                                      (1000, 4096, 4)])
def test_ternarize_bit_exact(N, K, seed):
    W = inputs.latent_weights(N, K, seed)
    t_ref, g_ref = O.absmean_ternarize(W.numpy(), 1e-6)
    t, g = tri.ternarize(W.to(DEV), 1e-6)
    assert _gamma_bits(g.item()) == _gamma_bits(g_ref)
    assert np.array_equal(t.cpu().numpy(), t_ref)


def test_ternarize_wide_range_and_ties():
    rng = np.random.default_rng(9)
    N, K = 64, 512
    W = (rng.standard_normal((N, K)) * np.exp2(rng.integers(-140, 100, (N, K)))).astype(np.float32)
    W[0, :8] = [0.0, -0.0, 2.0 ** -149, -(2.0 ** -149), 2.0 ** -126, 1.0, -1.0, 3e38]
    t_ref, g_ref = O.absmean_ternarize(W, 1e-6)
    t, g = tri.ternarize(torch.from_numpy(W).to(DEV), 1e-6)
    assert _gamma_bits(g.item()) == _gamma_bits(g_ref)
    assert np.array_equal(t.cpu().numpy(), t_ref)
    # exact tie: W/gamma = +-0.5 rounds to 0 (half to even)
    W = np.zeros((1, 256), np.float32)
    W[0, :4] = [2.0, 0.5, -0.5, -1.0]
    t_ref, g_ref = O.absmean_ternarize(W, 0.0)
    t, g = tri.ternarize(torch.from_numpy(W).to(DEV), 0.0)
    assert _gamma_bits(g.item()) == _gamma_bits(g_ref)
    assert np.array_equal(t.cpu().numpy(), t_ref)


def test_ternarize_degenerate():
    # all-zero W with eps = 0: gamma = 0, every quotient is NaN -> trit 0
    W = torch.zeros(4, 256)
    t, g = tri.ternarize(W.to(DEV), 0.0)
    assert g.item() == 0.0 and int(t.abs().sum()) == 0
    # non-finite weights: gamma NaN, wrapper raises, raw ABI gives zero trits
    W = inputs.latent_weights(8, 256, 5)
    W[3, 7] = float("inf")
    with pytest.raises(tri.TriError):
        tri.ternarize(W.to(DEV))
    t, g = tri.ternarize(W.to(DEV), check_finite=False)
    assert np.isnan(g.item()) and int(t.abs().sum()) == 0
    assert np.isnan(O.absmean_gamma(W.numpy(), 1e-6))


def test_absmean_large_matrix_bit_exact():
    """Full-size weight of the 70B-like block (gate projection 28672 x 8192)."""
    W = inputs.latent_weights(28672, 8192, 12)
    g_ref = O.absmean_gamma(W.numpy(), 1e-6)
    Wd = W.to(DEV)
    g = tri.absmean(Wd, 1e-6)
    assert _gamma_bits(g.item()) == _gamma_bits(g_ref)
    t, g2 = tri.ternarize(Wd, 1e-6)
    assert g2.item() == g.item()
    rows = np.random.default_rng(0).choice(28672, 64, replace=False)
    t_rows = t[torch.from_numpy(rows).to(DEV)].cpu().numpy()
    assert np.array_equal(t_rows, O.ternarize(W.numpy()[rows], g_ref))
    frac0 = float((t == 0).float().mean())
    assert abs(frac0 - 0.3101) < 2e-3


@pytest.mark.parametrize("fmt", ["tq2", "tq1"])
@pytest.mark.parametrize("N,K,per_block", [(1, 256, False), (19, 768, True), (256, 1024, False),
                                           (129, 11008, True)])
def test_pack_bit_exact(fmt, N, K, per_block):
    trits = inputs.random_trits(N, K, 0.4, 31 + N)
    scales = inputs.block_scales(N, K, 7) if per_block else torch.tensor([0.0234], dtype=torch.float32)
    qs_ref, d_ref = O.pack(fmt, trits.numpy(), scales.numpy())
    qs, d, inv = tri.pack(trits.to(DEV), scales.to(DEV), fmt, return_invalid=True)
    assert np.array_equal(qs.cpu().numpy(), qs_ref)
    assert np.array_equal(d.cpu().numpy().view(np.uint16), d_ref.view(np.uint16))
    assert int(inv.item()) == 0
    back, inv2 = tri.unpack(qs, N, K, fmt, return_invalid=True)
    assert np.array_equal(back.cpu().numpy(), trits.numpy()) and int(inv2.item()) == 0


@pytest.mark.parametrize("fmt", ["tq2", "tq1"])
def test_pack_counts_invalid_trits(fmt):
    trits = inputs.random_trits(8, 512, 0.3, 3)
    trits[2, 5] = 7
    trits[5, 511] = -2
    trits[7, 255] = 100
    qs_ref, _ = O.pack(fmt, trits.numpy(), np.float32(0.5))
    qs, d, inv = tri.pack(trits.to(DEV), torch.tensor([0.5]).to(DEV), fmt, return_invalid=True)
    assert int(inv.item()) == O.invalid_trit_count(trits.numpy()) == 3
    assert np.array_equal(qs.cpu().numpy(), qs_ref)


@pytest.mark.parametrize("fmt", ["tq2", "tq1"])
@pytest.mark.parametrize("N,K", [(3, 256), (50, 1024)])
def test_unpack_random_bytes_bit_exact(fmt, N, K):
    """Every byte value, valid or not, decodes like the oracle; counts agree."""
    nbytes = N * tri.packed_row_bytes(fmt, K)
    qs = inputs.random_bytes(nbytes, 17 + N).reshape(N, -1)
    t_ref, bad_ref = O.unpack(fmt, qs.numpy(), N, K)
    t, inv = tri.unpack(qs.to(DEV), N, K, fmt, return_invalid=True)
    assert np.array_equal(t.cpu().numpy(), t_ref)
    assert int(inv.item()) == bad_ref > 0


def test_tq1_all_243_codes_on_gpu():
    import itertools
    digs = np.array(list(itertools.product(range(3), repeat=5)), np.int8) - 1   # 243 x 5
    flat = digs.reshape(-1)
    N = 5
    trits = np.zeros((N, 256), np.int8)
    for r in range(N):
        chunk = flat[r * 255:(r + 1) * 255]
        trits[r, :chunk.size] = chunk
    qs_ref, _ = O.pack_tq1(trits, np.float32(1.0))
    qs, _ = tri.pack(torch.from_numpy(trits).to(DEV), torch.tensor([1.0]).to(DEV), "tq1")
    assert np.array_equal(qs.cpu().numpy(), qs_ref)
    assert len(set(qs_ref[:, :51].reshape(-1).tolist())) == 243
    assert np.array_equal(tri.unpack(qs, N, 256, "tq1").cpu().numpy(), trits)


def test_absmean_exponent_window_paths():
    """gamma bit-exact where the bins pass's per-warp exponent window has to
    move up many times (magnitudes growing along W), where it starts high and
    most later values fall below it (magnitudes shrinking), where warps start
    on zeros, and where most values of a step sit far below its largest."""
    rng = np.random.default_rng(17)
    n = 64 * 4096
    ramp = (rng.standard_normal(n) * np.exp2(np.linspace(-100, 100, n))).astype(np.float32)
    half_zero = np.zeros(n, np.float32)
    half_zero[n // 2:] = rng.standard_normal(n - n // 2).astype(np.float32) * 7
    spikes = (rng.standard_normal(n) * 1e-12).astype(np.float32)
    spikes[::37] = 1e30
    for w in (ramp, ramp[::-1].copy(), half_zero, spikes):
        W = w.reshape(64, 4096)
        g_ref = O.absmean_gamma(W, 1e-6)
        g = tri.absmean(torch.from_numpy(W).to(DEV), 1e-6)
        assert _gamma_bits(g.item()) == _gamma_bits(g_ref)
