"""GPU parity of the ternary GEMM against the FP64 CPU oracle, for every
kernel path, through the C ABI.  Bar (from the workload statement):
|y - y_ref| <= 1e-3 * gamma_n * sum_k |x_mk| + 2^-10 * |y_ref|, gamma_n the
largest block scale of output row n."""
import numpy as np
import pytest
import torch

import bit_mixed_precision_tri_b200 as tri
from bit_mixed_precision_tri_b200 import inputs
from oracle import tri_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
PATHS = {"simt": tri.PATH_SIMT, "i8": tri.PATH_I8, "mma": tri.PATH_MMA,
         "tcgen05": tri.PATH_TCGEN05}


def _supported(path, fmt, M, N, K):
    """Whether an explicit path serves this shape (the library answers)."""
    if path == tri.PATH_SIMT:
        return True
    X = torch.zeros(M, K, dtype=torch.float16, device=DEV)
    qs = torch.zeros(N, tri.packed_row_bytes(fmt, K), dtype=torch.uint8, device=DEV)
    d = torch.zeros(N, K // 256, dtype=torch.float16, device=DEV)
    try:
        tri.gemm(X, qs, d, N, K, fmt, path=path)
        return True
    except tri.TriError as e:
        if e.status == 7:
            return False
        raise


def _check(Y, X, trits, d, rows=None):
    y_ref = O.gemm_f64(X, trits, d)
    y = Y.float().cpu().numpy().astype(np.float64)
    if rows is not None:
        y = y[:, rows]
    tol = O.gemm_tolerance(X, d, y_ref)
    err = np.abs(y - y_ref)
    bad = err > tol
    assert not bad.any(), f"{bad.sum()} outputs out of tolerance; worst {(err - tol).max()}"
    assert np.all(np.isfinite(y))


def _case(M, N, K, seed, fmt, per_block=False, p_zero=None):
    if p_zero is None:
        W = inputs.latent_weights(N, K, seed)
        trits, g = O.absmean_ternarize(W.numpy(), 1e-6)
        scales = np.array([g], np.float32)
    else:
        trits = inputs.random_trits(N, K, p_zero, seed).numpy()
        scales = inputs.block_scales(N, K, seed + 1).numpy() if per_block else np.array([0.03], np.float32)
    qs, d = O.pack(fmt, trits, scales)
    X = inputs.activations(M, K, seed + 100).numpy()
    return X, trits, qs, d


SMALL = [(1, 256, 1024), (1, 1, 256), (2, 37, 768), (3, 300, 1024), (5, 1000, 512), (8, 64, 2048),
         (13, 129, 768), (16, 256, 4096), (16, 17, 256)]
MID = [(33, 256, 1024), (64, 256, 512), (100, 384, 768), (128, 512, 1024), (200, 640, 2048)]


@pytest.mark.parametrize("fmt", ["tq2", "tq1"])
@pytest.mark.parametrize("pname", list(PATHS))
@pytest.mark.parametrize("M,N,K", SMALL + MID)
def test_gemm_paths_vs_oracle(fmt, pname, M, N, K):
    path = PATHS[pname]
    if not _supported(path, fmt, M, N, K):
        pytest.skip(f"{pname} does not serve {fmt} M={M} N={N} K={K}")
    X, trits, qs, d = _case(M, N, K, 1000 + 7 * M + N, fmt)
    Y = tri.gemm(torch.from_numpy(X).to(DEV), torch.from_numpy(qs).to(DEV),
                 torch.from_numpy(d).to(DEV), N, K, fmt, path=path)
    _check(Y, X, trits, d)


@pytest.mark.parametrize("fmt", ["tq2", "tq1"])
@pytest.mark.parametrize("M", [1, 16, 128])
@pytest.mark.parametrize("p_zero", [0.3, 0.9])
def test_gemm_per_block_scales_and_sparsity(fmt, M, p_zero):
    N, K = 512, 4096
    X, trits, qs, d = _case(M, N, K, 20 + int(10 * p_zero), fmt, per_block=True, p_zero=p_zero)
    Y = tri.gemm(torch.from_numpy(X).to(DEV), torch.from_numpy(qs).to(DEV),
                 torch.from_numpy(d).to(DEV), N, K, fmt)
    _check(Y, X, trits, d)


@pytest.mark.parametrize("fmt", ["tq2", "tq1"])
def test_gemm_special_cases(fmt):
    M, N, K = 4, 96, 1024
    X = inputs.activations(M, K, 5).numpy()
    Xd = torch.from_numpy(X).to(DEV)
    for pname, path in PATHS.items():
        if not _supported(path, fmt, M, N, K):
            continue
        for kind in ("zero", "ones", "single"):
            trits = np.zeros((N, K), np.int8)
            if kind == "ones":
                trits[:] = 1
            elif kind == "single":
                trits[5, 700] = -1
            qs, d = O.pack(fmt, trits, np.float32(0.0234))
            Y = tri.gemm(Xd, torch.from_numpy(qs).to(DEV), torch.from_numpy(d).to(DEV), N, K, fmt,
                         path=path)
            _check(Y, X, trits, d)
            if kind == "single" and path == tri.PATH_SIMT:
                y = Y.float().cpu().numpy()
                exp = (-np.float64(d[5, 2]) * X[:, 700].astype(np.float64)).astype(np.float16)
                assert np.array_equal(y[:, 5].astype(np.float16), exp)
                assert np.all(np.delete(y, 5, axis=1) == 0)


def test_gemm_tiny_config_all_formats():
    """Tiny correctness case: W 256x1024 ~ N(0, 0.02) seed 0, X 1x1024 seed 1."""
    W = inputs.latent_weights(256, 1024, 0)
    X = inputs.activations(1, 1024, 1)
    for fmt in ("tq2", "tq1"):
        layer = tri.TernaryLinear.from_latent(W.to(DEV), fmt)
        Y = layer(X.to(DEV))
        t_ref, g_ref = O.absmean_ternarize(W.numpy(), 1e-6)
        _, d_ref = O.pack(fmt, t_ref, np.array([g_ref], np.float32))
        assert np.array_equal(layer.d.cpu().numpy().view(np.uint16), d_ref.view(np.uint16))
        _check(Y, X.numpy(), t_ref, d_ref)


@pytest.mark.parametrize("fmt", ["tq2", "tq1"])
@pytest.mark.parametrize("M", [1, 16, 256])
def test_gemm_full_size_sampled(fmt, M):
    """Largest layer shape (8192 x 28672): sampled output rows against the oracle,
    in the launch configuration the bench uses (AUTO path)."""
    N, K = 8192, 28672
    trits = inputs.random_trits(N, K, 0.31, 77)
    scale = torch.tensor([0.0159], dtype=torch.float32)
    qs, d = tri.pack(trits.to(DEV), scale.to(DEV), fmt)
    X = inputs.activations(M, K, 78)
    Y = tri.gemm(X.to(DEV), qs, d, N, K, fmt)
    rows = np.sort(np.random.default_rng(M).choice(N, 48, replace=False))
    rows[0], rows[-1] = 0, N - 1
    t_rows = trits.numpy()[rows]
    _, d_rows = O.pack(fmt, t_rows, scale.numpy())
    y_ref = O.gemm_f64(X.numpy(), t_rows, d_rows)
    y = Y.float().cpu().numpy()[:, rows].astype(np.float64)
    tol = O.gemm_tolerance(X.numpy(), d_rows, y_ref)
    assert np.all(np.abs(y - y_ref) <= tol)


def test_gemm_repeat_deterministic():
    M, N, K = 8, 4096, 4096
    X, trits, qs, d = _case(M, N, K, 4, "tq2")
    args = (torch.from_numpy(X).to(DEV), torch.from_numpy(qs).to(DEV), torch.from_numpy(d).to(DEV),
            N, K, "tq2")
    Y1 = tri.gemm(*args)
    Y2 = tri.gemm(*args)
    assert torch.equal(Y1, Y2)


@pytest.mark.parametrize("fmt", ["tq2", "tq1"])
@pytest.mark.parametrize("M,N,K", [(1, 65536, 1024), (2, 1000, 11008), (1, 129, 256), (2, 3, 512)])
def test_i8_path_shapes(fmt, M, N, K):
    """The integer path at shapes that exercise its work split: more units per
    CTA than block pairs per row (slot wrap), an odd number of blocks per row
    (a half-empty last pair), ragged row tiles and a grid smaller than the SMs."""
    X, trits, qs, d = _case(M, N, K, 300 + M + N % 97, fmt, per_block=True, p_zero=0.31)
    Y = tri.gemm(torch.from_numpy(X).to(DEV), torch.from_numpy(qs).to(DEV),
                 torch.from_numpy(d).to(DEV), N, K, fmt, path=tri.PATH_I8)
    _check(Y, X, trits, d)


@pytest.mark.parametrize("fmt", ["tq2", "tq1"])
@pytest.mark.parametrize("M", [1, 2])
def test_i8_path_activation_extremes(M, fmt):
    """Fixed-point activations: a block holding one value near the fp16 maximum
    among tiny ones (the quantisation step is set by the largest |x| of the
    block), an all-zero block, subnormal values and signed extremes."""
    N, K = 384, 2048
    X, trits, qs, d = _case(M, N, K, 41, fmt, per_block=True, p_zero=0.5)
    X = X.copy()
    X[:, 0] = 60000.0
    X[:, 1:256] = (np.random.default_rng(3).standard_normal((M, 255)) * 1e-3).astype(np.float16)
    X[:, 256:512] = 0.0
    X[:, 512:768] = np.float16(6e-8)
    X[:, 768] = -65504.0
    X[:, 769] = 65504.0
    Y = tri.gemm(torch.from_numpy(X).to(DEV), torch.from_numpy(qs).to(DEV),
                 torch.from_numpy(d).to(DEV), N, K, fmt, path=tri.PATH_I8)
    _check(Y, X, trits, d)


@pytest.mark.parametrize("M", [1, 2])
def test_i8_path_tq1_any_byte(M):
    """TQ1 planes read directly at M <= 2: every byte value, the ones no packer
    writes included, decodes as the inverse formula does (N5 = floor(243 b /
    256), digits first-most-significant; the last byte of a block gives one
    trit), so the product matches the oracle's product of its decoded trits."""
    N, K = 640, 2816
    rng = np.random.default_rng(55 + M)
    qs = rng.integers(0, 256, size=(N, (K // 256) * 52), dtype=np.uint8)
    for r in range(4):                    # every byte value in every position of a row
        qs[r] = np.resize(np.roll(np.arange(256, dtype=np.uint8), 64 * r), qs.shape[1])
    trits, invalid = O.unpack_tq1(qs, N, K)
    assert invalid > 0
    d = O.block_scales_fp16(rng.uniform(0.005, 0.05, size=N * (K // 256)).astype(np.float32), N, K)
    X = inputs.activations(M, K, 56).numpy()
    Y = tri.gemm(torch.from_numpy(X).to(DEV), torch.from_numpy(qs).to(DEV),
                 torch.from_numpy(d).to(DEV), N, K, "tq1", path=tri.PATH_I8)
    _check(Y, X, trits, d)


@pytest.mark.parametrize("M", [1, 2])
def test_i8_path_tq1_plane_4_byte_aligned(M):
    """A TQ1 plane that starts 4 bytes past a 16-byte boundary (the format
    only needs 4): the rows are then copied word by word instead of in
    16-byte chunks, with the same result."""
    N, K = 300, 4096
    X, trits, qs, d = _case(M, N, K, 61 + M, "tq1", per_block=True, p_zero=0.31)
    buf = torch.zeros(qs.size + 16, dtype=torch.uint8, device=DEV)
    shifted = buf[4:4 + qs.size].view(qs.shape)
    shifted.copy_(torch.from_numpy(qs).to(DEV))
    assert shifted.data_ptr() % 16 == 4
    Xd, dd = torch.from_numpy(X).to(DEV), torch.from_numpy(d).to(DEV)
    Y = tri.gemm(Xd, shifted, dd, N, K, "tq1", path=tri.PATH_I8)
    _check(Y, X, trits, d)
    Y16 = tri.gemm(Xd, torch.from_numpy(qs).to(DEV), dd, N, K, "tq1", path=tri.PATH_I8)
    assert torch.equal(Y, Y16)


def test_i8_path_deterministic():
    M, N, K = 1, 8192, 28672 // 4
    X, trits, qs, d = _case(M, N, K, 9, "tq2")
    args = (torch.from_numpy(X).to(DEV), torch.from_numpy(qs).to(DEV), torch.from_numpy(d).to(DEV),
            N, K, "tq2")
    Y1 = tri.gemm(*args, path=tri.PATH_I8)
    Y2 = tri.gemm(*args, path=tri.PATH_I8)
    assert torch.equal(Y1, Y2)


def test_i8_path_graph_replay_new_inputs():
    """A captured call replayed with new activations in the same buffers: the
    split-tile partial sums of one replay must never stand in for the next's."""
    M, N, K = 1, 4096, 7168
    X, trits, qs, d = _case(M, N, K, 61, "tq2")
    Xd = torch.from_numpy(X).to(DEV)
    qd, dd = torch.from_numpy(qs).to(DEV), torch.from_numpy(d).to(DEV)
    Y = torch.empty(M, N, dtype=torch.float16, device=DEV)
    ws = tri.Workspace(DEV)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        tri.gemm(Xd, qd, dd, N, K, "tq2", out=Y, workspace=ws, stream=s, path=tri.PATH_I8)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        tri.gemm(Xd, qd, dd, N, K, "tq2", out=Y, workspace=ws, stream=s, path=tri.PATH_I8)
    for seed in (7, 8, 9):
        Xn = inputs.activations(M, K, seed).numpy()
        Xd.copy_(torch.from_numpy(Xn).to(DEV))
        g.replay()
        torch.cuda.synchronize()
        _check(Y, Xn, trits, d)


def test_i8_path_workspace_shared_with_other_paths():
    """The same workspace alternates between the integer path and the others
    (which leave their own bytes in it): results stay correct."""
    N, K = 2048, 7168
    X1, trits, qs, d = _case(1, N, K, 62, "tq2", per_block=True, p_zero=0.4)
    X8 = inputs.activations(8, K, 63).numpy()
    qd, dd = torch.from_numpy(qs).to(DEV), torch.from_numpy(d).to(DEV)
    ws = tri.Workspace(DEV)
    for rep in range(3):
        Y1 = tri.gemm(torch.from_numpy(X1).to(DEV), qd, dd, N, K, "tq2", workspace=ws, path=tri.PATH_I8)
        _check(Y1, X1, trits, d)
        Y8 = tri.gemm(torch.from_numpy(X8).to(DEV), qd, dd, N, K, "tq2", workspace=ws, path=tri.PATH_MMA)
        _check(Y8, X8, trits, d)


@pytest.mark.parametrize("M", [1, 2])
def test_i8_path_beside_a_concurrent_kernel(M):
    """The decode kernel sums split row tiles through tickets (the last CTA to
    finish a tile adds the partial sums), so no CTA waits for another: while
    matrix products on a second stream hold a share of the SMs, the result is
    still right."""
    N, K = 8192, 7168
    X, trits, qs, d = _case(M, N, K, 91 + M, "tq2")
    Xd, qd, dd = torch.from_numpy(X).to(DEV), torch.from_numpy(qs).to(DEV), torch.from_numpy(d).to(DEV)
    A = torch.randn(4096, 4096, dtype=torch.float16, device=DEV)
    busy, mine = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    outs = []
    with torch.cuda.stream(busy):
        for _ in range(20):
            A = (A @ A).clamp_(-1, 1)
    with torch.cuda.stream(mine):
        for _ in range(8):
            outs.append(tri.gemm(Xd, qd, dd, N, K, "tq2", path=tri.PATH_I8, stream=mine))
    torch.cuda.synchronize()
    rows = np.arange(0, N, 7)
    for Y in outs:
        _check(Y[:, rows], X, trits[rows], d[rows])
        assert torch.equal(Y, outs[0])


@pytest.mark.parametrize("M", [1, 2])
def test_i8_path_chained_layers(M):
    """Back-to-back decode GEMMs: the second reads the first one's output as
    its activations (the kernel streams its weights before waiting for the
    preceding grid, and reads X only after the wait)."""
    K = 4096
    trits1, g1 = O.absmean_ternarize(inputs.latent_weights(K, K, 85).numpy(), 1e-6)
    trits2, g2 = O.absmean_ternarize(inputs.latent_weights(K, K, 86).numpy(), 1e-6)
    q1, d1 = O.pack("tq2", trits1, np.array([g1], np.float32))
    q2, d2 = O.pack("tq2", trits2, np.array([g2], np.float32))
    X = inputs.activations(M, K, 87).numpy() * np.float16(0.05)
    H = tri.gemm(torch.from_numpy(X).to(DEV), torch.from_numpy(q1).to(DEV), torch.from_numpy(d1).to(DEV),
                 K, K, "tq2", path=tri.PATH_I8)
    Y = tri.gemm(H, torch.from_numpy(q2).to(DEV), torch.from_numpy(d2).to(DEV), K, K, "tq2",
                 path=tri.PATH_I8)
    Hh = H.cpu().numpy()
    _check(H, X, trits1, d1)
    _check(Y, Hh, trits2, d2)


def test_i8_path_many_workspaces():
    """More workspaces than the library keeps ticket rows for: rows pass from
    one workspace to the next (their tickets are zero between calls)."""
    M, N, K = 1, 1024, 4096
    X, trits, qs, d = _case(M, N, K, 95, "tq2")
    Xd, qd, dd = torch.from_numpy(X).to(DEV), torch.from_numpy(qs).to(DEV), torch.from_numpy(d).to(DEV)
    wss = [tri.Workspace(DEV) for _ in range(300)]
    outs = [tri.gemm(Xd, qd, dd, N, K, "tq2", path=tri.PATH_I8, workspace=w) for w in wss]
    for Y in outs[::37] + outs[-2:]:
        _check(Y, X, trits, d)
    assert all(torch.equal(Y, outs[0]) for Y in outs)


@pytest.mark.parametrize("M,N,K", [(17, 384, 512), (33, 256, 1024), (300, 520, 2304), (513, 384, 1280),
                                   (1024, 256, 768), (256, 1000, 11008), (129, 8192, 1024)])
def test_tcgen05_path_shapes(M, N, K):
    """The tensor-memory kernel at shapes that exercise its tiling: activation
    tiles of 32..256 rows (ragged last tile), ragged weight tiles, several
    activation tiles, and K split over clusters of 2..4 CTAs (few tiles, many
    blocks) including a split whose parts hold different numbers of blocks."""
    X, trits, qs, d = _case(M, N, K, 400 + M + N % 89, "tq2", per_block=True, p_zero=0.31)
    Y = tri.gemm(torch.from_numpy(X).to(DEV), torch.from_numpy(qs).to(DEV),
                 torch.from_numpy(d).to(DEV), N, K, "tq2", path=tri.PATH_TCGEN05)
    _check(Y, X, trits, d)


def test_tcgen05_path_deterministic_split_k():
    """Split-K partial sums are added in cluster-rank order: bitwise repeatable."""
    M, N, K = 256, 2048, 8192
    X, trits, qs, d = _case(M, N, K, 71, "tq2")
    args = (torch.from_numpy(X).to(DEV), torch.from_numpy(qs).to(DEV), torch.from_numpy(d).to(DEV),
            N, K, "tq2")
    Y1 = tri.gemm(*args, path=tri.PATH_TCGEN05)
    Y2 = tri.gemm(*args, path=tri.PATH_TCGEN05)
    assert torch.equal(Y1, Y2)
    rows = np.arange(0, N, 37)
    _check(Y1[:, rows], X, trits[rows], d[rows])


def test_tcgen05_path_graph_replay_new_inputs():
    """A captured call replayed with new activations in the same buffers: the
    split-K scratch in the workspace is rewritten by every replay."""
    M, N, K = 96, 1024, 6144
    X, trits, qs, d = _case(M, N, K, 72, "tq2")
    Xd = torch.from_numpy(X).to(DEV)
    qd, dd = torch.from_numpy(qs).to(DEV), torch.from_numpy(d).to(DEV)
    Y = torch.empty(M, N, dtype=torch.float16, device=DEV)
    ws = tri.Workspace(DEV)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        tri.gemm(Xd, qd, dd, N, K, "tq2", out=Y, workspace=ws, stream=s, path=tri.PATH_TCGEN05)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        tri.gemm(Xd, qd, dd, N, K, "tq2", out=Y, workspace=ws, stream=s, path=tri.PATH_TCGEN05)
    for seed in (17, 18):
        Xn = inputs.activations(M, K, seed).numpy()
        Xd.copy_(torch.from_numpy(Xn).to(DEV))
        g.replay()
        torch.cuda.synchronize()
        _check(Y, Xn, trits, d)


def test_tcgen05_path_back_to_back_layers():
    """Consecutive launches chained by programmatic dependent launch: each
    layer reads the previous layer's output as its activations."""
    M, K = 64, 1024
    trits1, g1 = O.absmean_ternarize(inputs.latent_weights(K, K, 81).numpy(), 1e-6)
    trits2, g2 = O.absmean_ternarize(inputs.latent_weights(K, K, 82).numpy(), 1e-6)
    q1, d1 = O.pack("tq2", trits1, np.array([g1], np.float32))
    q2, d2 = O.pack("tq2", trits2, np.array([g2], np.float32))
    X = inputs.activations(M, K, 83).numpy() * np.float16(0.05)
    Xd = torch.from_numpy(X).to(DEV)
    H = tri.gemm(Xd, torch.from_numpy(q1).to(DEV), torch.from_numpy(d1).to(DEV), K, K, "tq2",
                 path=tri.PATH_TCGEN05)
    Y = tri.gemm(H, torch.from_numpy(q2).to(DEV), torch.from_numpy(d2).to(DEV), K, K, "tq2",
                 path=tri.PATH_TCGEN05)
    Hh = H.cpu().numpy()
    _check(H, X, trits1, d1)
    _check(Y, Hh, trits2, d2)


@pytest.mark.parametrize("fmt", ["tq2", "tq1"])
@pytest.mark.parametrize("M,N,K", [(3, 384, 512), (5, 1000, 2304), (9, 129, 256), (12, 2048, 4096),
                                   (16, 520, 11008), (16, 4096, 28672), (8, 1024, 8192)])
def test_i8_path_batch_up_to_16(fmt, M, N, K):
    """The integer path for 3 <= M <= 16 (three or six column tiles of digits):
    ragged row tiles, K split over clusters of 1..8 CTAs, per-block scales."""
    X, trits, qs, d = _case(M, N, K, 500 + M + N % 83, fmt, per_block=True, p_zero=0.31)
    Y = tri.gemm(torch.from_numpy(X).to(DEV), torch.from_numpy(qs).to(DEV),
                 torch.from_numpy(d).to(DEV), N, K, fmt, path=tri.PATH_I8)
    rows = np.arange(N) if N <= 2048 else np.arange(0, N, 41)
    _check(Y[:, rows], X, trits[rows], d[rows])


@pytest.mark.parametrize("M", [4, 16])
def test_i8_path_batch_activation_extremes(M):
    """Per (block, batch row) quantisation steps: rows with different ranges, a
    huge value among tiny ones, zero blocks and signed extremes."""
    N, K = 384, 2048
    X, trits, qs, d = _case(M, N, K, 42, "tq2", per_block=True, p_zero=0.5)
    X = X.copy()
    X[0, 0] = 60000.0
    X[0, 1:256] = (np.random.default_rng(4).standard_normal(255) * 1e-3).astype(np.float16)
    X[1 % M, 256:512] = 0.0
    X[M - 1, 512:768] = np.float16(6e-8)
    X[:, 768] = -65504.0
    X[:, 769] = 65504.0
    X[M // 2] *= np.float16(1e-3)
    Y = tri.gemm(torch.from_numpy(X).to(DEV), torch.from_numpy(qs).to(DEV),
                 torch.from_numpy(d).to(DEV), N, K, "tq2", path=tri.PATH_I8)
    _check(Y, X, trits, d)


def test_i8_path_batch_deterministic_and_graph_replay():
    """Split-K sums in cluster-rank order are bitwise repeatable, and a captured
    call replayed with new activations recomputes its activation records."""
    M, N, K = 16, 2048, 8192
    X, trits, qs, d = _case(M, N, K, 73, "tq2")
    Xd = torch.from_numpy(X).to(DEV)
    qd, dd = torch.from_numpy(qs).to(DEV), torch.from_numpy(d).to(DEV)
    Y1 = tri.gemm(Xd, qd, dd, N, K, "tq2", path=tri.PATH_I8)
    Y2 = tri.gemm(Xd, qd, dd, N, K, "tq2", path=tri.PATH_I8)
    assert torch.equal(Y1, Y2)
    Y = torch.empty(M, N, dtype=torch.float16, device=DEV)
    ws = tri.Workspace(DEV)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        tri.gemm(Xd, qd, dd, N, K, "tq2", out=Y, workspace=ws, stream=s, path=tri.PATH_I8)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        tri.gemm(Xd, qd, dd, N, K, "tq2", out=Y, workspace=ws, stream=s, path=tri.PATH_I8)
    for seed in (27, 28):
        Xn = inputs.activations(M, K, seed).numpy()
        Xd.copy_(torch.from_numpy(Xn).to(DEV))
        g.replay()
        torch.cuda.synchronize()
        rows = np.arange(0, N, 13)
        _check(Y[:, rows], Xn, trits[rows], d[rows])


def _swiglu_case(M, F, K, seed, fmt, per_block=True):
    rng = np.random.default_rng(seed)
    tg = inputs.random_trits(F, K, 0.31, seed).numpy()
    tu = inputs.random_trits(F, K, 0.31, seed + 1).numpy()
    sg = inputs.block_scales(F, K, seed + 2).numpy() if per_block else np.array([0.03], np.float32)
    su = inputs.block_scales(F, K, seed + 3).numpy() if per_block else np.array([0.02], np.float32)
    qg, dg = O.pack(fmt, tg, sg)
    qu, du = O.pack(fmt, tu, su)
    X = inputs.activations(M, K, seed + 4).numpy()
    q, d = tri.interleave_gate_up(torch.from_numpy(qg), torch.from_numpy(dg), torch.from_numpy(qu),
                                  torch.from_numpy(du))
    return X, tg, dg, tu, du, q.to(DEV), d.to(DEV)


@pytest.mark.parametrize("fmt", ["tq2", "tq1"])
@pytest.mark.parametrize("M,F,K", [(1, 520, 2304), (2, 128, 512), (4, 520, 2304), (16, 1024, 8192),
                                   (9, 64, 256), (40, 264, 1024), (16, 8, 256)])
def test_gemm_swiglu_vs_oracle(fmt, M, F, K):
    """silu(X Wg^T) * (X Wu^T) on every regime: fused epilogue (3 <= M <= 16,
    split K included) and the product-then-combine route (M <= 2, M > 16)."""
    X, tg, dg, tu, du, q, d = _swiglu_case(M, F, K, 600 + M + F % 37, fmt)
    Y = tri.gemm_swiglu(torch.from_numpy(X).to(DEV), q, d, F, K, fmt)
    y = Y.float().cpu().numpy().astype(np.float64)
    ref, G, U = O.swiglu_f64(X, tg, dg, tu, du)
    tol = O.swiglu_tolerance(X, dg, du, G, U)
    bad = np.abs(y - ref) > tol
    assert not bad.any(), f"{bad.sum()} outputs out of tolerance; worst {(np.abs(y - ref) - tol).max()}"


def test_gemm_swiglu_fused_matches_separate_products():
    """The fused epilogue agrees with two plain GEMMs combined on the host."""
    M, F, K = 16, 2048, 4096
    X, tg, dg, tu, du, q, d = _swiglu_case(M, F, K, 77, "tq2", per_block=False)
    Xd = torch.from_numpy(X).to(DEV)
    Y = tri.gemm_swiglu(Xd, q, d, F, K, "tq2", path=tri.PATH_I8).float()
    Y2 = tri.gemm(Xd, q, d, 2 * F, K, "tq2", path=tri.PATH_I8).float().reshape(M, F // 8, 2, 8)
    g, u = Y2[:, :, 0, :].reshape(M, F), Y2[:, :, 1, :].reshape(M, F)
    ref = torch.nn.functional.silu(g) * u
    assert torch.allclose(Y, ref, rtol=2e-3, atol=2e-3)
