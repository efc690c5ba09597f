"""Host-side accounting of bench.py on CPU: the algorithmic bytes behind the
roofline figures, the launch counts claimed per call, workload overrides and
the reference arm's JSON line (the CPU oracle timed on the host)."""
import argparse

import pytest

import bench

PATH_SIMT, PATH_MMA, PATH_TCGEN05, PATH_I8 = 1, 2, 3, 4


@pytest.mark.parametrize("fmt,bits", [("tq2", 2.0625), ("tq1", 1.6875)])
@pytest.mark.parametrize("M,N,K", [(1, 4096, 4096), (1, 11008, 4096), (16, 8192, 28672), (256, 8192, 8192)])
def test_algorithmic_bytes_are_storage_bits_plus_activations(fmt, bits, M, N, K):
    # TQ2: 64 B of fields + 2 B of scale per 256 weights = 2.0625 bit/weight;
    # TQ1: 52 B of five-trit bytes + 2 B of scale = 1.6875 bit/weight stored
    expected = N * K * bits / 8 + 2 * M * K + 2 * M * N
    assert bench.algo_bytes(fmt, M, N, K) == pytest.approx(expected, rel=0, abs=0.5)


def test_decode_set_weight_bytes_per_layer():
    # weights + scales = 66 N K / 256 bytes: 4.33 MB and 11.62 MB for the
    # LLaMA-7B-like layers (X and Y add 2 K + 2 N bytes at M = 1)
    got = [bench.algo_bytes("tq2", 1, N, K) - 2 * K - 2 * N for N, K in bench.WORKLOADS["llama7b_decode_m1"]["layers"]]
    assert got == [4325376, 11624448, 11624448]


@pytest.mark.parametrize("path,M,fmt,swiglu,n", [
    (PATH_I8, 1, "tq2", False, 1),        # M <= 2: one kernel, activations quantised in its prologue
    (PATH_I8, 2, "tq2", False, 1),
    (PATH_I8, 3, "tq2", False, 2),        # 3 <= M <= 16: prep + main
    (PATH_I8, 16, "tq2", False, 2),
    (PATH_I8, 1, "tq1", False, 1),        # M <= 2 reads TQ1 planes directly
    (PATH_I8, 2, "tq1", True, 2),         # + the SwiGLU combine
    (PATH_I8, 4, "tq1", False, 3),        # 3 <= M <= 16: + the TQ1 -> TQ2 transcode
    (PATH_I8, 8, "tq2", True, 2),         # SwiGLU fused into the integer kernel's epilogue
    (PATH_I8, 2, "tq2", True, 2),         # ... but not for M <= 2: + the combine kernel
    (PATH_MMA, 4, "tq2", False, 2),       # prep + main
    (PATH_TCGEN05, 256, "tq2", False, 1),
    (PATH_TCGEN05, 256, "tq1", False, 2),
    (PATH_TCGEN05, 64, "tq2", True, 2),
    (PATH_SIMT, 4, "tq1", False, 1),      # the CUDA-core path reads TQ1 directly
])
def test_kernels_per_call(path, M, fmt, swiglu, n):
    assert bench.kernels_per_call(path, M, fmt, swiglu) == n


def test_workload_overrides_do_not_touch_the_table():
    w = bench.workload_from_args("square_8192_m256", M=16, fmt="tq1")
    assert (w["M"], w["fmt"], w["name"]) == (16, "tq1", "square_8192_m256")
    assert bench.WORKLOADS["square_8192_m256"]["M"] == 256
    assert bench.WORKLOADS["square_8192_m256"]["fmt"] == "tq2"


def test_fused_block_layers():
    w = bench.WORKLOADS["block70b_m16_fused"]
    # q/k/v concatenated (8192 + 1024 + 1024 rows), gate/up interleaved (2 x 28672)
    assert w["layers"][0] == (10240, 8192) and w["layers"][2] == (57344, 8192)
    assert w["swiglu"] == [2]
    unfused = bench.WORKLOADS["block70b_m16"]["layers"]
    assert sum(N * K for N, K in w["layers"]) == sum(N * K for N, K in unfused)


def test_oracle_sample_on_a_small_layer():
    w = dict(layers=[(256, 1024)], seeds=[0], M=1, fmt="tq2", name="tiny")
    r = bench.oracle_sample(w, budget_s=0.2)
    assert r["unit"] == "GB/s" and r["value"] > 0 and r["threads"] >= 1 and "256x1024" in r["sample"]
    assert r["elapsed_s"] >= 0.2
    w = dict(w, M=64)
    r = bench.oracle_sample(w, budget_s=0.2, threads=1)
    assert r["unit"] == "TFLOP/s" and r["value"] > 0 and r["threads"] == 1


def test_reference_arm_line(monkeypatch):
    calls = []

    def fake_sample(w, budget_s=12.0, threads=None):
        calls.append(budget_s)
        return {"value": 0.025, "unit": "GB/s", "threads": 16, "elapsed_s": 2.5,
                "sample": "2 passes over the first min(N, 2048) rows of each layer"}

    monkeypatch.setattr(bench, "oracle_sample", fake_sample)
    args = argparse.Namespace(workload="llama7b_decode_m1", M=None, fmt=None, steps=4, warmup=3)
    line = bench.run_reference(args, 0, 1)
    assert len(calls) == 7                                # warm-up samples are taken and dropped
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["impl"] == "reference" and line["unit"] == "GB/s" and line["value"] == 0.025
    assert line["ms_per_step"] == 2500.0                  # the measured time per step, not a budget
    assert line["config"]["workload"] == "llama7b_decode_m1" and line["dtype"] == "f64"
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] == 16 and cb["value"] == line["value"]
    assert line["e2e"] == {"value": line["value"], "unit": "GB/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert bench.run_reference(args, 1, 2) is None        # only rank 0 runs the oracle


def test_default_workload_is_the_down_projection_decode():
    src = open(bench.__file__).read()
    assert 'ap.add_argument("--workload", default="down_8192x28672_m1"' in src
    w = bench.WORKLOADS["down_8192x28672_m1"]
    assert w["layers"] == [(8192, 28672)] and w["M"] == 1 and w["fmt"] == "tq2"
    assert bench.TARGET_WORKLOADS == ("square_8192_m256", "llama7b_decode_m1")
