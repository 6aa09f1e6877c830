"""bench.py's accounting on the CPU: the step's FLOPs and the kernels'
algorithmic bytes against the workload's figures worked out by hand, the
launches per step against the kernels a step runs, and the rule that a
recorded DRAM-traffic figure is reported only while the kernel sources still
hash to the value recorded beside it."""

import os
import shutil

import pytest

import bench
import workloads as WL


def test_step_flops_and_bytes_of_the_qkv_workload():
    M, K, N, r = WL.QKV.M, WL.QKV.K, WL.QKV.N, WL.QKV.r
    assert (M, K, N, r) == (4608, 3072, 9216, 32)
    # 2 M N K of the 4-bit GEMM = 260.9 GFLOP, plus the rank-32 branch 2 M r (K + N)
    assert 2 * 4608 * 9216 * 3072 == 260_919_263_232
    assert bench.layer_flops(M, K, N, r) == 260_919_263_232 + 2 * 4608 * 32 * (3072 + 9216)
    # the AWQ adaLN projection adds 2 M N K at M = 4, N = 18432
    assert bench.step_flops() == bench.layer_flops(M, K, N, r) + 2 * 4 * 18432 * 3072
    # the quantizer moves X (28.3 MB), codes (7.1), scales (0.9), xl1 (0.6), L1 and smooth_inv: 37.1 MB
    assert round(bench.quantize_bytes(M, K, r) / 1e6, 1) == 37.1
    # AWQ: 4-bit weights (28.3 MB), (scale, zero) pairs (3.5 MB), X, Y and bias: 32.1 MB
    assert round(bench.awq_bytes(4, 3072, 18432) / 1e6, 1) == 32.1


def test_launches_per_step():
    # quantizer, its split-K reduction, the GEMM and one AWQ launch per 16 tokens
    assert bench.launches_per_step(4608, 3072, 32, 4) == 4
    assert bench.launches_per_step(18432, 3072, 32, 4) == 3   # one K split: no reduction
    assert bench.launches_per_step(4608, 3072, 0, 4) == 3     # no low-rank branch
    assert bench.launches_per_step(4608, 3072, 32, 40) == 6   # three AWQ launches


def test_recorded_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    root = tmp_path / "repo"
    shutil.copytree(os.path.join(bench.ROOT, "bit_quantized_diffusion_b200", "csrc"),
                    root / "bit_quantized_diffusion_b200" / "csrc")
    (root / "profiles").mkdir()
    monkeypatch.setattr(bench, "ROOT", str(root))
    sha = bench.kernel_source_sha()
    assert sha == bench.kernel_source_sha() and len(sha) == 16
    (root / "profiles" / "traffic.md").write_text(
        "| kernel | bytes per launch | csrc sha |\n|---|---|---|\n"
        f"| w4a4_nvfp4_gemm_kernel | 56292096 | {sha} |\n"
        "| awq_gemv_kernel | 31944448 | 0000000000000000 |\n")
    assert bench.recorded_traffic("w4a4_nvfp4_gemm_kernel") == 56292096.0
    assert bench.recorded_traffic("awq_gemv_kernel") is None       # another hash
    assert bench.recorded_traffic("quantize_act_kernel") is None   # no row
    # any change to a kernel source retires the figure
    f = root / "bit_quantized_diffusion_b200" / "csrc" / "pack.cuh"
    f.write_text(f.read_text() + "\n")
    assert bench.kernel_source_sha() != sha
    assert bench.recorded_traffic("w4a4_nvfp4_gemm_kernel") is None


def test_peaks_come_from_the_measured_file():
    peaks = bench.measured_peaks()
    if not os.path.exists(os.path.join(bench.ROOT, "MEASURED_PEAKS.json")):
        pytest.skip("no measured peaks here")
    assert peaks["source"] == "measured" and peaks["hbm_gbs"] > 1000 and peaks["bf16_tflops"] > 100
