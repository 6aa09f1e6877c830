#!/usr/bin/env python
"""Benchmark of the SVDQuant W4A4 hot path on B200.

One step is one pass of the whole hot path over one batch of synthetic input:
  1. svdq_quantize_act  -- smoothing, NVFP4 quantization and the rank-32
                           down-projection of X [4608, 3072] (FLUX-like QKV input)
  2. svdq_w4a4_linear   -- the NVFP4 GEMM to N = 9216 with the fused low-rank
                           up-projection and bias
  3. awq_w4a16_linear   -- the AWQ W4A16 adaLN modulation projection
                           (M = 4, K = 3072, N = 18432)
The metric is TFLOP/s over the step: 2MNK + 2Mr(K+N) for the SVDQ layer plus
2MNK for the AWQ layer, divided by the device time of the step. L2 is flushed
before every step, outside the timed events: a 256 MiB write, then a 256 MiB
read, so the step starts with none of its inputs in L2 and with no dirty lines
left from the flush (their write-back would otherwise land inside the step).
The kernels of a step are launched with programmatic dependent launch, so each one's launch
and prologue overlap the previous kernel's tail; the timed region therefore
records events only at step boundaries, and the per-kernel times (and the
roofline of the GEMM) come from a second pass of the same steps with an event
between every two kernels.

Beside the step, and not part of it, two variants of the same layer are timed
call by call after the flush: two-level NVFP4 (svdq_tensor_scale,
svdq_quantize_act_two_level, svdq_w4a4_linear_two_level) and the fused QKV
projection (svdq_w4a4_linear_qkv_norm_rope: the layer's 9216 columns as 24 heads
each of Q, K, V, with the heads of Q and K RMS-normalised and rotated in the
GEMM's epilogue). They appear under "kernels".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With N > 1 (torchrun, one process per GPU) every rank runs the same layer on
its own token batch (data parallel, no collective on the data path); the
reported value is the work of all ranks over the slowest rank's device time.
Prints one JSON line on rank 0.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

# The oracle legs run on every host core this process may use; BLAS thread pools
# size themselves from the environment when numpy loads, so pin them first.
HOST_CORES = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
for _var in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS"):
    os.environ.setdefault(_var, str(HOST_CORES))

import numpy as np  # noqa: E402

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as WL  # noqa: E402

METRIC = "SVDQ W4A4 linear TFLOPS (NVFP4, r=32) and % of FP4 tensor roofline"
UNIT = "TFLOP/s"
SHAPE = WL.QKV
AWQ = WL.AWQ_MOD
FP4_OVER_BF16 = 4.0  # nominal dense FP4 / BF16 tensor throughput ratio (9 / 2.25 PFLOP/s)
NOMINAL_FP4_TFLOPS = 9000.0  # B200 dense FP4, nominal
AWQ_KERNEL = "awq_gemv_kernel"  # the kernel awq_w4a16_linear runs at the step's 4 tokens


def layer_flops(M: int, K: int, N: int, r: int) -> float:
    return 2.0 * M * N * K + 2.0 * M * r * (K + N)


def launches_per_step(M: int, K: int, r: int, m_awq: int) -> int:
    """Kernels one step launches: the quantizer, its split-K down-projection
    reduction when K is split, the GEMM, and one AWQ launch per 16 tokens."""
    import bit_quantized_diffusion_b200 as bq

    splits = bq.svdq_xl1_splits(M, K, r)
    return 1 + (1 if r > 0 and splits > 1 else 0) + 1 + (m_awq + 15) // 16


def step_flops() -> float:
    return layer_flops(SHAPE.M, SHAPE.K, SHAPE.N, SHAPE.r) + 2.0 * AWQ.M * AWQ.N * AWQ.K


def quantize_bytes(M: int, K: int, r: int) -> float:
    """Algorithmic HBM bytes of svdq_quantize_act (NVFP4)."""
    return 2.0 * M * K + M * K / 2 + M * K / 16 + 4.0 * M * r + 2.0 * K * r + 4.0 * K


def awq_bytes(M: int, K: int, N: int) -> float:
    return N * K / 2 + N * (K / 64) * 4 + 2.0 * M * K + 2.0 * M * N + 2.0 * N


def quantize_bytes_fmt(fmt: str, M: int, K: int, r: int) -> float:
    """Algorithmic HBM bytes of svdq_quantize_act: X, codes, scales, xl1, L1, smooth_inv."""
    sc = M * K / 16 if fmt == "nvfp4" else 2.0 * M * K / 64
    return 2.0 * M * K + M * K / 2 + sc + 4.0 * M * r + 2.0 * K * r + 4.0 * K


def median_us(fn, flush, n: int) -> float:
    """Median device time of fn() in microseconds: n calls, each after the L2
    flush, with CUDA events on the launch stream right around the call."""
    import torch
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(n + 3)]
    for a, b in ev:
        flush()
        a.record()
        fn()
        b.record()
    torch.cuda.synchronize()
    return statistics.median(a.elapsed_time(b) for a, b in ev[3:]) * 1e3


def sweep_layers(bq, prep, dev, flush, n: int, fp4_peak: float) -> dict:
    """The other workloads of the build, each as one SVDQ layer (quantizer, then
    the 4-bit GEMM with the fused low-rank branch and bias), timed call by call
    after the flush: the tiny layer, the FLUX-like MLP pair fc1 / fc2 (rank 128,
    NVFP4) and fc1 in INT4, the rank sweep at hidden 3840 (N 3840 and 15360, rank
    0 / 32 / 128 / 256; the overhead of the low-rank branch against rank 0), and
    the QKV projection at batch 4 (M 18432). Weights are prepared on the device
    from the same seeded draws the tests use; one float32 SVD per weight serves
    all of its ranks (timing only: parity is pinned on the float64 prep)."""
    import torch
    to_dev = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).to(dev).view(torch.bfloat16)  # noqa: E731
    out = {}
    svd_cache = {}
    shapes = [WL.TINY, WL.FC1, WL.FC2, WL.FC1_INT4, *WL.RANK_SWEEP, WL.BIG]
    for sh in shapes:
        d = WL.svdq_inputs(sh)
        X = to_dev(d["X"])
        W = to_dev(d["W"])
        bias = to_dev(d["bias"]) if d["bias"] is not None else None
        x_absmax = bq.svdq_column_absmax(X)
        svd = None
        if sh.r > 0:
            key = (sh.seed, sh.N, sh.K)
            if key not in svd_cache:
                _, w_hat = prep.smoothed_weight(W, x_absmax)
                svd_cache[key] = torch.linalg.svd(w_hat.float(), full_matrices=False)
            svd = svd_cache[key]
        w = prep.prepare_svdq_weights(W, x_absmax, sh.r, sh.fmt, svd=svd)
        del W
        M, K, N, r = sh.M, sh.K, sh.N, sh.r
        codes = torch.empty(bq.svdq_codes_bytes(sh.fmt, M, K), dtype=torch.uint8, device=dev)
        scales = torch.empty(bq.svdq_scales_bytes(sh.fmt, M, K), dtype=torch.uint8, device=dev)
        xl1 = (torch.empty((bq.svdq_xl1_splits(M, K, r), M, r), dtype=torch.float32, device=dev)
               if r else None)
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        quant = lambda: bq.svdq_quantize_act(X, w["L1s"], w["smooth_inv"], fmt=sh.fmt,  # noqa: E731
                                             codes=codes, scales=scales, xl1=xl1)
        _, _, xv = quant()
        gemm = lambda: bq.svdq_w4a4_linear(codes, scales, xv, w["w_codes"], w["w_scales"], w["L2"],  # noqa: E731
                                           bias, M, N, K, fmt=sh.fmt, Y=Y)
        t_q = median_us(quant, flush, n)
        t_g = median_us(gemm, flush, n)
        f4 = 2.0 * M * N * K
        e = {"M": M, "K": K, "N": N, "r": r, "format": sh.fmt,
             "svdq_quantize_act_us": round(t_q, 2),
             "svdq_quantize_act_gbs": round(quantize_bytes_fmt(sh.fmt, M, K, r) / (t_q * 1e-6) / 1e9, 1),
             "svdq_w4a4_linear_us": round(t_g, 2),
             "svdq_w4a4_linear_tflops_4bit": round(f4 / (t_g * 1e-6) / 1e12, 1),
             "layer_tflops": round(f4 / ((t_q + t_g) * 1e-6) / 1e12, 1)}
        if sh.fmt == "nvfp4":
            e["gemm_frac_of_fp4_peak"] = round(f4 / (t_g * 1e-6) / 1e12 / fp4_peak, 3)
        out[sh.name] = e
        del X, w, codes, scales, xl1, Y
        assert bq.svdq_check_device_status() == 0
    for n_ in (3840, 15360):
        base = out[f"dit3840_n{n_}_r0"]
        for r in (32, 128, 256):
            e = out[f"dit3840_n{n_}_r{r}"]
            e["lowrank_overhead_gemm"] = round(e["svdq_w4a4_linear_us"] / base["svdq_w4a4_linear_us"] - 1, 3)
            e["lowrank_overhead_layer"] = round(
                (e["svdq_w4a4_linear_us"] + e["svdq_quantize_act_us"])
                / (base["svdq_w4a4_linear_us"] + base["svdq_quantize_act_us"]) - 1, 3)
    return out


def mlp_pair(bq, prep, dev, flush, n: int) -> dict:
    """The FLUX-like MLP pair (fc1 4608 x 3072 -> 12288, GELU, fc2 12288 -> 3072, rank 128,
    NVFP4), fused and unfused, each timed as a whole (event to event after the flush).
    Unfused: quantizer, fc1 GEMM to bf16, GELU (tanh form, torch, bf16), fc2's quantizer
    on that bf16 activation, fc2 GEMM. Fused: quantizer, svdq_mlp_fc1 (GELU, fc2's
    smoothing, codes, scales and down-projection in fc1's epilogue, plus the reduction
    of its partial down-projections), fc2 GEMM."""
    import torch
    to_dev = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).to(dev).view(torch.bfloat16)  # noqa: E731
    s1, s2 = WL.FC1, WL.FC2
    d1, d2 = WL.svdq_inputs(s1), WL.svdq_inputs(s2)
    X1, X2c = to_dev(d1["X"]), to_dev(d2["X"])
    ws = []
    for d, sh, X in ((d1, s1, X1), (d2, s2, X2c)):
        W = to_dev(d["W"])
        xa = bq.svdq_column_absmax(X)
        _, w_hat = prep.smoothed_weight(W, xa)
        svd = torch.linalg.svd(w_hat.float(), full_matrices=False)
        ws.append(prep.prepare_svdq_weights(W, xa, sh.r, svd=svd))
        del W, w_hat, svd
    w1, w2 = ws
    del X2c
    b1, b2 = to_dev(d1["bias"]), to_dev(d2["bias"])
    M, K1, N1, N2, r1, r2 = s1.M, s1.K, s1.N, s2.N, s1.r, s2.r
    L1t_2 = w2["L1"].t().contiguous()
    c1 = torch.empty(bq.svdq_codes_bytes("nvfp4", M, K1), dtype=torch.uint8, device=dev)
    sc1 = torch.empty(bq.svdq_scales_bytes("nvfp4", M, K1), dtype=torch.uint8, device=dev)
    x1 = torch.empty((bq.svdq_xl1_splits(M, K1, r1), M, r1), dtype=torch.float32, device=dev)
    c2 = torch.empty(bq.svdq_codes_bytes("nvfp4", M, N1), dtype=torch.uint8, device=dev)
    sc2 = torch.empty(bq.svdq_scales_bytes("nvfp4", M, N1), dtype=torch.uint8, device=dev)
    x2f = torch.empty((bq.svdq_mlp_splits(M, N1), M, r2), dtype=torch.float32, device=dev)
    x2u = torch.empty((bq.svdq_xl1_splits(M, N1, r2), M, r2), dtype=torch.float32, device=dev)
    Y1 = torch.empty((M, N1), dtype=torch.bfloat16, device=dev)
    Y2 = torch.empty((M, N2), dtype=torch.bfloat16, device=dev)

    def quant1():
        return bq.svdq_quantize_act(X1, w1["L1s"], w1["smooth_inv"], codes=c1, scales=sc1, xl1=x1)[2]

    def unfused():
        xv = quant1()
        bq.svdq_w4a4_linear(c1, sc1, xv, w1["w_codes"], w1["w_scales"], w1["L2"], b1, M, N1, K1, Y=Y1)
        h = torch.nn.functional.gelu(Y1, approximate="tanh")
        _, _, xv2 = bq.svdq_quantize_act(h, w2["L1s"], w2["smooth_inv"], codes=c2, scales=sc2, xl1=x2u)
        bq.svdq_w4a4_linear(c2, sc2, xv2, w2["w_codes"], w2["w_scales"], w2["L2"], b2, M, N2, N1, Y=Y2)

    def fused_fc1():
        xv = quant1()
        return bq.svdq_mlp_fc1(c1, sc1, xv, w1["w_codes"], w1["w_scales"], w1["L2"], b1, w2["smooth_inv"],
                               L1t_2, M, N1, K1, codes2=c2, scales2=sc2, xl1_2=x2f)[2]

    def fused():
        xv2 = fused_fc1()
        bq.svdq_w4a4_linear(c2, sc2, xv2, w2["w_codes"], w2["w_scales"], w2["L2"], b2, M, N2, N1, Y=Y2)

    xv = quant1()
    t = {"unfused_us": median_us(unfused, flush, n), "fused_us": median_us(fused, flush, n),
         "fused_fc1_us": median_us(lambda: bq.svdq_mlp_fc1(
             c1, sc1, xv, w1["w_codes"], w1["w_scales"], w1["L2"], b1, w2["smooth_inv"], L1t_2, M, N1, K1,
             codes2=c2, scales2=sc2, xl1_2=x2f), flush, n)}
    assert bq.svdq_check_device_status() == 0
    flops = 2.0 * M * N1 * K1 + 2.0 * M * N2 * N1
    return {"workload": f"{s1.name} -> GELU -> {s2.name}: M={M} K1={K1} N1={N1} N2={N2} r={r1}",
            **{k: round(v, 2) for k, v in t.items()},
            "fused_speedup": round(t["unfused_us"] / t["fused_us"], 3),
            "fused_fc1_tflops_4bit": round(2.0 * M * N1 * K1 / (t["fused_fc1_us"] * 1e-6) / 1e12, 1),
            "fused_pair_tflops_4bit": round(flops / (t["fused_us"] * 1e-6) / 1e12, 1),
            "hidden_bytes_avoided": 2 * M * N1 * 2}


def awq_by_tokens(bq, awq_w, bias_a, dev, flush, n: int) -> dict:
    """The adaLN projection (K 3072, N 18432) at more tokens: the tensor-core
    GEMM above 64 tokens, and both kernels at 4 and 64 tokens."""
    import torch
    out = {}
    g = torch.Generator(device=dev)
    g.manual_seed(11)
    for M in (4, 16, 64, 128, 256):
        X = torch.randn(M, AWQ.K, device=dev, generator=g).to(torch.bfloat16)
        Y = torch.empty((M, AWQ.N), dtype=torch.bfloat16, device=dev)
        for path in ("0", "1"):
            if path == "0" and M > 64:
                continue
            os.environ["SVDQ_AWQ_PATH"] = path
            t = median_us(lambda: bq.awq_w4a16_linear(X, awq_w["qweight"], awq_w["sz"], bias_a, AWQ.N, Y=Y),
                          flush, n)
            name = "gemv" if path == "0" else "tensor_cores"
            out[f"m{M}_{name}_us"] = round(t, 2)
            out[f"m{M}_{name}_gbs"] = round(awq_bytes(M, AWQ.K, AWQ.N) / (t * 1e-6) / 1e9, 1)
        os.environ.pop("SVDQ_AWQ_PATH", None)
    assert bq.svdq_check_device_status() == 0
    return out


def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def kernel_source_sha() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_quantized_diffusion_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        if name.endswith((".cu", ".cuh")):
            with open(os.path.join(csrc, name), "rb") as f:
                h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str) -> float | None:
    """DRAM bytes per launch of `kernel` recorded from an ncu capture in
    profiles/, if the capture was taken on the current kernel sources."""
    path = os.path.join(ROOT, "profiles", "traffic.md")
    if not os.path.exists(path):
        return None
    sha = kernel_source_sha()
    for line in open(path):
        parts = line.strip().strip("|").split("|")
        if len(parts) >= 3 and parts[0].strip() == kernel and parts[2].strip() == sha:
            return float(parts[1])
    return None


def sum_traffic(kernels) -> float | None:
    """DRAM bytes per call summed over the call's kernels, or None if any is unrecorded."""
    vals = [recorded_traffic(k) for k in kernels]
    return None if any(v is None for v in vals) else float(sum(vals))


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x100: "display_clock_setting"}

    def __init__(self, cuda_index: int, period_s: float = 0.002):
        self.period = period_s
        self.samples: list[tuple[int, int]] = []
        self.max_mhz = None
        self._stop = threading.Event()
        self._h = None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            self._nv = pynvml
            pr = torch.cuda.get_device_properties(cuda_index)
            bus = "%08X:%02X:%02X.0" % (pr.pci_domain_id, pr.pci_bus_id, pr.pci_device_id)
            self._h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                pynvml.nvmlDeviceGetCurrentClocksThrottleReasons
        except Exception:  # NVML missing: report no clocks rather than guess
            self._h = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM)
                rs = self._reasons(self._h)
                self.samples.append((mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._h is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        if self._h is not None:
            self._stop.set()
            self._t.join()

    def summary(self) -> dict:
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = [s[0] for s in self.samples]
        bits = 0
        for _, rs in self.samples:
            bits |= rs
        reasons = [name for b, name in self.REASONS.items() if bits & b and name != "gpu_idle"]
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(mhz)}


# --------------------------------------------------------------------- oracle
def oracle_sample_step(rows: int, cols: int, awq_rows: int, host: dict) -> float:
    """The CPU oracle, as it stands, on a sample of the same step: `rows` token
    rows x `cols` output features of the SVDQ layer (a1..a6) and `awq_rows`
    output features of the AWQ layer (a7). Returns the sample's flops."""
    from oracle import awq as OA
    from oracle import svdq as S
    bias = None if host["bias_bits"] is None else host["bias_bits"][:cols]
    fwd = S.svdq_forward("nvfp4", host["x_bits"][:rows], host["smooth_inv"], host["L1"],
                         host["L2"][:, :cols], host["w_codes"][:cols], host["w_scales"][:cols], bias)
    assert fwd["Y"].shape == (rows, cols)
    ya = OA.linear(host["xa"], host["q"][:awq_rows], host["s"][:awq_rows], host["z"][:awq_rows])
    assert ya.shape == (AWQ.M, awq_rows)
    return (2.0 * rows * cols * SHAPE.K + 2.0 * rows * SHAPE.r * (SHAPE.K + cols)
            + 2.0 * AWQ.M * awq_rows * AWQ.K)


def sample_text(rows: int, cols: int, awq_rows: int) -> str:
    return (f"{rows} of {SHAPE.M} token rows x {cols} of {SHAPE.N} output features of the QKV "
            f"layer (a1..a6, weights dequantized per call) + {awq_rows} of {AWQ.N} AWQ output "
            f"features (a7)")


def oracle_inputs_from_device(dev: dict) -> dict:
    """Host copies of the prepared layer, in the oracle's plain formats."""
    from oracle import formats as F
    from oracle import layout as LO
    from oracle import svdq as S
    w = dev["svdq"]
    K, N, r = SHAPE.K, SHAPE.N, SHAPE.r
    bits = lambda t: t.view(__import__("torch").int16).cpu().numpy().view(np.uint16)  # noqa: E731
    wq = S.unpack_nibbles(w["w_codes"].cpu().numpy().reshape(N, K // 2))
    ws = LO.untile_nvfp4_scales(w["w_scales"].cpu().numpy(), N, K)
    a = dev["awq_plain"]
    return {"x_bits": dev["x_bits"], "smooth_inv": w["smooth_inv"].cpu().numpy().astype(np.float64),
            "L1": F.bf16_from_bits(bits(w["L1"])), "L2": F.bf16_from_bits(bits(w["L2"])),
            "w_codes": wq, "w_scales": ws, "bias_bits": dev["bias_bits"],
            "xa": F.bf16_from_bits(dev["xa_bits"]), "q": a["q"], "s": a["s"], "z": a["z"]}


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


def time_oracle(host: dict, budget_s: float, rows: int, cols: int,
                awq_rows: int) -> tuple[float, float, int]:
    """Repeat the oracle sample until `budget_s` elapses; returns (flops, seconds, reps)."""
    flops, t0, reps = 0.0, time.perf_counter(), 0
    while True:
        flops += oracle_sample_step(rows, cols, awq_rows, host)
        reps += 1
        if time.perf_counter() - t0 >= budget_s:
            break
    return flops, time.perf_counter() - t0, reps


def oracle_tiny_layer(budget_s: float) -> dict:
    """The oracle's whole tiny layer (M 256, K 512, N 512, r 16: a1..a6 with the
    weights' prep outside the clock), on one BLAS thread and on all of them."""
    from threadpoolctl import threadpool_limits

    from oracle import prep as P
    from oracle import svdq as S
    sh = WL.TINY
    d = WL.svdq_inputs(sh)
    pr = P.prepare_svdq_layer("nvfp4", d["X"], d["W"], sh.r)
    flops = layer_flops(sh.M, sh.K, sh.N, sh.r)

    def run():
        t0, reps = time.perf_counter(), 0
        while True:
            S.svdq_forward("nvfp4", d["X"], pr["smooth_inv"], pr["L1"], pr["L2"], pr["w_codes"],
                           pr["w_scales"], d["bias"])
            reps += 1
            if time.perf_counter() - t0 >= budget_s:
                return flops * reps / (time.perf_counter() - t0) / 1e9, reps
    with threadpool_limits(1):
        one, reps1 = run()
    allc, repsn = run()
    return {"workload": f"{sh.name}: M={sh.M} K={sh.K} N={sh.N} r={sh.r} NVFP4, the whole layer",
            "gflops_1_thread": round(one, 3), "gflops_all_threads": round(allc, 3),
            "threads": blas_threads(), "reps": [reps1, repsn]}


def awq_plain_host(w_bits: np.ndarray) -> dict:
    from oracle import awq as OA
    from oracle import formats as F
    q, s, z = OA.quantize_weight(F.bf16_from_bits(w_bits))
    return {"q": q, "s": s, "z": z}


def run_reference(args, rank: int) -> None:
    """--impl reference: the oracle on the host cores, bounded samples of the same step."""
    if rank != 0:
        return
    import torch  # noqa: F401  (only for symmetry of the environment)
    from oracle import formats as F
    from oracle import prep as P
    from oracle import svdq as S
    d = WL.svdq_inputs(SHAPE)
    pr = P.prepare_svdq_layer("nvfp4", d["X"], d["W"], SHAPE.r)
    da = WL.awq_inputs(AWQ)
    ap = awq_plain_host(da["W"])
    host = {"x_bits": d["X"], "smooth_inv": pr["smooth_inv"], "L1": pr["L1"], "L2": pr["L2"],
            "w_codes": pr["w_codes"], "w_scales": pr["w_scales"], "bias_bits": d["bias"],
            "xa": F.bf16_from_bits(da["X"]), **ap}
    # size each step so that warmup + steps fit in about two minutes
    per_step = 120.0 / max(1, args.steps + args.warmup)
    rows, cols, awq_rows = 8, 1152, 1152
    t0 = time.perf_counter()
    oracle_sample_step(rows, cols, awq_rows, host)
    base = time.perf_counter() - t0
    if base > per_step:
        shrink = max(1, int(np.ceil(base / per_step)))
        cols, awq_rows = max(16, cols // shrink), max(16, awq_rows // shrink)
    for _ in range(args.warmup):
        oracle_sample_step(rows, cols, awq_rows, host)
    flops, t0 = 0.0, time.perf_counter()
    for _ in range(args.steps):
        flops += oracle_sample_step(rows, cols, awq_rows, host)
    secs = time.perf_counter() - t0
    value = flops / secs / 1e12
    cores = blas_threads()
    sample = sample_text(rows, cols, awq_rows) + " per step"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_block(args.gpus),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


# ------------------------------------------------------------- multi-rank host logic
def rank_rows(x_bits: np.ndarray, rank: int) -> np.ndarray:
    """This rank's token batch (weak scaling: every rank has its own M rows):
    the workload's rows rotated by 37 per rank, so ranks never share a batch."""
    return x_bits if rank == 0 else np.roll(x_bits, 37 * rank, axis=0)


def max_over_ranks(values, world: int, device) -> list:
    """Every rank's per-step times -> their maxima over ranks (the slowest
    rank defines the job's step time). world == 1 returns the values."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.cpu()]


def job_tflops(flops_per_rank_step: float, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: the work of all ranks over the (max-over-ranks) step time."""
    return flops_per_rank_step * world / (ms_per_step * 1e-3) / 1e12


def config_block(n_gpus: int) -> dict:
    return {"workload": f"{SHAPE.name}: SVDQ W4A4 linear M={SHAPE.M} K={SHAPE.K} N={SHAPE.N} "
                        f"r={SHAPE.r} NVFP4 g16 + bias; AWQ W4A16 M={AWQ.M} K={AWQ.K} N={AWQ.N} g64",
            "M": SHAPE.M, "K": SHAPE.K, "N": SHAPE.N, "r": SHAPE.r, "format": "nvfp4_g16",
            "awq": {"M": AWQ.M, "K": AWQ.K, "N": AWQ.N, "group": AWQ.group},
            "l2": "flushed before every step: 256 MiB write, then 256 MiB read (clean lines), "
                  "outside the timed events",
            "parallelism": f"dp{n_gpus} (independent token batches per GPU, no collective)"}


# ------------------------------------------------------------------- our arm
def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-budget", type=float, default=12.0,
                    help="seconds of oracle time for the cpu_baseline leg")
    ap.add_argument("--no-sweep", action="store_true",
                    help="skip the other workloads (for profiling runs of the step)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return

    import torch
    import torch.distributed as dist

    import bit_quantized_diffusion_b200 as bq
    from bit_quantized_diffusion_b200 import prep

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                device_id=dev)

    # ---------------------------------------------------------------- inputs
    d = WL.svdq_inputs(SHAPE)
    x_bits = rank_rows(d["X"], rank)
    to_dev = lambda b: torch.from_numpy(np.ascontiguousarray(b).view(np.int16)).to(dev).view(torch.bfloat16)  # noqa: E731
    X = to_dev(x_bits)
    W = to_dev(d["W"])
    bias = to_dev(d["bias"])
    x_absmax = bq.svdq_column_absmax(X)
    svdq_w = prep.prepare_svdq_weights(W, x_absmax, SHAPE.r, "nvfp4")
    da = WL.awq_inputs(AWQ)
    Xa = to_dev(da["X"])
    awq_w = prep.prepare_awq_weights(to_dev(da["W"]))
    bias_a = to_dev(da["bias"])
    del W
    M, K, N, r = SHAPE.M, SHAPE.K, SHAPE.N, SHAPE.r
    codes = torch.empty(bq.svdq_codes_bytes("nvfp4", M, K), dtype=torch.uint8, device=dev)
    scales = torch.empty(bq.svdq_scales_bytes("nvfp4", M, K), dtype=torch.uint8, device=dev)
    xl1 = torch.empty((bq.svdq_xl1_splits(M, K, r), M, r), dtype=torch.float32, device=dev)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    Ya = torch.empty((AWQ.M, AWQ.N), dtype=torch.bfloat16, device=dev)
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(64 << 20, dtype=torch.float32, device=dev)

    def flush():
        # evict the step's inputs, then replace the dirty lines the write left
        # in L2 with clean ones
        flush_w.zero_()
        flush_r.sum()
    stream = torch.cuda.current_stream()

    def step(ev=None):
        bq.svdq_quantize_act(X, svdq_w["L1s"], svdq_w["smooth_inv"], codes=codes, scales=scales,
                             xl1=xl1, stream=stream)
        if ev is not None:
            ev[0].record(stream)
        bq.svdq_w4a4_linear(codes, scales, xl1, svdq_w["w_codes"], svdq_w["w_scales"], svdq_w["L2"],
                            bias, M, N, K, Y=Y, stream=stream)
        if ev is not None:
            ev[1].record(stream)
        bq.awq_w4a16_linear(Xa, awq_w["qweight"], awq_w["sz"], bias_a, AWQ.N, Y=Ya, stream=stream)

    for _ in range(args.warmup):
        flush()
        step()
    torch.cuda.synchronize()
    if bq.svdq_check_device_status() != 0:
        raise SystemExit("device status reported a timeout during warm-up")

    mk = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    ev_s = [mk() for _ in range(args.steps)]
    ev_e = [mk() for _ in range(args.steps)]
    ev_ks = [mk() for _ in range(args.steps)]
    ev_ke = [mk() for _ in range(args.steps)]
    ev_k = [(mk(), mk()) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        # the timed region: K whole steps, events at step boundaries only (an
        # event recorded between two kernels keeps the second from being
        # launched while the first finishes)
        for i in range(args.steps):
            flush()
            ev_s[i].record(stream)
            step()
            ev_e[i].record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        # the kernel-timing pass: the same K steps with an event between every
        # two kernels; each kernel's time here includes its launch gap
        for i in range(args.steps):
            flush()
            ev_ks[i].record(stream)
            step(ev_k[i])
            ev_ke[i].record(stream)
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    step_ms = sum(a.elapsed_time(b) for a, b in zip(ev_s, ev_e))
    k1_ms = sum(a.elapsed_time(b[0]) for a, b in zip(ev_ks, ev_k)) / args.steps
    k2_ms = sum(b[0].elapsed_time(b[1]) for b in ev_k) / args.steps
    k3_ms = sum(b[1].elapsed_time(e) for b, e in zip(ev_k, ev_ke)) / args.steps
    status = bq.svdq_check_device_status()
    # The event floor: a one-element torch kernel timed the same way (flush, event,
    # kernel, event). Every event-to-event figure above carries it; for the short
    # kernels it is a large part of their time.
    tiny = torch.zeros(1, device=dev)
    ev_f = [(mk(), mk()) for _ in range(args.steps + 3)]
    for i in range(args.steps + 3):
        flush()
        ev_f[i][0].record(stream)
        tiny.add_(1.0)
        ev_f[i][1].record(stream)
    torch.cuda.synchronize()
    floor_ms = sorted(a.elapsed_time(b) for a, b in ev_f[3:])[args.steps // 2]

    # ------------------------------ two-level NVFP4 on the same layer (per-tensor scales)
    # The same X and weights, quantized with a per-tensor float32 scale above the
    # group scales: the tensor scale of the smoothed activation, the two-level
    # quantizer and the two-level GEMM, each timed event to event after the flush.
    w_tscale = bq.svdq_tensor_scale(svdq_w["R"])
    wc2, ws2, _ = bq.svdq_quantize_act_two_level(svdq_w["R"], w_tscale)
    a_tscale = torch.empty(2, dtype=torch.float32, device=dev)
    codes2, scales2 = torch.empty_like(codes), torch.empty_like(scales)
    xl1_2 = torch.empty_like(xl1)
    Y2 = torch.empty_like(Y)
    n2 = max(3, min(args.steps, 200))
    ev2 = [[mk() for _ in range(4)] for _ in range(n2 + 3)]
    for i in range(n2 + 3):
        flush()
        ev2[i][0].record(stream)
        bq.svdq_tensor_scale(X, svdq_w["smooth_inv"], a_tscale, stream=stream)
        ev2[i][1].record(stream)
        _, _, xl1_view = bq.svdq_quantize_act_two_level(X, a_tscale, svdq_w["L1s"], svdq_w["smooth_inv"],
                                                        codes=codes2, scales=scales2, xl1=xl1_2,
                                                        stream=stream)
        ev2[i][2].record(stream)
        bq.svdq_w4a4_linear_two_level(codes2, scales2, a_tscale, xl1_view, wc2, ws2, w_tscale,
                                      svdq_w["L2"], bias, M, N, K, Y=Y2, stream=stream)
        ev2[i][3].record(stream)
    torch.cuda.synchronize()
    tl = [sum(e[j].elapsed_time(e[j + 1]) for e in ev2[3:]) / n2 for j in range(3)]
    status = status or bq.svdq_check_device_status()

    # ------------------- the same layer as a fused QKV projection (norm + rotation epilogue)
    # The QKV layer's 9216 columns are 24 heads each of Q, K and V; the GEMM with the
    # per-head RMS norm of Q and K and the rotation by row-position angles in its
    # epilogue, timed event to event after the flush, against the plain GEMM above.
    qe = WL.qkv_epilogue_inputs(M, seed=SHAPE.seed + 100, angles="positions")
    norm_q, norm_k = to_dev(qe["norm_q"]), to_dev(qe["norm_k"])
    rope_cos = torch.from_numpy(np.ascontiguousarray(qe["cos"].T)).to(dev)  # angle-major [64, M]
    rope_sin = torch.from_numpy(np.ascontiguousarray(qe["sin"].T)).to(dev)
    Y3 = torch.empty_like(Y)
    ev3 = [[mk() for _ in range(2)] for _ in range(n2 + 3)]
    for i in range(n2 + 3):
        flush()
        ev3[i][0].record(stream)
        bq.svdq_w4a4_linear_qkv_norm_rope(codes, scales, xl1, svdq_w["w_codes"], svdq_w["w_scales"],
                                          svdq_w["L2"], bias, norm_q, norm_k, rope_cos, rope_sin, M, N, K,
                                          Y=Y3, stream=stream)
        ev3[i][1].record(stream)
    torch.cuda.synchronize()
    t_qkv = sum(e[0].elapsed_time(e[1]) for e in ev3[3:]) / n2
    status = status or bq.svdq_check_device_status()

    # ------------------------------- the other workloads and AWQ at more tokens
    sweep, awq_tokens, mlp = None, None, None
    if not args.no_sweep and rank == 0:
        peaks0 = measured_peaks()
        sweep = sweep_layers(bq, prep, dev, flush, max(3, min(args.steps, 50)),
                             peaks0["bf16_tflops"] * FP4_OVER_BF16)
        awq_tokens = awq_by_tokens(bq, awq_w, bias_a, dev, flush, max(3, min(args.steps, 50)))
        mlp = mlp_pair(bq, prep, dev, flush, max(3, min(args.steps, 50)))

    # ----------------------------------------------- end to end, host buffers
    Xh = torch.empty(X.shape, dtype=X.dtype, pin_memory=True)
    Xh.copy_(X)
    Xah = torch.empty(Xa.shape, dtype=Xa.dtype, pin_memory=True)
    Xah.copy_(Xa)
    Yh = torch.empty(Y.shape, dtype=Y.dtype, pin_memory=True)
    Yah = torch.empty(Ya.shape, dtype=Ya.dtype, pin_memory=True)
    e2e_steps = max(3, min(args.steps, 50))
    e_s = [mk() for _ in range(e2e_steps)]
    e_e = [mk() for _ in range(e2e_steps)]
    for _ in range(3):
        X.copy_(Xh, non_blocking=True)
        step()
        Yh.copy_(Y, non_blocking=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    for i in range(e2e_steps):
        flush()
        e_s[i].record(stream)
        X.copy_(Xh, non_blocking=True)
        Xa.copy_(Xah, non_blocking=True)
        step()
        Y_host = Yh.copy_(Y, non_blocking=True)
        Yah.copy_(Ya, non_blocking=True)
        e_e[i].record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e2e_ms = sum(a.elapsed_time(b) for a, b in zip(e_s, e_e)) / e2e_steps
    del Y_host

    # ------------------------------------------------- max over ranks
    ms_step, ms_e2e, ms_k2 = max_over_ranks([step_ms / args.steps, e2e_ms, k2_ms], world, dev)

    # ------------------------------------------------- context: cuBLAS bf16
    cublas_tflops = None
    if rank == 0:
        A = torch.randn((M, K), dtype=torch.bfloat16, device=dev)
        B = torch.randn((N, K), dtype=torch.bfloat16, device=dev)
        for _ in range(3):
            torch.matmul(A, B.T)
        e0, e1 = mk(), mk()
        e0.record(stream)
        for _ in range(20):
            torch.matmul(A, B.T)
        e1.record(stream)
        torch.cuda.synchronize()
        cublas_tflops = 2.0 * M * N * K / (e0.elapsed_time(e1) / 20 * 1e-3) / 1e12
        del A, B

    # ------------------------------------------------- CPU baseline (oracle)
    cpu = None
    if rank == 0 and world == 1 and args.cpu_budget > 0:
        host = oracle_inputs_from_device({"svdq": svdq_w, "x_bits": x_bits, "bias_bits": d["bias"],
                                          "xa_bits": da["X"], "awq_plain": awq_plain_host(da["W"])})
        flops, secs, reps = time_oracle(host, args.cpu_budget, 8, 1152, 1152)
        cpu = {"value": flops / secs / 1e12, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
               "sample": f"{reps} x ({sample_text(8, 1152, 1152)}), {secs:.1f} s",
               "host_cores": HOST_CORES,
               "tiny_layer": oracle_tiny_layer(min(3.0, args.cpu_budget / 4))}

    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return
    peaks = measured_peaks()
    clk = clocks.summary()
    # The burst GEMM figure applies while the clocks stay at their maximum; once
    # the power cap pulls them down, the sustained one does.
    capped = "sw_power_cap" in clk.get("reasons", [])
    peak_kind = "sustained" if capped else "burst"
    bf16_peak = peaks["bf16_tflops_sustained"] if capped else peaks["bf16_tflops"]
    fp4_peak = bf16_peak * FP4_OVER_BF16
    k2_flops = 2.0 * M * N * K
    achieved = k2_flops / (ms_k2 * 1e-3) / 1e12
    value = job_tflops(step_flops(), world, ms_step)
    traffic = recorded_traffic("w4a4_nvfp4_gemm_kernel")
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "nvfp4 (e2m1 x ue4m3, f32 accumulate)", "data": "synthetic",
        "config": config_block(world),
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": fp4_peak, "unit": "TFLOP/s",
                     "frac": achieved / fp4_peak, "traffic": traffic,
                     "frac_vs_nominal": achieved / NOMINAL_FP4_TFLOPS,
                     "kernel": "w4a4_nvfp4_gemm_kernel",
                     "peak_note": f"peak = {peaks['source']} bf16 {peak_kind} x {FP4_OVER_BF16:g} "
                                  f"(nominal FP4/BF16 ratio; no FP4 peak is measured), so frac is of the "
                                  f"measured-bf16-scaled FP4 peak; frac_vs_nominal is of the nominal dense "
                                  f"FP4 {NOMINAL_FP4_TFLOPS:g} TFLOP/s"},
        "roofline_hbm": {
            "svdq_quantize_act": {
                "bound": "hbm", "unit": "GB/s", "peak": peaks["hbm_gbs"],
                "achieved": quantize_bytes(M, K, r) / (k1_ms * 1e-3) / 1e9,
                "frac": quantize_bytes(M, K, r) / (k1_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                "algorithmic_bytes": quantize_bytes(M, K, r),
                "traffic": sum_traffic(("quantize_act_kernel", "xl1_reduce_kernel")),
                "kernels": "quantize_act_kernel + xl1_reduce_kernel (K-split partial sums)",
                "us": k1_ms * 1e3,
                "frac_net_of_event_floor": quantize_bytes(M, K, r) / ((k1_ms - floor_ms) * 1e-3) / 1e9
                / peaks["hbm_gbs"]},
            "awq_w4a16_linear": {
                "bound": "hbm", "unit": "GB/s", "peak": peaks["hbm_gbs"],
                "achieved": awq_bytes(AWQ.M, AWQ.K, AWQ.N) / (k3_ms * 1e-3) / 1e9,
                "frac": awq_bytes(AWQ.M, AWQ.K, AWQ.N) / (k3_ms * 1e-3) / 1e9 / peaks["hbm_gbs"],
                "algorithmic_bytes": awq_bytes(AWQ.M, AWQ.K, AWQ.N),
                "traffic": sum_traffic((AWQ_KERNEL,)),
                "kernels": AWQ_KERNEL,
                "us": k3_ms * 1e3,
                "frac_net_of_event_floor": awq_bytes(AWQ.M, AWQ.K, AWQ.N) / ((k3_ms - floor_ms) * 1e-3) / 1e9
                / peaks["hbm_gbs"]},
            "event_floor_us": floor_ms * 1e3,
            "peak_note": f"{peaks['source']} HBM copy bandwidth; achieved = algorithmic bytes / "
                         f"event-to-event time in the kernel-timing pass; frac_net_of_event_floor "
                         f"takes event_floor_us (a one-element torch kernel timed the same way, "
                         f"flush, event, kernel, event) off that time"},
        "cpu_baseline": cpu,
        "e2e": {"value": job_tflops(step_flops(), world, ms_e2e), "unit": UNIT,
                "h2d_bytes_per_step": X.numel() * 2 + Xa.numel() * 2,
                "d2h_bytes_per_step": Y.numel() * 2 + Ya.numel() * 2, "ms_per_step": ms_e2e},
        "gpu_launches": launches_per_step(M, K, r, AWQ.M) * args.steps,
        "clocks": clk,
        "kernels": {
            "timing": "kernel-timing pass: the timed region's K steps again, one CUDA event "
                      "between every two kernels on the launch stream (no launch overlap)",
            "svdq_quantize_act_us": k1_ms * 1e3,
            "svdq_quantize_act_gbs": quantize_bytes(M, K, r) / (k1_ms * 1e-3) / 1e9,
            "svdq_w4a4_linear_us": k2_ms * 1e3,
            "svdq_w4a4_linear_tflops_4bit": achieved,
            "svdq_w4a4_linear_tflops_incl_lowrank": layer_flops(M, K, N, r) / (k2_ms * 1e-3) / 1e12,
            "layer_tflops": k2_flops / ((k1_ms + k2_ms) * 1e-3) / 1e12,
            "awq_w4a16_linear_us": k3_ms * 1e3,
            "awq_w4a16_linear_gbs": awq_bytes(AWQ.M, AWQ.K, AWQ.N) / (k3_ms * 1e-3) / 1e9,
            "hbm_peak_gbs": peaks["hbm_gbs"],
            "cublas_bf16_tflops_same_shape": cublas_tflops,
            "two_level_nvfp4": {
                "timing": f"the same layer with per-tensor float32 scales, {n2} steps, event to event",
                "svdq_tensor_scale_us": tl[0] * 1e3,
                "svdq_quantize_act_two_level_us": tl[1] * 1e3,
                "svdq_w4a4_linear_two_level_us": tl[2] * 1e3,
                "svdq_w4a4_linear_two_level_tflops_4bit": k2_flops / (tl[2] * 1e-3) / 1e12,
            },
            "fused_qkv_norm_rope": {
                "timing": f"the same layer as Q, K, V of 24 heads of 128, per-head RMS norm of Q and K "
                          f"and the pairwise rotation in the GEMM epilogue, {n2} steps, event to event",
                "svdq_w4a4_linear_qkv_norm_rope_us": t_qkv * 1e3,
                "svdq_w4a4_linear_qkv_norm_rope_tflops_4bit": k2_flops / (t_qkv * 1e-3) / 1e12,
            },
        },
        "device_status": status,
    }
    if sweep is not None:
        out["kernels"]["workloads"] = {
            "timing": "each layer's quantizer and GEMM called alone after the L2 flush, event to event, "
                      "median of the calls",
            **sweep}
        out["kernels"]["fused_mlp"] = {
            "timing": "the whole MLP pair per call, event to event after the flush, median", **mlp}
        out["kernels"]["awq_by_tokens"] = {
            "timing": f"awq_w4a16_linear at K={AWQ.K} N={AWQ.N}, event to event after the flush, median; "
                      f"the GEMV (warp-level MMA) serves M <= 64, the tensor-core GEMM any M",
            **awq_tokens}
    print(json.dumps(out), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
