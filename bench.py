"""Benchmark of the Hadamard-rotated INT8 linear layer on B200.

One step = one pass of the online hot path over one batch of synthetic input: rotate +
quantize the activations (per-token scales) and run the tensor-core int8 matmul with the
fused fp32 de-quant epilogue (plus the LoRA term, or the MLP chain, for those workloads).
Weights are rotated and quantized once before timing (offline, as on the pages).

Default workload: the DiT MLP pair, x [4608, 3840] bf16 Student-t(4) activations through the
up-projection W_up [10240, 3840] with GELU in its epilogue, per-token requantisation of the
hidden layer and the down-projection W_down [3840, 10240], Hadamard group 256 (725 GOP of int8
matmul per step).

Output: one JSON line on rank 0. ``value`` is int8 TOPS of the whole step (2*M*N*K per
GEMM over the device time of every kernel of the step), summed over ranks (replicas:
each rank runs its own copy of the workload, no data-path collective).

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--group G]
  python bench.py --impl reference   # the CPU oracle on a bounded sample, same metric
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "int8 rotated-linear TOPS and % of dense INT8 peak; rotate+quant HBM GB/s"
INT8_SPEC_TOPS = 4500.0        # B200 dense INT8, NVIDIA public spec
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
NOMINAL_INT8_OVER_BF16 = 2.0   # 4.5 / 2.25 PFLOP/s dense
HBM_SPEC_GBS = 8000.0          # B200 HBM3e, NVIDIA public spec (8 TB/s)


def clock_scaled_peak(peak, clocks):
    """The peak scaled by the run's median SM clock under load over the GPU's maximum SM
    clock (the tensor cores' rate is proportional to the SM clock); None without samples."""
    mhz, max_mhz = clocks.get("sm_mhz"), clocks.get("sm_max_mhz")
    if not mhz or not max_mhz:
        return None
    return peak * min(1.0, float(mhz) / float(max_mhz))


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# The sources each profiled kernel is compiled from (its own header and the shared PTX
# helpers): an ncu summary stays valid until one of these changes.
KERNEL_SOURCES = {
    "gemm_s8": ("device.cuh", "gemm.cuh", "gemm_pair.cuh", "gelu.cuh", "rotquant.cuh"),
    "lora_down": ("device.cuh", "lora_down.cuh"),
    "rotquant": ("device.cuh", "rotquant.cuh"),
    "attn_kernel": ("device.cuh", "rotquant.cuh", "attention.cuh"),
}


def _code_only(text: str) -> str:
    """Source text without comments and with whitespace collapsed: a comment edit does not
    change the kernel, so it does not make a profile stale."""
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "hadamard_rotated_int8_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode() + _code_only(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(profile: str, kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary `profiles/<profile>_<workload>.md`
    of a kernel of family `kernel`, if it was taken on the current kernel sources; else
    None."""
    path = os.path.join(ROOT, "profiles", f"{profile}_{workload}.md")
    try:
        text = open(path).read()
    except OSError:
        return None
    fields = {}
    for line in text.splitlines():
        if line.startswith("- ") and ":" in line:
            k, v = line[2:].split(":", 1)
            fields[k.strip()] = v.strip().strip("`")
    if fields.get("kernel_source_hash") != kernel_source_hash(kernel):
        return None
    try:
        return float(fields["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------------- workloads

def workload_ops(case, name):
    """int8 GEMM ops (2*M*N*K summed over the step's GEMMs) and extra bf16 LoRA flops; for
    attention, the int8 QK ops and the bf16 PV flops (2 L^2 D per head each)."""
    if case.extra.get("attn"):
        qk = 2 * case.extra["B"] * case.N * case.M * case.M * case.K
        return 2 * qk, 0
    if name.startswith("grad_"):
        return 2 * case.M * case.N * case.K, 0   # dy [M, N] x qW [N, K]
    if name.startswith("dit_mlp"):
        return 2 * 2 * case.M * case.N * case.K, 0
    lora = 0
    if case.A is not None:
        r = case.A.shape[1]
        lora = 2 * case.M * case.K * r + 2 * case.M * r * case.N
    return 2 * case.M * case.N * case.K, lora


def rotquant_bytes(M, K):
    return M * K * 2 + M * K + M * 4   # read bf16, write int8 codes, write fp32 scale


def rotquant_kernel_name(case, rows_k, grad, fp8):
    """The quantizer kernel the library launches for rows of `rows_k` elements (the run-per-lane
    kernel up to 512 runs of 64; the input gradient's column-multiplier mode on the
    chunk-per-warp kernels)."""
    if case.extra.get("attn"):
        return "attention quantizers (smooth_k means, q and k short-row quantizers)"
    f = str(fp8).lower()
    if grad:
        # the output gradient is quantized per token without a rotation (group 1), with the
        # weight's row scales as column multipliers
        kind = "rotquant_persistent_kernel" if (rows_k + 1023) // 1024 <= 16 else "rotquant_kernel"
        return f"{kind}<1,true,{f}>"
    if rows_k <= 32768:
        return f"rotquant_run_kernel<{case.g},{f},V8>"
    return f"rotquant_kernel<{case.g},false,{f}>"


class Step:
    """Device buffers and the stages of one step of a workload."""

    def __init__(self, name, case, sd, torch):
        self.name, self.case, self.sd, self.torch = name, case, sd, torch
        dev = "cuda"
        g = case.g
        self.x = case.x.to(dev)
        self.qx = torch.empty((case.M, case.K), dtype=torch.int8, device=dev)
        self.sx = torch.empty((case.M,), dtype=torch.float32, device=dev)
        self.bias = case.bias.to(dev) if case.bias is not None else None
        if not case.extra.get("attn") and not name.startswith("fp8_"):
            self.qW, self.sW = sd.sdnq_rotate_quant_weight(case.W.to(dev), g)
        self.out = torch.empty((case.M, case.N), dtype=torch.bfloat16, device=dev)
        self.gemm_stages = []
        if case.extra.get("attn"):
            B, L, H, D = case.extra["B"], case.M, case.N, case.K
            self.k = case.W.to(dev)
            self.v = case.extra["v"].to(dev)
            self.out = torch.empty((B, L, H, D), dtype=torch.bfloat16, device=dev)
            total, _ = sd._native.attention_workspace(B, L, L, H, D)
            self.ws = torch.empty(total, dtype=torch.uint8, device=dev)
            self.stages = [
                ("rotquant", lambda: sd._native.sdnq_attention_prep(self.x, self.k, g, ws=self.ws)),
                ("attention", lambda: sd._native.sdnq_attention_core(self.v, L, self.ws, out=self.out)),
            ]
            self.gemm_stages = ["attention"]
            self.launches = 5   # two for the key means, two quantizers, the attention kernel
        elif name.startswith("fp8_"):
            # the FP8 (e4m3) variant: rotate + quantize to e4m3, then the kind::f8f6f4 GEMM
            self.qW, self.sW = sd.sdnq_rotquant_fp8(case.W.to(dev), g)
            self.qx = torch.empty((case.M, case.K), dtype=torch.uint8, device=dev)
            self.stages = [
                ("rotquant", lambda: sd.sdnq_rotquant_fp8(self.x, g, self.qx, self.sx)),
                ("gemm", lambda: sd.sdnq_fp8_linear(self.qx, self.sx, self.qW, self.sW,
                                                    self.bias, out=self.out)),
            ]
            self.gemm_stages = ["gemm"]
            self.launches = 2
        elif name.startswith("grad_"):
            # backward through the frozen layer: x holds dy [M, N]; W is [N, K]
            self.out = torch.empty((case.M, case.K), dtype=torch.bfloat16, device=dev)
            self.qx = torch.empty((case.M, case.N), dtype=torch.int8, device=dev)
            self.stages = [
                ("rotquant", lambda: sd.sdnq_quant_grad_output(self.x, self.sW, self.qx, self.sx)),
                ("gemm_grad", lambda: sd.sdnq_int8_grad_input_gemm(self.qx, self.sx, self.qW,
                                                                   g, out=self.out)),
            ]
            self.gemm_stages = ["gemm_grad"]
            self.launches = 2
        elif name.startswith("dit_mlp"):
            Wd = case.extra["W_down"].to(dev)
            self.qWd, self.sWd = sd.sdnq_rotate_quant_weight(Wd, g)
            self.h = torch.empty((case.M, case.N), dtype=torch.bfloat16, device=dev)
            self.qh = torch.empty((case.M, case.N), dtype=torch.int8, device=dev)
            self.sh = torch.empty((case.M,), dtype=torch.float32, device=dev)
            self.down = torch.empty((case.M, case.K), dtype=torch.bfloat16, device=dev)
            self.stages = [
                ("rotquant", lambda: sd.sdnq_rotquant_act(self.x, g, self.qx, self.sx)),
                # up-projection with GELU in its epilogue: h = bf16(GELU(bf16(up)))
                ("gemm_up", lambda: sd.sdnq_int8_linear_gelu(self.qx, self.sx, self.qW, self.sW,
                                                             None, out=self.h)),
                ("rotquant_h", lambda: sd.sdnq_rotquant_act(self.h, g, self.qh, self.sh)),
                ("gemm_down", lambda: sd.sdnq_int8_linear(self.qh, self.sh, self.qWd, self.sWd,
                                                          None, out=self.down)),
            ]
            self.gemm_stages = ["gemm_up", "gemm_down"]
            self.launches = 4
        elif case.A is not None:
            self.A, self.B = case.A.to(dev), case.B.to(dev)
            self.u = torch.empty((case.M, case.A.shape[1]), dtype=torch.bfloat16, device=dev)
            # sdnq_int8_linear_lora as its two calls (the same kernels and bits), so that the
            # GEMM with the adapter term is timed on its own
            self.stages = [
                ("rotquant", lambda: sd.sdnq_rotquant_act(self.x, g, self.qx, self.sx)),
                ("lora_down", lambda: sd.sdnq_lora_down(self.x, self.A, u=self.u)),
                ("gemm_lora", lambda: sd.sdnq_int8_linear_lora_up(
                    self.qx, self.sx, self.qW, self.sW, self.bias, self.u, self.B,
                    case.lora_scale, out=self.out)),
            ]
            self.gemm_stages = ["gemm_lora"]
            self.launches = 3  # rotquant, LoRA down-projection, GEMM with the adapter term
        elif sd.sdnq_int8_linear_fused_plan(case.M, case.N, case.K):
            # the library's own choice for sdnq_int8_linear_fused (one launch here)
            # one launch: the activation quantizer runs inside the GEMM kernel
            self.sync = torch.zeros(4 * ((case.M + 127) // 128) + 64, dtype=torch.int32,
                                    device=dev)
            self.stages = [
                ("fused", lambda: sd.sdnq_int8_linear_fused(
                    self.x, g, self.qW, self.sW, self.bias, qx_ws=self.qx, sx_ws=self.sx,
                    sync_ws=self.sync, out=self.out)),
            ]
            self.gemm_stages = ["fused"]
            self.launches = 1
        else:
            self.stages = [
                ("rotquant", lambda: sd.sdnq_rotquant_act(self.x, g, self.qx, self.sx)),
                ("gemm", lambda: sd.sdnq_int8_linear(self.qx, self.sx, self.qW, self.sW,
                                                     self.bias, out=self.out)),
            ]
            self.gemm_stages = ["gemm"]
            self.launches = 2

    def run(self):
        for _, fn in self.stages:
            fn()


class ClockSampler:
    """Samples SM clock and throttle reasons with NVML while the timed region runs."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.01):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # pragma: no cover - NVML missing
            log(f"clock sampling unavailable: {e}")
            self.nvml = None

    def _loop(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nvml.nvmlDeviceGetClockInfo(self.h, self.nvml.NVML_CLOCK_SM))
                mask = self.nvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in self.REASONS.items():
                    if mask & bit and bit != 0x1:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nvml is not None:
            self._t = threading.Thread(target=self._loop, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples)}


# ---------------------------------------------------------------------- CPU oracle timing

def oracle_step(case, rows, nthreads):
    """The oracle's pass over `rows` tokens of the workload (weights already quantized)."""
    import oracle
    from hadamard_rotated_int8_b200 import synthetic
    if case.extra.get("attn"):
        import numpy as np
        qb = np.ascontiguousarray(synthetic.bits(case.x)[:, :rows])
        oracle.attention(qb, synthetic.bits(case.W), synthetic.bits(case.extra["v"]), case.g,
                         nthreads=nthreads)
        return
    xb = synthetic.bits(case.x)[:rows]
    if case.extra.get("fp8"):
        qx, sx = oracle.rotate_quantize_fp8(xb, case.g, nthreads)
        acc = oracle.gemm_fp8(qx, case._oracle_qW, nthreads)
        bias = synthetic.bits(case.bias) if case.bias is not None else None
        oracle.dequant_epilogue_f32(acc, sx, case._oracle_sW, bias, nthreads)
        return
    if case.extra.get("grad"):
        qg, sg = oracle.colscale_quantize(xb, case._oracle_sW, nthreads)
        acc = oracle.gemm_s8_nn(qg, case._oracle_qW, nthreads)
        oracle.grad_input_epilogue(acc, sg, case.g, nthreads)
        return
    qx, sx = oracle.rotate_quantize(xb, case.g, nthreads)
    acc = oracle.gemm_s8(qx, case._oracle_qW, nthreads)
    L = None
    if case.A is not None:
        u = oracle.lora_down(xb, synthetic.bits(case.A), nthreads)
        L = oracle.lora_up(u, synthetic.bits(case.B), nthreads)
    bias = synthetic.bits(case.bias) if case.bias is not None else None
    out = oracle.dequant_epilogue(acc, sx, case._oracle_sW, bias, L, case.lora_scale, nthreads)
    if case._oracle_down is not None:
        h = oracle.gelu_bf16(out, nthreads)
        qh, sh = oracle.rotate_quantize(h, case.g, nthreads)
        acc2 = oracle.gemm_s8(qh, case._oracle_down[0], nthreads)
        oracle.dequant_epilogue(acc2, sh, case._oracle_down[1], None, None, 1.0, nthreads)


def oracle_prepare(case, name, nthreads):
    import oracle
    from hadamard_rotated_int8_b200 import synthetic
    if case.extra.get("attn"):
        case._oracle_down = None
        return
    quant = oracle.rotate_quantize_fp8 if case.extra.get("fp8") else oracle.rotate_quantize
    case._oracle_qW, case._oracle_sW = quant(synthetic.bits(case.W), case.g, nthreads)
    case._oracle_down = None
    if name.startswith("dit_mlp"):
        case._oracle_down = oracle.rotate_quantize(synthetic.bits(case.extra["W_down"]), case.g,
                                                   nthreads)


def oracle_rows_for(case, name, nthreads, seconds):
    """Rows (tokens) of the workload the oracle processes in about `seconds`."""
    ops_full, _ = workload_ops(case, name)
    probe = max(1, min(case.M, 16))
    t0 = time.perf_counter()
    oracle_step(case, probe, nthreads)
    dt = max(time.perf_counter() - t0, 1e-4)
    per_row = dt / probe
    return int(max(1, min(case.M, seconds / per_row))), ops_full / case.M


def cpu_baseline(case, name, budget_s=12.0):
    nthreads = os.cpu_count() or 1
    oracle_prepare(case, name, nthreads)
    rows, ops_per_row = oracle_rows_for(case, name, nthreads, budget_s / 2)
    reps, total, t_start = 0, 0.0, time.perf_counter()
    while reps < 1 or (time.perf_counter() - t_start < budget_s and reps < 64):
        t0 = time.perf_counter()
        oracle_step(case, rows, nthreads)
        total += time.perf_counter() - t0
        reps += 1
    tops = ops_per_row * rows * reps / total / 1e12
    return {"value": tops, "unit": "TOPS", "cores": nthreads, "kind": "oracle",
            "sample": (f"{rows} of {case.M} query tokens of {name} x{reps} (smooth_k means, "
                       f"rotate + int8 of q and k, int32 logits, fp64 softmax and PV over all "
                       f"{case.M} keys of {case.N} heads), {total:.2f} s") if case.extra.get("attn") else
                      (f"{rows} of {case.M} tokens of {name} x{reps} (int8 of dy*sW, NN int8 "
                       f"GEMM against the {case.N}x{case.K} codes, inverse-rotation epilogue), "
                       f"{total:.2f} s") if case.extra.get("grad") else
                      (f"{rows} of {case.M} tokens of {name} x{reps} (rotate+quantize, int8 GEMM "
                       f"against all {case.N} weight rows, fp32 epilogue), {total:.2f} s")}


def run_reference(args):
    """The reference arm: the CPU oracle as it stands, on the machine's host cores, timed on a
    bounded sample of the same workload per step."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from hadamard_rotated_int8_b200 import synthetic
    case = synthetic.workload(args.workload, g=args.group)
    nthreads = os.cpu_count() or 1
    oracle_prepare(case, args.workload, nthreads)
    per_step_budget = max(0.05, 150.0 / max(1, args.steps + args.warmup))
    rows, ops_per_row = oracle_rows_for(case, args.workload, nthreads, per_step_budget)
    for _ in range(args.warmup):
        oracle_step(case, rows, nthreads)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_step(case, rows, nthreads)
    dt = time.perf_counter() - t0
    tops = ops_per_row * rows * args.steps / dt / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": tops, "unit": "TOPS",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e4m3" if args.workload.startswith("fp8_") else "int8",
        "data": "synthetic",
        "config": config_of(case, args),
        "cpu_baseline": {"value": tops, "unit": "TOPS", "cores": nthreads, "kind": "oracle",
                         "sample": f"{rows} of {case.M} tokens per step"},
        "e2e": {"value": tops, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


class L2Flush:
    """Leaves L2 cold before a timed step: writes a buffer of twice the L2 size (evicting
    everything the step could reuse), then reads a second one of the same size, so that the
    flush's own dirty lines are written back here, outside the timed region, and not during
    the step."""

    def __init__(self, torch, l2_bytes):
        n = max(2 * l2_bytes, 256 << 20)
        self.w = torch.empty(n, dtype=torch.uint8, device="cuda")
        self.r = torch.ones(n // 4, dtype=torch.int32, device="cuda")
        self.sink = torch.empty((), dtype=torch.int32, device="cuda")

    def __call__(self):
        self.w.zero_()
        import torch as _t
        _t.amax(self.r, dim=0, out=self.sink)


def standalone_rotquant_ms(step, flush, torch, sd, reps):
    times = []
    for i in range(reps + 3):
        flush()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        sd.sdnq_rotquant_act(step.x, step.case.g, step.qx, step.sx)
        e1.record()
        torch.cuda.synchronize()
        if i >= 3:
            times.append(e0.elapsed_time(e1))
    return sum(times) / len(times)


def reduce_max_over_ranks(values, dist=None, world=1, device="cuda"):
    """Element-wise max of a list of floats over all ranks (the slowest rank's times)."""
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t]


def whole_job_tops(ops_per_rank, world, ms_per_step):
    """Aggregate throughput of N replicas: every rank's work over the slowest rank's time."""
    return world * ops_per_rank / (ms_per_step * 1e-3) / 1e12


def config_of(case, args):
    c = {"workload": args.workload, "M": case.M, "N": case.N, "K": case.K,
         "hadamard_group": case.g, "bias": case.bias is not None,
         "lora_rank": case.A.shape[1] if case.A is not None else 0,
         "parallelism": f"replicas x{args.gpus}",
         "l2": "flushed before every timed step: write of 2x the L2 size, then a read of "
               "another 2x the L2 size (the flush's dirty lines are written back before the "
               "step, not during it)"}
    if args.workload.startswith("dit_mlp"):
        c["chain"] = "rotquant -> up GEMM with GELU epilogue -> rotquant -> down GEMM"
    if case.extra.get("attn"):
        c["attention"] = {"B": case.extra["B"], "L": case.M, "H": case.N, "D": case.K,
                          "qk": "int8, Hadamard-rotated, smooth_k", "pv": "bf16",
                          "ops": "int8 QK 2 L^2 D H + bf16 PV 2 L^2 D H"}
    if args.workload.startswith("grad_"):
        c["chain"] = ("input gradient of a frozen [N, K] layer: int8 of dy*sW [M, N] -> "
                      "NN int8 GEMM with row scale + inverse Hadamard epilogue -> dx [M, K]")
    return c


# ---------------------------------------------------------------------- GPU arm

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="sdnq", choices=["sdnq", "reference"])
    ap.add_argument("--workload", default="dit_mlp_4608x3840x10240")
    ap.add_argument("--group", type=int, default=None)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        log("warmup raised to 3 (timing rules)")
        args.warmup = 3

    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist
    import hadamard_rotated_int8_b200 as sd
    from hadamard_rotated_int8_b200 import _build, synthetic

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    if rank == 0:
        _build.build()
    if world > 1:
        dist.barrier()
    sd.lib()

    case = synthetic.workload(args.workload, g=args.group)
    step = Step(args.workload, case, sd, torch)
    l2 = torch.cuda.get_device_properties(local).L2_cache_size
    flush = L2Flush(torch, l2)
    names = [n for n, _ in step.stages]

    for _ in range(args.warmup):
        flush()
        step.run()
    torch.cuda.synchronize()
    assert sd.sdnq_device_status() == 0

    # timed region: K steps, L2 flushed before each, one CUDA event pair around each step on
    # the stream (nothing between the step's launches, so a kernel launched programmatically
    # may overlap the tail of the one before it, as in use)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        for i in range(args.steps):
            flush()
            evs[i][0].record()
            for _, fn in step.stages:
                fn()
            evs[i][1].record()
        torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    step_ms_each = [e[0].elapsed_time(e[1]) for e in evs]
    step_ms_total = sum(step_ms_each)

    # per-kernel times for the rooflines: the same K steps again with an event between the
    # stages (which serialises them)
    sevs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(names) + 1)]
            for _ in range(args.steps)]
    for i in range(args.steps):
        flush()
        e = sevs[i]
        e[0].record()
        for j, (_, fn) in enumerate(step.stages):
            fn()
            e[j + 1].record()
    torch.cuda.synchronize()
    stage_ms = {n: 0.0 for n in names}
    for e in sevs:
        for j, n in enumerate(names):
            stage_ms[n] += e[j].elapsed_time(e[j + 1])
    t = reduce_max_over_ranks([step_ms_total, statistics.median(step_ms_each), min(step_ms_each)]
                              + [stage_ms[n] for n in names], dist, world)
    step_ms_total, step_ms_median, step_ms_best = t[0], t[1], t[2]
    stage_ms = {n: t[3 + j] for j, n in enumerate(names)}
    assert sd.sdnq_device_status() == 0

    ops, lora_flops = workload_ops(case, args.workload)
    ms_per_step = step_ms_total / args.steps
    value = whole_job_tops(ops, world, ms_per_step)

    # end to end through the public API: every step copies its input from pinned host memory
    # to the device, runs, and copies its result back, inside the timed region. Copies in,
    # compute and copies out run on three streams over two sets of device buffers, so step
    # i + 1's upload and step i - 1's download overlap step i (PCIe is full duplex), as a
    # serving loop would run them.
    e2e = None
    if not args.no_e2e:
        n_e2e = max(3, min(args.steps, 50))
        sets = [step, Step(args.workload, case, sd, torch)]
        mlp = args.workload.startswith("dit_mlp")
        x_host = case.x.pin_memory()
        extra_host = ([case.W.pin_memory(), case.extra["v"].pin_memory()]
                      if case.extra.get("attn") else [])

        def device_inputs(st):
            return [st.x] + ([st.k, st.v] if case.extra.get("attn") else [])

        def result(st):
            return st.down if mlp else st.out

        out_hosts = [torch.empty(result(st).shape, dtype=torch.bfloat16).pin_memory()
                     for st in sets]
        s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        ev = {k: [torch.cuda.Event() for _ in sets] for k in ("in", "comp", "out")}

        def pipelined(n):
            for i in range(n):
                b = i % 2
                st = sets[b]
                with torch.cuda.stream(s_in):
                    if i >= 2:
                        s_in.wait_event(ev["comp"][b])      # step i - 2 has read this set
                    for dst, src in zip(device_inputs(st), [x_host] + extra_host):
                        dst.copy_(src, non_blocking=True)
                    ev["in"][b].record(s_in)
                with torch.cuda.stream(s_comp):
                    s_comp.wait_event(ev["in"][b])
                    if i >= 2:
                        s_comp.wait_event(ev["out"][b])     # step i - 2's result is downloaded
                    st.run()
                    ev["comp"][b].record(s_comp)
                with torch.cuda.stream(s_out):
                    s_out.wait_event(ev["comp"][b])
                    out_hosts[b].copy_(result(st), non_blocking=True)
                    ev["out"][b].record(s_out)

        torch.cuda.synchronize()
        pipelined(4)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        cur = torch.cuda.current_stream()
        e0.record(cur)
        for s_ in (s_in, s_comp, s_out):
            s_.wait_event(e0)
        pipelined(n_e2e)
        for s_ in (s_in, s_comp, s_out):
            done = torch.cuda.Event()
            done.record(s_)
            cur.wait_event(done)
        e1.record(cur)
        torch.cuda.synchronize()
        te = reduce_max_over_ranks([e0.elapsed_time(e1)], dist, world)
        e2e = {"value": whole_job_tops(ops, world, te[0] / n_e2e), "unit": "TOPS",
               "h2d_bytes_per_step": sum(t.numel() for t in [x_host] + extra_host) * 2,
               "d2h_bytes_per_step": out_hosts[0].numel() * 2, "steps": n_e2e,
               "streams": "copy in / compute / copy out, two buffer sets"}

    peaks, peak_src = measured_peaks()
    # committed ncu summaries are named <stage>_<workload>[_g<group>].md
    profile_key = args.workload + (f"_g{args.group}" if args.group else "")
    # GEMM rooflines against the published dense INT8 peak of the B200 (the denominator the
    # targets are stated against); the measured cuBLAS bf16 peak x 2 (the nominal int8/bf16
    # ratio) is given beside it: the burst figure for a kernel that ran at full clock, the
    # sustained one when the timed region itself reached the power cap
    capped = "sw_power_cap" in clocks.summary()["reasons"] and "bf16_tflops_sustained" in peaks
    bf16_peak = peaks["bf16_tflops_sustained"] if capped else peaks["bf16_tflops"]
    bf16_kind = "sustained (the timed region reached the power cap)" if capped else "burst"
    measured_int8 = bf16_peak * NOMINAL_INT8_OVER_BF16
    spec_peak = INT8_SPEC_TOPS
    if case.extra.get("attn"):
        # half the ops run int8 (QK), half bf16 (PV): the ceiling of that mix
        measured_int8 = 2.0 / (1.0 / measured_int8 + 1.0 / bf16_peak)
        spec_peak = 2.0 / (1.0 / INT8_SPEC_TOPS + 1.0 / (INT8_SPEC_TOPS / 2))
    grad = args.workload.startswith("grad_")
    # the kernel each GEMM stage launches: the CTA-pair kernel above 128 rows, template
    # arguments as in the library
    pair = case.M >= 129
    fp8 = bool(case.extra.get("fp8"))
    if case.extra.get("attn"):
        gemm_kernel = "attn_kernel"
    elif grad:
        gemm_kernel = (f"gemm_s8_pair_kernel<false,false,false,0,{case.g}>" if pair else
                       f"gemm_s8_kernel<256,false,false,{case.g}>") + " (input gradient)"
    elif "fused" in stage_ms:
        gemm_kernel = (f"gemm_s8_pair_kernel<false,false,false,{case.g}>" if pair else
                       f"gemm_s8_kernel<256,false,false,0,{case.g}>") \
            + " (quantizer warps inside)"
    elif args.workload.startswith("fp8_"):
        gemm_kernel = ("gemm_s8_pair_kernel<false,true,false,0>" if pair else
                       "gemm_s8_kernel<256,false,false,0,0,true>") + " (e4m3)"
    elif case.A is not None:
        gemm_kernel = ("gemm_s8_pair_kernel<false,false,true,0>" if pair else
                       "gemm_s8_kernel<SDNQ_LORA_BN,true>") + " (LoRA second accumulator)"
    else:
        gemm_kernel = ("gemm_s8_pair_kernel<false,false,false,0>" if pair else
                       "gemm_s8_kernel<256,false>")
    kernel_of = {"gemm_up": ("gemm_s8_pair_kernel<true,false,false,0>" if pair else
                             "gemm_s8_kernel<256,false,true>") + " (GELU epilogue)",
                 "gemm_down": gemm_kernel}
    ops_per_gemm = ops / len(step.gemm_stages)
    scaled_peak = clock_scaled_peak(spec_peak, clocks.summary())
    gemm_lines = {}
    for n in step.gemm_stages:
        ms = stage_ms[n] / args.steps
        tops = ops_per_gemm / (ms * 1e-3) / 1e12
        gemm_lines[n] = {
            "kernel": kernel_of.get(n, gemm_kernel), "bound": "tensor", "achieved": tops,
            "peak": spec_peak, "unit": "TFLOP/s", "frac": tops / spec_peak,
            "traffic": profiled_traffic(n, "attn_kernel" if case.extra.get("attn") else "gemm_s8",
                                        profile_key),
            "ops_per_launch": ops_per_gemm, "ms_per_launch": ms,
            "peak_source": ("NVIDIA B200 dense INT8 spec, 4500 TOPS"
                            + (" (int8 QK / bf16 PV mix)" if case.extra.get("attn") else "")),
            "measured_peak": measured_int8,
            "frac_of_measured": tops / measured_int8,
            "measured_peak_source": f"{peak_src} cuBLAS bf16 {bf16_kind} x "
                                    f"{NOMINAL_INT8_OVER_BF16} (int8/bf16 nominal)",
            "clock_scaled_peak": scaled_peak,
            "frac_of_clock_scaled": tops / scaled_peak if scaled_peak else None,
        }
    dominant = max(step.gemm_stages, key=lambda n: stage_ms[n])
    gemm_tops = ops / (sum(stage_ms[n] for n in step.gemm_stages) / args.steps * 1e-3) / 1e12

    rq_rows_k = case.N if grad else case.K        # row length of the quantized operand
    rq_lines = {}
    rq_stages = [n for n in names if n.startswith("rotquant")]
    if not rq_stages:
        # the step's quantizer runs inside the fused kernel: time the standalone kernel on
        # the same input (L2 flushed before each launch) for its own roofline
        rq_ms = standalone_rotquant_ms(step, flush, torch, sd, max(args.steps // 4, 10))
        rq_timed = {"rotquant": (rq_ms, rq_rows_k, "standalone rotquant kernel on the step's "
                                 "input (the step itself runs it fused)")}
    else:
        rq_timed = {n: (stage_ms[n] / args.steps,
                        case.N if n == "rotquant_h" else rq_rows_k,
                        "the stage's time in the per-stage pass of the same steps")
                    for n in rq_stages}
    for n, (ms, rows_k, note) in rq_timed.items():
        nbytes = rotquant_bytes(case.M, rows_k)
        if case.extra.get("attn"):
            # q and k rows of D (read bf16, write int8 + scale) and k read once more for the
            # means
            n_el = case.extra["B"] * case.M * case.N * case.K
            nbytes = 2 * (3 * n_el + 4 * n_el // case.K) + 2 * n_el
        gbs = nbytes / (ms * 1e-3) / 1e9
        rq_lines[n] = {
            "kernel": rotquant_kernel_name(case, rows_k, grad, fp8),
            "bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": gbs / peaks["hbm_gbs"],
            "traffic": profiled_traffic(n, "attn_kernel" if case.extra.get("attn") else "rotquant",
                                        profile_key),
            "bytes_per_launch": nbytes, "row_length": rows_k, "ms_per_launch": ms,
            "peak_source": f"{peak_src} copy bandwidth", "timing": note,
            "frac_of_spec": gbs / HBM_SPEC_GBS,
        }
    if "lora_down" in stage_ms:
        # u = bf16(x A): reads x and A, writes u
        r = case.A.shape[1]
        ms = stage_ms["lora_down"] / args.steps
        nbytes = 2 * (case.M * case.K + case.K * r + case.M * r)
        gbs = nbytes / (ms * 1e-3) / 1e9
        rq_lines["lora_down"] = {
            "kernel": f"lora_down_kernel<{(r + 63) // 64 * 64}>", "bound": "hbm",
            "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": gbs / peaks["hbm_gbs"],
            "traffic": profiled_traffic("lora_down", "lora_down", profile_key),
            "bytes_per_launch": nbytes, "ms_per_launch": ms,
            "peak_source": f"{peak_src} copy bandwidth",
            "timing": "the stage's time in the per-stage pass of the same steps",
        }
    line = {
        "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3" if args.workload.startswith("fp8_") else "int8",
        "data": "synthetic (seeded DiT-shaped bf16 activations with outlier channels, "
                "random-init weights)",
        "config": config_of(case, args),
        "roofline": gemm_lines[dominant],
        "gemm_tops": gemm_tops,
        "step_stats": {"median_ms": step_ms_median, "best_ms": step_ms_best,
                       "median_value": whole_job_tops(ops, world, step_ms_median),
                       "best_value": whole_job_tops(ops, world, step_ms_best),
                       "note": "per-step event times (each step alone between its L2 flush "
                               "and the next); value is the mean over the timed steps"},
        "stage_ms_per_step": {n: stage_ms[n] / args.steps for n in names},
        "stage_timing": "a second pass of the same steps with an event between the stages",
        "clocks": clocks.summary(),
        "gpu_launches": step.launches * args.steps,
        "e2e": e2e,
    }
    line["stages"] = names   # outside `config`, which the reference arm prints identically
    for n in step.gemm_stages:
        if len(step.gemm_stages) > 1:
            line[f"roofline_{n}"] = gemm_lines[n]
    for n, r in rq_lines.items():
        line[f"roofline_{n}"] = r
    if lora_flops:
        line["tops_with_lora_flops"] = whole_job_tops(ops + lora_flops, world, ms_per_step)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(case, args.workload)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
