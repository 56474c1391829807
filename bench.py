#!/usr/bin/env python
"""Benchmark of the fine-grained FP8 hot path on B200.

One step = one pass of the whole path over one batch of the dense workload
(A bf16 [4096, 7168] ~N(0,1) with 0.1% x100 outliers, W bf16 [7168, 7168] ~N(0,0.006),
power-of-two scales, bf16 output):
    quant_act_1x128(A) -> quant_weight_128x128(W) -> gemm_blockscaled(qA, sA, qW, sW)

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload NAME]

Prints one JSON line (rank 0).  ``value`` is GEMM FLOPs of all ranks / device time of
the whole step (quantization included), max over ranks; per-kernel event times give the
live roofline of the dominant kernel.  L2 is flushed between steps (a 512 MB write,
then a read of it so no dirty lines remain), outside the per-step events.  ``--impl reference`` times the CPU oracle (the reference
arm of this project) on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "FP8 block-scaled GEMM TFLOP/s and % of FP8 tensor peak; quant GB/s and % of HBM"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FP8_PER_BF16 = 2.0   # nominal dense fp8 : bf16 tensor throughput ratio


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return (float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d["bf16_tflops_sustained"]),
                "measured")
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS * 0.88, "fallback"


# ------------------------------------------------------------------------------ clocks (NVML)

class ClockSampler:
    """Samples SM clock and throttle reasons every ~20 ms in a thread while active."""

    REASONS = {0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x4: "sw_power_cap", 0x1: "gpu_idle",
               0x2: "applications_clocks_setting"}

    def __init__(self, device_index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.02)

    def __enter__(self):
        if self._nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._nv is not None:
            self._stop.set()
            self._t.join()

    def summary(self):
        return {"sm_mhz": float(statistics.median(self.samples)) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons - {"gpu_idle"}),
                "samples": len(self.samples)}


# ------------------------------------------------------------------------------ distributed

def dist_init(args):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and args.impl != "reference":
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The largest of the ranks' values (a collective: every rank calls it)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def bench_config(w, world: int) -> dict:
    """The `config` object of the bench line (both arms)."""
    return {"workload": w.name, "M": w.M, "N": w.N, "K": w.K, "pow2_scales": bool(w.pow2_a and w.pow2_b),
            "out": "fp32" if w.out_fp32 else "bf16",
            "parallelism": f"replicas x{world} (dense: each GPU its own {w.M}-token batch)",
            "l2": "flush between steps (512 MB write, then read back), outside the per-step events"}


# ------------------------------------------------------------------------------ GPU arm

def dev_bf16(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def run_gpu(args, rank, world):
    import torch
    import fp8_fine_grained_weight_b200 as fq

    w = workloads.ALL[args.workload]()
    assert not w.experts, "the bench times the dense path"
    M, N, K = w.M, w.N, w.K
    G = K // 128
    a_bits, b_bits = w.gen_a(), w.gen_b()
    A, W = dev_bf16(a_bits), dev_bf16(b_bits)
    qA = torch.empty((M, K), dtype=torch.uint8, device="cuda")
    sA = torch.empty((G, M), dtype=torch.float32, device="cuda")
    qW = torch.empty((N, K), dtype=torch.uint8, device="cuda")
    sW = torch.empty((N // 128, G), dtype=torch.float32, device="cuda")
    out_dtype = torch.float32 if w.out_fp32 else torch.bfloat16
    C = torch.empty((M, N), dtype=out_dtype, device="cuda")
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    # The GEMM of the step: with power-of-two scales on both operands the tensor core
    # applies them (fp8_gemm_blockscaled_ue8m0); otherwise the per-group promoted GEMM.
    path = gemm_path(args, w)
    gemms = {"ue8m0": lambda: fq.gemm_blockscaled_ue8m0(qA, sA, qW, sW, out=C),
             "promoted": lambda: fq.gemm_blockscaled(qA, sA, qW, sW, out=C)}
    gemm = gemms[path]

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        fq.quant_act_1x128(A, w.pow2_a, out=(qA, sA))
        if ev is not None:
            ev[1].record(stream)
        fq.quant_weight_128x128(W, w.pow2_b, out=(qW, sW))
        if ev is not None:
            ev[2].record(stream)
        gemm()
        if ev is not None:
            ev[3].record(stream)

    def flush_l2():
        # write a buffer 4x the L2, then read it back: the inputs are evicted and the
        # L2 holds no dirty lines that the first timed kernel would have to write back
        flush.zero_()
        flush.view(torch.int64).sum()

    for _ in range(max(args.warmup, 3)):
        flush_l2()
        step()
    torch.cuda.synchronize()
    err = fq.device_error()
    if err:
        raise RuntimeError(f"device error word {err:#x} after warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()

    def enqueue_steps():
        for i in range(args.steps):
            flush_l2()             # outside the step's events
            step(evs[i])

    with ClockSampler(torch.cuda.current_device()) as clk:
        # every step is enqueued behind a spin that outlasts the enqueueing, so the GPU runs
        # the steps back to back and no host latency falls inside a step's events
        _enqueue_ahead(enqueue_steps, lead_ms=max(20.0, 0.6 * args.steps))
    barrier(world)
    t_act = [e[0].elapsed_time(e[1]) for e in evs]
    t_w = [e[1].elapsed_time(e[2]) for e in evs]
    t_gemm = [e[2].elapsed_time(e[3]) for e in evs]
    t_step = [e[0].elapsed_time(e[3]) for e in evs]
    ms_step = max_over_ranks(sum(t_step) / len(t_step), world)
    ms_act = sum(t_act) / len(t_act)
    ms_w = sum(t_w) / len(t_w)
    ms_gemm = sum(t_gemm) / len(t_gemm)
    if fq.device_error():
        raise RuntimeError("device error word set after the timed region")

    hbm, bf16_burst, bf16_sust, peak_src = peaks()
    fp8_peak = bf16_burst * FP8_PER_BF16
    flops = w.gemm_flops
    gemm_tflops = flops / (ms_gemm * 1e-3) / 1e12
    act_bytes = M * K * 2 + M * K + M * G * 4
    w_bytes = N * K * 2 + N * K + (N // 128) * G * 4
    value = world * flops / (ms_step * 1e-3) / 1e12

    kernel = GEMM_KERNEL[path]
    traffic = None
    tp = os.path.join(ROOT, "profiles", f"{kernel}_dense_traffic.json")
    if os.path.exists(tp):
        try:
            tj = json.load(open(tp))
            if (tj.get("workload") == w.name and tj.get("kernel") == kernel
                    and tj.get("kernel_rev") == kernel_rev()):
                traffic = tj.get("dram_bytes_per_launch")
        except Exception:
            traffic = None
    # both GEMM paths on this step's operands (L2 flushed before each launch)
    paths = {}
    for name in (("ue8m0", "promoted") if w.pow2_a and w.pow2_b else ("promoted",)):
        t = _time_ms(gemms[name], 20, flush_l2)
        tf = flops / (t * 1e-3) / 1e12
        paths[name] = {"kernel": GEMM_KERNEL[name], "ms": round(t, 5), "tflops": round(tf, 1),
                       "frac_of_fp8_peak": round(tf / fp8_peak, 4)}
    if fq.device_error():
        raise RuntimeError("device error word set after the GEMM path timings")
    gemm_launches = 1 if path == "ue8m0" else (2 if fq.workspace_bytes(M, N, K) else 1)

    res = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "e4m3 x e4m3 -> f32 accumulate, bf16 out", "data": "synthetic",
        "config": bench_config(w, world),
        "kernels_ms": {"quant_act_1x128": round(ms_act, 5), "quant_weight_128x128": round(ms_w, 5),
                       kernel: round(ms_gemm, 5)},
        "kernels_ms_stats": {name: _spread(ts) for name, ts in
                             (("step", t_step), ("quant_act_1x128", t_act),
                              ("quant_weight_128x128", t_w), (kernel, t_gemm))},
        "gemm_path": path,
        "gemm_paths": paths,
        "gemm_tflops": round(gemm_tflops, 1),
        "gemm_frac_of_fp8_peak": round(gemm_tflops / fp8_peak, 4),
        "gemm_frac_of_fp8_spec_4500": round(gemm_tflops / 4500.0, 4),
        "quant_act_gbs": round(act_bytes / (ms_act * 1e-3) / 1e9, 1),
        "quant_act_frac_hbm": round(act_bytes / (ms_act * 1e-3) / 1e9 / hbm, 4),
        "quant_weight_gbs": round(w_bytes / (ms_w * 1e-3) / 1e9, 1),
        "quant_weight_frac_hbm": round(w_bytes / (ms_w * 1e-3) / 1e9 / hbm, 4),
        "roofline": {"bound": "tensor", "achieved": round(gemm_tflops, 1),
                     "peak": round(fp8_peak, 1), "unit": "TFLOP/s",
                     "frac": round(gemm_tflops / fp8_peak, 4), "traffic": traffic,
                     "kernel": kernel,
                     "peak_source": f"{peak_src} bf16 burst {bf16_burst} x {FP8_PER_BF16} (fp8:bf16)"},
        "gpu_launches": (2 + gemm_launches) * args.steps,
        "clocks": clk.summary(),
    }

    # ---- end to end through the public API with host buffers
    e2e_steps = max(3, min(args.steps, args.e2e_steps))
    A_h = torch.from_numpy(a_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    W_h = torch.from_numpy(b_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    C_h = torch.empty((M, N), dtype=out_dtype).pin_memory()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def e2e_step():
        A.copy_(A_h, non_blocking=True)
        W.copy_(W_h, non_blocking=True)
        step()
        C_h.copy_(C, non_blocking=True)

    e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    ev0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    ev1.record(stream)
    torch.cuda.synchronize()
    ms_e2e = max_over_ranks(ev0.elapsed_time(ev1) / e2e_steps, world)
    res["e2e"] = {"value": round(world * flops / (ms_e2e * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
                  "h2d_bytes_per_step": int(A_h.numel() * 2 + W_h.numel() * 2),
                  "d2h_bytes_per_step": int(C_h.numel() * C_h.element_size()),
                  "ms_per_step": round(ms_e2e, 4), "steps": e2e_steps}

    # ---- spot check of this run's output against a float64 product of its codes (rank 0)
    if rank == 0 and not args.no_check:
        res["spot_check"] = spot_check(w, qA, sA, qW, sW, C)

    if rank == 0 and not args.no_configs:
        res["configs"] = config_throughput(fq, flush_l2)
        res["library_fp8_ceiling"] = library_fp8_ceiling(flush_l2)
    if rank == 0 and not args.no_study:
        res["accumulation_study"] = accumulation_study(fq)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(w, a_bits, b_bits, budget_s=args.cpu_budget)
        if not args.no_configs:
            res["cpu_baseline_configs"] = cpu_baseline_configs()
    return res


# ------------------------------------------------------------------------------ other workloads

def _spread(ts) -> dict:
    """Mean, median and best of a list of per-launch times (ms) on this rank."""
    return {"mean": round(sum(ts) / len(ts), 5), "median": round(statistics.median(ts), 5),
            "best": round(min(ts), 5)}


def _enqueue_ahead(enqueue, lead_ms=20.0, max_ms=4000.0):
    """Runs enqueue() -- which only enqueues GPU work (and timing events) on the current
    stream -- behind a spin kernel on that stream that outlasts the host's enqueueing, so
    that the GPU never waits for the host between the enqueued events: host-side latency (a
    busy host, Python argument checks) cannot show up inside a timed region.  If the spin
    ended before the host finished enqueueing, the work is run again behind a spin twice as
    long.  Returns enqueue()'s result once its work has completed."""
    import torch
    stream = torch.cuda.current_stream()
    while True:
        torch.cuda.synchronize()
        torch.cuda._sleep(int(lead_ms * 2.0e6))    # ~lead_ms at 2 GHz (longer at lower clocks)
        lead_end = torch.cuda.Event()
        lead_end.record(stream)
        out = enqueue()
        caught_up = lead_end.query()
        torch.cuda.synchronize()
        if not caught_up or lead_ms >= max_ms:
            return out
        lead_ms *= 2


def _time_ms(fn, reps, flush_l2, warmup=2):
    """Mean device time of fn() over reps, L2 flushed before each (outside the events).
    Untimed warm-up calls first: a kernel variant's first launch pays one-time setup.
    All reps are enqueued behind a spin that outlasts the enqueueing (_enqueue_ahead)."""
    import torch
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()

    def enqueue():
        evs = []
        for _ in range(reps):
            flush_l2()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            evs.append((e0, e1))
        return evs

    evs = _enqueue_ahead(enqueue, lead_ms=max(20.0, 1.0 * reps))
    return sum(e0.elapsed_time(e1) for e0, e1 in evs) / reps


def _dev_normal(shape, std, seed, outlier_frac=0.0):
    """Seeded bf16 samples of N(0, std) generated on the device (timing-only inputs), with
    about `outlier_frac` of the entries (positions drawn with replacement) scaled x100 in
    fp32 before the bf16 rounding, as the workloads' outliers are."""
    import torch
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    out = torch.empty(shape, dtype=torch.bfloat16, device="cuda")
    flat = out.view(-1)
    step = 1 << 26
    for lo in range(0, flat.numel(), step):
        hi = min(flat.numel(), lo + step)
        v = torch.randn(hi - lo, generator=g, device="cuda") * std
        n_out = int(round(outlier_frac * (hi - lo)))
        if n_out:
            idx = torch.randint(0, hi - lo, (n_out,), generator=g, device="cuda")
            v[idx] *= 100.0
        flat[lo:hi] = v.to(torch.bfloat16)
    return out


DEVICE_INPUTS = ("seeded device draws of the workload's shapes and distributions (N(0, std), "
                 "0.1% x100 outliers where the workload has them); parity on the workload's own "
                 "host-drawn inputs is covered by the GPU tests")


def config_throughput(fq, flush_l2, reps=10):
    """Kernel times of the other workloads (inputs drawn on the device, same shapes and
    distributions as the parity tests; their parity is covered by the GPU tests)."""
    import torch
    hbm, bf16_burst, _, _ = peaks()
    fp8_peak = bf16_burst * FP8_PER_BF16
    out = {}
    # MoE prefill: 32 experts, Zipf routing, W [4096, 7168]
    w = workloads.prefill()
    off = torch.from_numpy(w.offsets).cuda()
    A = _dev_normal((w.M, w.K), w.a_std, 3001, w.a_outliers)
    W = _dev_normal((w.experts, w.N, w.K), w.b_std, 3002)
    qA, sA = fq.quant_act_1x128(A, False)
    qW, sW = fq.quant_weight_128x128(W, False)
    C = torch.empty((w.M, w.N), dtype=torch.bfloat16, device="cuda")
    t_a = _time_ms(lambda: fq.quant_act_1x128(A, False, out=(qA, sA)), reps, flush_l2)
    t_w = _time_ms(lambda: fq.quant_weight_128x128(W, False, out=(qW, sW)), reps, flush_l2)
    t_g = _time_ms(lambda: fq.gemm_grouped(qA, sA, qW, sW, off, out=C), reps, flush_l2)
    tf = w.gemm_flops / (t_g * 1e-3) / 1e12
    out["moe_prefill"] = {
        "workload": w.name, "inputs": DEVICE_INPUTS, "sum_M": w.M, "max_M": int(w.counts.max()), "min_M": int(w.counts.min()),
        "gemm_ms": round(t_g, 4), "gemm_tflops": round(tf, 1), "gemm_frac_of_fp8_peak": round(tf / fp8_peak, 4),
        "quant_act_gbs": round(w.M * w.K * (3 + 4 / 128) / (t_a * 1e-3) / 1e9, 1),
        "quant_weight_gbs": round(W.numel() * (3 + 4 / 16384) / (t_w * 1e-3) / 1e9, 1)}
    # the same shapes with power-of-two scales on both operands, scaled in the tensor core
    qA, sA = fq.quant_act_1x128(A, True, out=(qA, sA))
    qW, sW = fq.quant_weight_128x128(W, True, out=(qW, sW))
    t_u = _time_ms(lambda: fq.gemm_grouped_ue8m0(qA, sA, qW, sW, off, out=C), reps, flush_l2)
    tf_u = w.gemm_flops / (t_u * 1e-3) / 1e12
    out["moe_prefill_pow2_ue8m0"] = {"workload": w.name + " (power-of-two scales)", "gemm_ms": round(t_u, 4),
                                     "gemm_tflops": round(tf_u, 1),
                                     "gemm_frac_of_fp8_peak": round(tf_u / fp8_peak, 4)}
    del A, W, qA, sA, qW, sW, C
    # MoE decode: 64 experts, M_e ~ U{1..256}, W [7168, 2048] already FP8
    w = workloads.decode()
    off = torch.from_numpy(w.offsets).cuda()
    A = _dev_normal((w.M, w.K), w.a_std, 4001, w.a_outliers)
    W = _dev_normal((w.experts, w.N, w.K), w.b_std, 4002)
    qA, sA = fq.quant_act_1x128(A, True)
    qW, sW = fq.quant_weight_128x128(W, False)
    C = torch.empty((w.M, w.N), dtype=torch.bfloat16, device="cuda")
    t_g = _time_ms(lambda: fq.gemm_grouped(qA, sA, qW, sW, off, out=C), reps, flush_l2)
    gemm_bytes = qW.numel() + sW.numel() * 4 + qA.numel() + sA.numel() * 4 + C.numel() * 2
    out["moe_decode"] = {
        "workload": w.name, "inputs": DEVICE_INPUTS, "sum_M": w.M, "gemm_ms": round(t_g, 4),
        "gemm_tflops": round(w.gemm_flops / (t_g * 1e-3) / 1e12, 1),
        "gemm_gbs": round(gemm_bytes / (t_g * 1e-3) / 1e9, 1),
        "gemm_frac_of_hbm": round(gemm_bytes / (t_g * 1e-3) / 1e9 / hbm, 4),
        "algorithmic_bytes": int(gemm_bytes)}
    # the same with power-of-two weight scales too, scaled in the tensor core
    qW, sW = fq.quant_weight_128x128(W, True, out=(qW, sW))
    t_u = _time_ms(lambda: fq.gemm_grouped_ue8m0(qA, sA, qW, sW, off, out=C), reps, flush_l2)
    out["moe_decode_pow2w_ue8m0"] = {
        "workload": w.name + " (power-of-two weight scales too)", "gemm_ms": round(t_u, 4),
        "gemm_gbs": round(gemm_bytes / (t_u * 1e-3) / 1e9, 1),
        "gemm_frac_of_hbm": round(gemm_bytes / (t_u * 1e-3) / 1e9 / hbm, 4)}
    del A, W, qA, sA, qW, sW, C
    # wgrad: dY [7168, 16384] x X [2048, 16384], 1x128 both, fp32 out
    w = workloads.wgrad()
    A = _dev_normal((w.M, w.K), w.a_std, 5001, w.a_outliers)
    B = _dev_normal((w.N, w.K), w.b_std, 5002)
    qA, sA = fq.quant_act_1x128(A, False)
    qB, sB = fq.quant_act_1x128(B, False)
    C = torch.empty((w.M, w.N), dtype=torch.float32, device="cuda")
    t_a = _time_ms(lambda: fq.quant_act_1x128(A, False, out=(qA, sA)), reps, flush_l2)
    t_g = _time_ms(lambda: fq.gemm_blockscaled(qA, sA, qB, sB, b_rowwise=True, out=C), reps, flush_l2)
    tf = w.gemm_flops / (t_g * 1e-3) / 1e12
    out["wgrad"] = {"workload": w.name, "inputs": DEVICE_INPUTS, "gemm_ms": round(t_g, 4), "gemm_tflops": round(tf, 1),
                    "gemm_frac_of_fp8_peak": round(tf / fp8_peak, 4),
                    "quant_act_gbs": round(w.M * w.K * (3 + 4 / 128) / (t_a * 1e-3) / 1e9, 1)}
    del A, B, qA, sA, qB, sB, C
    # rows and the transposed copy in one pass: a gradient dY of 16384 tokens x 7168
    T, Nc = 16384, 7168
    dY = _dev_normal((T, Nc), 1e-3, 6001)
    bufs = fq.quant_act_dual(dY, False)
    t_d = _time_ms(lambda: fq.quant_act_dual(dY, False, out=bufs), reps, flush_l2)
    dual_bytes = T * Nc * (2 + 2 + 8 / 128)
    out["quant_dual"] = {"workload": f"quant_act_dual_{T}x{Nc}", "ms": round(t_d, 4),
                         "gbs": round(dual_bytes / (t_d * 1e-3) / 1e9, 1),
                         "frac_of_hbm": round(dual_bytes / (t_d * 1e-3) / 1e9 / hbm, 4),
                         "algorithmic_bytes": int(dual_bytes)}
    del dY, bufs
    # output quantized in the GEMM's epilogue against a GEMM then a separate 1x128 pass,
    # on the dense shape with FP32 scales (the promoted path)
    wd = workloads.dense()
    A = _dev_normal((wd.M, wd.K), wd.a_std, 6101)
    B = _dev_normal((wd.N, wd.K), wd.b_std, 6102)
    qA, sA = fq.quant_act_1x128(A, False)
    qB, sB = fq.quant_weight_128x128(B, False)
    bq = fq.gemm_blockscaled_quant(qA, sA, qB, sB)
    Cs = torch.empty((wd.M, wd.N), dtype=torch.bfloat16, device="cuda")
    qs = fq.quant_act_1x128(Cs, False)
    t_fc = _time_ms(lambda: fq.gemm_blockscaled_quant(qA, sA, qB, sB, out=bq), reps, flush_l2)
    t_fq = _time_ms(lambda: fq.gemm_blockscaled_quant(qA, sA, qB, sB, out=(None, bq[1], bq[2])),
                    reps, flush_l2)

    def two_pass():
        fq.gemm_blockscaled(qA, sA, qB, sB, out=Cs, split_k=False)
        fq.quant_act_1x128(Cs, False, out=qs)

    t_2 = _time_ms(two_pass, reps, flush_l2)
    out["gemm_quant_out"] = {"workload": f"dense_{wd.M}x{wd.N}x{wd.K}_fp32_scales_quantized_output",
                             "fused_with_c_ms": round(t_fc, 4), "fused_codes_only_ms": round(t_fq, 4),
                             "gemm_then_quant_pass_ms": round(t_2, 4), "launches_fused": 1,
                             "launches_two_pass": 2}
    del A, B, qA, sA, qB, sB, bq, Cs, qs
    # FP8 linear layer, one forward + backward (Fprop, Dgrad, Wgrad), dense shapes, pow2
    from fp8_fine_grained_weight_b200.linear import fp8_linear
    Tl, Kl, Nl = 4096, 7168, 7168
    x = _dev_normal((Tl, Kl), 1.0, 6002).requires_grad_(True)
    wl = _dev_normal((Nl, Kl), 0.006, 6003).requires_grad_(True)
    dyl = _dev_normal((Tl, Nl), 1e-3, 6004)

    def fwd_bwd():
        x.grad = None
        wl.grad = None
        fp8_linear(x, wl, True).backward(dyl)

    t_l = _time_ms(fwd_bwd, reps, flush_l2)
    tf = 3 * 2 * Tl * Kl * Nl / (t_l * 1e-3) / 1e12
    out["fp8_linear"] = {"workload": f"fp8_linear_fwd_bwd_{Tl}x{Kl}x{Nl}_pow2", "ms": round(t_l, 4),
                         "tflops_3_gemms": round(tf, 1), "frac_of_fp8_peak": round(tf / fp8_peak, 4),
                         "launches": 7}
    return out


def library_fp8_ceiling(flush_l2, n: int = 8192, reps: int = 20) -> dict:
    """The box's FP8 GEMM ceiling as a vendor library reaches it: torch._scaled_mm
    (cuBLASLt) on [n, n] x [n, n]^T E4M3 operands with one FP32 scale per tensor, bf16 out,
    L2 flushed before each launch.  Context for the block-scaled kernels' fraction of peak,
    not one of this library's kernels and not part of the timed step.  A failure is
    reported in the result, never raised."""
    try:
        import torch
        g = torch.Generator(device="cuda")
        g.manual_seed(7001)
        a = torch.randn(n, n, generator=g, device="cuda").to(torch.float8_e4m3fn)
        b = torch.randn(n, n, generator=g, device="cuda").to(torch.float8_e4m3fn)
        one = torch.ones((), dtype=torch.float32, device="cuda")

        def mm():
            return torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)

        t = _time_ms(mm, reps, flush_l2, warmup=5)
        del a, b
        _, bf16_burst, _, _ = peaks()
        tf = 2.0 * n * n * n / (t * 1e-3) / 1e12
        return {"call": "torch._scaled_mm (cuBLASLt), E4M3, per-tensor scales, bf16 out",
                "M": n, "N": n, "K": n, "ms": round(t, 4), "tflops": round(tf, 1),
                "frac_of_fp8_peak": round(tf / (FP8_PER_BF16 * bf16_burst), 4)}
    except Exception as e:     # reported, not raised: this leg is context only
        return {"unavailable": f"{type(e).__name__}: {str(e).splitlines()[0][:200] if str(e) else ''}"}


def accumulation_study(fq, rows_sampled=128, seeds=(0, 1, 2), ks=(4096, 8192, 16384), w=None):
    """Error of the promoted GEMM and of the no-promotion GEMM versus K on the wgrad workload
    (dY [7168, K] x X [2048, K], K = 4096 / 8192 / 16384 prefixes of one draw per seed),
    against the float64 product of the same codes and scales on `rows_sampled` rows.
    Promoted: 1x128 codes (and, apples to apples, the 1xK codes with their row scales
    repeated per group); no-promotion: 1xK codes, one TMEM accumulator over all of K.
    Per K: each statistic's value per seed, and its min / max over the seeds.  `w`: the
    shapes and spreads to draw (default: the wgrad workload)."""
    import torch
    w = workloads.wgrad() if w is None else w
    per_seed = []

    def stats(Cs, C_ref, T):
        d = np.abs(Cs.astype(np.float64) - C_ref)
        r = d / np.maximum(T, 1e-300)
        return {"max_rel_T": float(r.max()), "median_rel_T": float(np.median(r)),
                "rel_frobenius": float(np.linalg.norm(d) / np.linalg.norm(C_ref))}

    for seed in seeds:
        kmax = max(ks)
        a_full = workloads.normal_bf16(workloads.rng_for(5, 100 + seed), (w.M, kmax), w.a_std)
        b_full = workloads.normal_bf16(workloads.rng_for(5, 200 + seed), (w.N, kmax), w.b_std)
        rows = np.sort(np.random.default_rng(5 + seed).choice(w.M, rows_sampled, replace=False))
        res = []
        for K in ks:
            A = dev_bf16(np.ascontiguousarray(a_full[:, :K]))
            B = dev_bf16(np.ascontiguousarray(b_full[:, :K]))
            rows_t = torch.from_numpy(rows).to(A.device)
            G = K // 128
            qa, sa = fq.quant_act_1x128(A, False)
            qb, sb = fq.quant_act_1x128(B, False)
            C_p = fq.gemm_blockscaled(qa, sa, qb, sb, out_dtype=torch.float32, b_rowwise=True)
            qa1, sa1 = fq.quant_rowwise(A)
            qb1, sb1 = fq.quant_rowwise(B)
            C_n = fq.gemm_nopromo(qa1, sa1, qb1, sb1)
            C_p1 = fq.gemm_blockscaled(qa1, sa1.expand(G, -1).contiguous(), qb1,
                                       sb1.expand(G, -1).contiguous(), out_dtype=torch.float32,
                                       b_rowwise=True)
            torch.cuda.synchronize()
            C_ref, T = _fp64_product(qa[rows_t].cpu().numpy(), sa[:, rows_t].cpu().numpy(),
                                     qb.cpu().numpy(), sb.cpu().numpy(), True)
            C1_ref, T1 = _fp64_product(qa1[rows_t].cpu().numpy(),
                                       sa1[rows_t].cpu().numpy()[None, :].repeat(G, 0),
                                       qb1.cpu().numpy(), sb1.cpu().numpy()[None, :].repeat(G, 0), True)
            res.append({"K": K,
                        "promoted_1x128": stats(C_p[rows_t].cpu().numpy(), C_ref, T),
                        "promoted_1xK_codes": stats(C_p1[rows_t].cpu().numpy(), C1_ref, T1),
                        "no_promotion_1xK_codes": stats(C_n[rows_t].cpu().numpy(), C1_ref, T1)})
            del A, B, qa, sa, qb, sb, C_p, qa1, sa1, qb1, sb1, C_n, C_p1
        per_seed.append(res)
    summary = []
    for i, K in enumerate(ks):
        entry = {"K": K}
        for path in ("promoted_1x128", "promoted_1xK_codes", "no_promotion_1xK_codes"):
            entry[path] = {}
            for stat in ("max_rel_T", "median_rel_T", "rel_frobenius"):
                vals = [per_seed[j][i][path][stat] for j in range(len(seeds))]
                entry[path][stat] = {"per_seed": vals, "min": min(vals), "max": max(vals)}
        summary.append(entry)
    return {"rows_sampled": int(rows_sampled), "seeds": list(seeds),
            "metric": "|C - C_ref| / sum_k|a b| (max, median) and relative Frobenius error",
            "results": summary}


def profile_case(args, name: str, launches: int = 3):
    """A few launches of one workload's kernels on device-drawn inputs (for ncu captures)."""
    import torch
    import fp8_fine_grained_weight_b200 as fq
    if name == "dual":     # rows + transposed copy of a 16384-token x 7168 gradient
        dY = _dev_normal((16384, 7168), 1e-3, 7003)
        bufs = fq.quant_act_dual(dY, False)
        for _ in range(launches):
            fq.quant_act_dual(dY, False, out=bufs)
        torch.cuda.synchronize()
        if fq.device_error():
            raise RuntimeError("device error word set")
        print(json.dumps({"profile_case": "quant_act_dual_16384x7168", "launches": launches}), flush=True)
        return
    pow2_grouped = name == "decode_pow2"   # decode with power-of-two weight scales too
    w = workloads.ALL["decode" if pow2_grouped else name]()
    if w.experts:
        off = torch.from_numpy(w.offsets).cuda()
        A = _dev_normal((w.M, w.K), w.a_std, 7001)
        W = _dev_normal((w.experts, w.N, w.K), w.b_std, 7002)
        qA, sA = fq.quant_act_1x128(A, w.pow2_a or pow2_grouped)
        qW, sW = fq.quant_weight_128x128(W, w.pow2_b or pow2_grouped)
        del A, W               # keep the captured program's device memory small
        C = torch.empty((w.M, w.N), dtype=torch.bfloat16, device="cuda")
        gemm = fq.gemm_grouped_ue8m0 if pow2_grouped else fq.gemm_grouped
        run = lambda: gemm(qA, sA, qW, sW, off, out=C)
    else:
        A = _dev_normal((w.M, w.K), w.a_std, 7001)
        B = _dev_normal((w.N, w.K), w.b_std, 7002)
        qA, sA = fq.quant_act_1x128(A, w.pow2_a)
        qB, sB = fq.quant_act_1x128(B, w.pow2_b) if w.b_rowwise else fq.quant_weight_128x128(B, w.pow2_b)
        del A, B
        C = torch.empty((w.M, w.N), dtype=torch.float32 if w.out_fp32 else torch.bfloat16, device="cuda")
        if gemm_path(args, w) == "ue8m0":
            run = lambda: fq.gemm_blockscaled_ue8m0(qA, sA, qB, sB, b_rowwise=w.b_rowwise, out=C)
        else:
            run = lambda: fq.gemm_blockscaled(qA, sA, qB, sB, b_rowwise=w.b_rowwise, out=C)
    for _ in range(launches):
        run()
    torch.cuda.synchronize()
    if fq.device_error():
        raise RuntimeError("device error word set")
    print(json.dumps({"profile_case": w.name, "launches": launches}), flush=True)


GEMM_KERNEL = {"ue8m0": "gemm_blockscaled_ue8m0", "promoted": "gemm_blockscaled"}


def gemm_path(args, w) -> str:
    """The dense step's GEMM: the tensor-core-scaled one when both operands have
    power-of-two scales (unless --gemm says otherwise), else the promoted one."""
    if args.gemm != "auto":
        if args.gemm == "ue8m0" and not (w.pow2_a and w.pow2_b):
            raise SystemExit("--gemm ue8m0 needs power-of-two scales on both operands")
        return args.gemm
    return "ue8m0" if (w.pow2_a and w.pow2_b) else "promoted"


def kernel_rev() -> str:
    """Short hash of the GEMM sources (the kernels and their launch code), to tie stored
    ncu counters of a GEMM to the code they measured."""
    import hashlib
    h = hashlib.sha1()
    for f in ("ptx.cuh", "quant.cuh", "gemm.cuh", "gemm_ue8m0.cuh", "fp8q.cu"):
        h.update(open(os.path.join(ROOT, "fp8_fine_grained_weight_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:12]


def _e4m3_values() -> np.ndarray:
    """Float64 value of each of the 256 E4M3 bytes, decoded by torch's float8_e4m3fn."""
    import torch
    return torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()


def _fp64_product(qa, sa, qb, sb, b_rowwise: bool):
    """Exact reference for rows of a block-scaled GEMM, from the codes and scales the GPU
    used: C_ref = sum_k a~ b~ and T = sum_k |a~ b~| in float64, with a~ = E4M3(qa) times
    its 1x128 scale and b~ likewise (128x128 blocks, or 1x128 along K when b_rowwise).
    qa uint8 [r, K]; sa float32 [K/128, r]; qb uint8 [N, K]; sb [N/128, K/128] or
    [K/128, N].  Measurement only: no quantization happens here."""
    v = _e4m3_values()
    r, K = qa.shape
    N, G = qb.shape[0], K // 128
    A = (v[qa].reshape(r, G, 128) * sa[:G, :r].T.astype(np.float64)[:, :, None]).reshape(r, K)
    if b_rowwise:
        B = (v[qb].reshape(N, G, 128) * sb[:G, :N].T.astype(np.float64)[:, :, None]).reshape(N, K)
    else:
        B = (v[qb].reshape(N // 128, 128, G, 128)
             * sb.astype(np.float64)[:, None, :, None]).reshape(N, K)
    return A @ B.T, np.abs(A) @ np.abs(B).T


def _within_band(C, C_ref, T, out_fp32: bool) -> np.ndarray:
    """The acceptance band of the parity tests: fp32 out within 2e-5 T; bf16 out within one
    bf16 spacing of C_ref, or (where the sum cancels) within 2e-5 T plus half a bf16
    spacing of C.  The bf16 spacing at x is float32's spacing times 2^16 (8 against 24
    significant bits; also right for subnormals)."""
    C = np.asarray(C, np.float64)
    d = np.abs(C - C_ref)
    band = 2e-5 * T + 1e-30
    if out_fp32:
        return d <= band

    def spacing(x):
        return np.spacing(np.abs(x).astype(np.float32)).astype(np.float64) * 65536.0

    return (d <= spacing(C_ref)) | (d <= band + 0.5 * spacing(C))


def spot_check(w, qA, sA, qB, sB, C, b_rowwise: bool = False):
    """Four rows of this run's C (first, second, middle, last) against the float64 product
    of this run's own codes and scales, in the parity tests' band.  The codes themselves
    are checked bit for bit against the oracle by the GPU tests.  b_rowwise: the B scale
    mode the GEMM ran with (the timed step always uses 128x128 weight blocks)."""
    import torch
    rows = np.array([0, 1, w.M // 2, w.M - 1])
    rt = torch.from_numpy(rows).to(C.device)
    C_ref, T = _fp64_product(qA[rt].cpu().numpy(), sA[:, rt].cpu().numpy(), qB.cpu().numpy(),
                             sB.cpu().numpy(), b_rowwise)
    ok = _within_band(C[rt].float().cpu().numpy(), C_ref, T, w.out_fp32)
    return {"rows": rows.tolist(), "within_band": bool(ok.all()), "entries": int(ok.size),
            "reference": "float64 product of this run's codes and scales"}


# ------------------------------------------------------------------------------ CPU oracle

class OracleSample:
    """The oracle on a sample of a workload, one component at a time, each time scaled to the
    whole workload by its share of the work (the oracle's work is linear in each):

      A quantization (1x128 tiles) of `a_rows` rows      x  (total A rows) / a_rows
      W quantization (128x128 blocks) of `w_rows` rows   x  (total W rows) / w_rows
      FP64 dequantize + dgemm of `a_rows` rows by one
        expert's full W                                  x  (GEMM FLOPs) / (sample FLOPs)

    The dequantized W of the GEMM leg is prepared once, outside the timed components.  W
    rows are taken in turn (a different 128-row-aligned slice each call).  Used by both the
    `cpu_baseline` leg and the reference arm, so that the two CPU figures measure the same."""

    def __init__(self, w, a_bits, b_bits, a_rows=64, w_rows=1024):
        import oracle
        self.oracle, self.w = oracle, w
        self.a_rows = min(a_rows, a_bits.shape[0])
        wb = b_bits if b_bits.ndim == 2 else b_bits[0]           # one expert's weights
        self.w_rows = min(w_rows, wb.shape[0])
        self.a_bits, self.wb = a_bits, wb
        if w.b_rowwise:
            qb, sb = oracle.quant_act_1x128(wb, w.pow2_b)
            self.Bd = oracle.dequant_rows_groupmajor(qb, sb)
        else:
            qb, sb = oracle.quant_weight_128x128(wb, w.pow2_b)
            self.Bd = oracle.dequant_blocks(qb, sb)
        self.w_rows_total = w.N * max(1, w.experts)
        self._next = 0

    def step(self) -> float:
        """Seconds the oracle takes for the whole workload, extrapolated from one sample."""
        o, w = self.oracle, self.w
        r0 = (self._next * self.a_rows) % max(1, self.a_bits.shape[0] - self.a_rows + 1)
        a = self.a_bits[r0:r0 + self.a_rows]
        w0 = (self._next * self.w_rows) % max(1, self.wb.shape[0] - self.w_rows + 1) // 128 * 128
        wslice = self.wb[w0:w0 + self.w_rows]
        self._next += 1
        t0 = time.perf_counter()
        qa, sa = o.quant_act_1x128(a, w.pow2_a)
        t1 = time.perf_counter()
        if w.b_rowwise:
            o.quant_act_1x128(wslice, w.pow2_b)
        else:
            o.quant_weight_128x128(wslice, w.pow2_b)
        t2 = time.perf_counter()
        Ad = o.dequant_rows_groupmajor(qa, sa)
        _ = Ad @ self.Bd.T
        t3 = time.perf_counter()
        sample_flops = 2.0 * self.a_rows * self.Bd.shape[0] * w.K
        return ((t1 - t0) * w.M / self.a_rows + (t2 - t1) * self.w_rows_total / self.w_rows
                + (t3 - t2) * w.gemm_flops / sample_flops)

    def describe(self) -> str:
        return (f"per sample: 1x128 quantization of {self.a_rows} A rows, "
                f"{'1x128' if self.w.b_rowwise else '128x128'} quantization of {self.w_rows} W rows, "
                f"FP64 dequantize + dgemm of {self.a_rows} rows x [{self.Bd.shape[0]}, {self.w.K}]; "
                f"each scaled to the whole workload by its share of the work")


def cpu_baseline(w, a_bits, b_bits, budget_s: float = 15.0):
    """The oracle, as it stands, on the host cores: samples of the workload (OracleSample)
    until the budget is spent; the median extrapolated step time gives the metric."""
    cores = os.cpu_count()
    smp = OracleSample(w, a_bits, b_bits)
    times, t_end = [], time.perf_counter() + budget_s
    while time.perf_counter() < t_end or len(times) < 3:
        times.append(smp.step())
    t_step = statistics.median(times)
    return {"value": round(w.gemm_flops / t_step / 1e12, 6), "unit": "TFLOP/s", "cores": cores,
            "kind": "oracle", "samples": len(times),
            "sample": smp.describe() + f"; median over {len(times)} samples; numpy BLAS and "
                                       f"OpenMP threads = host cores"}


def cpu_baseline_configs(budget_s: float = 4.0) -> dict:
    """The oracle per workload (prefill and decode per expert, wgrad), a few seconds each, on
    the workloads' own seeded inputs (the first rows of A; one expert's weights)."""
    out = {}
    for name in ("prefill", "decode", "wgrad"):
        w = workloads.ALL[name]()
        rng = workloads.rng_for(3 if name == "prefill" else (4 if name == "decode" else 5), 7)
        a_bits = workloads.normal_bf16(rng, (256, w.K), w.a_std, w.a_outliers)
        b_bits = workloads.normal_bf16(rng, (w.N, w.K), w.b_std)
        smp = OracleSample(w, a_bits, b_bits, a_rows=64, w_rows=min(1024, w.N))
        times, t_end = [], time.perf_counter() + budget_s
        while time.perf_counter() < t_end or len(times) < 2:
            times.append(smp.step())
        t = statistics.median(times)
        out[name] = {"workload": w.name, "value": round(w.gemm_flops / t / 1e12, 6), "unit": "TFLOP/s",
                     "seconds_per_pass": round(t, 3), "samples": len(times),
                     "sample": smp.describe() + (f"; weights of one expert, W quantization scaled "
                                                 f"to all {w.experts} experts" if w.experts else "")}
    return out


def run_reference(args):
    """Reference arm: the CPU oracle (this project's reference: the pages hold no code) on the
    dense workload, one OracleSample per step, with the same sampling as `cpu_baseline`;
    the step time is the median of the steps' extrapolated times."""
    w = workloads.ALL[args.workload]()
    rows = min(w.M, 256)
    a_bits = w.gen_a()[:rows] if w.M <= 4096 else workloads.normal_bf16(
        np.random.default_rng(0), (rows, w.K), w.a_std, w.a_outliers)
    b_bits = w.gen_b()
    smp = OracleSample(w, a_bits, b_bits)
    for _ in range(max(args.warmup, 3)):
        smp.step()
    t_wall0 = time.perf_counter()
    times = [smp.step() for _ in range(args.steps)]
    wall = time.perf_counter() - t_wall0
    t_step = statistics.median(times)
    v = round(w.gemm_flops / t_step / 1e12, 6)
    return {"impl": "reference", "metric": METRIC, "value": v, "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": max(args.warmup, 3), "ms_per_step": round(t_step * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f64 (oracle)", "data": "synthetic",
            "config": bench_config(w, 1),
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
                             "sample": smp.describe() + f"; {args.steps} samples in {wall:.1f} s of "
                                                        f"wall time, median extrapolated step"},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="dense", choices=["tiny", "dense", "wgrad"],
                    help="the dense workload timed as one step (the bench line)")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--gemm", default="auto", choices=["auto", "ue8m0", "promoted"],
                    help="dense GEMM: auto = tensor-core scaling when both operands have "
                         "power-of-two scales, else per-group promotion")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-check", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the other workloads' timings")
    ap.add_argument("--no-study", action="store_true", help="skip the accumulation study")
    ap.add_argument("--profile-case",
                    choices=["tiny", "dense", "prefill", "decode", "decode_pow2", "wgrad", "dual"],
                    help="only run a few GEMM launches of one workload (for ncu) and exit")
    args = ap.parse_args()

    if args.profile_case:
        import torch
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
        profile_case(args, args.profile_case)
        return

    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) != 0:
            return
        print(json.dumps(run_reference(args)), flush=True)
        return

    rank, world, _ = dist_init(args)
    res = run_gpu(args, rank, world)
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
