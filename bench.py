#!/usr/bin/env python
"""Benchmark of the SERQ W4A4 linear on B200; prints one JSON line.

One step = the whole hot path over one batch of the LLaMA-3-8B-shaped MLP
workload at M = 2048 tokens, r = 128, MXFP4:
    serq_quant_act(X^_gu) -> serq_linear(gate|up, N = 2 x 14336)
    serq_quant_act(X^_dn) -> serq_linear(down, K = 14336)
value = sum over the step of 2*M*N*(K+r) / device time (TOPS), max over ranks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

--impl reference times the CPU oracle (the only other implementation of the
method here) on a bounded row sample of the same workload.
Multi-GPU runs are independent replicas (the linear has no exchange step).
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "serq_linear TOPS (2·M·N·(K+r)/t) and % of FP4 peak; decode GB/s; overhead vs r=0"
WORKLOAD = "mlp_mxfp4"
FP4_OVER_BF16 = 4.0  # nominal dense FP4 / dense BF16 tensor throughput on B200 (9 / 2.25 PFLOP/s)
INT8_OVER_BF16 = 2.0  # nominal dense INT8 / dense BF16 (4.5 / 2.25)
INT_KERNEL = "serq_linear_int4_kernel"  # INT4 and W4A8 prefill
CAPTURED_TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
DOMINANT_KERNEL = "serq_linear_mxfp4_pair_kernel"  # M > 128 MXFP4 prefill (CTA pairs)


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-rows", type=int, default=64, help="token rows of the oracle's timed sample")
    ap.add_argument("--no-extras", action="store_true", help="skip the r=0, INT4 and e2e side measurements")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-clocks", action="store_true", help="do not sample nvidia-smi (for profiler runs)")
    ap.add_argument("--only", default=None, help="time only the named linear of the workload (profiling)")
    ap.add_argument("--workload", default=WORKLOAD, choices=[WORKLOAD, "qproj_int4"],
                    help="the step's workload (default: the MXFP4 MLP); qproj_int4 is for profiling the INT4 kernel")
    ap.add_argument("--profile-decode", default=None, metavar="SHAPE",
                    help="run a few plain small-M launches of one decode shape (q, kv, gate_up, down) at "
                         "--decode-m tokens and exit (for profilers)")
    ap.add_argument("--decode-m", type=int, default=16)
    return ap.parse_args()


# ----------------------------------------------------------------- distributed
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    pg = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        backend = "nccl" if _cuda_ok() else "gloo"
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
        pg = dist
    return world, rank, local, pg


def _cuda_ok():
    import torch
    return torch.cuda.is_available()


def barrier(pg):
    if pg is not None:
        import torch
        if torch.cuda.is_available():
            pg.barrier(device_ids=[torch.cuda.current_device()])
        else:
            pg.barrier()


def whole_job_tops(world: int, step_flops: float, ms_per_step: float) -> float:
    """Aggregate throughput of `world` replicas that each ran one step of
    `step_flops` in `ms_per_step` (the slowest rank's time)."""
    return world * step_flops / (ms_per_step * 1e-3) / 1e12


def max_over_ranks(pg, value: float) -> float:
    if pg is None:
        return value
    import torch
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------- clocks
class ClockSampler:
    """NVML samples (every `period_s`, 1 ms by default) of the SM clock, power and clock-event reasons.

    Read-only queries; sampling runs in a thread from start() to stop().
    """

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake", "nvmlClocksEventReasonHwPowerBrakeSlowdown"))

    def __init__(self, device_index: int, period_s: float = 0.001):
        import threading
        self.period = period_s
        self.samples = []
        self.window = None
        self._stop = threading.Event()
        self._thread = None
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nv = nv
            self.h = nv.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
        except Exception:  # no NVML: no clock record
            self.nv = None
            return
        self._thread = threading.Thread(target=self._run, daemon=True)
        self._thread.start()

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                self.samples.append((time.perf_counter(), nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM),
                                     nv.nvmlDeviceGetCurrentClocksEventReasons(self.h),
                                     nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0))
            except Exception:
                pass
            time.sleep(self.period)

    def mark(self, t0, t1):
        self.window = (t0, t1)

    def stop(self):
        if self._thread is None:
            return None
        self._stop.set()
        self._thread.join(timeout=2)
        if not self.samples:
            return None
        nv = self.nv
        reasons = set()
        for _, _, mask, _ in self.samples:
            for name, attr in self.REASONS:
                if hasattr(nv, attr) and mask & getattr(nv, attr):
                    reasons.add(name)
        inside = [s for s in self.samples if self.window and self.window[0] <= s[0] <= self.window[1]]
        return {"sm_mhz": statistics.median(s[1] for s in self.samples), "sm_max_mhz": self.max_mhz,
                "power_w_max": max(s[3] for s in self.samples), "samples": len(self.samples),
                "samples_in_timed_region": len(inside),
                "sm_mhz_timed_region": statistics.median(s[1] for s in inside) if inside else None,
                "reasons": sorted(reasons),
                "source": f"NVML, {self.period * 1e3:g} ms period, 0.5 s pre-roll + timed region"}


# ----------------------------------------------------------------- workload
def linear_flops(M, lin):
    return 2.0 * M * lin.N * (lin.K + lin.r)


def build_layers(wl, r_override=None, device="cuda"):
    """Device-resident inputs of the step: prepared weights, folded activations, buffers."""
    import torch
    import w4a4_post_quantization_serq_b200 as S
    layers = []
    for lin in wl.linears:
        r = lin.r if r_override is None else r_override
        X = torch.from_numpy(lin.X(wl.M)).to(torch.bfloat16).to(device)
        W = torch.from_numpy(lin.W()).to(torch.bfloat16).to(device)
        a = S.serq_calib_absmax(torch.from_numpy(lin.X_calib(wl.M)).to(torch.bfloat16).to(device))
        w = S.serq_prepare(W, r, lin.fmt, act_absmax=a)
        Xh = S.serq_fold_producer(w, X)
        del W, X
        layers.append({"lin": lin, "r": r, "w": w, "Xh": Xh, "qa": S.alloc_act(wl.M, lin.K, r, lin.fmt, device),
                       "Y": torch.empty(wl.M, lin.N, dtype=torch.bfloat16, device=device),
                       "flops": 2.0 * wl.M * lin.N * (lin.K + r)})
    torch.cuda.synchronize()
    return layers


def quant_act_bytes(M: int, K: int, r: int, fmt: str) -> int:
    """Algorithmic HBM bytes of one serq_quant_act: read X^ (bf16), write the
    packed codes of X^_q and X~_{s,q} and their scales."""
    rp = ((r + 63) // 64) * 64 if r > 0 else 0
    scales = (M * K // 32 + M * rp // 32) if fmt == "mxfp4" else (4 * M + (4 * M if rp else 0))
    codes = (M * K + M * rp) if fmt == "w4a8" else (M * K // 2 + M * rp // 2)  # W4A8: one byte per code
    return 2 * M * K + codes + scales


def quant_roofline(layers, quant_ms, hbm_gbs):
    """HBM roofline of serq_quant_act over the step's launches (CUDA events)."""
    if not quant_ms:
        return None
    nbytes = [quant_act_bytes(L["qa"].M, L["lin"].K, L["r"], L["lin"].fmt) for L in layers]
    tot_b, tot_ms = sum(nbytes), sum(quant_ms)
    return {"bound": "hbm", "kernel": "quant_act", "bytes_per_step": tot_b,
            "us_per_step": round(tot_ms * 1e3, 2), "achieved": tot_b / (tot_ms * 1e-3) / 1e9, "unit": "GB/s",
            "peak": hbm_gbs, "frac": tot_b / (tot_ms * 1e-3) / 1e9 / hbm_gbs,
            "per_launch": {L["lin"].name: {"bytes": b, "us": round(t * 1e3, 2),
                                           "GBs": round(b / (t * 1e-3) / 1e9, 1)}
                           for L, b, t in zip(layers, nbytes, quant_ms)}}


def run_step(layers, events=None):
    """One step: per linear, serq_quant_act then serq_linear. With `events`
    ([layer][3] CUDA events) the quant launch is bracketed by events 0-1 and
    the linear by events 1-2, on the launching (current) stream."""
    import w4a4_post_quantization_serq_b200 as S
    for i, L in enumerate(layers):
        if events is not None:
            events[i][0].record()
        S.serq_quant_act(L["Xh"], L["r"], L["lin"].fmt, out=L["qa"])
        if events is not None:
            events[i][1].record()
        S.serq_linear(L["w"], L["qa"], Y=L["Y"])
        if events is not None:
            events[i][2].record()


def time_steps(layers, steps, warmup, pg, per_gemm=True, sampler=None):
    """Device time of `steps` steps (CUDA events on the launching stream).

    Returns (total_ms, gemm_ms, quant_ms): the per-layer means over the timed
    steps of the serq_linear and serq_quant_act launches (None without
    per-launch events)."""
    import torch
    import w4a4_post_quantization_serq_b200 as S
    for _ in range(warmup):
        run_step(layers)
    S.serq_device_status()
    if sampler is not None:
        # untimed pre-roll under the same load so the clock record has samples
        t_end = time.perf_counter() + 0.5
        while time.perf_counter() < t_end:
            run_step(layers)
            torch.cuda.synchronize()
    ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in layers] for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(pg)
    torch.cuda.synchronize()
    switch = sys.getswitchinterval()
    sys.setswitchinterval(2e-4)  # let the clock sampler thread in while this one launches
    t0 = time.perf_counter()
    start.record()
    for k in range(steps):
        run_step(layers, ev[k] if per_gemm else None)
    end.record()
    torch.cuda.synchronize()
    if sampler is not None:
        sampler.mark(t0, time.perf_counter())
    sys.setswitchinterval(switch)
    barrier(pg)
    S.serq_device_status()
    total_ms = start.elapsed_time(end)
    gemm_ms = quant_ms = None
    if per_gemm:
        gemm_ms = [sum(ev[k][i][1].elapsed_time(ev[k][i][2]) for k in range(steps)) / steps
                   for i in range(len(layers))]
        quant_ms = [sum(ev[k][i][0].elapsed_time(ev[k][i][1]) for k in range(steps)) / steps
                    for i in range(len(layers))]
    return total_ms, gemm_ms, quant_ms


def time_e2e(layers, steps, warmup, pg=None):
    """Same step through the public API with host buffers: pinned H2D of X^, D2H of Y, every step."""
    import torch
    import w4a4_post_quantization_serq_b200 as S
    host_in = [L["Xh"].cpu().pin_memory() for L in layers]
    host_out = [torch.empty(L["Y"].shape, dtype=L["Y"].dtype).pin_memory() for L in layers]

    def step():
        for L, hi, ho in zip(layers, host_in, host_out):
            L["Xh"].copy_(hi, non_blocking=True)
            S.serq_quant_act(L["Xh"], L["r"], L["lin"].fmt, out=L["qa"])
            S.serq_linear(L["w"], L["qa"], Y=L["Y"])
            ho.copy_(L["Y"], non_blocking=True)
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(pg)
    torch.cuda.synchronize()
    start.record()
    for _ in range(steps):
        step()
    end.record()
    torch.cuda.synchronize()
    barrier(pg)
    S.serq_device_status()
    h2d = sum(t.numel() * t.element_size() for t in host_in)
    d2h = sum(t.numel() * t.element_size() for t in host_out)
    return start.elapsed_time(end) / steps, h2d, d2h


def bench_small_m(tokens=(32, 64, 128), reps: int = 50):
    """serq_linear for 16 < M <= 128 (the one-CTA tensor-core kernel) on the
    gate/up shape (K = 4096, N = 2 x 14336, MXFP4, r = 128), one weight, CUDA
    events over back-to-back launches. At these M the 59 MB weight stream
    bounds it, so both the TFLOP/s and the weight GB/s are reported."""
    import torch
    import w4a4_post_quantization_serq_b200 as S
    from synth import workload
    lin = workload("mlp_mxfp4").linears[0]
    K, N, r = lin.K, lin.N, lin.r
    rp = ((r + 63) // 64) * 64
    W = torch.from_numpy(lin.W()).to(torch.bfloat16).cuda()
    a = S.serq_calib_absmax(torch.from_numpy(lin.X_calib(128)).to(torch.bfloat16).cuda())
    w = S.serq_prepare(W, r, lin.fmt, act_absmax=a)
    del W
    w_bytes = N * K // 2 + N * K // 32 + N * rp // 2 + N * rp // 32
    peaks = measured_peaks()[0]
    out = {"K": K, "N": N, "r": r}
    for M in tokens:
        qa = S.serq_quant_act(S.serq_fold_producer(w, torch.from_numpy(lin.X(M)).to(torch.bfloat16).cuda()),
                              r, lin.fmt)
        Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        for _ in range(5):
            S.serq_linear(w, qa, Y=Y)
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record()
        for _ in range(reps):
            S.serq_linear(w, qa, Y=Y)
        end.record()
        torch.cuda.synchronize()
        us = start.elapsed_time(end) / reps * 1e3
        tflops = 2.0 * M * N * (K + r) / (us * 1e-6) / 1e12
        out[f"M{M}"] = {"us": round(us, 2), "TFLOPs": round(tflops, 1),
                        "frac_fp4": round(tflops / (peaks["bf16_tflops"] * FP4_OVER_BF16), 3),
                        "weight_GBs": round(w_bytes / (us * 1e-6) / 1e9, 1),
                        "frac_hbm": round(w_bytes / (us * 1e-6) / 1e9 / peaks["hbm_gbs"], 3)}
    S.serq_device_status()
    return out


def bench_decode(reps: int = 10, tokens=(1, 4, 16)):
    """HBM-bound small-M serq_linear on the LLaMA-3-8B decode shapes.

    For each shape, a pool of independently prepared copies of the weight
    (total bytes >= 4x the L2 size) is swept by a CUDA graph of back-to-back
    launches, so every launch streams its weight from HBM.
    Returns {shape: {M: {us, GBs, frac}}} with algorithmic bytes per call:
    W^_q + its E8M0 + Q(R) + its E8M0 + token codes and scales + bf16 Y.
    """
    import torch
    import w4a4_post_quantization_serq_b200 as S
    from synth import workload
    import dataclasses
    wl = workload("decode_mxfp4")
    l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
    hbm = measured_peaks()[0]["hbm_gbs"]
    out = {}
    # beside the four shapes, q, k and v as the one launch a decoder issues for them
    # (they read the same input): 4096 x 6144
    qkv = dataclasses.replace(wl.linears[0], name="qkv_fused", N=6144, w_seeds=(14,), x_seed=14, calib_seed=104)
    for lin in list(wl.linears) + [qkv]:
        K, N, r = lin.K, lin.N, lin.r
        rp = ((r + 63) // 64) * 64 if r else 0
        W = torch.from_numpy(lin.W()).to(torch.bfloat16).cuda()
        a = S.serq_calib_absmax(torch.from_numpy(lin.X_calib(16)).to(torch.bfloat16).cuda())
        w_bytes = N * K // 2 + N * K // 32 + N * rp // 2 + N * rp // 32
        n_pool = max(2, -(-4 * l2 // w_bytes))
        pool = [S.serq_prepare(W, r, lin.fmt, act_absmax=a) for _ in range(n_pool)]
        del W
        out[lin.name] = {"K": K, "N": N, "pool": n_pool}
        for M in tokens:
            X = torch.from_numpy(lin.X(M)).to(torch.bfloat16).cuda()
            qa = S.serq_quant_act(S.serq_fold_producer(pool[0], X), r, lin.fmt)
            Y = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
            for w in pool:
                S.serq_linear(w, qa, Y=Y)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for w in pool:
                    S.serq_linear(w, qa, Y=Y)
            g.replay()
            g.replay()
            start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            start.record()
            for _ in range(reps):
                g.replay()
            end.record()
            torch.cuda.synchronize()
            S.serq_device_status()
            t = start.elapsed_time(end) * 1e-3 / (reps * n_pool)
            nbytes = w_bytes + M * (K // 2 + K // 32 + rp // 2 + rp // 32) + 2 * M * N
            out[lin.name][f"M{M}"] = {"us": round(t * 1e6, 3), "GBs": round(nbytes / t / 1e9, 1),
                                      "frac": round(nbytes / t / 1e9 / hbm, 3)}
            del g
        del pool
        torch.cuda.empty_cache()
    return out


def bench_stack(ranks=(0, 16, 128, 256), reps: int = 3):
    """The 32-block LLaMA-3-8B-shaped MXFP4 stack at M = 2048, per swept r.

    Per block: qkv (4096 -> 6144), o (4096 -> 4096), gate/up (4096 -> 2x14336),
    down (14336 -> 4096), each with its own prepared weight buffer (128
    distinct buffers, ~3.7 GB at r = 128, so nothing stays in L2 between uses);
    the block-0 weight and activation of each shape are prepared once and
    copied into the 32 buffers (timing does not depend on the values).
    Returns {r: {linears_ms, total_ms, TOPS_linears, TOPS_total}} where total
    adds one serq_quant_act per linear input.
    """
    import torch
    import w4a4_post_quantization_serq_b200 as S
    from synth import workload
    out = {}
    for r in ranks:
        wl = workload("stack_mxfp4", r=r)
        shapes = [l for l in wl.linears if l.name.startswith("b0.")]
        blocks = len(wl.linears) // len(shapes)
        per_shape = []
        flops = 0.0
        for lin in shapes:
            W = torch.from_numpy(lin.W()).to(torch.bfloat16).cuda()
            a = S.serq_calib_absmax(torch.from_numpy(lin.X_calib(wl.M)).to(torch.bfloat16).cuda())
            pool = [S.serq_prepare(W, r, lin.fmt, act_absmax=a) for _ in range(blocks)]
            del W
            Xh = S.serq_fold_producer(pool[0], torch.from_numpy(lin.X(wl.M)).to(torch.bfloat16).cuda())
            qa = S.serq_quant_act(Xh, r, lin.fmt)
            Y = torch.empty(wl.M, lin.N, dtype=torch.bfloat16, device="cuda")
            per_shape.append((lin, pool, Xh, qa, Y))
            flops += blocks * 2.0 * wl.M * lin.N * (lin.K + r)

        def run(with_quant):
            for b in range(blocks):
                for lin, pool, Xh, qa, Y in per_shape:
                    if with_quant:
                        S.serq_quant_act(Xh, r, lin.fmt, out=qa)
                    S.serq_linear(pool[b], qa, Y=Y)

        res = {}
        for key, wq in (("linears_ms", False), ("total_ms", True)):
            run(wq)
            torch.cuda.synchronize()
            start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            start.record()
            for _ in range(reps):
                run(wq)
            end.record()
            torch.cuda.synchronize()
            S.serq_device_status()
            res[key] = round(start.elapsed_time(end) / reps, 3)
        res["TOPS_linears"] = round(flops / (res["linears_ms"] * 1e-3) / 1e12, 1)
        res["TOPS_total"] = round(flops / (res["total_ms"] * 1e-3) / 1e12, 1)
        out[f"r{r}"] = res
        del per_shape
        torch.cuda.empty_cache()
    if "r0" in out:
        for k, v in out.items():
            v["overhead_vs_r0"] = round(v["total_ms"] / out["r0"]["total_ms"] - 1, 4)
    return out


def bench_mlp_fused(wl, steps: int, warmup: int):
    """The MLP block with the producers fused (MXFP4, M = 2048): per step
    serq_rmsnorm_quant_act (RMSNorm -> gate/up input, quantized) ->
    serq_linear_swiglu_quant (gate/up whose epilogue writes down's quantized
    input) -> serq_linear (down). Same linear flops as the headline step.
    Returns (ms per step, per-launch us)."""
    import torch
    import w4a4_post_quantization_serq_b200 as S
    from synth import norm_weight
    gu, dn = wl.linears
    dev = "cuda"
    Wd = torch.from_numpy(dn.W()).to(torch.bfloat16).to(dev)
    w_d = S.serq_prepare(Wd, dn.r, dn.fmt,
                         act_absmax=S.serq_calib_absmax(torch.from_numpy(dn.X_calib(wl.M)).to(torch.bfloat16).to(dev)))
    Wgu = torch.from_numpy(gu.W()).to(torch.bfloat16).to(dev)
    w_gu = S.serq_prepare_swiglu(Wgu, gu.r, w_d, act_absmax=S.serq_calib_absmax(
        torch.from_numpy(gu.X_calib(wl.M)).to(torch.bfloat16).to(dev)))
    del Wd, Wgu
    H = torch.from_numpy(gu.X(wl.M)).to(torch.bfloat16).to(dev)      # the residual stream entering the MLP
    gamma = torch.from_numpy(norm_weight(77, gu.K)).to(torch.bfloat16).to(dev)
    qa = S.alloc_act(wl.M, gu.K, gu.r, gu.fmt, dev)
    h = S.alloc_act(wl.M, dn.K, dn.r, dn.fmt, dev)
    Y = torch.empty(wl.M, dn.N, dtype=torch.bfloat16, device=dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]

    def step(record=False):
        if record:
            ev[0].record()
        S.serq_rmsnorm_quant_act(w_gu, H, gamma, 1e-5, out=qa)
        if record:
            ev[1].record()
        S.serq_linear_swiglu_quant(w_gu, qa, out=h)
        if record:
            ev[2].record()
        S.serq_linear(w_d, h, Y=Y)
        if record:
            ev[3].record()
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    parts = [0.0, 0.0, 0.0]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps):
        step(record=True)
        # per-launch split from the last step's events (read after the loop)
    end.record()
    torch.cuda.synchronize()
    S.serq_device_status()
    parts = [ev[i].elapsed_time(ev[i + 1]) * 1e3 for i in range(3)]
    return start.elapsed_time(end) / steps, {"rmsnorm_quant_act": round(parts[0], 2),
                                             "gate_up_swiglu_quant": round(parts[1], 2), "down": round(parts[2], 2)}


def bench_prefill_block(M: int = 2048, blocks: int = 32, reps: int = 3, r: int = 128):
    """Time to first token of a random-init LLaMA-3-8B-shaped stack at a 2K
    prefill (hidden 4096, 32 query / 8 key-value heads of 128, FFN 14336,
    MXFP4, r = 128): per block RMSNorm+quant -> qkv -> RoPE (q, k) -> causal
    GQA attention -> fold+quant -> o -> add -> RMSNorm+quant -> gate/up with
    the SwiGLU epilogue -> down -> add. 32 distinct weight sets (block 0's
    prepared weights copied; timing does not depend on the values).
    Embedding and LM head are not included. Returns a dict of ms."""
    import torch
    import w4a4_post_quantization_serq_b200 as S
    from synth import activations, norm_weight, weights
    Hd, nq, nkv, D, F = 4096, 32, 8, 128, 14336
    nqkv = (nq + 2 * nkv) * D
    dev = "cuda"
    bf = lambda a: torch.from_numpy(a).to(torch.bfloat16).to(dev)
    cal = lambda seed, K: S.serq_calib_absmax(bf(activations(seed, 256, K, K // 100, "lognormal", 10.0)))
    fmt = "mxfp4"
    Wd = bf(weights(1004, F, Hd))
    a_d = cal(1005, F)
    blk = [None] * blocks
    # prepare every block's weights (distinct buffers, same values)
    Wqkv, Wo, Wgu = bf(weights(1000, Hd, nqkv)), bf(weights(1002, nq * D, Hd)), bf(weights(1003, Hd, 2 * F))
    a_qkv, a_o, a_gu = cal(1001, Hd), cal(1006, nq * D), cal(1007, Hd)
    for b in range(blocks):
        d = S.serq_prepare(Wd, r, fmt, act_absmax=a_d)
        blk[b] = {"qkv": S.serq_prepare(Wqkv, r, fmt, act_absmax=a_qkv),
                  "o": S.serq_prepare(Wo, r, fmt, act_absmax=a_o),
                  "d": d, "gu": S.serq_prepare_swiglu(Wgu, r, d, act_absmax=a_gu)}
    del Wqkv, Wo, Wgu, Wd
    torch.cuda.empty_cache()
    g1, g2 = bf(norm_weight(1010, Hd)), bf(norm_weight(1011, Hd))
    H = [bf(activations(1012, M, Hd, 41, "lognormal", 10.0)), torch.empty(M, Hd, dtype=torch.bfloat16, device=dev)]
    qa1 = S.alloc_act(M, Hd, r, fmt)
    qa2 = S.alloc_act(M, nq * D, r, fmt)
    qa3 = S.alloc_act(M, Hd, r, fmt)
    hq = S.alloc_act(M, F, r, fmt)
    qkv = torch.empty(M, nqkv, dtype=torch.bfloat16, device=dev)
    att = torch.empty(M, nq * D, dtype=torch.bfloat16, device=dev)
    y = torch.empty(M, Hd, dtype=torch.bfloat16, device=dev)
    h1 = torch.empty(M, Hd, dtype=torch.bfloat16, device=dev)

    def forward():
        h = H[0]
        for b in range(blocks):
            w = blk[b]
            S.serq_rmsnorm_quant_act(w["qkv"], h, g1, 1e-5, out=qa1)
            S.serq_linear(w["qkv"], qa1, Y=qkv)
            S.serq_rope(qkv[:, :nq * D], nq, D, 500000.0)
            S.serq_rope(qkv[:, nq * D:(nq + nkv) * D], nkv, D, 500000.0)
            S.serq_attention_prefill(qkv[:, :nq * D], qkv[:, nq * D:(nq + nkv) * D], qkv[:, (nq + nkv) * D:], nq,
                                     nkv, out=att)
            S.serq_fold_quant_act(w["o"], att, out=qa2)
            S.serq_linear(w["o"], qa2, Y=y)
            S.serq_add(h, y, out=h1)
            S.serq_rmsnorm_quant_act(w["gu"], h1, g2, 1e-5, out=qa3)
            S.serq_linear_swiglu_quant(w["gu"], qa3, out=hq)
            S.serq_linear(w["d"], hq, Y=y)
            S.serq_add(h1, y, out=H[1])
            h = H[1]
    forward()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(reps):
        forward()
    end.record()
    torch.cuda.synchronize()
    S.serq_device_status()
    ttft = start.elapsed_time(end) / reps
    # one block's attention alone (after two untimed calls)
    for _ in range(2):
        S.serq_attention_prefill(qkv[:, :nq * D], qkv[:, nq * D:(nq + nkv) * D], qkv[:, (nq + nkv) * D:], nq, nkv,
                                 out=att)
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record()
    for _ in range(10):
        S.serq_attention_prefill(qkv[:, :nq * D], qkv[:, nq * D:(nq + nkv) * D], qkv[:, (nq + nkv) * D:], nq, nkv,
                                 out=att)
    a1.record()
    torch.cuda.synchronize()
    att_us = a0.elapsed_time(a1) / 10 * 1e3
    att_flops = 4.0 * nq * D * M * (M + 1) / 2
    del blk
    torch.cuda.empty_cache()
    return {"ttft_ms": round(ttft, 3), "blocks": blocks, "M": M, "attention_us_per_block": round(att_us, 2),
            "attention_TFLOPs": round(att_flops / (att_us * 1e-6) / 1e12, 1),
            "note": "random-init LLaMA-3-8B-shaped blocks, MXFP4 SERQ linears r=128, bf16 causal GQA attention; "
                    "no embedding / LM head. The pages' LLaMA-3-8B 2K TTFT (RTX PRO 6000 Blackwell): "
                    "FP16 132.38 ms, MXFP4 56.03 ms, SERQ-MXFP4 62.31 ms (other hardware; context only)"}


def bench_l2qer(wl, steps: int, warmup: int, k: int = 128):
    """The two-factor baseline on the same workload: per linear, serq_quant_act
    (r = 0) then serq_linear_l2qer (T = X_q L1_q, Q(T), X_q W_q + Q(T) L2_q).
    Synthetic factors L1 (K x k), L2 (k x N): the timing does not depend on
    their values. Returns ms per step."""
    import torch
    import w4a4_post_quantization_serq_b200 as S
    from synth import weights
    layers = []
    for i, lin in enumerate(wl.linears):
        X = torch.from_numpy(lin.X(wl.M)).to(torch.bfloat16).cuda()
        W = torch.from_numpy(lin.W()).to(torch.bfloat16).cuda()
        L1 = torch.from_numpy(weights(900 + i, lin.K, k, 0.05)).to(torch.bfloat16).cuda()
        L2 = torch.from_numpy(weights(950 + i, k, lin.N, 0.01)).to(torch.bfloat16).cuda()
        a = S.serq_calib_absmax(torch.from_numpy(lin.X_calib(wl.M)).to(torch.bfloat16).cuda())
        main = S.serq_prepare(W, k, lin.fmt, act_absmax=a, R=L2)
        l1 = S.serq_prepare(L1, 0, lin.fmt, s=main.view()["s"])
        Xh = S.serq_fold_producer(main, X)
        del X, W, L1, L2
        layers.append({"main": main, "l1": l1, "Xh": Xh, "fmt": lin.fmt,
                       "qa": S.alloc_act(wl.M, lin.K, 0, lin.fmt),
                       "scratch": {"T": torch.empty(wl.M, k, dtype=torch.bfloat16, device="cuda"),
                                   "tq": S.alloc_act(wl.M, k, k, lin.fmt)},
                       "Y": torch.empty(wl.M, lin.N, dtype=torch.bfloat16, device="cuda")})

    def step():
        for L in layers:
            S.serq_quant_act(L["Xh"], 0, L["fmt"], out=L["qa"])
            S.serq_linear_l2qer(L["main"], L["l1"], L["qa"], Y=L["Y"], scratch=L["scratch"])
    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps):
        step()
    end.record()
    torch.cuda.synchronize()
    S.serq_device_status()
    return start.elapsed_time(end) / steps


# ----------------------------------------------------------------- CPU oracle
def cpu_oracle_prepare(wl, r_override=None):
    """The oracle's offline preparation of every linear (not timed)."""
    from oracle import serq_oracle as O
    out = []
    for lin in wl.linears:
        r = lin.r if r_override is None else r_override
        prep = O.prepare(lin.W(), r, lin.fmt, act_absmax=O.calib_absmax(lin.X_calib(wl.M)))
        out.append((lin, r, prep, lin.X(wl.M)))
    return out


def cpu_oracle_step(prepared, rows):
    """One timed oracle step on `rows` tokens: activation quantization + linear.

    Returns (seconds, flops, cores)."""
    from threadpoolctl import threadpool_info

    from oracle import serq_oracle as O
    t_total, flops = 0.0, 0.0
    for lin, r, prep, X in prepared:
        Xh = O.fold_activation(X[:rows], prep.s, prep.perm)
        t0 = time.perf_counter()
        qa = O.quant_act(Xh, r, lin.fmt)
        O.linear(prep, qa)
        t_total += time.perf_counter() - t0
        flops += 2.0 * rows * lin.N * (lin.K + r)
    cores = max([p.get("num_threads", 1) for p in threadpool_info()] + [1])
    return t_total, flops, cores


# ----------------------------------------------------------------- main
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return d, "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def captured_traffic():
    """DRAM bytes per launch from the committed ncu capture, or None once the
    kernel source differs from the one the counters were taken on."""
    import hashlib
    try:
        rec = json.load(open(CAPTURED_TRAFFIC_FILE))
        src = os.path.join(ROOT, "w4a4_post_quantization_serq_b200", "csrc", rec.get("source", "gemm_mxfp4.cuh"))
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    except (OSError, ValueError):
        return None
    if rec.get("source_sha256_prefix") != sha or rec.get("kernel") != DOMINANT_KERNEL:
        return None
    return rec.get("dram_bytes_per_launch")


def profile_decode(shape: str, M: int, launches: int = 4):
    """A few plain launches of one decode-shape linear on separate weight copies
    (no graph), so a profiler sees ordinary kernels that stream from HBM."""
    import torch
    import w4a4_post_quantization_serq_b200 as S
    from synth import workload
    lin = [l for l in workload("decode_mxfp4").linears if l.name == shape][0]
    W = torch.from_numpy(lin.W()).to(torch.bfloat16).cuda()
    a = S.serq_calib_absmax(torch.from_numpy(lin.X_calib(16)).to(torch.bfloat16).cuda())
    pool = [S.serq_prepare(W, lin.r, lin.fmt, act_absmax=a) for _ in range(launches)]
    qa = S.serq_quant_act(S.serq_fold_producer(pool[0], torch.from_numpy(lin.X(M)).to(torch.bfloat16).cuda()),
                          lin.r, lin.fmt)
    for w in pool:
        S.serq_linear(w, qa)
    torch.cuda.synchronize()
    S.serq_device_status()


def reference_main(args, world, rank, pg):
    """The CPU oracle on a bounded token sample of the same workload (rank 0 only)."""
    from synth import workload
    if rank != 0:
        return
    wl = workload(WORKLOAD)
    rows = args.cpu_rows
    prepared = cpu_oracle_prepare(wl)
    for _ in range(args.warmup):
        cpu_oracle_step(prepared, rows)
    secs, flops, cores = [], 0.0, 1
    t_start = time.perf_counter()
    for _ in range(max(1, args.steps)):
        t, flops, cores = cpu_oracle_step(prepared, rows)
        secs.append(t)
        if time.perf_counter() - t_start > 150:  # keep the run to a few minutes
            break
    mean_t = sum(secs) / len(secs)
    tops = flops / mean_t / 1e12
    sample = (f"{rows} of {wl.M} tokens of every linear ({', '.join(l.name for l in wl.linears)}), r=128: "
              f"oracle quant_act + linear per step; offline prepare untimed")
    line = {"impl": "reference", "metric": METRIC, "value": tops, "unit": "TOPS", "n_gpus": world,
            "steps": len(secs), "warmup": args.warmup, "ms_per_step": mean_t * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64 (fp32 quantization decisions)",
            "data": "synthetic", "config": {"workload": wl.description, "M_sampled": rows},
            "cpu_baseline": {"value": tops, "unit": "TOPS", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": tops, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    world, rank, local, pg = dist_setup(args.gpus)
    if args.impl == "reference":
        reference_main(args, world, rank, pg)
        if pg is not None:
            pg.destroy_process_group()
        return

    import torch
    import w4a4_post_quantization_serq_b200 as S  # noqa: F401  (fails loudly without libserq.so)
    from synth import workload
    if args.profile_decode:
        profile_decode(args.profile_decode, args.decode_m)
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local)
    wl = workload(args.workload)
    if args.only:
        wl.linears = [l for l in wl.linears if l.name == args.only]
        if not wl.linears:
            raise SystemExit(f"no linear named {args.only}")
    layers = build_layers(wl)
    step_flops = sum(L["flops"] for L in layers)

    sampler = ClockSampler(local) if (rank == 0 and not args.no_clocks) else None
    total_ms, gemm_ms, quant_ms = time_steps(layers, args.steps, args.warmup, pg, sampler=sampler)
    clocks = sampler.stop() if sampler is not None else None
    total_ms = max_over_ranks(pg, total_ms)
    ms_per_step = total_ms / args.steps
    value = whole_job_tops(world, step_flops, ms_per_step)

    # dominant kernel: the CTA-pair MXFP4 linear; its largest launch (gate/up,
    # two thirds of the step's flops) is the roofline's unit. The launch lasts
    # ~0.16 ms inside a ~0.3 ms step, so the burst (not the seconds-long
    # sustained) GEMM peak is its denominator.
    peaks, peak_src = measured_peaks()
    dom = max(range(len(layers)), key=lambda i: layers[i]["flops"])
    mx = layers[dom]["lin"].fmt == "mxfp4"
    ratio, ratio_name = (FP4_OVER_BF16, "FP4") if mx else (INT8_OVER_BF16, "INT8")
    peak = peaks["bf16_tflops"] * ratio
    achieved = layers[dom]["flops"] / (gemm_ms[dom] * 1e-3) / 1e12
    traffic = captured_traffic() if mx else None  # the committed capture is of the CTA-pair kernel
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s" if mx else "TOPS",
                "frac": achieved / peak, "traffic": traffic,
                "kernel": DOMINANT_KERNEL if mx else INT_KERNEL, "launch": layers[dom]["lin"].name,
                "flops_per_launch": layers[dom]["flops"],
                "peak_source": f"{peak_src} bf16 burst {peaks['bf16_tflops']} TFLOP/s x "
                               f"{ratio:g} (nominal dense {ratio_name}/BF16 ratio); of measured",
                "frac_of_sustained": achieved / (peaks["bf16_tflops_sustained"] * ratio),
                "quant_act": quant_roofline(layers, quant_ms, peaks["hbm_gbs"]),
                "per_launch_us": {L["lin"].name: round(t * 1e3, 2) for L, t in zip(layers, gemm_ms)},
                "all_launches_tflops": sum(L["flops"] for L in layers) / (sum(gemm_ms) * 1e-3) / 1e12,
                "gemm_share_of_step": sum(gemm_ms) / ms_per_step}

    line = {"metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None,
            "dtype": "mxfp4 (e2m1 x e2m1, e8m0 per 32, fp32 accumulate)" if mx else
                     "int4 (s4 x s4 on the int8 path, int32 accumulate)",
            "data": "synthetic",
            "config": {"workload": wl.description, "M": wl.M, "r": 128,
                       "linears": [{"name": L["lin"].name, "K": L["lin"].K, "N": L["lin"].N} for L in layers],
                       "parallelism": f"replicas x{world}",
                       "l2": "inputs larger than L2 (a step touches ~300 MB)"},
            "roofline": roofline, "gpu_launches": 2 * len(layers) * args.steps, "clocks": clocks}

    if not args.no_extras:
        # end to end through the public API with host buffers, on every rank
        e2e_ms, h2d, d2h = time_e2e(layers, max(3, args.steps // 4), 2, pg)
        e2e_ms = max_over_ranks(pg, e2e_ms)
        line["e2e"] = {"value": whole_job_tops(world, step_flops, e2e_ms), "unit": "TOPS",
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}
    del layers
    torch.cuda.empty_cache()
    if not args.no_extras and rank == 0:
        # SERQ overhead: the same step with r = 0 (plain W4A4)
        layers0 = build_layers(wl, r_override=0)
        t0, g0, _ = time_steps(layers0, args.steps, args.warmup, None)
        del layers0
        torch.cuda.empty_cache()
        line["overhead_vs_r0"] = {"ms_per_step_r0": t0 / args.steps, "step": ms_per_step / (t0 / args.steps) - 1,
                                  "serq_linear": sum(gemm_ms) / sum(g0) - 1}
        # the MLP block with the producers fused (RMSNorm -> quant, SwiGLU -> quant in the gate/up epilogue)
        t_f, parts_f = bench_mlp_fused(wl, args.steps, args.warmup)
        line["mlp_fused"] = {"ms_per_step": t_f, "TOPS": step_flops / (t_f * 1e-3) / 1e12, "per_launch_us": parts_f,
                             "vs_unfused_step": ms_per_step / t_f,
                             "note": "serq_rmsnorm_quant_act -> serq_linear_swiglu_quant -> serq_linear(down); "
                                     "the unfused step has no RMSNorm or SwiGLU kernel at all"}
        # the two-factor baseline (L2QER) at the same rank: its overhead over plain W4A4 against SERQ's
        t_l2 = bench_l2qer(wl, args.steps, args.warmup)
        ms_r0 = t0 / args.steps
        line["l2qer"] = {"ms_per_step": t_l2, "rank": 128,
                         "overhead_ms": t_l2 - ms_r0, "serq_overhead_ms": ms_per_step - ms_r0,
                         "overhead_ratio_l2qer_over_serq": (t_l2 - ms_r0) / max(ms_per_step - ms_r0, 1e-9),
                         "note": "steps with serq_quant_act; L2QER = T = X_q L1_q (bf16), Q(T), X_q W_q + Q(T) L2_q"}
        # INT4: LLaMA-2-7B q_proj shape
        wl2 = workload("qproj_int4")
        layers2 = build_layers(wl2)
        t2, g2, q2 = time_steps(layers2, args.steps, args.warmup, None)
        f2 = sum(L["flops"] for L in layers2)
        line["int4_qproj"] = {"TOPS": f2 / (t2 / args.steps * 1e-3) / 1e12, "ms_per_step": t2 / args.steps,
                              "serq_linear_us": g2[0] * 1e3,
                              "frac_of_int8_peak": f2 / (g2[0] * 1e-3) / 1e12 / (peaks["bf16_tflops"] * 2),
                              "int8_peak_tops": peaks["bf16_tflops"] * 2,
                              "peak_source": "measured bf16 burst x 2 (nominal dense INT8/BF16 ratio); of measured",
                              "quant_act": quant_roofline(layers2, q2, peaks["hbm_gbs"])}
        del layers2
        # W4A8: the same q_proj shape with INT8 activations (the abstract's second setting)
        import dataclasses
        wl8 = workload("qproj_int4")
        wl8.linears = [dataclasses.replace(l, fmt="w4a8") for l in wl8.linears]
        layers8 = build_layers(wl8)
        t8, g8, q8 = time_steps(layers8, args.steps, args.warmup, None)
        f8 = sum(L["flops"] for L in layers8)
        line["w4a8_qproj"] = {"TOPS": f8 / (t8 / args.steps * 1e-3) / 1e12, "ms_per_step": t8 / args.steps,
                              "serq_linear_us": g8[0] * 1e3,
                              "frac_of_int8_peak": f8 / (g8[0] * 1e-3) / 1e12 / (peaks["bf16_tflops"] * 2),
                              "quant_act": quant_roofline(layers8, q8, peaks["hbm_gbs"])}
        del layers8
    if not args.no_extras and rank == 0:
        dec = bench_decode()
        line["decode"] = dec
        m16 = [v["M16"]["GBs"] for k, v in dec.items() if k != "qkv_fused" and isinstance(v, dict) and "M16" in v]
        line["decode_GBs_M16_mean"] = sum(m16) / len(m16)
        line["small_m"] = bench_small_m()
        line["stack"] = bench_stack()
        line["prefill_block"] = bench_prefill_block()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        secs, flops, cores = cpu_oracle_step(cpu_oracle_prepare(wl), args.cpu_rows)
        line["cpu_baseline"] = {"value": flops / secs / 1e12, "unit": "TOPS", "cores": cores, "kind": "oracle",
                                "sample": f"{args.cpu_rows} of {wl.M} tokens of every linear, oracle quant_act + "
                                          f"linear ({secs:.1f} s); offline prepare untimed"}
    if "e2e" not in line:
        line["e2e"] = None
    if rank == 0:
        print(json.dumps(line), flush=True)
    if pg is not None:
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
