#!/usr/bin/env python3
"""Benchmark: shifted-window attention forward + backward on B200.

One step = one pass of the whole path (pad, shift, partition, masked window
attention with relative-position bias, reverse, unshift; then the backward with
dq, dk, dv and the bias-table gradient) over one batch of the synthetic
1/12-degree-shaped workload (256 x 544 tokens, 16 heads x 64, 8 x 8 windows,
shift 4, bf16), inputs resident in HBM. Prints ONE JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
  (N > 1: launched by torch.distributed.run, one process per GPU; every rank
  runs its own batch -- windows and batches are independent, so there is no
  data-path collective; scaling is weak.)

--impl reference times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload (the pages ship no runnable implementation).
"""
import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from shifted_window_attention_pad_b200 import WORKLOADS, BENCH_WORKLOAD  # noqa: E402
from shifted_window_attention_pad_b200.synth import make_inputs  # noqa: E402

FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
L2_BYTES = 126 * 1024 * 1024
METRIC = "shifted-window attn fwd+bwd tokens/s"
# The backward kernel of each kernel family (75-80 % of a step on every workload).
def dominant_kernel(kpath, wl):
    if kpath == 1:
        return ("bwd_kernel<%d,%d> (tcgen05/TMA fused backward: S, dP, dV, dQ, dK, dT)" %
                (wl.head_dim, 8 if wl.win == 8 else 0))
    if kpath == 3:
        return ("wide_bwd_kernel<%d,%d> (tcgen05/TMA backward of 256-token windows: row "
                "statistics, S^T, dP^T, dV, dK, dQ, dT)" % (wl.head_dim, 16 if wl.win == 16 else 0))
    if kpath == 4:
        return ("large_bwdq_kernel<%d> + large_bwdk_kernel<%d> (tcgen05/TMA backward of "
                "1024-token windows: row statistics, dQ and dT by query block; dK and dV by "
                "key block)" % (wl.head_dim, wl.head_dim))
    if kpath == 2:
        return ("tiled_bwd_kernel<%d,%d,32> (warp-MMA backward, one CTA per window and head)" %
                (wl.head_dim, 64 if wl.win ** 2 <= 64 else (128 if wl.win ** 2 <= 128 else 256)))
    return "generic backward kernels (portable, per token)"
# Sources each family's kernels are built from (recorded ncu traffic is used
# only while they are unchanged).
KERNEL_SOURCES = {
    1: ("shifted_window_attention_pad_b200/csrc/fast_sm100.cu",
        "shifted_window_attention_pad_b200/csrc/fast_common.cuh",
        "shifted_window_attention_pad_b200/csrc/sm100_ptx.cuh"),
    3: ("shifted_window_attention_pad_b200/csrc/wide_sm100.cu",
        "shifted_window_attention_pad_b200/csrc/fast_common.cuh",
        "shifted_window_attention_pad_b200/csrc/sm100_ptx.cuh"),
    4: ("shifted_window_attention_pad_b200/csrc/large_sm100.cu",
        "shifted_window_attention_pad_b200/csrc/fast_common.cuh",
        "shifted_window_attention_pad_b200/csrc/sm100_ptx.cuh"),
    2: ("shifted_window_attention_pad_b200/csrc/tiled_mma.cu",
        "shifted_window_attention_pad_b200/csrc/sm100_ptx.cuh"),
    0: ("shifted_window_attention_pad_b200/csrc/generic_kernels.cu",),
}


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=BENCH_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the end-to-end leg (and its second buffer set): profiler captures")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-budget-s", type=float, default=20.0,
                    help="CPU seconds for the oracle baseline sample")
    return ap.parse_args(argv)


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("LOCAL_RANK", 0)),
            int(os.environ.get("WORLD_SIZE", 1)))


def init_dist(world, backend):
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def max_over_ranks(x: float, device=None) -> float:
    """Maximum of a per-rank float over all ranks (identity without a group)."""
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(wl, rank):
    """Each rank draws its own batch of the same shape."""
    return wl.seed + 1000 * rank


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d.get("bf16_tflops", FALLBACK_BF16_TFLOPS)), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def input_bytes(wl):
    """Bytes of q, k, v and dO one step reads (bf16)."""
    return 4 * wl.tokens * wl.heads * wl.head_dim * 2


def needs_l2_flush(wl):
    """Inputs smaller than twice L2 would be served from L2 on the next step."""
    return input_bytes(wl) < 2 * L2_BYTES


def kernel_source_hash(path=1):
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[path]:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload, kpath):
    """DRAM bytes per launch of the dominant kernel from the committed ncu
    summary, or None when absent or taken on a different kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        e = d[workload]
        if e.get("path", 1) != kpath or e.get("source_hash") != kernel_source_hash(kpath):
            return None
        return float(e["bytes_per_launch"])
    except Exception:
        return None


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML (read-only) on a thread."""

    def __init__(self, device, period_s=0.02):
        self.period, self.samples, self.ok = period_s, [], False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            try:
                uuid = "GPU-" + str(torch.cuda.get_device_properties(device).uuid)
                self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(device.index or 0)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((mhz, rs))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        nv = self.nv
        names = {"hw_slowdown": getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8),
                 "hw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
                 "sw_thermal_slowdown": getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
                 "sw_power_cap": getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4)}
        seen = set()
        for _, rs in self.samples:
            for n, bit in names.items():
                if rs & bit:
                    seen.add(n)
        return {"sm_mhz": statistics.median(m for m, _ in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": sorted(seen),
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# CPU oracle legs (baseline and reference arm)
# ---------------------------------------------------------------------------
def oracle_sample_step(wl, rows, nh, inp_np):
    """One oracle forward + backward on the sample: heads 0..nh-1 of the
    workload's first `rows` grid rows of image 0 (a problem of the same window,
    shift and head size). Returns (tokens of the full workload the work stands
    for, seconds)."""
    import oracle
    s = oracle.make_shape(1, rows, wl.W, wl.win, wl.shift, nh, wl.head_dim)
    q, k, v, do = (np.ascontiguousarray(a[:1, :rows, :, :nh].to(torch.float64).numpy())
                   for a in inp_np[:4])
    T = np.ascontiguousarray(inp_np[4][:, :nh].to(torch.float64).numpy())
    t0 = time.perf_counter()
    oracle.forward(s, q, k, v, T)
    oracle.backward(s, q, k, v, T, do)
    dt = time.perf_counter() - t0
    # work is uniform per (token, head): the sample stands for rows*W*nh token-heads
    return rows * wl.W * nh / wl.heads, dt


def oracle_inputs(wl):
    """The workload's inputs (CPU tensors in their storage type; each sample
    widens its own slice to fp64)."""
    inp = make_inputs(wl)
    return inp["q"], inp["k"], inp["v"], inp["dout"], inp["table"]


def pick_sample(wl, budget_s):
    """(rows, heads) of image 0 whose oracle step fits the budget: whole window
    rows of head 0 first, then more heads of the whole grid, from a calibration
    step on one window row of head 0."""
    import oracle
    rows0 = min(wl.win, wl.H)
    inp = oracle_inputs(wl)
    _, dt = oracle_sample_step(wl, rows0, 1, inp)
    per_row = dt / rows0
    rows = max(rows0, min(wl.H, int(budget_s / max(per_row, 1e-9)) // wl.win * wl.win))
    nh = 1
    if rows == wl.H:
        nh = max(1, min(wl.heads, int(budget_s / max(per_row * wl.H, 1e-9))))
    return rows, nh, inp, oracle.num_threads()


def cpu_baseline(wl, budget_s):
    rows, nh, inp, cores = pick_sample(wl, budget_s)
    tok, dt = oracle_sample_step(wl, rows, nh, inp)
    return {"value": tok / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": "fp64 oracle fwd+bwd on heads 0..%d of grid rows 0..%d (x %d cols) of "
                      "image 0; %.1f s; scaled to tokens/s of the full %d-head workload" %
                      (nh - 1, rows - 1, wl.W, dt, wl.heads)}


def run_reference(args):
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    wl = WORKLOADS[args.workload]
    steps, warmup = args.steps, args.warmup
    per_step = max(0.5, min(20.0, 150.0 / max(1, steps + warmup)))
    rows, nh, inp, cores = pick_sample(wl, per_step)
    for _ in range(warmup):
        oracle_sample_step(wl, rows, nh, inp)
    tok_total, t_total = 0.0, 0.0
    for _ in range(steps):
        tok, dt = oracle_sample_step(wl, rows, nh, inp)
        tok_total += tok
        t_total += dt
    value = tok_total / t_total
    sample = ("fp64 oracle fwd+bwd per step on heads 0..%d of grid rows 0..%d (x %d cols) of "
              "image 0, scaled to tokens/s of the full %d-head workload" %
              (nh - 1, rows - 1, wl.W, wl.heads))
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": steps, "warmup": warmup, "ms_per_step": 1e3 * t_total / max(1, steps),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": wl.name, "grid": [wl.B, wl.H, wl.W], "window": wl.win,
                       "shift": wl.shift, "heads": wl.heads, "head_dim": wl.head_dim},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def run_ours(args):
    from shifted_window_attention_pad_b200 import binding as sb

    rank, local, world = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_dist(world, "nccl")
    wl = WORKLOADS[args.workload]
    desc = sb.desc_for(wl)
    inp = make_inputs(wl, seed=rank_seed(wl, rank))
    q, k, v, do = (inp[n].to(dev) for n in ("q", "k", "v", "dout"))
    T = inp["table"].to(dev)
    out, dq, dk, dv = (torch.empty_like(q) for _ in range(4))
    dT = torch.empty_like(T)
    ws = sb.new_workspace(desc, dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        sb.swin_wattn_fwd(desc, q, k, v, T, out, None, ws, stream)
        sb.swin_wattn_bwd(desc, q, k, v, T, do, dq, dk, dv, dT, ws, stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    if sb.swin_wattn_poll_status(ws) != 0:
        raise RuntimeError("device-side timeout during warm-up")

    K = args.steps
    # Inputs smaller than twice the 126 MB L2 would be served from L2 on the
    # next step: flush it before the forward and again before the backward
    # (which would otherwise find q, k, v in L2 from the forward) by writing a
    # 256 MB buffer, and time the steps by their own fwd and bwd events (the
    # flushes are left out).
    in_bytes = input_bytes(wl)
    flush = torch.empty(64 << 20, dtype=torch.float32, device=dev) if needs_l2_flush(wl) else None
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches0 = sb.swin_wattn_launch_count()
    with ClockSampler(dev) as clocks:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        start.record(stream)
        for i in range(K):
            if flush is not None:
                flush.zero_()
            ev[i][0].record(stream)
            sb.swin_wattn_fwd(desc, q, k, v, T, out, None, ws, stream)
            ev[i][1].record(stream)
            if flush is not None:
                flush.zero_()
            ev[i][2].record(stream)
            sb.swin_wattn_bwd(desc, q, k, v, T, do, dq, dk, dv, dT, ws, stream)
            ev[i][3].record(stream)
        end.record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
    launches = sb.swin_wattn_launch_count() - launches0
    if flush is None:
        ms = max_over_ranks(start.elapsed_time(end), dev)
    else:
        ms = max_over_ranks(sum(e[0].elapsed_time(e[1]) + e[2].elapsed_time(e[3]) for e in ev), dev)
    if sb.swin_wattn_poll_status(ws) != 0:
        raise RuntimeError("device-side timeout in the timed region")
    fwd_ms = sum(e[0].elapsed_time(e[1]) for e in ev) / K
    bwd_ms = sum(e[2].elapsed_time(e[3]) for e in ev) / K

    secs = ms / 1e3
    tokens = wl.tokens * K * world
    value = tokens / secs
    tflops = wl.flops_fwd_bwd() * K * world / secs / 1e12
    hbm, _, peak_src = measured_peaks()
    bwd_bytes = wl.alg_bytes_bwd()
    achieved = bwd_bytes / (bwd_ms / 1e3) / 1e9
    fwd_achieved = wl.alg_bytes_fwd() / (fwd_ms / 1e3) / 1e9
    step_gbs = (wl.alg_bytes_fwd() + wl.alg_bytes_bwd()) * K / secs / 1e9

    if args.no_e2e:
        return _finish(args, wl, desc, rank, world, ms, K, fwd_ms, bwd_ms, value, tflops, hbm,
                       peak_src, achieved, fwd_achieved, step_gbs, bwd_bytes, launches, clocks,
                       None, flush, in_bytes)
    # End to end through the public API with pinned host buffers: every step
    # uploads its own inputs and downloads its own results inside the timed
    # region. Two device buffer sets and three streams (upload, compute,
    # download) let step i+1's upload run while step i computes and downloads,
    # as a caller streaming batches would; PCIe is full duplex.
    IN, OUTS = ("q", "k", "v", "dout", "table"), ("o", "dq", "dk", "dv", "dT")
    h_in = {n: inp[n].pin_memory() for n in IN}
    d_in = [{"q": q, "k": k, "v": v, "dout": do, "table": T},
            {n: torch.empty_like(h_in[n], device=dev) for n in IN}]
    d_out = [{"o": out, "dq": dq, "dk": dk, "dv": dv, "dT": dT},
             {"o": torch.empty_like(out), "dq": torch.empty_like(dq), "dk": torch.empty_like(dk),
              "dv": torch.empty_like(dv), "dT": torch.empty_like(dT)}]
    h_out = {n: torch.empty_like(d_out[0][n], device="cpu").pin_memory() for n in OUTS}
    s_up, s_comp, s_down = (torch.cuda.Stream(dev) for _ in range(3))
    up_done, comp_done, down_done = ([torch.cuda.Event() for _ in range(2)] for _ in range(3))

    def e2e_steps(n, start=None, end=None):
        torch.cuda.synchronize(dev)
        if start is not None:
            start.record(s_up)
        for i in range(n):
            b = i & 1
            I, O = d_in[b], d_out[b]
            if i >= 2:
                s_up.wait_event(comp_done[b])      # step i-2 has consumed these inputs
            with torch.cuda.stream(s_up):
                for nm in IN:
                    I[nm].copy_(h_in[nm], non_blocking=True)
            up_done[b].record(s_up)
            s_comp.wait_event(up_done[b])
            if i >= 2:
                s_comp.wait_event(down_done[b])    # step i-2's results are read out
            sb.swin_wattn_fwd(desc, I["q"], I["k"], I["v"], I["table"], O["o"], None, ws, s_comp)
            sb.swin_wattn_bwd(desc, I["q"], I["k"], I["v"], I["table"], I["dout"], O["dq"],
                              O["dk"], O["dv"], O["dT"], ws, s_comp)
            comp_done[b].record(s_comp)
            s_down.wait_event(comp_done[b])
            with torch.cuda.stream(s_down):
                for nm in OUTS:
                    h_out[nm].copy_(O[nm], non_blocking=True)
            down_done[b].record(s_down)
        if end is not None:
            end.record(s_down)                     # the last download ends the chain
        torch.cuda.synchronize(dev)

    e2e_steps(2)
    E = max(1, args.e2e_steps)
    if world > 1:
        dist.barrier()
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_steps(E, s0, s1)
    e2e_ms = max_over_ranks(s0.elapsed_time(s1), dev)
    if sb.swin_wattn_poll_status(ws) != 0:
        raise RuntimeError("device-side timeout in the end-to-end steps")
    h2d = sum(t.numel() * t.element_size() for t in h_in.values())
    d2h = sum(t.numel() * t.element_size() for t in h_out.values())
    e2e = {"value": wl.tokens * E * world / (e2e_ms / 1e3), "unit": "tokens/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
    return _finish(args, wl, desc, rank, world, ms, K, fwd_ms, bwd_ms, value, tflops, hbm,
                   peak_src, achieved, fwd_achieved, step_gbs, bwd_bytes, launches, clocks, e2e,
                   flush, in_bytes)


def roofline_entry(kpath, wl, bwd_ms, achieved_gbs, hbm, peak_src, traffic, bwd_bytes):
    """The backward against its bound. 1024-token windows do N/2 = 512 FLOP per
    byte, past the ridge of the measured peaks, so they are held to the bf16
    tensor peak (burst figure); every other family to HBM bandwidth."""
    if kpath == 4:
        _, tf, src = measured_peaks()
        flops = wl.flops_bwd()
        ach = flops / (bwd_ms / 1e3) / 1e12
        return {"bound": "tensor", "kernel": dominant_kernel(kpath, wl), "achieved": ach,
                "peak": tf, "unit": "TFLOP/s", "frac": ach / tf, "peak_source": src,
                "traffic": traffic, "alg_flops_per_launch": flops,
                "hbm_gbs": achieved_gbs}
    return {"bound": "hbm", "kernel": dominant_kernel(kpath, wl), "achieved": achieved_gbs,
            "peak": hbm, "unit": "GB/s", "frac": achieved_gbs / hbm, "peak_source": peak_src,
            "traffic": traffic, "alg_bytes_per_launch": bwd_bytes}


def _finish(args, wl, desc, rank, world, ms, K, fwd_ms, bwd_ms, value, tflops, hbm, peak_src,
            achieved, fwd_achieved, step_gbs, bwd_bytes, launches, clocks, e2e, flush, in_bytes):
    from shifted_window_attention_pad_b200 import binding as sb

    clk = clocks.summary()
    if world > 1:
        allc = [None] * world
        dist.all_gather_object(allc, clk)
        clk["reasons"] = sorted(set(r for c in allc for r in (c["reasons"] or [])))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, args.cpu_budget_s)

    if rank == 0:
        kpath = sb.swin_wattn_path(desc)
        traffic = recorded_traffic(wl.name, kpath)
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": K, "warmup": max(3, args.warmup), "ms_per_step": ms / K,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl.name, "grid": [wl.B, wl.H, wl.W], "window": wl.win,
                       "shift": wl.shift, "heads": wl.heads, "head_dim": wl.head_dim,
                       "tokens_per_rank_step": wl.tokens, "parallelism": "dp%d" % world,
                       "l2": ("inputs larger than L2 (q,k,v,dO = %.2f GB per step)" % (in_bytes / 1e9)
                              if flush is None else
                              "L2 flushed before the forward and before the backward of every "
                              "step (256 MB write, outside the timed fwd and bwd events; "
                              "q,k,v,dO = %.1f MB per step)" % (in_bytes / 1e6))},
            "tflops": tflops,
            "fwd_ms": fwd_ms, "bwd_ms": bwd_ms,
            "hbm_gbs_step": step_gbs, "hbm_gbs_fwd": fwd_achieved,
            "roofline": roofline_entry(kpath, wl, bwd_ms, achieved, hbm, peak_src, traffic,
                                       bwd_bytes),
            "cpu_baseline": cpu,
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
