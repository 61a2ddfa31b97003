#!/usr/bin/env python
"""Benchmark of the MiMo-V2 attention forward on B200.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step = one attention forward (one layer) over one batch of the workload.
Default workload: the 4096-token sliding-window layer with sink, 64 query /
8 KV heads (the single-GPU configuration the metric is quoted on).

Our arm: inputs already resident in HBM, rotated over several buffer sets
whose total footprint exceeds the 126 MB L2, so consecutive steps never hit
L2 and one CUDA-event pair brackets all K steps (barrier + synchronize on both
sides, max over ranks).  Under torchrun every rank runs its own batch of the
same shape (weak scaling; no data-path collective).  Rank 0 prints one JSON
line.  The reference arm (--impl reference) times the FP64 CPU oracle on
bounded samples of the same workload.
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from global_attention_moe_b200 import workloads as W  # noqa: E402

METRIC = "attn fwd tokens/s and TFLOP/s on 1 B200 (SWA-sink and global); % of roofline"
L2_BYTES = 126 * 2 ** 20
FLOPS_PER_PAIR = 2 * 192 + 2 * 128
# Device code of each forward kernel: the traffic recorded in profiles/traffic.json for a kernel is
# valid only while its files are unchanged.
_COMMON_SOURCES = ["csrc/sm100.cuh", "csrc/rope_smem.cuh", "csrc/params.cuh"]
KERNEL_SOURCES = {
    "attn_fwd_pipelined_kernel": _COMMON_SOURCES + ["csrc/attn_fwd_pipelined.cuh"],
    "attn_fwd_swa_kernel": _COMMON_SOURCES + ["csrc/rope_k_prepass.cuh", "csrc/attn_fwd_swa.cuh"],
    "attn_fwd_swa_packed_kernel": _COMMON_SOURCES + ["csrc/attn_fwd_swa_packed.cuh"],
}
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="swa4096", choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-parity", action="store_true")
    ap.add_argument("--no-secondary", action="store_true",
                    help="SWA-4096 only: skip the global layer's record that the line otherwise carries")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--ref-budget-s", type=float, default=90.0, help="reference arm: total CPU seconds to aim for")
    ap.add_argument("--decode", choices=W.DECODE_KINDS, default=None,
                    help="time the KV-cache path (64 requests x 8 new tokens) instead of the forward")
    ap.add_argument("--decode-requests", type=int, default=64,
                    help="requests in the KV-cache batch (fewer: a smaller case for profiling)")
    ap.add_argument("--step", choices=("bwd", "bwd_tc", "dequant", "split", "proj", "route"), default=None,
                    help="time a step beside the forward instead (backward, FP8 dequant, QKV split, output "
                         "projection, MoE routing)")
    ap.add_argument("--decode-contiguous", action="store_true",
                    help="each request's cache rows in order instead of a random permutation")
    return ap.parse_args()


# ------------------------------------------------------------------ accounting
def bytes_per_step(w: W.Workload) -> int:
    """Algorithmic bytes: q, k, v read once, out and lse written once."""
    T = w.total_tokens
    return T * (2 * w.num_q_heads * w.head_dim_qk + 2 * w.num_kv_heads * w.head_dim_qk
                + 2 * w.num_kv_heads * w.head_dim_v + 2 * w.num_q_heads * w.head_dim_v + 4 * w.num_q_heads)


def flops_per_step(w: W.Workload) -> int:
    return FLOPS_PER_PAIR * W.attended_pairs(w.lengths, w.window, w.num_q_heads)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in ("hbm_gbs", "bf16_tflops", "bf16_tflops_sustained")}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def dominant_kernel(w) -> str:
    """The attention kernel the library's default choice launches for this shape."""
    group = w.num_q_heads // w.num_kv_heads
    if w.layer_kind == W.LAYER_SWA and 0 <= w.window <= 128 and group in (4, 8):
        return "attn_fwd_swa_packed_kernel"
    if group % 2 != 0:
        return "attn_fwd_simple_kernel"
    if w.layer_kind == W.LAYER_SWA and 0 <= w.window <= 128:
        return "attn_fwd_swa_kernel"
    return "attn_fwd_pipelined_kernel"


def host_lead(torch, steps: int, per_step_ms: float = 0.5) -> None:
    """Queues a bounded GPU spin (at most 50 ms) ahead of a timed region, so that the host enqueues the
    first steps while it runs: the events then time the device, not the launch overhead of calls that
    take less GPU time than host time.  The spin ends before the region's first event."""
    ms = min(50.0, max(2.0, steps * per_step_ms))
    torch.cuda._sleep(int(ms * 1e-3 * 1.965e9))


def kernel_sources_sha(kernel: str) -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "global_attention_moe_b200", rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel, {}).get(workload)
    if not e or kernel not in KERNEL_SOURCES or e.get("sources_sha") != kernel_sources_sha(kernel):
        return None
    return float(e["dram_bytes_per_launch"])


# ------------------------------------------------------------------ multi-rank plumbing
def rank_workload(name: str, rank: int) -> W.Workload:
    """Weak scaling: every rank draws its own batch of the workload's shape (seed = rank)."""
    w = W.WORKLOADS[name](seed=0)
    if rank:
        w.seed = rank
    return w


def max_over_ranks(value: float, device=None) -> float:
    """Largest value over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_rate(world: int, units_per_rank_step: int, steps: int, ms_max: float) -> float:
    """Whole-job throughput: the units all ranks processed / the slowest rank's time."""
    return world * units_per_rank_step * steps / (ms_max / 1e3)


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, device_index: int):
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:  # NVML missing: clocks reported as unavailable
            self._ok = False

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.0002)  # short timed regions still get several samples

    def __enter__(self):
        if self._ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self._ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": float(statistics.median(self.samples)), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ------------------------------------------------------------------ CPU oracle
def cpu_oracle_rate(w: W.Workload, x: W.Inputs, target_s: float, max_rows_per_call: int | None = None,
                    threads: int | None = None):
    """Time the oracle (as it stands) on samples of the workload's rows.
    Returns (tokens/s, cores, description)."""
    import oracle
    cores = threads or oracle.default_threads()
    rng = np.random.default_rng(0)
    order = rng.permutation(w.total_tokens)
    # calibrate on a small sample
    n = min(w.total_tokens, 64)
    t0 = time.perf_counter()
    oracle.attn_fwd(x.q, x.k, x.v, x.sink, x.cu_seqlens, w.window, w.rope_base, w.rope_dims, w.v_scale,
                    rows=order[:n], threads=cores)
    t_small = time.perf_counter() - t0
    per_row = max(t_small / n, 1e-6)
    rows = int(min(w.total_tokens, max(1, target_s / per_row)))
    if max_rows_per_call:
        rows = min(rows, max_rows_per_call)
    done, elapsed, calls = 0, 0.0, 0
    while elapsed < target_s and calls < 1000:
        start = (calls * rows) % w.total_tokens
        sel = np.take(order, np.arange(start, start + rows), mode="wrap")
        t0 = time.perf_counter()
        oracle.attn_fwd(x.q, x.k, x.v, x.sink, x.cu_seqlens, w.window, w.rope_base, w.rope_dims, w.v_scale,
                        rows=sel, threads=cores)
        elapsed += time.perf_counter() - t0
        done += rows
        calls += 1
        if rows == w.total_tokens and elapsed >= 0.5 * target_s:
            break
    desc = (f"{calls} oracle call(s) of {rows} seeded-random token rows (all {w.num_q_heads} heads each) of "
            f"{w.name} on {cores} host thread(s); {elapsed:.1f} s of CPU time")
    return done / elapsed, cores, desc


# ------------------------------------------------------------------ reference arm
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    w = W.WORKLOADS[args.workload]()
    x = W.make_inputs(w)
    import oracle
    cores = oracle.default_threads()
    rng = np.random.default_rng(0)
    order = rng.permutation(w.total_tokens)
    n = min(w.total_tokens, 32)
    t0 = time.perf_counter()
    oracle.attn_fwd(x.q, x.k, x.v, x.sink, x.cu_seqlens, w.window, w.rope_base, w.rope_dims, w.v_scale,
                    rows=order[:n], threads=cores)
    per_call_fixed_and_rows = time.perf_counter() - t0
    per_row = per_call_fixed_and_rows / n
    total_steps = max(1, args.steps + args.warmup)
    rows = int(max(1, min(w.total_tokens, args.ref_budget_s / total_steps / max(per_row, 1e-6))))

    def step(i):
        start = (i * rows) % w.total_tokens
        sel = np.take(order, np.arange(start, start + rows), mode="wrap")
        oracle.attn_fwd(x.q, x.k, x.v, x.sink, x.cu_seqlens, w.window, w.rope_base, w.rope_dims, w.v_scale,
                        rows=sel, threads=cores)

    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(args.warmup + i)
    el = time.perf_counter() - t0
    value = args.steps * rows / el
    sample = (f"each step: {rows} seeded-random token rows (all {w.num_q_heads} heads) of {w.name}, "
              f"FP64 C oracle on {cores} host threads")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / max(args.steps, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {**w.describe(), "rows_per_step": rows},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm
TC_FLOP_PER_CLK_SM = 8192  # dense BF16 tcgen05: one M128 N256 K16 MMA (1 MFLOP) per 128 cycles per SM
SECONDARY = {"swa4096": "global"}  # the metric names both layer kinds: the SWA line carries the global one


def launches_per_step(w) -> int:
    """This library's kernels per forward: the attention kernel, plus the K RoPE pre-pass where the
    chosen kernel reads K's rope dims pre-rotated."""
    return 2 if dominant_kernel(w) in ("attn_fwd_pipelined_kernel", "attn_fwd_swa_kernel") else 1


def percentiles(xs):
    xs = sorted(xs)
    pick = lambda f: xs[min(len(xs) - 1, max(0, int(round(f * (len(xs) - 1)))))]
    return {"p10": pick(0.10), "p50": pick(0.50), "p90": pick(0.90), "n": len(xs)}


def measure(args, w, rank, world, dev, with_cpu: bool):
    """Times one workload on this rank: K steps over rotating input sets (one event pair around all,
    one per step), the attention kernel alone (library events), a repeat on one input set, the
    end-to-end host-buffer entry, a parity spot check and the CPU oracle.  Returns a dict of fields."""
    import torch
    import torch.distributed as dist

    from global_attention_moe_b200 import mimo_attn

    x = W.make_inputs(w)
    T = w.total_tokens
    stream = torch.cuda.current_stream()
    sh = ctypes.c_void_p(stream.cuda_stream)

    def dev_set():
        q = torch.from_numpy(x.q.view(np.int16)).to(dev).view(torch.bfloat16)
        k = torch.from_numpy(x.k.view(np.int16)).to(dev).view(torch.bfloat16)
        v = torch.from_numpy(x.v.view(np.int16)).to(dev).view(torch.bfloat16)
        s = None if x.sink is None else torch.from_numpy(x.sink).to(dev)
        cu = torch.from_numpy(x.cu_seqlens).to(dev)
        out = torch.empty(T, w.num_q_heads, w.head_dim_v, dtype=torch.bfloat16, device=dev)
        lse = torch.empty(w.num_q_heads, T, dtype=torch.float32, device=dev)
        return q, k, v, s, cu, out, lse

    set_bytes = bytes_per_step(w)
    n_sets = max(2, -(-3 * L2_BYTES // set_bytes))
    sets = [dev_set() for _ in range(n_sets)]
    dims = mimo_attn.make_dims(w.num_seqs, T, w.max_seqlen, w.num_q_heads, w.num_kv_heads)
    calls = [(q.data_ptr(), k.data_ptr(), v.data_ptr(), s.data_ptr() if s is not None else None, cu.data_ptr(),
              out.data_ptr(), lse.data_ptr()) for (q, k, v, s, cu, out, lse) in sets]
    fn = mimo_attn.LIB.mimo_attn_fwd
    dref = ctypes.byref(dims)
    lk, win, base, rd, vs = w.layer_kind, w.window, w.rope_base, w.rope_dims, w.v_scale

    def step(i):
        a = calls[i % n_sets]
        st = fn(a[0], a[1], a[2], a[3], a[4], dref, lk, win, base, rd, vs, a[5], a[6], sh)
        if st != 0:
            raise mimo_attn.MimoAttnError(st, "mimo_attn_fwd")

    for i in range(max(args.warmup, 0)):
        step(i)
    st = mimo_attn.check()
    if st != mimo_attn.OK:
        raise mimo_attn.MimoAttnError(st, "warm-up")

    # K steps: one event pair around all of them (the value), one event per step boundary (spread)
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    # the attention kernel's own launches are timed by library-recorded event pairs around every 16th
    # launch, on the launching stream, over this same region (a pair around every launch adds about
    # 5 us to a 72 us step)
    mimo_attn.profile_set_stride(16 if args.steps >= 64 else 1)
    mimo_attn.profile_start()
    with ClockSampler(dev.index) as clk:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        host_lead(torch, args.steps)
        ev0.record(stream)
        for i in range(args.steps):
            evs[i].record(stream)
            step(i)
        evs[args.steps].record(stream)
        ev1.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
    n_rec, tot = mimo_attn.profile_stop()
    kernel_ms = max_over_ranks(tot / n_rec, dev) if n_rec else None
    ms = ev0.elapsed_time(ev1)
    per_step = [evs[i].elapsed_time(evs[i + 1]) for i in range(args.steps)]
    st = mimo_attn.check()
    if st != mimo_attn.OK:
        raise mimo_attn.MimoAttnError(st, "timed region")
    ms = max_over_ranks(ms, dev)
    ms_per_step = ms / max(args.steps, 1)
    n_launch = launches_per_step(w)

    # the same K steps on one input set (its inputs partly L2-resident between steps): context only
    torch.cuda.synchronize()
    w0, w1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    w0.record(stream)
    for _ in range(args.steps):
        step(0)
    w1.record(stream)
    torch.cuda.synchronize()
    warm_ms = max_over_ranks(w0.elapsed_time(w1), dev) / max(args.steps, 1)

    # end to end through the host-buffer C-ABI entry (pinned host memory, copies inside the region)
    e2e = None
    if not args.no_e2e:
        pin = lambda a: torch.from_numpy(a).pin_memory()
        qh, kh, vh = (pin(a.view(np.int16)) for a in (x.q, x.k, x.v))
        shh = pin(x.sink) if x.sink is not None else None
        ch = pin(x.cu_seqlens)
        oh = torch.empty(T, w.num_q_heads, w.head_dim_v, dtype=torch.int16).pin_memory()
        lh = torch.empty(w.num_q_heads, T, dtype=torch.float32).pin_memory()
        ws = torch.empty(mimo_attn.host_workspace_size(dims, x.sink is not None), dtype=torch.uint8, device=dev)
        h2d = sum(a.numel() * a.element_size() for a in (qh, kh, vh, ch) + ((shh,) if shh is not None else ()))
        d2h = oh.numel() * 2 + lh.numel() * 4
        for _ in range(2):
            mimo_attn.fwd_host(qh, kh, vh, shh, ch, dims, lk, win, base, rd, vs, oh, lh, ws)
        ne = max(1, min(args.e2e_steps, args.steps))
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(ne):
            mimo_attn.fwd_host(qh, kh, vh, shh, ch, dims, lk, win, base, rd, vs, oh, lh, ws)
        e1.record(stream)
        torch.cuda.synchronize()
        ems = max_over_ranks(e0.elapsed_time(e1), dev)
        e2e = {"value": aggregate_rate(world, T, ne, ems), "unit": "tokens/s", "h2d_bytes_per_step": int(h2d),
               "d2h_bytes_per_step": int(d2h), "steps": ne}
        del qh, kh, vh, shh, ch, oh, lh, ws

    # parity spot check of this run's output against the oracle (rank 0)
    parity = None
    if rank == 0 and not args.no_parity:
        import oracle
        q, k, v, s, cu, out, lse = sets[(args.steps - 1) % n_sets]
        rng = np.random.default_rng(1)
        rows = np.unique(np.concatenate([[0, T - 1, min(T - 1, 128)], rng.integers(0, T, 24)])).astype(np.int64)
        ro, rl = oracle.attn_fwd(x.q, x.k, x.v, x.sink, x.cu_seqlens, w.window, w.rope_base, w.rope_dims, w.v_scale,
                                 rows=rows)
        idx = torch.from_numpy(rows).to(dev)
        go = out.index_select(0, idx).float().cpu().numpy().astype(np.float64)
        gl = lse.index_select(1, idx).cpu().numpy().astype(np.float64)
        d = go - ro
        parity = {"rows": int(len(rows)), "max_abs": float(np.abs(d).max()),
                  "rel_l2": float(np.linalg.norm(d) / np.linalg.norm(ro)), "lse_max_abs": float(np.abs(gl - rl).max())}

    cpu = None
    if rank == 0 and world == 1 and with_cpu and not args.no_cpu_baseline:
        rate, cores, desc = cpu_oracle_rate(w, x, target_s=10.0)
        cpu = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": desc}
        if w.name in ("swa_sink_T4096_h64_kv8", "tiny_swa_sink_T512_h4_kv1"):
            r1, _, d1 = cpu_oracle_rate(w, x, target_s=3.0, threads=1)
            cpu["single_thread"] = {"value": r1, "unit": "tokens/s", "cores": 1, "sample": d1}
    del sets
    torch.cuda.empty_cache()

    clocks = clk.summary()
    peaks, peak_src = load_peaks()
    flops = flops_per_step(w)
    nbytes = bytes_per_step(w)
    t_s = ms_per_step / 1e3
    tk_s = (kernel_ms if kernel_ms else ms_per_step) / 1e3  # the attention kernel's own launch duration
    t_hbm = nbytes / (peaks["hbm_gbs"] * 1e9)
    long_region = ms > 1000.0
    tc_peak = peaks["bf16_tflops_sustained" if long_region else "bf16_tflops"]
    t_tc = flops / (tc_peak * 1e12)
    kernel = dominant_kernel(w)
    if t_hbm >= t_tc:
        ach = nbytes / tk_s / 1e9
        roof = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": ach / peaks["hbm_gbs"]}
    else:
        ach = flops / tk_s / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": tc_peak, "unit": "TFLOP/s", "frac": ach / tc_peak}
        if clocks.get("sm_mhz"):
            issue_peak = 148 * TC_FLOP_PER_CLK_SM * clocks["sm_mhz"] * 1e6 / 1e12
            roof["tcgen05_issue_peak"] = {
                "tflops": issue_peak, "frac": ach / issue_peak,
                "basis": "148 SMs x 8192 dense BF16 FLOP/clk/SM (M128 N256 K16 MMA in 128 cycles) x the median "
                         "SM clock sampled in the timed region; a labelled second ratio, not the roofline peak"}
    roof.update({"traffic": recorded_traffic(kernel, w.name),
                 "peak_source": f"{peak_src} ({'sustained' if long_region and roof['bound'] == 'tensor' else 'burst'})",
                 "kernel": kernel, "algorithmic_bytes": nbytes, "algorithmic_flops": flops,
                 "kernel_us": tk_s * 1e6, "step_frac": tk_s / t_s})
    return {
        "value": aggregate_rate(world, T, args.steps, ms), "ms_per_step": ms_per_step,
        "per_step_ms": percentiles(per_step), "warm_l2_ms_per_step": warm_ms,
        "config": {**w.describe(), "parallelism": f"replicas{world}" if world > 1 else "single",
                   "l2": f"inputs rotated over {n_sets} device buffer sets ({n_sets * set_bytes / 2**20:.0f} MiB > "
                         f"126 MiB L2), no flush"},
        "tflops": flops / t_s / 1e12, "gbs": nbytes / t_s / 1e9, "roofline_time_us": max(t_hbm, t_tc) * 1e6,
        "roofline": roof, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": args.steps * n_launch,
        "clocks": clocks, "parity": parity,
    }


def run_ours(args):
    import torch
    import torch.distributed as dist

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus and rank == 0:
        print(f"warning: WORLD_SIZE={world} but --gpus={args.gpus}", file=sys.stderr)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    main = measure(args, rank_workload(args.workload, rank), rank, world, dev, with_cpu=True)
    second = None
    if args.workload in SECONDARY and not args.no_secondary:
        second = measure(args, rank_workload(SECONDARY[args.workload], rank), rank, world, dev, with_cpu=True)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": main["value"], "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": main["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
    }
    line.update({k: v for k, v in main.items() if k not in ("value", "ms_per_step")})
    if second is not None:
        # the other layer kind of the metric, measured the same way in the same run
        line["gpu_launches"] += second["gpu_launches"]
        line["global_layer"] = {"metric": METRIC, "unit": "tokens/s", "steps": args.steps, "warmup": args.warmup,
                                **second}
    print(json.dumps(line), flush=True)
    return 0


DECODE_METRIC = "KV-cache attention (page size 1) new tokens/s on 1 B200; % of HBM roofline"


def decode_bytes_flops(x, window):
    """Algorithmic bytes (K/V rows the queries can see, read once with their indices; q read, out
    and lse written once) and FLOPs (640 per attended pair) of one KV-cache step."""
    hq, hkv = x.q.shape[1], x.k_cache.shape[1]
    keys = pairs = 0
    for kv, q in zip(x.kv_lens, x.q_lens):
        keys += min(kv, window + q) if window >= 0 else kv
        for i in range(q):
            p = kv - q + i
            pairs += min(p + 1, window + 1) if window >= 0 else p + 1
    Tq = x.q.shape[0]
    nbytes = keys * (hkv * (192 + 128) * 2 + 4) + Tq * hq * (192 * 2 + 128 * 2 + 4)
    return nbytes, FLOPS_PER_PAIR * pairs * hq


def run_decode(args):
    """The KV-cache path on a serving-shaped batch; one JSON line (single GPU)."""
    import torch
    import oracle
    from global_attention_moe_b200 import mimo_attn

    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    n_sets = 4 if args.decode == "swa" else 1  # the sliding layer's rows per step fit in L2: rotate
    sets = []
    for seed in range(n_sets):
        x, layer, window, base = W.decode_batch(args.decode, seed=seed, num_seqs=args.decode_requests,
                                                contiguous=args.decode_contiguous)
        t = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
        i32 = lambda a: torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).cuda()
        dev = (t(x.q), t(x.k_cache), t(x.v_cache), i32(x.kv_indices), i32(x.kv_indptr), i32(x.cu_q),
               None if x.sink is None else torch.from_numpy(x.sink).cuda())
        out = torch.empty(x.q.shape[0], 64, 128, dtype=torch.bfloat16, device="cuda")
        lse = torch.empty(64, x.q.shape[0], dtype=torch.float32, device="cuda")
        sets.append((x, dev, out, lse))
    x0 = sets[0][0]
    Tq = x0.q.shape[0]
    set_bytes = sum(a.numel() * a.element_size() for a in sets[0][1] if a is not None)

    def step(i):
        x, (q, kc, vc, idx, indptr, cuq, sk), out, lse = sets[i % n_sets]
        mimo_attn.decode(q, kc, vc, idx, indptr, cuq, sk, max(x.q_lens), max(x.kv_lens), layer, window, base,
                         out=out, lse=lse)

    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize()
    assert mimo_attn.check() == mimo_attn.OK
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        torch.cuda.synchronize()
        host_lead(torch, args.steps)  # a step's host work (allocation, three launches) exceeds its GPU time
        e0.record()
        for i in range(args.steps):
            step(i)
        e1.record()
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    st = mimo_attn.check()
    if st != mimo_attn.OK:
        raise RuntimeError(mimo_attn.status_string(st))
    # parity spot check and CPU baseline: the first two requests of set 0 through the oracle
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from decode_helpers import decode_reference
    sub = W.decode_subset(x0, [0, 1])
    t0 = time.time()
    ro, rl = decode_reference(sub, window, base)
    cpu_s = time.time() - t0
    step(0)
    torch.cuda.synchronize()
    rows = int(sub.q.shape[0])
    g_out = sets[0][2][:rows].float().cpu().numpy().astype(np.float64)
    g_lse = sets[0][3][:, :rows].cpu().numpy().astype(np.float64)
    d = g_out - ro
    parity = {"rows": rows, "max_abs": float(np.abs(d).max()), "rel_l2": float(np.linalg.norm(d) / np.linalg.norm(ro)),
              "lse_max_abs": float(np.abs(g_lse - rl).max())}
    nbytes, flops = decode_bytes_flops(x0, window)
    peaks, peak_src = load_peaks()
    ach = nbytes / (ms / 1e3) / 1e9
    line = {
        "metric": DECODE_METRIC, "value": Tq / (ms / 1e3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": f"decode_{args.decode}_B{len(x0.kv_lens)}_q{max(x0.q_lens)}_kv1024-8192",
                   "layer": "swa_sink" if args.decode == "swa" else "global_causal", "requests": len(x0.kv_lens),
                   "new_tokens": Tq, "context_tokens": int(sum(x0.kv_lens)), "q_heads": 64,
                   "kv_heads": int(x0.k_cache.shape[1]), "page_size": 1,
                   "cache_rows": "in request order" if args.decode_contiguous else "random permutation",
                   "l2": f"{n_sets} input sets rotated ({n_sets * set_bytes / 2**20:.0f} MiB on the device)"},
        "tflops": flops / (ms / 1e3) / 1e12, "gbs": ach,
        "roofline": {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": ach / peaks["hbm_gbs"], "traffic": None, "peak_source": f"{peak_src} (burst)",
                     "kernel": "attn_decode_tc_kernel + attn_decode_combine_kernel",
                     "algorithmic_bytes": nbytes, "algorithmic_flops": flops},
        "cpu_baseline": {"value": rows / cpu_s, "unit": "tokens/s", "cores": oracle.default_threads(),
                         "kind": "oracle", "sample": f"the first two requests of the batch ({rows} new tokens)"},
        "e2e": None,
        "gpu_launches": args.steps * 2,
        "clocks": clk.summary(),
        "parity": parity,
    }
    print(json.dumps(line), flush=True)
    return 0


STEP_KINDS = ("bwd", "bwd_tc", "dequant", "split", "proj", "route")
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12  # CUDA-core FP32 FMA peak at the maximum SM clock


# Shapes of the step lines (synthetic, layer-shaped) and their algorithmic FLOPs / bytes: every tensor
# moved once, masked work and the exponentials not counted.
STEP_SHAPES = {
    "dequant": dict(M=8 * (8 * 192 + 320), N=4096, block=128),  # a fused qkv_proj weight, hidden 4096
    "split": dict(T=16384, hq=64, hkv=8),
    "proj": dict(T=4096, K=64 * 128, N=4096),  # 64 heads x 128 dims -> hidden 4096
    "route": dict(T=262144, E=256, k=8),
}


def step_accounting(kind):
    """(FLOPs, bytes, units) of one call of a step line; the backward on the swa4096 workload."""
    if kind in ("bwd", "bwd_tc"):
        w = W.WORKLOADS["swa4096"]()
        flops = W.attended_pairs(w.lengths, w.window, w.num_q_heads) * (2 * 192 * 3 + 2 * 128 * 2)  # S dQ dK; dP dV
        nbytes = w.total_tokens * (w.num_q_heads * (192 * 2 + 128 * 2 * 2 + 4 + 192 * 4)  # q, out, dout, lse, dq
                                   + w.num_kv_heads * (192 * 2 + 128 * 2 + 192 * 4 + 128 * 4))  # k, v, dk, dv
        return flops, nbytes, w.total_tokens
    s = STEP_SHAPES[kind]
    if kind == "dequant":
        M, N, b = s["M"], s["N"], s["block"]
        return 0, M * N * 3 + (-(-M // b)) * (-(-N // b)) * 4, M * N  # codes in, bf16 out, scales
    if kind == "split":
        width = s["hkv"] * (s["hq"] // s["hkv"] * 192 + 320)
        return 0, s["T"] * width * 2 * 2, s["T"]  # every element read once and written once
    if kind == "proj":
        T, K, N = s["T"], s["K"], s["N"]
        return 2 * T * K * N, 2 * (T * K + N * K + T * N), T
    T, E, k = s["T"], s["E"], s["k"]
    return 0, T * E * 4 + E * 4 + T * k * 8, T  # logits, bias, ids + weights


def run_step(args):
    """One of the steps beside the forward (backward, FP8 dequant, fused-QKV split, MoE routing) on a
    layer-shaped synthetic input; one JSON line (single GPU)."""
    import torch
    from global_attention_moe_b200 import mimo_attn, synth

    if int(os.environ.get("RANK", "0")) != 0:
        return 0
    torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", "0")))
    rng = np.random.default_rng(0)
    peaks, peak_src = load_peaks()
    kind = args.step
    tensor_bwd = kind == "bwd_tc"
    if kind in ("bwd", "bwd_tc"):  # bwd: the FP32 CUDA-core kernel; bwd_tc: the tensor-core one (the default)
        mimo_attn.set_bwd_kernel(mimo_attn.BWD_TENSOR if tensor_bwd else mimo_attn.BWD_CUDA_CORES)
        kind = "bwd"
    if kind == "bwd":
        w = W.WORKLOADS["swa4096"]()
        x = W.make_inputs(w)
        dev = lambda a: torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)
        q, k, v = dev(x.q), dev(x.k), dev(x.v)
        sk = torch.from_numpy(x.sink).cuda()
        cu = torch.from_numpy(x.cu_seqlens).cuda()
        out, lse = mimo_attn.fwd(q, k, v, sk, cu, w.max_seqlen, w.layer_kind, w.window, w.rope_base)
        go = dev(synth.f32_to_bf16_bits(rng.standard_normal((w.total_tokens, w.num_q_heads, 128)).astype(np.float32)))
        call = lambda: mimo_attn.bwd(q, k, v, sk, cu, w.max_seqlen, w.layer_kind, w.window, w.rope_base, out, lse, go)
        flops, nbytes, units = step_accounting("bwd")
        unit = "tokens/s"
        config = {"workload": ("bwd_tc_" if tensor_bwd else "bwd_") + w.name, "grads": "fp32",
                  "kernel": "tcgen05, bf16 operands" if tensor_bwd else "fp32 cuda cores"}
        bound = "tensor" if tensor_bwd else "alu"  # BF16 tcgen05 MMAs / FP32 FMAs on the CUDA cores
    elif kind == "dequant":
        # a fused qkv_proj weight of the sliding layer (hidden 4096, synthetic): 61 MB of codes, 122 MB out
        M_, N_ = STEP_SHAPES["dequant"]["M"], STEP_SHAPES["dequant"]["N"]
        codes = rng.integers(0, 256, size=(M_, N_)).astype(np.uint8)
        codes[(codes & 0x7F) == 0x7F] = 0x3F
        scale = rng.uniform(0.5, 2.0, size=(-(-M_ // 128), -(-N_ // 128))).astype(np.float32)
        ct, st = torch.from_numpy(codes).cuda(), torch.from_numpy(scale).cuda()
        call = lambda: mimo_attn.fp8_dequant_blockwise(ct, st)
        flops, nbytes, units = step_accounting("dequant")
        unit, config, bound = "elements/s", {"workload": f"fp8_dequant_{M_}x{N_}_block128"}, "hbm"
    elif kind == "split":
        T, hq, hkv = (STEP_SHAPES["split"][n] for n in ("T", "hq", "hkv"))  # 486 MB in and out: larger than L2
        fused = torch.from_numpy(rng.integers(0, 1 << 16, size=(T, hkv * (hq // hkv * 192 + 320))).astype(np.uint16)
                                 .view(np.int16)).cuda().view(torch.bfloat16)
        call = lambda: mimo_attn.qkv_split(fused, hq, hkv)
        flops, nbytes, units = step_accounting("split")
        unit, config, bound = "tokens/s", {"workload": f"qkv_split_T{T}_hq{hq}_hkv{hkv}"}, "hbm"
    elif kind == "proj":
        # the sliding layer's output projection: 64 heads x 128 dims -> hidden 4096 (synthetic), T = 4096
        T, K_, N_ = (STEP_SHAPES["proj"][n] for n in ("T", "K", "N"))
        bf = lambda a: torch.from_numpy((a.astype(np.float32).view(np.uint32) >> np.uint32(16)).astype(np.uint16)
                                        .view(np.int16)).cuda().view(torch.bfloat16)
        xt, wt = bf(rng.standard_normal((T, K_))), bf(rng.standard_normal((N_, K_)) / np.sqrt(K_))
        call = lambda: mimo_attn.linear_proj(xt, wt)
        flops, nbytes, units = step_accounting("proj")
        unit, config, bound = "tokens/s", {"workload": f"linear_proj_T{T}_in{K_}_out{N_}"}, "tensor"
    else:
        T, E = STEP_SHAPES["route"]["T"], STEP_SHAPES["route"]["E"]  # 268 MB of logits: larger than L2
        lg = torch.from_numpy((rng.standard_normal((T, E)) * 2).astype(np.float32)).cuda()
        bias = torch.from_numpy((rng.standard_normal(E) * 0.1).astype(np.float32)).cuda()
        call = lambda: mimo_attn.moe_route(lg, bias, 8)
        flops, nbytes, units = step_accounting("route")
        unit, config, bound = "tokens/s", {"workload": f"moe_route_T{T}_E{E}_top8"}, "hbm"
    for _ in range(max(3, args.warmup)):
        call()
    torch.cuda.synchronize()
    assert mimo_attn.check() == mimo_attn.OK
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    steps = args.steps
    with ClockSampler(torch.cuda.current_device()) as clk:
        torch.cuda.synchronize()
        host_lead(torch, steps)
        e0.record()
        for _ in range(steps):
            call()
        e1.record()
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    assert mimo_attn.check() == mimo_attn.OK
    if bound == "hbm":
        ach, peak, runit = nbytes / (ms / 1e3) / 1e9, peaks["hbm_gbs"], "GB/s"
    elif bound == "tensor":
        ach, peak, runit = flops / (ms / 1e3) / 1e12, peaks["bf16_tflops"], "TFLOP/s"
    else:
        ach, peak, runit = flops / (ms / 1e3) / 1e12, FP32_ALU_TFLOPS, "TFLOP/s"
        peak_src = "derived: 148 SMs x 128 FP32 lanes x 2 FLOP per FMA x 1965 MHz"
    line = {
        "metric": f"{'bwd_tc' if tensor_bwd else kind} throughput on 1 B200; % of roofline", "value": units / (ms / 1e3),
        "unit": unit,
        "n_gpus": 1, "steps": steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if kind != "route" else "f32", "data": "synthetic",
        "config": dict(config, l2="inputs larger than L2"),
        "roofline": {"bound": bound, "achieved": ach, "peak": peak, "unit": runit, "frac": ach / peak, "traffic": None,
                     "peak_source": peak_src if bound == "alu" else f"{peak_src} (burst)", "algorithmic_bytes": nbytes, "algorithmic_flops": flops},
        "e2e": None, "clocks": clk.summary(),
        # this library's kernels per step (the projection's GEMM runs in cuBLAS)
        "gpu_launches": steps * ({"bwd": 3, "dequant": 1, "split": 1, "route": 1, "proj": 0}[kind] - tensor_bwd),
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    if args.decode:
        return run_decode(args)
    if args.step:
        return run_step(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
