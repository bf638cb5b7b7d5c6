"""Benchmark of the partitioned-attention step with selective state reuse.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

A step is one pass of the whole hot path over one batch: the plan, the
partial attention of the fresh pairs and the log-sum-exp merge (with the
cache refreshed in place), through the library's C ABI.  The default
workload is the frame-tile sparse attention over a 29-frame 720p latent
(8 frames x 3600 tokens, B=1, H=24, d=96).  Metric: effective attention
TFLOP/s, counting only the freshly computed (query partition, KV partition)
blocks: 4 * d * B * H * sum over fresh pairs of L_i * L_j.

Several GPUs run independent replicas (one process per GPU under torchrun);
the path has no exchange between GPUs.  --impl reference times the fp64 CPU
oracle on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import configs, inputs  # noqa: E402

DEFAULT_WORKLOAD = configs.DENSE.name
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ------------------------------------------------------------------ counting
def pair_mask(w):
    """Active pairs of the workload, from the library's host logic."""
    import sparse_state_reuse_b200 as dt
    g = dt.Geometry(w.B, w.H, w.N, w.d, w.part_off(), w.frame_off(), w.frame_mask())
    return np.array(dt.ditango_slot_table(g)) >= 0


def effective_flops(w, fresh_mask):
    """4 d B H sum over fresh active pairs of L_i L_j (fresh_mask: [P, P])."""
    po = np.array(w.part_off())
    L = np.diff(po)
    return float(4.0 * w.d * w.BH * (np.outer(L, L) * fresh_mask).sum())


def fresh_pairs_of_units(w, plan_units, A_pairs):
    """[P, P] fresh active pairs of a plan over KV groups: pair (i, j) is
    computed when it is active and the unit (i, group of j) is fresh."""
    go = w.group_off()
    col = np.zeros(w.P, dtype=np.int64)
    for c in range(len(go) - 1):
        col[go[c]:go[c + 1]] = c
    return A_pairs & (plan_units[:, col] == 1)


def merge_bytes(w, A, fresh_mask, out_bytes_per_elem=2, writeback=False, state_o_bytes=4,
                mass_partials=True):
    """Algorithmic HBM bytes of the merge: every active state read once
    (d O values of state_o_bytes each + an fp32 lse per row), the output
    written once (d elements + fp32 lse), the mass partials (one float per
    KV column per block of 128 rows of each (b*h, partition)), plus the
    write-back of fresh states when they are copied."""
    po = np.array(w.part_off())
    L = np.diff(po)
    rows_states = (A.sum(axis=1) * L).sum() * w.BH
    row_state = w.d * state_o_bytes + 4
    b = rows_states * row_state + w.BH * w.N * (w.d * out_bytes_per_elem + 4)
    if mass_partials:
        b += float(np.ceil(L / 128.0).sum()) * w.BH * A.shape[1] * 4
    if writeback:
        b += (fresh_mask.sum(axis=1) * L).sum() * w.BH * row_state
    return float(b)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d, "measured"
    return PEAKS_FALLBACK, "fallback"


def kernel_source_hash(name):
    csrc = os.path.join(ROOT, "sparse_state_reuse_b200", "csrc")
    files = [name, "common.cuh"] + (["weights.cuh"] if name in ("merge.cu", "plan.cu") else [])
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel_file, workload):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current source of the kernel; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(kernel_file, {}).get(workload)
    if not e or e.get("source_hash") != kernel_source_hash(kernel_file):
        return None
    return e.get("dram_bytes_per_launch")


# ------------------------------------------------------------------ ranks
def max_over_ranks(x, device, dist=None):
    """Max of a per-rank float over all ranks (the slowest replica sets the
    time); identity on one process."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(world, flops_per_replica, ms_per_step):
    """Whole-job effective TFLOP/s: every replica does the same step."""
    return world * flops_per_replica / (ms_per_step * 1e-3) / 1e12


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi in a process of its own (it takes nothing from this one)
    samples the GPU every 20 ms with a timestamp; stop(t0, t1) keeps the
    samples taken inside the timed region [t0, t1] (host wall clock), or the
    first one after t0 when the region is shorter than the sampling period.
    Reads only, changes nothing."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index, period_ms=20):
        self.idx = gpu_index
        self.period_ms = period_ms
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", str(self.period_ms)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self, t0=None, t1=None):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        return summarise_clocks(out, t0, t1)


def _smi_time(stamp):
    """Host epoch seconds of an nvidia-smi timestamp (local time,
    "YYYY/MM/DD HH:MM:SS.mmm"), or None."""
    try:
        day, clock = stamp.split(" ")
        whole, _, frac = clock.partition(".")
        st = time.strptime(f"{day} {whole}", "%Y/%m/%d %H:%M:%S")
        return time.mktime(st) + (float("0." + frac) if frac else 0.0)
    except ValueError:
        return None


def summarise_clocks(csv_text, t0=None, t1=None):
    """Median SM clock, the highest max clock and every throttle reason seen
    Active, from nvidia-smi lines of ClockSampler.FIELDS (no header, no
    units); with t0/t1, only the lines stamped inside [t0, t1], else the
    first line after t0.  None when no line qualifies."""
    lines = []
    for line in csv_text.strip().splitlines():
        parts = [x.strip() for x in line.split(",")]
        if len(parts) < 10:
            continue
        lines.append((_smi_time(parts[0]), parts[1:]))
    if t0 is not None and t1 is not None:
        inside = [ln for ln in lines if ln[0] is not None and t0 <= ln[0] <= t1]
        if not inside:
            after = [ln for ln in lines if ln[0] is not None and ln[0] >= t0]
            inside = after[:1]
        lines = inside
    sm, mx, reasons = [], 0.0, set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for _, parts in lines:
        try:
            sm.append(float(parts[1]))
            mx = max(mx, float(parts[2]))
        except ValueError:
            continue
        for n, v in zip(names, parts[5:9]):
            if v.lower() == "active":
                reasons.add(n)
    if not sm:
        return None
    return {"sm_mhz": float(np.median(sm)), "sm_max_mhz": mx, "reasons": sorted(reasons),
            "samples": len(sm)}


# ------------------------------------------------------------------ GPU arm
def run_ours(args, w, rank, world, local_rank):
    import torch
    import sparse_state_reuse_b200 as dt

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    stream = torch.cuda.Stream(device=dev)

    def up(bits):
        return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16)

    hq, hk, hv = (up(inputs.full(w, t)) for t in "qkv")
    Q, K, V = (x.to(dev) for x in (hq, hk, hv))
    group_off = w.group_off() if w.grouped else None
    pa = dt.PartitionedAttention(w.B, w.H, w.N, w.d, w.part_off(), w.frame_off(), w.frame_mask(),
                                 device=dev, state_bf16=args.state_bf16, group_off=group_off)
    if w.reuses:
        Kp = up(inputs.full(w, "k", prev=True)).to(dev)
        Vp = up(inputs.full(w, "v", prev=True)).to(dev)
        pa.plan_step(anchor=True)
        pa.partial(Q, Kp, Vp)          # anchor step: the cache of the previous denoising step
        torch.cuda.synchronize()
        del Kp, Vp
    out = torch.empty((w.B, w.H, w.N, w.d), dtype=torch.bfloat16, device=dev)
    out_lse = torch.empty((w.B, w.H, w.N), dtype=torch.float32, device=dev)
    kw = dict(band_k=w.band_k, budget=w.budget, anchor=w.anchor)

    # one step to learn the plan (the fresh count, and so the work, is the
    # same every step here); its output rows are kept for the error check
    with torch.cuda.stream(stream):
        pa.step(Q, K, V, out, out_lse, stream=stream, **kw)
    stream.synchronize()
    plan = pa.plan.cpu().numpy().reshape(w.P, pa.G)
    check_rows = sample_check_rows(w)
    first_out = {(b, h, i): out[b, h].index_select(0, torch.as_tensor(rows, device=dev)).float().cpu().numpy()
                 for (b, h, i, rows) in check_rows}
    A = plan != 0
    fresh = plan == 1
    flops = effective_flops(w, fresh_pairs_of_units(w, plan, pair_mask(w)))
    mbytes = merge_bytes(w, A, fresh, state_o_bytes=2 if args.state_bf16 else 4)
    # plan (anchor: the selection alone; reuse: the mean of the mass block sums
    # the previous merge left, then the selection), attention, merge
    launches_per_step = (1 if w.anchor else 2) + 1 + 1

    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    n_ev = args.steps
    e_part0, e_part1 = [ev() for _ in range(n_ev)], [ev() for _ in range(n_ev)]
    e_merge1 = [ev() for _ in range(n_ev)]
    e_plan0 = [ev() for _ in range(n_ev)]
    e_start, e_end = ev(), ev()

    def one_step(t=None):
        with torch.cuda.stream(stream):
            if t is not None:
                e_plan0[t].record(stream)
            pa.plan_step(w.band_k, w.budget, w.anchor, stream=stream)
            if t is not None:
                e_part0[t].record(stream)
            pa.partial(Q, K, V, stream=stream)
            if t is not None:
                e_part1[t].record(stream)
            pa.merge(out, out_lse, stream=stream)
            if t is not None:
                e_merge1[t].record(stream)

    for _ in range(args.warmup):
        one_step()
    stream.synchronize()
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    clk = ClockSampler(local_rank)
    clk.start()
    time.sleep(0.5)                           # nvidia-smi is sampling by now
    stream.synchronize()
    t_wall0 = time.time()
    e_start.record(stream)
    for t in range(args.steps):
        one_step(t)
    e_end.record(stream)
    stream.synchronize()
    t_wall1 = time.time()
    clocks = clk.stop(t_wall0, t_wall1)       # the samples of the timed region
    torch.cuda.synchronize()
    ms = e_start.elapsed_time(e_end)
    part_ms = float(np.mean([e_part0[t].elapsed_time(e_part1[t]) for t in range(n_ev)]))
    merge_ms = float(np.mean([e_part1[t].elapsed_time(e_merge1[t]) for t in range(n_ev)]))
    plan_us = 1e3 * float(np.mean([e_plan0[t].elapsed_time(e_part0[t]) for t in range(n_ev)]))
    ms = max_over_ranks(ms, dev, dist)
    if world > 1:
        dist.barrier()
    status = int(pa.status.item())
    if status != 0:
        raise RuntimeError(f"device status {status}")

    # End to end through the public API: every step copies its Q/K/V in from
    # pinned host memory and its output (bf16 O and fp32 lse) back out.  Two
    # sets of device buffers let step s+1's uploads overlap step s's compute
    # (copy-in stream -> compute stream -> copy-out stream, ordered by events).
    hq_p, hk_p, hv_p = (x.pin_memory() for x in (hq, hk, hv))
    h_out = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    h_lse = torch.empty(out_lse.shape, dtype=out_lse.dtype).pin_memory()
    bufs = [(Q, K, V, out, out_lse)]
    bufs.append((torch.empty_like(Q), torch.empty_like(K), torch.empty_like(V),
                 torch.empty_like(out), torch.empty_like(out_lse)))
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    done = [torch.cuda.Event() for _ in range(2)]
    loaded = [torch.cuda.Event() for _ in range(2)]
    drained = [torch.cuda.Event() for _ in range(2)]
    e2e_steps = max(3, min(args.steps, 20))

    def e2e_run(n):
        for i in range(n):
            bq, bk, bv, bo, bl = bufs[i % 2]
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(done[i % 2])
                bq.copy_(hq_p, non_blocking=True)
                bk.copy_(hk_p, non_blocking=True)
                bv.copy_(hv_p, non_blocking=True)
                loaded[i % 2].record(s_in)
            with torch.cuda.stream(stream):
                stream.wait_event(loaded[i % 2])
                if i >= 2:
                    stream.wait_event(drained[i % 2])
                pa.step(bq, bk, bv, bo, bl, stream=stream, **kw)
                done[i % 2].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done[i % 2])
                h_out.copy_(bo, non_blocking=True)
                h_lse.copy_(bl, non_blocking=True)
                drained[i % 2].record(s_out)

    e2e_run(2)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    a, b = ev(), ev()
    a.record(s_in)
    e2e_run(e2e_steps)
    s_in.wait_stream(s_out)
    b.record(s_in)
    torch.cuda.synchronize()
    e2e_ms = a.elapsed_time(b) / e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, dev, dist)
    h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv))
    d2h = h_out.numel() * h_out.element_size() + h_lse.numel() * h_lse.element_size()
    del bufs

    ms_step = ms / args.steps
    peaks, peak_src = load_peaks()
    compose = None
    if w.grouped:
        compose = measure_compose(w, pa, Q, K, V, dev, stream, args, peaks)
    tflops_part = flops / (part_ms * 1e-3) / 1e12
    peak_t = float(peaks.get("bf16_tflops"))          # burst figure: the conservative denominator
    peak_ts = float(peaks.get("bf16_tflops_sustained", peak_t))
    merge_gbs = mbytes / (merge_ms * 1e-3) / 1e9
    # recorded DRAM bytes are per state format (a bf16 cache moves half the bytes)
    tkey = w.name + (":bf16" if args.state_bf16 else "")
    traffic = recorded_traffic("attn_partial.cu", tkey)
    res = {
        "metric": "effective attention TFLOP/s (fresh blocks only) at 1 B200; tokens/s",
        "value": round(aggregate_tflops(world, flops, ms_step), 3),
        "unit": "TFLOP/s",
        "tokens_per_s": round(world * w.B * w.N / (ms_step * 1e-3), 1),
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16, shaped like the pages' workloads)",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "P": w.P,
                   "frames": w.F, "kv_groups": int(pa.G), "fresh_units": int(fresh.sum()),
                   "active_units": int(A.sum()),
                   "state_format": "bf16 O + fp32 lse" if args.state_bf16 else "fp32 O + fp32 lse",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "l2": "inputs larger than L2 (Q/K/V %.0f MB, states %.0f MB)" % (
                       h2d / 1e6, pa.state_O.numel() * pa.state_O.element_size() / 1e6)},
        "roofline": {"bound": "tensor", "kernel": "attn_partial", "achieved": round(tflops_part, 2),
                     "peak": peak_t, "unit": "TFLOP/s", "frac": round(tflops_part / peak_t, 4),
                     "peak_source": peak_src, "traffic": traffic,
                     "frac_of_sustained_peak": round(tflops_part / peak_ts, 4),
                     "kernel_ms": round(part_ms, 4),
                     "algorithmic_flops_per_launch": flops},
        "merge_roofline": {"bound": "hbm", "achieved": round(merge_gbs, 1),
                           "peak": float(peaks.get("hbm_gbs")), "unit": "GB/s",
                           "frac": round(merge_gbs / float(peaks.get("hbm_gbs")), 4),
                           "kernel_ms": round(merge_ms, 4),
                           "algorithmic_bytes_per_launch": mbytes,
                           "traffic": recorded_traffic("merge.cu", tkey)},
        "plan": {"us": round(plan_us, 2), "launches": 1 if w.anchor else 2,
                 "note": "anchor steps: the selection alone; reuse steps: the mass score from the "
                         "previous step's merge (its block sums reduced per unit) and the selection"},
        "e2e": {"value": round(aggregate_tflops(world, flops, e2e_ms), 3), "unit": "TFLOP/s",
                "ms_per_step": round(e2e_ms, 3), "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "plan_sha16": hashlib.sha256(plan.astype(np.int8).tobytes()).hexdigest()[:16],
    }
    res["_check"] = (plan, first_out, check_rows)
    if compose is not None:
        res["compose"] = compose
    if args.schedule > 0:
        del pa
        torch.cuda.empty_cache()
        res["schedule"] = measure_schedule(w, args, dev, stream, Q, K, V, flops)
    return res


def measure_schedule(w, args, dev, stream, Q, K0, V0, plain_flops):
    """A run of denoising steps with the error-growth planner (DiTango,
    1. Anchor-Guided Selection Planner): anchor steps every --anchor-every
    steps, predicted-error reuse between them.  K/V walk from step to step
    (K_s = bf16(K_0 + sigma * (e_1 + ... + e_s)), drawn on the device with
    torch's seeded generator, outside the timed region).  For every step it
    times the error planner's step, and the w planner's step on the same
    inputs, and reports each output's mean |difference| from unpartitioned
    all-fresh attention (computed by the library with one partition) -- the
    quality of reuse, reported and not gated."""
    import torch
    import sparse_state_reuse_b200 as dt
    go = w.group_off() if w.grouped else None
    mk = lambda **kw: dt.PartitionedAttention(w.B, w.H, w.N, w.d, w.part_off(), w.frame_off(),  # noqa: E731
                                              w.frame_mask(), device=dev, state_bf16=args.state_bf16,
                                              **kw)
    pa_e = mk(group_off=go)
    pa_w = mk(group_off=go)
    ep = dt.ErrorPlanner(pa_e, w.band_k, w.budget, args.anchor_every)
    # one partition: unpartitioned attention (unavailable under a frame mask,
    # which needs partitions inside frames)
    dense = None if w.F else dt.PartitionedAttention(w.B, w.H, w.N, w.d, [0, w.N], device=dev)
    outs = {k: torch.empty((w.B, w.H, w.N, w.d), dtype=torch.float32, device=dev) for k in "ewf"}
    gen = torch.Generator(device=dev)
    gen.manual_seed(w.drift_seed * 1000 + 17)
    K0f, V0f = K0.float(), V0.float()
    accK, accV = torch.zeros_like(K0f), torch.zeros_like(V0f)
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    rows = []
    for s in range(args.schedule + 1):
        if s > 0:
            accK.add_(torch.randn(accK.shape, generator=gen, device=dev))
            accV.add_(torch.randn(accV.shape, generator=gen, device=dev))
        K = (K0f + w.drift_sigma * accK).to(torch.bfloat16)
        V = (V0f + w.drift_sigma * accV).to(torch.bfloat16)
        stream.wait_stream(torch.cuda.current_stream())    # K/V were made on the default stream
        anchor = ep.is_anchor(s)
        e = [ev() for _ in range(4)]
        with torch.cuda.stream(stream):
            e[0].record(stream)
            ep.step(Q, K, V, outs["e"], stream=stream)
            e[1].record(stream)
            pa_w.step(Q, K, V, outs["w"], band_k=w.band_k, budget=w.budget, anchor=anchor,
                      stream=stream)
            e[2].record(stream)
            if dense is not None:
                dense.step(Q, K, V, outs["f"], anchor=True, stream=stream)
        stream.synchronize()
        fresh_e = pa_e.plan.cpu().numpy().reshape(w.P, pa_e.G) == 1
        fl = effective_flops(w, fresh_pairs_of_units(w, np.where(fresh_e, 1, 0), pair_mask(w)))
        row = {"step": s, "anchor": bool(anchor), "error_planner_ms": round(e[0].elapsed_time(e[1]), 4),
               "w_planner_ms": round(e[1].elapsed_time(e[2]), 4),
               "error_planner_tflops": round(fl / (e[0].elapsed_time(e[1]) * 1e-3) / 1e12, 2),
               "mean_local_drift": float(ep.delta.mean().item())}
        if dense is not None:
            row["error_planner_err"] = float((outs["e"] - outs["f"]).abs().mean().item())
            row["w_planner_err"] = float((outs["w"] - outs["f"]).abs().mean().item())
        rows.append(row)
    if int(pa_e.status.item()) != 0 or int(pa_w.status.item()) != 0:
        raise RuntimeError("device status in the schedule")
    reuse = [r for r in rows if not r["anchor"]]
    summary = {"steps": args.schedule + 1, "anchor_every": args.anchor_every,
               "sigma_per_step": w.drift_sigma,
               "mean_error_planner_ms_reuse_steps": round(float(np.mean([r["error_planner_ms"] for r in reuse])), 4),
               "mean_w_planner_ms_reuse_steps": round(float(np.mean([r["w_planner_ms"] for r in reuse])), 4),
               "per_step": rows}
    if dense is not None:
        summary["mean_abs_err_vs_fresh_error_planner"] = float(np.mean([r["error_planner_err"] for r in reuse]))
        summary["mean_abs_err_vs_fresh_w_planner"] = float(np.mean([r["w_planner_err"] for r in reuse]))
    return summary


def measure_compose(w, pa, Q, K, V, dev, stream, args, peaks):
    """Dynamic group composition: a cache of one state per (query partition,
    KV partition) merged into this workload's KV groups, no recomputation.
    The pair cache is built by an anchor step on the current K/V; the
    composition is timed alone (CUDA events, after warm-up).  Algorithmic
    bytes: every pair state read once, every group state written once."""
    import torch
    import sparse_state_reuse_b200 as dt
    fine = dt.PartitionedAttention(w.B, w.H, w.N, w.d, w.part_off(), w.frame_off(), w.frame_mask(),
                                   device=dev, state_bf16=args.state_bf16)
    with torch.cuda.stream(stream):
        fine.plan_step(anchor=True, stream=stream)
        fine.partial(Q, K, V, stream=stream)
    stream.synchronize()
    row = w.d * (2 if args.state_bf16 else 4) + 4
    nbytes = float((fine.n_slots + pa.n_slots) * w.BH * w.Lp * row)
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    reps = 5
    for _ in range(2):
        dt.ditango_cache_compose(fine.geom, pa.geom, fine.state_O, fine.state_lse, fine.valid,
                                 pa.state_O, pa.state_lse, pa.valid, args.state_bf16, stream)
    a, b = ev(), ev()
    a.record(stream)
    for _ in range(reps):
        dt.ditango_cache_compose(fine.geom, pa.geom, fine.state_O, fine.state_lse, fine.valid,
                                 pa.state_O, pa.state_lse, pa.valid, args.state_bf16, stream)
    b.record(stream)
    stream.synchronize()
    pa.mass_from_merge = False      # its cache was rewritten by the composition
    ms = a.elapsed_time(b) / reps
    gbs = nbytes / (ms * 1e-3) / 1e9
    out = {"from_slots": int(fine.n_slots), "to_slots": int(pa.n_slots),
           "cache_bytes_before": int(fine.state_O.numel() * fine.state_O.element_size()
                                     + fine.state_lse.numel() * 4),
           "cache_bytes_after": int(pa.state_O.numel() * pa.state_O.element_size()
                                    + pa.state_lse.numel() * 4),
           "ms": round(ms, 4), "bound": "hbm", "achieved": round(gbs, 1), "unit": "GB/s",
           "peak": float(peaks.get("hbm_gbs")), "frac": round(gbs / float(peaks.get("hbm_gbs")), 4),
           "algorithmic_bytes_per_launch": nbytes,
           "traffic": recorded_traffic("merge.cu", w.name + (":bf16" if args.state_bf16 else "") + ":compose")}
    del fine
    torch.cuda.empty_cache()
    return out


# ------------------------------------------------------------------ CPU oracle
def sample_check_rows(w, n_rows=32):
    """(b, h, partition, token rows) whose output the benchmark checks against
    the oracle: the first and last rows of the first and last partitions of
    the first and last (b, h)."""
    po = w.part_off()
    out = []
    for bh in sorted({0, w.BH - 1}):
        b, h = divmod(bh, w.H)
        for i in sorted({0, w.P - 1}):
            lo, hi = po[i], po[i + 1]
            rows = np.unique(np.concatenate([np.arange(lo, min(hi, lo + n_rows // 2)),
                                             np.arange(max(lo, hi - n_rows // 2), hi)]))
            out.append((b, h, i, rows))
    return out


def error_vs_oracle(w, check):
    """Max and mean |GPU - oracle| of the first step's sampled output rows:
    the oracle composes the same plan's states in fp64 (fresh states from the
    current K/V, reused ones from the previous step's)."""
    from oracle import groups as OG, step as OS
    plan, first_out, rows_list = check
    errs = []
    for (b, h, i, rows) in rows_list:
        q = inputs.slab_f64(w, "q", b, h)
        k = inputs.slab_f64(w, "k", b, h)
        v = inputs.slab_f64(w, "v", b, h)
        kp, vp = (inputs.slab_f64(w, "k", b, h, prev=True), inputs.slab_f64(w, "v", b, h, prev=True)) \
            if w.reuses else (k, v)
        if w.grouped:
            O, _ = OG.step_rows_units(q, k, v, kp, vp, plan, w.part_off(), w.group_off(), i, rows,
                                      w.frame_off(), w.frame_mask())
        else:
            O, _, _ = OS.step_rows(q, k, v, kp, vp, plan, w.part_off(), i, rows, w.frame_off(),
                                   w.frame_mask())
        errs.append(np.abs(first_out[(b, h, i)] - O).ravel())
    e = np.concatenate(errs)
    return {"max_abs": float(e.max()), "mean_abs": float(e.mean()),
            "rows": int(sum(r.size for (_, _, _, r) in rows_list)),
            "output": "bf16", "tolerance": {"max_abs": 2e-2, "mean_abs": 2e-3}}



def oracle_sample(w, rng_seed, rows_per_sample, deadline_s, n_slabs=4):
    """Time the fp64 oracle on seeded (b, h, partition, row-block) samples of
    the workload until deadline_s of CPU work; returns (flops, seconds, desc).
    The samples are drawn from n_slabs seeded (b, h) slabs, generated once
    (outside the timed region) and reused, so that the run's wall time stays
    close to the CPU time it measures."""
    from oracle import groups as OG, masks as OM, step as OS
    from oracle.plan import PLAN_FRESH
    A = OM.pair_mask(w.part_off(), w.frame_off(), w.frame_mask())
    plan = np.where(A, PLAN_FRESH, 0).astype(np.int8)  # the fresh work of the step
    if w.grouped:
        plan = np.where(OG.unit_mask(A, w.group_off()), PLAN_FRESH, 0).astype(np.int8)
    rng = np.random.default_rng(rng_seed)
    po = w.part_off()
    bh_set = sorted({int(x) for x in rng.integers(w.BH, size=n_slabs)})
    cache = {}
    flops, secs, n = 0.0, 0.0, 0
    while secs < deadline_s:
        bh = bh_set[int(rng.integers(len(bh_set)))]
        b, h = divmod(bh, w.H)
        i = int(rng.integers(w.P))
        lo, hi = po[i], po[i + 1]
        r0 = int(rng.integers(lo, max(lo + 1, hi - rows_per_sample)))
        rows = np.arange(r0, min(hi, r0 + rows_per_sample))
        if bh not in cache:
            cache[bh] = tuple(inputs.slab_f64(w, t, b, h) for t in "qkv")
        q, k, v = cache[bh]
        t0 = time.perf_counter()
        if w.grouped:
            OG.step_rows_units(q, k, v, k, v, plan, po, w.group_off(), i, rows, w.frame_off(),
                               w.frame_mask())
        else:
            OS.step_rows(q, k, v, k, v, plan, po, i, rows, w.frame_off(), w.frame_mask())
        secs += time.perf_counter() - t0
        keys = sum(po[j + 1] - po[j] for j in range(w.P) if A[i, j])
        flops += 4.0 * w.d * rows.size * keys
        n += 1
    return flops, secs, (f"{n} samples of {rows_per_sample} query rows x all active KV partitions, "
                         f"one (b,h) each, from {len(bh_set)} seeded (b,h) slabs")


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([x.get("num_threads", 1) for x in info] or [1])
    except Exception:
        return cpu_cores()


def run_reference(args, w, world=1):
    # a bounded sample per step: the whole run stays within a few minutes
    per_step = max(0.2, min(10.0, 90.0 / max(1, args.steps + args.warmup), args.cpu_baseline_seconds))
    for _ in range(args.warmup):
        oracle_sample(w, 7, 128, per_step / 4)
    tot_f, tot_s, desc = 0.0, 0.0, ""
    for s in range(args.steps):
        f, sec, desc = oracle_sample(w, 1000 + s, 128, per_step)
        tot_f += f
        tot_s += sec
    val = tot_f / tot_s / 1e12
    return {
        "impl": "reference",
        "metric": "effective attention TFLOP/s (fresh blocks only) at 1 B200; tokens/s",
        "value": round(val, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(1e3 * tot_s / args.steps, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1) bf16 values)",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d": w.d, "P": w.P},
        "cpu_baseline": {"value": round(val, 6), "unit": "TFLOP/s", "cores": blas_threads(),
                         "kind": "oracle", "sample": desc},
        "e2e": {"value": round(val, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=400)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(configs.BY_NAME))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-baseline-seconds", type=float, default=12.0)
    ap.add_argument("--state-bf16", action="store_true",
                    help="compressed attention-state cache: O stored as bf16")
    ap.add_argument("--schedule", type=int, default=0,
                    help="also run this many denoising steps with the error-growth planner "
                         "(K/V drifting step by step) and report them under 'schedule'")
    ap.add_argument("--anchor-every", type=int, default=5)
    ap.add_argument("--heads", type=int, default=0,
                    help="replace the workload's head count (a reduced case for profiling; "
                         "the line then names the reduced H and is not the workload's figure)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    w = configs.BY_NAME[args.workload]
    if args.heads > 0 and args.heads != w.H:
        w = configs.scaled(w, H=args.heads, name=f"{w.name}@H{args.heads}")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        # the oracle runs on rank 0's host cores only; the line names the
        # launch's GPU count so that it pairs with this arm's own line
        if rank == 0:
            print(json.dumps(run_reference(args, w, max(world, args.gpus))), flush=True)
        return

    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        res = run_ours(args, w, rank, world, local_rank)
        check = res.pop("_check")
        if rank == 0:
            if world == 1:
                res["error_vs_oracle"] = error_vs_oracle(w, check)
                f, s, desc = oracle_sample(w, 5, 128, args.cpu_baseline_seconds)
                res["cpu_baseline"] = {"value": round(f / s / 1e12, 6), "unit": "TFLOP/s",
                                       "cores": blas_threads(), "kind": "oracle", "sample": desc}
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
