"""Benchmark of the NABLA block-sparse attention path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload wan480p] [--impl ours|reference]

A step is one pass of the whole path over one batch of seeded synthetic
input: reorder Q, K, V -> block mask (pool, reduced attention, CDF threshold)
-> block-sparse attention -> inverse reorder.  Inputs are resident in HBM when
the timed region starts; L2 is flushed (a 2x-L2 buffer write) between steps,
outside the per-step CUDA events.  ``value`` is the effective throughput
4 * N^2 * d * heads * B * density / step time (TFLOP/s), summed over ranks.
With N > 1 GPUs (torchrun) every rank runs an independent replica of the
workload with its own seed (weak scaling; the path has no exchange step).

``e2e`` is the same metric through the public API with host buffers: each
step copies Q, K, V from pinned host memory, runs the path and copies the
output back to pinned host memory; the copies of neighbouring steps overlap
the compute (two device buffer sets, one copy stream per direction).  ``--impl reference`` times the fp64 CPU oracle instead, on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "block-sparse attn fwd ms & effective TFLOPS (% bf16 peak), Wan-480p shape"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Fine-selection timing: fraction of the 4-token KV blocks each query block
# keeps (the budget the AB-Attention article quotes for ideal top-k, 10.8 %).
FINE_FRAC = 0.108


def kernel_launches_per_step(w) -> int:
    """Our kernels in one step: the Q/K reorder with block pooling, V's
    reorder, the mask (reduced scores + selection, adaptive workloads), the
    plan (overlap + matching with 64-token blocks, one kernel with 128),
    attention, inverse reorder."""
    return 2 + (0 if w.iid else 2) + (2 if w.block == 64 else 1) + 1 + 1


# ------------------------------------------------------------------ helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# the kernel source each recorded traffic figure was taken from (the shared
# headers count for all of them)
TRAFFIC_SOURCES = {"attn": "attn_fwd.cu", "fine": "attn_fine.cu"}


def kernel_source_hash(kernel: str) -> str:
    csrc = os.path.join(ROOT, "block_sparse_attention_fractal_b200", "csrc")
    h = hashlib.sha256()
    for fn in sorted(os.listdir(csrc)):
        if fn == TRAFFIC_SOURCES[kernel] or fn.endswith((".cuh", ".h")):
            with open(os.path.join(csrc, fn), "rb") as f:
                h.update(fn.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` on `workload` from the committed ncu
    summary, if the kernel sources have not changed since it was taken (else None)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    ent = rec.get(kernel)
    if not ent or ent.get("source_hash") != kernel_source_hash(kernel) or ent.get("workload") != workload:
        return None
    return ent.get("bytes_per_launch")


class ClockSampler:
    """Samples SM clocks and throttle reasons while running: NVML every 5 ms
    (the counters nvidia-smi reports), else nvidia-smi -lms 50."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        self.t0 = None
        if self._start_nvml():
            self.t0 = time.monotonic()
            return self
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.first = threading.Event()
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
            self.first.wait(timeout=5.0)   # sampling is live before the timed region starts
        except (OSError, ValueError):
            self.proc = None
        self.t0 = time.monotonic()
        return self

    def _start_nvml(self) -> bool:
        """Polls NVML every 5 ms (the same counters nvidia-smi reads) in a
        thread; False when NVML is not available."""
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByIndex(self.index)
            smax = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
        except Exception:
            return False
        bits = {"hw_slowdown": pynvml.nvmlClocksEventReasonHwSlowdown,
                "hw_thermal_slowdown": pynvml.nvmlClocksEventReasonHwThermalSlowdown,
                "sw_thermal_slowdown": pynvml.nvmlClocksEventReasonSwThermalSlowdown,
                "sw_power_cap": pynvml.nvmlClocksEventReasonSwPowerCap}
        self.stop = threading.Event()

        def poll():
            while not self.stop.is_set():
                try:
                    sm = pynvml.nvmlDeviceGetClockInfo(h, pynvml.NVML_CLOCK_SM)
                    rs = pynvml.nvmlDeviceGetCurrentClocksEventReasons(h)
                except Exception:
                    break
                flags = ["Active" if rs & bits[k] else "Not Active" for k in
                         ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")]
                self.lines.append((time.monotonic(), ", ".join([str(self.index), str(sm), str(smax), "", hex(rs)]
                                                               + flags)))
                time.sleep(0.005)

        self.thread = threading.Thread(target=poll, daemon=True)
        self.thread.start()
        self.nvml = True
        return True

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.monotonic(), line.strip()))
            self.first.set()
        self.first.set()

    def __exit__(self, *exc):
        self.t1 = time.monotonic()
        if getattr(self, "nvml", False):
            self.stop.set()
            self.thread.join(timeout=2)
            return
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.thread.join(timeout=2)

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for t, line in self.lines:
            if not (self.t0 <= t <= self.t1):      # only samples taken during the timed region
                continue
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


def plan_work_ratio(bsa, shape, w, plan) -> float:
    """KV tiles the attention kernel runs (each tile 128 x 128) over the kept
    (query block, key block) pairs, in pair units: 1 for 128-token blocks;
    with 64-token blocks two query blocks share a tile and walk the union of
    their lists."""
    qb = 128 // w.block
    per_bh = -(-plan.nb // qb)
    off = bsa.plan_items_offset(shape)
    n = w.B * w.heads * per_bh
    items = plan.ws[off:off + 8 * n].view(torch.int32).view(n, 2).cpu().numpy()
    keep = lists_to_keep(plan.kv_count.cpu().numpy(), plan.kv_idx.cpu().numpy(), plan.nb).reshape(-1, plan.nb,
                                                                                                   plan.nb)
    bh = np.arange(n) // per_bh
    a = np.clip(items[:, 0], 0, plan.nb - 1)
    rows = keep[bh, a]
    if qb == 2:
        second = items[:, 1] >= 0
        rows = rows | (keep[bh, np.clip(items[:, 1], 0, plan.nb - 1)] & second[:, None])
    tiles = -(-rows.sum(axis=1) // qb)
    return float(tiles.sum() * qb * qb / keep.sum())


def lists_to_keep(kv_count: np.ndarray, kv_idx: np.ndarray, nb: int) -> np.ndarray:
    """KV lists -> bool block mask [B, heads, nb, nb] (entries past the count ignored)."""
    keep = np.zeros(kv_count.shape + (nb,), dtype=bool)
    flat_k, flat_c, flat_i = keep.reshape(-1, nb), kv_count.reshape(-1), kv_idx.reshape(-1, kv_idx.shape[-1])
    for r in range(flat_c.size):
        flat_k[r, flat_i[r, :flat_c[r]]] = True
    return keep


def max_over_ranks(value: float, dist, device) -> float:
    """The largest `value` over all ranks (the value itself without a process group)."""
    if dist is None:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(per_rank_ms, per_rank_flops):
    """Whole-job throughput: total effective FLOPs over the slowest rank's time."""
    t = max(per_rank_ms)
    return sum(per_rank_flops) / (t * 1e-3) / 1e12, t


# ------------------------------------------------------------------ oracle timing

def block_flops(w, count: int) -> float:
    """Effective FLOPs of one query block that keeps `count` KV blocks: its share
    of 4 * N^2 * d (the metric's formula, summed over all blocks of a call)."""
    return 4.0 * (w.N / w.nb) ** 2 * w.d * count


def oracle_head_path(pool, w, b, h, blocks, counts):
    """One sampled step of the fp64 oracle on the host cores: the whole path of
    head (b, h) -- reorder of its Q, K and V, its block mask (adaptive
    workloads), the attention of the query blocks `blocks` and the inverse
    reorder of its output -- each stage spread over the pool.  Returns (wall
    seconds, effective FLOPs of the attention done)."""
    t = pool.reorder([(b, h)])
    if not w.iid:
        _, _, tm = pool.masks([(b, h)])
        t += tm
    t += pool.attention(b, h, blocks)
    t += pool.inverse()
    return t, sum(block_flops(w, int(counts[b, h, I])) for I in blocks)


def oracle_block_seconds(pool, w):
    """Wall seconds of one query block's oracle attention (a probe: one block
    per worker, in parallel), with Q, K, V of head (0, 0) reordered first."""
    pool.reorder([(0, 0)])
    n = min(w.nb, pool.workers)
    blocks = list(range(0, w.nb, max(1, w.nb // n)))[:n]
    pool.attention(0, 0, blocks, chunk=1)          # first touch of the mapped inputs in every worker
    return pool.attention(0, 0, blocks, chunk=1)


def sample_blocks(w, workers, t_block, budget_s):
    """The query blocks of a head that one sampled step runs: all of them when
    the estimated wall time fits `budget_s`, else every k-th (first block 0,
    the ragged last block always included)."""
    fit = max(1, int(budget_s * workers / max(t_block, 1e-6)))
    k = max(1, -(-w.nb // fit))
    blocks = list(range(0, w.nb, k))
    if blocks[-1] != w.nb - 1:
        blocks.append(w.nb - 1)
    return blocks, k


def oracle_baseline(w, q, k, v, gpu_keep, budget_s=15.0):
    """The GPU arm's ``cpu_baseline``: the fp64 oracle on the host cores.

    First the oracle's block mask of every head (its ambiguous blocks counted,
    and compared with the GPU's mask ``gpu_keep``), then one sampled step:
    the whole path of head (0, 0) with as many query blocks as `budget_s` of
    wall time allows.  Returns (cpu_baseline dict, mask report dict)."""
    from oracle.parallel import OraclePool
    with OraclePool(w, q, k, v) as pool:
        report = {}
        if not w.iid:
            pool.reorder(pool.pairs(), (0, 1))
            keep, amb, _ = pool.masks(pool.pairs())
            report = {"ambiguous_blocks": int(amb.sum()),
                      "mask_mismatch_unambiguous": int(((keep != gpu_keep) & ~amb).sum()),
                      "oracle_density": float(keep.mean())}
        else:
            pool.set_keep(gpu_keep)
        counts = gpu_keep.sum(-1)
        t_block = oracle_block_seconds(pool, w)
        blocks, kstride = sample_blocks(w, pool.workers, t_block, budget_s)
        secs, flops = oracle_head_path(pool, w, 0, 0, blocks, counts)
        desc = (f"fp64 oracle, {pool.workers} host processes: the whole path of head 0 of {w.heads} (reorder Q, K, V; "
                f"{'block mask; ' if not w.iid else ''}attention of {len(blocks)} of {w.nb} query blocks"
                f"{'' if kstride == 1 else f' (every {kstride}th)'}; inverse reorder), {secs:.1f} s wall; "
                f"value = effective FLOPs of those blocks / that time")
        cpu = {"value": flops / secs / 1e12, "unit": "TFLOP/s", "cores": pool.workers, "kind": "oracle",
               "sample": desc}
    return cpu, report


# ------------------------------------------------------------------ main legs

def run_reference(args, w):
    """--impl reference: the fp64 oracle on the host cores.  Untimed set-up: the
    oracle's block mask of every head (so the workload and its density are the
    GPU arm's).  Each step then runs the whole path of one head (heads in
    turn), with as many of its query blocks as the step's time budget allows;
    value = effective FLOPs done / wall time of the timed steps."""
    import block_sparse_attention_fractal_b200.synth as synth
    from oracle.parallel import OraclePool
    q, k, v = synth.make_qkv(w)
    with OraclePool(w, q, k, v) as pool:
        if w.iid:
            dens_req = args.density if args.density is not None else 0.2
            cnt, idx = synth.random_block_lists(w.B, w.heads, w.nb, dens_req, w.seed)
            keep = np.zeros((w.B, w.heads, w.nb, w.nb), dtype=bool)
            c, ix = cnt.numpy(), idx.numpy()
            for b in range(w.B):
                for h in range(w.heads):
                    for I in range(w.nb):
                        keep[b, h, I, ix[b, h, I, :c[b, h, I]]] = True
            pool.set_keep(keep)
        else:
            pool.reorder(pool.pairs(), (0, 1))
            keep, _, _ = pool.masks(pool.pairs())
        dens = float(keep.mean())
        counts = keep.sum(-1)
        budget = max(1.5, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
        t_block = oracle_block_seconds(pool, w)
        blocks, kstride = sample_blocks(w, pool.workers, t_block, budget)
        times, flops = [], []
        for s in range(args.warmup + args.steps):
            b, h = (s // w.heads) % w.B, s % w.heads
            t, f = oracle_head_path(pool, w, b, h, blocks, counts)
            if s >= args.warmup:
                times.append(t)
                flops.append(f)
        workers = pool.workers
    value = sum(flops) / sum(times) / 1e12
    desc = (f"fp64 oracle, {workers} host processes; each step is the whole path of one head (heads in turn): "
            f"reorder Q, K, V; {'block mask; ' if not w.iid else ''}attention of {len(blocks)} of {w.nb} query blocks"
            f"{'' if kstride == 1 else f' (every {kstride}th)'}; inverse reorder")
    line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": statistics.mean(times) * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "density": dens, "sample": desc},
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": workers, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_ours(args, w, rank, world, dist):
    import block_sparse_attention_fractal_b200 as bsa
    import block_sparse_attention_fractal_b200.synth as synth

    dev = torch.device("cuda", torch.cuda.current_device())
    wr = dataclasses.replace(w, seed=w.seed + 1000 * rank) if rank else w
    q_h, k_h, v_h = synth.make_qkv(wr)
    q_pin, k_pin, v_pin = q_h.pin_memory(), k_h.pin_memory(), v_h.pin_memory()
    qd, kd, vd = q_pin.to(dev), k_pin.to(dev), v_pin.to(dev)
    out = torch.empty_like(qd)
    out_pin = torch.empty_like(q_pin).pin_memory()
    shape = bsa.make_shape(w.B, w.T, w.H, w.W, w.heads, w.d, w.block, w.patch)
    plan = bsa.NablaAttention(shape, device=dev)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush = torch.empty(max(2 * l2, 64 << 20), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    sweep_lists = None
    if w.iid:
        dens_req = args.density if args.density is not None else 0.2
        sweep_lists = synth.random_block_lists(w.B, w.heads, plan.nb, dens_req, w.seed)
        plan.kv_count.copy_(sweep_lists[0])
        plan.kv_idx.copy_(sweep_lists[1])

    ev = lambda: torch.cuda.Event(enable_timing=True)

    def step(times=None):
        # events on the launching stream: 0 | Q/K reorder + pooling | 1 | mask | 2 |
        # wait for V's reorder (side stream, overlapping the mask) | 3 | attention | 4 | inverse | 5
        e = [ev() for _ in range(6)] if times is not None else None
        if e: e[0].record(stream)
        plan.reorder_inputs(qd, kd, vd)
        if e: e[1].record(stream)
        if not w.iid:
            plan.mask_step(w.thr, w.sta)
        if e: e[2].record(stream)
        plan.join_side()
        if e: e[3].record(stream)
        plan.attention_step(baseline=args.baseline_kernel)
        if e: e[4].record(stream)
        bsa.inverse_reorder(shape, plan.o, out)
        if e:
            e[5].record(stream)
            times.append(e)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    if plan.status() != 0:
        raise RuntimeError("device status not OK after warm-up")
    dens = float(plan.kv_count.sum().item()) / (w.B * w.heads * plan.nb * plan.nb)
    work_ratio = plan_work_ratio(bsa, shape, w, plan)
    flops_step = 4.0 * w.N * w.N * w.d * w.heads * w.B * dens

    # ---- device-timed steps
    events = []
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clocks:
        for _ in range(args.steps):
            flush.fill_(1)
            step(events)
        torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    parts = np.array([[e[i].elapsed_time(e[i + 1]) for i in range(5)] for e in events])  # ms
    step_ms = float(parts.sum(axis=1).sum())   # total over K steps
    t_max = max_over_ranks(step_ms, dist, dev)
    total_flops = flops_step * args.steps * world
    value = total_flops / (t_max * 1e-3) / 1e12
    ms_per_step = t_max / args.steps
    br = parts.mean(axis=0)
    attn_ms = float(br[3])

    # ---- end to end through the public API with host buffers: every step
    # copies its Q, K, V from pinned host memory and its output back to pinned
    # host memory, all inside the timed region.  As a serving loop would run
    # it, the copies of neighbouring steps overlap the compute: two sets of
    # device input/output buffers, one copy stream per direction, events for
    # the dependencies (a set's inputs are overwritten only after the step that
    # read them, its output only after it has been copied out).
    h2d = 3 * q_pin.numel() * q_pin.element_size()
    d2h = out_pin.numel() * out_pin.element_size()
    h2d_stream, d2h_stream = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    sets = [(qd, kd, vd, out),
            (torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd), torch.empty_like(out))]
    outs_pin = [out_pin, torch.empty_like(out_pin).pin_memory()]
    in_ready = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    out_free = [torch.cuda.Event() for _ in range(2)]

    def run_path(qs, ks, vs, os_):
        if not w.iid:
            plan(qs, ks, vs, w.thr, w.sta, out=os_)
        else:
            plan.reorder_inputs(qs, ks, vs)
            plan.join_side()
            plan.attention_step()
            bsa.inverse_reorder(shape, plan.o, os_)

    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = ev(), ev()
    e0.record(stream)
    h2d_stream.wait_stream(stream)
    d2h_stream.wait_stream(stream)
    for i in range(args.steps):
        si = i % 2
        qs, ks, vs, os_ = sets[si]
        with torch.cuda.stream(h2d_stream):
            if i >= 2:
                h2d_stream.wait_event(comp_done[si])
            qs.copy_(q_pin, non_blocking=True)
            ks.copy_(k_pin, non_blocking=True)
            vs.copy_(v_pin, non_blocking=True)
            in_ready[si].record(h2d_stream)
        stream.wait_event(in_ready[si])
        if i >= 2:
            stream.wait_event(out_free[si])
        run_path(qs, ks, vs, os_)
        comp_done[si].record(stream)
        with torch.cuda.stream(d2h_stream):
            d2h_stream.wait_event(comp_done[si])
            outs_pin[si].copy_(os_, non_blocking=True)
            out_free[si].record(d2h_stream)
    stream.wait_stream(h2d_stream)
    stream.wait_stream(d2h_stream)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), dist, dev)
    if dist is not None:
        dist.barrier()
    e2e_value = total_flops / (e2e_ms * 1e-3) / 1e12
    if plan.status() != 0:
        raise RuntimeError("device status not OK after the timed steps")

    # ---- the backward pass (not part of `value`): K steps of bsa_attn_bwd on
    # the same lists, CUDA events on the launching stream, L2 flushed between
    bwd = None
    if args.bwd and not args.baseline_kernel:
        g = torch.Generator().manual_seed(99)
        dO = torch.randn(plan.o.shape, generator=g).to(torch.bfloat16).to(dev)
        if plan.lse is None:
            plan.lse = torch.empty(w.B, w.heads, plan.Npad, dtype=torch.float32, device=dev)
        plan.attention_step()
        dq, dk, dv = (torch.empty_like(plan.q) for _ in range(3))
        bws = torch.zeros((bsa.attn_bwd_workspace_bytes(shape) + 15) // 16 * 16, dtype=torch.uint8, device=dev)
        bsa.workspace_init(bws)
        run_bwd = lambda: bsa.attn_bwd(shape, plan.q, plan.k, plan.v, plan.o, dO, plan.lse, plan.kv_count,
                                       plan.kv_idx, 0.0, dq, dk, dv, bws)
        for _ in range(args.warmup):
            run_bwd()
        torch.cuda.synchronize()
        if bsa.check_device_status(bws) != 0:
            raise RuntimeError("device status not OK after the backward warm-up")
        bt = []
        for _ in range(args.steps):
            flush.fill_(1)
            b0, b1 = ev(), ev()
            b0.record(stream)
            run_bwd()
            b1.record(stream)
            bt.append((b0, b1))
        torch.cuda.synchronize()
        bwd_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in bt) / args.steps, dist, dev)
        bwd = {"ms": bwd_ms, "flops": 2.5 * flops_step}
    # ---- fine-grained KV selection (not part of `value`): K calls of
    # bsa_attn_fwd_fine on the same Q, K, V (kernel order) with lists of
    # 4-token blocks covering 10.8 % of the keys per 128-row query block,
    # weighted, L2 flushed between calls
    fine = None
    if args.fine and not args.baseline_kernel:
        fshape = bsa.make_shape(w.B, w.T, w.H, w.W, w.heads, w.d, 128, w.patch)
        fNpad = bsa.padded_len(fshape)
        nq, nkb = fNpad // 128, -(-w.N // 4)
        fq, fk, fv = (torch.zeros(w.B, w.heads, fNpad, w.d, dtype=torch.bfloat16, device=dev) for _ in range(3))
        for dst, src_t in ((fq, plan.q), (fk, plan.k), (fv, plan.v)):
            dst[:, :, :w.N].copy_(src_t[:, :, :w.N])
        off, idx, wt = synth.random_fine_lists(w.B, w.heads, nq, nkb, FINE_FRAC, w.seed + 1000 * rank)
        keys = torch.clamp(w.N - 4 * idx.to(torch.int64), max=4)
        rows_valid = torch.clamp(w.N - 128 * (torch.arange(off.numel() - 1) % nq), max=128)
        per_row = torch.zeros(off.numel() - 1, dtype=torch.int64)
        per_row.index_add_(0, torch.repeat_interleave(torch.arange(off.numel() - 1), off[1:] - off[:-1]), keys)
        fine_flops = 4.0 * w.d * float((per_row * rows_valid).sum())
        offd, idxd, wtd = off.to(dev), idx.to(dev), wt.to(dev)
        fo = torch.empty_like(fq)
        flse = torch.empty(w.B, w.heads, fNpad, dtype=torch.float32, device=dev)
        fws = torch.zeros(bsa.attn_fine_workspace_bytes(fshape), dtype=torch.uint8, device=dev)
        run_fine = lambda: bsa.attn_fwd_fine(fshape, fq, fk, fv, offd, idxd, wtd, 0.0, fo, flse, fws)
        for _ in range(args.warmup):
            run_fine()
        torch.cuda.synchronize()
        if bsa.check_device_status(fws) != 0:
            raise RuntimeError("device status not OK after the fine-selection warm-up")
        ft = []
        for _ in range(args.steps):
            flush.fill_(1)
            f0, f1 = ev(), ev()
            f0.record(stream)
            run_fine()
            f1.record(stream)
            ft.append((f0, f1))
        torch.cuda.synchronize()
        if bsa.check_device_status(fws) != 0:
            raise RuntimeError("device status not OK after the fine-selection calls")
        fine_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in ft) / args.steps, dist, dev)
        fine = {"ms": fine_ms, "flops": fine_flops, "entries_per_block": int(off[1] - off[0]), "nkb": nkb}
    if rank != 0:
        return
    peaks, src = load_peaks()
    peak_tf = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_tf_sus = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    attn_tf = flops_step / (attn_ms * 1e-3) / 1e12
    traffic = recorded_traffic("attn", w.name)
    # algorithmic bytes: the fused Q/K pass reads Q and K once, writes them
    # reordered (zero tail included) and writes the block means; the mask
    # kernel reads the means and writes the lists; V's reorder moves V
    tok_bytes = w.B * w.heads * w.N * w.d * 2
    pad_bytes = w.B * w.heads * (plan.Npad - w.N) * w.d * 2
    means_bytes = 2 * w.B * w.heads * plan.nb * w.d * 8
    kept = float(plan.kv_count.sum().item())
    qk_pool_bytes = 2 * (2 * tok_bytes + pad_bytes) + means_bytes
    # (the fp64 reduced scores the two mask kernels pass through the workspace are
    # an implementation choice, not algorithmic bytes: not counted)
    mask_kernel_bytes = means_bytes + 4 * (kept + w.B * w.heads * plan.nb)
    v_bytes = 2 * tok_bytes + pad_bytes
    qk_ms, mask_ms, vjoin_ms = float(br[0]), float(br[1]), float(br[2])
    gbs = lambda nbytes, ms: nbytes / (ms * 1e-3) / 1e9 if ms > 0 else None
    mask_gbs = gbs(qk_pool_bytes + mask_kernel_bytes, qk_ms + mask_ms)
    stage_gbs = gbs(qk_pool_bytes + mask_kernel_bytes + v_bytes, qk_ms + mask_ms + vjoin_ms)
    reduced_flops = 2.0 * w.B * w.heads * plan.nb * plan.nb * w.d
    cpu, mask_report = None, {}
    if args.cpu_baseline and world == 1:
        gpu_keep = lists_to_keep(plan.kv_count.cpu().numpy(), plan.kv_idx.cpu().numpy(), plan.nb)
        cpu, mask_report = oracle_baseline(w, q_h, k_h, v_h, gpu_keep, budget_s=args.cpu_budget)
    clk = clocks.summary()
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {
            "workload": w.name, "B": w.B, "T": w.T, "H": w.H, "W": w.W, "N": w.N, "Npad": plan.Npad,
            "heads": w.heads, "d": w.d, "block": w.block, "patch": w.patch, "thr": w.thr,
            "sta": list(w.sta) if w.sta else None, "density": dens, "parallelism": f"replicas x{world}",
            "attn_kernel": "mma.sync (legacy baseline)" if args.baseline_kernel else "tcgen05",
            "l2": "flushed between steps (write of a 2x L2 buffer, outside the step events)",
            "plan_work_ratio": work_ratio,
            "attn_ms": attn_ms, "attn_tflops": attn_tf, "attn_pct_bf16_peak": 100.0 * attn_tf / peak_tf,
            "breakdown_ms": {"reorder_pool_qk": qk_ms, "mask": mask_ms, "wait_reorder_v": vjoin_ms, "attn": attn_ms,
                             "inverse_reorder": float(br[4])},
            "reorder_pool_qk_gbs": gbs(qk_pool_bytes, qk_ms),
            "reorder_pool_qk_pct_hbm": 100.0 * gbs(qk_pool_bytes, qk_ms) / hbm,
            "mask_kernel_f64_tflops": reduced_flops / (mask_ms * 1e-3) / 1e12 if mask_ms > 0 else None,
            # mask construction: the fused Q/K reorder + pooling and the mask kernel
            "mask_gbs": mask_gbs,
            "mask_pct_hbm": 100.0 * mask_gbs / hbm if mask_gbs else None,
            # the whole stage before attention: the above with V's reorder overlapping the mask kernel
            "mask_stage_gbs": stage_gbs,
            "mask_stage_pct_hbm": 100.0 * stage_gbs / hbm if stage_gbs else None,
            "inverse_reorder_gbs": gbs(v_bytes - pad_bytes, float(br[4])),
            "mask_precision": "f64 pooled means, dots and masses",
            **mask_report,
            "step_ms_median": float(np.median(parts.sum(axis=1))),
            "step_ms_min": float(parts.sum(axis=1).min()),
            "attn_ms_median": float(np.median(parts[:, 3])),
            "attn_ms_min": float(parts[:, 3].min()),
        },
        "roofline": {"bound": "tensor", "achieved": attn_tf, "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": attn_tf / peak_tf, "traffic": traffic,
                     "kernel": "attention", "peak_source": f"{src} bf16 burst",
                     "frac_of_sustained": attn_tf / peak_tf_sus},
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": kernel_launches_per_step(w) * args.steps,
        "clocks": clk,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    if bwd is not None:
        bt_tf = bwd["flops"] / (bwd["ms"] * 1e-3) / 1e12
        line["config"]["bwd"] = {"ms": bwd["ms"], "tflops": bt_tf, "pct_bf16_peak": 100.0 * bt_tf / peak_tf,
                                 "flops": "2.5 x the forward's effective FLOPs (the five products of the "
                                          "definition per kept tile pair)",
                                 "launches_per_call": 3 + (4 if w.block == 64 else 2) + 2}
    if fine is not None:
        ft_tf = fine["flops"] / (fine["ms"] * 1e-3) / 1e12
        line["config"]["fine"] = {"ms": fine["ms"], "tflops": ft_tf, "pct_bf16_peak": 100.0 * ft_tf / peak_tf,
                                  "query_block": 128, "key_block": 4, "key_frac": FINE_FRAC,
                                  "entries_per_block": fine["entries_per_block"], "weighted": True,
                                  "flops": "4 d x valid query rows x valid selected keys",
                                  "launches_per_call": 1}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="wan480p")
    ap.add_argument("--density", type=float, default=None, help="density-sweep workload: kept fraction")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--no-bwd", dest="bwd", action="store_false", help="skip the backward-pass timing")
    ap.add_argument("--no-fine", dest="fine", action="store_false", help="skip the fine-selection timing")
    ap.add_argument("--baseline-kernel", action="store_true",
                    help="time the legacy mma.sync attention kernel instead of the tcgen05 one")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    from block_sparse_attention_fractal_b200 import synth
    w = synth.WORKLOADS[args.workload]
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))

    if args.impl == "reference":
        if rank == 0:
            run_reference(args, w)
        return 0

    dist = None
    if world > 1:
        import torch.distributed as dist_mod
        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        import datetime
        dist_mod.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", local))
        dist = dist_mod
    else:
        torch.cuda.set_device(0)
    try:
        run_ours(args, w, rank, world, dist)
    finally:
        if dist is not None:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
