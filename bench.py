#!/usr/bin/env python
"""Benchmark of the dynamic block-sparse attention hot path on B200.

One step = one pass of the whole hot path over one batch:
  kv_append (the batch's new tokens) -> index_score -> topk_blocks -> attention.
Default workload: 1M-context decode (8 sequences x 1,048,576 tokens, Top-K 32
blocks of 64 tokens, 64 query / 8 KV heads, 16 indexer heads).  The step is
captured in a CUDA graph.  The timed steps run back to back and rotate through
several independent batches (their own sequences, KV pools and queries) whose
step traffic together exceeds the L2 by half, so no step finds its data in L2;
the K steps are timed with one pair of CUDA events on the launching stream.
Workloads too small for that are timed one step at a time after a cold-L2
flush (512 MiB written, then 256 MiB read so no dirty lines remain), which is
also reported for the first batch as the isolated step time.  Decode lines
also carry an `overlapped` record: the same batches all in flight at once,
each on a stream of its own (a serving schedule; not part of `value`).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Under torchrun every rank runs its own batch (weak scaling, no collective on
the data path); rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "sparse-attn decode tokens/s @1M ctx; achieved HBM GB/s vs ~8 TB/s peak"
UNIT = "tokens/s"
L2_FLUSH_BYTES = 512 << 20
L2_BYTES = 126 << 20            # B200 L2
ROTATE_L2_MULTIPLE = 1.5        # rotated batches' step traffic, in L2 capacities
MAX_ROTATE = 4
# DRAM bytes (read + write) per launch of the roofline kernel, from an ncu
# capture of the current kernel ((workload, path) -> bytes); absent = not
# captured since the kernel last changed.  The decode attention figure comes
# from the 128K-context case, which processes the same units (8 queries x 8 KV
# heads x 32 selected blocks) and so the same selected bytes per launch.
TRAFFIC = {("decode_1m", "attention"): 68_514_048}


# ----------------------------------------------------------------------------- distributed plumbing
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world: int, backend: str):
    if world > 1 and not torch.distributed.is_initialized():
        import datetime
        torch.distributed.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))


def _reduce_device(device):
    # gloo reduces host tensors, nccl device tensors
    if torch.distributed.get_backend() == "gloo":
        return torch.device("cpu")
    return device


def max_over_ranks(x: float, world: int, device) -> float:
    """Max of a per-rank float over all ranks (identity when world == 1)."""
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=_reduce_device(device))
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=_reduce_device(device))
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def weak_scaling_throughput(units_per_step_per_rank: int, steps: int, world: int, seconds_max: float) -> float:
    """Whole-job throughput: every rank processes its own batch each step, and
    the job takes as long as its slowest rank."""
    return units_per_step_per_rank * steps * world / seconds_max


def barrier(world: int):
    if world > 1:
        torch.distributed.barrier()


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
        0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
        0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting",
    }

    def __init__(self, device_index: int, period_s: float = 0.0002):
        self.samples, self.reasons, self.stamps = [], set(), []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thr = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None
        self.period = period_s

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                self.stamps.append(time.monotonic())
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._nv is not None:
            # the thread that issues the timed graph replays holds the GIL
            # between them; a short switch interval lets the sampler run every
            # ~0.1 ms instead of every 5 ms (the work is queued on the GPU
            # well ahead of the host, so the timed region does not notice)
            self._switch = sys.getswitchinterval()
            sys.setswitchinterval(1e-4)
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thr is not None:
            self._thr.join()
            sys.setswitchinterval(self._switch)

    def count_between(self, t0: float, t1: float) -> int:
        return sum(1 for t in list(self.stamps) if t0 <= t <= t1)

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ----------------------------------------------------------------------------- workload accounting
def algorithmic_bytes(wl) -> dict:
    """Bytes the method must move per step (decode roofline): every visible
    block's coarse key plus the K/V page slices of the selected blocks."""
    spec = wl.spec
    idx = 0
    kv = 0
    flops = 0
    for s in range(spec.num_seqs):
        for i in range(spec.n_new[s]):
            p = spec.seq_lens[s] - spec.n_new[s] + i
            n_vis = p // spec.block_size + 1
            idx += n_vis * spec.idx_dim
            k = min(spec.k_per_seq[s], n_vis)
            kv += k * spec.block_size * spec.num_kv_heads * spec.head_dim * 2 * 2
            # QK^T and PV: 2 x 2 x (query heads) x 64 tokens x 128 per selected block
            flops += k * 4 * spec.num_q_heads * spec.block_size * spec.head_dim
    return {"coarse_keys": idx, "kv": kv, "total": idx + kv, "flops": flops}


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def _bf16_sustained():
    """dense bf16 TFLOP/s for a kernel timed inside a long run"""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops_sustained"]), "measured sustained"
    except Exception:
        return 1400.0, "fallback sustained"


# ----------------------------------------------------------------------------- one batch and its graphs
class StepCase:
    """One independent batch of a workload (its own sequences, KV pool, queries
    and output buffers) with its step captured in CUDA graphs: the whole step,
    the attention launch alone, and each phase alone (events only at the
    graphs' ends, so the kernels' programmatic dependent launches overlap)."""

    def __init__(self, spec, seed, device, stream, err, path):
        import dynamic_block_sparse_dsa_b200 as dsa
        from dynamic_block_sparse_dsa_b200 import workloads as wk
        self.dsa, self.spec, self.stream, self.err, self.device = dsa, spec, stream, err, device
        self.decode = all(n == 1 for n in spec.n_new)
        self.path = path
        self.fused = path in ("fused_select", "fused_decode")
        self.fused_decode = path == "fused_decode"
        self.wl = wl = wk.make_workload(spec, seed=seed, device=device)
        self.cache = dsa.PagedKVCache(wl.k_pool, wl.v_pool, wl.kc_pool)
        self.seqs = dsa.SeqBatch(wl.block_table, wl.seq_lens)
        self.queries = dsa.QueryBatch(wl.cu_q, wl.q_pos)
        with torch.cuda.stream(stream):
            self.bufs = dsa.step(self.cache, self.seqs, self.queries, k_new=wl.k_new, v_new=wl.v_new,
                                 kc_new=wl.kc_new, q=wl.q, q_idx=wl.q_idx, w=wl.w, k_per_seq=wl.k_per_seq,
                                 k_max=spec.k_max, decode=self.decode, fused_select=self.fused,
                                 overlap_append=self.fused and self.decode, fused_decode=self.fused_decode,
                                 dev_err=err)
        torch.cuda.synchronize(device)
        if int(err.item()) != 0:
            raise RuntimeError(f"device error bits {int(err.item())} in the first step of {spec.name}")
        self.graph, self.ev = self.capture(self.run_step)
        self.graph_attn, self.ev_attn = self.capture(self.attn)

    def capture(self, fn):
        """A graph of ``fn`` between two events it records; the graph keeps
        the events alive (they must outlive every replay)."""
        ev = (torch.cuda.Event(enable_timing=True, external=True), torch.cuda.Event(enable_timing=True, external=True))
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream):
            ev[0].record()
            fn()
            ev[1].record()
        torch.cuda.synchronize(self.device)
        g.dsa_events = ev
        return g, ev

    def run_step(self):
        if self.fused_decode:
            self.whole_step()
        else:
            self.front()
            self.attn()

    def append(self):
        wl = self.wl
        self.dsa.kv_append(self.cache, self.seqs, self.queries.cu_q, wl.k_new, wl.v_new, wl.kc_new, dev_err=self.err)

    def select(self):
        wl, b, spec = self.wl, self.bufs, self.spec
        if self.fused and self.decode:   # a decode batch: the append overlaps the selection in one launch
            self.dsa.select_blocks_append(self.cache, self.seqs, self.queries, self.queries.cu_q, wl.k_new,
                                          wl.v_new, wl.kc_new, wl.q_idx, wl.w, wl.k_per_seq, spec.k_max, 16,
                                          sel=b["sel"], cnt=b["cnt"], workspace=b["select_ws"], dev_err=self.err)
        else:
            self.dsa.select_blocks(self.cache, self.seqs, self.queries, wl.q_idx, wl.w, wl.k_per_seq, spec.k_max,
                                   16, sel=b["sel"], cnt=b["cnt"], workspace=b["select_ws"], dev_err=self.err)

    def score(self):
        wl, b = self.wl, self.bufs
        self.dsa.index_score(self.cache, self.seqs, self.queries, wl.q_idx, wl.w, 16, scores=b["scores"],
                             dev_err=self.err)

    def topk(self):
        wl, b = self.wl, self.bufs
        self.dsa.topk_blocks(self.seqs, self.queries, b["scores"], wl.k_per_seq, self.spec.k_max, sel=b["sel"],
                             cnt=b["cnt"], dev_err=self.err, block_size=self.spec.block_size)

    def front(self):
        if self.fused and self.decode:
            self.select()
            return
        self.append()
        if self.fused:
            self.select()
        else:
            self.score()
            self.topk()

    def attn(self):
        wl, b = self.wl, self.bufs
        if self.decode:
            self.dsa.sparse_attn_decode(self.cache, self.seqs, self.queries, wl.q, b["sel"], b["cnt"], out=b["out"],
                                        lse=b["lse"], workspace=b["workspace"], dev_err=self.err)
        else:
            self.dsa.sparse_attn_prefill(self.cache, self.seqs, self.queries, wl.q, b["sel"], b["cnt"],
                                         out=b["out"], lse=b["lse"], dev_err=self.err)

    def whole_step(self):
        wl, b = self.wl, self.bufs
        self.dsa.decode_fused(self.cache, self.seqs, self.queries, self.queries.cu_q, wl.k_new, wl.v_new,
                              wl.kc_new, wl.q_idx, wl.w, wl.k_per_seq, self.spec.k_max, wl.q, sel=b["sel"],
                              cnt=b["cnt"], out=b["out"], lse=b["lse"], workspace=b["fused_ws"], dev_err=self.err)

    def phases(self):
        """(name, call) of the step's separate launches, in order."""
        if self.fused_decode:
            return [("decode_fused", self.whole_step)]
        if self.fused and self.decode:
            return [("select_append", self.select), ("attention", self.attn)]
        if self.fused:
            return [("append", self.append), ("select", self.select), ("attention", self.attn)]
        return [("append", self.append), ("index_score", self.score), ("topk", self.topk), ("attention", self.attn)]


class Timer:
    """Cold-L2 flushes and CUDA-event timing of graph replays on one stream."""

    def __init__(self, device, stream):
        self.device, self.stream = device, stream
        self.flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
        self.flush_rd = torch.ones(L2_FLUSH_BYTES // 2 // 4, dtype=torch.int32, device=device)

    def cold_l2(self):
        # write a buffer larger than the L2, then read another one so that the
        # timed work starts on a cold L2 holding no dirty lines
        self.flush.fill_(1)
        self.flush_rd.sum(dtype=torch.int32)

    def isolated(self, graph, ev, n):
        """n replays of ``graph``, each after a cold-L2 flush; ms per replay from
        the graph's own events."""
        ms = []
        for _ in range(n):
            with torch.cuda.stream(self.stream):
                self.cold_l2()
                graph.replay()
            self.stream.synchronize()
            ms.append(ev[0].elapsed_time(ev[1]))
        return ms

    def rotated(self, whole, singles, n):
        """n replays back to back: ``whole`` holds one of each batch's graphs in
        turn, ``singles`` the per-batch graphs for the remainder; seconds."""
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        k = len(singles)
        with torch.cuda.stream(self.stream):
            e0.record()
            for _ in range(n // k):
                whole.replay()
            for i in range(n % k):
                singles[i].replay()
            e1.record()
        self.stream.synchronize()
        return e0.elapsed_time(e1) / 1e3


def rotation_graph(cases, fn_of, stream, device):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for c in cases:
            fn_of(c)()
    torch.cuda.synchronize(device)
    return g


OVERLAP_PASSES = 8   # steps of each batch in one graph of the overlapped schedule


def overlap_graph(cases, stream, device, passes=OVERLAP_PASSES):
    """One CUDA graph in which every batch runs ``passes`` steps in order on a
    stream of its own, forked from and joined back into ``stream``: the batches
    are independent, so one batch's latency-bound selection runs while another
    batch's attention streams its pages (the steps of one batch stay in order;
    the results are those of the same steps one after another)."""
    g = torch.cuda.CUDAGraph()
    sides = [torch.cuda.Stream(device) for _ in cases]
    with torch.cuda.graph(g, stream=stream):
        for s in sides:
            s.wait_stream(stream)
        for _ in range(passes):
            for c, s in zip(cases, sides):
                with torch.cuda.stream(s):
                    c.run_step()
        for s in sides:
            stream.wait_stream(s)
    torch.cuda.synchronize(device)
    g.dsa_streams = sides   # the captured streams outlive the graph's replays
    return g


def time_overlapped(cases, stream, device, steps, passes=OVERLAP_PASSES):
    """Seconds per step of ``overlap_graph`` replayed back to back (at least
    ``steps`` steps, after one untimed replay)."""
    g = overlap_graph(cases, stream, device, passes)
    per = passes * len(cases)
    n = max(1, math.ceil(steps / per))
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        g.replay()
        e0.record()
        for _ in range(n):
            g.replay()
        e1.record()
    stream.synchronize()
    del g
    return e0.elapsed_time(e1) / 1e3 / (n * per), n * per


def overlapped_record(cases, spec, ab, stream, device, steps, peak):
    s, n = time_overlapped(cases, stream, device, steps)
    gbs = ab["total"] / s / 1e9
    return {"batches_in_flight": len(cases), "ms_per_step": round(s * 1e3, 5),
            "tokens_per_s": round(spec.total_q / s, 1), "step_gbs": round(gbs, 1),
            "step_frac_of_measured": round(gbs / peak, 4), "steps_timed": n,
            "how": (f"the {len(cases)} independent batches each on a stream of their own, {OVERLAP_PASSES} steps of "
                    f"each in one CUDA graph replayed back to back, so one batch's selection overlaps another's "
                    f"attention; a serving schedule with {len(cases)} batches in flight, not the headline's "
                    f"one-step-after-another timing")}


def pick_path(spec, path):
    decode = all(n == 1 for n in spec.n_new)
    if path == "auto":   # decode batches: the fused select chain; otherwise the separate calls
        path = "fused_select" if decode and spec.k_max <= 64 else "score_topk"
    if path == "fused_decode" and not decode:
        raise SystemExit("--path fused_decode needs a decode workload")
    return path, decode


def indexer_ops(spec):
    """int8 ops of the block scoring: every (query, visible block) pair x heads x 64 x 2."""
    pairs = 0
    for s in range(spec.num_seqs):
        for i in range(spec.n_new[s]):
            p = spec.seq_lens[s] - spec.n_new[s] + i
            pairs += p // spec.block_size + 1
    return pairs * spec.num_idx_heads * spec.idx_dim * 2


def _int8_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return 2.0 * float(json.load(f)["bf16_tflops"]), "measured bf16 burst x 2 (nominal int8/bf16 ratio)"
    except Exception:
        return 2.0 * 1590.0, "fallback bf16 x 2"


# ----------------------------------------------------------------------------- our arm: the headline
def run_ours(args, world, rank, device):
    import dynamic_block_sparse_dsa_b200 as dsa
    from dynamic_block_sparse_dsa_b200 import workloads as wk

    spec = wk.NAMED[args.workload]()
    path, decode = pick_path(spec, args.path)
    fused = path in ("fused_select", "fused_decode")
    fused_decode = path == "fused_decode"
    err = torch.zeros(1, dtype=torch.int32, device=device)
    stream = torch.cuda.Stream(device)
    tm = Timer(device, stream)

    # independent batches whose step traffic together exceeds the L2: the timed
    # steps rotate through them back to back, so no step finds its data in L2
    # (workloads too small for that, more than MAX_ROTATE batches, are timed one
    # step at a time after a cold-L2 flush instead)
    cases = [StepCase(spec, args.seed + rank, device, stream, err, path)]
    ab = algorithmic_bytes(cases[0].wl)
    need = max(args.rotate, math.ceil(ROTATE_L2_MULTIPLE * L2_BYTES / ab["total"]))
    rotate = need <= MAX_ROTATE and not args.no_rotate
    while rotate and len(cases) < need:
        cases.append(StepCase(spec, args.seed + rank + 7919 * len(cases), device, stream, err, path))
    case0 = cases[0]
    wl = case0.wl
    n_case = len(cases)

    # one graph holding a step of every batch in turn (as consecutive layers'
    # steps would sit in one graph), and one holding their attention launches
    if rotate:
        rot_graph = rotation_graph(cases, lambda c: c.run_step, stream, device)
        rot_attn = rotation_graph(cases, lambda c: c.attn, stream, device)
    steps_g = [c.graph for c in cases]
    attn_g = [c.graph_attn for c in cases]

    for _ in range(args.warmup):
        if rotate:
            tm.rotated(rot_graph, steps_g, n_case)
            tm.rotated(rot_attn, attn_g, n_case)
        else:
            tm.isolated(case0.graph, case0.ev, 1)
    barrier(world)
    torch.cuda.synchronize(device)
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        time.sleep(0.002)   # the sampler's first samples, before the timed region
        t_begin = time.monotonic()
        if rotate:
            total_s = tm.rotated(rot_graph, steps_g, args.steps)
        else:
            total_s = sum(tm.isolated(case0.graph, case0.ev, args.steps)) / 1e3
        torch.cuda.synchronize(device)
        n_timed_samples = clk.count_between(t_begin, time.monotonic())
        # the same steps again, untimed, so that the clock record has more than
        # a handful of samples of the load the timed region ran under
        if rotate:
            tm.rotated(rot_graph, steps_g, max(args.steps, 2000))
    torch.cuda.synchronize(device)
    barrier(world)
    n_attn = max(3 * n_case, min(args.steps, 300))
    iso_step_ms = tm.isolated(case0.graph, case0.ev, max(5, min(args.steps, 50)))
    iso_attn_ms = tm.isolated(case0.graph_attn, case0.ev_attn, max(5, min(args.steps, 50)))
    attn_mean_s = tm.rotated(rot_attn, attn_g, n_attn) / n_attn if rotate else statistics.mean(iso_attn_ms) / 1e3
    if int(err.item()) != 0:
        raise RuntimeError(f"device error bits {int(err.item())} during timing")

    total_s_max = max_over_ranks(total_s, world, device)
    tokens_per_step = spec.total_q
    value = weak_scaling_throughput(tokens_per_step, args.steps, world, total_s_max)
    step_mean_s = total_s / args.steps
    peak, peak_kind = _peaks()
    if fused_decode:
        # the step is one kernel: its bytes are the coarse keys plus the selected K/V
        achieved = ab["total"] / step_mean_s / 1e9
        roofline = {"bound": "hbm", "kernel": "sparse_attn_kernel<1,true> (single-launch decode step)",
                    "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4),
                    "peak_source": peak_kind, "bytes_per_launch": ab["total"],
                    "traffic": TRAFFIC.get((spec.name, "fused_decode"))}
    elif not decode:
        # prefill attention: a contraction; each query's selected page slices
        # are its own (re-read from L2 across queries), so it is reported in
        # bf16 TFLOP/s against the sustained dense peak
        tpk, tsrc = _bf16_sustained()
        achieved = ab["flops"] / attn_mean_s / 1e12
        roofline = {"bound": "tensor", "kernel": "sparse_attn_kernel (prefill entry)", "achieved": round(achieved, 2),
                    "peak": tpk, "unit": "TFLOP/s", "frac": round(achieved / tpk, 4), "peak_source": tsrc,
                    "flops_per_launch": ab["flops"], "traffic": None,
                    "timing": (f"mean over {n_attn} launches back to back ({n_case} per graph)"
                               if rotate else "mean of single launches after a cold-L2 flush"),
                    "selected_kv_bytes_per_launch": ab["kv"]}
    else:
        achieved = ab["kv"] / attn_mean_s / 1e9
        iso = statistics.median(iso_attn_ms) * 1e-3
        roofline = {"bound": "hbm", "kernel": "sparse_attn_kernel (decode entry)",
                    "achieved": round(achieved, 1),
                    "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4), "peak_source": peak_kind,
                    "bytes_per_launch": ab["kv"], "traffic": TRAFFIC.get((spec.name, "attention")),
                    "timing": (f"mean over {n_attn} launches back to back ({n_case} per graph, one per "
                               f"independent batch, PDL between them)"
                               if rotate else "mean of single launches after a cold-L2 flush"),
                    "isolated": {"us": round(iso * 1e6, 2), "achieved": round(ab["kv"] / iso / 1e9, 1),
                                 "frac": round(ab["kv"] / iso / 1e9 / peak, 4),
                                 "how": "one launch after a cold-L2 flush, in-graph events (median)"}}
    step_gbs = ab["total"] / step_mean_s / 1e9
    step_roof = {"bytes_per_step": ab["total"], "achieved_gbs": round(step_gbs, 1),
                 "frac_of_measured": round(step_gbs / peak, 4), "frac_of_8tbs": round(step_gbs / 8000.0, 4)}

    # independent batches in flight at once (decode only; not part of `value`)
    overlapped = (overlapped_record(cases, spec, ab, stream, device, args.steps, peak)
                  if rotate and decode and not fused_decode and world == 1 else None)
    if int(err.item()) != 0:
        raise RuntimeError(f"device error bits {int(err.item())} during the overlapped steps")

    e2e = end_to_end(cases, spec, path, decode, rotate, tm, world, device, stream, err, args.steps)

    res = {
        "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(total_s_max / args.steps * 1e3, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16+int8",
        "data": "synthetic (seeded; N(0,1)/sqrt(128) bf16 q/k/v, uniform int8 indexer, planted blocks)",
        "config": {"workload": spec.name, "batch_per_gpu": spec.num_seqs, "context": max(spec.seq_lens),
                   "top_k": spec.k_max, "block_size": spec.block_size,
                   "heads_q_kv_idx": [spec.num_q_heads, spec.num_kv_heads, spec.num_idx_heads],
                   "global_batch": spec.num_seqs * world, "parallelism": f"dp{world} (independent sequences)",
                   "l2": (f"inputs larger than L2: steps back to back over {n_case} independent batches "
                          f"({n_case * ab['total'] / 2**20:.0f} MiB of step traffic, L2 126 MiB)" if rotate else
                          "cold before every timed step: 512 MiB written, then 256 MiB read (no dirty lines)"),
                   "graph": (f"one CUDA graph per {n_case} steps, one step of each batch in turn"
                             if rotate else "one CUDA graph per step") + ("" if fused_decode else " (PDL between kernels)"),
                   "path": {"fused_decode": "single launch: append + fused score/Top-K + attention",
                            "fused_select": "fused score+Top-K with the token append overlapping it, attention",
                            "score_topk": "kv_append, index_score, topk_blocks, attention"}[path]},
        "roofline": roofline,
        "step_roofline": step_roof,
        "overlapped": overlapped,
        "attn_ms_mean": round(attn_mean_s * 1e3, 5),
        "step_isolated_ms_median": round(statistics.median(iso_step_ms), 5),
        "e2e": e2e,
        "gpu_launches": len(case0.phases()) * args.steps,
        "clocks": dict(clk.summary(), samples_in_timed_region=n_timed_samples,
                       how="NVML every 0.2 ms during the timed steps and the same steps repeated untimed"),
    }
    if rotate:
        del rot_graph, rot_attn
    return res, cases


def end_to_end(cases, spec, path, decode, rotate, tm, world, device, stream, err, steps):
    """The same metric through the public API with host buffers: every step
    copies its inputs H2D from pinned memory, runs dsa.step (its C-ABI calls,
    launched from Python) and copies out/lse back D2H; the timed region holds
    all of it.  Each batch's inputs are staged in one pinned buffer (one H2D
    copy) and the library writes out and lse into one device buffer (one D2H
    copy), each tensor a 256-byte-aligned view.  The steps run back to back
    over the same independent batches as the device-side timing (or one step
    at a time after an L2 flush for small workloads).  The same steps
    replayed from CUDA graphs (how a serving loop would launch them) are
    timed as well."""
    import dynamic_block_sparse_dsa_b200 as dsa
    fused = path in ("fused_select", "fused_decode")
    fused_decode = path == "fused_decode"
    n_case = len(cases)

    def pack_layout(ts):
        offs, off = {}, 0
        for k, t in ts.items():
            off = (off + 255) // 256 * 256
            offs[k] = off
            off += t.numel() * t.element_size()
        return offs, off

    def view(buf, off, t):
        return buf[off:off + t.numel() * t.element_size()].view(t.dtype).view(t.shape)

    class Staged:
        """One batch's pinned input buffer, device input and output buffers."""

        def __init__(self, c):
            w = c.wl
            src = {k: getattr(w, k) for k in ("k_new", "v_new", "kc_new", "q", "q_idx", "w")}
            in_offs, self.in_bytes = pack_layout(src)
            self.host_in = torch.empty(self.in_bytes, dtype=torch.uint8).pin_memory()
            self.dev_in_buf = torch.empty(self.in_bytes, dtype=torch.uint8, device=device)
            for k, t in src.items():
                view(self.host_in, in_offs[k], t).copy_(t.cpu())
            self.dev_in = {k: view(self.dev_in_buf, in_offs[k], t) for k, t in src.items()}
            out_offs, self.out_bytes = pack_layout({"out": c.bufs["out"], "lse": c.bufs["lse"]})
            self.dev_out_buf = torch.empty(self.out_bytes, dtype=torch.uint8, device=device)
            self.host_out = torch.empty(self.out_bytes, dtype=torch.uint8).pin_memory()
            self.bufs = dict(c.bufs)
            self.bufs["out"] = view(self.dev_out_buf, out_offs["out"], c.bufs["out"])
            self.bufs["lse"] = view(self.dev_out_buf, out_offs["lse"], c.bufs["lse"])
            self.c = c
            d = self.dev_in
            kw = dict(bufs=self.bufs, k_new=d["k_new"], v_new=d["v_new"], kc_new=d["kc_new"], q=d["q"],
                      q_idx=d["q_idx"], w=d["w"], k_per_seq=c.wl.k_per_seq, k_max=spec.k_max, decode=decode,
                      fused_select=fused, overlap_append=fused and decode, fused_decode=fused_decode, dev_err=err)
            # the step's calls with their arguments marshalled once (the public
            # PreparedStep: a serving loop's way of issuing the same step
            # again), once with the library's host staging of this batch's
            # inputs and results (slot = the batch) and once bare, for capture
            self.prep_staged = dsa.PreparedStep(c.cache, c.seqs, c.queries, stager=stager, slot=len(staged),
                                                host_in=[(self.dev_in_buf, self.host_in)],
                                                host_out=[(self.dev_out_buf, self.host_out)], **kw)
            self.prep = dsa.PreparedStep(c.cache, c.seqs, c.queries, **kw)
            self.in_ready = torch.cuda.Event()   # graph only: this batch's inputs landed
            self.consumed = torch.cuda.Event()   # its step ran
            self.out_done = torch.cuda.Event()   # its outputs read back

        def compute(self):
            self.prep()

        def step(self):
            """copy in, step, copy out: the copies on the stager's streams, the
            step on `stream`"""
            self.prep_staged()

    stager = dsa.Stager(n_case, stream)
    staged = []
    for c in cases:
        staged.append(Staged(c))
    h2d, d2h = staged[0].in_bytes, staged[0].out_bytes
    for st in staged:   # first use outside any capture
        st.step()
    stager.join()
    torch.cuda.synchronize(device)
    # the graph: a rotation's input copies on one side stream, its steps on the
    # main stream, each step's read-back on another side stream as soon as that
    # step is done, so the copies overlap the other batches' steps; with
    # rotating batches three rotations per graph (a batch's next input copy
    # waits until its previous step has read its inputs, and its next step
    # until its previous read-back has landed), so the join at the end of a
    # replay comes once per nine steps
    reps = 3 if rotate else 1
    s_in, s_out = torch.cuda.Stream(device), torch.cuda.Stream(device)
    graph_e2e = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph_e2e, stream=stream):
        fork = torch.cuda.Event()
        fork.record(stream)
        s_in.wait_event(fork)
        s_out.wait_event(fork)
        for r in range(reps):
            for st in staged:
                if r > 0:
                    s_in.wait_event(st.consumed)
                with torch.cuda.stream(s_in):
                    st.dev_in_buf.copy_(st.host_in, non_blocking=True)
                    st.in_ready.record(s_in)
            for st in staged:
                stream.wait_event(st.in_ready)
                if r > 0:
                    stream.wait_event(st.out_done)
                st.compute()
                st.consumed.record(stream)
                s_out.wait_event(st.consumed)
                with torch.cuda.stream(s_out):
                    st.host_out.copy_(st.dev_out_buf, non_blocking=True)
                    st.out_done.record(s_out)
        for st in staged:
            stream.wait_event(st.out_done)
    torch.cuda.synchronize(device)
    n_e2e = max(3 * n_case, min(steps, 150)) // n_case * n_case
    n_graph = max(1, n_e2e // (n_case * reps))   # replays in the graph timing
    e_s, e_e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)

    def time_e2e(eager):
        if rotate:
            with torch.cuda.stream(stream):
                e_s.record()
            if eager:
                e_s.synchronize()   # as below: the copy streams do not wait for `stream`
                for i in range(n_e2e):
                    staged[i % n_case].step()
                stager.join()
            else:
                with torch.cuda.stream(stream):
                    for i in range(n_graph):
                        graph_e2e.replay()
            with torch.cuda.stream(stream):
                e_e.record()
            stream.synchronize()
            total = e_s.elapsed_time(e_e) / 1e3
        else:
            total = 0.0
            for _ in range(n_e2e):
                with torch.cuda.stream(stream):
                    tm.cold_l2()
                    e_s.record()
                    if eager:
                        # the copy streams do not wait for `stream`: let the flush
                        # and the start event pass before the input copy is issued
                        e_s.synchronize()
                        staged[0].step()
                        stager.join()
                    else:
                        graph_e2e.replay()
                    e_e.record()
                stream.synchronize()
                total += e_s.elapsed_time(e_e) / 1e3
        total = max_over_ranks(total, world, device)
        n_steps = n_graph * n_case * reps if (rotate and not eager) else n_e2e
        return round(weak_scaling_throughput(spec.total_q, n_steps, world, total), 1)

    time_e2e(True)   # warm-up
    e2e_eager = time_e2e(True)
    e2e_graph = time_e2e(False)
    if int(err.item()) != 0:
        raise RuntimeError(f"device error bits {int(err.item())} in the end-to-end loop")
    del graph_e2e
    stager.close()
    return {"value": e2e_eager, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "how": ("the step issued from Python every step through dsa.PreparedStep (the step's library calls "
                    "with their arguments marshalled once) with the library's host staging (dsa_stager): each "
                    "step's inputs copied from one pinned buffer (one H2D copy) and out/lse read back into one "
                    "(one D2H copy) on the library's two copy streams, so one batch's copies overlap the other "
                    "batches' kernels; steps back to back over the independent batches, every copy inside the "
                    "timed region"),
            "graph_value": e2e_graph,
            "graph_how": ("the same copies and calls captured in a CUDA graph (three rotations per graph when the "
                          "batches rotate) whose input copies and read-backs run on side streams, overlapping the "
                          "other batches' steps; replayed")}


# ----------------------------------------------------------------------------- the other workloads
def measure_workload(name, device, steps=30, iso=15, seed=None, path="auto"):
    """A compact record of one of the other workloads: its step time (back to
    back over independent batches whose traffic exceeds the L2, or one step at
    a time after a cold-L2 flush when that would take more than MAX_ROTATE
    batches), and each launch of the step alone after a cold-L2 flush with the
    roofline that bounds it."""
    from dynamic_block_sparse_dsa_b200 import workloads as wk
    spec = wk.NAMED[name]()
    path, decode = pick_path(spec, path)
    err = torch.zeros(1, dtype=torch.int32, device=device)
    stream = torch.cuda.Stream(device)
    tm = Timer(device, stream)
    seed = {"tiny_decode": 1001, "batched_gqa_decode": 1002, "chunked_prefill": 1004,
            "mixed_ragged": 1005}.get(name, 1003) if seed is None else seed
    cases = [StepCase(spec, seed, device, stream, err, path)]
    ab = algorithmic_bytes(cases[0].wl)
    need = max(2, math.ceil(ROTATE_L2_MULTIPLE * L2_BYTES / ab["total"]))
    rotate = need <= MAX_ROTATE
    while rotate and len(cases) < need:
        cases.append(StepCase(spec, seed + 7919 * len(cases), device, stream, err, path))
    c0 = cases[0]
    for _ in range(3):
        tm.isolated(c0.graph, c0.ev, 1)
    if rotate:
        rot = rotation_graph(cases, lambda c: c.run_step, stream, device)
        tm.rotated(rot, [c.graph for c in cases], len(cases))
        step_s = tm.rotated(rot, [c.graph for c in cases], steps) / steps
        how = f"back to back over {len(cases)} independent batches (inputs larger than L2)"
        del rot
        if decode:
            ov_s, _ = time_overlapped(cases, stream, device, steps * len(cases) * OVERLAP_PASSES)
    else:
        step_s = statistics.median(tm.isolated(c0.graph, c0.ev, steps)) / 1e3
        how = "one step at a time after a cold-L2 flush (median; includes one graph launch)"
    peak, peak_kind = _peaks()
    rec = {"path": path, "queries": spec.total_q, "block_size": spec.block_size, "top_k": spec.k_max,
           "step_us": round(step_s * 1e6, 2),
           "tokens_per_s": round(spec.total_q / step_s, 1), "step_timing": how, "phases": {}}
    kv_gb, flops = ab["kv"], ab["flops"]
    if decode:
        rec["step_bytes"] = ab["total"]
        rec["step_gbs"] = round(ab["total"] / step_s / 1e9, 1)
        rec["step_frac_of_measured_hbm"] = round(ab["total"] / step_s / 1e9 / peak, 4)
        if rotate:
            rec["overlapped"] = {"batches_in_flight": len(cases), "step_us": round(ov_s * 1e6, 2),
                                 "tokens_per_s": round(spec.total_q / ov_s, 1),
                                 "step_frac_of_measured_hbm": round(ab["total"] / ov_s / 1e9 / peak, 4),
                                 "how": f"each batch on a stream of its own, {OVERLAP_PASSES} steps of each per graph"}
    for i, (pname, _) in enumerate(c0.phases()):
        if rotate:
            # the launch alone, back to back over the batches (as in the step)
            singles = [c.capture(c.phases()[i][1])[0] for c in cases]
            whole = rotation_graph(cases, lambda c: c.phases()[i][1], stream, device)
            tm.rotated(whole, singles, len(cases))
            n = max(steps, 3 * len(cases))
            us = tm.rotated(whole, singles, n) / n * 1e6
            del whole, singles
        else:
            g, ev = c0.capture(c0.phases()[i][1])
            us = statistics.median(tm.isolated(g, ev, iso)) * 1e3
            del g
        ph = {"us": round(us, 2)}
        if pname == "attention":
            gbs = kv_gb / us / 1e3
            ph.update({"selected_kv_bytes": kv_gb, "tflops": round(flops / us / 1e6, 2)})
            if decode:
                ph.update({"gbs": round(gbs, 1), "frac_of_measured_hbm": round(gbs / peak, 4)})
            else:
                # prefill queries re-read shared pages from L2: the gather rate is
                # not an HBM rate; the bound reported is the bf16 contraction's
                tpk, _ = _bf16_sustained()
                ph.update({"gather_gbs_l2_and_hbm": round(gbs, 1),
                           "frac_of_bf16_sustained": round(flops / us / 1e6 / tpk, 4)})
        elif pname in ("index_score", "select", "select_append"):
            ops = indexer_ops(spec)
            ipk, _ = _int8_peak()
            ph.update({"int8_ops": ops, "tops": round(ops / us / 1e6, 1), "frac_of_int8_peak": round(ops / us / 1e6 / ipk, 4),
                       "coarse_key_bytes": ab["coarse_keys"]})
        rec["phases"][pname] = ph
    rec["phase_timing"] = (f"each launch alone, back to back over the {len(cases)} batches (mean)" if rotate else
                           "each launch alone after a cold-L2 flush (median of %d, in-graph events; includes one "
                           "graph launch)" % iso)
    if int(err.item()) != 0:
        raise RuntimeError(f"device error bits {int(err.item())} while timing {name}")
    del cases
    torch.cuda.synchronize(device)
    torch.cuda.empty_cache()
    return rec


# ----------------------------------------------------------------------------- prefill indexer
def prefill_indexer(device, seed=1004, iters=20):
    """The prefill indexer contraction (dsa_index_score on the 4096-query chunk
    after a 128K prefix) timed alone with a cold L2, against the int8 tensor
    roofline: ops = causal (query, block) pairs x 16 heads x 64 x 2."""
    import dynamic_block_sparse_dsa_b200 as dsa
    from dynamic_block_sparse_dsa_b200 import workloads as wk
    spec = wk.chunked_prefill()
    wl = wk.make_workload(spec, seed=seed, device=device)
    cache = dsa.PagedKVCache(wl.k_pool, wl.v_pool, wl.kc_pool)
    seqs = dsa.SeqBatch(wl.block_table, wl.seq_lens)
    queries = dsa.QueryBatch(wl.cu_q, wl.q_pos)
    err = torch.zeros(1, dtype=torch.int32, device=device)
    scores = torch.empty((spec.total_q, wl.block_table.shape[1]), dtype=torch.int32, device=device)
    stream = torch.cuda.Stream(device)
    tm = Timer(device, stream)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ops = indexer_ops(spec)
    ms = []
    with torch.cuda.stream(stream):
        for i in range(iters + 3):
            tm.cold_l2()
            e0.record()
            dsa.index_score(cache, seqs, queries, wl.q_idx, wl.w, 16, scores=scores, dev_err=err)
            e1.record()
            stream.synchronize()
            if i >= 3:
                ms.append(e0.elapsed_time(e1))
    if int(err.item()) != 0:
        raise RuntimeError(f"device error bits {int(err.item())} in the prefill indexer")
    t = statistics.median(ms) * 1e-3
    peak, src = _int8_peak()
    tops = ops / t / 1e12
    return {"workload": spec.name, "kernel": "index_score_tc_kernel (tcgen05 kind::i8)", "us": round(t * 1e6, 2),
            "int8_ops": ops, "achieved": round(tops, 1), "peak": round(peak, 1), "unit": "TOPS",
            "frac": round(tops / peak, 4), "peak_source": src, "frac_of_datasheet_4500": round(tops / 4500.0, 4),
            "l2": "cold before every launch"}


# ----------------------------------------------------------------------------- oracle (CPU) arm
def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or "unknown"


def usable_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def oracle_all_cores(inp, budget_s, workers):
    """``workers`` separate processes (one per core), each running whole
    oracle steps on its own memory-mapped copy of ``inp`` for about
    ``budget_s`` seconds once all of them are ready; returns (steps summed,
    seconds maxed)."""
    import shutil
    import subprocess
    import tempfile
    from oracle import harness
    d = tempfile.mkdtemp(prefix="dsa_oracle_")
    procs = []
    try:
        harness.save_inputs(inp, os.path.join(d, "inputs"))
        env = dict(os.environ, PYTHONPATH=ROOT + os.pathsep + os.environ.get("PYTHONPATH", ""))
        go = os.path.join(d, "go")
        for i in range(workers):
            procs.append(subprocess.Popen(
                [sys.executable, "-m", "oracle.harness", os.path.join(d, "inputs"), str(budget_s),
                 os.path.join(d, f"ready{i}"), go, os.path.join(d, f"out{i}")], cwd=ROOT, env=env))
        t0 = time.time()
        while not all(os.path.exists(os.path.join(d, f"ready{i}")) for i in range(workers)):
            if time.time() - t0 > 300 or any(p.poll() not in (None, 0) for p in procs):
                raise RuntimeError("oracle workers failed to start")
            time.sleep(0.01)
        open(go, "w").close()
        for p in procs:
            if p.wait(timeout=budget_s * 20 + 300) != 0:
                raise RuntimeError("an oracle worker failed")
        got = []
        for i in range(workers):
            with open(os.path.join(d, f"out{i}")) as f:
                n, sec = f.read().split()
            got.append((int(n), float(sec)))
    finally:
        for p in procs:
            if p.poll() is None:
                p.kill()
        shutil.rmtree(d, ignore_errors=True)
    return sum(g[0] for g in got), max(g[1] for g in got)


def cpu_baseline(wl, budget_s=10.0, max_steps=50):
    """The oracle as it stands (plain single-threaded C), on whole steps of the
    same workload: once on one core until about ``budget_s`` seconds of oracle
    time are spent, then as one process per usable core for about ``budget_s``
    seconds of wall time."""
    from oracle.harness import host_inputs, run_host
    inp = host_inputs(wl)
    spent, steps = 0.0, 0
    while steps < max_steps and (spent < budget_s or steps == 0):
        spent += run_host(inp)["seconds"]
        steps += 1
    tok = wl.spec.total_q
    single = tok * steps / spent
    cores = usable_cores()
    all_steps, all_s = oracle_all_cores(inp, budget_s, cores)
    multi = tok * all_steps / all_s
    return {"value": round(multi, 3), "unit": UNIT, "cores": cores, "kind": "oracle",
            "cpu_model": cpu_model(),
            "sample": (f"whole steps of {wl.spec.name} ({tok} queries each) on the oracle's host copies of the step's "
                       f"inputs: {all_steps} steps over {cores} processes (one per usable core, "
                       f"sched_getaffinity) in {all_s:.1f} s of wall time"),
            "single_thread": {"value": round(single, 3), "unit": UNIT, "cores": 1,
                              "sample": f"{steps} steps, {spent:.1f} s of oracle time on one core"}}


def run_reference(args, world, rank, device):
    from dynamic_block_sparse_dsa_b200 import workloads as wk
    from oracle.harness import host_inputs, run_host
    spec = wk.NAMED[args.workload]()
    wl = wk.make_workload(spec, seed=args.seed, device=device)
    inp = host_inputs(wl)
    for _ in range(args.warmup):
        run_host(inp)
    # the K steps as a bounded sample: about 20 s of wall time on all cores
    cores = usable_cores()
    one = run_host(inp)["seconds"]
    budget = min(20.0, max(2.0, one * args.steps / cores))
    steps, secs = oracle_all_cores(inp, budget, cores)
    value = spec.total_q * steps / secs
    return {"impl": "reference", "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(secs / steps * 1e3, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64+int64",
            "data": "synthetic (same seeded workload as our arm)",
            "config": {"workload": spec.name, "batch_per_gpu": spec.num_seqs, "context": max(spec.seq_lens),
                       "top_k": spec.k_max},
            "cpu_baseline": {"value": round(value, 3), "unit": UNIT, "cores": cores, "kind": "oracle",
                             "cpu_model": cpu_model(),
                             "sample": (f"{steps} whole steps of {spec.name} over {cores} processes (one per usable "
                                        f"core) in {secs:.1f} s of wall time; plain single-threaded C oracle in "
                                        f"each")},
            "e2e": {"value": round(value, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="decode_1m")
    ap.add_argument("--seed", type=int, default=1003)
    ap.add_argument("--rotate", type=int, default=2,
                    help="independent batches the timed steps rotate through (more if needed to exceed the L2)")
    ap.add_argument("--no-rotate", action="store_true",
                    help="one batch, each step timed after a cold-L2 flush (small profiling runs)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true", help="skip the prefill-indexer measurement")
    ap.add_argument("--no-configs", action="store_true", help="skip the other workloads' records")
    ap.add_argument("--path", choices=["auto", "fused_decode", "fused_select", "score_topk"], default="auto",
                    help="decode step as one launch, or as the chain of separate calls")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    world, rank, local = dist_env()
    if world != args.gpus and world > 1:
        print(f"warning: WORLD_SIZE={world} but --gpus={args.gpus}", file=sys.stderr)
    if args.impl == "reference" and rank != 0:
        return 0   # the oracle arm runs on rank 0 alone
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)

    if args.impl == "reference":
        print(json.dumps(run_reference(args, world, rank, device)), flush=True)
        return 0

    init_dist(world, "nccl")
    res, cases = run_ours(args, world, rank, device)
    wl = cases[0].wl
    if world == 1 and not args.no_cpu_baseline:   # the CPU baseline and the extra records: one GPU only
        res["cpu_baseline"] = cpu_baseline(wl)
    del cases, wl
    torch.cuda.synchronize(device)
    torch.cuda.empty_cache()
    if world == 1 and not args.no_prefill:
        res["prefill_indexer"] = prefill_indexer(device)
    if world == 1 and not args.no_configs:
        # the other workloads, one GPU: step time and each launch against its roofline
        # the prefill workloads also through the fused prefill pipeline:
        # scoring and selection in one kernel (no score matrix), then attention
        runs = [("tiny_decode", "auto"), ("batched_gqa_decode", "auto"), ("chunked_prefill", "auto"),
                ("chunked_prefill", "fused_select"), ("mixed_ragged", "auto"), ("mixed_ragged", "fused_select"),
                ("decode_1m_b128", "auto"), ("decode_1m_b256", "auto"), ("decode_1m_b512", "auto")]
        res["configs"] = {(n if p == "auto" else f"{n}@{p}"): measure_workload(n, device, path=p) for n, p in runs
                          if n != args.workload}
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        barrier(world)
        torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
