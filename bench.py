"""Benchmark of the Velox geometry-routed attention path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload headline|sweep|pipeline|robustness|rollout|overlap] [--P 48]

One step = one pass of the whole hot path over one chunk's synthetic inputs,
with the KV cache resident in HBM: frustum slices of every past chunk, slice
overlap counts, geometry-modulated top-k routing (pooling + scores + select)
and block-sparse attention over the routed blocks. The slices and counts are
built on a side stream one step ahead: chunk n+1's are built while chunk n's
attention runs (a step's routing waits only for its own counts, built during
the step before), as the method builds its slices asynchronously to
denoising; the timed steps therefore hold one extra geometry pass (the next
chunk's). `value` is the whole-job throughput in TFLOP/s of attention work on
the kept blocks
(4 * B * H * m * topk * T^2 * d per step) divided by the step time. The dense
attention over every block (this library's own dense attention) is timed
separately for the speedup.

Multi-GPU (torchrun, one process per GPU): by default the ranks split the 24
heads of one chunk (routing and attention of a head read only that head's
Q/K/V; the geometry is replicated) and all-gather O in place every step
("scaling": "strong"); with --shard chunks every rank runs its own chunk
(seed + rank) with no data-path collective ("scaling": "weak"). The time is the
max over ranks.

--impl reference times the fp64 CPU oracle on the host cores on a bounded
sample of the same workload (the oracle stands in for a reference
implementation: the method's pages publish no code).

--workload robustness (one GPU) measures how depth-estimation error moves
the selection: at P = 48, 96, 192 and 224 past chunks (or --P) the routing
from ground-truth depth is compared, row by row, with the routing of the
full geometry pipeline (multiwarp -> slices -> overlap) fed with perturbed
past depth (scale bias, multiplicative noise, holes); it also times routing,
sparse and dense attention at each P.

--workload rollout runs --chunks consecutive chunks from --P, each denoised
in --denoise-steps steps of --layers layers (pooled-key-cache routing and
sparse attention over a KV cache sized for all of them), with the geometry
built at each chunk boundary or pipelined one chunk ahead.

--workload overlap times the slice-overlap kernel at the headline size and on a
stress shape (64 scenes at 256 x 384 against 96 slices) against a measured
float64 FMA rate.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from geometry_routed_block_b200 import synth  # noqa: E402

METRIC = "chunk-48 routed attention ms & TFLOP/s (kept blocks), speedup vs dense; routing GB/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one sparse attention
# launch at the headline workload, from a one-pass ncu capture of this kernel at full
# size; reported only while the kernel sources still hash to what was captured.
ATTN_TRAFFIC = {
    "bytes_per_launch": 642.31e6 + 23.48e6,
    "sources": {"attention_pp.cu": "b928acde795e1f93", "attn_common.cuh": "f9d878738244f2cb",
                "ptx.cuh": "16d190c725154d53"},
}


def attn_traffic():
    import hashlib
    base = os.path.join(ROOT, "geometry_routed_block_b200", "csrc")
    for name, want in ATTN_TRAFFIC["sources"].items():
        with open(os.path.join(base, name), "rb") as f:
            if hashlib.sha256(f.read()).hexdigest()[:16] != want:
                return None
    return ATTN_TRAFFIC["bytes_per_launch"]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(PEAKS_FALLBACK), "fallback"


def workload_desc(s: synth.Shape) -> str:
    return (f"chunk-{s.P} routed attention: B{s.B} H{s.H} d{s.d} T{s.T}, chunk {s.F}x{s.Hp}x{s.Wp}"
            f"={s.Nq} tokens, {s.P} past chunks, Nk={s.Nk}, {s.nKB} key blocks, topk={s.topk}, "
            f"alpha={s.alpha}")


def kept_flops(s: synth.Shape) -> float:
    return 4.0 * s.B * s.H * s.m * s.topk * s.T * s.T * s.d


def dense_flops(s: synth.Shape) -> float:
    return 4.0 * s.B * s.H * s.m * s.nKB * s.T * s.T * s.d


def routing_bytes(s: synth.Shape) -> float:
    """Algorithmic bytes of routing: Q + past K read once, idx written, counts read."""
    return (2.0 * s.B * s.H * s.d * (s.Nq + s.P * s.Nq) + 4.0 * s.B * s.H * s.m * s.topk
            + 4.0 * s.B * s.m * s.P)


# ----------------------------------------------------------------------------
# clocks during the timed region
# ----------------------------------------------------------------------------

class ClockSampler:
    """nvidia-smi queries (read only) every 50 ms while it is open; begin() and
    end() mark the timed region on the host clock, and summary() keeps the
    samples taken inside it (all of them, flagged, if the region was shorter
    than the sampling interval)."""
    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.t0 = self.t1 = None

    def begin(self):
        self.t0 = time.time()

    def end(self):
        self.t1 = time.time()

    def __enter__(self):
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not self.path or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        import datetime
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                rows.append((ts, float(parts[1]), float(parts[2]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        inside = [r for r in rows if self.t0 is not None and self.t1 is not None
                  and self.t0 <= r[0] <= self.t1]
        use = inside if inside else rows
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = set()
        for r in use:
            for n, v in zip(names, r[3]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        sm = [r[1] for r in use]
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": use[-1][2] if use else None, "samples": len(sm),
                "window": "timed region" if inside else "whole sampler run (no sample inside "
                                                        "the timed region)",
                "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------
# CPU oracle sample (cpu_baseline and the reference arm)
# ----------------------------------------------------------------------------

def cpu_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return int(max(n)) if n else 1
    except Exception:
        return os.cpu_count() or 1


SAMPLE_ROWS = 4  # query blocks of the sampled head whose attention the oracle computes


def oracle_sample(case, head: int = 0, n_rows: int = SAMPLE_ROWS) -> dict:
    """Runs the oracle on one bounded sample of a step: all geometry (slices +
    overlap counts), the routing of one (batch, head) pair and the attention
    of `n_rows` evenly spaced query blocks of that pair. Returns the measured
    seconds of each part, the whole step extrapolated from them (geometry +
    B*H routings + B*H*m query blocks at the sampled per-block time), and the
    sample's counts and selection (for the parity check of the GPU's)."""
    from oracle import velox_oracle as vo
    s = case.shape
    n_rows = max(1, min(s.m, n_rows))
    t0 = time.perf_counter()
    sl = vo.slices_build(case.past_depth[0], case.past_poses[0], case.past_intr[0])
    counts = vo.block_overlap(case.cur_depth, case.cur_cam, sl[None], s.F, s.T)
    t1 = time.perf_counter()
    q, k, v = case.q[0][:, head:head + 1], case.k[0][:, head:head + 1], case.v[0][:, head:head + 1]
    idx, s_mod = vo.route_topk(q, k, counts, s.alpha, s.topk, s.T)
    t2 = time.perf_counter()
    qbs = [int(round(i * (s.m - 1) / max(1, n_rows - 1))) for i in range(n_rows)]
    vo.sparse_attention(q, k, v, idx, s.T, rows=[(0, 0, qb) for qb in qbs])
    t3 = time.perf_counter()
    pairs = s.B * s.H
    per_row = (t3 - t2) / len(qbs)
    est = (t1 - t0) + pairs * (t2 - t1) + pairs * s.m * per_row
    desc = (f"oracle (numpy fp64) on a bounded sample of one step: all geometry (slices + "
            f"overlap counts), routing of (batch 0, head {head}) and attention of {len(qbs)} of "
            f"its {s.m} query blocks (qb {qbs}); the whole step is extrapolated as geometry + "
            f"{pairs} x routing + {pairs * s.m} x per-block attention")
    return {"geometry_s": t1 - t0, "routing_s_per_head": t2 - t1,
            "attention_s_per_query_block": per_row, "sample_s": t3 - t0, "est_step_s": est,
            "desc": desc, "counts": counts, "idx": idx, "s_mod": s_mod}


def oracle_repeated(case, min_seconds: float, max_repeats: int = 64) -> dict:
    """oracle_sample run again and again until `min_seconds` of host time have
    gone by (at least once); every timing is the mean over the repeats."""
    runs = [oracle_sample(case)]
    t = runs[0]["sample_s"]
    while t < min_seconds and len(runs) < max_repeats:
        runs.append(oracle_sample(case))
        t += runs[-1]["sample_s"]
    r = dict(runs[0])
    for key in ("geometry_s", "routing_s_per_head", "attention_s_per_query_block", "sample_s",
                "est_step_s"):
        r[key] = statistics.mean(x[key] for x in runs)
    r["repeats"] = len(runs)
    return r


def oracle_single_thread(case, min_seconds: float = 2.0) -> dict:
    """oracle_repeated with the BLAS thread pool limited to one thread."""
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1):
        return oracle_repeated(case, min_seconds)


def baseline_record(kf: float, r: dict, r1: dict | None) -> dict:
    """The cpu_baseline object: the oracle's whole-step throughput extrapolated
    from the sample `r` (all host threads) and, when given, `r1` (one thread)."""
    out = {"value": round(kf / r["est_step_s"] / 1e12, 6), "unit": "TFLOP/s",
           "cores": cpu_threads(), "kind": "oracle", "sample": r["desc"], "extrapolated": True,
           "sample_seconds": round(r["sample_s"], 3), "repeats": r.get("repeats", 1),
           "est_step_seconds": round(r["est_step_s"], 2),
           "geometry_s": round(r["geometry_s"], 4),
           "routing_s_per_head": round(r["routing_s_per_head"], 4),
           "attention_s_per_query_block": round(r["attention_s_per_query_block"], 4)}
    if r1 is not None:
        out["single_thread"] = {
            "value": round(kf / r1["est_step_s"] / 1e12, 6), "cores": 1,
            "sample_seconds": round(r1["sample_s"], 3), "repeats": r1.get("repeats", 1),
            "est_step_seconds": round(r1["est_step_s"], 2),
            "routing_s_per_head": round(r1["routing_s_per_head"], 4),
            "attention_s_per_query_block": round(r1["attention_s_per_query_block"], 4)}
    return out


def selection_ties(gpu_idx, oracle_idx, s_mod, m) -> dict:
    """GPU selection vs the oracle's on the same rows under the parity rule
    (equal, or differing only at blocks within 1e-4 of the threshold)."""
    from tests.parity_utils import TIE_TOL, compare_selection
    try:
        ties = compare_selection(gpu_idx, oracle_idx, s_mod, m)
        return {"rows": int(np.prod(gpu_idx.shape[:-1])), "near_tie_rows": ties,
                "tie_tol": TIE_TOL, "ok": True}
    except AssertionError as e:
        return {"rows": int(np.prod(gpu_idx.shape[:-1])), "ok": False, "error": str(e)[:200]}


# ----------------------------------------------------------------------------
# GPU workload
# ----------------------------------------------------------------------------

class Workload:
    def __init__(self, case, device):
        import torch
        from geometry_routed_block_b200 import velox as vx
        self.vx, self.torch = vx, torch
        self.case, self.s = case, case.shape
        s = self.s
        self.device = device

        def dev(a):
            if a.dtype == np.uint16:
                return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(
                    torch.bfloat16).to(device)
            return torch.from_numpy(np.ascontiguousarray(a)).to(device)

        self.q, self.k, self.v = dev(case.q[0]), dev(case.k[0]), dev(case.v[0])
        H = self.q.shape[1]  # the heads this process holds (all, or its share)
        self.past_depth = dev(case.past_depth[0])
        self.past_poses = dev(case.past_poses[0])
        self.past_intr = dev(case.past_intr[0])
        self.cur_depth, self.cur_cam = dev(case.cur_depth), dev(case.cur_cam)
        self.slices = torch.empty((s.P, 18), dtype=torch.float32, device=device)
        self.counts = torch.empty((s.B, s.m, s.P), dtype=torch.int32, device=device)
        self.ws = vx.route_workspace(s.B, H, s.Nq, s.Nk, s.d, s.T, device)
        self.idx = torch.empty((s.B, H, s.m, s.topk), dtype=torch.int32, device=device)
        self.o = torch.empty_like(self.q)
        self.o_dense = torch.empty_like(self.q)
        self.lse = torch.empty((s.B, H, s.Nq), dtype=torch.float32, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.launches_per_step = 6  # slices, overlap, pool_q, pool_score, select, attention
        # the geometry runs on a side stream; only the selection waits for its counts
        self.side = torch.cuda.Stream(device=device)
        self.geo_ready = torch.cuda.Event()
        self.after_attend = None  # e.g. the all-gather of O when heads are sharded
        # geometry one step ahead (step_ahead): double-buffered counts, with events
        # for "counts j built" and "the selection reading counts j done"
        self.counts2 = [self.counts, torch.empty_like(self.counts)]
        self.geo_ev = [torch.cuda.Event(), torch.cuda.Event()]
        self.sel_ev = [torch.cuda.Event(), torch.cuda.Event()]
        self.cur = None

    def geometry(self, counts=None, depth=None, cam=None):
        vx, s = self.vx, self.s
        vx.slices_build(self.past_depth, self.past_poses, self.past_intr, out=self.slices)
        vx.block_overlap(self.cur_depth if depth is None else depth,
                         self.cur_cam if cam is None else cam, self.slices[None], s.F, s.T,
                         out=self.counts if counts is None else counts)

    def route(self, ready=None, counts=None):
        s = self.s
        self.vx.route_topk(self.q, self.k, self.counts if counts is None else counts, s.alpha,
                           s.topk, s.T, ws=self.ws, out=self.idx, counts_ready=ready)

    def attend(self):
        self.vx.sparse_attn_fwd(self.q, self.k, self.v, self.idx, self.s.T, out=self.o,
                                lse=self.lse, status=self.status)
        if self.after_attend is not None:
            self.after_attend()

    def dense(self):
        self.vx.sparse_attn_fwd(self.q, self.k, self.v, None, self.s.T, out=self.o_dense,
                                want_lse=False, status=self.status)

    def step(self, ev=None, route=None):
        """Slices and overlap counts on the side stream while the keys are pooled
        on the current one (the selection waits for the counts through an
        event), then attention. ev: events for geometry (ev0 -> ev1, side
        stream), routing (ev0 -> ev2, including any wait for the counts) and
        attention (ev2 -> ev3)."""
        torch = self.torch
        main = torch.cuda.current_stream()
        self.side.wait_stream(main)  # this step's inputs were written on `main`
        if ev is not None:
            ev[0].record(main)
        with torch.cuda.stream(self.side):
            self.geometry()
            if ev is not None:
                ev[1].record(self.side)
            self.geo_ready.record(self.side)
        (route or self.route)(ready=self.geo_ready)
        if ev is not None:
            ev[2].record(main)
        self.attend()
        if ev is not None:
            ev[3].record(main)

    def prime(self, depth=None, cam=None, ready=None):
        """Builds the first step's counts on the side stream (step_ahead's prologue)."""
        torch = self.torch
        self.side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(self.side):
            if ready is not None:
                self.side.wait_event(ready)
            self.geometry(self.counts2[0], depth, cam)
            self.geo_ev[0].record(self.side)
        self.cur = 0

    def step_ahead(self, ev=None, route=None, next_depth=None, next_cam=None, next_ready=None):
        """One step with the geometry pipelined one step ahead: routing (after
        the stream waits for the counts built during the previous step), then
        attention; the next step's slices and counts are built on the side stream
        once this step's selection is done, so they run under this step's
        attention instead of competing with the scorer for SMs (the method builds
        slices asynchronously to denoising). next_depth / next_cam: the next
        step's inputs (default: this step's), next_ready: an event they wait for.
        ev: routing (ev0 -> ev2) and attention (ev2 -> ev3)."""
        torch = self.torch
        main = torch.cuda.current_stream()
        if self.cur is None:
            self.prime()
        j = self.cur
        # the counts were built on the side stream during the previous step's
        # attention, so they are ready long before this point on the GPU
        # timeline: the main stream waits for them here (in the step time, not
        # in the routing interval), and the routing runs without a mid-stream
        # event wait (which would keep the selection from overlapping the
        # scorer's tail)
        main.wait_event(self.geo_ev[j])
        if ev is not None:
            ev[0].record(main)
        (route or self.route)(ready=None, counts=self.counts2[j])
        self.sel_ev[j].record(main)
        if ev is not None:
            ev[2].record(main)
        # counts2[1 - j] was last read by the previous step's selection, which the
        # stream order puts before this one
        self.side.wait_event(self.sel_ev[j])
        with torch.cuda.stream(self.side):
            if next_ready is not None:
                self.side.wait_event(next_ready)
            self.geometry(self.counts2[1 - j], next_depth, next_cam)
            self.geo_ev[1 - j].record(self.side)
        self.attend()
        if ev is not None:
            ev[3].record(main)
        self.cur = 1 - j


def reduce_max(values, device=None):
    """Element-wise max of `values` over all ranks (identity on one rank)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_throughput(world: int, units_per_rank: float, ms: float) -> float:
    """Whole-job rate: every rank processed `units_per_rank` in at most `ms`."""
    return world * units_per_rank / (ms * 1e-3)


def head_range(H: int, world: int, rank: int) -> tuple:
    """Heads [h0, h1) of `rank` when the H heads are split evenly over `world` ranks."""
    if H % world:
        raise ValueError(f"{H} heads do not split evenly over {world} ranks")
    n = H // world
    return rank * n, (rank + 1) * n


def gather_heads(o_all, o_local, world: int):
    """Every rank's [B, H/world, N, d] output o_local -> o_all [world * B, H/world, N, d]
    (rank r's share at rows r*B .. r*B+B-1) on every rank, by one all-gather into
    the preallocated buffer: in place when o_local is this rank's slice of
    o_all. Returns the whole output as [B, H, N, d], heads in order (rank-major,
    as head_range splits them): a view of o_all when B = 1, a permuted copy
    otherwise."""
    import torch.distributed as dist
    if world > 1:
        dist.all_gather_into_tensor(o_all, o_local)
    WB, h, N, d = o_all.shape
    B = WB // world
    if B == 1:
        return o_all.view(1, world * h, N, d)
    return o_all.view(world, B, h, N, d).permute(1, 0, 2, 3, 4).reshape(B, world * h, N, d)


def rank_seed(cfg: int, rank: int) -> int:
    """Each rank runs its own chunk: the workload's seed offset by the rank."""
    return 1000 + cfg + rank


def time_loop(torch, fn, reps):
    st = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a.record(st)
    for _ in range(reps):
        fn()
    b.record(st)
    torch.cuda.synchronize()
    return a.elapsed_time(b) / reps


SWEEP_P = (8, 16, 24, 32, 96)


def sweep_point(torch, vx, device, P: int, reps: int, peaks: dict, status, T: int = 128,
                d: int = 128):
    """Workload 4 at P past chunks on this GPU (geometry from the synthetic
    trajectory, Q/K/V drawn on the device with workload 3's structure; other
    block sizes T and head dims d on request): routing, sparse attention and
    dense attention timed alone with CUDA events. Returns the record and, for
    the oracle check, head 0's inputs and selection."""
    geo = synth.geometry_only(4, P=P)
    s = synth.shape_for(4, P=P, T=T, d=d)
    q, k, v = draw_qkv_on_device(torch, s, geo.meta["view_overlap"], 1004 + P, device)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    slices = vx.slices_build(dev(geo.past_depth[0]), dev(geo.past_poses[0]), dev(geo.past_intr[0]))
    counts = vx.block_overlap(dev(geo.cur_depth), dev(geo.cur_cam), slices[None], s.F, s.T)
    ws = vx.route_workspace(s.B, s.H, s.Nq, s.Nk, s.d, s.T, device)
    idx = torch.empty((s.B, s.H, s.m, s.topk), dtype=torch.int32, device=device)
    o, o2 = torch.empty_like(q), torch.empty_like(q)
    lse = torch.empty((s.B, s.H, s.Nq), dtype=torch.float32, device=device)
    route = lambda: vx.route_topk(q, k, counts, s.alpha, s.topk, s.T, ws=ws, out=idx)
    attend = lambda: vx.sparse_attn_fwd(q, k, v, idx, s.T, out=o, lse=lse, status=status)
    dense = lambda: vx.sparse_attn_fwd(q, k, v, None, s.T, out=o2, want_lse=False, status=status)
    for _ in range(3):
        route()
        attend()
    dense()
    t_route = time_loop(torch, route, reps)
    t_attn = time_loop(torch, attend, reps)
    t_dense = time_loop(torch, dense, max(2, reps // 4))
    rbytes = routing_bytes(s)
    kf, df = kept_flops(s), dense_flops(s)
    attn_tf = kf / (t_attn * 1e-3) / 1e12
    route_gbs = rbytes / (t_route * 1e-3) / 1e9
    rec = {
        "P": P, "T": s.T, "d": s.d, "key_blocks": s.nKB, "topk": s.topk,
        "kept_fraction": round(s.topk / s.nKB, 4),
        "routing_ms": round(t_route, 4), "routing_gbs": round(route_gbs, 1),
        "routing_hbm_frac": round(route_gbs / peaks["hbm_gbs"], 4),
        "sparse_attn_ms": round(t_attn, 4), "attn_tflops_kept": round(attn_tf, 1),
        "attn_tensor_frac": round(attn_tf / peaks["bf16_tflops"], 4),
        "dense_attn_ms": round(t_dense, 4),
        "dense_tflops": round(df / (t_dense * 1e-3) / 1e12, 1),
        "speedup_vs_dense": round(t_dense / (t_route + t_attn), 3),
        "attn_speedup_vs_dense": round(t_dense / t_attn, 3),
        "allowed_speedup": round(s.nKB / s.topk, 3),
    }
    check = {"q": q[:, :1].cpu(), "k": k[:, :1].cpu(), "idx": idx[:, :1].cpu().numpy(),
             "counts": counts.cpu().numpy(), "shape": s}
    return rec, check


def run_gpu(args):
    import torch
    import torch.distributed as dist
    from geometry_routed_block_b200 import velox as vx

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=device)

    cfg = 4 if args.workload == "sweep" else 3
    by_heads = args.shard == "heads"
    extra = {"T": args.T, "d": args.d} if cfg == 4 else {}
    if by_heads:
        # one chunk for the whole job; each rank routes and attends its share of the
        # heads (geometry replicated) and the heads' outputs are all-gathered
        h0, h1 = head_range(synth.shape_for(cfg, P=args.P, **extra).H, world, rank)
        heads = None if (h0, h1) == (0, synth.shape_for(cfg, P=args.P, **extra).H) else tuple(range(h0, h1))
        case = synth.make_case(cfg, seed=1000 + cfg, P=args.P, heads=heads, **extra)
    else:
        case = synth.make_case(cfg, seed=rank_seed(cfg, rank), P=args.P, **extra)
    s = case.shape
    w = Workload(case, device)
    o_all = None
    if by_heads and world > 1:
        # this rank's heads are written straight into its slice of the gathered output
        B_ = w.o.shape[0]
        o_all = torch.empty((world * B_,) + tuple(w.o.shape[1:]), dtype=w.o.dtype, device=device)
        w.o = o_all[rank * B_:(rank + 1) * B_]
        w.after_attend = lambda: gather_heads(o_all, w.o, world)
    peaks, peak_kind = load_peaks()

    # warm-up (also the first-call costs: tensor-map encode, attribute set)
    for _ in range(max(3, args.warmup)):
        w.step_ahead()
    w.dense()
    torch.cuda.synchronize()

    # ---- timed region: K whole steps, with per-stage events
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    with ClockSampler(local) as clk:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        clk.begin()
        t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t_start.record()
        for i in range(args.steps):
            w.step_ahead(evs[i])
        t_end.record()
        torch.cuda.synchronize()
        clk.end()
        if world > 1:
            dist.barrier()
    clocks = clk.summary()
    ms_total = t_start.elapsed_time(t_end)
    route_ms = statistics.mean(e[0].elapsed_time(e[2]) for e in evs)
    attn_ms = statistics.mean(e[2].elapsed_time(e[3]) for e in evs)
    status = int(w.status.item())
    gpu_idx = w.idx.cpu().numpy()
    # the geometry (slices + overlap counts) alone; in the steps it runs on the side
    # stream under the previous step's attention
    geo_ms = time_loop(torch, w.geometry, 20)

    # ---- pooled-key cache: each past chunk's key blocks pooled once when the chunk
    # was appended; per step the routing reads the 21 MB cache instead of 1.36 GB of K
    kbar = w.vx.kbar_cache(s.B, w.q.shape[1], s.P, s.Nq, s.d, s.T, device)
    append_ms = time_loop(torch, lambda: [w.vx.kbar_append(w.k, s.Nq, s.T, j, kbar)
                                          for j in range(s.P)], 3) / s.P

    def route_cached(ready=None, counts=None):
        w.vx.route_topk_cached(w.q, kbar, s.P, w.counts if counts is None else counts, s.alpha,
                               s.topk, s.T, ws=w.ws, out=w.idx, counts_ready=ready)

    def step_cached():
        w.step_ahead(route=route_cached)

    route_cached()
    route_cached_ms = time_loop(torch, route_cached, 20)
    step_cached_ms = time_loop(torch, step_cached, max(3, min(50, args.steps // 2)))

    # ---- dense baseline, timed alone (inputs > L2, so no flush is needed)
    dense_reps = max(3, min(20, args.steps // 10))
    dense_ms = time_loop(torch, w.dense, dense_reps)
    # context only, not on the path: PyTorch's own dense attention on the same tensors
    sdpa_ms = None
    try:
        import torch.nn.functional as F
        sdpa = lambda: F.scaled_dot_product_attention(w.q, w.k, w.v)
        sdpa()
        sdpa_ms = time_loop(torch, sdpa, dense_reps)
    except RuntimeError:
        pass

    # ---- end to end through the public API with host buffers: each step copies
    # the chunk's new inputs (Q, the current chunk's K and V, its depth map and
    # camera) from pinned host memory and reads O back. The copies run on their
    # own streams, double-buffered: step i+1's inputs go up and step i's O comes
    # down while step i computes; the current chunk's K/V are moved from the
    # staging buffer into the KV cache on the compute stream.
    h_q = w.q.cpu().pin_memory()
    h_k = w.k[:, :, s.P * s.Nq:].contiguous().cpu().pin_memory()
    h_v = w.v[:, :, s.P * s.Nq:].contiguous().cpu().pin_memory()
    h_depth = w.cur_depth.cpu().pin_memory()
    h_cam = w.cur_cam.cpu().pin_memory()
    h_o = torch.empty(w.o.shape, dtype=w.o.dtype).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in (h_q, h_k, h_v, h_depth, h_cam))
    d2h = h_o.numel() * h_o.element_size()
    stage = [{"q": torch.empty_like(w.q), "k": torch.empty(h_k.shape, dtype=h_k.dtype, device=device),
              "v": torch.empty(h_v.shape, dtype=h_v.dtype, device=device),
              "depth": torch.empty_like(w.cur_depth), "cam": torch.empty_like(w.cur_cam),
              "o": torch.empty_like(w.o)} for _ in range(2)]
    up, down = torch.cuda.Stream(device=device), torch.cuda.Stream(device=device)
    compute = torch.cuda.current_stream()
    ev = lambda: torch.cuda.Event()
    uploaded, consumed, o_ready, o_read = ([ev() for _ in range(2)] for _ in range(4))
    q0, depth0, cam0, o0 = w.q, w.cur_depth, w.cur_cam, w.o

    def upload(b):
        with torch.cuda.stream(up):
            up.wait_event(consumed[b])
            for key, h in (("q", h_q), ("k", h_k), ("v", h_v), ("depth", h_depth), ("cam", h_cam)):
                stage[b][key].copy_(h, non_blocking=True)
            uploaded[b].record(up)

    def e2e_run(n):
        for b in range(2):
            consumed[b].record(compute)
            o_read[b].record(compute)
        upload(0)
        # the first step's geometry from its uploaded depth and camera; every later
        # step's is built during the step before it (step_ahead)
        w.prime(stage[0]["depth"], stage[0]["cam"], uploaded[0])
        for i in range(n):
            b = i & 1
            if i + 1 < n:
                upload(b ^ 1)
            compute.wait_event(uploaded[b])
            compute.wait_event(o_read[b])  # stage[b]["o"] was copied down two steps ago
            w.k[:, :, s.P * s.Nq:].copy_(stage[b]["k"])
            w.v[:, :, s.P * s.Nq:].copy_(stage[b]["v"])
            w.q, w.cur_depth, w.cur_cam, w.o = (stage[b]["q"], stage[b]["depth"], stage[b]["cam"],
                                                stage[b]["o"])
            nxt = stage[b ^ 1] if i + 1 < n else stage[b]
            w.step_ahead(next_depth=nxt["depth"], next_cam=nxt["cam"],
                         next_ready=uploaded[b ^ 1] if i + 1 < n else None)
            consumed[b].record(compute)
            o_ready[b].record(compute)
            with torch.cuda.stream(down):
                down.wait_event(o_ready[b])
                h_o.copy_(stage[b]["o"], non_blocking=True)
                o_read[b].record(down)
        compute.wait_stream(down)
        compute.wait_stream(up)
        compute.wait_stream(w.side)
        w.q, w.cur_depth, w.cur_cam, w.o = q0, depth0, cam0, o0
        w.cur = None  # the next step primes its own geometry again

    e2e_reps = max(3, min(50, args.steps // 4))
    e2e_run(2)
    if world > 1:
        dist.barrier()
    e2e_ms = time_loop(torch, lambda: e2e_run(e2e_reps), 1) / e2e_reps
    h_o_ok = bool(torch.equal(h_o, w.o.cpu()))

    # the host links alone: one step's uploads, its download, and both at once
    def copies(up_on=True, down_on=True):
        if up_on:
            with torch.cuda.stream(up):
                for key, h in (("q", h_q), ("k", h_k), ("v", h_v), ("depth", h_depth),
                               ("cam", h_cam)):
                    stage[0][key].copy_(h, non_blocking=True)
        if down_on:
            with torch.cuda.stream(down):
                h_o.copy_(stage[1]["o"], non_blocking=True)
        compute.wait_stream(up)
        compute.wait_stream(down)

    copies()
    h2d_ms = time_loop(torch, lambda: copies(True, False), 10)
    d2h_ms = time_loop(torch, lambda: copies(False, True), 10)
    both_ms = time_loop(torch, lambda: copies(True, True), 10)

    # ---- max over ranks
    ms_total, e2e_ms = reduce_max([ms_total, e2e_ms], device)
    ms_step = ms_total / args.steps

    # per-rank work: the whole chunk, or this rank's share of the heads
    share = world if by_heads else 1
    kf, df = kept_flops(s) / share, dense_flops(s) / share
    value = job_throughput(world, kf, ms_step) / 1e12
    attn_tflops = kf / (attn_ms * 1e-3) / 1e12
    rbytes = routing_bytes(s) / share
    route_gbs = rbytes / (route_ms * 1e-3) / 1e9
    peak_b = peaks["bf16_tflops"]
    peak_s = peaks.get("bf16_tflops_sustained", peak_b)
    out = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "strong" if by_heads else "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {
            "workload": workload_desc(s),
            "l2": "inputs larger than L2 (past K and V are 1.39 GB each at chunk 48); no flush",
            "kept_fraction": round(s.topk / s.nKB, 4),
            "parallelism": (f"heads split over {world} GPU(s), geometry replicated, O all-gathered "
                            "each step" if by_heads
                            else f"replicated chunks x{world} (one per GPU, no collective)"),
        },
        "routed_attn_ms": round(attn_ms, 4),
        "routing_ms": round(route_ms, 4),
        "geometry_ms": round(geo_ms, 4),
        "dense_attn_ms": round(dense_ms, 4),
        "attn_tflops_kept": round(attn_tflops, 2),
        "dense_tflops": round(df / (dense_ms * 1e-3) / 1e12, 2),
        "routing_gbs": round(route_gbs, 1),
        "routing_hbm_frac": round(route_gbs / peaks["hbm_gbs"], 4),
        "speedup_vs_dense": round(dense_ms / (route_ms + attn_ms), 3),
        "attn_speedup_vs_dense": round(dense_ms / attn_ms, 3),
        "torch_sdpa_dense": (None if sdpa_ms is None else
                             {"ms": round(sdpa_ms, 4),
                              "tflops": round(df / (sdpa_ms * 1e-3) / 1e12, 2),
                              "routed_step_speedup": round(sdpa_ms / (route_ms + attn_ms), 3),
                              "note": "torch.nn.functional.scaled_dot_product_attention on the "
                                      "same tensors, every key block: context only"}),
        "allowed_speedup": round(s.nKB / s.topk, 3),
        "pooled_key_cache": {
            "append_ms_per_chunk": round(append_ms, 4),
            "routing_ms": round(route_cached_ms, 4),
            "step_ms": round(step_cached_ms, 4),
            "speedup_vs_dense": round(dense_ms / (route_cached_ms + attn_ms), 3),
            "note": "routing from past chunks' pooled keys (pooled once per chunk)",
        },
        "roofline": {
            "bound": "tensor",
            "kernel": ("attn_pp_kernel (sparse walk, kept blocks)" if (s.T, s.d) == (128, 128)
                       else f"attn_fwd_kernel<d={s.d},T={s.T}> (sparse walk, kept blocks)"),
            "achieved": round(attn_tflops, 2),
            "peak": peak_b,
            "peak_kind": f"bf16 burst ({peak_kind}): the kernel is timed per launch",
            "unit": "TFLOP/s",
            "frac": round(attn_tflops / peak_b, 4),
            "frac_of_sustained": round(attn_tflops / peak_s, 4),
            "sustained_peak": peak_s,
            "traffic": attn_traffic() if s.P == 48 and cfg == 3 and share == 1 else None,
        },
        "routing_roofline": {
            "bound": "hbm", "achieved": round(route_gbs, 1), "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": round(route_gbs / peaks["hbm_gbs"], 4),
            "algorithmic_bytes": rbytes,
        },
        "e2e": {
            "value": round(job_throughput(world, kf, e2e_ms) / 1e12, 3),
            "unit": "TFLOP/s",
            "ms_per_step": round(e2e_ms, 4),
            "h2d_bytes_per_step": int(h2d),
            "d2h_bytes_per_step": int(d2h),
            "copies_alone_ms": {"h2d": round(h2d_ms, 4), "d2h": round(d2h_ms, 4),
                                "both": round(both_ms, 4)},
            "h2d_gbs": round(h2d / (h2d_ms * 1e-3) / 1e9, 1),
            "d2h_gbs": round(d2h / (d2h_ms * 1e-3) / 1e9, 1),
            "note": "past KV cache resident; per step the chunk's Q/K/V, depth and camera go "
                    "host->device and O comes back, on copy streams overlapped with the previous "
                    "/ next step's compute (double-buffered); copies_alone_ms times the same "
                    "copies with no compute",
            "o_matches_device": h_o_ok,
        },
        "gpu_launches": w.launches_per_step * args.steps,
        "device_status": status,
        "clocks": clocks,
    }

    extras = world == 1 and not args.no_extras and cfg == 3 and args.P in (None, 48)
    checks = []
    if extras:
        # ---- rollout-length sweep (workload 4) and the 30-layer pipeline (workload 5)
        sweep = []
        for P in SWEEP_P:
            rec, chk = sweep_point(torch, vx, device, P, max(3, min(10, args.steps // 20)), peaks,
                                   w.status)
            sweep.append(rec)
            checks.append(chk)
            torch.cuda.empty_cache()
        out["sweep"] = sweep
        # the other block sizes and head dims the kernels support, at chunk 48
        shapes = []
        for T, d in ((64, 128), (64, 64), (128, 64)):
            rec, _ = sweep_point(torch, vx, device, 48, max(3, min(10, args.steps // 20)), peaks,
                                 w.status, T=T, d=d)
            shapes.append(rec)
            torch.cuda.empty_cache()
        out["tile_shapes"] = shapes
        pipe = pipeline_measure(torch, vx, device, layers=30, steps=3, warmup=3, seed=1005)
        out["pipeline"] = {key: pipe[key] for key in (
            "layers", "ms_per_step", "tflops_kept", "geometry_ms", "geometry_done_after_ms",
            "layer0_routing_done_after_ms", "geometry_exposed_ms", "interleaved_async_step_ms",
            "interleaved_serial_step_ms")}
        out["pipeline"]["workload"] = pipe["workload"]
        out["gpu_launches_outside_timed_region"] = "sweep and pipeline records are timed separately"
        out["device_status"] = int(w.status.item())
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        # the reference arm's sample, repeated for about 10 s of host work (all
        # threads), then for about 2 s on one thread
        r = oracle_repeated(case, 10.0)
        r1 = oracle_single_thread(case)
        out["cpu_baseline"] = baseline_record(kf, r, r1)
        # the sampled head's selection against the GPU's, and head 0 of every sweep point
        ties = {"chunk 48 (workload 3), head 0": selection_ties(gpu_idx[:, :1], r["idx"],
                                                                 r["s_mod"], s.m)}
        if extras:
            from oracle import velox_oracle as vo
            for chk in checks:
                cs = chk["shape"]
                qh = chk["q"].view(torch.int16).numpy().view(np.uint16)
                kh = chk["k"].view(torch.int16).numpy().view(np.uint16)
                want, s_mod = vo.route_topk(qh, kh, chk["counts"], cs.alpha, cs.topk, cs.T)
                ties[f"P = {cs.P} (workload 4), head 0"] = selection_ties(chk["idx"], want, s_mod,
                                                                           cs.m)
        out["selection_vs_oracle"] = ties
    if rank == 0:
        print(json.dumps(out), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def layer_inputs_on_device(torch, case, layers: int, device, seed: int):
    """Layer 0 is the host-generated case; layers 1.. are drawn on the device
    with the same structure (Q = N(0,1) + mu_h, past chunk c's K shifted by the
    chunk's view-overlap proxy times mu_h, V = N(0,1)), one seeded generator per
    layer. Returns lists of bf16 tensors q[l], k[l], v[l]."""
    s = case.shape
    w0 = Workload(case, device)
    qs, ks, vs = [w0.q], [w0.k], [w0.v]
    ov = torch.tensor(case.meta["view_overlap"], dtype=torch.float32, device=device)
    for l in range(1, layers):
        g = torch.Generator(device=device)
        g.manual_seed(seed * 1000 + l)
        mu = 0.5 * torch.randn((s.H, 1, s.d), generator=g, device=device)
        q = (torch.randn((s.B, s.H, s.Nq, s.d), generator=g, device=device) + mu).to(torch.bfloat16)
        k = torch.randn((s.B, s.H, s.P + 1, s.Nq, s.d), generator=g, device=device)
        k[:, :, : s.P] += ov.view(1, 1, s.P, 1, 1) * mu.view(1, s.H, 1, 1, s.d)
        k = k.view(s.B, s.H, s.Nk, s.d).to(torch.bfloat16)
        v = torch.randn((s.B, s.H, s.Nk, s.d), generator=g, device=device).to(torch.bfloat16)
        qs.append(q), ks.append(k), vs.append(v)
        del k
    return w0, qs, ks, vs


def pipeline_measure(torch, vx, device, layers: int, steps: int, warmup: int, seed: int) -> dict:
    """One denoising step of the 30-layer pipeline at chunk 48: the geometry
    (recency-priority multiwarp of the 48 past depth maps -> slices -> overlap
    counts) runs on a side stream while layer 0 pools its keys; layer 0's
    selection waits for the counts; then routing + attention for every layer.
    Returns the timings, the geometry's exposure and the clocks."""
    case = synth.make_case(5, seed=seed, layers=1)
    s = case.shape
    s.layers = layers
    w, qs, ks, vs = layer_inputs_on_device(torch, case, layers, device, seed)

    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    past_depth = dev(case.past_depth[0])
    past_poses, past_intr = dev(case.past_poses[0]), dev(case.past_intr[0])
    past_cams = dev(np.stack([synth.camera_record(case.past_poses[0, j], case.past_intr[0, j])
                              for j in range(s.P)]))
    cur_cam = dev(case.cur_cam)
    cur_depth = torch.empty((1, s.Hp, s.Wp), dtype=torch.float32, device=device)
    mw_ws = vx.depth_multiwarp_workspace(s.Hp, s.Wp, device)
    slices = torch.empty((s.P, 18), dtype=torch.float32, device=device)
    counts = torch.empty((s.B, s.m, s.P), dtype=torch.int32, device=device)
    idx = torch.empty((s.B, s.H, s.m, s.topk), dtype=torch.int32, device=device)
    o = torch.empty_like(qs[0])
    lse = torch.empty((s.B, s.H, s.Nq), dtype=torch.float32, device=device)
    ws = w.ws
    main = torch.cuda.current_stream()
    side = torch.cuda.Stream(device=device)
    ev_start = torch.cuda.Event()
    ev_geo = torch.cuda.Event()

    def geometry(stream):
        vx.depth_multiwarp(past_depth, past_cams, cur_cam[0], 0.01, ws=mw_ws, out=cur_depth[0],
                           stream=stream)
        vx.slices_build(past_depth, past_poses, past_intr, out=slices, stream=stream)
        vx.block_overlap(cur_depth, cur_cam, slices[None], s.F, s.T, out=counts, stream=stream)

    def layer(l, ready=None, routed=None):
        vx.route_topk(qs[l], ks[l], counts, s.alpha, s.topk, s.T, ws=ws, out=idx, counts_ready=ready)
        if routed is not None:
            routed.record(main)
        vx.sparse_attn_fwd(qs[l], ks[l], vs[l], idx, s.T, out=o, lse=lse, status=w.status)

    def step_async(ev=None):
        ev_start.record(main)
        if ev is not None:
            ev[0].record(main)  # origin, before any geometry is enqueued
        side.wait_event(ev_start)
        geometry(side)
        ev_geo.record(side)
        if ev is not None:
            ev[1].record(side)  # geometry done
        for l in range(layers):
            layer(l, ev_geo if l == 0 else None, ev[2] if (ev is not None and l == 0) else None)
        if ev is not None:
            ev[3].record(main)

    def step_serial():
        geometry(main)
        for l in range(layers):
            layer(l)

    for _ in range(max(3, warmup)):
        step_async()
    step_serial()
    torch.cuda.synchronize()
    steps = max(1, steps)
    # the timed region: K whole steps with the geometry in flight on the side stream
    with ClockSampler(device.index or 0) as clk:
        clk.begin()
        t_async = time_loop(torch, step_async, steps)
        clk.end()
    clocks = clk.summary()
    # exposure, per step, from events: when the geometry is done vs when layer 0's
    # routing (whose selection waited for it) is done; plus the same steps run
    # serially, interleaved with async ones so clock drift cancels
    mk = lambda: torch.cuda.Event(enable_timing=True)
    geo_done, route0_done, a_ms, s_ms = [], [], [], []
    for _ in range(max(2, steps // 2)):
        ev = [mk() for _ in range(4)]
        step_async(ev)
        torch.cuda.synchronize()
        geo_done.append(ev[0].elapsed_time(ev[1]))
        route0_done.append(ev[0].elapsed_time(ev[2]))
        a_ms.append(ev[0].elapsed_time(ev[3]))
        e0, e1 = mk(), mk()
        e0.record(main)
        step_serial()
        e1.record(main)
        torch.cuda.synchronize()
        s_ms.append(e0.elapsed_time(e1))
    g0, g1 = mk(), mk()
    torch.cuda.synchronize()
    g0.record(side)
    for _ in range(20):
        geometry(side)
    g1.record(side)
    torch.cuda.synchronize()
    t_geo = g0.elapsed_time(g1) / 20
    med = statistics.median
    kf = kept_flops(s) * layers
    out = {
        "layers": layers, "steps": steps, "ms_per_step": round(t_async, 4),
        "tflops_kept": round(kf / (t_async * 1e-3) / 1e12, 3), "kept_flops": kf,
        "workload": f"denoising step, {layers} layers x " + workload_desc(s)
                    + "; current depth from the multiwarp of the past depth maps",
        "geometry_ms": round(t_geo, 4),
        "geometry_done_after_ms": round(med(geo_done), 4),
        "layer0_routing_done_after_ms": round(med(route0_done), 4),
        "geometry_exposed_ms": round(max(0.0, med(geo_done) - med(route0_done)), 4),
        "interleaved_async_step_ms": round(med(a_ms), 4),
        "interleaved_serial_step_ms": round(med(s_ms), 4),
        "gpu_launches": (7 + 4 * layers) * steps,
        "device_status": int(w.status.item()),
        "clocks": clocks,
    }
    del qs, ks, vs, w
    torch.cuda.empty_cache()
    return out


def run_pipeline(args):
    """The 30-layer pipeline (workload 5) as its own bench line."""
    import torch
    from geometry_routed_block_b200 import velox as vx
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    r = pipeline_measure(torch, vx, device, args.layers, args.steps, args.warmup, 1005 + rank)
    out = {
        "metric": METRIC, "value": round(world * r["tflops_kept"], 3), "unit": "TFLOP/s",
        "n_gpus": world, "steps": r["steps"], "warmup": args.warmup,
        "ms_per_step": r["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": r["workload"], "l2": "inputs larger than L2; no flush"},
        **{k: r[k] for k in ("geometry_ms", "geometry_done_after_ms",
                             "layer0_routing_done_after_ms", "geometry_exposed_ms",
                             "interleaved_async_step_ms", "interleaved_serial_step_ms",
                             "gpu_launches", "device_status", "clocks")},
    }
    if rank == 0:
        print(json.dumps(out), flush=True)


ROBUST_P = (48, 96, 192, 224)
DEPTH_ERRORS = (
    ("none", {}),
    ("scale x0.8", {"scale": 0.8}), ("scale x0.9", {"scale": 0.9}),
    ("scale x1.1", {"scale": 1.1}), ("scale x1.25", {"scale": 1.25}),
    ("noise 2%", {"noise_sd": 0.02}), ("noise 5%", {"noise_sd": 0.05}),
    ("noise 10%", {"noise_sd": 0.10}), ("noise 20%", {"noise_sd": 0.20}),
    ("holes 10%", {"hole_frac": 0.10}), ("holes 30%", {"hole_frac": 0.30}),
    ("holes 50%", {"hole_frac": 0.50}),
)


def selection_change(ref: np.ndarray, got: np.ndarray, n_past: int) -> dict:
    """Rows of ascending key-block lists [..., k]: how the past blocks `got`
    keeps differ from those `ref` keeps (current-chunk blocks, always kept,
    are left out). Mean Jaccard index and recall of `ref`'s blocks, and the
    fraction of rows whose past sets are identical."""
    ref = ref.reshape(-1, ref.shape[-1])
    got = got.reshape(-1, got.shape[-1])
    R = ref.shape[0]
    a = np.zeros((R, n_past), dtype=bool)
    b = np.zeros((R, n_past), dtype=bool)
    for mask, lst in ((a, ref), (b, got)):
        rows = np.broadcast_to(np.arange(R)[:, None], lst.shape)
        keep = lst < n_past
        mask[rows[keep], lst[keep]] = True
    inter = (a & b).sum(1)
    union = (a | b).sum(1)
    na = a.sum(1)
    jac = np.where(union > 0, inter / np.maximum(union, 1), 1.0)
    rec = np.where(na > 0, inter / np.maximum(na, 1), 1.0)
    return {"jaccard": round(float(jac.mean()), 4), "recall": round(float(rec.mean()), 4),
            "rows_identical": round(float((inter == union).mean()), 4)}


def draw_qkv_on_device(torch, s, view_overlap, seed: int, device):
    """Workload 3's Q/K/V structure drawn on the device, one head at a time
    (bounded temporaries at any P): Q = N(0,1) + mu_h, past chunk c's K =
    N(0,1) + view_overlap[c] * mu_h, current K and V = N(0,1)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    mu = 0.5 * torch.randn((s.H, s.d), generator=g, device=device)
    ov = torch.tensor(np.asarray(view_overlap), dtype=torch.float32, device=device)
    q = torch.empty((s.B, s.H, s.Nq, s.d), dtype=torch.bfloat16, device=device)
    k = torch.empty((s.B, s.H, s.Nk, s.d), dtype=torch.bfloat16, device=device)
    v = torch.empty((s.B, s.H, s.Nk, s.d), dtype=torch.bfloat16, device=device)
    for b in range(s.B):
        for h in range(s.H):
            q[b, h] = torch.randn((s.Nq, s.d), generator=g, device=device) + mu[h]
            kh = torch.randn((s.P + 1, s.Nq, s.d), generator=g, device=device)
            kh[: s.P] += ov.view(s.P, 1, 1) * mu[h].view(1, 1, s.d)
            k[b, h] = kh.view(s.Nk, s.d)
            del kh
            v[b, h] = torch.randn((s.Nk, s.d), generator=g, device=device)
    return q, k, v


def run_robustness(args):
    import torch
    from geometry_routed_block_b200 import velox as vx
    if int(os.environ.get("RANK", "0")) != 0:
        return
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    reps = max(3, min(args.steps, 10))
    status = torch.zeros(1, dtype=torch.int32, device=device)
    per_p = []
    for P in ([args.P] if args.P else ROBUST_P):
        geo = synth.geometry_only(4, P=P)
        s = synth.shape_for(4, P=P)
        q, k, v = draw_qkv_on_device(torch, s, geo.meta["view_overlap"], 1004 + P, device)
        dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
        past_poses, past_intr = dev(geo.past_poses[0]), dev(geo.past_intr[0])
        past_cams, cur_cam = dev(geo.past_cams[0]), dev(geo.cur_cam)
        mw_ws = vx.depth_multiwarp_workspace(s.Hp, s.Wp, device)
        ws = vx.route_workspace(s.B, s.H, s.Nq, s.Nk, s.d, s.T, device)
        n_past = s.P * s.m

        def counts_for(past_depth, cur_depth):
            sl = vx.slices_build(past_depth, past_poses, past_intr)
            return vx.block_overlap(cur_depth, cur_cam, sl[None], s.F, s.T)

        def route(counts):
            return vx.route_topk(q, k, counts, s.alpha, s.topk, s.T, ws=ws).cpu().numpy()

        gt_counts = counts_for(dev(geo.past_depth[0]), dev(geo.cur_depth))
        gtc = gt_counts.cpu().numpy()
        idx_gt = route(gt_counts)
        rows = [{"depth_error": "no geometry (alpha = 0)",
                 **selection_change(idx_gt, route(None), n_past)}]
        for e, (name, kw) in enumerate(DEPTH_ERRORS):
            rng = np.random.default_rng([1004, P, e])
            past = synth.perturb_depth(geo.past_depth[0], rng, **kw) if kw else geo.past_depth[0]
            past_t = dev(past)
            cur = vx.depth_multiwarp(past_t, past_cams, cur_cam[0], 0.01, ws=mw_ws)
            counts = counts_for(past_t, cur[None])
            c = counts.cpu().numpy()
            rows.append({"depth_error": name + " (multiwarp current depth)",
                         **selection_change(idx_gt, route(counts), n_past),
                         "count_mae_over_T": round(float(np.abs(c - gtc).mean()) / s.T, 4),
                         "covered_query_blocks": int((c.sum(-1) > 0).sum())})
        # timing at this P on the ground-truth route
        idx = torch.from_numpy(idx_gt).to(device)
        o, o2 = torch.empty_like(q), torch.empty_like(q)
        route_dev = lambda: vx.route_topk(q, k, gt_counts, s.alpha, s.topk, s.T, ws=ws, out=idx)
        attend = lambda: vx.sparse_attn_fwd(q, k, v, idx, s.T, out=o, want_lse=False, status=status)
        dense = lambda: vx.sparse_attn_fwd(q, k, v, None, s.T, out=o2, want_lse=False, status=status)
        for _ in range(3):
            route_dev()
            attend()
        dense()
        t_route = time_loop(torch, route_dev, reps)
        t_attn = time_loop(torch, attend, reps)
        t_dense = time_loop(torch, dense, 2)
        per_p.append({
            "P": P, "key_blocks": s.nKB, "topk": s.topk, "covered_query_blocks_gt":
            int((gtc.sum(-1) > 0).sum()), "selection_vs_ground_truth_depth": rows,
            "routing_ms": round(t_route, 4), "routing_gbs": round(routing_bytes(s) / t_route / 1e6, 1),
            "sparse_attn_ms": round(t_attn, 4),
            "sparse_attn_tflops": round(kept_flops(s) / t_attn / 1e9, 1),
            "dense_attn_ms": round(t_dense, 4),
            "speedup_vs_dense": round(t_dense / (t_route + t_attn), 3),
        })
        del q, k, v, o, o2, ws
        torch.cuda.empty_cache()
    out = {"workload": "robustness: depth error vs selection, rollouts P = "
           + "/".join(str(r["P"]) for r in per_p) + " (B1 H24 d128 T128, 3x32x48 chunks, k = 20%)",
           "data": "synthetic", "n_gpus": 1, "device_status": int(status.item()), "per_P": per_p}
    print(json.dumps(out), flush=True)


def run_rollout(args):
    """Several consecutive chunks of a rollout, each denoised in S steps of L
    layers: pooled-key-cache routing + sparse attention per layer, the pooled
    keys of a chunk appended when it is done, and the geometry either built
    at each chunk boundary or pipelined one chunk ahead. Reports both
    schedules' time per chunk and how much the look-ahead geometry (built from
    the previous chunk's warped depth, its final depth not yet known) changes
    the selection."""
    import torch
    from geometry_routed_block_b200 import velox as vx
    from geometry_routed_block_b200.rollout import Rollout
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    P0 = args.P or 48
    C, S, L = args.chunks, args.denoise_steps, args.layers
    cap = P0 + C  # chunks 0..cap-1 live in the KV cache
    seed = 1004 + rank
    geo = synth.geometry_only(4, seed=seed, P=cap)  # cameras and depth of chunks 0..cap
    s = synth.shape_for(4, P=cap - 1)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    cams = dev(np.concatenate([geo.past_cams[0], geo.cur_cam], 0))
    poses, intr = dev(geo.past_poses[0]), dev(geo.past_intr[0])
    final_depth = dev(np.concatenate([geo.past_depth[0], geo.cur_depth], 0))
    ov = np.asarray(geo.meta["view_overlap"])[: cap - 1]
    qs, ks, vs = [], [], []
    for layer in range(L):
        q, k, v = draw_qkv_on_device(torch, s, ov, seed * 1000 + layer, device)
        qs.append(q), ks.append(k), vs.append(v)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    o = torch.empty_like(qs[0])
    topk_of = lambda n: synth.topk_for(n, s.m)
    idx_buf = {n: torch.empty((s.B, s.H, s.m, topk_of(n)), dtype=torch.int32, device=device)
               for n in range(P0, cap)}
    states = {}
    for sched in ("boundary", "pipelined"):
        R = Rollout(ks, B=s.B, H=s.H, d=s.d, T=s.T, F=s.F, Hp=s.Hp, Wp=s.Wp, capacity=cap,
                    cams=cams, poses=poses, intr=intr, alpha=s.alpha, topk_of=topk_of,
                    schedule=sched)
        R.prefill(P0, final_depth[:P0])
        states[sched] = R

    def rollout(R, marks=None):
        for n in range(P0, cap):
            if marks is not None:
                marks[n][0].record()
            R.begin_chunk(n)
            for step in range(S):
                for layer in range(L):
                    idx = R.route(layer, qs[layer], out=idx_buf[n])
                    if marks is not None and step == 0 and layer == 0:
                        marks[n][1].record()
                    R.attend(layer, qs[layer], vs[layer], idx, out=o, status=status)
            R.end_chunk(n, final_depth[n])

    mk = lambda: torch.cuda.Event(enable_timing=True)
    times = {k: [] for k in states}
    first_route = {k: [] for k in states}
    reps = max(1, min(args.steps, 3))
    for it in range(1 + reps):  # one untimed rollout per schedule, then interleaved reps
        for sched, R in states.items():
            R.start(P0)
            torch.cuda.synchronize()
            marks = {n: (mk(), mk()) for n in range(P0, cap)}
            a, b = mk(), mk()
            a.record()
            rollout(R, marks)
            b.record()
            torch.cuda.synchronize()
            if it > 0:
                times[sched].append(a.elapsed_time(b) / C)
                first_route[sched] += [marks[n][0].elapsed_time(marks[n][1])
                                       for n in range(P0, cap)]
    med = statistics.median
    t = reduce_max([med(times["boundary"]), med(times["pipelined"])], device)
    # selection change of the look-ahead geometry: layer 0 of every chunk
    rows = []
    Rb, Rp = states["boundary"], states["pipelined"]
    for n in range(P0, cap):
        ib = vx.route_topk_cached(qs[0], Rb.kbar[0], n, Rb.counts[n], s.alpha, topk_of(n), s.T)
        ip = vx.route_topk_cached(qs[0], Rp.kbar[0], n, Rp.counts[n], s.alpha, topk_of(n), s.T)
        cb, cp = Rb.counts[n].cpu().numpy(), Rp.counts[n].cpu().numpy()
        rows.append({"chunk": n, **selection_change(ib.cpu().numpy(), ip.cpu().numpy(), n * s.m),
                     "count_mae_over_T": round(float(np.abs(cb - cp).mean()) / s.T, 4)})
    kf = sum(S * L * 4.0 * s.B * s.H * s.m * topk_of(n) * s.T * s.T * s.d for n in range(P0, cap))
    value = world * kf / (t[1] * C * 1e-3) / 1e12
    launches_chunk = S * L * 4 + L + 8  # route (3) + attention per layer; appends; geometry
    out = {
        "metric": METRIC, "value": round(value, 3), "unit": "TFLOP/s", "n_gpus": world,
        "steps": reps, "warmup": 1, "ms_per_step": round(t[1] * C, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": f"rollout of chunks {P0}..{cap - 1}, {S} denoising steps x {L} "
                   f"layers per chunk, pooled-key-cache routing, KV cache of {cap} chunks; "
                   + workload_desc(s), "l2": "inputs larger than L2; no flush"},
        "chunk_ms": {"boundary": round(t[0], 3), "pipelined": round(t[1], 3)},
        "geometry_exposed_ms_per_chunk": round(t[0] - t[1], 4),
        "first_route_done_ms": {k: round(med(v), 4) for k, v in first_route.items()},
        "lookahead_selection_vs_boundary": rows,
        "gpu_launches": launches_chunk * C * reps,
        "device_status": int(status.item()),
    }
    if rank == 0:
        print(json.dumps(out), flush=True)


# float64 operations of one overlap point test, from the method's formulas (a
# division counts as one): per (point, slice) q = R p + t (9 mul + 9 add) and
# u, v = f * (q_xy / q_z) + c (2 div + 2 mul + 2 add); per point, shared by the P
# slices, the back-projection (2 sub + 2 div + 2 mul) and p_w = R^T (p_c - t)
# (3 sub + 9 mul + 6 add).
OVERLAP_FLOPS_PER_TEST = 24.0
OVERLAP_FLOPS_PER_POINT = 24.0


def run_overlap(args):
    """The slice-overlap kernel at the headline size (latency-bound: us and
    point tests per second) and on a stress shape where its float64 ALU work
    dominates: 64 scenes at 256 x 384 (one frame per chunk) against 96 past
    slices, 604 M point tests. Its rate is set against a measured float64 FMA
    ceiling (velox_fp64_fma_bench). Also the multiwarp's candidate splats per
    second, at the headline size and with 96 past maps of 256 x 384."""
    import torch
    from geometry_routed_block_b200 import velox as vx
    if int(os.environ.get("RANK", "0")) != 0:
        return
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
    reps = max(3, min(args.steps, 50))
    # headline size
    geo = synth.geometry_only(3)
    s = synth.shape_for(3)
    sl = vx.slices_build(dev(geo.past_depth[0]), dev(geo.past_poses[0]), dev(geo.past_intr[0]))
    cd, cc = dev(geo.cur_depth), dev(geo.cur_cam)
    counts = vx.block_overlap(cd, cc, sl[None], s.F, s.T)
    for _ in range(3):
        vx.block_overlap(cd, cc, sl[None], s.F, s.T, out=counts)
    t_small = time_loop(torch, lambda: vx.block_overlap(cd, cc, sl[None], s.F, s.T, out=counts), reps)
    tests_small = s.B * s.Nq * s.P
    # float64 FMA ceiling
    props = torch.cuda.get_device_properties(device)
    fma_out = torch.zeros(1, dtype=torch.float64, device=device)
    blocks, threads, iters = props.multi_processor_count * 8, 256, 1 << 14
    fl = vx.fp64_fma_bench(fma_out, blocks, threads, iters)
    t_fma = time_loop(torch, lambda: vx.fp64_fma_bench(fma_out, blocks, threads, iters), 5)
    fp64_peak = fl / (t_fma * 1e-3) / 1e12
    # stress shape
    B, P, Hp, Wp, T = 64, 96, 256, 384, 128
    g = synth.stress_geometry(B, P, Hp, Wp, seed=1010)
    pd = dev(g["past_depth"].reshape(B * P, *g["past_depth"].shape[2:]))
    slices = vx.slices_build(pd, dev(g["past_poses"].reshape(B * P, 12)),
                             dev(g["past_intr"].reshape(B * P, 4))).view(B, P, 18)
    cd, cc = dev(g["cur_depth"]), dev(g["cur_cam"])
    counts = vx.block_overlap(cd, cc, slices, 1, T)
    for _ in range(2):
        vx.block_overlap(cd, cc, slices, 1, T, out=counts)
    t_big = time_loop(torch, lambda: vx.block_overlap(cd, cc, slices, 1, T, out=counts), 10)
    points = B * Hp * Wp
    tests = points * P
    flops = tests * OVERLAP_FLOPS_PER_TEST + points * OVERLAP_FLOPS_PER_POINT
    achieved = flops / (t_big * 1e-3) / 1e12
    covered = float((counts.sum(-1) > 0).float().mean().item())

    # the multiwarp (recency-priority splat of the past depth maps into the
    # current view): candidate splats per second at the headline size and with
    # 96 past maps at the stress grid
    def multiwarp_rate(past_depth, poses, intr, cur_cam, n_reps):
        P_, Hp_, Wp_ = past_depth.shape
        pd = dev(past_depth)
        cams = dev(np.stack([synth.camera_record(poses[j], intr[j]) for j in range(P_)]))
        cc = dev(cur_cam)
        ws = vx.depth_multiwarp_workspace(Hp_, Wp_, device)
        cur = torch.empty((Hp_, Wp_), dtype=torch.float32, device=device)
        call = lambda: vx.depth_multiwarp(pd, cams, cc, 0.01, ws=ws, out=cur)
        for _ in range(3):
            call()
        t_ = time_loop(torch, call, n_reps)
        splats = P_ * Hp_ * Wp_
        return {"shape": f"{P_} past maps of {Hp_}x{Wp_}", "ms": round(t_, 4), "candidate_splats": splats,
                "splats_per_s": round(splats / (t_ * 1e-3), 1),
                "holes_fraction": round(float(torch.isnan(cur).float().mean().item()), 4)}

    geo3 = synth.geometry_only(3)
    mw_head = multiwarp_rate(geo3.past_depth[0], geo3.past_poses[0], geo3.past_intr[0],
                             geo3.cur_cam[0], reps)
    g_mw = synth.stress_geometry(1, 96, Hp, Wp, seed=1011, past_grid=(Hp, Wp))
    mw_big = multiwarp_rate(g_mw["past_depth"][0], g_mw["past_poses"][0], g_mw["past_intr"][0],
                            g_mw["cur_cam"][0], 10)
    out = {
        "workload": "slice overlap (step 3 of the method's geometry): headline size and a stress shape",
        "data": "synthetic", "n_gpus": 1,
        "headline": {"shape": "B1, 3x32x48 tokens (T 128), 48 slices", "ms": round(t_small, 4),
                     "point_tests": tests_small,
                     "point_tests_per_s": round(tests_small / (t_small * 1e-3), 1),
                     "note": "one launch, latency-bound; an HBM fraction is meaningless here"},
        "stress": {"shape": f"B{B} scenes, {Hp}x{Wp} (1 frame per chunk, T {T}), {P} slices",
                   "ms": round(t_big, 4), "point_tests": tests,
                   "point_tests_per_s": round(tests / (t_big * 1e-3), 1),
                   "fp64_flops_per_test": OVERLAP_FLOPS_PER_TEST,
                   "achieved_fp64_tflops": round(achieved, 3),
                   "covered_query_block_fraction": round(covered, 4)},
        "roofline": {"bound": "alu", "achieved": round(achieved, 3), "peak": round(fp64_peak, 3),
                     "unit": "TFLOP/s", "frac": round(achieved / fp64_peak, 4),
                     "peak_kind": "measured float64 FMA rate (velox_fp64_fma_bench, FMA = 2 FLOP)",
                     "traffic": None},
        "multiwarp": {"headline": mw_head, "stress": mw_big,
                      "note": "every valid past pixel is a candidate: back-projection, projection and "
                              "64-bit atomic minima on the target pixel (float64 geometry)"},
    }
    print(json.dumps(out), flush=True)


def run_reference(args):
    """The reference arm: the fp64 CPU oracle (the method's pages publish no
    code) on the host cores. Each step is one bounded sample of the workload
    (oracle_sample); the line reports the time a sample really took and the
    whole step extrapolated from it, flagged as such."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return
    cfg = 4 if args.workload == "sweep" else 3
    case = synth.make_case(cfg, seed=1000 + cfg, P=args.P, heads=(0,))
    s = synth.shape_for(cfg, P=args.P)
    case.shape = s
    kf = kept_flops(s)
    for _ in range(args.warmup):
        oracle_sample(case)
    samples = [oracle_sample(case) for _ in range(args.steps)]
    r = {key: statistics.mean(x[key] for x in samples)
         for key in ("geometry_s", "routing_s_per_head", "attention_s_per_query_block",
                     "sample_s", "est_step_s")}
    r["desc"] = samples[0]["desc"]
    r["repeats"] = len(samples)
    r1 = oracle_single_thread(case)
    value = kf / r["est_step_s"] / 1e12
    out = {
        "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(r["sample_s"] * 1e3, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "impl": "reference",
        "extrapolated": True,
        "est_full_step_ms": round(r["est_step_s"] * 1e3, 1),
        "config": {"workload": workload_desc(s), "l2": "n/a (host)",
                   "parallelism": "host cores, rank 0 only",
                   "step": "one bounded sample of the workload per step (ms_per_step is its "
                           "measured time); value is the whole step extrapolated from the "
                           "sample (est_full_step_ms)"},
        "cpu_baseline": baseline_record(kf, r, r1),
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(out), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="velox", choices=["velox", "reference"])
    ap.add_argument("--workload", default="headline",
                    choices=["headline", "sweep", "pipeline", "robustness", "rollout", "overlap"])
    ap.add_argument("--chunks", type=int, default=4, help="chunks (rollout workload)")
    ap.add_argument("--denoise-steps", type=int, default=4, help="steps per chunk (rollout)")
    ap.add_argument("--layers", type=int, default=30, help="layers (pipeline workload)")
    ap.add_argument("--P", type=int, default=None, help="past chunks (sweep workload)")
    ap.add_argument("--T", type=int, default=None, help="block size (sweep workload: 64 or 128)")
    ap.add_argument("--d", type=int, default=None, help="head dim (sweep workload: 64 or 128)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extras", action="store_true",
                    help="leave the sweep and pipeline records out of the default line")
    ap.add_argument("--shard", default="heads", choices=["heads", "chunks"],
                    help="multi-GPU: the heads of one chunk split over the GPUs with an "
                         "all-gather of O every step (default, strong scaling), or one "
                         "independent chunk per GPU with no collective (weak scaling)")
    args = ap.parse_args()
    if args.impl == "reference":
        run_reference(args)
    elif args.workload == "pipeline":
        run_pipeline(args)
    elif args.workload == "robustness":
        run_robustness(args)
    elif args.workload == "rollout":
        run_rollout(args)
    elif args.workload == "overlap":
        run_overlap(args)
    else:
        run_gpu(args)


if __name__ == "__main__":
    main()
