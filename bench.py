#!/usr/bin/env python
"""Benchmark of the fused short-convolution step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step is one pass of the hot path over one batch: the per-token metadata
build (sconv_seq_metadata_ahead, each step having its own metadata buffers)
followed by the fused insert + conv (sconv_fused), on the single-token decode workload (256 requests over
histories of 1..4096 cached tokens, H=32, D=128, stream ws=32 at off_s=32,
C=1024, W=4, N=16, SiLU + residual, bf16).  Inputs are resident in HBM; the
step rotates over enough independent input sets (each touching its own
cache blocks) that the data touched between two visits of one set is
larger than L2.  Steps are replayed from CUDA graphs and timed with CUDA
events; with N GPUs each rank runs its own requests (weak scaling, no
collective on the data path) and the time is the maximum over ranks.

Also reported: the fused kernel's own launch duration against the HBM
roofline, end-to-end throughput through the public API with host buffers
(H2D of the step's inputs, D2H of its output), the other workloads' kernel
throughput, SM clocks sampled during the timed region, and the CPU oracle's
throughput on the host cores (rank 0, N = 1).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import platform
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "fused sconv Mtokens/s and achieved HBM GB/s (% of B200 peak) per config"
UNIT = "Mtokens/s"
HEADLINE = "decode_bf16"
# The headline step: its form (DecodeSets mode) and schedule (see
# run_steps_graphs), the fastest single-layer decode step measured.
STEP_MODE = "taps"
STEP_SCHEDULE = "next"
STEP_KERNEL = {"paged": "fused_token_kernel (sconv_fused at decode sizes)",
               "taps": "fused_taps_next_kernel (sconv_fused_taps_next: this step's "
                       "convolution and the next step's tap table in one launch)"}
STEP_CALLS = {"paged": "sconv_seq_metadata_ahead + sconv_fused",
              "taps": "sconv_fused_taps_next (one launch: this step's convolution and the "
                      "next step's metadata and tap table)"}
L2_BYTES = 126 * 1024 * 1024
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    p = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=192000)
    p.add_argument("--warmup", type=int, default=960)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--sets", type=int, default=96, help="rotating input sets (decode)")
    p.add_argument("--no-extras", action="store_true",
                   help="skip the per-workload table, e2e and the CPU baseline")
    p.add_argument("--seed", type=int, default=1002)
    p.add_argument("--only", choices=["chunked_prefill_bf16", "long_prefill_bf16",
                                      "spec_decode_bf16", "dense", "dense_prefill_bf16",
                                      "dense_long_prefill_bf16", "dense_decode_bf16",
                                      "decode_chain", "chunked_prefill_f32_w4",
                                      "chunked_prefill_bf16_w8", "chunked_prefill_taps"],
                   help="time just this workload's kernels and print its table row")
    p.add_argument("--max-hist", type=int, default=4096,
                   help="longest cached history of the decode requests (smaller only for "
                        "profiling captures; the workload itself uses 4096)")
    return p.parse_args()


# --------------------------------------------------------------------------
# distributed plumbing

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _reduce(value: float, world: int, op_name: str) -> float:
    """All-reduce one float over the ranks (timing and token counts only;
    nothing on the data path is exchanged)."""
    if world == 1:
        return value
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=getattr(dist.ReduceOp, op_name))
    return float(t.item())


def max_over_ranks(value: float, world: int) -> float:
    return _reduce(value, world, "MAX")


def sum_over_ranks(value: float, world: int) -> float:
    return _reduce(value, world, "SUM")


def rank_seed(base: int, rank: int) -> int:
    """Each rank draws its own requests (weak scaling: per-GPU work fixed)."""
    return base + 100003 * rank


# --------------------------------------------------------------------------
# algorithmic bytes (what one launch must move, no re-reads)

def algorithmic_bytes_taps(wl) -> int:
    """Bytes of one sconv_fused_taps launch: as algorithmic_bytes, with the
    per-token metadata being the slot (8 B) and the resolved table row
    (8 B per lag) instead of 24 B of metadata plus block-table entries."""
    e, C, W = wl.elem_bytes, wl.C, wl.W
    live = int((wl.slot_mapping != -1).sum())
    hist_rows = sum(min(W - 1, int(wl.hist[r])) for r in range(wl.R) if wl.new[r] > 0)
    return (wl.T * C * e + 2 * live * C * e + hist_rows * C * e + C * W * e
            + (8 + 8 * (W - 1)) * wl.T)


def algorithmic_bytes_resolve(wl) -> int:
    """Bytes of one step's tap resolution: positions and slots read (16 B
    per token), query_start_loc (4 B per request + 4), the distinct
    block-table entries of the pre-forward taps (4 B each), and seq_idx,
    query_start and the table row written (8 + 8 (W-1) B per token)."""
    W, N = wl.W, wl.N
    bt_entries = 0
    for r in range(wl.R):
        if wl.new[r] == 0:
            continue
        h = int(wl.hist[r])
        rows = min(W - 1, h)
        bt_entries += len({p // N for p in range(h - rows, h)})
    return 16 * wl.T + 4 * (wl.R + 1) + 4 * bt_entries + (8 + 8 * (W - 1)) * wl.T


def algorithmic_bytes(wl) -> int:
    """x rows read + inserts + outputs + the distinct pre-forward cache rows
    of each request (min(W-1, history) rows of C elements) + weights + 24 B
    of per-token metadata + 4 B per distinct block-table entry read."""
    e, C, W, N = wl.elem_bytes, wl.C, wl.W, wl.N
    live = int((wl.slot_mapping != -1).sum())
    hist_rows, bt_entries = 0, 0
    for r in range(wl.R):
        if wl.new[r] == 0:
            continue
        h = int(wl.hist[r])
        rows = min(W - 1, h)
        hist_rows += rows
        bt_entries += len({p // N for p in range(h - rows, h)})
    return (wl.T * C * e + 2 * live * C * e + hist_rows * C * e + C * W * e
            + 24 * wl.T + 4 * bt_entries)


def measured_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            v = float(json.load(f)["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash() -> str:
    """Hash of the sources of the decode step's kernels (fused.cu and the
    headers it includes), to tell whether a committed ncu record is
    current."""
    h = hashlib.sha256()
    for name in ("fused.cu", "fused_common.cuh", "common.cuh", "taps_resolve.cuh"):
        with open(os.path.join(ROOT, "hybrid_sconv_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per launch of the fused kernel from the committed ncu
    record (profiles/fused_sconv_<workload>.json), if it was taken on the
    current kernel source; None otherwise."""
    path = os.path.join(ROOT, "profiles", f"fused_sconv_{workload}.json")
    try:
        with open(path) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("kernel_source_sha256_16") != kernel_source_hash():
        return None
    v = rec.get("traffic_bytes_per_launch")
    return int(v) if v is not None else None


# --------------------------------------------------------------------------
# clocks sampled while the GPU is busy

class ClockSampler:
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")

    def __init__(self, device_index):
        self.proc = None
        self.lines = []
        self.device_index = device_index

    def _gpu_id(self):
        try:
            u = str(torch.cuda.get_device_properties(self.device_index).uuid)
            return u if u.startswith("GPU-") else "GPU-" + u
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            if vis:
                return vis.split(",")[self.device_index]
            return str(self.device_index)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self._gpu_id(), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        self.lines += [ln for ln in out.splitlines() if ln.strip()]

    def samples(self, t0=None, t1=None):
        """Parsed samples, optionally only those stamped within [t0, t1]
        (host wall-clock seconds)."""
        import datetime
        out = []
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                sm, mx = float(parts[2]), float(parts[3])
            except ValueError:
                continue
            if t0 is not None and not (t0 <= ts <= t1):
                continue
            reasons = {n for n, v in zip(self.NAMES, parts[6:10]) if v.lower().startswith("active")}
            out.append((sm, mx, reasons))
        return out

    @staticmethod
    def summary(samples, window):
        if not samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "window": window}
        reasons = set().union(*[r for _, _, r in samples])
        return {"sm_mhz": statistics.median(s for s, _, _ in samples),
                "sm_max_mhz": max(m for _, m, _ in samples), "reasons": sorted(reasons),
                "samples": len(samples), "window": window}


# --------------------------------------------------------------------------
# CUDA-graph helpers

def capture(fn, stream):
    """Capture fn() (which launches on the current stream) into a graph."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        fn()  # eager warm-up on the capture stream (loads the kernels)
    stream.synchronize()
    with torch.cuda.graph(g, stream=stream):
        fn()
    return g


def replay_steps(graphs_full, graph_tail, reps):
    for _ in range(reps):
        graphs_full.replay()
    if graph_tail is not None:
        graph_tail.replay()


# --------------------------------------------------------------------------
# the decode workload: rotating input sets over one shared cache

class DecodeSets:
    """``n`` independent decode batches sharing one weight and one paged
    cache; each has its own requests, histories, block permutation, x,
    metadata buffers (seq_idx, query_start and the resolved tap table) and
    output.

    mode "taps" (the benchmark's step): sconv_seq_metadata_taps(_ahead)
    builds the step's metadata and tap table, sconv_fused_taps convolves.
    mode "paged": sconv_seq_metadata(_ahead), then sconv_fused reading
    positions, request metadata and the block table itself."""

    def __init__(self, n, seed, device, max_hist=4096, ahead=False, mode="taps", min_hist=1):
        # ahead: build each step's metadata with the *_ahead builder, whose
        # precondition holds because every set has its own buffers and a
        # graph replay touches each set once.
        self.ahead = ahead
        self.mode = mode
        self.wls = [workloads.decode_bf16(seed=seed + 7919 * i, max_hist=max_hist,
                                          min_hist=min_hist) for i in range(n)]
        self.device = device
        nb = max(w.num_blocks for w in self.wls)
        w0 = self.wls[0]
        g = torch.Generator(device=device).manual_seed(seed)
        self.weight = workloads.normal((w0.C, w0.W), w0.w_sigma, torch.bfloat16, g, device)
        self.cache = torch.empty((nb, w0.H, w0.N, w0.D), dtype=torch.bfloat16, device=device)
        workloads.fill_normal_(self.cache, 1.0, g, device)
        self.sets = []
        for wl in self.wls:
            md = wl.metadata(device)
            s = {
                "x": workloads.normal((wl.T, wl.C), 1.0, torch.bfloat16, g, device),
                "positions": md["positions"], "slot_mapping": md["slot_mapping"],
                "block_table": md["block_table"], "query_start_loc": md["query_start_loc"],
                "seq_idx": torch.empty(wl.T, dtype=torch.int32, device=device),
                "query_start": torch.empty(wl.T, dtype=torch.int32, device=device),
                "taps": torch.empty((wl.T, wl.W - 1), dtype=torch.int64, device=device),
                "out": torch.empty((wl.T, wl.C), dtype=torch.bfloat16, device=device),
            }
            self.sets.append(s)
        self.alg_bytes = [algorithmic_bytes(wl) for wl in self.wls]
        self.alg_bytes_taps = [algorithmic_bytes_taps(wl) for wl in self.wls]
        # one sconv_fused_taps_next launch: set i's convolution, set i+1's table
        self.alg_bytes_next = [algorithmic_bytes_taps(wl) +
                               algorithmic_bytes_resolve(self.wls[(i + 1) % n])
                               for i, wl in enumerate(self.wls)]

    def step_next(self, i, j):
        """Set i's convolution and set j's tap table in one launch
        (sconv_fused_taps_next; taps mode)."""
        import hybrid_sconv_b200 as hs
        wl, s, wn, sn = self.wls[i], self.sets[i], self.wls[j], self.sets[j]
        hs.sconv_fused_taps_next(
            s["x"], self.weight, self.cache, s["slot_mapping"], s["taps"], out=s["out"],
            next_step=dict(query_start_loc=sn["query_start_loc"], num_reqs=wn.R,
                           num_actual_tokens=wn.T, positions=sn["positions"],
                           slot_mapping=sn["slot_mapping"], block_table=sn["block_table"],
                           seq_idx_out=sn["seq_idx"], query_start_out=sn["query_start"],
                           taps_out=sn["taps"]),
            **wl.kwargs())

    def kernel_alg_bytes(self, schedule=None):
        """Algorithmic bytes of one convolution launch in this mode (with the
        next step's table build for the "next" schedule)."""
        if schedule == "next":
            return self.alg_bytes_next
        return self.alg_bytes_taps if self.mode == "taps" else self.alg_bytes

    def step(self, i, fused=True, metadata=True, ready=False):
        """Metadata build and/or convolution of set i.  ready: the set's
        metadata was complete before the kernel ahead of the convolution on
        its stream began (sconv_fused_taps may then read it before its
        wait)."""
        import hybrid_sconv_b200 as hs
        wl, s = self.wls[i], self.sets[i]
        if metadata:
            if self.mode == "taps":
                build = (hs.sconv_seq_metadata_taps_ahead if self.ahead
                         else hs.sconv_seq_metadata_taps)
                build(s["query_start_loc"], wl.R, wl.T, s["positions"], s["slot_mapping"],
                      s["block_table"], wl.num_blocks, wl.N, wl.W, seq_idx_out=s["seq_idx"],
                      query_start_out=s["query_start"], taps_out=s["taps"])
            else:
                build = hs.sconv_seq_metadata_ahead if self.ahead else hs.sconv_seq_metadata
                build(s["query_start_loc"], wl.R, wl.T, s["seq_idx"], s["query_start"])
        if fused:
            if self.mode == "taps":
                hs.sconv_fused_taps(s["x"], self.weight, self.cache, s["slot_mapping"],
                                    s["taps"], out=s["out"], metadata_ready=ready,
                                    **wl.kwargs())
            else:
                hs.sconv_fused(s["x"], self.weight, self.cache, s["positions"],
                               s["block_table"], s["seq_idx"], s["slot_mapping"],
                               s["query_start"], out=s["out"], **wl.kwargs())


def pipelined_steps(sets_obj, idxs, side, carry=None):
    """Steps idxs in order, each metadata build + convolution over its
    batch, with the next step's metadata built beside the current step's
    convolution, as a serving engine prepares step i+1's inputs while step
    i runs: metadata(i+1) goes to `side` once conv(i-1) has finished (its
    buffers are the next batch's own), and conv(i+1) waits for both
    conv(i) (its cache inserts are the next step's history) and
    metadata(i+1).  carry: the index of the step after idxs; then the first
    step's metadata is taken as already built (by the call before this one)
    and the last build is for step `carry` -- still one build and one
    convolution per step, as in a serving loop's steady state."""
    main = torch.cuda.current_stream()
    side.wait_stream(main)
    meta_done = None
    if carry is None:
        with torch.cuda.stream(side):
            sets_obj.step(idxs[0], fused=False)
        meta_done = torch.cuda.Event()
        meta_done.record(side)
    nxt = list(idxs[1:]) + ([] if carry is None else [carry])
    for j, i in enumerate(idxs):
        if meta_done is not None:
            main.wait_event(meta_done)
        before = torch.cuda.Event()
        before.record(main)  # everything up to conv(i-1)
        # Not ready: under stream capture the event join becomes a
        # programmatic edge, which orders this launch after the builder's
        # trigger, not after its completion.
        sets_obj.step(i, metadata=False)
        if j < len(nxt):
            side.wait_event(before)
            with torch.cuda.stream(side):
                sets_obj.step(nxt[j], fused=False)
            meta_done = torch.cuda.Event()
            meta_done.record(side)
    main.wait_stream(side)


def interleaved_steps(sets_obj, idxs):
    """Steps idxs in order on one stream, each convolution preceded by the
    NEXT step's metadata build (the set's builder; an *_ahead builder looks
    up before its wait, beside the convolution ahead of it): metadata(0),
    metadata(1), conv(0), metadata(2), conv(1), ...  A convolution other
    than the first reads its table before its wait, since the builder of
    that table is two launches back, with the previous convolution between
    them.  Each step still launches both kernels."""
    sets_obj.step(idxs[0], fused=False)
    for j, i in enumerate(idxs):
        if j + 1 < len(idxs):
            sets_obj.step(idxs[j + 1], fused=False)
        sets_obj.step(i, metadata=False, ready=j > 0)


def next_steps(sets_obj, idxs, carry):
    """Steps idxs in order, one launch each: the step's convolution and the
    next step's tap table (sconv_fused_taps_next), the last one building
    step `carry`'s; the first step's table comes from before.  One table
    build and one convolution per step."""
    for i, j in zip(idxs, list(idxs[1:]) + [carry]):
        sets_obj.step_next(i, j)


def run_steps_graphs(sets_obj, K, stream, pipeline=False, carry=False, **step_kw):
    """Graphs that together replay exactly K steps over the rotating sets.
    pipeline: False (metadata then convolution, one stream), "side" (next
    step's metadata on a second stream beside the current convolution) or
    "interleaved" (next step's metadata ahead of the current convolution on
    one stream) or "next" (one sconv_fused_taps_next launch per step, which
    always carries).  carry (with "side"): each graph takes its first step's
    metadata as built by whatever ran before it and builds the metadata of
    the step after its last (see pipelined_steps); carry_prologue() builds
    the first one before the first replay."""
    M = len(sets_obj.sets)
    side = torch.cuda.Stream(stream.device)

    def steps(n):
        if pipeline == "next":
            next_steps(sets_obj, list(range(n)), n % M)
        elif pipeline == "side":
            pipelined_steps(sets_obj, list(range(n)), side, n % M if carry else None)
        elif pipeline == "interleaved":
            interleaved_steps(sets_obj, list(range(n)))
        else:
            for i in range(n):
                sets_obj.step(i, **step_kw)
    full = capture(lambda: steps(M), stream) if K >= M else None
    tail = capture(lambda: steps(K % M), stream) if K % M else None
    return full, tail, K // M


def carry_prologue(sets_obj, stream, i=0):
    """The metadata of set i (0 unless given), built before the first replay
    of carry graphs (the build a previous window of the serving loop would
    have made)."""
    with torch.cuda.stream(stream):
        sets_obj.step(i, fused=False)
    torch.cuda.synchronize()


# Untimed steps at the head of the timed graph: the serving loop's steps
# before the measured window, so the first timed step starts with the
# launch pipeline already running, as every later one does.
LEAD_STEPS = 4
# Up to this many timed steps go into one graph with the lead steps and the
# two event nodes; longer runs replay graphs of one rotation each between
# events on the stream (each graph boundary then costs a launch gap, about
# 1 % of a rotation).
EVENT_GRAPH_MAX_STEPS = 768


class StepEvents:
    """The start and end of a timed window of steps inside one captured
    graph.  start() records an event node on a branch off the step chain,
    after the last untimed step: it is recorded when that step completes,
    while the first timed step follows that step on the chain exactly as
    every step follows its predecessor (its launch and its work before its
    wait may overlap the step before, as in the serving loop).  end()
    joins the branch and records an event node after the last timed step
    completes.  The interval is then K step periods of the running loop,
    with nothing of the graph's own launch in it."""

    def __init__(self, device):
        self.begin = torch.cuda.Event(enable_timing=True, external=True)
        self.finish = torch.cuda.Event(enable_timing=True, external=True)
        self.branch = torch.cuda.Stream(device)

    def start(self):
        self.branch.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(self.branch):
            self.begin.record()

    def end(self):
        torch.cuda.current_stream().wait_stream(self.branch)
        self.finish.record()

    def seconds(self):
        return self.begin.elapsed_time(self.finish) / 1e3


def timed_steps_graph(sets_obj, K, stream, lead=LEAD_STEPS):
    """For the one-launch schedule ("next"): one graph of `lead` untimed
    steps (the sets before set 0 in the rotation), then exactly K timed
    steps (sets 0, 1, ... mod M) between the StepEvents marks.
    carry_prologue(sets_obj, stream, idx) with the returned idx builds the
    first lead step's table before each replay."""
    M = len(sets_obj.sets)
    lead_idx = [(M - lead + i) % M for i in range(lead)]
    timed_idx = [i % M for i in range(K)]
    marks = StepEvents(stream.device)

    def body():
        next_steps(sets_obj, lead_idx, timed_idx[0])
        marks.start()
        next_steps(sets_obj, timed_idx, K % M)
        marks.end()
    return capture(body, stream), marks, lead_idx[0]


class L2Flush:
    """A device buffer larger than L2 (256 MiB), written right before a timed
    region so that no input of the timed steps is still cached from the
    warm-up."""

    def __init__(self, device):
        self.buf = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device=device)

    def __call__(self):
        self.buf.zero_()


# GPU cycles of the spin kernel enqueued before a timed region (about 1 ms at
# the B200's 1.965 GHz): the device stays busy while the host enqueues the
# start event and the graph launches, so the region measures the GPU's work
# and not the host's submission latency.
HOST_LEAD_CYCLES = 2_000_000


class nvtx_range:
    """An NVTX range around a phase of the benchmark (host-side markers for
    a timeline profiler; they add nothing to the device's work)."""

    def __init__(self, name):
        self.name = name

    def __enter__(self):
        torch.cuda.nvtx.range_push(self.name)

    def __exit__(self, *exc):
        torch.cuda.nvtx.range_pop()


def time_region(full, tail, reps, stream, world, sampler=None, flush=None, label="timed"):
    """Seconds for the replays, by CUDA events on the launching stream,
    bracketed by a barrier and a device synchronisation on both sides.
    flush: written on the stream before the start event (L2 cold for the
    timed steps).  A spin kernel precedes the start event so the device does
    not wait for the host's launches inside the region.  With a sampler,
    also returns the host wall-clock span of the region."""
    barrier(world)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if sampler:
        sampler.start()
        time.sleep(1.0)  # nvidia-smi takes a moment before its first reading
    w0 = time.time()
    with torch.cuda.stream(stream), nvtx_range(label):
        if flush is not None:
            flush()
        torch.cuda._sleep(HOST_LEAD_CYCLES)
        start.record()
        replay_steps(full, tail, reps)
        end.record()
    end.synchronize()
    w1 = time.time()
    barrier(world)
    torch.cuda.synchronize()
    if sampler:
        time.sleep(0.3)
        sampler.stop()
    return start.elapsed_time(end) / 1e3, (w0, w1)  # seconds


def time_graph_events(graph, marks, stream, world, sampler=None, flush=None, label="timed"):
    """Seconds between the StepEvents marks of one replay of graph,
    bracketed by a barrier and a device synchronisation on both sides;
    flush and the spin kernel as in time_region.  With a sampler, also
    returns the host wall-clock span of the replay."""
    barrier(world)
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(1.0)
    w0 = time.time()
    with torch.cuda.stream(stream), nvtx_range(label):
        if flush is not None:
            flush()
        torch.cuda._sleep(HOST_LEAD_CYCLES)
        graph.replay()
    torch.cuda.synchronize()
    w1 = time.time()
    barrier(world)
    torch.cuda.synchronize()
    if sampler:
        time.sleep(0.3)
        sampler.stop()
    return marks.seconds(), (w0, w1)


def prime(full, tail, stream):
    """Replay each graph that is about to be timed once, untimed: the first
    replay of a freshly instantiated graph also uploads it."""
    with torch.cuda.stream(stream):
        for g in (full, tail):
            if g is not None:
                g.replay()
    torch.cuda.synchronize()


def l2_statement(sets_obj, K):
    """What the timed region does about L2, computed for this run: which
    sets the K timed steps read and how many bytes one pass over them
    touches."""
    M = len(sets_obj.sets)
    if K <= M:
        touched = sum(sets_obj.alg_bytes[:K])
        lead = (f"; the {LEAD_STEPS} untimed steps ahead of them read other sets"
                if K + LEAD_STEPS <= M and K <= EVENT_GRAPH_MAX_STEPS else "")
        return (f"L2 flushed (256 MiB written) before the timed region; the {K} timed steps "
                f"each read their own input set (none repeats within the region; "
                f"{touched / 1e6:.0f} MB touched in all){lead}")
    touched = sum(sets_obj.alg_bytes)
    verdict = "> 126 MB L2" if touched > L2_BYTES else "NOT above the 126 MB L2"
    return (f"L2 flushed (256 MiB written) before the timed region; the steps rotate over "
            f"{M} input sets, each rotation touching {touched / 1e6:.0f} MB {verdict}")


def step_launch_duration(sets_obj, stream, reps=200):
    """Average duration of one launch of the headline step's kernel: with
    the "next" schedule the step is one launch, so a graph of the full
    rotation of steps (after the prologue) replayed `reps` times; otherwise
    the convolution launches alone (fused_launch_duration)."""
    if STEP_SCHEDULE != "next":
        return fused_launch_duration(sets_obj, stream, reps)
    carry_prologue(sets_obj, stream)
    full, _, _ = run_steps_graphs(sets_obj, len(sets_obj.sets), stream, pipeline="next")
    prime(full, None, stream)
    secs, _ = time_region(full, None, reps, stream, 1)
    del full
    return secs / (reps * len(sets_obj.sets))


def fused_launch_duration(sets_obj, stream, reps=200):
    """Average duration of one fused launch: a graph of the fused launches
    alone (one per rotating set, metadata built beforehand, so complete
    before any of them starts) replayed `reps` times, timed by CUDA events
    on the launching stream, divided by the number of launches."""
    n = len(sets_obj.sets)
    for i in range(n):
        sets_obj.step(i, fused=False)
    torch.cuda.synchronize()
    g = capture(lambda: [sets_obj.step(i, metadata=False, ready=True) for i in range(n)], stream)
    with torch.cuda.stream(stream):  # on the timed stream, finished before timing
        for _ in range(3):
            g.replay()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        s.record()
        for _ in range(reps):
            g.replay()
        e.record()
    e.synchronize()
    del g
    return s.elapsed_time(e) * 1e-3 / (reps * n)


# --------------------------------------------------------------------------
# other workloads: kernel-only throughput

def _kernel_time(step_fns, reps, stream):
    """Mean seconds per call of the launches in step_fns, replayed from one
    CUDA graph and timed with CUDA events on the launching stream."""
    g = capture(lambda: [f() for f in step_fns], stream)
    # Warm-up replays (clocks, caches, lazy module loads) on the timed stream,
    # finished device-wide before the first event: a warm-up left running on
    # another stream would overlap the timed replays and inflate them.
    with torch.cuda.stream(stream):
        for _ in range(3):
            g.replay()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        s.record()
        for _ in range(reps):
            g.replay()
        e.record()
    e.synchronize()
    del g
    return s.elapsed_time(e) * 1e-3 / (reps * len(step_fns))


def _entry(wl, secs, nbytes, peak):
    live = int((wl.slot_mapping != -1).sum())
    gbs = nbytes / secs / 1e9
    return {"kernel_us": round(secs * 1e6, 3), "mtokens_s": round(live / secs / 1e6, 2),
            "alg_bytes": nbytes, "alg_gbs": round(gbs, 1), "frac": round(gbs / peak, 4)}


PREFILL_SHAPES = (("f32_w4", "f32", 4), ("bf16_w8", "bf16", 8))


def prefill_shape_workload(tag, dtype, W):
    """The chunked prefill's requests (seed 1003: 16 requests, cached
    prefixes U{0..2048}, new tokens U{1..2048}) and channel count in another
    dtype or tap count."""
    rng = np.random.default_rng(1003)
    hist = rng.integers(0, 2049, size=16)
    new = rng.integers(1, 2049, size=16)
    return workloads.build(f"chunked_prefill_{tag}", dtype=dtype, H=32, D=128, ws=128,
                           off_s=0, W=W, N=16, hist=hist, new=new, act="silu",
                           residual=False, seed=1003, rng=rng)


def bench_prefill_taps(device, stream, peak, reps=50):
    """The chunked prefill (W 4) and its W 8 shape in the resolved-tap form:
    the step's table built once (sconv_seq_metadata_taps, shared by every
    layer of a step; timed alone too), then sconv_fused_taps with the table
    ready, which runs the TMA-pipelined kernel with the table rows in its
    tiles.  One set each (134 MB of x, larger than L2)."""
    import hybrid_sconv_b200 as hs
    table = {}
    for name, wl in (("chunked_prefill_bf16", workloads.chunked_prefill_bf16()),
                     ("chunked_prefill_bf16_w8", prefill_shape_workload("bf16_w8", "bf16", 8))):
        t = wl.tensors(device)
        out = torch.empty_like(t["x"])
        taps = torch.empty((wl.T, wl.W - 1), dtype=torch.int64, device=device)

        def build():
            hs.sconv_seq_metadata_taps(t["query_start_loc"], wl.R, wl.T, t["positions"],
                                       t["slot_mapping"], t["block_table"], wl.num_blocks,
                                       wl.N, wl.W, taps_out=taps)

        def conv():
            hs.sconv_fused_taps(t["x"], t["weight"], t["cache"], t["slot_mapping"], taps,
                                out=out, metadata_ready=True, **wl.kwargs())
        with torch.cuda.stream(stream):
            build()
        torch.cuda.synchronize()
        table[f"{name}_fused_taps"] = _entry(wl, _kernel_time([conv], reps, stream),
                                             algorithmic_bytes_taps(wl), peak)
        table[f"{name}_seq_metadata_taps"] = {
            "kernel_us": round(_kernel_time([build], reps, stream) * 1e6, 3),
            "alg_bytes": algorithmic_bytes_resolve(wl)}
        del t, out, taps
        torch.cuda.empty_cache()
    return table


def bench_prefill_shapes(device, stream, peak, reps=50, only=None):
    """The chunked prefill's requests and channel count (T = 16 070, C =
    4096) in fp32 with W = 4 and in bf16 with W = 8: the tiled prefill form
    outside the named workloads' dtype and tap count.  only: one tag."""
    import hybrid_sconv_b200 as hs
    table = {}
    for tag, dtype, W in PREFILL_SHAPES:
        if only is not None and tag != only:
            continue
        wl = prefill_shape_workload(tag, dtype, W)
        t = wl.tensors(device)
        out = torch.empty_like(t["x"])

        def f():
            hs.sconv_fused(t["x"], t["weight"], t["cache"], t["positions"], t["block_table"],
                           t["seq_idx"], t["slot_mapping"], t["query_start"], out=out,
                           **wl.kwargs())
        table[wl.name] = _entry(wl, _kernel_time([f], reps, stream), algorithmic_bytes(wl), peak)
        del t, out
        torch.cuda.empty_cache()
    return table


def bench_prefill(name, device, stream, peak, reps=None):
    """One prefill workload (a single set, larger than L2): the fused
    kernel's throughput; for the long prefill also the window extraction
    (48 rotating window sets, 48 x 5.2 MB > L2)."""
    import hybrid_sconv_b200 as hs
    out_table = {}
    wl = workloads.NAMED[name]()
    t = wl.tensors(device)
    out = torch.empty_like(t["x"])

    def f():
        hs.sconv_fused(t["x"], t["weight"], t["cache"], t["positions"], t["block_table"],
                       t["seq_idx"], t["slot_mapping"], t["query_start"], out=out, **wl.kwargs())
    reps = reps or (20 if name.startswith("long") else 100)
    out_table[name] = _entry(wl, _kernel_time([f], reps, stream), algorithmic_bytes(wl), peak)
    if name.startswith("long"):
        e = wl.extra
        rng = np.random.default_rng(wl.seed)
        fns = []
        rc = torch.tensor([e["real_count"]], dtype=torch.int32, device=device)
        for _ in range(48):
            pos = torch.from_numpy(rng.integers(e["d_conv"], wl.T + 1, size=e["max_count"])
                                   .astype(np.int32)).to(device)
            o = torch.empty((e["max_count"], wl.C, e["d_conv"]), dtype=torch.bfloat16,
                            device=device)
            fns.append(lambda pos=pos, o=o: hs.sconv_extract_windows(
                t["x"], pos, rc, o, e["d_conv"]))
        secs = _kernel_time(fns, 50, stream)
        nbytes = 2 * e["real_count"] * e["d_conv"] * wl.C * wl.elem_bytes + 4 + 4 * e["max_count"]
        gbs = nbytes / secs / 1e9
        out_table["extract_windows_long_prefill"] = {
            "kernel_us": round(secs * 1e6, 3), "alg_bytes": nbytes,
            "alg_gbs": round(gbs, 1), "frac": round(gbs / peak, 4)}
        # the same windows read through the block table from the paged cache
        req = torch.zeros(e["max_count"], dtype=torch.int32, device=device)
        pfns = []
        for _ in range(48):
            pos = torch.from_numpy(rng.integers(e["d_conv"], wl.T + 1, size=e["max_count"])
                                   .astype(np.int32)).to(device)
            o = torch.empty((e["max_count"], wl.C, e["d_conv"]), dtype=torch.bfloat16,
                            device=device)
            pfns.append(lambda pos=pos, o=o: hs.sconv_extract_windows_paged(
                t["cache"], t["block_table"], req, pos, rc, o, e["d_conv"], wl.off_s, wl.ws))
        secs = _kernel_time(pfns, 50, stream)
        nbytes += 4 * e["max_count"] + 4 * 2 * e["real_count"]  # requests, block-table entries
        gbs = nbytes / secs / 1e9
        out_table["extract_windows_paged_long_prefill"] = {
            "kernel_us": round(secs * 1e6, 3), "alg_bytes": nbytes,
            "alg_gbs": round(gbs, 1), "frac": round(gbs / peak, 4)}
    del t, out
    torch.cuda.empty_cache()
    return out_table


def bench_spec_decode(device, stream, peak, n_sets=40):
    """Speculative decode: rotating sets (each 7.5 MB, 40 sets > L2) over one
    shared cache; the convolution launch alone, as sconv_fused and as
    sconv_fused_taps on tables built beforehand."""
    import hybrid_sconv_b200 as hs
    wls = [workloads.spec_decode_bf16(seed=1004 + 7919 * i) for i in range(n_sets)]
    nb = max(w.num_blocks for w in wls)
    w0 = wls[0]
    g = torch.Generator(device=device).manual_seed(1004)
    cache = torch.empty((nb, w0.H, w0.N, w0.D), dtype=torch.bfloat16, device=device)
    workloads.fill_normal_(cache, 1.0, g, device)
    weight = workloads.normal((w0.C, w0.W), 0.5, torch.bfloat16, g, device)
    fns, tfns = [], []
    for wl in wls:
        md = wl.metadata(device)
        x = workloads.normal((wl.T, wl.C), 1.0, torch.bfloat16, g, device)
        out = torch.empty_like(x)
        taps = hs.sconv_seq_metadata_taps(md["query_start_loc"], wl.R, wl.T, md["positions"],
                                          md["slot_mapping"], md["block_table"], wl.num_blocks,
                                          wl.N, wl.W)
        fns.append(lambda wl=wl, md=md, x=x, out=out: hs.sconv_fused(
            x, weight, cache, md["positions"], md["block_table"], md["seq_idx"],
            md["slot_mapping"], md["query_start"], out=out, **wl.kwargs()))
        tfns.append(lambda wl=wl, md=md, x=x, out=out, taps=taps: hs.sconv_fused_taps(
            x, weight, cache, md["slot_mapping"], taps, out=out, metadata_ready=True,
            **wl.kwargs()))
    torch.cuda.synchronize()
    res = {}
    secs = _kernel_time(fns, 200, stream)
    res["spec_decode_bf16"] = _entry(w0, secs, int(np.mean([algorithmic_bytes(w) for w in wls])),
                                     peak)
    secs = _kernel_time(tfns, 200, stream)
    res["spec_decode_bf16_fused_taps"] = _entry(
        w0, secs, int(np.mean([algorithmic_bytes_taps(w) for w in wls])), peak)
    del cache, fns, tfns
    torch.cuda.empty_cache()
    return res


def bench_serial_step(sets_obj, stream, peak, reps=200):
    """Decode steps in steady state (a full graph of all rotating sets
    replayed many times): the headline's pipelined step, and for comparison
    the other step shapes.  side: the next step's metadata is built on a
    second stream beside the current convolution (joined by an event);
    interleaved: one stream, the next step's metadata enqueued ahead of the
    current convolution; serial: one stream, metadata then convolution.  taps: sconv_seq_metadata_taps + sconv_fused_taps; paged:
    sconv_seq_metadata + sconv_fused.  With a plain builder each step's
    metadata waits for the previous step's convolution before its lookup;
    with an *_ahead builder the lookup overlaps it and only the completion
    waits."""
    saved = (sets_obj.ahead, sets_obj.mode)
    res = {}
    for key, mode, ahead, pipeline in (
            ("decode_step_pipelined", STEP_MODE, True, STEP_SCHEDULE),
            ("decode_step_taps_next", "taps", True, "next"),
            ("decode_step_taps_side", "taps", True, "side"),
            ("decode_step_taps_interleaved", "taps", True, "interleaved"),
            ("decode_step_serial_taps", "taps", False, False),
            ("decode_step_serial_taps_ahead", "taps", True, False),
            ("decode_step_paged_side", "paged", True, "side"),
            ("decode_step_paged_interleaved", "paged", True, "interleaved"),
            ("decode_step_serial", "paged", False, False),
            ("decode_step_serial_ahead", "paged", True, False),
            ("decode_step_paged_side_plain_metadata", "paged", False, "side")):
        sets_obj.ahead, sets_obj.mode = ahead, mode
        if pipeline == "next":
            carry_prologue(sets_obj, stream)
        full, _, _ = run_steps_graphs(sets_obj, len(sets_obj.sets), stream, pipeline=pipeline)
        prime(full, None, stream)
        secs, _ = time_region(full, None, reps, stream, 1)
        del full
        per = secs / (reps * len(sets_obj.sets))
        names = {("taps", True): "sconv_seq_metadata_taps_ahead",
                 ("taps", False): "sconv_seq_metadata_taps",
                 ("paged", True): "sconv_seq_metadata_ahead",
                 ("paged", False): "sconv_seq_metadata"}
        res[key] = {"step_us": round(per * 1e6, 3),
                    "mtokens_s": round(sets_obj.wls[0].T / per / 1e6, 2),
                    "metadata": ("built by the previous launch (sconv_fused_taps_next)"
                                 if pipeline == "next" else names[(mode, ahead)]),
                    "conv": ("sconv_fused_taps_next" if pipeline == "next" else
                             "sconv_fused_taps" if mode == "taps" else "sconv_fused"),
                    "schedule": pipeline or "serial"}
    sets_obj.ahead, sets_obj.mode = saved
    return res


def bench_metadata_kernels(sets_obj, stream, reps=200):
    """The metadata builders alone, one launch per rotating set back to back:
    sconv_seq_metadata (request index and start) and
    sconv_seq_metadata_taps (the same plus the tap table)."""
    saved = (sets_obj.ahead, sets_obj.mode)
    res = {}
    for key, mode in (("decode_bf16_seq_metadata", "paged"),
                      ("decode_bf16_seq_metadata_taps", "taps")):
        sets_obj.ahead, sets_obj.mode = False, mode
        n = len(sets_obj.sets)
        secs = _kernel_time([lambda i=i: sets_obj.step(i, fused=False) for i in range(n)], reps,
                            stream)
        res[key] = {"kernel_us": round(secs * 1e6, 3)}
    sets_obj.ahead, sets_obj.mode = saved
    return res


def bench_decode_kernels(sets_obj, stream, peak, zero_sets=None):
    """The convolution launch alone (metadata built beforehand), both forms,
    on the decode sets and on a batch of the same shape with no history
    (every token at position 0: no cache taps, so the difference is the
    cost of the cache trip)."""
    res = {}
    for tag, so in (("", sets_obj), ("_zero_history", zero_sets)):
        if so is None:
            continue
        saved = so.mode
        for mode, kernel in (("taps", "fused_taps_kernel"), ("paged", "fused_token_kernel")):
            so.mode = mode
            secs = fused_launch_duration(so, stream)
            nbytes = float(np.mean(so.kernel_alg_bytes()))
            gbs = nbytes / secs / 1e9
            res[f"decode_bf16{tag}_{'fused_taps' if mode == 'taps' else 'fused'}"] = {
                "kernel_us": round(secs * 1e6, 3), "kernel": kernel,
                "mtokens_s": round(so.wls[0].T / secs / 1e6, 2), "alg_bytes": int(nbytes),
                "alg_gbs": round(gbs, 1), "frac": round(gbs / peak, 4)}
        so.mode = saved
    return res


def bench_update(sets_obj, stream, peak, reps=200):
    """The decode workload through sconv_update (token b is request b; no
    metadata build needed): one launch per rotating set."""
    import hybrid_sconv_b200 as hs
    fns = []
    for wl, s in zip(sets_obj.wls, sets_obj.sets):
        fns.append(lambda wl=wl, s=s: hs.sconv_update(
            s["x"], sets_obj.weight, sets_obj.cache, s["positions"], s["block_table"],
            s["slot_mapping"], out=s["out"], **wl.kwargs()))
    secs = _kernel_time(fns, reps, stream)
    nbytes = int(np.mean(sets_obj.alg_bytes)) - 8 * sets_obj.wls[0].T  # no seq_idx / query_start
    return {"decode_bf16_update": _entry(sets_obj.wls[0], secs, nbytes, peak)}


def bench_streams(sets_obj, stream, peak, reps=200):
    """Two conv streams of the decode layer in one launch: the workload's
    stream (lanes 32..63) and a second stream on lanes 0..31, sharing
    tokens, metadata and cache; as sconv_fused_streams and as
    sconv_fused_streams_taps (tables built beforehand)."""
    import hybrid_sconv_b200 as hs
    wl0 = sets_obj.wls[0]
    g = torch.Generator(device=sets_obj.device).manual_seed(7)
    w2 = workloads.normal((wl0.C, wl0.W), 0.5, torch.bfloat16, g, sets_obj.device)
    for i in range(len(sets_obj.sets)):
        sets_obj.step(i, fused=False)     # seq_idx, query_start (and the table in taps mode)
    fns, tfns = [], []
    for wl, s in zip(sets_obj.wls, sets_obj.sets):
        x2 = workloads.normal((wl.T, wl.C), 1.0, torch.bfloat16, g, sets_obj.device)
        o2 = torch.empty_like(x2)
        streams = [dict(x=s["x"], weight=sets_obj.weight, off_s=wl.off_s, ws=wl.ws,
                        activation=wl.act, use_residual=wl.residual, out=s["out"]),
                   dict(x=x2, weight=w2, off_s=0, ws=wl.ws, activation=wl.act,
                        use_residual=wl.residual, out=o2)]
        fns.append(lambda s=s, streams=streams, wl=wl: hs.sconv_fused_streams(
            streams, sets_obj.cache, s["positions"], s["block_table"], s["seq_idx"],
            s["slot_mapping"], s["query_start"], wl.N))
        if sets_obj.mode == "taps":
            tfns.append(lambda s=s, streams=streams, wl=wl: hs.sconv_fused_streams_taps(
                streams, sets_obj.cache, s["slot_mapping"], s["taps"], wl.N,
                metadata_ready=True))
    torch.cuda.synchronize()
    res = {}
    for key, f, nbytes in (("decode_bf16_two_streams", fns,
                            2 * int(np.mean(sets_obj.alg_bytes)) - 24 * wl0.T),
                           ("decode_bf16_two_streams_taps", tfns,
                            2 * int(np.mean(sets_obj.alg_bytes_taps)) - 32 * wl0.T)):
        if not f:
            continue
        secs = _kernel_time(f, reps, stream)
        gbs = nbytes / secs / 1e9
        res[key] = {
            "kernel_us": round(secs * 1e6, 3), "streams": 2,
            "mtokens_s_per_stream": round(wl0.T / secs / 1e6, 2),
            "stream_mtokens_s": round(2 * wl0.T / secs / 1e6, 2), "alg_bytes": nbytes,
            "alg_gbs": round(gbs, 1), "frac": round(gbs / peak, 4)}
    return res


def decode_chain_step(hs, sets_obj, i, layers, pdl, side):
    """One decode step through a stack of layers: the metadata build (the
    set's builder and mode, see DecodeSets), then one convolution per layer
    (its own cache and weight), layer l+1 convolving layer l's output; in
    taps mode every layer reads the step's one table, and a layer other
    than the first reads it before its wait (the layer ahead of it on the
    stream began only after the builder had finished).  pdl: every launch
    on the current stream (programmatic dependent launch between
    neighbours).  Otherwise the layers alternate between the current stream
    and `side`, joined by events, so each launch waits for its predecessor
    to finish."""
    wl, s = sets_obj.wls[i], sets_obj.sets[i]
    main = torch.cuda.current_stream()
    sets_obj.step(i, fused=False)
    x, cur = s["x"], main
    for l, (cache, weight, out) in enumerate(layers):
        target = main if (pdl or l % 2 == 0) else side
        if target is not cur:
            ev = torch.cuda.Event()
            ev.record(cur)
            target.wait_event(ev)
        with torch.cuda.stream(target):
            if sets_obj.mode == "taps":
                hs.sconv_fused_taps(x, weight, cache, s["slot_mapping"], s["taps"], out=out,
                                    metadata_ready=l > 0, **wl.kwargs())
            else:
                hs.sconv_fused(x, weight, cache, s["positions"], s["block_table"],
                               s["seq_idx"], s["slot_mapping"], s["query_start"], out=out,
                               **wl.kwargs())
        cur, x = target, out
    if cur is not main:
        ev = torch.cuda.Event()
        ev.record(cur)
        main.wait_event(ev)


def bench_decode_chain(sets_obj, stream, peak, n_layers=4, reps=50):
    """The decode workload through a stack of n_layers layers (each its own
    4.2 GB cache and weight; layer l+1 convolves layer l's output, the chain
    a model's decode step runs, without the projections between), over the
    96 rotating sets, in both modes (taps: one table per step read by every
    layer; paged: every layer resolves its taps itself).  Timed with every
    launch on one stream (PDL: a launch becomes resident while its
    predecessor runs and prefetches before waiting) and with the layers
    alternating between two streams joined by events (each launch starts
    only when its predecessor has finished)."""
    import hybrid_sconv_b200 as hs
    dev = sets_obj.device
    w0 = sets_obj.wls[0]
    g = torch.Generator(device=dev).manual_seed(4242)
    layers = []
    for l in range(n_layers):
        if l == 0:
            cache, weight = sets_obj.cache, sets_obj.weight
        else:
            cache = torch.empty_like(sets_obj.cache)
            workloads.fill_normal_(cache, 1.0, g, dev)
            weight = workloads.normal((w0.C, w0.W), w0.w_sigma, torch.bfloat16, g, dev)
        layers.append((cache, weight, torch.zeros((w0.T, w0.C), dtype=torch.bfloat16, device=dev)))
    side = torch.cuda.Stream(dev)
    n = len(sets_obj.sets)
    saved = sets_obj.mode
    table = {}
    for mode, key in (("taps", f"decode_chain_{n_layers}_layers"),
                      ("paged", f"decode_chain_{n_layers}_layers_paged")):
        sets_obj.mode = mode
        res = {}
        for kind, pdl in (("pdl", True), ("serialised", False)):
            res[kind] = _kernel_time([lambda i=i: decode_chain_step(hs, sets_obj, i, layers, pdl,
                                                                    side)
                                      for i in range(n)], reps, stream)
        table[key] = {
            "step_us_pdl": round(res["pdl"] * 1e6, 3),
            "step_us_serialised": round(res["serialised"] * 1e6, 3),
            "layer_us_pdl": round(res["pdl"] * 1e6 / n_layers, 3),
            "layer_us_serialised": round(res["serialised"] * 1e6 / n_layers, 3),
            "mtokens_s_layers": round(w0.T * n_layers / res["pdl"] / 1e6, 2),
            "launches_per_step": 1 + n_layers,
            "metadata": ("sconv_seq_metadata_taps" if mode == "taps" else "sconv_seq_metadata")
                        + ("_ahead" if sets_obj.ahead else ""),
            "conv": "sconv_fused_taps" if mode == "taps" else "sconv_fused"}
    sets_obj.mode = saved
    del layers
    torch.cuda.empty_cache()
    return table


def bench_ssm_gather(device, stream, peak, reps=50):
    """Conditional SSM state gather: 256 chunk-scan states of [64, 64, 128]
    fp32 (2 MB rows), 64 slots of which 40 real, 8 rotating index sets over
    4 state tensors (1 GiB of distinct rows > L2)."""
    import hybrid_sconv_b200 as hs
    g = torch.Generator(device=device).manual_seed(11)
    shape, nchunks, max_count, real = (64, 64, 128), 128, 64, 40
    states = [workloads.normal((nchunks,) + shape, 1.0, torch.float32, g, device)
              for _ in range(4)]
    rng = np.random.default_rng(11)
    rc = torch.tensor([real], dtype=torch.int32, device=device)
    fns = []
    for j in range(8):
        idx = torch.from_numpy(rng.integers(0, nchunks, size=max_count)).to(device)
        out = torch.empty((max_count,) + shape, dtype=torch.float32, device=device)
        st = states[j % 4]
        fns.append(lambda st=st, idx=idx, out=out: hs.sconv_scatter_intermediate_ssm(
            st, idx, rc, out))
    secs = _kernel_time(fns, reps, stream)
    nbytes = 2 * real * int(np.prod(shape)) * 4 + 8 * max_count + 4
    gbs = nbytes / secs / 1e9
    del states, fns
    torch.cuda.empty_cache()
    return {"scatter_intermediate_ssm": {
        "kernel_us": round(secs * 1e6, 3), "alg_bytes": nbytes, "alg_gbs": round(gbs, 1),
        "frac": round(gbs / peak, 4)}}


def dense_fwd_bytes(d) -> int:
    """Bytes sconv_causal_conv1d_fwd must move: x read and out written for
    every row of a computed sequence, each computed line read (when the
    sequence starts from it) and written, weights, bias and metadata."""
    T, dim = d["x"].shape
    e = d["x"].element_size()
    L = d["conv_states"].shape[2]
    W = d["weight"].shape[1]
    qsl = d["query_start_loc"].cpu().numpy()
    lines = d["cache_indices"].cpu().numpy()
    init = d["has_initial_state"].cpu().numpy()
    live = lines != d["pad_slot_id"]
    rows = int(((qsl[1:] - qsl[:-1]) * live).sum())
    state = int((live * (1 + init)).sum()) * L * dim * e
    meta = 4 * (len(qsl) + len(lines)) + len(init)
    return 2 * rows * dim * e + state + (W + 1) * dim * e + meta


def bench_dense_prefill(name, device, stream, peak):
    """sconv_causal_conv1d_fwd (causal_conv1d_fwd of the Sglang Mamba ops
    page) in place: the mixed prefill over 2 input sets (2 x 147 MB > L2),
    or the long single-sequence prefill (1 GB)."""
    import hybrid_sconv_b200 as hs
    nsets, reps = (2, 50) if name == "dense_prefill_bf16" else (1, 10)
    sets = [workloads.DENSE_NAMED[name](seed=1011 + 17 * i if name == "dense_prefill_bf16"
                                        else 1012, device=device) for i in range(nsets)]
    fns = [lambda d=d: hs.sconv_causal_conv1d_fwd(
        d["x"], d["weight"], d["bias"], d["conv_states"], d["query_start_loc"],
        d["cache_indices"], d["has_initial_state"], True) for d in sets]
    secs = _kernel_time(fns, reps, stream)
    nbytes = int(np.mean([dense_fwd_bytes(d) for d in sets]))
    rows = int(sets[0]["query_start_loc"][-1])
    gbs = nbytes / secs / 1e9
    del sets, fns
    torch.cuda.empty_cache()
    return {name: {"kernel_us": round(secs * 1e6, 3), "mtokens_s": round(rows / secs / 1e6, 2),
                   "alg_bytes": nbytes, "alg_gbs": round(gbs, 1), "frac": round(gbs / peak, 4)}}


def bench_dense_decode(device, stream, peak, nsets=96, reps=200):
    """sconv_causal_conv1d_update (causal_conv1d_update) in place: 256
    sequences, 96 rotating sets of 256 distinct lines each from a 151 MB
    line pool (> L2)."""
    import hybrid_sconv_b200 as hs
    u0 = workloads.dense_decode_bf16(device=device)
    B, dim = u0["x"].shape
    g = torch.Generator(device=device).manual_seed(1013)
    pool = torch.empty((nsets * B, dim, 3), dtype=torch.bfloat16, device=device)
    workloads.fill_normal_(pool, 1.0, g, device)
    perm = torch.randperm(nsets * B, generator=torch.Generator().manual_seed(1013))
    fns = []
    for i in range(nsets):
        x = workloads.normal((B, dim), 1.0, torch.bfloat16, g, device)
        idx = perm[i * B:(i + 1) * B].to(torch.int32).to(device)
        fns.append(lambda x=x, idx=idx: hs.sconv_causal_conv1d_update(
            x, pool, u0["weight"], u0["bias"], True, None, idx))
    secs = _kernel_time(fns, reps, stream)
    nbytes = 2 * B * dim * 2 + 2 * B * dim * 3 * 2 + 5 * dim * 2 + 4 * B
    gbs = nbytes / secs / 1e9
    del pool, fns
    torch.cuda.empty_cache()
    return {"dense_decode_bf16": {"kernel_us": round(secs * 1e6, 3),
                                  "mtokens_s": round(B / secs / 1e6, 2), "alg_bytes": nbytes,
                                  "alg_gbs": round(gbs, 1), "frac": round(gbs / peak, 4)}}


def bench_dense(device, stream, peak):
    table = {}
    for name in ("dense_prefill_bf16", "dense_long_prefill_bf16"):
        table.update(bench_dense_prefill(name, device, stream, peak))
    table.update(bench_dense_decode(device, stream, peak))
    return table


def per_workload_table(device, stream, peak, sets_obj=None, zero_sets=None):
    table = {}
    if sets_obj is not None:
        table.update(bench_serial_step(sets_obj, stream, peak))
        table.update(bench_decode_kernels(sets_obj, stream, peak, zero_sets))
        table.update(bench_metadata_kernels(sets_obj, stream))
        table.update(bench_update(sets_obj, stream, peak))
        table.update(bench_streams(sets_obj, stream, peak))
        table.update(bench_decode_chain(sets_obj, stream, peak))
    table.update(bench_prefill("chunked_prefill_bf16", device, stream, peak))
    table.update(bench_prefill("long_prefill_bf16", device, stream, peak))
    table.update(bench_prefill_shapes(device, stream, peak))
    table.update(bench_prefill_taps(device, stream, peak))
    table.update(bench_spec_decode(device, stream, peak))
    table.update(bench_ssm_gather(device, stream, peak))
    table.update(bench_dense(device, stream, peak))
    return table


# --------------------------------------------------------------------------
# CPU oracle baseline

def cpu_baseline(sets_obj, seconds=8.0, all_cores_seconds=5.0):
    """The oracle as it stands on the host cores: one core (the contract's
    figure), and every logical core running whole decode steps side by side
    (one thread per core; the oracle's C code runs outside the interpreter
    lock and keeps no global state, so the steps proceed in parallel)."""
    import threading

    import oracle
    wl, s = sets_obj.wls[0], sets_obj.sets[0]
    cache = sets_obj.cache.cpu()
    x, w = s["x"].cpu(), sets_obj.weight.cpu()
    md = wl.metadata("cpu")

    def one_step():
        oracle.fused(dtype=wl.dtype, x=x, weight=w, cache=cache, positions=md["positions"],
                     block_table=md["block_table"], seq_idx=md["seq_idx"],
                     slot_mapping=md["slot_mapping"], query_start=md["query_start"],
                     write_cache=False, **wl.kwargs())

    n, t0 = 0, time.perf_counter()
    while True:
        one_step()
        n += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break

    cores = os.cpu_count() or 1
    counts = [0] * cores
    stop = time.perf_counter() + all_cores_seconds

    def worker(i):
        while time.perf_counter() < stop:
            one_step()
            counts[i] += 1

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(cores)]
    t1 = time.perf_counter()
    for th in threads:
        th.start()
    for th in threads:
        th.join()
    el_all = time.perf_counter() - t1
    return {"value": round(n * wl.T / el / 1e6, 6), "unit": UNIT, "cores": 1,
            "kind": "oracle",
            "sample": f"{n} full decode steps ({wl.T} tokens each, C={wl.C}) on one core, "
                      f"{el:.1f} s",
            "all_cores": {"value": round(sum(counts) * wl.T / el_all / 1e6, 6), "unit": UNIT,
                          "cores": cores,
                          "sample": f"{sum(counts)} full decode steps, one thread per logical "
                                    f"core, {el_all:.1f} s"},
            "host": host_cpu()}


def host_cpu() -> dict:
    """The host's logical CPU count and model name (for the CPU baseline)."""
    model = platform.processor() or "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "model": model}


# --------------------------------------------------------------------------
# e2e: the public API with host buffers

class MappedOut:
    """Pinned host memory mapped into the device's address space
    (cudaHostAlloc with cudaHostAllocMapped), presented with the tensor
    interface the binding reads (data_ptr, shape, stride, dtype, device):
    the fused kernel stores a step's output straight into host memory, so
    the result crosses to the host without a copy-engine transfer.  The
    device address comes from cudaHostGetDevicePointer; both calls' return
    codes are checked and any failure raises before a kernel sees the
    buffer."""

    _rt = None

    @classmethod
    def runtime(cls):
        if cls._rt is None:
            import ctypes
            rt = ctypes.CDLL("libcudart.so.12")  # the runtime torch and libsconv share
            rt.cudaHostAlloc.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.c_size_t,
                                         ctypes.c_uint]
            rt.cudaHostGetDevicePointer.argtypes = [ctypes.POINTER(ctypes.c_void_p),
                                                    ctypes.c_void_p, ctypes.c_uint]
            rt.cudaFreeHost.argtypes = [ctypes.c_void_p]
            cls._rt = rt
        return cls._rt

    def __init__(self, shape, dtype, device):
        import ctypes
        rt = self.runtime()
        self.shape = torch.Size(shape)
        self.dtype = dtype
        self.device = torch.device(device)
        self.nbytes = int(np.prod(shape)) * torch.empty((), dtype=dtype).element_size()
        host = ctypes.c_void_p()
        err = rt.cudaHostAlloc(ctypes.byref(host), self.nbytes, 2)  # cudaHostAllocMapped
        if err != 0:
            raise RuntimeError(f"cudaHostAlloc(mapped) failed: {err}")
        dev = ctypes.c_void_p()
        err = rt.cudaHostGetDevicePointer(ctypes.byref(dev), host, 0)
        if err != 0 or not dev.value:
            rt.cudaFreeHost(host)
            raise RuntimeError(f"cudaHostGetDevicePointer failed: {err}")
        self.host_ptr, self.dev_ptr = host.value, dev.value

    def data_ptr(self):
        return self.dev_ptr

    def dim(self):
        return len(self.shape)

    def stride(self, i=None):
        st = (self.shape[1], 1)
        return st if i is None else st[i]

    def host_view(self):
        """A CPU tensor over the same bytes (valid until free())."""
        import ctypes
        buf = (ctypes.c_uint8 * self.nbytes).from_address(self.host_ptr)
        return torch.frombuffer(buf, dtype=self.dtype).view(self.shape)

    def free(self):
        if self.host_ptr:
            self.runtime().cudaFreeHost(self.host_ptr)
            self.host_ptr = self.dev_ptr = 0


def _packed_inputs(sets_obj, keys):
    """Per set, one pinned host buffer and one device buffer holding all of
    a step's inputs back to back (each 256-byte aligned), and device views
    of them shaped like the originals."""
    packed = []
    for s in sets_obj.sets:
        offs, total = {}, 0
        for k in keys:
            offs[k] = total
            total += (s[k].numel() * s[k].element_size() + 255) // 256 * 256
        host = torch.empty(total, dtype=torch.uint8).pin_memory()
        dev = torch.empty(total, dtype=torch.uint8, device=s["x"].device)
        views = {}
        for k in keys:
            n = s[k].numel() * s[k].element_size()
            host[offs[k]:offs[k] + n].copy_(s[k].reshape(-1).view(torch.uint8).cpu())
            views[k] = dev[offs[k]:offs[k] + n].view(s[k].dtype).view(s[k].shape)
        out_host = torch.empty_like(s["out"], device="cpu").pin_memory()
        packed.append({"host": host, "dev": dev, "views": views, "out_host": out_host,
                       "h2d": sum(s[k].numel() * s[k].element_size() for k in keys)})
    return packed


def e2e(sets_obj, K, stream, world, flush):
    """End to end through the public API with host buffers.  Every step
    copies its inputs (x, positions, slot_mapping, block_table,
    query_start_loc) from pinned host memory to the device, builds the
    metadata (and, in taps mode, the tap table) and runs the fused step,
    whose output lands in host memory: the fused kernel stores it straight
    into mapped pinned host memory (MappedOut), so the copy engine carries
    only the uploads, or, where host memory cannot be mapped, a copy-engine
    download on its own stream follows.  The inputs of a step travel as one
    copy (they sit back to back in one pinned buffer and are used in place
    on the device), since every copy has a fixed cost of microseconds on top
    of its bytes (measured: five copies per step 5.9 Mtok/s, one 9.7).  As a
    serving engine does, uploads and kernels run on their own streams
    (joined by events), so step i+1's upload overlaps step i's kernels;
    each step still moves all of its own bytes."""
    import hybrid_sconv_b200 as hs
    keys = ("x", "positions", "slot_mapping", "block_table", "query_start_loc")
    packed = _packed_inputs(sets_obj, keys)
    h2d = packed[0]["h2d"]
    d2h = packed[0]["out_host"].numel() * packed[0]["out_host"].element_size()
    try:
        mapped = [MappedOut(tuple(s["out"].shape), s["out"].dtype, s["out"].device)
                  for s in sets_obj.sets]
    except (OSError, RuntimeError):
        mapped = None
    up, down = torch.cuda.Stream(), torch.cuda.Stream()

    def kernels(i, out):
        wl, s, v = sets_obj.wls[i], sets_obj.sets[i], packed[i]["views"]
        if sets_obj.mode == "taps":
            hs.sconv_seq_metadata_taps(v["query_start_loc"], wl.R, wl.T, v["positions"],
                                       v["slot_mapping"], v["block_table"], wl.num_blocks,
                                       wl.N, wl.W, seq_idx_out=s["seq_idx"],
                                       query_start_out=s["query_start"], taps_out=s["taps"])
            hs.sconv_fused_taps(v["x"], sets_obj.weight, sets_obj.cache, v["slot_mapping"],
                                s["taps"], out=out, **wl.kwargs())
        else:
            hs.sconv_seq_metadata(v["query_start_loc"], wl.R, wl.T, s["seq_idx"],
                                  s["query_start"])
            hs.sconv_fused(v["x"], sets_obj.weight, sets_obj.cache, v["positions"],
                           v["block_table"], s["seq_idx"], v["slot_mapping"], s["query_start"],
                           out=out, **wl.kwargs())

    if mapped:
        # One step of set 0 into device memory, then the same step into the
        # mapped buffer (a step never reads its own inserts, so the history
        # is the same): the bytes must agree.
        packed[0]["dev"].copy_(packed[0]["host"])
        kernels(0, sets_obj.sets[0]["out"])
        kernels(0, mapped[0])
        torch.cuda.synchronize()
        assert torch.equal(mapped[0].host_view().view(torch.int16),
                           sets_obj.sets[0]["out"].cpu().view(torch.int16)), "mapped output"

    def steps(idxs):
        cur = torch.cuda.current_stream()
        up.wait_stream(cur)
        down.wait_stream(cur)
        for i in idxs:
            s, p = sets_obj.sets[i], packed[i]
            with torch.cuda.stream(up):
                p["dev"].copy_(p["host"], non_blocking=True)
            cur.wait_stream(up)
            kernels(i, mapped[i] if mapped else s["out"])
            if not mapped:
                down.wait_stream(cur)
                with torch.cuda.stream(down):
                    p["out_host"].copy_(s["out"], non_blocking=True)
        cur.wait_stream(up)
        cur.wait_stream(down)

    # As for the headline: up to EVENT_GRAPH_MAX_STEPS, LEAD_STEPS untimed
    # steps and then the K timed steps between two event-record nodes of
    # one graph; beyond, graphs of one rotation replayed between events.
    M = len(sets_obj.sets)
    if K <= EVENT_GRAPH_MAX_STEPS:
        marks = StepEvents(stream.device)

        def body():
            steps([(M - LEAD_STEPS + i) % M for i in range(LEAD_STEPS)])
            marks.start()
            steps([i % M for i in range(K)])
            marks.end()
        graph = capture(body, stream)
        prime(graph, None, stream)
        secs = time_graph_events(graph, marks, stream, world, flush=flush)[0]
        del graph
    else:
        full = capture(lambda: steps(range(M)), stream) if K >= M else None
        tail = capture(lambda: steps(range(K % M)), stream) if K % M else None
        prime(full, tail, stream)
        secs = time_region(full, tail, K // M, stream, world, flush=flush)[0]
        del full, tail
    secs = max_over_ranks(secs, world)
    torch.cuda.synchronize()
    if mapped:
        for m in mapped:
            m.free()
    tokens = sum_over_ranks(float(sets_obj.wls[0].T * K), world)
    return {"value": round(tokens / secs / 1e6, 3), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": K,
            "launch": "cuda_graph; one packed upload per step on its own stream, kernels on "
                      "another",
            "d2h": ("the fused kernel stores the step's output in mapped pinned host memory"
                    if mapped else "copy-engine download on a third stream")}


# --------------------------------------------------------------------------

def config_block(world, l2, K=None):
    block = {"workload": "decode_bf16: 256 single-token requests over cached histories "
                        "U{1..4096}; H=32, D=128, ws=32, off_s=32, C=1024, W=4, N=16; "
                        "SiLU + residual",
            "global_batch": 256 * world, "seq_len": 1,
            "parallelism": f"dp{world}" if world > 1 else "single",
            "step": STEP_CALLS[STEP_MODE],
            "pipelining": "each step is one launch that convolves this step and, in "
                          "extra blocks, builds the next step's metadata and tap table, as "
                          "a serving engine prepares step i+1's inputs while step i runs; "
                          "the convolutions run in order, each waiting for the previous "
                          "one; the timed region holds K convolutions and K table builds "
                          "(the first step's table comes from the step before the region, "
                          "the last build is for the step after it)",
            "metadata": "one metadata buffer set per step, so the *_ahead builder may look "
                        "up before the launch's wait on its predecessors",
            "l2": l2}
    if K is not None:
        block["timing"] = (f"one graph replay: {LEAD_STEPS} untimed steps, then the K timed "
                           "steps; CUDA events recorded by graph nodes when the last untimed "
                           "step and the last timed step complete (device time)"
                           if K <= EVENT_GRAPH_MAX_STEPS and STEP_SCHEDULE == "next" else
                           "graphs of one rotation of steps replayed between CUDA events on "
                           "the launching stream (device time)")
    return block


def main_reference(args, rank, world):
    """The oracle, as it stands, timed on the host cores on the same
    workload and metric.  Exactly K steps; each step is a bounded sample of
    the decode batch (a window of its tokens, the whole batch when the
    budget allows) so the run ends within a few minutes."""
    if rank != 0:
        return
    import oracle
    device = "cuda" if torch.cuda.is_available() else "cpu"
    wl = workloads.decode_bf16(seed=args.seed)
    t = wl.tensors(device)
    cache, x, w = t["cache"].cpu(), t["x"].cpu(), t["weight"].cpu()
    del t
    md = wl.metadata("cpu")

    def run(a, b):
        oracle.fused(dtype=wl.dtype, x=x, weight=w, cache=cache, positions=md["positions"],
                     block_table=md["block_table"], seq_idx=md["seq_idx"],
                     slot_mapping=md["slot_mapping"], query_start=md["query_start"],
                     write_cache=False, t_range=(a, b), **wl.kwargs())
    # cost per token, then the sample size that keeps K steps near 60 s
    t0 = time.perf_counter()
    run(0, wl.T)
    per_token = (time.perf_counter() - t0) / wl.T
    K, W = args.steps, max(3, min(args.warmup, 20))
    n = int(max(1, min(wl.T, 60.0 / (K * per_token))))
    for i in range(W):
        a = (i * n) % wl.T
        run(a, min(wl.T, a + n))
    done, t0 = 0, time.perf_counter()
    for i in range(K):
        a = (i * n) % wl.T
        b = min(wl.T, a + n)
        run(a, b)
        done += b - a
    el = time.perf_counter() - t0
    v = done / el / 1e6
    sample = f"{n} of the {wl.T} tokens of the decode batch per step, {K} steps, one core"
    line = {"impl": "reference", "metric": METRIC, "value": round(v, 6), "unit": UNIT,
            "n_gpus": world, "steps": K, "warmup": W,
            "ms_per_step": round(el / K * 1e3, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config_block(1, "oracle on the host: no GPU cache involved"),
            "cpu_baseline": {"value": round(v, 6), "unit": UNIT, "cores": 1, "kind": "oracle",
                             "sample": sample, "host": host_cpu()},
            "e2e": {"value": round(v, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    rank, world, local = dist_setup(args)
    if args.impl == "reference":
        main_reference(args, rank, world)
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the sconv kernels have no CPU path)")
    import hybrid_sconv_b200  # noqa: F401  (fails loudly if libsconv.so is missing)
    device = torch.device("cuda", local)
    stream = torch.cuda.Stream(device)
    peak, peak_kind = measured_hbm_peak()
    if args.only:
        if args.only == "spec_decode_bf16":
            row = bench_spec_decode(device, stream, peak)
        elif args.only == "dense":
            row = bench_dense(device, stream, peak)
        elif args.only == "decode_chain":
            sets_obj = DecodeSets(args.sets, rank_seed(args.seed, rank), device, args.max_hist)
            row = bench_decode_chain(sets_obj, stream, peak)
        elif args.only == "chunked_prefill_taps":
            row = bench_prefill_taps(device, stream, peak, reps=max(3, args.steps))
        elif args.only in ("chunked_prefill_f32_w4", "chunked_prefill_bf16_w8"):
            row = bench_prefill_shapes(device, stream, peak, reps=max(3, args.steps),
                                       only=args.only[len("chunked_prefill_"):])
        elif args.only == "dense_decode_bf16":
            row = bench_dense_decode(device, stream, peak, nsets=args.sets,
                                     reps=max(3, args.steps))
        elif args.only.startswith("dense"):
            row = bench_dense_prefill(args.only, device, stream, peak)
        else:
            row = bench_prefill(args.only, device, stream, peak, reps=max(3, args.steps))
        print(json.dumps({"only": args.only, "peak_gbs": peak, "table": row}), flush=True)
        return
    K, W = args.steps, max(3, args.warmup)

    sets_obj = DecodeSets(args.sets, rank_seed(args.seed, rank), device, args.max_hist,
                          ahead=True, mode=STEP_MODE)
    flush = L2Flush(device)

    # warm-up, then exactly K timed steps (each step's metadata built during
    # the step before it; set 0's by the prologue for the first replay)
    carry_prologue(sets_obj, stream)
    wfull, wtail, wreps = run_steps_graphs(sets_obj, W, stream, pipeline=STEP_SCHEDULE,
                                           carry=True)
    with torch.cuda.stream(stream), nvtx_range("warm-up"):
        replay_steps(wfull, wtail, wreps)
    torch.cuda.synchronize()
    del wfull, wtail
    sampler = ClockSampler(local) if rank == 0 else None
    if K <= EVENT_GRAPH_MAX_STEPS and STEP_SCHEDULE == "next":
        graph, marks, first = timed_steps_graph(sets_obj, K, stream)
        carry_prologue(sets_obj, stream, first)
        prime(graph, None, stream)
        carry_prologue(sets_obj, stream, first)
        secs, (w0, w1) = time_graph_events(graph, marks, stream, world, sampler, flush,
                                           label=f"timed decode steps (K={K})")
        del graph
    else:
        carry_prologue(sets_obj, stream)
        full, tail, reps = run_steps_graphs(sets_obj, K, stream, pipeline=STEP_SCHEDULE,
                                            carry=True)
        prime(full, tail, stream)
        carry_prologue(sets_obj, stream)
        secs, (w0, w1) = time_region(full, tail, reps, stream, world, sampler, flush,
                                     label=f"timed decode steps (K={K})")
        del full, tail
    secs = max_over_ranks(secs, world)
    clocks = None
    if sampler is not None:
        inside = sampler.samples(w0, w1)
        clocks = ClockSampler.summary(inside, "timed region")
        if len(inside) < 3:
            # The timed region was too short for 100 ms sampling: sample a
            # separate ~2 s replay of the same steps instead.
            load = ClockSampler(local)
            carry_prologue(sets_obj, stream)
            full, _, _ = run_steps_graphs(sets_obj, len(sets_obj.sets), stream,
                                          pipeline=STEP_SCHEDULE, carry=True)
            prime(full, None, stream)
            n = max(1, int(2.0 / max(secs / K * len(sets_obj.sets), 1e-6)))
            _, (l0, l1) = time_region(full, None, n, stream, 1, load)
            clocks = ClockSampler.summary(load.samples(l0, l1),
                                          "2 s replay of the step graphs after the timed region")
            del full
    T = sets_obj.wls[0].T
    tokens = sum_over_ranks(float(T * K), world)
    value = tokens / secs / 1e6
    step_bytes = sum_over_ranks(float(np.mean(sets_obj.alg_bytes)) * K, world)

    # the step kernel's own average launch duration
    avg = step_launch_duration(sets_obj, stream)
    bytes_per_launch = float(np.mean(sets_obj.kernel_alg_bytes(STEP_SCHEDULE)))
    achieved = bytes_per_launch / avg / 1e9
    traffic = profiled_traffic(HEADLINE)

    line = {
        "metric": METRIC, "value": round(value, 3), "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": W, "ms_per_step": round(secs / K * 1e3, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded generator; random-normal x, weight and cache)",
        "config": config_block(world, l2_statement(sets_obj, K) if args.max_hist == 4096
                               else "NOT a benchmark figure: profiling case "
                                    f"(histories up to {args.max_hist} tokens)", K),
        "hbm_gbs": round(step_bytes / secs / 1e9, 1),
        "gpu_launches": (1 if STEP_SCHEDULE == "next" else 2) * K,
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": traffic,
                     "kernel": STEP_KERNEL[STEP_MODE],
                     "alg_bytes_per_launch": int(bytes_per_launch),
                     "launch_us": round(avg * 1e6, 3),
                     "kernel_source_sha256_16": kernel_source_hash(),
                     "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs, copy)"},
    }
    if clocks is not None:
        line["clocks"] = clocks

    if not args.no_extras:
        with nvtx_range("e2e"):
            line["e2e"] = e2e(sets_obj, min(K, 24000), stream, world, flush)
        if rank == 0:
            with nvtx_range("per-configuration table"):
                zero = DecodeSets(args.sets, rank_seed(args.seed, rank) + 1, device, max_hist=0,
                                  min_hist=0)
                line["per_config"] = per_workload_table(device, stream, peak, sets_obj, zero)
                del zero
        if rank == 0 and world == 1:
            with nvtx_range("cpu baseline"):
                line["cpu_baseline"] = cpu_baseline(sets_obj)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
