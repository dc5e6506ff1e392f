#!/usr/bin/env python
"""Benchmark of the fused IPA forward (one JSON line on rank 0).

python bench.py [--gpus N] [--steps K] [--warmup W] [--workload KEY] [--impl fipa|reference]

A step is one full forward (prologue, fused attention core with the feature
epilogue, output projection) over one batch of the workload's synthetic
inputs, resident in HBM, replayed from a captured CUDA graph.  The L2 cache
is flushed (a 256 MB write) between timed steps, outside the timed events.
The default workload is the longest chain of the length-scaling workload
(B=1, N=16384), the largest that the configurations run on one GPU; its line
also carries the whole length sweep (N = 512 ... 32768: time, peak device
memory, fitted time exponent and memory line) under "sweep".  Metric: query-key pairs per second, B*H*N^2 / t (padded
N), summed over all ranks.  With N > 1 GPUs (torchrun) every rank either runs
its own replica of the workload on its own seed (weak scaling; the default for
batched workloads), or, for a single-sample workload, lifts all keys of the
same sample and computes its own contiguous range of query tiles through
fipa_forward_rows (strong scaling; --shard).  No collective on the data path;
the step time is the max over ranks.

--impl reference times the CPU fp64 oracle on the host cores instead (each
step: one sample of the batch, or a block of its query rows for long chains),
same metric and unit.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import re
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "fused IPA fwd query-key pairs/sec (B·H·N²/s), % of B200 BF16 tensor peak"
UNIT = "pairs/s"
DEFAULT_WORKLOAD = "3-16384"
MATH = {"bf16": "fp16 tensor-core products, fp32 accumulate; bf16 inputs",
        "f32": "fp16 tensor-core products of hi/lo splits (every float32 value as 2-3 fp16 parts), fp32 "
               "accumulate, point distances in fp32 on the CUDA cores; float32 inputs"}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    help="0, 1, 2, 4 or 3-<N> (length sweep, N in 512..16384)")
    ap.add_argument("--impl", choices=("fipa", "reference"), default="fipa")
    ap.add_argument("--dtype", choices=("bf16", "f32"), default=None,
                    help="input dtype of the workload (default: the workload's own)")
    ap.add_argument("--n", type=int, default=None,
                    help="residues per sample (default: the workload's own N); the other widths stay")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--shard", choices=("auto", "replicas", "rows"), default="auto",
                    help="N > 1 GPUs: independent replicas (weak scaling) or the query rows of one "
                         "batch split across ranks (strong scaling); auto = rows for a single-sample "
                         "workload, replicas otherwise")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-knn", action="store_true", help="leave the kNN distogram timing out of the bench line")
    ap.add_argument("--no-backward", action="store_true",
                    help="leave the backward pass (training step) out of the bench line")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--sweep", action="store_true",
                    help="length sweep N=512..32768 only: time, peak memory, fitted exponents (JSON lines)")
    ap.add_argument("--no-sweep", action="store_true",
                    help="leave the length sweep out of the bench line (it runs after the timed steps)")
    return ap.parse_args()


def dist_info():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def flops_per_pair(wl) -> int:
    """Algorithmic lifted-contraction flops per (b,h,i,j): 2 Ka + 2 Va."""
    ka = wl.D + 3 * wl.P + wl.R * wl.Cz
    va = wl.Dv + 3 * wl.Q + wl.R * wl.Cz
    return 2 * ka + 2 * va


def bwd_flops_per_pair(wl) -> int:
    """Algorithmic flops of the backward's contractions per (b,h,i,j), counted
    as flash-attention backward passes are: the logits once (2 Ka), dP (2 Va),
    dQhat (2 Ka), dKhat (2 Ka), dVhat (2 Va) = 6 Ka + 4 Va.  The second
    recompute of S and dP (one per side) is not counted."""
    ka = wl.D + 3 * wl.P + wl.R * wl.Cz
    va = wl.Dv + 3 * wl.Q + wl.R * wl.Cz
    return 6 * ka + 4 * va


def pair_counts(wl, inp):
    valid = inp["mask"].sum(axis=1).astype(np.int64)
    return wl.B * wl.H * wl.N * wl.N, int(wl.H * np.sum(valid * valid))


def workload_config(wl, extra=None):
    cfg = {"workload": f"{wl.name} ({workloads_key(wl)})", "B": wl.B, "N": wl.N, "H": wl.H, "D": wl.D,
           "Dv": wl.Dv, "P": wl.P, "Q": wl.Q, "Cz": wl.Cz, "R": wl.R, "Cout": wl.Cout,
           "input_dtype": wl.dtype, "frames": f"{wl.frames} {wl.t_scale}",
           "lengths": "all valid" if wl.len_range is None else f"U{{{wl.len_range[0]}..{wl.len_range[1]}}}"}
    if extra:
        cfg.update(extra)
    return cfg


def workloads_key(wl):
    return f"3-{wl.N}" if wl.index == 3 else str(wl.index)


# ---------------------------------------------------------------- clocks
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits", "-lms", "200",
                 "-i", str(self.dev)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for ln in out.splitlines():
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None,
                "sm_max_mhz": float(max(smax)) if smax else None,
                "samples": len(sm), "reasons": sorted(reasons)}


# ---------------------------------------------------------------- roofline inputs
def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d.get("bf16_tflops"), d.get("bf16_tflops_sustained"), d.get("hbm_gbs"), "measured"
    return 1590.0, 1400.0, 6650.0, "fallback"


# Sources of each timed kernel; a committed ncu summary counts only while its
# recorded hash of these files matches.
KERNEL_SOURCES = {
    "fipa_lift_kernel": ("prologue.cu", "sm100.cuh", "plan.h", "kernels.h"),
    "fipa_core_kernel": ("core.cu", "sm100.cuh", "plan.h", "kernels.h"),
    "fipa_out_proj_kernel": ("epilogue.cu", "sm100.cuh", "plan.h", "kernels.h"),
    "bwd_q_kernel": ("backward.cu", "sm100.cuh", "plan.h", "bwd_plan.h", "kernels.h"),
    "bwd_k_kernel": ("backward.cu", "sm100.cuh", "plan.h", "bwd_plan.h", "kernels.h"),
}


def source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "protein_structure_models_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel: str, wl):
    """DRAM bytes per launch of `kernel` from a committed ncu summary, if it
    was taken on the current source of that kernel for this workload."""
    path = os.path.join(ROOT, "profiles", f"{kernel}-{wl.name}.md")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    m_h = re.search(r"source_sha256_16:\s*([0-9a-f]+)", text)
    m_b = re.search(r"dram_bytes_per_launch:\s*([0-9]+)", text)
    if not m_h or not m_b or m_h.group(1) != source_hash(kernel):
        return None
    return int(m_b.group(1))


def _rup(a, b):
    return (a + b - 1) // b * b


def lifted_widths(wl):
    """Column widths of the lifted fp16 rows the prologue writes (the layout of
    csrc/plan.h): Qhat Kq, key head part KHp, value head part VHp, pair rows Zp."""
    f32 = wl.dtype == "f32"
    nsq, nsv, nz, nqz = (3, 2, 3, 1) if f32 else (1, 1, 1, 2)
    D8, P38, Dv8, Q38, RC8 = _rup(wl.D, 8), _rup(3 * wl.P, 8), _rup(wl.Dv, 8), _rup(3 * wl.Q, 8), _rup(wl.R * wl.Cz, 8)
    KHp = _rup(nsq * D8 + (0 if f32 else 3 * P38), 64)
    Zp = _rup(nz * RC8, 64)
    return {"Kq": KHp + nqz * Zp, "KHp": KHp, "VHp": _rup(nsv * Dv8 + 2 * Q38, 64), "Zp": Zp}


def prologue_bytes(wl) -> int:
    """Bytes the prologue must move: every input it reads once, and the lifted
    rows plus per-row fp32 vectors it writes."""
    es = 4 if wl.dtype == "f32" else 2
    BN, BHN = wl.B * wl.N, wl.B * wl.H * wl.N
    reads = es * (BHN * (2 * wl.D + wl.Dv + 6 * wl.P + 3 * wl.Q) + BN * (12 + 2 * wl.R * wl.Cz)) + BN
    w = lifted_widths(wl)
    writes = 2 * (BHN * (w["Kq"] + w["KHp"] + w["VHp"]) + BN * w["Zp"]) + 32 * BHN
    if wl.dtype == "f32":
        writes += 2 * BHN * 3 * wl.P * 4
    return int(reads + writes)


def live_rows(inp) -> int:
    """Rows with a non-empty neighbourhood (mask_i and some permitted j): the
    rows whose update the projection actually computes."""
    mask = np.asarray(inp["mask"]).astype(bool)
    pm = inp.get("pair_mask")
    if pm is None:
        return int(np.sum(mask & mask.any(axis=1, keepdims=True)))
    permitted = mask[:, :, None] & mask[:, None, :] & np.asarray(pm).astype(bool)
    return int(np.sum(permitted.any(axis=2)))


def out_proj_flops(wl, rows: int) -> int:
    """Algorithmic flops of update = features @ w_out over `rows` rows."""
    F = wl.H * (wl.Dv + 4 * wl.Q + wl.Cz)
    return 2 * rows * F * wl.Cout


# ---------------------------------------------------------------- CPU baseline (oracle)
def cpu_oracle_rate(wl, inp, seconds: float):
    """Time the fp64 oracle on the host cores for about `seconds`.

    Short samples: whole samples of the batch, all query rows.  When one sample
    would take longer than `seconds` (the long chains), seeded query rows of
    sample 0 against all N keys, in blocks of 128, at least 512 rows (each row
    is exact on its own, so the rate carries over to the whole forward).
    Returns (pairs/s in B*H*N^2 units, description of the sample)."""
    import oracle
    rng = np.random.default_rng(wl.seed + 7)
    t0 = time.perf_counter()
    oracle.ipa_forward_dense(workloads.slice_batch(inp, [0]), rows=np.arange(min(16, wl.N)))
    per_row = (time.perf_counter() - t0) / min(16, wl.N)
    if per_row * wl.N <= seconds / 2:
        done, t0 = 0, time.perf_counter()
        while True:
            oracle.ipa_forward_dense(workloads.slice_batch(inp, [done % wl.B]))
            done += 1
            el = time.perf_counter() - t0
            if el >= seconds or done >= 10000:
                break
        return (done * wl.H * wl.N * wl.N / el,
                f"{done} whole sample(s) of the batch, all query rows, fp64 NumPy, {el:.1f} s")
    order = rng.permutation(wl.N)
    one = workloads.slice_batch(inp, [0])
    rows_done, t0 = 0, time.perf_counter()
    while True:
        blk = np.sort(order[rows_done:rows_done + 128])
        oracle.ipa_forward_dense(one, rows=blk)
        rows_done += len(blk)
        el = time.perf_counter() - t0
        if (el >= seconds and rows_done >= min(512, wl.N)) or rows_done >= wl.N:
            break
    full = el * wl.B * wl.N / rows_done
    return (rows_done * wl.H * wl.N / el,
            f"{rows_done} seeded query rows of sample 0 against all {wl.N} keys, fp64 NumPy, {el:.1f} s "
            f"(whole forward extrapolated: {full:.0f} s = {el:.1f} s x {wl.B * wl.N}/{rows_done} rows)")


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max([x.get("num_threads", 1) for x in info] or [1])
    except Exception:
        return len(os.sched_getaffinity(0))


# ---------------------------------------------------------------- GPU arm
def shard_mode(shard: str, wl, world: int) -> str:
    """'rows' (every rank lifts all keys and computes its own query tiles of the
    same inputs) or 'replicas' (every rank runs the whole workload on its own
    seed)."""
    if shard == "auto":
        return "rows" if (wl.B == 1 and world > 1) else "replicas"
    return shard


def row_range(mask, rank: int, world: int):
    """Query rows [r0, r1) of rank `rank` when the 128-row query tiles are split
    into `world` contiguous ranges balanced by valid query rows (mask [B, N])."""
    from protein_structure_models_b200.sharding import TILE, tile_rows, tile_shards
    B, N = mask.shape
    T = (N + TILE - 1) // TILE
    weights = [int(mask[:, t * TILE:(t + 1) * TILE].sum()) for t in range(T)]
    r0, r1 = tile_rows(tile_shards(weights, world)[rank], N)
    if r0 >= r1:
        raise ValueError(f"rank {rank} of {world} gets no query tile (N={N}): use fewer GPUs or --shard replicas")
    return r0, r1


def replica_seed(wl, rank: int) -> int:
    """Seed of rank `rank`'s replica: rank 0 runs the workload's own inputs."""
    return wl.seed + 1000 * rank


def to_device(inp, dtype, dev):
    import torch
    td = torch.bfloat16 if dtype == "bf16" else torch.float32
    out = {}
    for k, v in inp.items():
        if isinstance(v, np.ndarray):
            t = torch.from_numpy(np.ascontiguousarray(v))
            out[k] = t.to(dev) if v.dtype == bool else t.to(device=dev, dtype=td)
        elif v is None:
            out[k] = None
    return out


def run_fipa(args, wl, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    from protein_structure_models_b200 import Fipa
    from protein_structure_models_b200.sharding import max_over_ranks

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    mode = shard_mode(args.shard, wl, world)
    inp = workloads.make_inputs(wl, seed=wl.seed if mode == "rows" else replica_seed(wl, rank))
    rows = row_range(inp["mask"], rank, world) if mode == "rows" else None
    d_in = to_device(inp, wl.dtype, dev)
    h = Fipa(wl.dtype, local_rank)
    dims = wl.dims()
    workspace = torch.empty(h.workspace_size(dims), dtype=torch.uint8, device=dev)
    out = {"update": torch.empty((wl.B, wl.N, wl.Cout), dtype=torch.float32, device=dev),
           "local_points": torch.empty((wl.B, wl.N, wl.H, wl.Q, 3), dtype=torch.float32, device=dev)}
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)     # > 126 MB L2
    stream = torch.cuda.current_stream(dev)

    def forward():
        h.forward(d_in, eps=inp["eps"], workspace=workspace, out=out, stream=stream, rows=rows)

    forward()                               # first call outside capture (one-time host setup)
    torch.cuda.synchronize()

    def capture(stage_timing):
        h.enable_stage_timing(stage_timing)
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(dev)
        cap.wait_stream(stream)
        with torch.cuda.graph(g, stream=cap):
            h.forward(d_in, eps=inp["eps"], workspace=workspace, out=out, stream=cap, rows=rows)
        torch.cuda.synchronize()
        return g

    # the timed step replays one captured forward (a CUDA graph), so host-side
    # submission cost stays out of the device timing; a second capture with
    # the library's per-kernel events gives the stage breakdown, replayed
    # separately so those events stay out of the timed steps
    graph = capture(False)
    sgraph = capture(True)      # holds the handle's events: timing stays on until it is released
    for _ in range(args.warmup):
        flush.zero_()
        graph.replay()
    torch.cuda.synchronize()
    h.sync_status()

    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler(local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.start()
    for k in range(args.steps):
        flush.zero_()                       # outside the timed events
        ev[k][0].record(stream)
        graph.replay()
        ev[k][1].record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    h.sync_status()
    launches = h.kernel_count(dims) * args.steps
    step_ms = sum(a.elapsed_time(b) for a, b in ev) / args.steps
    step_ms_max = max_over_ranks(step_ms, dev)

    # ---- stage breakdown (not part of the timed steps).  Each stage-graph
    # replay is also timed as a whole and clocks are sampled: when the replays
    # run more than 25% away from the timed steps (a clock drop outside the
    # timed region), the stage times are rescaled to the timed step and the
    # factor is reported.
    nb = max(1, min(args.steps, 200))
    stage_sum = {}
    rep_ms = 0.0
    sclocks = ClockSampler(local_rank)
    sclocks.start()
    for _ in range(nb):
        flush.zero_()
        graph.replay()                       # keeps the GPU busy right before the measured replay
        r0, r1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        r0.record(stream)
        sgraph.replay()
        r1.record(stream)
        for name, ms in h.stage_times().items():   # waits for this replay
            stage_sum[name] = stage_sum.get(name, 0.0) + ms
        rep_ms += r0.elapsed_time(r1)
    torch.cuda.synchronize()
    stage_clk = sclocks.stop()
    h.sync_status()
    del graph, sgraph
    h.enable_stage_timing(False)
    stage_scale = step_ms / (rep_ms / nb)
    if abs(stage_scale - 1.0) > 0.25:
        stage_sum = {k: v * stage_scale for k, v in stage_sum.items()}
    else:
        stage_scale = 1.0
    stage_avg = {k: v / nb for k, v in stage_sum.items()}
    stage_check = {"replay_ms": rep_ms / nb, "scale": stage_scale, "clocks": stage_clk}
    core_ms = stage_avg["core"]

    # ---- backward (training step): fipa_backward replayed from a graph, L2
    # flushed between steps; stage breakdown from a second graph with the
    # library's events (not part of the timed steps)
    bwd = None
    if wl.dtype == "bf16" and mode == "replicas" and not args.no_backward:
        from protein_structure_models_b200.fipa import Fipa as _F
        rng = np.random.default_rng(wl.seed + 31)
        d_update = torch.from_numpy(rng.standard_normal((wl.B, wl.N, wl.Cout)).astype(np.float32)).to(dev)
        d_local = torch.from_numpy(rng.standard_normal((wl.B, wl.N, wl.H, wl.Q, 3)).astype(np.float32)).to(dev)
        bws = torch.empty(h.backward_workspace_size(dims), dtype=torch.uint8, device=dev)
        grads = {key: torch.empty(d_in[key].shape, dtype=torch.float32, device=dev) for key in _F.GRAD_KEYS.values()}

        def backward(st):
            h.backward(d_in, d_update, d_local, eps=inp["eps"], workspace=bws, grads=grads, stream=st)

        backward(stream)
        torch.cuda.synchronize()
        h.sync_status()

        def bcapture(stage_timing):
            h.enable_stage_timing(stage_timing)
            g = torch.cuda.CUDAGraph()
            cap = torch.cuda.Stream(dev)
            cap.wait_stream(stream)
            with torch.cuda.graph(g, stream=cap):
                backward(cap)
            torch.cuda.synchronize()
            return g

        def train_step(st):
            h.forward_train(d_in, bws, eps=inp["eps"], out=out, stream=st)
            h.backward(d_in, d_update, d_local, eps=inp["eps"], workspace=bws, grads=grads, stream=st, saved=True)

        def tcapture():
            h.enable_stage_timing(False)
            g = torch.cuda.CUDAGraph()
            cap = torch.cuda.Stream(dev)
            cap.wait_stream(stream)
            with torch.cuda.graph(g, stream=cap):
                train_step(cap)
            torch.cuda.synchronize()
            return g

        train_step(stream)
        torch.cuda.synchronize()
        tgraph = tcapture()
        bgraph = bcapture(False)
        sbgraph = bcapture(True)
        nbs = max(3, min(args.steps, 20))
        for _ in range(max(3, args.warmup)):
            flush.zero_()
            bgraph.replay()
        bev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nbs)]
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        for k in range(nbs):
            flush.zero_()
            bev[k][0].record(stream)
            bgraph.replay()
            bev[k][1].record(stream)
        torch.cuda.synchronize()
        h.sync_status()
        bwd_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in bev) / nbs, dev)
        # the training step without the recompute: forward_train + backward from its state
        for _ in range(3):
            flush.zero_()
            tgraph.replay()
        tev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nbs)]
        torch.cuda.synchronize()
        for k in range(nbs):
            flush.zero_()
            tev[k][0].record(stream)
            tgraph.replay()
            tev[k][1].record(stream)
        torch.cuda.synchronize()
        h.sync_status()
        train_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in tev) / nbs, dev)
        bst = {}
        for _ in range(nbs):
            flush.zero_()
            sbgraph.replay()
            for name, ms in h.backward_stage_times().items():
                bst[name] = bst.get(name, 0.0) + ms
        torch.cuda.synchronize()
        h.sync_status()
        del bgraph, sbgraph, tgraph
        h.enable_stage_timing(False)
        bwd = {"ms": bwd_ms, "train_ms": train_ms, "steps": nbs, "stage_ms": {k: v / nbs for k, v in bst.items()},
               "launches_per_call": 11}
        del bws, grads

    # ---- kNN distogram features of the same structures (k = 20, 39 bins)
    knn = None
    if not args.no_knn:
        from protein_structure_models_b200.fipa import knn_distogram
        kk, nbins = 20, 39
        edges = torch.linspace(3.25, 50.75, nbins - 1, device=dev, dtype=torch.float32)
        kout = {"idx": torch.empty((wl.B, wl.N, kk), dtype=torch.int32, device=dev),
                "dist": torch.empty((wl.B, wl.N, kk), dtype=torch.float32, device=dev),
                "bin": torch.empty((wl.B, wl.N, kk), dtype=torch.int32, device=dev),
                "onehot": torch.empty((wl.B, wl.N, kk, nbins), dtype=torch.float32, device=dev)}
        tr, mk = d_in["translation"], d_in["mask"]
        for _ in range(3):
            knn_distogram(tr, mk, kk, edges, out=kout, stream=stream)
        torch.cuda.synchronize()
        nk = max(3, min(args.steps, 50))
        kev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(nk)]
        for k in range(nk):
            flush.zero_()
            kev[k][0].record(stream)
            knn_distogram(tr, mk, kk, edges, out=kout, stream=stream)
            kev[k][1].record(stream)
        torch.cuda.synchronize()
        knn_ms = sum(a.elapsed_time(b) for a, b in kev) / nk
        knn = {"ms": knn_ms, "k": kk, "n_bins": nbins, "steps": nk,
               "pairs_per_s": wl.B * wl.N * wl.N / (knn_ms / 1e3),
               "how": "fipa_knn_distogram on the workload's translations and mask (indices, distances, bins, "
                      "one-hot [B,N,k,n_bins]); every query scans all keys of its sample, block-wise"}
        del kout

    # ---- end to end through the public API: each step copies its inputs from
    # pinned host memory (one packed buffer), runs the forward and copies the
    # update and local points back (one packed buffer).  Two steps are in
    # flight: step k+1's upload and step k-1's download overlap step k's
    # forward (separate copy streams, two device buffer sets, event-ordered).
    h.enable_stage_timing(False)
    names = [k for k, v in d_in.items() if v is not None]

    def packed_layout(tensors):
        offs, o = {}, 0
        for k, t in tensors.items():
            offs[k] = o
            o = (o + t.numel() * t.element_size() + 255) // 256 * 256
        return offs, o

    in_offs, in_bytes = packed_layout({k: d_in[k] for k in names})
    out_offs, out_bytes = packed_layout(out)
    host_in = torch.empty(in_bytes, dtype=torch.uint8).pin_memory()
    for k in names:
        t = d_in[k].cpu().contiguous().view(torch.uint8).reshape(-1)
        host_in[in_offs[k]:in_offs[k] + t.numel()].copy_(t)
    host_out = [torch.empty(out_bytes, dtype=torch.uint8).pin_memory() for _ in range(2)]

    def views(buf, offs, like):
        return {k: buf[offs[k]:offs[k] + like[k].numel() * like[k].element_size()].view(like[k].dtype)
                .reshape(like[k].shape) for k in offs}

    dbuf_in = [torch.empty(in_bytes, dtype=torch.uint8, device=dev) for _ in range(2)]
    dbuf_out = [torch.empty(out_bytes, dtype=torch.uint8, device=dev) for _ in range(2)]
    dev_in = [dict(views(b, in_offs, {k: d_in[k] for k in names}), pair_mask=None) if "pair_mask" not in names
              else views(b, in_offs, {k: d_in[k] for k in names}) for b in dbuf_in]
    dev_out = [views(b, out_offs, out) for b in dbuf_out]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_fwd = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    h2d, d2h = in_bytes, out_bytes
    e2e_steps = max(2, min(args.e2e_steps, args.steps))

    def e2e_step(k):
        j = k % 2
        if k >= 2:
            s_in.wait_event(ev_fwd[j])          # forward k-2 has read buffer j
        with torch.cuda.stream(s_in):
            dbuf_in[j].copy_(host_in, non_blocking=True)
            ev_in[j].record(s_in)
        stream.wait_event(ev_in[j])
        if k >= 2:
            stream.wait_event(ev_out[j])        # download k-2 has read output j
        h.forward(dev_in[j], eps=inp["eps"], workspace=workspace, out=dev_out[j], stream=stream, rows=rows)
        ev_fwd[j].record(stream)
        s_out.wait_event(ev_fwd[j])
        with torch.cuda.stream(s_out):
            host_out[j].copy_(dbuf_out[j], non_blocking=True)
            ev_out[j].record(s_out)

    for k in range(2):                          # warm-up (first-call host setup)
        e2e_step(k)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for k in range(e2e_steps):
        e2e_step(k)
    s_out.wait_stream(stream)
    e1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, dev)
    h.sync_status()
    h.close()
    return dict(inp=inp, mode=mode, step_ms=step_ms_max, core_ms=core_ms, launches=launches,
                stage_ms=stage_avg, clocks=clk, stage_check=stage_check,
                e2e_ms=e2e_ms, h2d=h2d, d2h=d2h, bwd=bwd, knn=knn)


def kernel_rooflines(wl, stage_ms, valid, fpp, burst, hbm, src, rows):
    """Achieved rate of each timed kernel against its roofline; the time of a
    kernel is its stage's mean CUDA-event time inside the timed steps."""
    lift_s = stage_ms["prologue"] / 1e3
    core_s = stage_ms["core"] / 1e3
    proj_s = stage_ms["out_proj"] / 1e3
    pb, pf, cf = prologue_bytes(wl), out_proj_flops(wl, rows), valid * fpp
    tensor_peak = f"{src} bf16 dense burst, {burst} TFLOP/s (fp16 operands run at the bf16 rate)"
    return {
        "fipa_lift_kernel": {
            "bound": "hbm", "achieved": pb / lift_s / 1e9, "peak": hbm, "unit": "GB/s",
            "frac": pb / lift_s / 1e9 / hbm, "peak_source": f"{src} HBM copy bandwidth",
            "work": f"{pb} bytes per launch (inputs read once + lifted rows written); "
                    f"time = prologue stage (origin + lift kernels)",
            "traffic": profiled_traffic("fipa_lift_kernel", wl)},
        "fipa_core_kernel": {
            "bound": "tensor", "achieved": cf / core_s / 1e12, "peak": burst, "unit": "TFLOP/s",
            "frac": cf / core_s / 1e12 / burst, "peak_source": tensor_peak,
            "frac_of_datasheet_2250": cf / core_s / 1e12 / 2250.0,
            "work": f"{fpp} flop per valid (b,h,i,j) x {valid} valid pairs per launch",
            "traffic": profiled_traffic("fipa_core_kernel", wl)},
        "fipa_out_proj_kernel": {
            "bound": "tensor", "achieved": pf / proj_s / 1e12, "peak": burst, "unit": "TFLOP/s",
            "frac": pf / proj_s / 1e12 / burst, "peak_source": tensor_peak,
            "work": f"2*F*Cout flop x {rows} rows with a non-empty neighbourhood = {pf} per launch; "
                    f"time = out_proj stage",
            "traffic": profiled_traffic("fipa_out_proj_kernel", wl)},
    }


def main_fipa(args, wl):
    rank, world, local_rank = dist_info()
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    r = run_fipa(args, wl, rank, world, local_rank)
    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return
    inp = r["inp"]
    padded, valid = pair_counts(wl, inp)
    fpp = flops_per_pair(wl)
    burst, sustained, hbm, src = measured_peaks()
    # replicas: every rank processed the whole workload; row shards: the ranks
    # together processed it once
    mult = world if r["mode"] == "replicas" else 1
    value = padded * mult / (r["step_ms"] / 1e3)
    kernels = kernel_rooflines(wl, r["stage_ms"], valid, fpp, burst, hbm, src, live_rows(inp))
    stage_of = {"fipa_lift_kernel": "prologue", "fipa_core_kernel": "core", "fipa_out_proj_kernel": "out_proj"}
    dominant = max(kernels, key=lambda k: r["stage_ms"][stage_of[k]])
    roofline = dict(kernels[dominant], kernel=dominant)
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        rate, what = cpu_oracle_rate(wl, inp, args.cpu_seconds)
        cpu = {"value": rate, "unit": UNIT, "cores": blas_threads(), "kind": "oracle", "sample": what}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": r["step_ms"], "higher_is_better": True,
        "scaling": "weak" if r["mode"] == "replicas" else "strong",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": workload_config(wl, {"parallelism": "single GPU" if world == 1 else
                                       (f"replicas x{world}" if r["mode"] == "replicas"
                                        else f"query-row shards x{world}"),
                                       "l2": "flushed (256 MB write) between timed steps",
                                       "math": MATH[wl.dtype]}),
        "valid_pairs_per_s": valid * mult / (r["step_ms"] / 1e3),
        "stage_ms": r["stage_ms"],
        "stage_check": r["stage_check"],
        "roofline": roofline,
        "kernels": kernels,
        "cpu_baseline": cpu,
        "e2e": {"value": padded * mult / (r["e2e_ms"] / 1e3), "unit": UNIT,
                "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"],
                "how": "public binding, pinned packed host buffers, one upload and one download per step, "
                       "two steps in flight (copies overlap the neighbouring forwards)"},
        "gpu_launches": r["launches"],
        "clocks": r["clocks"],
    }
    if r["bwd"] is not None:
        b = r["bwd"]
        bf = bwd_flops_per_pair(wl)
        gemm_ms = b["stage_ms"]["q_side"] + b["stage_ms"]["k_side"]
        ach = bf * valid / (gemm_ms / 1e3) / 1e12
        line["backward"] = {
            "ms": b["ms"], "train_step_ms": b["train_ms"],
            "train_step_recompute_ms": r["step_ms"] + b["ms"],
            "pairs_per_s": padded * mult / (b["ms"] / 1e3),
            "train_step_pairs_per_s": padded * mult / (b["train_ms"] / 1e3),
            "stage_ms": b["stage_ms"], "steps": b["steps"],
            "roofline": {"bound": "tensor", "kernel": "bwd_q_kernel + bwd_k_kernel", "achieved": ach,
                         "peak": burst, "unit": "TFLOP/s", "frac": ach / burst,
                         "work": f"{bf} flop per valid (b,h,i,j) (6 Ka + 4 Va) x {valid} valid pairs; "
                                 f"time = q-side + k-side stages"},
            "how": "ms: fipa_backward (recomputes the lift and the core, then the backward kernels); "
                   "train_step_ms: fipa_forward_train + fipa_backward_saved (no recompute); "
                   "train_step_recompute_ms: forward + fipa_backward; each replayed from a CUDA graph, "
                   "L2 flushed between steps; cotangents N(0,1)"}
    if r["knn"] is not None:
        line["knn_distogram"] = r["knn"]
    if world == 1 and wl.index == 3 and not args.no_sweep:
        line["sweep"] = run_sweep(args.warmup)
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ---------------------------------------------------------------- reference arm (oracle)
def main_reference(args, wl):
    """The fp64 oracle on the host cores, same metric and unit.  Each step is one
    sample of the batch, or, when K whole samples would take more than about two
    minutes, a block of that sample's query rows against all keys (every output
    row is exact on its own); the block size comes from the time of a small row
    block in warm-up."""
    rank, world, _ = dist_info()
    if rank != 0:
        return
    import oracle
    inp = workloads.make_inputs(wl)
    probe = np.arange(min(16, wl.N))
    oracle.ipa_forward_dense(workloads.slice_batch(inp, [0]), rows=probe)      # library start-up
    t_row = []
    for k in range(max(1, args.warmup)):
        t0 = time.perf_counter()
        oracle.ipa_forward_dense(workloads.slice_batch(inp, [k % wl.B]), rows=probe)
        t_row.append((time.perf_counter() - t0) / len(probe))
        if sum(t_row) * len(probe) > 20.0:
            break
    per_sample = float(np.median(t_row)) * wl.N
    budget = 120.0
    nrows = wl.N if args.steps * per_sample <= budget else max(1, int(wl.N * budget / (args.steps * per_sample)))
    t0 = time.perf_counter()
    for k in range(args.steps):
        b = k % wl.B
        r0 = (k * nrows) % wl.N
        rows = None if nrows == wl.N else [(r0 + r) % wl.N for r in range(nrows)]
        oracle.ipa_forward_dense(workloads.slice_batch(inp, [b]), rows=rows)
    el = time.perf_counter() - t0
    value = args.steps * wl.H * nrows * wl.N / el
    what = "one sample (B=1 slice), all query rows" if nrows == wl.N else \
        f"{nrows} query rows of one sample (B=1 slice) against all N keys"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": workload_config(wl, {"step": what}),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": f"{args.steps} steps x {what}, fp64 NumPy oracle, {el:.1f} s"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def fit_loglog(ns, ts):
    """Least-squares exponent of log t against log N with its 95% confidence
    interval (Student t, n - 2 degrees of freedom)."""
    from scipy import stats
    x, y = np.log(np.asarray(ns, float)), np.log(np.asarray(ts, float))
    n = len(x)
    A = np.vstack([x, np.ones(n)]).T
    (slope, icpt), *_ = np.linalg.lstsq(A, y, rcond=None)
    resid = y - (slope * x + icpt)
    dof = n - 2
    se = float(np.sqrt(resid @ resid / dof / np.sum((x - x.mean()) ** 2))) if dof > 0 else float("nan")
    half = float(stats.t.ppf(0.975, dof)) * se if dof > 0 else float("nan")
    return {"exponent": float(slope), "ci95": [float(slope - half), float(slope + half)], "points": n}


def fit_linear(ns, ys):
    """Least-squares line y = a N + c and its R^2."""
    x, y = np.asarray(ns, float), np.asarray(ys, float)
    a, c = np.polyfit(x, y, 1)
    pred = a * x + c
    ss = float(np.sum((y - y.mean()) ** 2))
    r2 = 1.0 - float(np.sum((y - pred) ** 2)) / ss if ss > 0 else 1.0
    return {"bytes_per_residue": float(a), "intercept_bytes": float(c), "r2": r2}


def run_sweep(warmup: int, emit=None) -> dict:
    """Length sweep (the length-scaling workload, N = 512 ... 16384, plus the
    32768 chain): per N the graph-timed forward (L2 flushed between steps) and
    the peak device bytes held by inputs, outputs and workspace (torch's peak
    counter, reset before they are allocated); then the least-squares exponent
    of time vs N (all N, and N >= 2048) and the line of memory vs N.  `emit`,
    if given, receives one dict per N."""
    import torch
    from protein_structure_models_b200 import Fipa
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    ns, ts, mems, wss = [], [], [], []
    for N in workloads.SWEEP_N + workloads.LONG_N:
        wl = workloads.workload(f"3-{N}")
        inp = workloads.make_inputs(wl)
        torch.cuda.synchronize()
        torch.cuda.reset_peak_memory_stats(dev)
        base = torch.cuda.memory_allocated(dev)
        d_in = to_device(inp, wl.dtype, dev)
        h = Fipa(wl.dtype, 0)
        ws = torch.empty(h.workspace_size(wl.dims()), dtype=torch.uint8, device=dev)
        out = {"update": torch.empty((wl.B, wl.N, wl.Cout), dtype=torch.float32, device=dev),
               "local_points": torch.empty((wl.B, wl.N, wl.H, wl.Q, 3), dtype=torch.float32, device=dev)}
        stream = torch.cuda.current_stream(dev)
        h.forward(d_in, eps=inp["eps"], workspace=ws, out=out, stream=stream)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(dev)
        cap.wait_stream(stream)
        with torch.cuda.graph(graph, stream=cap):
            h.forward(d_in, eps=inp["eps"], workspace=ws, out=out, stream=cap)
        torch.cuda.synchronize()
        steps = max(5, min(200, int(2000 * 512 * 512 / N ** 2)))
        for _ in range(max(3, warmup)):
            flush.zero_()
            graph.replay()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
        for k in range(steps):
            flush.zero_()
            ev[k][0].record(stream)
            graph.replay()
            ev[k][1].record(stream)
        torch.cuda.synchronize()
        h.sync_status()
        ms = float(np.median([a.elapsed_time(b) for a, b in ev]))
        peak = torch.cuda.max_memory_allocated(dev) - base
        del graph
        h.close()
        ns.append(N); ts.append(ms); mems.append(int(peak)); wss.append(int(ws.numel()))
        if emit is not None:
            emit({"sweep": "length", "N": N, "ms_per_forward": ms, "steps": steps,
                  "pairs_per_s": wl.B * wl.H * N * N / (ms / 1e3), "peak_device_bytes": int(peak),
                  "workspace_bytes": int(ws.numel())})
        del d_in, ws, out
        torch.cuda.empty_cache()
    big = [i for i, n in enumerate(ns) if n >= 2048]
    return {"N": ns, "ms_per_forward": ts, "peak_device_bytes": mems, "workspace_bytes": wss,
            "fit_time_all": fit_loglog(ns, ts),
            "fit_time_N_ge_2048": fit_loglog([ns[i] for i in big], [ts[i] for i in big]),
            "fit_memory": fit_linear(ns, mems),
            "how": "graph-replayed forward per N, median of CUDA-event steps, L2 flushed between steps; "
                   "peak = torch max_memory_allocated of inputs + outputs + workspace"}


def main_sweep(args):
    """--sweep: one JSON line per N, then one with the fits."""
    res = run_sweep(args.warmup, emit=lambda d: print(json.dumps(d), flush=True))
    print(json.dumps({"sweep": "length", "fit_time_all": res["fit_time_all"],
                      "fit_time_N_ge_2048": res["fit_time_N_ge_2048"],
                      "fit_memory": res["fit_memory"]}), flush=True)


def main():
    args = parse_args()
    if args.sweep:
        main_sweep(args)
        return
    wl = workloads.workload(args.workload)
    if args.dtype is not None:
        wl = wl.with_(dtype=args.dtype)
    if args.n is not None:
        wl = wl.with_(N=args.n, name=f"{wl.name}-N{args.n}")
    if args.impl == "reference":
        main_reference(args, wl)
    else:
        main_fipa(args, wl)


if __name__ == "__main__":
    main()
