#!/usr/bin/env python
"""Benchmark of Re-ttention's attention path on B200.

One step is one pass of the whole hot path on one batch of synthetic input:
the capture step at t0 (block mask from Q0/K0, then full attention with the
statistics cache) followed by the sparse step at t1 (kept blocks only, with
the reshape) on drifted Q1/K1/V1 -- the video-DiT 5B workload's "one sparse
step after a full-capture step".

The headline metric is the sparse step: its device time, its dense-equivalent
TFLOP/s (4*B*H*N^2*d over the sparse-step time) and the tensor-pipe share of
the bf16 peak on the flops it executes.  ``value`` is the dense-equivalent
TFLOP/s of the sparse step summed over all ranks (each rank runs one replica;
weak scaling).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import json
import os
import statistics
import subprocess
import sys
import time
from fractions import Fraction

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from ultra_sparse_attention_b200.workloads import WORKLOADS, denoising_inputs  # noqa: E402

METRIC = "sparse-step ms & dense-equiv TFLOP/s; tensor-pipe % of BF16 peak (1xB200)"
UNIT = "TFLOP/s (dense-equivalent, sparse step)"
# Kernels the library launches per step: block pooling and score/select (mask),
# pairing candidates and matching (tile pairing), max |v| per head, the scaled
# f16 copy of V and the capture kernel (capture), the sparse kernel.
LAUNCHES_PER_STEP = 8
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    p = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=60)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=("ours", "reference"), default="ours")
    p.add_argument("--workload", default="video5b", choices=sorted(WORKLOADS))
    p.add_argument("--keep", default=None, help="keep ratio as a fraction, e.g. 1/32 (default: the workload's)")
    p.add_argument("--heads", type=int, default=None,
                   help="override the workload's head count (small profiling cases of the same kernels)")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--cpu-rows", type=int, default=4096, help="rows in the oracle's bounded sample")
    p.add_argument("--no-sweep", action="store_true", help="skip the per-workload sweep (single-GPU runs only)")
    p.add_argument("--sweep-steps", type=int, default=10)
    p.add_argument("--sweep-warmup", type=int, default=3)
    return p.parse_args()


# --------------------------------------------------------------------------- plumbing
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {k: float(p[k]) for k in FALLBACK_PEAKS}, "measured"
    except (OSError, KeyError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled while the timed region runs."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, period_ms: int = 50):
        self.proc = None
        self.gpu = gpu_index
        self.period = period_ms

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", str(self.period)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


def stored_traffic(kernel: str, workload: str):
    """dram bytes per launch from the committed ncu summary, if it matches the current sources."""
    from ultra_sparse_attention_b200 import build as _b
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return None
    cur = _b.source_hash()
    for ln in lines:
        if ln.startswith("#") or "=" not in ln:
            continue
        kv = dict(x.split("=", 1) for x in ln.split())
        if kv.get("kernel") == kernel and kv.get("workload") == workload and kv.get("src_hash") == cur:
            return float(kv["dram_bytes_per_launch"])
    return None


def max_over_ranks(values, device, world: int):
    """Element-wise max of per-rank timings (every rank takes part; no-op at world 1)."""
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    if world > 1:
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


def job_throughput(units_per_rank: float, world: int, slowest_ms: float) -> float:
    """Whole-job TFLOP/s: the units of all ranks over the slowest rank's time."""
    return world * units_per_rank / (slowest_ms / 1e3) / 1e12


# --------------------------------------------------------------------------- work accounting
def kept_work(row_ptr: np.ndarray, col_idx: np.ndarray, N: int, bs: int, bh: int):
    """Executed sparse-step flop factor: sum over query blocks of rows(qb) * kept key columns."""
    nb = -(-N // bs)
    sizes = np.minimum(bs, N - np.arange(nb) * bs).astype(np.int64)
    total = 0
    for r in range(bh * nb):
        kept = col_idx[row_ptr[r]:row_ptr[r + 1]]
        total += int(sizes[r % nb]) * int(sizes[kept].sum())
    return total


def key_tiles_per_query_tile(row_ptr: np.ndarray, col_idx: np.ndarray, tiles: np.ndarray | None, nb: int, bs: int,
                             bh: int, N: int) -> float:
    """Mean key-tile steps of the sparse kernel per 128-row query tile: the union of the
    kept blocks of the tile's query blocks (neighbouring blocks when `tiles` is None)."""
    n_tiles = -(-N // 128)
    if tiles is None:
        per = 128 // bs
        tiles = np.full((bh, n_tiles, 2), -1, np.int64)
        for t in range(n_tiles):
            for h in range(per):
                if t * per + h < nb:
                    tiles[:, t, h] = t * per + h
    total = 0
    for b in range(bh):
        for t in range(n_tiles):
            u = set()
            for qb in tiles[b, t]:
                if 0 <= qb < nb:
                    u.update(col_idx[row_ptr[b * nb + qb]:row_ptr[b * nb + qb + 1]].tolist())
            total += len(u) * (bs // 64)
    return total / (bh * n_tiles)


def workload_numbers(w, keep: int, row_ptr, col_idx):
    B, H, N, d, D = w.batch, w.heads, w.seq_len, w.head_dim, w.head_dim_padded
    bh = B * H
    dense = 4.0 * bh * N * N * d
    executed = 4.0 * d * kept_work(row_ptr, col_idx, N, w.block_size, bh)
    sparse_bytes = bh * N * (D * 2 * 2 + D * 4 + 12) + 2 * bh * N * D * 2  # Q, O, U, stats; K and V once
    sparse_bytes_c = bh * N * (D * 2 * 2 + D * 2 + 16) + 2 * bh * N * D * 2  # the same with f16 U and its row scale
    capture_bytes = 3 * bh * N * D * 2 + bh * N * (D * 2 + D * 4 + 12)     # Q, K, V; O, U, stats
    mask_bytes = 2 * bh * N * D * 2                                       # Q and K read once
    return {"dense_flops": dense, "executed_flops": executed, "sparse_bytes": sparse_bytes,
            "sparse_bytes_compressed": sparse_bytes_c,
            "capture_bytes": capture_bytes, "mask_bytes": mask_bytes}


# --------------------------------------------------------------------------- our arm
def run_ours(args, rank, world, local):
    import ultra_sparse_attention_b200 as usa

    w = WORKLOADS[args.workload]
    if args.heads:
        w = dataclasses.replace(w, heads=args.heads)
    keep_ratio = Fraction(args.keep) if args.keep else w.keep[0]
    keep = w.keep_blocks(keep_ratio)
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    usa.load_library()
    steps = list(denoising_inputs(w, 2))
    host0, host1 = steps[0][1:], steps[1][1:]
    q0, k0, v0 = (x.to(device) for x in host0)
    q1, k1, v1 = (x.to(device) for x in host1)
    kw = dict(head_dim=w.head_dim, block_size=w.block_size, scale=w.scale)
    B, H, N, D = q0.shape
    nb = w.n_blocks
    row_ptr = torch.empty(B * H * nb + 1, dtype=torch.int32, device=device)
    col_idx = torch.empty(B * H * nb * keep, dtype=torch.int32, device=device)
    out0, out1 = torch.empty_like(q0), torch.empty_like(q1)
    stats = usa.Stats(torch.empty(B, H, N, device=device), torch.empty(B, H, N, device=device),
                      torch.empty(B, H, N, device=device), torch.empty(B, H, N, D, device=device))
    tiles = torch.empty(B * H, -(-N // 128), 2, dtype=torch.int32, device=device)
    stream = torch.cuda.current_stream(device)
    ev = {k: [torch.cuda.Event(enable_timing=True) for _ in range(2)] for k in ("mask", "pair", "capture", "sparse")}
    times = {k: [] for k in ev}

    def step(record: bool):
        def mark(name, i):
            if record:
                ev[name][i].record(stream)
        mark("mask", 0)
        usa.rt_build_block_mask(q0, k0, keep_blocks=keep, forced_prefix_tokens=w.forced_prefix_tokens,
                                row_ptr=row_ptr, col_idx=col_idx, **kw)
        mark("mask", 1)
        mark("pair", 0)
        usa.rt_pair_query_blocks(q0, row_ptr, col_idx, head_dim=w.head_dim, block_size=w.block_size, tile_blocks=tiles)
        mark("pair", 1)
        mark("capture", 0)
        usa.rt_attn_full_capture(q0, k0, v0, row_ptr=row_ptr, col_idx=col_idx, out=out0, stats=stats, **kw)
        mark("capture", 1)
        mark("sparse", 0)
        usa.rt_attn_sparse_reshape(q1, k1, v1, row_ptr=row_ptr, col_idx=col_idx, stats=stats, tile_blocks=tiles,
                                   out=out1, **kw)
        mark("sparse", 1)

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    for _ in range(args.warmup):
        step(False)
    torch.cuda.synchronize()
    if usa.rt_take_device_error() != 0:
        raise RuntimeError("a kernel reported a device error during warm-up")

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize()
    t_start.record(stream)
    for _ in range(args.steps):
        step(True)
        # per-kernel durations are read after the loop; keep the events of every step
        for k in ev:
            times[k].append((ev[k][0], ev[k][1]))
            ev[k] = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
    t_end.record(stream)
    torch.cuda.synchronize()
    barrier()
    clk = clocks.stop()
    total_ms = t_start.elapsed_time(t_end)
    per_kernel = {k: statistics.mean(a.elapsed_time(b) for a, b in times[k]) for k in times}
    if usa.rt_take_device_error() != 0:
        raise RuntimeError("a kernel reported a device error in the timed region")

    # The sparse step reading the compressed residual cache (f16 U with a per-row scale),
    # timed on its own after the main loop: the same launch on the same inputs.
    _, stats_c = usa.rt_attn_full_capture(q0, k0, v0, row_ptr=row_ptr, col_idx=col_idx, compressed=True, **kw)
    out1c = torch.empty_like(q1)
    for _ in range(args.warmup):
        usa.rt_attn_sparse_reshape(q1, k1, v1, row_ptr=row_ptr, col_idx=col_idx, stats=stats_c, tile_blocks=tiles,
                                   out=out1c, **kw)
    ev_c = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize()
    for a, b in ev_c:
        a.record(stream)
        usa.rt_attn_sparse_reshape(q1, k1, v1, row_ptr=row_ptr, col_idx=col_idx, stats=stats_c, tile_blocks=tiles,
                                   out=out1c, **kw)
        b.record(stream)
    torch.cuda.synchronize()
    barrier()
    sparse_c_ms = statistics.mean(a.elapsed_time(b) for a, b in ev_c)
    if usa.rt_take_device_error() != 0:
        raise RuntimeError("a kernel reported a device error in the compressed-cache loop")
    del stats_c, out1c

    rp, ci = row_ptr.cpu().numpy(), col_idx.cpu().numpy()
    nums = workload_numbers(w, keep, rp, ci)
    nums["key_tiles_per_query_tile"] = key_tiles_per_query_tile(rp, ci, tiles.cpu().numpy(), nb, w.block_size, B * H, N)
    nums["key_tiles_per_query_tile_neighbours"] = key_tiles_per_query_tile(rp, ci, None, nb, w.block_size, B * H, N)

    # e2e: the sparse step through the public API with host buffers (pinned), copies inside the
    # timed region.  Steps are pipelined as a server would run them: step k+1's host-to-device
    # copy (its own stream, double-buffered inputs) overlaps step k's kernel and step k's
    # device-to-host copy (a third stream); every step's copies and kernel lie between the first
    # copy and the last read-back.
    e2e = None
    if not args.no_e2e:
        h_in = [x.pin_memory() for x in host1]
        h_out = [torch.empty(out1.shape, dtype=out1.dtype, pin_memory=True) for _ in range(2)]
        d_in = [[torch.empty_like(x, device=device) for x in host1] for _ in range(2)]
        d_out = [torch.empty_like(out1) for _ in range(2)]
        s_h2d, s_d2h = torch.cuda.Stream(device), torch.cuda.Stream(device)
        ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs of slot b landed
        ev_used = [torch.cuda.Event() for _ in range(2)]   # the kernel of slot b is done
        ev_out = [torch.cuda.Event() for _ in range(2)]    # the read-back of slot b is done
        n_total = args.warmup + args.steps
        e_start = torch.cuda.Event(enable_timing=True)
        e_end = torch.cuda.Event(enable_timing=True)
        for it in range(n_total):
            b = it % 2
            if it == args.warmup:
                barrier()
                torch.cuda.synchronize()
                e_start.record(s_h2d)
            with torch.cuda.stream(s_h2d):
                if it >= 2:
                    s_h2d.wait_event(ev_used[b])
                for dx, hx in zip(d_in[b], h_in):
                    dx.copy_(hx, non_blocking=True)
                ev_in[b].record(s_h2d)
            stream.wait_event(ev_in[b])
            if it >= 2:
                stream.wait_event(ev_out[b])
            usa.rt_attn_sparse_reshape(*d_in[b], row_ptr=row_ptr, col_idx=col_idx, stats=stats, tile_blocks=tiles,
                                       out=d_out[b], **kw)
            ev_used[b].record(stream)
            with torch.cuda.stream(s_d2h):
                s_d2h.wait_event(ev_used[b])
                h_out[b].copy_(d_out[b], non_blocking=True)
                ev_out[b].record(s_d2h)
        stream.wait_stream(s_h2d)
        stream.wait_stream(s_d2h)
        e_end.record(stream)
        torch.cuda.synchronize()
        barrier()
        e2e_ms = e_start.elapsed_time(e_end) / args.steps
        e2e = {"ms_per_step": e2e_ms,
               "h2d_bytes_per_step": int(sum(x.numel() * x.element_size() for x in h_in)),
               "d2h_bytes_per_step": int(h_out[0].numel() * h_out[0].element_size())}
        del d_in, d_out

    total_ms, mask_ms, pair_ms, cap_ms, sp_ms, e2e_ms, sp_c_ms = max_over_ranks(
        [total_ms, per_kernel["mask"], per_kernel["pair"], per_kernel["capture"], per_kernel["sparse"],
         e2e["ms_per_step"] if e2e else 0.0, sparse_c_ms], device, world)
    return {"w": w, "keep": keep, "keep_ratio": keep_ratio, "total_ms": total_ms, "mask_ms": mask_ms,
            "pair_ms": pair_ms, "capture_ms": cap_ms, "sparse_ms": sp_ms, "sparse_compressed_ms": sp_c_ms,
            "e2e": e2e, "e2e_ms": e2e_ms, "clocks": clk, "nums": nums,
            "host1": host1, "host0": host0, "gpu": {"row_ptr": rp, "col_idx": ci, "out0": out0, "out1": out1,
                                                    "stats": stats}}


# --------------------------------------------------------------------------- configuration sweep
def run_sweep(args, device, checker=None) -> list:
    """Per-kernel times of one mask + capture + sparse cycle on every workload
    (the 5B shape at every keep ratio), L2 flushed between cycles.  With a
    `checker` (the CPU-baseline leg's OracleChecker) each row also carries the
    oracle's error figures on sampled rows of that cycle's outputs."""
    import ultra_sparse_attention_b200 as usa

    peaks, _ = load_peaks()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=device)  # twice the L2
    stream = torch.cuda.current_stream(device)
    cases = [("tiny", None), ("image", None), ("video2b", None)]
    cases += [("video5b", r) for r in WORKLOADS["video5b"].keep] + [("long", None)]
    out = []
    for name, ratio in cases:
        w = WORKLOADS[name]
        ratio = w.keep[0] if ratio is None else ratio
        keep = w.keep_blocks(ratio)
        steps = denoising_inputs(w, 2)
        host0 = next(steps)[1:]
        host1 = next(steps)[1:]
        q0, k0, v0 = (x.to(device) for x in host0)
        q1, k1, v1 = (x.to(device) for x in host1)
        kw = dict(head_dim=w.head_dim, block_size=w.block_size, scale=w.scale)
        times = {"mask": [], "pair": [], "capture": [], "sparse": [], "sparse_c": []}
        rp = ci = tb = None
        for it in range(args.sweep_warmup + args.sweep_steps):
            flush.zero_()
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
            ev[0].record(stream)
            rp, ci = usa.rt_build_block_mask(q0, k0, keep_blocks=keep, forced_prefix_tokens=w.forced_prefix_tokens, **kw)
            ev[1].record(stream)
            tb = usa.rt_pair_query_blocks(q0, rp, ci, head_dim=w.head_dim, block_size=w.block_size)
            ev[2].record(stream)
            out0, st = usa.rt_attn_full_capture(q0, k0, v0, row_ptr=rp, col_idx=ci, **kw)
            ev[3].record(stream)
            out1 = usa.rt_attn_sparse_reshape(q1, k1, v1, row_ptr=rp, col_idx=ci, stats=st, tile_blocks=tb, **kw)
            ev[4].record(stream)
            if it >= args.sweep_warmup:
                for i, k in enumerate(("mask", "pair", "capture", "sparse")):
                    times[k].append((ev[i], ev[i + 1]))
        # the sparse step on the compressed cache (same mask and tiles), L2 flushed likewise
        _, st_c = usa.rt_attn_full_capture(q0, k0, v0, row_ptr=rp, col_idx=ci, compressed=True, **kw)
        for it in range(args.sweep_warmup + args.sweep_steps):
            flush.zero_()
            e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
            e[0].record(stream)
            usa.rt_attn_sparse_reshape(q1, k1, v1, row_ptr=rp, col_idx=ci, stats=st_c, tile_blocks=tb, **kw)
            e[1].record(stream)
            if it >= args.sweep_warmup:
                times["sparse_c"].append((e[0], e[1]))
        del st_c
        # How close the reshaped sparse step comes to full attention of its own inputs (the
        # capture kernel's output on them), against plain block-sparse attention.
        full1, _ = usa.rt_attn_full_capture(q1, k1, v1, row_ptr=rp, col_idx=ci, **kw)
        resh1 = usa.rt_attn_sparse_reshape(q1, k1, v1, row_ptr=rp, col_idx=ci, stats=st, tile_blocks=tb, **kw)
        plain1 = usa.rt_attn_sparse_reshape(q1, k1, v1, row_ptr=rp, col_idx=ci, stats=None, **kw)
        torch.cuda.synchronize()
        if usa.rt_take_device_error() != 0:
            raise RuntimeError(f"a kernel reported a device error in the sweep ({name})")
        ref_norm = torch.linalg.vector_norm(full1.float()).item()
        err_r = torch.linalg.vector_norm(resh1.float() - full1.float()).item() / ref_norm
        err_p = torch.linalg.vector_norm(plain1.float() - full1.float()).item() / ref_norm
        del resh1, plain1
        # The same cycle with the mask chosen by exact block attention mass (one extra
        # full-attention pass at the capture step): its time and the reshape's distance to full
        # attention, beside the pooled mask's.
        exact = None
        if name != "tiny" and (name != "video5b" or ratio == w.keep[0]):
            ex_ms = []
            for it in range(args.sweep_warmup + 3):
                flush.zero_()
                e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
                e[0].record(stream)
                rpx, cix = usa.rt_build_block_mask_exact(q0, k0, v0, keep_blocks=keep,
                                                         forced_prefix_tokens=w.forced_prefix_tokens, **kw)
                e[1].record(stream)
                if it >= args.sweep_warmup:
                    ex_ms.append((e[0], e[1]))
            tbx = usa.rt_pair_query_blocks(q0, rpx, cix, head_dim=w.head_dim, block_size=w.block_size)
            _, stx = usa.rt_attn_full_capture(q0, k0, v0, row_ptr=rpx, col_idx=cix, **kw)
            reshx = usa.rt_attn_sparse_reshape(q1, k1, v1, row_ptr=rpx, col_idx=cix, stats=stx, tile_blocks=tbx, **kw)
            plainx = usa.rt_attn_sparse_reshape(q1, k1, v1, row_ptr=rpx, col_idx=cix, stats=None, tile_blocks=tbx,
                                                **kw)
            torch.cuda.synchronize()
            if usa.rt_take_device_error() != 0:
                raise RuntimeError(f"a kernel reported a device error in the exact-mask cycle ({name})")
            exact = {"mask_ms": statistics.mean(a.elapsed_time(b) for a, b in ex_ms),
                     "reshape_rel_l2_vs_full": torch.linalg.vector_norm(reshx.float() - full1.float()).item() / ref_norm,
                     "plain_sparse_rel_l2_vs_full":
                         torch.linalg.vector_norm(plainx.float() - full1.float()).item() / ref_norm,
                     "kept_sets_differing_from_pooled": float((cix.view(-1, keep) != ci.view(-1, keep)).any(1)
                                                              .float().mean().item()),
                     "what": "rt_build_block_mask_exact (one full-attention pass, block masses, top-k) "
                             "instead of the pooled mask; same capture and sparse kernels"}
            del rpx, cix, tbx, stx, reshx, plainx
        # The image grids with their tokens in Hilbert order (each 64-token block an 8 x 8 patch
        # square): the permutation's cost and the reshape's distance to full attention.
        hilbert = None
        if w.kind in ("smooth", "smooth_outliers"):
            perm = usa.rt_hilbert_order(w.grid, w.grid).to(device)
            pq0 = torch.empty_like(q0)
            pm_ms = []
            for it in range(args.sweep_warmup + 5):
                flush.zero_()
                e = [torch.cuda.Event(enable_timing=True) for _ in range(2)]
                e[0].record(stream)
                usa.rt_permute_tokens(q0, perm, out=pq0, head_dim=w.head_dim)
                e[1].record(stream)
                if it >= args.sweep_warmup:
                    pm_ms.append((e[0], e[1]))
            hp0 = [usa.rt_permute_tokens(x, perm, head_dim=w.head_dim) for x in (q0, k0, v0)]
            hp1 = [usa.rt_permute_tokens(x, perm, head_dim=w.head_dim) for x in (q1, k1, v1)]
            rph, cih = usa.rt_build_block_mask(hp0[0], hp0[1], keep_blocks=keep,
                                               forced_prefix_tokens=w.forced_prefix_tokens, **kw)
            tbh = usa.rt_pair_query_blocks(hp0[0], rph, cih, head_dim=w.head_dim, block_size=w.block_size)
            _, sth = usa.rt_attn_full_capture(*hp0, row_ptr=rph, col_idx=cih, **kw)
            resh = usa.rt_permute_tokens(usa.rt_attn_sparse_reshape(*hp1, row_ptr=rph, col_idx=cih, stats=sth,
                                                                    tile_blocks=tbh, **kw), perm, inverse=True,
                                         head_dim=w.head_dim)
            plainh = usa.rt_permute_tokens(usa.rt_attn_sparse_reshape(*hp1, row_ptr=rph, col_idx=cih, stats=None,
                                                                      tile_blocks=tbh, **kw), perm, inverse=True,
                                           head_dim=w.head_dim)
            torch.cuda.synchronize()
            if usa.rt_take_device_error() != 0:
                raise RuntimeError(f"a kernel reported a device error in the Hilbert cycle ({name})")
            pm = statistics.mean(a.elapsed_time(b) for a, b in pm_ms)
            hilbert = {"permute_ms_per_tensor": pm,
                       "permute_gbs": 2 * q0.numel() * 2 / (pm / 1e3) / 1e9,
                       "reshape_rel_l2_vs_full": torch.linalg.vector_norm(resh.float() - full1.float()).item() / ref_norm,
                       "plain_sparse_rel_l2_vs_full":
                           torch.linalg.vector_norm(plainh.float() - full1.float()).item() / ref_norm,
                       "what": "Q/K/V of both steps reordered along the Hilbert curve of the patch grid "
                               "(rt_hilbert_order, rt_permute_tokens), the pooled mask and the same kernels on "
                               "the reordered tokens, the output mapped back"}
            del perm, pq0, hp0, hp1, rph, cih, tbh, sth, resh, plainh
        del full1
        ms = {k: statistics.mean(a.elapsed_time(b) for a, b in v) for k, v in times.items()}
        nums = workload_numbers(w, keep, rp.cpu().numpy(), ci.cpu().numpy())
        sp_s, cap_s = ms["sparse"] / 1e3, ms["capture"] / 1e3
        exe = nums["executed_flops"] / sp_s / 1e12
        cap = nums["dense_flops"] / cap_s / 1e12
        out.append({"workload": name, "shape": f"B={w.batch} H={w.heads} N={w.seq_len} d={w.head_dim} D={w.head_dim_padded} "
                                               f"block={w.block_size}",
                    "keep": f"{keep}/{w.n_blocks} ({ratio})", "sparse_step_ms": ms["sparse"],
                    "sparse_step_ms_compressed_cache": ms["sparse_c"],
                    "full_step_ms": ms["mask"] + ms["pair"] + ms["capture"], "mask_ms": ms["mask"],
                    "pair_ms": ms["pair"], "capture_ms": ms["capture"],
                    "dense_equiv_tflops": nums["dense_flops"] / sp_s / 1e12, "executed_tflops": exe,
                    "sparse_tensor_frac_of_bf16_peak": exe / peaks["bf16_tflops"],
                    "capture_tflops": cap, "capture_frac_of_bf16_peak": cap / peaks["bf16_tflops"],
                    "reshape_rel_l2_vs_full": err_r, "plain_sparse_rel_l2_vs_full": err_p,
                    "exact_mass_mask": exact, "hilbert_order": hilbert,
                    "steps": args.sweep_steps, "warmup": args.sweep_warmup, "l2": "flushed between cycles"})
        if checker is not None:
            out[-1]["oracle_check"] = checker.check(w, keep, host0, host1, rp, ci, out0, st, out1)
        del q0, k0, v0, q1, k1, v1, st, rp, ci, tb, out0, out1, host0, host1
    return out


# --------------------------------------------------------------------------- oracle timing (CPU)
class OracleSample:
    """The fp64 oracle's sparse step on a bounded row sample of the workload.

    Its block mask and the capture statistics of the sampled rows are computed
    once, untimed; ``time_step`` then times one sparse step with the reshape."""

    def __init__(self, w, keep: int, host0, host1, rows: int, seed: int = 0):
        import oracle
        self.oracle, self.w, self.keep, self.host1 = oracle, w, keep, host1
        d, bs = w.head_dim, w.block_size
        self.rp, self.ci = oracle.build_block_mask(host0[0], host0[1], d, bs, w.scale, keep, w.forced_prefix_tokens)
        rng = np.random.default_rng(seed)
        total = w.batch * w.heads * w.seq_len
        self.rows = np.sort(rng.choice(total, size=min(rows, total), replace=False)).astype(np.int64)
        self.threads = oracle.default_threads()
        self.stats = oracle.full_capture(*host0, d, bs, w.scale, self.rp, self.ci, rows=self.rows, threads=self.threads)
        self.dense_flops = 4.0 * w.seq_len * d * len(self.rows)
        self.desc = (f"{len(self.rows)} query rows sampled uniformly (seed {seed}) of {total} of {w.name} at keep "
                     f"{keep}/{w.n_blocks}: fp64 oracle sparse step with reshape on {self.threads} threads; its mask "
                     f"and the capture statistics of those rows computed beforehand, untimed")

    def time_step(self) -> float:
        w = self.w
        t0 = time.perf_counter()
        self.oracle.sparse_reshape(*self.host1, w.head_dim, w.block_size, w.scale, self.rp, self.ci, self.stats,
                                   rows=self.rows, threads=self.threads)
        return time.perf_counter() - t0

    def baseline(self, repeats: int = 3) -> dict:
        secs = min(self.time_step() for _ in range(repeats))
        return {"value": self.dense_flops / secs / 1e12, "unit": UNIT, "cores": self.threads, "kind": "oracle",
                "sample": self.desc}


class OracleChecker:
    """Part of the CPU-baseline leg: the GPU outputs of a cycle against the fp64 oracle on a
    few sampled rows (capture output and statistics, sparse output), with the oracle's own
    block mask.  Rows are sampled only from query blocks whose kept sets the GPU mask and the
    oracle's agree on (a near tie may make them differ; the count is reported)."""

    def __init__(self, rows: int = 64, seed: int = 1):
        import oracle
        self.oracle, self.rows, self.seed = oracle, rows, seed

    def check(self, w, keep, host0, host1, rp_gpu, ci_gpu, out0, st, out1) -> dict:
        orc = self.oracle
        d, bs, D, N = w.head_dim, w.block_size, w.head_dim_padded, w.seq_len
        rp_o, ci_o = orc.build_block_mask(host0[0], host0[1], d, bs, w.scale, keep, w.forced_prefix_tokens)
        rp_g = rp_gpu.cpu().numpy() if torch.is_tensor(rp_gpu) else rp_gpu
        ci_g = ci_gpu.cpu().numpy() if torch.is_tensor(ci_gpu) else ci_gpu
        nb = w.n_blocks
        n_qb = w.batch * w.heads * nb
        same = np.array([np.array_equal(ci_g[rp_g[r]:rp_g[r + 1]], ci_o[rp_o[r]:rp_o[r + 1]]) for r in range(n_qb)])
        rng = np.random.default_rng(self.seed)
        cand = rng.choice(w.batch * w.heads * N, size=min(w.batch * w.heads * N, 8 * self.rows), replace=False)
        cand = cand[same[(cand // N) * nb + (cand % N) // bs]]
        rows = np.sort(cand[:self.rows]).astype(np.int64)
        cap = orc.full_capture(*host0, d, bs, w.scale, rp_o, ci_o, rows=rows)
        cap_abs = orc.full_capture(host0[0], host0[1], host0[2].abs(), d, bs, w.scale, rp_o, ci_o, rows=rows)["u"]
        sp = orc.sparse_reshape(*host1, d, bs, w.scale, rp_o, ci_o, cap, rows=rows)
        sel = torch.as_tensor(rows, device=out0.device)

        def errs(got, want):
            g = got.reshape(-1, D)[sel].double().cpu().numpy()[:, :d]
            e = np.abs(g - want)
            big = np.abs(want) > 1.0  # where the unit-scale reading of the max-abs bound differs
            return {"max_abs_unit_scale": float(np.max(e / np.maximum(1.0, np.abs(want)))),
                    "mean_abs": float(e.mean()), "max_abs_raw": float(e.max()),
                    "max_abs_where_above_1": float(e[big].max()) if big.any() else None,
                    "max_rel_where_above_1": float((e[big] / np.abs(want[big])).max()) if big.any() else None}

        zf = st.zfull.reshape(-1)[sel].double().cpu().numpy()
        zk = st.zkept.reshape(-1)[sel].double().cpu().numpy()
        m = st.m.reshape(-1)[sel].double().cpu().numpy()
        u = st.u.reshape(-1, D)[sel].double().cpu().numpy()[:, :d]
        bound = 1e-3 * cap_abs / cap["zfull"][:, None] + 1e-7
        stats = {"ratio_rel": float(np.max(np.abs((zf / zk) / (cap["zfull"] / cap["zkept"]) - 1))),
                 "lse_abs": float(np.max(np.abs(m + np.log(zf) - cap["m"] - np.log(cap["zfull"])))),
                 "u_err_over_bound": float(np.max(np.abs(u / zf[:, None] - cap["u"] / cap["zfull"][:, None]) / bound))}
        return {"rows": int(len(rows)), "mask_rows_differing": int(n_qb - int(same.sum())),
                "capture_o": errs(out0, cap["o"]), "capture_stats": stats, "sparse_o": errs(out1, sp),
                "tolerance": "o: max-abs 1.5e-2 at unit scale, mean-abs 1.5e-3; stats: 1e-3 relative"}


def run_reference(args, rank, world):
    """The base contract's reference arm: the fp64 oracle on the host cores."""
    if rank != 0:
        return None
    w = WORKLOADS[args.workload]
    if args.heads:
        w = dataclasses.replace(w, heads=args.heads)
    keep_ratio = Fraction(args.keep) if args.keep else w.keep[0]
    keep = w.keep_blocks(keep_ratio)
    steps = list(denoising_inputs(w, 2))
    sample = OracleSample(w, keep, steps[0][1:], steps[1][1:], args.cpu_rows)
    for _ in range(args.warmup):
        sample.time_step()
    secs = sum(sample.time_step() for _ in range(args.steps))
    value = sample.dense_flops * args.steps / secs / 1e12
    cpu = {"value": value, "unit": UNIT, "cores": sample.threads, "kind": "oracle", "sample": sample.desc}
    return {"metric": METRIC, "value": value, "unit": UNIT, "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": _config(w, keep, keep_ratio, args.gpus),
            "cpu_baseline": cpu, "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                                         "d2h_bytes_per_step": 0}}


def _config(w, keep, keep_ratio, gpus):
    return {"workload": (f"{w.name}: B={w.batch} H={w.heads} N={w.seq_len} d={w.head_dim} D={w.head_dim_padded} "
                         f"block={w.block_size} keep={keep}/{w.n_blocks} ({keep_ratio})"),
            "step": "mask + tile pairing + full capture at t0, sparse reshape at t1 (drifted inputs)",
            "forced_prefix_tokens": w.forced_prefix_tokens,
            "l2": "inputs larger than L2 (about 1.1 GB touched per step; no flush)",
            "parallelism": f"replicas x{gpus}"}


# --------------------------------------------------------------------------- main
def main():
    args = parse_args()
    rank, world, local = dist_env()
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=180),
                                             device_id=torch.device("cuda", local))
    r = run_ours(args, rank, world, local)
    if rank == 0:
        peaks, peak_src = load_peaks()
        # The CPU-baseline leg (rank 0 at one GPU): the oracle's timed sample, and its error
        # check of the GPU outputs on sampled rows of the main cycle and of every sweep cycle.
        cpu_leg = not args.no_cpu_baseline and world == 1
        checker = OracleChecker() if cpu_leg else None
        sweep = None
        if not args.no_sweep and world == 1:
            sweep = run_sweep(args, torch.device("cuda", local), checker)
        cpu = None
        if cpu_leg:
            cpu = OracleSample(r["w"], r["keep"], r["host0"], r["host1"], args.cpu_rows).baseline()
            g = r["gpu"]
            cpu["oracle_check"] = checker.check(r["w"], r["keep"], r["host0"], r["host1"], g["row_ptr"],
                                                g["col_idx"], g["out0"], g["stats"], g["out1"])
        print(json.dumps(build_line(args, r, world, peaks, peak_src, sweep, cpu)), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


def build_line(args, r: dict, world: int, peaks: dict, peak_src: str, sweep, cpu) -> dict:
    """The JSON line of our arm from one measurement `r` of run_ours (rank 0)."""
    w, nums = r["w"], r["nums"]
    sp_s = r["sparse_ms"] / 1e3
    value = job_throughput(nums["dense_flops"], world, r["sparse_ms"])
    exec_tflops = nums["executed_flops"] / sp_s / 1e12
    cap_tflops = nums["dense_flops"] / (r["capture_ms"] / 1e3) / 1e12
    kernels = {
        "rt_build_block_mask": {"ms": r["mask_ms"], "bound": "hbm",
                                "achieved_gbs": nums["mask_bytes"] / (r["mask_ms"] / 1e3) / 1e9},
        "rt_pair_query_blocks": {"ms": r["pair_ms"], "bound": "latency (one CTA per head, once per mask)"},
        "rt_attn_full_capture": {"ms": r["capture_ms"], "bound": "tensor", "achieved_tflops": cap_tflops,
                                 "algorithmic_tflop": nums["dense_flops"] / 1e12,
                                 "achieved_gbs": nums["capture_bytes"] / (r["capture_ms"] / 1e3) / 1e9},
        "rt_attn_sparse_reshape": {"ms": r["sparse_ms"], "bound": "tensor+hbm",
                                   "executed_tflops": exec_tflops,
                                   "executed_tflop": nums["executed_flops"] / 1e12,
                                   "dense_equiv_tflops": nums["dense_flops"] / sp_s / 1e12,
                                   "tensor_frac_of_bf16_peak": exec_tflops / peaks["bf16_tflops"],
                                   "achieved_gbs": nums["sparse_bytes"] / sp_s / 1e9,
                                   "hbm_frac": nums["sparse_bytes"] / sp_s / 1e9 / peaks["hbm_gbs"],
                                   "algorithmic_bytes": nums["sparse_bytes"],
                                   "key_tiles_per_query_tile": nums.get("key_tiles_per_query_tile"),
                                   "key_tiles_per_query_tile_neighbours": nums.get("key_tiles_per_query_tile_neighbours")},
    }
    if r.get("sparse_compressed_ms"):
        spc_s = r["sparse_compressed_ms"] / 1e3
        exc = nums["executed_flops"] / spc_s / 1e12
        kernels["rt_attn_sparse_reshape_u16"] = {
            "ms": r["sparse_compressed_ms"], "bound": "tensor+hbm", "executed_tflops": exc,
            "tensor_frac_of_bf16_peak": exc / peaks["bf16_tflops"],
            "dense_equiv_tflops": nums["dense_flops"] / spc_s / 1e12,
            "achieved_gbs": nums["sparse_bytes_compressed"] / spc_s / 1e9,
            "algorithmic_bytes": nums["sparse_bytes_compressed"],
            "what": "the sparse step reading the compressed residual cache (f16 U, one power-of-two scale per row), "
                    "timed in its own loop after the main one"}
    # dominant kernel of the step (by device time)
    dom = max(("rt_attn_full_capture", r["capture_ms"]), ("rt_attn_sparse_reshape", r["sparse_ms"]),
              ("rt_build_block_mask", r["mask_ms"]), key=lambda t: t[1])[0]
    wl_tag = f"{w.name}@{r['keep']}"
    if dom == "rt_attn_full_capture":
        ach = cap_tflops
        roof = {"kernel": dom, "bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": ach / peaks["bf16_tflops"],
                "traffic": stored_traffic("full_capture_kernel", wl_tag),
                "peak_source": f"bf16_tflops ({peak_src}, burst)",
                "per_launch": f"{nums['dense_flops'] / 1e12:.3f} TFLOP algorithmic (4*B*H*N^2*d)"}
    elif dom == "rt_attn_sparse_reshape":
        ach = exec_tflops
        roof = {"kernel": dom, "bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": ach / peaks["bf16_tflops"],
                "traffic": stored_traffic("sparse_reshape_kernel", wl_tag),
                "peak_source": f"bf16_tflops ({peak_src}, burst)"}
    else:
        ach = kernels["rt_build_block_mask"]["achieved_gbs"]
        roof = {"kernel": dom, "bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": ach / peaks["hbm_gbs"], "traffic": None, "peak_source": f"hbm_gbs ({peak_src})"}
    # The kernel the target is stated for: the sparse step on its executed (kept-block) flops,
    # beside its achieved HBM bandwidth on the algorithmic bytes.
    sp_ach = exec_tflops
    roof_sparse = {"kernel": "rt_attn_sparse_reshape", "bound": "tensor", "achieved": sp_ach,
                   "peak": peaks["bf16_tflops"], "unit": "TFLOP/s", "frac": sp_ach / peaks["bf16_tflops"],
                   "traffic": stored_traffic("sparse_reshape_kernel", wl_tag),
                   "peak_source": f"bf16_tflops ({peak_src}, burst)",
                   "per_launch": f"{nums['executed_flops'] / 1e12:.4f} TFLOP executed (kept blocks, 4*d*rows*cols)",
                   "hbm_achieved_gbs": nums["sparse_bytes"] / sp_s / 1e9,
                   "hbm_frac": nums["sparse_bytes"] / sp_s / 1e9 / peaks["hbm_gbs"],
                   "algorithmic_bytes": nums["sparse_bytes"], "target_frac": 0.5}
    kept_tokens = nums["executed_flops"] / nums["dense_flops"]
    claims = [
        {"claim": "quality on par with full attention while attending to 3.1% of the tokens", "source":
         "Re-ttention project page, Abstract", "hardware": "not stated",
         "here": f"{r['keep']}/{w.n_blocks} key blocks per query block = {100.0 * r['keep'] / w.n_blocks:.2f}% of the "
                 f"keys; {100.0 * kept_tokens:.2f}% of the dense score work executed"},
        {"claim": "more than 95% of the attention compute avoided", "source": "Re-ttention project page, teaser",
         "hardware": "not stated", "here": f"{100.0 * (1.0 - kept_tokens):.2f}% of the dense QK^T and PV flops skipped "
                                           "in the sparse step"},
    ]
    e2e = None
    if r["e2e"]:
        e2e = {"value": job_throughput(nums["dense_flops"], world, r["e2e_ms"]), "unit": UNIT,
               "ms_per_step": r["e2e_ms"], "h2d_bytes_per_step": r["e2e"]["h2d_bytes_per_step"],
               "d2h_bytes_per_step": r["e2e"]["d2h_bytes_per_step"],
               "what": "sparse step through the public API: pinned host Q1/K1/V1 -> device, "
                       "rt_attn_sparse_reshape, output -> pinned host; steps pipelined on three "
                       "streams (next step's upload overlaps this step's kernel and read-back)"}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": r["total_ms"] / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": _config(w, r["keep"], r["keep_ratio"], world),
        "sparse_step_ms": r["sparse_ms"], "full_step_ms": r["mask_ms"] + r["pair_ms"] + r["capture_ms"],
        "dense_equiv_tflops": nums["dense_flops"] / sp_s / 1e12, "executed_tflops": exec_tflops,
        "tensor_pct_of_bf16_peak": 100.0 * exec_tflops / peaks["bf16_tflops"],
        "roofline": roof, "roofline_sparse": roof_sparse, "pages_claims": claims,
        "kernels": kernels, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": LAUNCHES_PER_STEP * args.steps, "clocks": r["clocks"],
        "peaks": {**peaks, "source": peak_src},
        "sweep": sweep,
    }
    return line


if __name__ == "__main__":
    main()
