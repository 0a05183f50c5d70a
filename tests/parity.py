"""Shared helpers of the GPU parity tests: run the CUDA path and the fp64
oracle on the same seeded inputs and compare them.

Tolerances (fixed by the target, not tuned): attention outputs within
max-abs 1.5e-2 and mean-abs 1.5e-3 of the oracle, the max-abs bound stated
for unit-scale outputs and so applied to |got - want| / max(1, |want|)
(bf16's own spacing is 2^-5 on [4, 8), so even a correctly rounded output of
magnitude 4 can be 1.56e-2 off; the video workloads reach |o| ~ 5); statistics within 1e-3
relative, compared in forms that do not depend on the exponent reference
(Z_full/Z_kept, m + ln Z_full, and U/Z_full against the absolute masked mass);
kept-block lists bit-exact wherever the oracle's decision is not a near tie.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
import ultra_sparse_attention_b200 as usa

OUT_MAX_ABS = 1.5e-2
OUT_MEAN_ABS = 1.5e-3
STAT_REL = 1e-3


def csr_sets(row_ptr, col_idx):
    rp = np.asarray(row_ptr)
    ci = np.asarray(col_idx)
    return [tuple(ci[rp[r]:rp[r + 1]].tolist()) for r in range(len(rp) - 1)]


def random_csr(bh, nb, keep, seed, forced=0):
    """Random kept sets (sorted, forced prefix included): int32 row_ptr, col_idx."""
    rng = np.random.default_rng(seed)
    sets = []
    for _ in range(bh * nb):
        rest = rng.choice(np.arange(forced, nb), size=keep - forced, replace=False) if keep > forced else []
        sets.append(sorted(set(range(forced)) | set(int(x) for x in rest)))
    row_ptr = np.array([0] + list(np.cumsum([len(s) for s in sets])), np.int32)
    col_idx = np.array([kb for s in sets for kb in s], np.int32)
    return row_ptr, col_idx


def to_dev(a, device, dtype=None):
    t = torch.as_tensor(np.ascontiguousarray(a)) if isinstance(a, np.ndarray) else a
    t = t.to(device)
    return t.to(dtype) if dtype is not None else t


def score_tol(scores: np.ndarray) -> float:
    """Bound on |fp32 GPU block score - fp64 oracle score| used for tie decisions."""
    return 1e-4 * (1.0 + float(np.max(np.abs(scores))))


def check_mask(rp_gpu, ci_gpu, scores64, keep, bs, forced_tokens, tol):
    """GPU CSR against the oracle's: identical on every row whose decision is not a
    near tie; on near-tie rows the GPU set must still be a valid top-k within tol.
    Returns the number of near-tie rows where the sets differ."""
    rp_gpu = np.asarray(rp_gpu)
    ci_gpu = np.asarray(ci_gpu)
    s = scores64.reshape(-1, scores64.shape[-1])
    rows, nkb = s.shape
    assert list(rp_gpu) == [r * keep for r in range(rows + 1)]
    rp_o, ci_o = oracle.select_blocks(s, keep, bs, forced_tokens)
    forced = min(nkb, -(-forced_tokens // bs)) if forced_tokens > 0 else 0
    differ = 0
    for r in range(rows):
        g = ci_gpu[r * keep:(r + 1) * keep]
        o = ci_o[r * keep:(r + 1) * keep]
        assert list(g) == sorted(set(g.tolist())), f"row {r}: not sorted/unique"
        if np.array_equal(g, o):
            continue
        rest = [kb for kb in range(nkb) if kb >= forced]
        order = sorted(rest, key=lambda kb: (-s[r, kb], kb))
        need = keep - forced
        kth = s[r, order[need - 1]]
        nxt = s[r, order[need]] if need < len(order) else -math.inf
        assert kth - nxt <= 2 * tol, f"row {r}: mask differs with decisive gap {kth - nxt}"
        assert set(range(forced)) <= set(g.tolist())
        for kb in g:
            if kb >= forced:
                assert s[r, kb] >= kth - 2 * tol
        differ += 1
    return differ


def compare_out(got: torch.Tensor, want: np.ndarray, d: int, what: str):
    """bf16 GPU rows [R, D] against fp64 oracle rows [R, d]: max-abs at unit scale, mean abs, pads zero."""
    g = got.float().cpu().numpy().astype(np.float64)
    assert np.all(g[:, d:] == 0.0), f"{what}: pad columns not zero"
    err = np.abs(g[:, :d] - want)
    assert np.all(np.isfinite(g)), f"{what}: non-finite output"
    mx = float(np.max(err / np.maximum(1.0, np.abs(want))))  # max-abs at unit scale
    mean = float(err.mean())
    assert mx <= OUT_MAX_ABS and mean <= OUT_MEAN_ABS, (
        f"{what}: max-abs (unit scale) {mx:.3e} (raw {float(err.max()):.3e}) mean-abs {mean:.3e}")
    return mx, mean


def compare_stats(st_gpu: usa.Stats, rows: np.ndarray, orc: dict, orc_abs_u: np.ndarray, d: int, what: str):
    """GPU capture statistics at global rows `rows` against the oracle's (same rows)."""
    m = st_gpu.m.reshape(-1)[rows].double().cpu().numpy()
    zf = st_gpu.zfull.reshape(-1)[rows].double().cpu().numpy()
    zk = st_gpu.zkept.reshape(-1)[rows].double().cpu().numpy()
    u = st_gpu.u.reshape(-1, st_gpu.u.shape[-1])[rows].double().cpu().numpy()
    assert np.all(u[:, d:] == 0.0), f"{what}: U pad columns not zero"
    r_g, r_o = zf / zk, orc["zfull"] / orc["zkept"]
    assert np.max(np.abs(r_g / r_o - 1.0)) <= STAT_REL, f"{what}: Z_full/Z_kept rel {np.max(np.abs(r_g / r_o - 1)):.2e}"
    lse_g, lse_o = m + np.log(zf), orc["m"] + np.log(orc["zfull"])
    assert np.max(np.abs(lse_g - lse_o)) <= STAT_REL, f"{what}: lse abs {np.max(np.abs(lse_g - lse_o)):.2e}"
    # U / Z_full, each element against the masked absolute mass sum_masked e|v| / Z_full
    ug = u[:, :d] / zf[:, None]
    uo = orc["u"] / orc["zfull"][:, None]
    bound = STAT_REL * orc_abs_u / orc["zfull"][:, None] + 1e-7
    worst = float(np.max(np.abs(ug - uo) / bound))
    assert worst <= 1.0, f"{what}: U/Z_full error {worst:.2f} x bound"


def sample_rows(bh: int, n: int, count: int, seed: int) -> np.ndarray:
    """Sorted global row ids: first/last rows of every head plus random ones."""
    rng = np.random.default_rng(seed)
    fixed = [h * n + i for h in {0, bh // 2, bh - 1} for i in (0, 1, 63, 64, 127, n - 1)]
    rand = rng.choice(bh * n, size=min(count, bh * n), replace=False)
    return np.unique(np.concatenate([np.array(fixed, np.int64), rand.astype(np.int64)]))
