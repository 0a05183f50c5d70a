"""fp64 CPU oracle of Re-ttention's attention path (ctypes shim over oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline / reference arm may import this package; the product
path (``ultra_sparse_attention_b200``) never does.  It shares no code with
the CUDA library.

Each wrapper below names the step of the method it computes.  The C source
(``oracle.c``) states which test pins each function to something other than
itself.
"""
from __future__ import annotations

import ctypes
import hashlib
import os
import subprocess
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_STAMP = _LIB + ".srchash"
_lock = threading.Lock()
_lib = None


def _src_hash() -> str:
    with open(_SRC, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()


def build(force: bool = False) -> str:
    """Compile oracle.c with gcc (plain -O2, IEEE fp64, no fast-math)."""
    h = _src_hash()
    if not force and os.path.exists(_LIB) and os.path.exists(_STAMP):
        with open(_STAMP) as f:
            if f.read().strip() == h:
                return _LIB
    tmp = f"{_LIB}.{os.getpid()}.tmp"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off",
           "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm", "-lpthread"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    with open(_STAMP, "w") as f:
        f.write(h)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB)
            i64, f64, vp = ctypes.c_int64, ctypes.c_double, ctypes.c_void_p
            lib.orc_pool_blocks.argtypes = [vp, i64, i64, i64, i64, i64, vp]
            lib.orc_block_scores.argtypes = [vp, vp, i64, i64, i64, f64, vp]
            lib.orc_select_blocks.argtypes = [vp, i64, i64, i64, i64, i64, vp, vp]
            lib.orc_full_capture.argtypes = [vp, vp, vp, i64, i64, i64, i64, i64, f64, vp, vp, vp,
                                             i64, vp, vp, vp, vp, vp, ctypes.c_int]
            lib.orc_sparse_reshape.argtypes = [vp, vp, vp, i64, i64, i64, i64, i64, f64, vp, vp,
                                               vp, vp, vp, vp, vp, i64, vp, ctypes.c_int]
            lib.orc_block_mass.argtypes = [vp, vp, i64, i64, i64, i64, i64, f64, vp, i64, vp, ctypes.c_int]
            for fn in ("orc_pool_blocks", "orc_block_scores", "orc_select_blocks",
                       "orc_full_capture", "orc_sparse_reshape", "orc_block_mass"):
                getattr(lib, fn).restype = ctypes.c_int
            _lib = lib
    return _lib


def _bf16_bits(x) -> np.ndarray:
    """bf16 torch tensor [B,H,N,D] -> contiguous uint16 numpy [B*H, N, D]."""
    if not (isinstance(x, torch.Tensor) and x.dtype == torch.bfloat16):
        raise TypeError("oracle inputs are bf16 torch tensors")
    x = x.detach().cpu().contiguous()
    return x.view(torch.int16).numpy().view(np.uint16).reshape(-1, x.shape[-2], x.shape[-1])


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, what: str):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed with code {rc}")


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count() or 1)


# --------------------------------------------------------------------------
# Mask (block pooling -> block scores -> top-k with forced prefix -> CSR)
# --------------------------------------------------------------------------
def pool_blocks(x, d: int, bs: int) -> np.ndarray:
    """Mean of each block's real tokens over the logical columns: fp64 [B*H, n_blocks, d]."""
    a = _bf16_bits(x)
    bh, n, dpad = a.shape
    nb = -(-n // bs)
    out = np.empty((bh, nb, d), dtype=np.float64)
    _check(_load().orc_pool_blocks(_ptr(a), bh, n, dpad, d, bs, _ptr(out)), "pool")
    return out


def block_scores(pq: np.ndarray, pk: np.ndarray, scale: float) -> np.ndarray:
    """scale * <pooled q block, pooled k block>: fp64 [B*H, n_blocks, n_blocks]."""
    pq = np.ascontiguousarray(pq, dtype=np.float64)
    pk = np.ascontiguousarray(pk, dtype=np.float64)
    bh, nb, d = pq.shape
    out = np.empty((bh, nb, nb), dtype=np.float64)
    _check(_load().orc_block_scores(_ptr(pq), _ptr(pk), bh, nb, d, float(scale), _ptr(out)), "scores")
    return out


def select_blocks(scores: np.ndarray, keep: int, bs: int, forced_tokens: int):
    """Top-k kept key blocks per row as CSR (row_ptr int32 [R+1], col_idx int32 [R*keep])."""
    s = np.ascontiguousarray(scores, dtype=np.float64)
    nkb = s.shape[-1]
    rows = s.size // nkb
    row_ptr = np.empty(rows + 1, dtype=np.int32)
    col_idx = np.empty(rows * keep, dtype=np.int32)
    _check(_load().orc_select_blocks(_ptr(s), rows, nkb, keep, bs, forced_tokens,
                                     _ptr(row_ptr), _ptr(col_idx)), "select")
    return row_ptr, col_idx


def build_block_mask(q, k, d: int, bs: int, scale: float, keep: int, forced_tokens: int,
                     return_scores: bool = False):
    """The whole mask step: pool Q and K, score block pairs, select, emit CSR."""
    s = block_scores(pool_blocks(q, d, bs), pool_blocks(k, d, bs), scale)
    row_ptr, col_idx = select_blocks(s, keep, bs, forced_tokens)
    return (row_ptr, col_idx, s) if return_scores else (row_ptr, col_idx)


def block_mass(q, k, d: int, bs: int, scale: float, qblocks=None, threads: int | None = None) -> np.ndarray:
    """Exact attention mass of every (query block, key block) pair: fp64 [B*H, n_blocks, n_blocks],
    the softmax probabilities of the block's query rows summed over the key block's keys.
    With ``qblocks`` (global query-block ids bh*n_blocks + qb) only those rows: [len, n_blocks]."""
    qa, ka = _bf16_bits(q), _bf16_bits(k)
    bh, n, dpad = qa.shape
    nb = -(-n // bs)
    qb = None if qblocks is None else np.ascontiguousarray(qblocks, dtype=np.int64)
    out = np.empty((bh, nb, nb) if qb is None else (qb.size, nb), dtype=np.float64)
    _check(_load().orc_block_mass(_ptr(qa), _ptr(ka), bh, n, dpad, d, bs, float(scale), _ptr(qb),
                                  0 if qb is None else qb.size, _ptr(out), threads or default_threads()),
           "block_mass")
    return out


def build_block_mask_exact(q, k, d: int, bs: int, scale: float, keep: int, forced_tokens: int,
                           return_mass: bool = False):
    """The mask from exact block masses: the same selection rule as the pooled mask, applied to
    block_mass instead of the pooled block scores."""
    a = block_mass(q, k, d, bs, scale)
    row_ptr, col_idx = select_blocks(a, keep, bs, forced_tokens)
    return (row_ptr, col_idx, a) if return_mass else (row_ptr, col_idx)


# --------------------------------------------------------------------------
# Attention steps
# --------------------------------------------------------------------------
def _rows_arg(rows):
    if rows is None:
        return None
    r = np.ascontiguousarray(rows, dtype=np.int64)
    return r


def full_capture(q, k, v, d: int, bs: int, scale: float, row_ptr, col_idx, rows=None,
                 threads: int | None = None) -> dict:
    """Full attention plus the cached statistics, per row (all rows if ``rows`` is None).

    ``rows`` holds global row ids bh*N + i.  Returns fp64 arrays: o [R, d],
    m [R], zfull [R], zkept [R], u [R, d].
    """
    qa, ka, va = _bf16_bits(q), _bf16_bits(k), _bf16_bits(v)
    bh, n, dpad = qa.shape
    r = _rows_arg(rows)
    nr = bh * n if r is None else r.size
    out = {"o": np.empty((nr, d)), "m": np.empty(nr), "zfull": np.empty(nr),
           "zkept": np.empty(nr), "u": np.empty((nr, d))}
    rp = np.ascontiguousarray(row_ptr, dtype=np.int32)
    ci = np.ascontiguousarray(col_idx, dtype=np.int32)
    rc = _load().orc_full_capture(_ptr(qa), _ptr(ka), _ptr(va), bh, n, dpad, d, bs, float(scale),
                                  _ptr(rp), _ptr(ci), _ptr(r), nr, _ptr(out["o"]), _ptr(out["m"]),
                                  _ptr(out["zfull"]), _ptr(out["zkept"]), _ptr(out["u"]),
                                  threads or default_threads())
    _check(rc, "full_capture")
    return out


def sparse_reshape(q, k, v, d: int, bs: int, scale: float, row_ptr, col_idx, stats: dict | None,
                   rows=None, threads: int | None = None) -> np.ndarray:
    """Sparse step over the kept blocks, reshaped with ``stats`` (or plain if None).

    ``stats`` holds per-row fp64 m, zfull, zkept, u for the same ``rows``.
    Returns fp64 [R, d].
    """
    qa, ka, va = _bf16_bits(q), _bf16_bits(k), _bf16_bits(v)
    bh, n, dpad = qa.shape
    r = _rows_arg(rows)
    nr = bh * n if r is None else r.size
    out = np.empty((nr, d))
    rp = np.ascontiguousarray(row_ptr, dtype=np.int32)
    ci = np.ascontiguousarray(col_idx, dtype=np.int32)
    if stats is None:
        cm = czf = czk = cu = None
    else:
        cm = np.ascontiguousarray(stats["m"], dtype=np.float64)
        czf = np.ascontiguousarray(stats["zfull"], dtype=np.float64)
        czk = np.ascontiguousarray(stats["zkept"], dtype=np.float64)
        cu = np.ascontiguousarray(stats["u"], dtype=np.float64)
    rc = _load().orc_sparse_reshape(_ptr(qa), _ptr(ka), _ptr(va), bh, n, dpad, d, bs, float(scale),
                                    _ptr(rp), _ptr(ci), _ptr(cm), _ptr(czf), _ptr(czk), _ptr(cu),
                                    _ptr(r), nr, _ptr(out), threads or default_threads())
    _check(rc, "sparse_reshape")
    return out


# --------------------------------------------------------------------------
# Hilbert-curve token order (HilbertA blog page, "Introducing HilbertA", first
# component, Reordering: tokens follow a Hilbert curve over the patch grid, so
# neighbours on the grid stay neighbours in the sequence).  Pinned by the
# curve's defining properties: a bijection onto the cells, consecutive cells
# 4-adjacent, each quarter of the curve filling one quadrant, the order-1 curve.
# --------------------------------------------------------------------------
def hilbert_curve(k: int) -> list[tuple[int, int]]:
    """Cells (x, y) of the 2^k x 2^k grid in Hilbert order, by the recursive definition:
    the curve of side 2s visits the lower-left quadrant along the transposed curve of side s,
    then the upper-left and upper-right quadrants along the curve itself, then the lower-right
    quadrant along the anti-transposed curve; it starts at (0, 0) and ends at (2s - 1, 0)."""
    if k == 0:
        return [(0, 0)]
    sub = hilbert_curve(k - 1)
    s = 1 << (k - 1)
    return ([(y, x) for x, y in sub] +
            [(x, y + s) for x, y in sub] +
            [(x + s, y + s) for x, y in sub] +
            [(2 * s - 1 - y, s - 1 - x) for x, y in sub])


def hilbert_order(grid_h: int, grid_w: int, frames: int = 1, prefix: int = 0) -> np.ndarray:
    """Token permutation perm (int64 [prefix + frames*grid_h*grid_w]): position t of the
    reordered sequence holds token perm[t] of the row-major one (cell (x, y) of frame f is
    token prefix + f*grid_h*grid_w + y*grid_w + x).  The first `prefix` tokens (text) keep
    their place; each frame's cells follow the Hilbert curve of the smallest power-of-two
    square that holds the grid, skipping the square's cells outside it."""
    k = 0
    while (1 << k) < max(grid_h, grid_w):
        k += 1
    cells = [y * grid_w + x for x, y in hilbert_curve(k) if x < grid_w and y < grid_h]
    hw = grid_h * grid_w
    order = list(range(prefix))
    for f in range(frames):
        order += [prefix + f * hw + c for c in cells]
    return np.array(order, dtype=np.int64)


def permute_tokens(x, perm, inverse: bool = False):
    """Reordered copy of a [B, H, N, D] tensor: out[..., t, :] = x[..., perm[t], :], or the
    inverse, out[..., perm[t], :] = x[..., t, :]."""
    p = torch.as_tensor(np.asarray(perm, dtype=np.int64))
    if not inverse:
        return x[..., p, :].clone()
    out = torch.empty_like(x)
    out[..., p, :] = x
    return out
