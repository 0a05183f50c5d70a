"""Save and reload what a capture step leaves for the later sparse steps.

A denoising run keeps, per attention layer, the kept-block CSR, the query-block
pairing table and the statistics cache (m, Z_full, Z_kept, U; fp32 or the
compressed f16 U with its row scale) from the latest capture step until the
next one.  ``save_cache`` writes them, with the shape and scale they belong
to, to one ``.npz`` file; ``load_cache`` reads it back onto a device.  Uses:
resuming a run between two capture steps without recomputing the capture,
and replaying a sparse step offline against the stored cache (the tests
replay one through the CUDA path and the CPU oracle).

Host-side I/O only: tensors are copied between the device and host memory,
nothing is computed.
"""
from __future__ import annotations

import numpy as np
import torch

from . import Stats

__all__ = ["save_cache", "load_cache", "CACHE_FORMAT"]

CACHE_FORMAT = 1


def _host(t: torch.Tensor | None) -> np.ndarray | None:
    if t is None:
        return None
    x = t.detach().cpu().contiguous()
    if x.dtype == torch.float16:
        return x.view(torch.int16).numpy().view(np.uint16)  # f16 bits, exactly
    return x.numpy()


def save_cache(path, *, head_dim: int, block_size: int, scale: float, row_ptr: torch.Tensor,
               col_idx: torch.Tensor, stats: Stats, tile_blocks: torch.Tensor | None = None) -> None:
    """Write the capture step's mask, pairing table and statistics cache to ``path`` (.npz)."""
    B, H, N = stats.m.shape
    D = stats.u.shape[-1]
    arrays = {
        "format": np.array(CACHE_FORMAT, np.int64),
        "shape": np.array([B, H, N, head_dim, D, block_size], np.int64),
        "scale": np.array(scale, np.float64),
        "row_ptr": _host(row_ptr),
        "col_idx": _host(col_idx),
        "m": _host(stats.m),
        "zfull": _host(stats.zfull),
        "zkept": _host(stats.zkept),
        "u": _host(stats.u),
        "u_is_f16": np.array(1 if stats.compressed else 0, np.int64),
    }
    if stats.compressed:
        arrays["u_scale"] = _host(stats.u_scale)
    if tile_blocks is not None:
        arrays["tile_blocks"] = _host(tile_blocks)
    with open(path, "wb") as f:
        np.savez(f, **arrays)


def load_cache(path, device: torch.device | str = "cuda") -> dict:
    """Read a file written by ``save_cache``.  Returns a dict with ``head_dim``, ``block_size``,
    ``scale``, ``shape`` (B, H, N, D), ``row_ptr``, ``col_idx``, ``stats`` (a Stats on
    ``device``) and ``tile_blocks`` (or None)."""
    with np.load(path) as z:
        fmt = int(z["format"])
        if fmt != CACHE_FORMAT:
            raise ValueError(f"cache format {fmt}, expected {CACHE_FORMAT}")
        B, H, N, d, D, bs = (int(x) for x in z["shape"])
        t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(device)
        u = z["u"]
        compressed = bool(int(z["u_is_f16"]))
        u_t = torch.from_numpy(np.ascontiguousarray(u).view(np.int16)).view(torch.float16).to(device) if compressed \
            else t(u)
        stats = Stats(t(z["m"]), t(z["zfull"]), t(z["zkept"]), u_t, t(z["u_scale"]) if compressed else None)
        for name, x, want in (("m", stats.m, (B, H, N)), ("zfull", stats.zfull, (B, H, N)),
                              ("zkept", stats.zkept, (B, H, N)), ("u", stats.u, (B, H, N, D))):
            if tuple(x.shape) != want:
                raise ValueError(f"cache {name} has shape {tuple(x.shape)}, expected {want}")
        nb = -(-N // bs)
        row_ptr = t(z["row_ptr"])
        if row_ptr.numel() != B * H * nb + 1:
            raise ValueError("cache row_ptr does not match the shape")
        return {"head_dim": d, "block_size": bs, "scale": float(z["scale"]), "shape": (B, H, N, D),
                "row_ptr": row_ptr, "col_idx": t(z["col_idx"]), "stats": stats,
                "tile_blocks": t(z["tile_blocks"]) if "tile_blocks" in z else None}
