"""Python binding of librettention.so: Re-ttention's attention path on B200.

Argument marshalling only.  Every step of the path (pooling, block scores,
top-k, full attention with the statistics cache, sparse attention with the
reshape) runs in the library's CUDA kernels; PyTorch only supplies device
memory and the current stream.  There is no CPU fallback: if the library
cannot be built or loaded, every call raises.

The functions carry the C ABI's names (see include/rettention.h):

    rt_build_block_mask(q, k, ...)      -> (row_ptr, col_idx)
    rt_attn_full_capture(q, k, v, ...)  -> (out, stats)
    rt_attn_sparse_reshape(q, k, v, ...) -> out
    rt_pair_query_blocks(q, row_ptr, col_idx, ...) -> tile_blocks  (schedule for the sparse step)
"""
from __future__ import annotations

import ctypes
import threading
from dataclasses import dataclass

import torch

from . import build as _build

__all__ = [
    "RtError",
    "Stats",
    "library_path",
    "load_library",
    "rt_build_block_mask",
    "rt_build_block_mask_exact",
    "rt_exact_mask_workspace_bytes",
    "rt_hilbert_order",
    "rt_permute_tokens",
    "rt_attn_full_capture",
    "rt_attn_sparse_reshape",
    "rt_pair_query_blocks",
    "rt_workspace_bytes",
    "rt_status_string",
    "rt_abi_version",
    "rt_take_device_error",
    "rt_selftest_wait_timeout",
    "rt_selftest_exp2_poly",
    "rt_build_block_mask_static",
    "STATIC_POOL_FLOATS",
]

# Capacity of rt_build_block_mask_static's fixed workspace (fp32 values).
STATIC_POOL_FLOATS = 2 * 1024 * 1024

RT_OK = 0
RT_ERR_INVALID_ARGUMENT = 1
RT_ERR_UNSUPPORTED = 2
RT_ERR_CUDA = 3
RT_ERR_TIMEOUT = 4


class RtError(RuntimeError):
    """A librettention call returned a status other than RT_OK."""

    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {rt_status_string(status)}")


class RtShape(ctypes.Structure):
    _fields_ = [(name, ctypes.c_int32) for name in
                ("batch", "heads", "seq_len", "head_dim", "head_dim_padded", "block_size")]


_lock = threading.Lock()
_lib = None


def library_path() -> str:
    return _build.LIB


def load_library(build_if_needed: bool = True) -> ctypes.CDLL:
    """Load librettention.so, compiling it first if it is missing or stale."""
    global _lib
    with _lock:
        if _lib is None:
            if build_if_needed:
                _build.build()
            lib = ctypes.CDLL(_build.LIB)
            vp, i32, f32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_int64
            shp = ctypes.POINTER(RtShape)
            lib.rt_build_block_mask.argtypes = [shp, vp, vp, f32, i32, i32, vp, vp, vp, vp]
            sz = ctypes.c_size_t
            lib.rt_attn_full_capture.argtypes = [shp, vp, vp, vp, f32, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]
            lib.rt_attn_sparse_reshape.argtypes = [shp, vp, vp, vp, f32, vp, vp, vp, vp, vp, vp, vp, vp, vp]
            lib.rt_attn_full_capture_u16.argtypes = [shp, vp, vp, vp, f32, vp, vp, vp, vp, vp, vp, vp, vp, vp, sz,
                                                     vp]
            lib.rt_attn_sparse_reshape_u16.argtypes = [shp, vp, vp, vp, f32, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                                       vp]
            lib.rt_pair_query_blocks.argtypes = [shp, vp, vp, vp, vp, sz, vp]
            lib.rt_workspace_bytes.argtypes = [shp, ctypes.POINTER(sz), ctypes.POINTER(sz)]
            lib.rt_build_block_mask_exact.argtypes = [shp, vp, vp, vp, f32, i32, i32, vp, vp, vp, vp, sz, vp]
            lib.rt_exact_mask_workspace_bytes.argtypes = [shp, ctypes.POINTER(sz)]
            lib.rt_hilbert_order.argtypes = [i32, i32, i32, i32, vp]
            lib.rt_permute_tokens.argtypes = [shp, vp, vp, i32, vp, vp]
            lib.rt_status_string.argtypes = [ctypes.c_int]
            lib.rt_status_string.restype = ctypes.c_char_p
            lib.rt_abi_version.argtypes = []
            lib.rt_abi_version.restype = i32
            lib.rt_take_device_error.argtypes = [ctypes.POINTER(i32)]
            lib.rt_selftest_wait_timeout.argtypes = [i64, vp]
            lib.rt_selftest_exp2_poly.argtypes = [vp, vp, i32, vp]
            lib.rt_build_block_mask_static.argtypes = [shp, vp, vp, f32, i32, i32, vp, vp, vp, vp]
            lib.rt_build_block_mask_static.restype = ctypes.c_int
            for fn in ("rt_build_block_mask", "rt_attn_full_capture", "rt_attn_sparse_reshape",
                       "rt_attn_full_capture_u16", "rt_attn_sparse_reshape_u16",
                       "rt_build_block_mask_exact", "rt_exact_mask_workspace_bytes",
                       "rt_hilbert_order", "rt_permute_tokens",
                       "rt_pair_query_blocks", "rt_workspace_bytes", "rt_take_device_error",
                       "rt_selftest_wait_timeout", "rt_selftest_exp2_poly"):
                getattr(lib, fn).restype = ctypes.c_int
            _lib = lib
    return _lib


def rt_status_string(status: int) -> str:
    return load_library().rt_status_string(int(status)).decode()


def rt_abi_version() -> int:
    return int(load_library().rt_abi_version())


@dataclass
class Stats:
    """Statistics cache of a capture step (device).

    ``u`` is fp32, or f16 for the compressed cache, where the residual numerator is
    ``u * u_scale[..., None]`` with one power-of-two scale per row."""

    m: torch.Tensor       # [B, H, N]   row max of the scaled scores
    zfull: torch.Tensor   # [B, H, N]   full softmax denominator
    zkept: torch.Tensor   # [B, H, N]   kept-key part of it
    u: torch.Tensor       # [B, H, N, D] masked-out residual numerator (fp32, or f16 with u_scale)
    u_scale: torch.Tensor | None = None  # [B, H, N] fp32, compressed cache only

    @property
    def compressed(self) -> bool:
        return self.u.dtype == torch.float16

    def residual(self) -> torch.Tensor:
        """U as fp32 [B, H, N, D] (decoded from the compressed form if needed)."""
        return self.u.float() * self.u_scale[..., None] if self.compressed else self.u


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _nbytes(t: torch.Tensor | None) -> int:
    return 0 if t is None else t.numel() * t.element_size()


def _stream_handle(device: torch.device, stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream if isinstance(stream, torch.cuda.Stream) else int(stream))


def _check_qkv(name: str, *xs: torch.Tensor) -> tuple[int, int, int, int]:
    shape = None
    for x in xs:
        if not isinstance(x, torch.Tensor) or not x.is_cuda:
            raise ValueError(f"{name}: Q/K/V must be CUDA tensors")
        if x.dtype != torch.bfloat16 or x.dim() != 4 or not x.is_contiguous():
            raise ValueError(f"{name}: Q/K/V must be contiguous bf16 [B, H, N, D]")
        if shape is None:
            shape = tuple(x.shape)
        elif tuple(x.shape) != shape:
            raise ValueError(f"{name}: Q/K/V shapes differ")
        if x.device != xs[0].device:
            raise ValueError(f"{name}: Q/K/V are on different devices")
    return shape


def _check_buf(name: str, what: str, t: torch.Tensor, dtype: torch.dtype, device: torch.device,
               shape: tuple | None = None, min_numel: int | None = None):
    """A caller-supplied buffer the library reads or writes: the C side cannot see its size."""
    if not isinstance(t, torch.Tensor) or t.device != device or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name}: {what} must be a contiguous {dtype} tensor on {device}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: {what} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if min_numel is not None and t.numel() < min_numel:
        raise ValueError(f"{name}: {what} holds {t.numel()} elements, needs at least {min_numel}")


def _check_stats(name: str, st: "Stats", dims, device: torch.device):
    B, H, N, D = dims
    for what, t in (("stats.m", st.m), ("stats.zfull", st.zfull), ("stats.zkept", st.zkept)):
        _check_buf(name, what, t, torch.float32, device, shape=(B, H, N))
    if isinstance(st.u, torch.Tensor) and st.u.dtype == torch.float16:
        _check_buf(name, "stats.u", st.u, torch.float16, device, shape=(B, H, N, D))
        _check_buf(name, "stats.u_scale", st.u_scale, torch.float32, device, shape=(B, H, N))
    else:
        _check_buf(name, "stats.u", st.u, torch.float32, device, shape=(B, H, N, D))


def _shape(dims, head_dim: int, block_size: int) -> RtShape:
    B, H, N, D = dims
    return RtShape(B, H, N, head_dim, D, block_size)


def _call(status: int, what: str):
    if status != RT_OK:
        raise RtError(status, what)


def rt_build_block_mask(q: torch.Tensor, k: torch.Tensor, *, head_dim: int, block_size: int, scale: float,
                        keep_blocks: int, forced_prefix_tokens: int = 0, row_ptr: torch.Tensor | None = None,
                        col_idx: torch.Tensor | None = None, block_scores: torch.Tensor | bool | None = None,
                        stream=None):
    """Kept key blocks per query block (CSR).  Returns (row_ptr, col_idx[, block_scores])."""
    name = "rt_build_block_mask"
    dims = _check_qkv(name, q, k)
    B, H, N, D = dims
    nb = -(-N // block_size) if block_size > 0 else 0
    dev = q.device
    if row_ptr is None:
        row_ptr = torch.empty(B * H * nb + 1, dtype=torch.int32, device=dev)
    if col_idx is None:
        col_idx = torch.empty(B * H * nb * max(keep_blocks, 0), dtype=torch.int32, device=dev)
    _check_buf(name, "row_ptr", row_ptr, torch.int32, dev, min_numel=B * H * nb + 1)
    _check_buf(name, "col_idx", col_idx, torch.int32, dev, min_numel=B * H * nb * max(keep_blocks, 0))
    want_scores = block_scores is True
    if want_scores:
        block_scores = torch.empty(B, H, nb, nb, dtype=torch.float32, device=dev)
    elif block_scores is False:
        block_scores = None
    if block_scores is not None:
        _check_buf(name, "block_scores", block_scores, torch.float32, dev, min_numel=B * H * nb * nb)
    shape = _shape(dims, head_dim, block_size)
    with torch.cuda.device(dev):
        _call(load_library().rt_build_block_mask(ctypes.byref(shape), _ptr(q), _ptr(k), float(scale),
                                                 int(keep_blocks), int(forced_prefix_tokens), _ptr(row_ptr),
                                                 _ptr(col_idx), _ptr(block_scores), _stream_handle(dev, stream)),
              name)
    return (row_ptr, col_idx, block_scores) if want_scores else (row_ptr, col_idx)


def rt_build_block_mask_exact(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, head_dim: int,
                              block_size: int, scale: float, keep_blocks: int, forced_prefix_tokens: int = 0,
                              row_ptr: torch.Tensor | None = None, col_idx: torch.Tensor | None = None,
                              block_mass: torch.Tensor | bool | None = None, workspace: torch.Tensor | None = None,
                              stream=None):
    """Kept key blocks chosen by exact block attention mass (CSR).  Returns (row_ptr, col_idx[, block_mass])."""
    name = "rt_build_block_mask_exact"
    dims = _check_qkv(name, q, k, v)
    B, H, N, D = dims
    nb = -(-N // block_size) if block_size > 0 else 0
    dev = q.device
    if row_ptr is None:
        row_ptr = torch.empty(B * H * nb + 1, dtype=torch.int32, device=dev)
    if col_idx is None:
        col_idx = torch.empty(B * H * nb * max(keep_blocks, 0), dtype=torch.int32, device=dev)
    _check_buf(name, "row_ptr", row_ptr, torch.int32, dev, min_numel=B * H * nb + 1)
    _check_buf(name, "col_idx", col_idx, torch.int32, dev, min_numel=B * H * nb * max(keep_blocks, 0))
    want_mass = block_mass is True
    if want_mass:
        block_mass = torch.empty(B, H, nb, nb, dtype=torch.float32, device=dev)
    elif block_mass is False:
        block_mass = None
    if block_mass is not None:
        _check_buf(name, "block_mass", block_mass, torch.float32, dev, min_numel=B * H * nb * nb)
    if workspace is not None:
        _check_buf(name, "workspace", workspace, torch.uint8, dev)
    shape = _shape(dims, head_dim, block_size)
    with torch.cuda.device(dev):
        _call(load_library().rt_build_block_mask_exact(
            ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), float(scale), int(keep_blocks),
            int(forced_prefix_tokens), _ptr(row_ptr), _ptr(col_idx), _ptr(block_mass), _ptr(workspace),
            _nbytes(workspace), _stream_handle(dev, stream)), name)
    return (row_ptr, col_idx, block_mass) if want_mass else (row_ptr, col_idx)


def rt_exact_mask_workspace_bytes(batch: int, heads: int, seq_len: int, *, head_dim: int, head_dim_padded: int,
                                  block_size: int) -> int:
    """Workspace bytes rt_build_block_mask_exact needs for this shape."""
    shape = RtShape(batch, heads, seq_len, head_dim, head_dim_padded, block_size)
    n = ctypes.c_size_t(0)
    _call(load_library().rt_exact_mask_workspace_bytes(ctypes.byref(shape), ctypes.byref(n)),
          "rt_exact_mask_workspace_bytes")
    return int(n.value)


def rt_hilbert_order(grid_h: int, grid_w: int, *, frames: int = 1, prefix_tokens: int = 0) -> torch.Tensor:
    """Hilbert-curve token order (host int32 [prefix + frames*grid_h*grid_w]): position t of the
    reordered sequence takes token perm[t] of the row-major one."""
    n = prefix_tokens + frames * grid_h * grid_w
    perm = torch.empty(max(n, 0), dtype=torch.int32)
    _call(load_library().rt_hilbert_order(int(prefix_tokens), int(frames), int(grid_h), int(grid_w),
                                          ctypes.c_void_p(perm.data_ptr())), "rt_hilbert_order")
    return perm


def rt_permute_tokens(x: torch.Tensor, perm: torch.Tensor, *, inverse: bool = False, head_dim: int | None = None,
                      out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Token-reordered copy of bf16 [B, H, N, D] ``x``: out[..., t, :] = x[..., perm[t], :], or with
    ``inverse`` out[..., perm[t], :] = x[..., t, :].  ``perm``: int32 [N] on x's device."""
    name = "rt_permute_tokens"
    dims = _check_qkv(name, x)
    B, H, N, D = dims
    dev = x.device
    _check_buf(name, "perm", perm, torch.int32, dev, shape=(N,))
    if out is None:
        out = torch.empty_like(x)
    _check_buf(name, "out", out, torch.bfloat16, dev, shape=dims)
    shape = _shape(dims, head_dim or D, 64)
    with torch.cuda.device(dev):
        _call(load_library().rt_permute_tokens(ctypes.byref(shape), _ptr(x), _ptr(perm), 1 if inverse else 0,
                                               _ptr(out), _stream_handle(dev, stream)), name)
    return out


def rt_attn_full_capture(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, head_dim: int, block_size: int,
                         scale: float, row_ptr: torch.Tensor, col_idx: torch.Tensor,
                         out: torch.Tensor | None = None, stats: Stats | None = None,
                         workspace: torch.Tensor | None = None, compressed: bool = False, stream=None):
    """Full attention at a capture step plus the statistics cache.  Returns (out, stats).

    ``compressed`` (or a ``stats`` whose ``u`` is f16) writes the compressed cache
    (rt_attn_full_capture_u16).  ``workspace`` (uint8, device, at least
    rt_workspace_bytes(...)[0] bytes) keeps the library from taking a transient
    buffer from its pool."""
    name = "rt_attn_full_capture"
    dims = _check_qkv(name, q, k, v)
    B, H, N, D = dims
    dev = q.device
    if out is None:
        out = torch.empty_like(q)
    if stats is None:
        f = lambda *shp, dt=torch.float32: torch.empty(*shp, dtype=dt, device=dev)
        stats = (Stats(f(B, H, N), f(B, H, N), f(B, H, N), f(B, H, N, D, dt=torch.float16), f(B, H, N))
                 if compressed else Stats(f(B, H, N), f(B, H, N), f(B, H, N), f(B, H, N, D)))
    _check_buf(name, "out", out, torch.bfloat16, dev, shape=dims)
    _check_stats(name, stats, dims, dev)
    _check_buf(name, "row_ptr", row_ptr, torch.int32, dev)
    _check_buf(name, "col_idx", col_idx, torch.int32, dev)
    if workspace is not None:
        _check_buf(name, "workspace", workspace, torch.uint8, dev)
    shape = _shape(dims, head_dim, block_size)
    lib = load_library()
    with torch.cuda.device(dev):
        head = (ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), float(scale), _ptr(row_ptr), _ptr(col_idx),
                _ptr(out), _ptr(stats.m), _ptr(stats.zfull), _ptr(stats.zkept))
        tail = (_ptr(workspace), _nbytes(workspace), _stream_handle(dev, stream))
        if stats.compressed:
            _call(lib.rt_attn_full_capture_u16(*head, _ptr(stats.u), _ptr(stats.u_scale), *tail),
                  "rt_attn_full_capture_u16")
        else:
            _call(lib.rt_attn_full_capture(*head, _ptr(stats.u), *tail), name)
    return out, stats


def rt_attn_sparse_reshape(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, *, head_dim: int, block_size: int,
                           scale: float, row_ptr: torch.Tensor, col_idx: torch.Tensor, stats: Stats | None,
                           tile_blocks: torch.Tensor | None = None, out: torch.Tensor | None = None,
                           stream=None) -> torch.Tensor:
    """Sparse step over the kept blocks, reshaped with ``stats`` (plain block-sparse if None).

    ``tile_blocks`` (from rt_pair_query_blocks) groups the query blocks into the
    kernel's 128-row tiles; None takes neighbouring blocks.  The result is the same."""
    name = "rt_attn_sparse_reshape"
    dims = _check_qkv(name, q, k, v)
    dev = q.device
    if tile_blocks is not None:
        _check_buf(name, "tile_blocks", tile_blocks, torch.int32, dev, shape=_tile_table_shape(dims))
    if out is None:
        out = torch.empty_like(q)
    _check_buf(name, "out", out, torch.bfloat16, dev, shape=dims)
    if stats is not None:
        _check_stats(name, stats, dims, dev)
    _check_buf(name, "row_ptr", row_ptr, torch.int32, dev)
    _check_buf(name, "col_idx", col_idx, torch.int32, dev)
    shape = _shape(dims, head_dim, block_size)
    s = stats
    lib = load_library()
    with torch.cuda.device(dev):
        head = (ctypes.byref(shape), _ptr(q), _ptr(k), _ptr(v), float(scale), _ptr(row_ptr), _ptr(col_idx),
                _ptr(tile_blocks), _ptr(s.m if s else None), _ptr(s.zfull if s else None),
                _ptr(s.zkept if s else None))
        if s is not None and s.compressed:
            _call(lib.rt_attn_sparse_reshape_u16(*head, _ptr(s.u), _ptr(s.u_scale), _ptr(out),
                                                 _stream_handle(dev, stream)), "rt_attn_sparse_reshape_u16")
        else:
            _call(lib.rt_attn_sparse_reshape(*head, _ptr(s.u if s else None), _ptr(out), _stream_handle(dev, stream)),
                  name)
    return out


def _tile_table_shape(dims) -> tuple[int, int, int]:
    B, H, N, _ = dims
    return (B * H, -(-N // 128), 2)


def rt_pair_query_blocks(q: torch.Tensor, row_ptr: torch.Tensor, col_idx: torch.Tensor, *, head_dim: int,
                         block_size: int, tile_blocks: torch.Tensor | None = None,
                         workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Group each head's query blocks into the sparse kernel's 128-row tiles (``q`` gives the shape).

    Returns int32 [B*H, ceil(N/128), 2]: the query blocks of each tile, -1 for an empty half.
    ``workspace`` (uint8, device, at least rt_workspace_bytes(...)[1] bytes) keeps the
    library from taking a transient buffer from its pool."""
    name = "rt_pair_query_blocks"
    dims = _check_qkv(name, q)
    dev = q.device
    if tile_blocks is None:
        tile_blocks = torch.empty(_tile_table_shape(dims), dtype=torch.int32, device=dev)
    _check_buf(name, "tile_blocks", tile_blocks, torch.int32, dev, shape=_tile_table_shape(dims))
    _check_buf(name, "row_ptr", row_ptr, torch.int32, dev)
    _check_buf(name, "col_idx", col_idx, torch.int32, dev)
    if workspace is not None:
        _check_buf(name, "workspace", workspace, torch.uint8, dev)
    shape = _shape(dims, head_dim, block_size)
    with torch.cuda.device(dev):
        _call(load_library().rt_pair_query_blocks(ctypes.byref(shape), _ptr(row_ptr), _ptr(col_idx),
                                                  _ptr(tile_blocks), _ptr(workspace), _nbytes(workspace),
                                                  _stream_handle(dev, stream)),
              name)
    return tile_blocks


def rt_workspace_bytes(batch: int, heads: int, seq_len: int, *, head_dim: int, head_dim_padded: int,
                       block_size: int) -> tuple[int, int]:
    """Device workspace bytes of (rt_attn_full_capture, rt_pair_query_blocks) for a shape."""
    shape = RtShape(batch, heads, seq_len, head_dim, head_dim_padded, block_size)
    cap, pair = ctypes.c_size_t(0), ctypes.c_size_t(0)
    _call(load_library().rt_workspace_bytes(ctypes.byref(shape), ctypes.byref(cap), ctypes.byref(pair)),
          "rt_workspace_bytes")
    return int(cap.value), int(pair.value)


def rt_take_device_error() -> int:
    """Read and clear the library's device status word (synchronises the device)."""
    code = ctypes.c_int32(0)
    _call(load_library().rt_take_device_error(ctypes.byref(code)), "rt_take_device_error")
    return int(code.value)


def rt_selftest_wait_timeout(timeout_ns: int, stream=None):
    """Launch the bounded-wait self test (records RT_ERR_TIMEOUT in the status word)."""
    dev = torch.device("cuda", torch.cuda.current_device())
    _call(load_library().rt_selftest_wait_timeout(int(timeout_ns), _stream_handle(dev, stream)),
          "rt_selftest_wait_timeout")


def rt_selftest_exp2_poly(x: torch.Tensor, stream=None) -> torch.Tensor:
    """2^x by the capture kernel's FMA-pipe exponential (fp32 CUDA tensor in, same shape out)."""
    if not isinstance(x, torch.Tensor) or not x.is_cuda or x.dtype != torch.float32 or not x.is_contiguous():
        raise ValueError("rt_selftest_exp2_poly: x must be a contiguous fp32 CUDA tensor")
    y = torch.empty_like(x)
    with torch.cuda.device(x.device):
        _call(load_library().rt_selftest_exp2_poly(_ptr(x), _ptr(y), int(x.numel()),
                                                   _stream_handle(x.device, stream)), "rt_selftest_exp2_poly")
    return y


def rt_build_block_mask_static(q: torch.Tensor, k: torch.Tensor, *, head_dim: int, block_size: int, scale: float,
                               keep_blocks: int, forced_prefix_tokens: int = 0, row_ptr: torch.Tensor | None = None,
                               col_idx: torch.Tensor | None = None, block_scores: torch.Tensor | None = None,
                               stream=None):
    """rt_build_block_mask without any device allocation inside the library.

    For callers that cannot let the library allocate (a framework that owns all
    device memory through its own pool, loops that must not block in an
    allocator).  The workspace is a fixed 8 MiB array of the library, shared
    by every call on a device: calls must not overlap on the GPU.  Pass
    preallocated ``row_ptr`` / ``col_idx`` to avoid allocations on the Python
    side as well.  Shapes with 2*B*H*n_blocks*D > STATIC_POOL_FLOATS raise.
    """
    name = "rt_build_block_mask_static"
    dims = _check_qkv(name, q, k)
    B, H, N, D = dims
    nb = -(-N // block_size) if block_size > 0 else 0
    if 2 * B * H * nb * D > STATIC_POOL_FLOATS:
        raise ValueError(f"{name}: workspace needs {2 * B * H * nb * D} fp32 values, "
                         f"the fixed array holds {STATIC_POOL_FLOATS}")
    dev = q.device
    if row_ptr is None:
        row_ptr = torch.empty(B * H * nb + 1, dtype=torch.int32, device=dev)
    if col_idx is None:
        col_idx = torch.empty(B * H * nb * max(keep_blocks, 0), dtype=torch.int32, device=dev)
    _check_buf(name, "row_ptr", row_ptr, torch.int32, dev, min_numel=B * H * nb + 1)
    _check_buf(name, "col_idx", col_idx, torch.int32, dev, min_numel=B * H * nb * max(keep_blocks, 0))
    if block_scores is not None:
        _check_buf(name, "block_scores", block_scores, torch.float32, dev, min_numel=B * H * nb * nb)
    shape = _shape(dims, head_dim, block_size)
    with torch.cuda.device(dev):
        _call(load_library().rt_build_block_mask_static(ctypes.byref(shape), _ptr(q), _ptr(k), float(scale),
                                                        int(keep_blocks), int(forced_prefix_tokens), _ptr(row_ptr),
                                                        _ptr(col_idx), _ptr(block_scores),
                                                        _stream_handle(dev, stream)),
              name)
    return row_ptr, col_idx
