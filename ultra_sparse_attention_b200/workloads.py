"""Seeded synthetic attention inputs for the Re-ttention workloads.

This module only draws numbers. It holds none of the method's arithmetic
(no pooling, no scores, no softmax, no statistics), so the CUDA path and the
CPU oracle can both take their inputs from it.

Re-ttention (project page, "Abstract") is evaluated on the attention layers
of CogVideoX and PixArt DiTs.  Trained weights and prompts are not available
here, so each workload below is a synthetic stand-in with the attention
shapes of those models: batch, heads, tokens, head dim, block size, keep
ratio and the denoising-step schedule (full capture every k-th step, sparse
steps in between; project page, teaser: the statistics are cached at one
denoising step and reused by the following ones).

Every tensor is built in fp32 on the host from one ``torch.Generator``
seeded with the workload's seed, rounded to bf16 (round-to-nearest-even) and
zero-padded from the logical head dim ``d`` to the stored head dim ``D``.
The draw order is fixed: base Q, K, V, then for each later step the drift of
Q, K, V in that order.
"""
from __future__ import annotations

import dataclasses
import math
from fractions import Fraction
from typing import Iterator

import torch

__all__ = [
    "Workload",
    "WORKLOADS",
    "keep_blocks",
    "base_inputs",
    "drift_inputs",
    "denoising_inputs",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    """Shape and input recipe of one synthetic attention workload."""

    name: str
    batch: int
    heads: int
    seq_len: int
    head_dim: int            # logical d (sets the softmax scale 1/sqrt(d))
    head_dim_padded: int     # stored D >= d, columns d..D-1 are zero
    block_size: int          # tokens per query block and per key block
    keep: tuple[Fraction, ...]  # keep ratios (first one is the default)
    forced_prefix_tokens: int   # key blocks overlapping [0, this) are always kept
    steps: int
    capture_every: int
    drift_sigma: float
    kind: str                # "iid", "smooth", "video" or "smooth_outliers"
    seed: int = 0
    # recipe parameters (meaning depends on ``kind``)
    iid_std: float = 1.0
    grid: int = 0            # smooth: side of the square patch grid
    rank: int = 0            # smooth: rank of the shared low-rank signal
    max_freq: int = 3        # smooth: largest integer frequency of a field
    noise_std: float = 0.5   # smooth: additive noise
    outlier_frac: float = 0.0  # smooth_outliers: fraction of K rows with heavy tails
    outlier_dof: int = 3       # smooth_outliers: Student-t degrees of freedom
    text_tokens: int = 0     # video: leading text tokens
    frames: int = 0          # video: latent frames
    frame_h: int = 0
    frame_w: int = 0
    frame_corr: float = 0.9  # video: correlation of a patch across frames

    @property
    def n_blocks(self) -> int:
        return -(-self.seq_len // self.block_size)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.head_dim)

    def keep_blocks(self, ratio: Fraction | None = None) -> int:
        return keep_blocks(self.n_blocks, self.keep[0] if ratio is None else ratio)

    def capture_steps(self) -> list[int]:
        return [t for t in range(self.steps) if t % self.capture_every == 0]


def keep_blocks(n_blocks: int, ratio: Fraction) -> int:
    """Kept key blocks per query block: ceil(n_blocks * ratio), clamped to [1, n_blocks].

    Integer arithmetic, so 278 blocks at 1/32 keep 9, at 1/16 keep 18.
    """
    ratio = Fraction(ratio)
    k = -(-(n_blocks * ratio.numerator) // ratio.denominator)
    return max(1, min(n_blocks, k))


_F = Fraction
WORKLOADS: dict[str, Workload] = {
    # B=1, H=2, N=512, d=64, i.i.d. N(0,1)/sqrt(64); keep 2 of 8 blocks.
    "tiny": Workload(
        name="tiny", batch=1, heads=2, seq_len=512, head_dim=64, head_dim_padded=64,
        block_size=64, keep=(_F(1, 4),), forced_prefix_tokens=0, steps=3,
        capture_every=3, drift_sigma=0.05, kind="iid", iid_std=1.0 / 8.0),
    # PixArt-like image: 64x64 patch grid, d=72 stored as 80, rank-32 smooth signal.
    "image": Workload(
        name="image", batch=2, heads=16, seq_len=4096, head_dim=72, head_dim_padded=80,
        block_size=64, keep=(_F(1, 16),), forced_prefix_tokens=0, steps=20,
        capture_every=5, drift_sigma=0.03, kind="smooth", grid=64, rank=32),
    # CogVideoX-2B-like video: 226 text tokens + 13 frames of 30x45 patches.
    "video2b": Workload(
        name="video2b", batch=1, heads=30, seq_len=17776, head_dim=64, head_dim_padded=64,
        block_size=64, keep=(_F(1, 32),), forced_prefix_tokens=226, steps=10,
        capture_every=5, drift_sigma=0.02, kind="video", text_tokens=226, frames=13,
        frame_h=30, frame_w=45),
    # CogVideoX-5B-like video: same token layout, 48 heads, keep-ratio sweep.
    "video5b": Workload(
        name="video5b", batch=1, heads=48, seq_len=17776, head_dim=64, head_dim_padded=64,
        block_size=64, keep=(_F(1, 32), _F(1, 16), _F(1, 8), _F(1, 4), _F(1, 1)),
        forced_prefix_tokens=226, steps=2, capture_every=2, drift_sigma=0.02, kind="video",
        text_tokens=226, frames=13, frame_h=30, frame_w=45),
    # High-resolution image: 128x128 grid, 128-token blocks, heavy-tailed outlier keys.
    "long": Workload(
        name="long", batch=1, heads=16, seq_len=16384, head_dim=72, head_dim_padded=80,
        block_size=128, keep=(_F(1, 32),), forced_prefix_tokens=0, steps=20,
        capture_every=10, drift_sigma=0.03, kind="smooth_outliers", grid=128, rank=64,
        outlier_frac=0.01, outlier_dof=3),
}


def _to_bf16_padded(x: torch.Tensor, dpad: int) -> torch.Tensor:
    """fp32 [..., d] -> bf16 [..., D] (RNE), zero in columns d..D-1."""
    d = x.shape[-1]
    out = torch.zeros(*x.shape[:-1], dpad, dtype=torch.bfloat16)
    out[..., :d] = x.to(torch.bfloat16)
    return out


def _smooth_fields(w: Workload, gen: torch.Generator) -> torch.Tensor:
    """Rank-r spatially smooth fields on the w.grid x w.grid patch grid (row-major).

    Column j is sqrt(2)*cos(2*pi*(fx*x + fy*y)/G + phi) with integer
    frequencies |fx|,|fy| <= max_freq, not both zero, and a uniform phase,
    so each column has unit variance over the grid.  Returns [B*H, N, r].
    """
    G, r, f = w.grid, w.rank, w.max_freq
    assert G * G == w.seq_len
    bh = w.batch * w.heads
    freqs = torch.randint(-f, f + 1, (bh, r, 2), generator=gen)
    zero = (freqs[..., 0] == 0) & (freqs[..., 1] == 0)
    freqs[..., 0] = torch.where(zero, torch.ones_like(freqs[..., 0]), freqs[..., 0])
    phase = torch.rand(bh, r, generator=gen, dtype=torch.float64) * (2 * math.pi)
    idx = torch.arange(w.seq_len, dtype=torch.float64)
    xs, ys = idx % G, torch.div(idx, G, rounding_mode="floor")
    arg = (2 * math.pi / G) * (xs[None, :, None] * freqs[:, None, :, 0].double()
                               + ys[None, :, None] * freqs[:, None, :, 1].double()) + phase[:, None, :]
    return (math.sqrt(2.0) * torch.cos(arg)).float()


def _student_t(shape, dof: int, gen: torch.Generator) -> torch.Tensor:
    z = torch.randn(*shape, generator=gen)
    chi2 = (torch.randn(*shape, dof, generator=gen) ** 2).sum(-1)
    return z / torch.sqrt(chi2 / dof)


def base_inputs(w: Workload, gen: torch.Generator | None = None):
    """Q, K, V of the first denoising step: bf16 [B, H, N, D] CPU tensors.

    If ``gen`` is None a fresh generator seeded with ``w.seed`` is used; the
    generator is advanced so later drift draws continue the same stream.
    """
    if gen is None:
        gen = torch.Generator().manual_seed(w.seed)
    B, H, N, d, D = w.batch, w.heads, w.seq_len, w.head_dim, w.head_dim_padded
    if w.kind == "iid":
        qkv = [torch.randn(B, H, N, d, generator=gen) * w.iid_std for _ in range(3)]
    elif w.kind in ("smooth", "smooth_outliers"):
        fields = _smooth_fields(w, gen)                       # [BH, N, r], shared by Q, K, V
        qkv = []
        for _ in range(3):
            mix = torch.randn(B * H, d, w.rank, generator=gen) / math.sqrt(w.rank)
            x = torch.bmm(fields, mix.transpose(1, 2))
            x += torch.randn(B * H, N, d, generator=gen) * w.noise_std
            qkv.append(x.view(B, H, N, d))
        if w.kind == "smooth_outliers":
            n_out = int(round(w.outlier_frac * N))
            k = qkv[1].view(B * H, N, d)
            for i in range(B * H):
                rows = torch.randperm(N, generator=gen)[:n_out]
                k[i, rows] += _student_t((n_out, d), w.outlier_dof, gen)
    elif w.kind == "video":
        T, F, P = w.text_tokens, w.frames, w.frame_h * w.frame_w
        assert T + F * P == N
        base = torch.randn(B * H, 1, P, d, generator=gen)          # per-patch, shared by frames and Q/K/V
        eps = torch.randn(B * H, F, P, d, generator=gen)           # per frame and patch, shared by Q/K/V
        frame = math.sqrt(w.frame_corr) * base + math.sqrt(1.0 - w.frame_corr) * eps
        frame = frame.reshape(B * H, F * P, d)
        qkv = []
        for _ in range(3):
            x = torch.empty(B * H, N, d)
            x[:, :T] = torch.randn(B * H, T, d, generator=gen)
            x[:, T:] = frame + torch.randn(B * H, F * P, d, generator=gen)
            qkv.append(x.view(B, H, N, d))
    else:
        raise ValueError(f"unknown workload kind {w.kind!r}")
    return tuple(_to_bf16_padded(x, D) for x in qkv)


def drift_inputs(w: Workload, qkv, gen: torch.Generator):
    """Next step's Q, K, V: bf16(X + N(0, sigma^2)) on the logical columns."""
    d = w.head_dim
    out = []
    for x in qkv:
        y = x.clone()
        noise = torch.randn(*x.shape[:-1], d, generator=gen) * w.drift_sigma
        y[..., :d] = (x[..., :d].float() + noise).to(torch.bfloat16)
        out.append(y)
    return tuple(out)


def denoising_inputs(w: Workload, steps: int | None = None) -> Iterator[tuple]:
    """Yield (step, q, k, v) for steps 0..steps-1 from one seeded stream."""
    gen = torch.Generator().manual_seed(w.seed)
    qkv = base_inputs(w, gen)
    n = w.steps if steps is None else steps
    for t in range(n):
        if t > 0:
            qkv = drift_inputs(w, qkv, gen)
        yield (t, *qkv)
