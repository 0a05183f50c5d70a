"""Every call writes its outputs and workspaces and nothing next to them.

Each output and caller workspace is a view into a larger buffer filled with a
canary value; after the call the canaries before and after the view must be
intact (a stand-in for a memory checker, which is not available on the GPU
pool).  Shapes have ragged tails (N = 1000: a 40-token last block and a
104-row last query tile), padded head dims and both block sizes.
"""
import math

import pytest
import torch

import ultra_sparse_attention_b200 as usa

pytestmark = pytest.mark.gpu

PAD = 4096  # elements of canary on each side (16-byte aligned views for every dtype)
FILL = {torch.int32: -123456789, torch.float32: 7.25, torch.float16: 3.5, torch.bfloat16: 7.0, torch.uint8: 0xA5}


class Canaried:
    """Views into canary-padded device buffers; `check` verifies every pad."""

    def __init__(self, device):
        self.device, self.bufs = device, []

    def __call__(self, shape, dtype):
        n = math.prod(shape)
        buf = torch.full((n + 2 * PAD,), FILL[dtype], dtype=dtype, device=self.device)
        self.bufs.append((buf, n, dtype))
        return buf[PAD:PAD + n].view(*shape)

    def check(self, what):
        torch.cuda.synchronize()
        for i, (buf, n, dtype) in enumerate(self.bufs):
            f = FILL[dtype]
            assert torch.all(buf[:PAD] == f), f"{what}: buffer {i} written before its start"
            assert torch.all(buf[PAD + n:] == f), f"{what}: buffer {i} written past its end"
        assert usa.rt_take_device_error() == 0


def _qkv(B, H, N, d, D, seed, device):
    g = torch.Generator().manual_seed(seed)
    out = []
    for _ in range(3):
        x = torch.zeros(B, H, N, D)
        x[..., :d] = torch.randn(B, H, N, d, generator=g)
        out.append(x.to(torch.bfloat16).to(device))
    return out


CASES = [(2, 3, 1000, 72, 80, 64, 4), (2, 3, 1000, 72, 80, 128, 3), (1, 2, 1000, 64, 64, 64, 5)]


@pytest.mark.parametrize("B,H,N,d,D,bs,keep", CASES)
def test_calls_write_only_their_outputs(cuda_device, B, H, N, d, D, bs, keep):
    q, k, v = _qkv(B, H, N, d, D, N + d + bs, cuda_device)
    nb = -(-N // bs)
    kw = dict(head_dim=d, block_size=bs, scale=d ** -0.5)
    c = Canaried(cuda_device)

    # mask (allocating and fixed-array variants), with the block scores
    rp, ci, sc = c((B * H * nb + 1,), torch.int32), c((B * H * nb * keep,), torch.int32), c((B, H, nb, nb), torch.float32)
    usa.rt_build_block_mask(q, k, keep_blocks=keep, forced_prefix_tokens=100, row_ptr=rp, col_idx=ci,
                            block_scores=sc, **kw)
    c.check("rt_build_block_mask")
    rp2, ci2 = c((B * H * nb + 1,), torch.int32), c((B * H * nb * keep,), torch.int32)
    usa.rt_build_block_mask_static(q, k, keep_blocks=keep, forced_prefix_tokens=100, row_ptr=rp2, col_idx=ci2, **kw)
    c.check("rt_build_block_mask_static")
    assert torch.equal(rp, rp2) and torch.equal(ci, ci2)

    # pairing and capture with caller workspaces
    cap_ws, pair_ws = usa.rt_workspace_bytes(B, H, N, head_dim=d, head_dim_padded=D, block_size=bs)
    tiles = c((B * H, -(-N // 128), 2), torch.int32)
    usa.rt_pair_query_blocks(q, rp, ci, head_dim=d, block_size=bs, tile_blocks=tiles,
                             workspace=c((max(pair_ws, 1),), torch.uint8))
    c.check("rt_pair_query_blocks")
    for compressed in (False, True):
        f = lambda *s: c(s, torch.float32)
        st = (usa.Stats(f(B, H, N), f(B, H, N), f(B, H, N), c((B, H, N, D), torch.float16), f(B, H, N))
              if compressed else usa.Stats(f(B, H, N), f(B, H, N), f(B, H, N), f(B, H, N, D)))
        out = c((B, H, N, D), torch.bfloat16)
        usa.rt_attn_full_capture(q, k, v, row_ptr=rp, col_idx=ci, out=out, stats=st,
                                 workspace=c((cap_ws,), torch.uint8), **kw)
        c.check(f"rt_attn_full_capture (compressed={compressed})")
        for t in (tiles, None):
            out1 = c((B, H, N, D), torch.bfloat16)
            usa.rt_attn_sparse_reshape(q, k, v, row_ptr=rp, col_idx=ci, stats=st, tile_blocks=t, out=out1, **kw)
            c.check(f"rt_attn_sparse_reshape (compressed={compressed}, table={t is not None})")

    # exact-mass mask with its workspace and the block masses
    ws = usa.rt_exact_mask_workspace_bytes(B, H, N, head_dim=d, head_dim_padded=D, block_size=bs)
    rp3, ci3 = c((B * H * nb + 1,), torch.int32), c((B * H * nb * keep,), torch.int32)
    usa.rt_build_block_mask_exact(q, k, v, keep_blocks=keep, forced_prefix_tokens=100, row_ptr=rp3, col_idx=ci3,
                                  block_mass=c((B, H, nb, nb), torch.float32), workspace=c((ws,), torch.uint8), **kw)
    c.check("rt_build_block_mask_exact")

    # token permutation both ways
    perm = torch.randperm(N, generator=torch.Generator().manual_seed(N)).to(torch.int32).to(cuda_device)
    y = c((B, H, N, D), torch.bfloat16)
    usa.rt_permute_tokens(q, perm, out=y, head_dim=d)
    z = c((B, H, N, D), torch.bfloat16)
    usa.rt_permute_tokens(y, perm, inverse=True, out=z, head_dim=d)
    c.check("rt_permute_tokens")
    assert torch.equal(z, q)
