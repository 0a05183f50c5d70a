"""rt_build_block_mask_static: the mask builder for callers that cannot let a
library allocate device memory (a framework that owns all device memory
through its own pool, or a loop that must never block in an allocator).

It keeps its workspace in a fixed array of the library instead of taking a
buffer from the allocator, so it must give exactly what rt_build_block_mask
gives.  Two calls in a row with different inputs also show that the shared
workspace carries nothing stale from one call into the next.  This file is
collected last so that a failing run stopped at the first failure has
already run every other test.
"""
import ctypes

import pytest
import torch

import ultra_sparse_attention_b200 as usa
from ultra_sparse_attention_b200 import RtShape
from ultra_sparse_attention_b200.workloads import WORKLOADS, base_inputs

pytestmark = pytest.mark.gpu


def _call(fn, q, k, bs, d, keep, forced, scale):
    B, H, N, D = q.shape
    nb = -(-N // bs)
    rp = torch.full((B * H * nb + 1,), -7, dtype=torch.int32, device=q.device)
    ci = torch.full((B * H * nb * keep,), -7, dtype=torch.int32, device=q.device)
    sc = torch.full((B, H, nb, nb), float("nan"), dtype=torch.float32, device=q.device)
    shape = RtShape(B, H, N, d, D, bs)
    stream = ctypes.c_void_p(torch.cuda.current_stream(q.device).cuda_stream)
    st = fn(ctypes.byref(shape), ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), scale, keep, forced,
            ctypes.c_void_p(rp.data_ptr()), ctypes.c_void_p(ci.data_ptr()), ctypes.c_void_p(sc.data_ptr()), stream)
    assert st == usa.RT_OK, usa.rt_status_string(st)
    return rp, ci, sc


def _seeded_qk(B, H, N, D, d, seed, device):
    g = torch.Generator().manual_seed(seed)
    q = torch.zeros(B, H, N, D, dtype=torch.bfloat16)
    k = torch.zeros(B, H, N, D, dtype=torch.bfloat16)
    q[..., :d] = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    k[..., :d] = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    return q.to(device), k.to(device)


def test_static_mask_equals_allocating_mask_on_two_calls_in_a_row(cuda_device):
    lib = usa.load_library()
    img = WORKLOADS["image"]
    cases = [
        # (q, k, block size, d, keep, forced prefix tokens)
        (*[x.to(cuda_device) for x in base_inputs(img)[:2]], 64, 72, img.keep_blocks(), 0),
        (*_seeded_qk(1, 48, 17776, 64, 64, 11, cuda_device), 64, 64, 9, 226),   # near the workspace limit
        (*_seeded_qk(2, 3, 1000, 80, 72, 12, cuda_device), 128, 72, 3, 100),    # ragged tail, 128-token blocks
    ]
    for q, k, bs, d, keep, forced in cases:
        scale = d ** -0.5
        first = _call(lib.rt_build_block_mask_static, q, k, bs, d, keep, forced, scale)
        # second call in a row on other inputs: nothing of the first may leak into it
        q2, k2 = k.flip(2).contiguous(), q.flip(2).contiguous()
        second = _call(lib.rt_build_block_mask_static, q2, k2, bs, d, keep, forced, scale)
        want1 = _call(lib.rt_build_block_mask, q, k, bs, d, keep, forced, scale)
        want2 = _call(lib.rt_build_block_mask, q2, k2, bs, d, keep, forced, scale)
        torch.cuda.synchronize()
        for got, want in ((first, want1), (second, want2)):
            assert torch.equal(got[0], want[0])       # row_ptr
            assert torch.equal(got[1], want[1])       # kept blocks, bit-exact
            assert torch.equal(got[2], want[2])       # block scores, same kernels
        assert not torch.equal(first[1], second[1])
    assert usa.rt_take_device_error() == 0


def test_static_mask_rejects_shapes_beyond_the_workspace(cuda_device):
    lib = usa.load_library()
    fake = ctypes.c_void_p(0x10000)                   # never dereferenced: rejected before any launch
    too_big = RtShape(1, 64, 17776, 64, 64, 64)       # 2*64*278*64 > 2097152 fp32 values
    st = lib.rt_build_block_mask_static(ctypes.byref(too_big), fake, fake, 0.125, 9, 0, fake, fake, None, None)
    assert st == usa.RT_ERR_UNSUPPORTED
    q = torch.zeros(1, 64, 17776, 64, dtype=torch.bfloat16, device=cuda_device)
    with pytest.raises(ValueError):
        usa.rt_build_block_mask_static(q, q, head_dim=64, block_size=64, scale=0.125, keep_blocks=9)


@pytest.mark.parametrize("bs,D,d", [(64, 64, 64), (128, 80, 72)])
def test_cycle_with_caller_workspaces_equals_pool_cycle(cuda_device, bs, D, d):
    """A whole denoising cycle without the library allocating: the static mask, the pairing
    and the capture with caller workspaces (sized by rt_workspace_bytes, filled with garbage
    first), then the sparse step; every output equals the pool-allocating cycle bit for bit."""
    from ultra_sparse_attention_b200.workloads import Workload, denoising_inputs
    from fractions import Fraction
    w = Workload(name="case", batch=2, heads=3, seq_len=1000, head_dim=d, head_dim_padded=D, block_size=bs,
                 keep=(Fraction(1, 4),), forced_prefix_tokens=70, steps=2, capture_every=2, drift_sigma=0.05,
                 kind="iid", iid_std=1.0, seed=5)
    steps = list(denoising_inputs(w, 2))
    d0 = [x.to(cuda_device) for x in steps[0][1:]]
    d1 = [x.to(cuda_device) for x in steps[1][1:]]
    kw = dict(head_dim=d, block_size=bs, scale=w.scale)
    keep = w.keep_blocks()
    cap_b, pair_b = usa.rt_workspace_bytes(2, 3, 1000, head_dim=d, head_dim_padded=D, block_size=bs)
    ws_cap = torch.randint(0, 255, (cap_b,), dtype=torch.uint8, device=cuda_device)
    ws_pair = torch.randint(0, 255, (max(pair_b, 16),), dtype=torch.uint8, device=cuda_device)

    def cycle(static):
        mask = usa.rt_build_block_mask_static if static else usa.rt_build_block_mask
        rp, ci = mask(d0[0], d0[1], keep_blocks=keep, forced_prefix_tokens=w.forced_prefix_tokens, **kw)
        tiles = usa.rt_pair_query_blocks(d0[0], rp, ci, head_dim=d, block_size=bs,
                                         workspace=ws_pair if static else None)
        out0, st = usa.rt_attn_full_capture(*d0, row_ptr=rp, col_idx=ci, workspace=ws_cap if static else None, **kw)
        out1 = usa.rt_attn_sparse_reshape(*d1, row_ptr=rp, col_idx=ci, stats=st, tile_blocks=tiles, **kw)
        return [rp, ci, tiles, out0, st.m, st.zfull, st.zkept, st.u, out1]

    got, want = cycle(True), cycle(False)
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0
    for g, x in zip(got, want):
        assert torch.equal(g.view(torch.uint8), x.view(torch.uint8))
