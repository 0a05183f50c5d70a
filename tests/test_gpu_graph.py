"""A whole denoising cycle recorded once in a CUDA graph and replayed on new inputs.

The library's calls take preallocated outputs, caller workspaces and the
fixed-array mask builder, so a cycle -- mask, query-block pairing, capture
with its statistics cache, and the reshaped sparse steps that follow -- can be
captured into one CUDA graph and replayed with no host work but the copy of
the next inputs into the captured buffers.  Each replay must give, bit for
bit, what the same calls give when launched one by one (every kernel on the
path is deterministic), and the captured graph must follow new input values
rather than replay the recorded ones.
"""
import dataclasses

import pytest
import torch

import ultra_sparse_attention_b200 as usa
from ultra_sparse_attention_b200.workloads import WORKLOADS, denoising_inputs

pytestmark = pytest.mark.gpu


class _Cycle:
    """Static device buffers of one cycle: a capture step and `n_sparse` sparse steps."""

    def __init__(self, w, device, n_sparse, compressed):
        B, H, N, D = w.batch, w.heads, w.seq_len, w.head_dim_padded
        self.w, self.compressed = w, compressed
        self.kw = dict(head_dim=w.head_dim, block_size=w.block_size, scale=w.scale)
        mk = lambda: torch.zeros(B, H, N, D, dtype=torch.bfloat16, device=device)
        self.inp = [[mk(), mk(), mk()] for _ in range(1 + n_sparse)]
        self.out = [mk() for _ in range(1 + n_sparse)]
        nb = w.n_blocks
        keep = w.keep_blocks()
        self.row_ptr = torch.empty(B * H * nb + 1, dtype=torch.int32, device=device)
        self.col_idx = torch.empty(B * H * nb * keep, dtype=torch.int32, device=device)
        self.tiles = torch.empty(B * H, -(-N // 128), 2, dtype=torch.int32, device=device)
        f = lambda *s, dt=torch.float32: torch.empty(*s, dtype=dt, device=device)
        self.stats = (usa.Stats(f(B, H, N), f(B, H, N), f(B, H, N), f(B, H, N, D, dt=torch.float16), f(B, H, N))
                      if compressed else usa.Stats(f(B, H, N), f(B, H, N), f(B, H, N), f(B, H, N, D)))
        cap_ws, pair_ws = usa.rt_workspace_bytes(B, H, N, head_dim=w.head_dim, head_dim_padded=D,
                                                 block_size=w.block_size)
        self.cap_ws = torch.empty(cap_ws, dtype=torch.uint8, device=device)
        self.pair_ws = torch.empty(pair_ws, dtype=torch.uint8, device=device)

    def load(self, steps):
        for dst, (q, k, v) in zip(self.inp, steps):
            for d, s in zip(dst, (q, k, v)):
                d.copy_(s, non_blocking=True)

    def run(self):
        w, kw = self.w, self.kw
        q0, k0, v0 = self.inp[0]
        usa.rt_build_block_mask_static(q0, k0, keep_blocks=w.keep_blocks(),
                                       forced_prefix_tokens=w.forced_prefix_tokens, row_ptr=self.row_ptr,
                                       col_idx=self.col_idx, **kw)
        usa.rt_pair_query_blocks(q0, self.row_ptr, self.col_idx, head_dim=w.head_dim, block_size=w.block_size,
                                 tile_blocks=self.tiles, workspace=self.pair_ws)
        usa.rt_attn_full_capture(q0, k0, v0, row_ptr=self.row_ptr, col_idx=self.col_idx, out=self.out[0],
                                 stats=self.stats, workspace=self.cap_ws, **kw)
        for (q, k, v), o in zip(self.inp[1:], self.out[1:]):
            usa.rt_attn_sparse_reshape(q, k, v, row_ptr=self.row_ptr, col_idx=self.col_idx, stats=self.stats,
                                       tile_blocks=self.tiles, out=o, **kw)

    def results(self):
        """Everything the cycle writes; the outputs of its steps come last."""
        s = self.stats
        res = [self.row_ptr, self.col_idx, self.tiles, s.m, s.zfull, s.zkept, s.u]
        if s.compressed:
            res.append(s.u_scale)
        return [x.clone() for x in res + self.out]


def _inputs(w, n_steps, seed_shift):
    st = denoising_inputs(dataclasses.replace(w, seed=w.seed + seed_shift), n_steps)
    return [tuple(x for x in step[1:]) for step in st]


@pytest.mark.parametrize("name,heads,compressed", [("video2b", 4, False), ("video2b", 4, True), ("image", 16, False),
                                                   ("long", 2, False)])
def test_cycle_replays_in_a_cuda_graph(cuda_device, name, heads, compressed):
    w = dataclasses.replace(WORKLOADS[name], heads=heads)
    n_sparse = 2
    cyc = _Cycle(w, cuda_device, n_sparse, compressed)
    first, second = _inputs(w, 1 + n_sparse, 0), _inputs(w, 1 + n_sparse, 1)

    side = torch.cuda.Stream(cuda_device)
    side.wait_stream(torch.cuda.current_stream(cuda_device))
    with torch.cuda.stream(side):  # eager reference for both input sets (also loads the module)
        cyc.load(first)
        cyc.run()
        want_first = cyc.results()
        cyc.load(second)
        cyc.run()
        want_second = cyc.results()
    torch.cuda.current_stream(cuda_device).wait_stream(side)
    torch.cuda.synchronize(cuda_device)

    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        cyc.run()
    for inputs, want in ((first, want_first), (second, want_second), (first, want_first)):
        cyc.load(inputs)
        graph.replay()
        torch.cuda.synchronize(cuda_device)
        got = cyc.results()
        for i, (g, e) in enumerate(zip(got, want)):
            assert torch.equal(g, e), f"result {i} of the replayed cycle differs from the eager one"
    assert not torch.equal(want_first[-1], want_second[-1])  # the last sparse step's output: the graph follows its inputs
    del graph
    assert usa.rt_take_device_error() == 0
