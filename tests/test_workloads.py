"""Host-side checks of the seeded input generators (no GPU)."""
from fractions import Fraction

import torch

from ultra_sparse_attention_b200.workloads import WORKLOADS, base_inputs, denoising_inputs, keep_blocks


def test_keep_counts_follow_integer_ceiling():
    assert keep_blocks(278, Fraction(1, 32)) == 9
    assert [keep_blocks(278, r) for r in WORKLOADS["video5b"].keep] == [9, 18, 35, 70, 278]
    assert WORKLOADS["tiny"].keep_blocks() == 2
    assert WORKLOADS["image"].keep_blocks() == 4
    assert WORKLOADS["long"].keep_blocks() == 4
    assert keep_blocks(10, Fraction(1, 1000)) == 1


def test_shapes_blocks_and_forced_prefix():
    w = WORKLOADS["video2b"]
    assert w.n_blocks == 278 and w.seq_len - 277 * 64 == 48
    assert -(-w.forced_prefix_tokens // w.block_size) == 4
    assert WORKLOADS["long"].n_blocks == 128


def test_tiny_is_seeded_padded_and_drifts():
    w = WORKLOADS["tiny"]
    a = [x for _, *x in denoising_inputs(w, 3)]
    b = [x for _, *x in denoising_inputs(w, 3)]
    for sa, sb in zip(a, b):
        for xa, xb in zip(sa, sb):
            assert xa.dtype == torch.bfloat16 and xa.shape == (1, 2, 512, 64)
            assert torch.equal(xa, xb)
    d = (a[1][0].float() - a[0][0].float())
    assert 0.03 < float(d.std()) < 0.07
    assert abs(float(a[0][0].float().std()) - 0.125) < 0.01


def test_padded_columns_are_zero():
    w = WORKLOADS["image"]
    small = type(w)(**{**w.__dict__, "batch": 1, "heads": 1})
    q, k, v = base_inputs(small)
    for x in (q, k, v):
        assert x.shape[-1] == 80
        assert torch.all(x[..., 72:] == 0)
        assert float(x[..., :72].float().std()) > 0.5
