"""The capture kernel's FMA-pipe exponential (one exponential pair in eight), against its
stated error bound: 2^x from Cody-Waite range reduction and a degree-3 minimax polynomial,
maximum relative error 7.5e-5 on [-125, 126], inputs below -125 clamped to 2^-125.  The
reference is numpy's exp2 in fp64 of the same fp32 inputs."""
import numpy as np
import pytest
import torch

import ultra_sparse_attention_b200 as usa

pytestmark = pytest.mark.gpu

BOUND = 7.6e-5


def test_exp2_poly_within_its_bound(cuda_device):
    g = torch.Generator().manual_seed(2)
    dense = torch.linspace(-125.0, 126.0, 1 << 21, dtype=torch.float64)
    near_int = torch.arange(-125, 127, dtype=torch.float64).repeat_interleave(9) + \
        torch.tensor([-0.5, -0.5 + 2 ** -20, -1e-6, -2 ** -24, 0.0, 2 ** -24, 1e-6, 0.5 - 2 ** -20, 0.5],
                     dtype=torch.float64).repeat(252)
    rand = (torch.rand(1 << 20, generator=g, dtype=torch.float64) * 251.0 - 125.0)
    x = torch.cat([dense, near_int.clamp(-125.0, 126.0), rand]).to(torch.float32)
    y = usa.rt_selftest_exp2_poly(x.to(cuda_device)).cpu().numpy().astype(np.float64)
    want = np.exp2(x.numpy().astype(np.float64))
    rel = np.abs(y / want - 1.0)
    assert np.all(np.isfinite(y))
    assert rel.max() <= BOUND, f"max relative error {rel.max():.3e} at x = {x.numpy()[rel.argmax()]}"
    # odd element count (the last pair has one lane)
    y3 = usa.rt_selftest_exp2_poly(torch.tensor([0.0, 1.0, -3.5], device=cuda_device)).cpu().numpy()
    assert np.all(np.abs(y3 / np.exp2([0.0, 1.0, -3.5]) - 1.0) <= BOUND)


def test_exp2_poly_clamps_below_range(cuda_device):
    x = torch.tensor([-float("inf"), -1e30, -300.0, -126.0, -125.5], device=cuda_device)
    y = usa.rt_selftest_exp2_poly(x).cpu().numpy().astype(np.float64)
    assert np.all(np.abs(y / 2.0 ** -125 - 1.0) <= BOUND), y
    assert usa.rt_take_device_error() == 0
