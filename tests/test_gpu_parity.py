"""GPU parity: the CUDA path against the fp64 oracle, element by element.

Sizes are chosen so the oracle finishes in seconds while the kernels still
see several 128-row query tiles, several 64-key tiles and a ragged tail.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import ultra_sparse_attention_b200 as usa
from ultra_sparse_attention_b200.workloads import Workload, denoising_inputs

from pairing_ref import check_table, pair_query_blocks
from parity import (check_mask, compare_out, compare_stats, random_csr, score_tol, to_dev)

pytestmark = pytest.mark.gpu


def _wl(N, d, D, bs, B=2, H=3, std=1.0, seed=0, drift=0.05):
    return Workload(name="case", batch=B, heads=H, seq_len=N, head_dim=d, head_dim_padded=D, block_size=bs,
                    keep=(Fraction(1, 4),), forced_prefix_tokens=0, steps=2, capture_every=2, drift_sigma=drift,
                    kind="iid", iid_std=std, seed=seed)


def _inputs(w, device):
    steps = list(denoising_inputs(w, 2))
    host = [s[1:] for s in steps]
    dev = [tuple(x.to(device) for x in s) for s in host]
    return host, dev


def _stats_to_dev(st, shape, device):
    B, H, N, D = shape
    u = np.zeros((B * H * N, D))
    u[:, :st["u"].shape[1]] = st["u"]
    f = lambda a: torch.as_tensor(a, dtype=torch.float32).reshape(B, H, N).to(device)
    return usa.Stats(f(st["m"]), f(st["zfull"]), f(st["zkept"]),
                     torch.as_tensor(u, dtype=torch.float32).reshape(B, H, N, D).to(device))


def _abs_v(v):
    return v.abs()


CASES = [
    # N, d, D, bs
    (1000, 64, 64, 64),     # 16 blocks, last one 40 tokens; 8 query tiles
    (1000, 72, 80, 64),
    (1000, 72, 80, 128),    # 8 blocks, last one 104 tokens
    (896, 64, 64, 128),     # exact multiple of the block size
    (200, 64, 64, 64),      # one ragged query tile, odd number of blocks (4: 64,64,64,8)
    (1000, 128, 128, 64),   # head dim 128: a second 64-column tile part
    (1000, 112, 128, 128),  # head dim 112 stored as 128 (zero pad)
]


# ------------------------------------------------------------------ mask builder
@pytest.mark.parametrize("N,d,D,bs", CASES)
@pytest.mark.parametrize("keep_frac", [Fraction(1, 4), Fraction(1, 1)])
def test_mask_matches_oracle(cuda_device, N, d, D, bs, keep_frac):
    w = _wl(N, d, D, bs, std=1.0, seed=N + d)
    (h0, _), (d0, _) = _inputs(w, cuda_device)
    nb = w.n_blocks
    keep = w.keep_blocks(keep_frac)
    forced = 70 if keep >= 2 else 0
    rp, ci, sc = usa.rt_build_block_mask(d0[0], d0[1], head_dim=d, block_size=bs, scale=w.scale, keep_blocks=keep,
                                         forced_prefix_tokens=forced, block_scores=True)
    torch.cuda.synchronize()
    _, _, s64 = oracle.build_block_mask(h0[0], h0[1], d, bs, w.scale, keep, forced, return_scores=True)
    tol = score_tol(s64)
    s32 = sc.double().cpu().numpy().reshape(s64.shape)
    assert np.max(np.abs(s32 - s64)) <= tol
    differ = check_mask(rp.cpu().numpy(), ci.cpu().numpy(), s64, keep, bs, forced, tol)
    assert differ <= max(1, (w.batch * w.heads * nb) // 100)


def test_mask_exact_scores_and_ties_bit_exact(cuda_device):
    """Inputs whose block scores are exact in fp32 and fp64 (multiples of 2^-k),
    with duplicated key blocks: the GPU CSR must equal the oracle's everywhere,
    ties included (lower block index wins)."""
    B, H, N, d, bs = 1, 2, 1024, 64, 64
    g = torch.Generator().manual_seed(3)
    q = (torch.randint(-1, 2, (B, H, N, d), generator=g).float() / 4).to(torch.bfloat16)
    k = (torch.randint(-1, 2, (B, H, N, d), generator=g).float() / 4).to(torch.bfloat16)
    k[:, :, 5 * bs:6 * bs] = k[:, :, 3 * bs:4 * bs]      # block 5 duplicates block 3
    k[:, :, 9 * bs:10 * bs] = k[:, :, 12 * bs:13 * bs]   # block 9 duplicates block 12
    scale = 0.125
    for keep, forced in ((1, 0), (3, 0), (4, 64), (7, 130), (16, 0)):
        rp, ci = usa.rt_build_block_mask(q.to(cuda_device), k.to(cuda_device), head_dim=d, block_size=bs,
                                         scale=scale, keep_blocks=keep, forced_prefix_tokens=forced)
        rp_o, ci_o = oracle.build_block_mask(q, k, d, bs, scale, keep, forced)
        assert np.array_equal(rp.cpu().numpy(), rp_o)
        assert np.array_equal(ci.cpu().numpy(), ci_o), (keep, forced)


def test_mask_threshold_selection_ties_bit_exact(cuda_device):
    """More than eight chosen blocks take the threshold path of the selection:
    64 blocks with exact scores and many duplicated key blocks, so the k-th
    score is shared by several blocks; the CSR must equal the oracle's."""
    B, H, N, d, bs = 1, 3, 4096, 64, 64
    g = torch.Generator().manual_seed(11)
    q = (torch.randint(-1, 2, (B, H, N, d), generator=g).float() / 4).to(torch.bfloat16)
    k = (torch.randint(-1, 2, (B, H, N, d), generator=g).float() / 4).to(torch.bfloat16)
    for dst in range(1, 64, 3):  # blocks 1, 4, 7, ... copy block dst // 2
        src = dst // 2
        k[:, :, dst * bs:(dst + 1) * bs] = k[:, :, src * bs:(src + 1) * bs]
    scale = 0.125
    for keep, forced in ((9, 0), (20, 0), (33, 130), (50, 0), (63, 64), (64, 0)):
        rp, ci = usa.rt_build_block_mask(q.to(cuda_device), k.to(cuda_device), head_dim=d, block_size=bs,
                                         scale=scale, keep_blocks=keep, forced_prefix_tokens=forced)
        rp_o, ci_o = oracle.build_block_mask(q, k, d, bs, scale, keep, forced)
        assert np.array_equal(rp.cpu().numpy(), rp_o)
        assert np.array_equal(ci.cpu().numpy(), ci_o), (keep, forced)


# ------------------------------------------------------------------ capture step
@pytest.mark.parametrize("N,d,D,bs", CASES)
@pytest.mark.parametrize("keep_frac", [Fraction(1, 4), Fraction(1, 1)])
def test_capture_matches_oracle(cuda_device, N, d, D, bs, keep_frac):
    w = _wl(N, d, D, bs, std=1.2, seed=7 * N + d)
    (h0, _), (d0, _) = _inputs(w, cuda_device)
    bh, nb = w.batch * w.heads, w.n_blocks
    keep = w.keep_blocks(keep_frac)
    rp, ci = random_csr(bh, nb, keep, seed=N)
    out, st = usa.rt_attn_full_capture(*d0, head_dim=d, block_size=bs, scale=w.scale,
                                       row_ptr=to_dev(rp, cuda_device), col_idx=to_dev(ci, cuda_device))
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0
    orc = oracle.full_capture(*h0, d, bs, w.scale, rp, ci)
    orc_abs = oracle.full_capture(h0[0], h0[1], h0[2].abs(), d, bs, w.scale, rp, ci)["u"]
    compare_out(out.reshape(-1, D), orc["o"], d, "capture O")
    compare_stats(st, np.arange(bh * N), orc, orc_abs, d, "capture stats")
    if keep == nb:
        assert torch.all(st.u == 0)


# ------------------------------------------------------------------ sparse step (oracle mask + oracle stats)
@pytest.mark.parametrize("N,d,D,bs", CASES)
@pytest.mark.parametrize("keep_frac", [Fraction(1, 4), Fraction(1, 2)])
@pytest.mark.parametrize("with_stats", [True, False])
def test_sparse_matches_oracle(cuda_device, N, d, D, bs, keep_frac, with_stats):
    w = _wl(N, d, D, bs, std=1.2, seed=11 * N + d, drift=0.05)
    (h0, h1), (d0, d1) = _inputs(w, cuda_device)
    bh, nb = w.batch * w.heads, w.n_blocks
    keep = w.keep_blocks(keep_frac)
    rp, ci = random_csr(bh, nb, keep, seed=N + 1)
    st_o = oracle.full_capture(*h0, d, bs, w.scale, rp, ci) if with_stats else None
    st_d = _stats_to_dev(st_o, d0[0].shape, cuda_device) if with_stats else None
    out = usa.rt_attn_sparse_reshape(*d1, head_dim=d, block_size=bs, scale=w.scale, row_ptr=to_dev(rp, cuda_device),
                                     col_idx=to_dev(ci, cuda_device), stats=st_d)
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0
    want = oracle.sparse_reshape(*h1, d, bs, w.scale, rp, ci, st_o)
    compare_out(out.reshape(-1, D), want, d, "sparse O")


# ------------------------------------------------------------------ tile pairing
def _random_table(bh, nb, bs, N, seed):
    """Each head's blocks in random tiles and halves (an odd count leaves a random empty half)."""
    rng = np.random.default_rng(seed)
    n_tiles = -(-N // 128)
    per = 2 if bs == 64 else 1
    t = np.full((bh, n_tiles, 2), -1, np.int32)
    for h in range(bh):
        slots = np.full(n_tiles * per, -1, np.int64)
        slots[:nb] = rng.permutation(nb)
        slots = rng.permutation(slots) if per == 2 else slots
        t[h, :, :per] = slots.reshape(n_tiles, per)
    return t


@pytest.mark.parametrize("N,bs,keep", [(1000, 64, 4), (200, 64, 2), (64 * 301, 64, 9), (1000, 128, 3), (64, 64, 1),
                                        (1000, 64, 16), (64 * 2048, 64, 20), (64 * 900 - 5, 64, 30)])
def test_pairing_matches_reference(cuda_device, N, bs, keep):
    bh, nb = 3, -(-N // bs)
    rp, ci = random_csr(bh, nb, keep, seed=N + keep, forced=1)
    q = torch.zeros(1, bh, N, 64, dtype=torch.bfloat16, device=cuda_device)
    got = usa.rt_pair_query_blocks(q, to_dev(rp, cuda_device), to_dev(ci, cuda_device), head_dim=64, block_size=bs)
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0
    got = got.cpu().numpy()
    check_table(got, nb, bs)
    np.testing.assert_array_equal(got, pair_query_blocks(rp, ci, bh, nb, bs, -(-N // 128)))


def test_pairing_of_a_malformed_csr_is_valid_and_matches(cuda_device):
    """Out-of-range entries, repeats, empty rows and rows longer than n_blocks: the
    table is still a valid one and the same as the reference's."""
    N, bs, bh = 1000, 64, 2
    nb = -(-N // bs)
    rng = np.random.default_rng(3)
    rows = []
    for r in range(bh * nb):
        n = int(rng.choice([0, 1, 3, nb + 5]))
        rows.append(rng.integers(-3, nb + 3, size=n))
    rp = np.array([0] + list(np.cumsum([len(x) for x in rows])), np.int32)
    ci = np.concatenate(rows).astype(np.int32)
    q = torch.zeros(1, bh, N, 64, dtype=torch.bfloat16, device=cuda_device)
    got = usa.rt_pair_query_blocks(q, to_dev(rp, cuda_device), to_dev(ci, cuda_device), head_dim=64, block_size=bs)
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0
    got = got.cpu().numpy()
    check_table(got, nb, bs)
    np.testing.assert_array_equal(got, pair_query_blocks(rp, ci, bh, nb, bs, -(-N // 128)))


@pytest.mark.parametrize("N,d,D,bs", CASES + [(1064, 64, 64, 64), (1064, 72, 80, 64)])  # 17 blocks: an empty half
def test_sparse_with_any_tile_table_is_bit_identical(cuda_device, N, d, D, bs):
    """The pairing only regroups rows: the sparse step with the computed pairing, with a
    random table (blocks in any tile and half, empty halves anywhere) and with the
    neighbouring blocks gives the same bits, with and without statistics, and matches
    the oracle."""
    w = _wl(N, d, D, bs, std=1.2, seed=13 * N + d, drift=0.05)
    (h0, h1), (d0, d1) = _inputs(w, cuda_device)
    bh, nb = w.batch * w.heads, w.n_blocks
    keep = w.keep_blocks(Fraction(1, 4))
    rp, ci = random_csr(bh, nb, keep, seed=N + 3, forced=1)
    rp_d, ci_d = to_dev(rp, cuda_device), to_dev(ci, cuda_device)
    kw = dict(head_dim=d, block_size=bs, scale=w.scale, row_ptr=rp_d, col_idx=ci_d)
    _, st = usa.rt_attn_full_capture(*d0, **kw)
    paired = usa.rt_pair_query_blocks(d1[0], rp_d, ci_d, head_dim=d, block_size=bs)
    rand = to_dev(_random_table(bh, nb, bs, N, seed=N), cuda_device)
    for stats in (st, None):
        base = usa.rt_attn_sparse_reshape(*d1, stats=stats, **kw)
        for table in (paired, rand):
            out = torch.full_like(base, float("nan"))
            usa.rt_attn_sparse_reshape(*d1, stats=stats, tile_blocks=table, out=out, **kw)
            torch.cuda.synchronize()
            assert usa.rt_take_device_error() == 0
            assert torch.equal(out.view(torch.int16), base.view(torch.int16))
    check_table(paired.cpu().numpy(), nb, bs)
    want = oracle.sparse_reshape(*h1, d, bs, w.scale, rp, ci, None)
    compare_out(out.reshape(-1, D), want, d, "sparse O (random tile table, no statistics)")


@pytest.mark.parametrize("D,d", [(64, 64), (80, 72)])
def test_sparse_tile_table_with_missing_and_repeated_blocks(cuda_device, D, d):
    """A table entry out of range is an empty half, a block in no tile leaves its rows
    unwritten, and a block in two halves is computed twice with the same result."""
    N, bs = 1000, 64
    w = _wl(N, d, D, bs, std=1.0, seed=29, drift=0.05)
    (h0, h1), (d0, d1) = _inputs(w, cuda_device)
    bh, nb = w.batch * w.heads, w.n_blocks
    rp, ci = random_csr(bh, nb, w.keep_blocks(Fraction(1, 4)), seed=31, forced=1)
    kw = dict(head_dim=d, block_size=bs, scale=w.scale, row_ptr=to_dev(rp, cuda_device), col_idx=to_dev(ci, cuda_device))
    _, st = usa.rt_attn_full_capture(*d0, **kw)
    base = usa.rt_attn_sparse_reshape(*d1, stats=st, **kw)
    n_tiles = -(-N // 128)
    table = np.arange(2 * n_tiles, dtype=np.int32).reshape(1, n_tiles, 2).repeat(bh, 0)
    table[:, 2, 1] = nb + 7       # block 5: out of range -> empty half, rows unwritten
    table[:, 3, 0] = 7            # block 6 missing, block 7 in both halves of tile 3
    table[:, n_tiles - 1, 1] = -1  # block 15 missing
    out = torch.full_like(base, float("nan"))
    usa.rt_attn_sparse_reshape(*d1, stats=st, tile_blocks=to_dev(table, cuda_device), out=out, **kw)
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0
    rows = torch.arange(N, device=cuda_device) // bs
    missing = (rows == 5) | (rows == 6) | (rows == 15)
    assert torch.isnan(out[:, :, missing].float()).all()
    assert torch.equal(out[:, :, ~missing].view(torch.int16), base[:, :, ~missing].view(torch.int16))


@pytest.mark.parametrize("N,d,D,bs", [(1000, 64, 64, 64), (1000, 72, 80, 64), (200, 64, 64, 64), (896, 64, 64, 128),
                                      (1000, 128, 128, 64)])
@pytest.mark.parametrize("gain", [3.0, 0.25])
def test_sparse_reshape_with_rescales(cuda_device, N, d, D, bs, gain):
    """Sparse step on Q scaled by `gain` against statistics of the unscaled step.

    With gain 3 the running maxima exceed the cached ones by far more than the
    lazy-rescale margin, so O is rescaled on the first kept tiles of most rows
    (including while the previous query tile's output is still pending); with
    gain 1/4 no rescale happens but e^{m_c - m'} is large.  The oracle evaluates
    the same reshape formula on the same inputs."""
    w = _wl(N, d, D, bs, std=1.2, seed=5 * N + d, drift=0.0)
    (h0, _), (d0, _) = _inputs(w, cuda_device)
    q1 = (h0[0].float() * gain).to(torch.bfloat16)
    h1 = (q1, h0[1], h0[2])
    d1 = (q1.to(cuda_device), d0[1], d0[2])
    bh, nb = w.batch * w.heads, w.n_blocks
    keep = w.keep_blocks(Fraction(1, 2))
    rp, ci = random_csr(bh, nb, keep, seed=N + 7)
    st_o = oracle.full_capture(*h0, d, bs, w.scale, rp, ci)
    st_d = _stats_to_dev(st_o, d0[0].shape, cuda_device)
    out = usa.rt_attn_sparse_reshape(*d1, head_dim=d, block_size=bs, scale=w.scale, row_ptr=to_dev(rp, cuda_device),
                                     col_idx=to_dev(ci, cuda_device), stats=st_d)
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0
    want = oracle.sparse_reshape(*h1, d, bs, w.scale, rp, ci, st_o)
    compare_out(out.reshape(-1, D), want, d, f"sparse O (Q x {gain})")


@pytest.mark.parametrize("N,d,D,bs,keep", [(896, 64, 64, 128, 1), (2048, 72, 80, 128, 1), (1000, 64, 64, 64, 1),
                                             (1000, 72, 80, 64, 1), (2048, 64, 64, 128, 2), (1000, 128, 128, 64, 1)])
def test_sparse_reshape_short_query_tiles(cuda_device, N, d, D, bs, keep):
    """Query tiles with one or two kept key tiles: fewer than the key tiles the MMA issuer
    keeps in flight, so a tile's PVs are still pending when the query tile two ahead needs
    its Q buffer back (the issuer must drain them first)."""
    w = _wl(N, d, D, bs, std=1.0, seed=7 * N + keep, drift=0.05)
    (h0, h1), (d0, d1) = _inputs(w, cuda_device)
    bh, nb = w.batch * w.heads, w.n_blocks
    rp, ci = random_csr(bh, nb, keep, seed=N + keep)
    st_o = oracle.full_capture(*h0, d, bs, w.scale, rp, ci)
    st_d = _stats_to_dev(st_o, d0[0].shape, cuda_device)
    out = usa.rt_attn_sparse_reshape(*d1, head_dim=d, block_size=bs, scale=w.scale, row_ptr=to_dev(rp, cuda_device),
                                     col_idx=to_dev(ci, cuda_device), stats=st_d)
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0
    want = oracle.sparse_reshape(*h1, d, bs, w.scale, rp, ci, st_o)
    compare_out(out.reshape(-1, D), want, d, f"sparse O (keep {keep} of {nb})")


@pytest.mark.parametrize("N,d,D,bs", [(1000, 64, 64, 64), (1000, 72, 80, 64)])
@pytest.mark.parametrize("shift", [50.0, -10.0, 3.0])
def test_sparse_reshape_cached_reference_shift(cuda_device, N, d, D, bs, shift):
    """The reshape formula does not depend on which reference the statistics are cached
    against: m_c + delta with Z_full, Z_kept and U scaled by e^-delta give the same output.

    delta = 50 puts every kept p below 2^-64 of the shifted reference, so the kernel's
    no-max fast path must hand the tile to the max-based path and rescale down; delta = -10
    makes the tile sums exceed 2^8, the rescale-up hand-off; delta = 3 stays on the fast
    path.  The expected output is the oracle's on the unshifted statistics."""
    w = _wl(N, d, D, bs, std=1.0, seed=11 * N + d, drift=0.05)
    (h0, h1), (d0, d1) = _inputs(w, cuda_device)
    bh, nb = w.batch * w.heads, w.n_blocks
    keep = w.keep_blocks(Fraction(1, 4))
    rp, ci = random_csr(bh, nb, keep, seed=N + 3)
    st_o = oracle.full_capture(*h0, d, bs, w.scale, rp, ci)
    f = np.exp(-shift)
    shifted = {"m": st_o["m"] + shift, "zfull": st_o["zfull"] * f, "zkept": st_o["zkept"] * f,
               "u": st_o["u"] * f}
    st_d = _stats_to_dev(shifted, d0[0].shape, cuda_device)
    out = usa.rt_attn_sparse_reshape(*d1, head_dim=d, block_size=bs, scale=w.scale, row_ptr=to_dev(rp, cuda_device),
                                     col_idx=to_dev(ci, cuda_device), stats=st_d)
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0
    want = oracle.sparse_reshape(*h1, d, bs, w.scale, rp, ci, st_o)
    compare_out(out.reshape(-1, D), want, d, f"sparse O (cached reference shifted by {shift})")


# ------------------------------------------------------------------ invariants the pages fix
@pytest.mark.parametrize("N,d,D,bs", [(1000, 72, 80, 64), (1000, 64, 64, 128)])
def test_reshape_keep_all_equals_full_attention(cuda_device, N, d, D, bs):
    """Keep ratio 100%: the reshaped sparse step is full attention of its own inputs."""
    w = _wl(N, d, D, bs, std=1.2, seed=5, drift=0.2)
    (h0, h1), (d0, d1) = _inputs(w, cuda_device)
    nb = w.n_blocks
    rp, ci = usa.rt_build_block_mask(d0[0], d0[1], head_dim=d, block_size=bs, scale=w.scale, keep_blocks=nb)
    _, st = usa.rt_attn_full_capture(*d0, head_dim=d, block_size=bs, scale=w.scale, row_ptr=rp, col_idx=ci)
    out = usa.rt_attn_sparse_reshape(*d1, head_dim=d, block_size=bs, scale=w.scale, row_ptr=rp, col_idx=ci, stats=st)
    torch.cuda.synchronize()
    rpo, cio = oracle.build_block_mask(h0[0], h0[1], d, bs, w.scale, nb, 0)
    want = oracle.full_capture(*h1, d, bs, w.scale, rpo, cio)["o"]
    compare_out(out.reshape(-1, D), want, d, "keep-all reshape vs full attention")


@pytest.mark.parametrize("N,d,D,bs", [(1000, 72, 80, 64), (1000, 64, 64, 128)])
def test_reshape_unchanged_inputs_recover_capture(cuda_device, N, d, D, bs):
    """Inputs unchanged since the capture step: reshape recovers full attention at 1/8 keep."""
    w = _wl(N, d, D, bs, std=1.5, seed=6)
    (h0, _), (d0, _) = _inputs(w, cuda_device)
    keep = w.keep_blocks(Fraction(1, 8))
    rp, ci = usa.rt_build_block_mask(d0[0], d0[1], head_dim=d, block_size=bs, scale=w.scale, keep_blocks=keep)
    _, st = usa.rt_attn_full_capture(*d0, head_dim=d, block_size=bs, scale=w.scale, row_ptr=rp, col_idx=ci)
    out = usa.rt_attn_sparse_reshape(*d0, head_dim=d, block_size=bs, scale=w.scale, row_ptr=rp, col_idx=ci, stats=st)
    torch.cuda.synchronize()
    want = oracle.full_capture(*h0, d, bs, w.scale, rp.cpu().numpy(), ci.cpu().numpy())["o"]
    compare_out(out.reshape(-1, D), want, d, "unchanged-input reshape vs capture")


def test_sparse_empty_rows_give_zero(cuda_device):
    N, d, D, bs = 512, 64, 64, 64
    w = _wl(N, d, D, bs, B=1, H=1, seed=2)
    (h0, _), (d0, _) = _inputs(w, cuda_device)
    # query blocks 0 and 5 keep nothing; block 1 keeps nothing while its tile partner 0 also keeps nothing
    sets = [[], [], [2], [0, 7], [3], [], [6], [1, 2]]
    rp = np.array([0] + list(np.cumsum([len(s) for s in sets])), np.int32)
    ci = np.array([x for s in sets for x in s], np.int32)
    for with_stats in (False, True):
        st_o = oracle.full_capture(*h0, d, bs, w.scale, rp, ci) if with_stats else None
        st_d = _stats_to_dev(st_o, d0[0].shape, cuda_device) if with_stats else None
        out = usa.rt_attn_sparse_reshape(*d0, head_dim=d, block_size=bs, scale=w.scale, row_ptr=to_dev(rp, cuda_device),
                                         col_idx=to_dev(ci, cuda_device), stats=st_d)
        torch.cuda.synchronize()
        want = oracle.sparse_reshape(*h0, d, bs, w.scale, rp, ci, st_o)
        o = out.reshape(-1, D)
        assert torch.all(o[:2 * bs] == 0) and torch.all(o[5 * bs:6 * bs] == 0)
        compare_out(o, want, d, "empty rows")


def test_malformed_csr_stays_in_bounds(cuda_device):
    """Out-of-range and duplicated block indices are skipped; the call completes
    and writes only its output (checked with canary-padded buffers)."""
    N, d, D, bs = 256, 64, 64, 64
    w = _wl(N, d, D, bs, B=1, H=1, seed=4)
    (_, _), (d0, _) = _inputs(w, cuda_device)
    ci = np.array([0, 0, 9, -3, 1, 2, 2, 1000, 3], np.int32)
    rp = np.array([0, 4, 5, 8, 9], np.int32)
    big = torch.full((3 * N * D,), 7.0, dtype=torch.bfloat16, device=cuda_device)
    out = big[N * D:2 * N * D].view(1, 1, N, D)
    usa.rt_attn_sparse_reshape(*d0, head_dim=d, block_size=bs, scale=w.scale, row_ptr=to_dev(rp, cuda_device),
                               col_idx=to_dev(ci, cuda_device), stats=None, out=out)
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0
    assert torch.all(big[:N * D] == 7.0) and torch.all(big[2 * N * D:] == 7.0)
    assert torch.isfinite(out.float()).all()


# ------------------------------------------------------------------ whole cycle (GPU mask -> capture -> sparse)
@pytest.mark.parametrize("N,d,D,bs", [(1000, 72, 80, 64), (1000, 72, 80, 128), (1000, 64, 64, 64)])
def test_denoising_cycle_matches_oracle_chain(cuda_device, N, d, D, bs):
    w = _wl(N, d, D, bs, std=1.2, seed=9, drift=0.05)
    (h0, h1), (d0, d1) = _inputs(w, cuda_device)
    keep = w.keep_blocks(Fraction(1, 4))
    rp, ci = usa.rt_build_block_mask(d0[0], d0[1], head_dim=d, block_size=bs, scale=w.scale, keep_blocks=keep)
    o0, st = usa.rt_attn_full_capture(*d0, head_dim=d, block_size=bs, scale=w.scale, row_ptr=rp, col_idx=ci)
    o1 = usa.rt_attn_sparse_reshape(*d1, head_dim=d, block_size=bs, scale=w.scale, row_ptr=rp, col_idx=ci, stats=st)
    torch.cuda.synchronize()
    rpo, cio = oracle.build_block_mask(h0[0], h0[1], d, bs, w.scale, keep, 0)
    assert np.array_equal(ci.cpu().numpy(), cio)
    st_o = oracle.full_capture(*h0, d, bs, w.scale, rpo, cio)
    compare_out(o0.reshape(-1, D), st_o["o"], d, "cycle capture O")
    want = oracle.sparse_reshape(*h1, d, bs, w.scale, rpo, cio, st_o)
    compare_out(o1.reshape(-1, D), want, d, "cycle sparse O")


def test_timeout_self_test_reports_and_recovers(cuda_device):
    """A bounded wait that runs out records RT_ERR_TIMEOUT; the context stays usable."""
    assert usa.rt_take_device_error() == 0
    usa.rt_selftest_wait_timeout(20_000_000)   # 20 ms
    assert usa.rt_take_device_error() == usa.RT_ERR_TIMEOUT
    assert usa.rt_take_device_error() == 0
    x = torch.ones(4, device=cuda_device)
    assert float(x.sum()) == 4.0


@pytest.mark.parametrize("v_scale", [1.0e5, 3.0e-7])
def test_capture_with_large_and_tiny_v(cuda_device, v_scale):
    """The capture's PV products run on an f16 copy of V scaled per head by a power of two:
    V far above the f16 range (1e5) or far below its normal range (3e-7) gives the same
    relative accuracy as unit-scale V, against the oracle on the same bf16 inputs; one head
    mixes a single huge value into unit-scale V (its scale follows the max)."""
    N, d, D, bs = 1000, 64, 64, 64
    w = _wl(N, d, D, bs, std=1.0, seed=41, drift=0.05)
    (h0, _), (d0, _) = _inputs(w, cuda_device)
    v = (h0[2].float() * v_scale).to(torch.bfloat16)
    v[1, 2] = h0[2][1, 2]
    v[1, 2, 777, 5] = 6.0e4 if v_scale > 1 else 1.0
    bh = w.batch * w.heads
    rp, ci = random_csr(bh, w.n_blocks, 4, seed=43, forced=1)
    out, st = usa.rt_attn_full_capture(d0[0], d0[1], v.to(cuda_device), head_dim=d, block_size=bs, scale=w.scale,
                                       row_ptr=to_dev(rp, cuda_device), col_idx=to_dev(ci, cuda_device))
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0
    orc = oracle.full_capture(h0[0], h0[1], v, d, bs, w.scale, rp, ci)
    orc_abs = oracle.full_capture(h0[0], h0[1], v.abs(), d, bs, w.scale, rp, ci)["u"]
    # outputs compared at unit scale, head by head (the mixed head at its own scale)
    head_scale = np.full(bh, v_scale)
    head_scale[1 * w.heads + 2] = 1.0
    row_scale = np.repeat(head_scale, N)[:, None]
    got = out.reshape(-1, D).float().cpu().numpy().astype(np.float64) / row_scale
    compare_out(torch.as_tensor(got), orc["o"] / row_scale, d, f"capture O, V x {v_scale:g}")
    compare_stats(st, np.arange(bh * N), orc, orc_abs, d, f"capture stats, V x {v_scale:g}")


# ------------------------------------------------------------------ sharply peaked rows
def _csr_with_block(bh, nb, keep, seed, block):
    """Random kept sets that all contain `block` (sorted): int32 row_ptr, col_idx."""
    rng = np.random.default_rng(seed)
    others = np.array([b for b in range(nb) if b != block])
    sets = [sorted({block} | set(int(x) for x in rng.choice(others, size=keep - 1, replace=False)))
            for _ in range(bh * nb)]
    row_ptr = np.array([0] + list(np.cumsum([len(s) for s in sets])), np.int32)
    col_idx = np.array([kb for s in sets for kb in s], np.int32)
    return row_ptr, col_idx


def _capture_vs_oracle(cuda_device, h, d, bs, scale, rp, ci, what):
    q, k, v = (x.to(cuda_device) for x in h)
    out, st = usa.rt_attn_full_capture(q, k, v, head_dim=d, block_size=bs, scale=scale,
                                       row_ptr=to_dev(rp, cuda_device), col_idx=to_dev(ci, cuda_device))
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0
    orc = oracle.full_capture(*h, d, bs, scale, rp, ci)
    orc_abs = oracle.full_capture(h[0], h[1], h[2].abs(), d, bs, scale, rp, ci)["u"]
    D = q.shape[-1]
    bh, N = q.shape[0] * q.shape[1], q.shape[2]
    compare_out(out.reshape(-1, D), orc["o"], d, f"{what}: capture O")
    compare_stats(st, np.arange(bh * N), orc, orc_abs, d, f"{what}: capture stats")


@pytest.mark.parametrize("N,d,D,bs", [(1000, 64, 64, 64), (1000, 72, 80, 64), (896, 64, 64, 128),
                                      (1000, 128, 128, 64)])
@pytest.mark.parametrize("gain", [3.0, 5.0])
def test_capture_sharp_scores(cuda_device, N, d, D, bs, gain):
    """Q scaled by 3 and 5: scores spread over tens of nats, so most terms of U and of the
    kept sum lie many binades below the row's largest term; statistics and output must
    still meet the tolerances against the oracle on the same bf16 inputs."""
    w = _wl(N, d, D, bs, std=1.2, seed=5 * N + d + int(gain))
    (h0, _), _ = _inputs(w, cuda_device)
    q = (h0[0].float() * gain).to(torch.bfloat16)
    bh = w.batch * w.heads
    rp, ci = random_csr(bh, w.n_blocks, max(2, w.n_blocks // 4), seed=N + int(gain), forced=1)
    _capture_vs_oracle(cuda_device, (q, h0[1], h0[2]), d, bs, w.scale, rp, ci, f"Q x {gain:g}")


@pytest.mark.parametrize("gap", [10.0, 14.0, 16.0, 18.0, 22.0, 30.0])
@pytest.mark.parametrize("N,d,D,bs,peak", [(2000, 64, 64, 64, 0), (2000, 64, 64, 64, 1500), (2000, 72, 80, 128, 1100),
                                           (2000, 128, 128, 64, 700)])
def test_capture_peaked_rows(cuda_device, N, d, D, bs, peak, gap):
    """Every row's maximum sits on one key (token `peak`, in a block that every query block
    keeps) about `gap` nats above all other keys, the masked ones among them: U is then a
    sum of many terms each near e^-gap of the row's largest, whose total still decides the
    tolerance.  Q shares a direction u; the peak key is c*u, the others small noise."""
    g = torch.Generator().manual_seed(int(gap * 10) + N + peak)
    B, H = 1, 2
    scale = 1.0 / np.sqrt(d)
    u = torch.randn(d, generator=g)
    q = u + 0.3 * torch.randn(B, H, N, d, generator=g)
    k = 0.5 * torch.randn(B, H, N, d, generator=g)
    c = gap / (scale * float(u @ u))
    k[:, :, peak] = c * u
    v = torch.randn(B, H, N, d, generator=g)

    def pad(x):
        out = torch.zeros(B, H, N, D)
        out[..., :d] = x
        return out.to(torch.bfloat16)

    nb = -(-N // bs)
    rp, ci = _csr_with_block(B * H, nb, max(2, nb // 4), seed=N + peak, block=peak // bs)
    _capture_vs_oracle(cuda_device, (pad(q), pad(k), pad(v)), d, bs, scale, rp, ci, f"peak gap {gap:g} nats")


def _csr_without_block(bh, nb, keep, seed, block):
    """Random kept sets that never contain `block` (sorted): int32 row_ptr, col_idx."""
    rng = np.random.default_rng(seed)
    others = np.array([b for b in range(nb) if b != block])
    sets = [sorted(int(x) for x in rng.choice(others, size=keep, replace=False)) for _ in range(bh * nb)]
    row_ptr = np.array([0] + list(np.cumsum([len(s) for s in sets])), np.int32)
    col_idx = np.array([kb for s in sets for kb in s], np.int32)
    return row_ptr, col_idx


@pytest.mark.parametrize("compressed", [False, True])
@pytest.mark.parametrize("gap", [30.0, 70.0, 95.0, 115.0, 130.0])
@pytest.mark.parametrize("N,d,D,bs,peak", [(2000, 64, 64, 64, 1500), (2000, 72, 80, 128, 700)])
def test_masked_dominant_rows(cuda_device, N, d, D, bs, peak, gap, compressed):
    """The mirror of the peaked rows: the row maximum sits on one key (token `peak`) in a
    block that no query block keeps, `gap` nats above every kept key.  Relative to the row
    max the kept sum is about e^-gap, beyond fp32 from ~87 nats on, so the cache has to
    hold it at another reference; the statistics (through the reference-free ratio,
    log-sum-exp and U / Z_full), the capture output and the reshaped sparse step -- on the
    same inputs and on drifted ones -- must all meet the tolerances against the oracle,
    with no non-finite value."""
    g = torch.Generator().manual_seed(int(gap) + N + peak + 7)
    B, H = 1, 2
    scale = 1.0 / np.sqrt(d)
    u = torch.randn(d, generator=g)
    q = u + 0.3 * torch.randn(B, H, N, d, generator=g)
    k = 0.5 * torch.randn(B, H, N, d, generator=g)
    c = gap / (scale * float(u @ u))
    k[:, :, peak] = c * u
    v = torch.randn(B, H, N, d, generator=g)

    def pad(x):
        out = torch.zeros(B, H, N, D)
        out[..., :d] = x
        return out.to(torch.bfloat16)

    nb = -(-N // bs)
    rp, ci = _csr_without_block(B * H, nb, max(2, nb // 4), seed=N + peak, block=peak // bs)
    h0 = (pad(q), pad(k), pad(v))
    h1 = (pad(q + 0.05 * torch.randn(B, H, N, d, generator=g)), pad(k + 0.05 * torch.randn(B, H, N, d, generator=g)),
          pad(v + 0.05 * torch.randn(B, H, N, d, generator=g)))
    q0, k0, v0 = (x.to(cuda_device) for x in h0)
    rp_d, ci_d = to_dev(rp, cuda_device), to_dev(ci, cuda_device)
    out, st = usa.rt_attn_full_capture(q0, k0, v0, head_dim=d, block_size=bs, scale=scale, row_ptr=rp_d,
                                       col_idx=ci_d, compressed=compressed)
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0
    orc = oracle.full_capture(*h0, d, bs, scale, rp, ci)
    orc_abs = oracle.full_capture(h0[0], h0[1], h0[2].abs(), d, bs, scale, rp, ci)["u"]
    assert np.log(orc["zfull"] / orc["zkept"]).max() > gap - 10.0  # the case is what it claims
    what = f"masked max {gap:g} nats up"
    compare_out(out.reshape(-1, D), orc["o"], d, f"{what}: capture O")
    st32 = usa.Stats(st.m, st.zfull, st.zkept, st.residual())
    for t in (st.m, st.zfull, st.zkept, st32.u):
        assert torch.isfinite(t).all(), f"{what}: non-finite statistics"
    compare_stats(st32, np.arange(B * H * N), orc, orc_abs, d, f"{what}: capture stats")
    for name, h in (("same inputs", h0), ("drifted inputs", h1)):
        x = [t.to(cuda_device) for t in h]
        got = usa.rt_attn_sparse_reshape(*x, head_dim=d, block_size=bs, scale=scale, row_ptr=rp_d, col_idx=ci_d,
                                         stats=st)
        torch.cuda.synchronize()
        assert usa.rt_take_device_error() == 0
        want = oracle.sparse_reshape(*h, d, bs, scale, rp, ci, orc)
        compare_out(got.reshape(-1, D), want, d, f"{what}: sparse step, {name}")


def test_masked_dominant_rows_beyond_the_cache_range(cuda_device):
    """A masked maximum ~200 nats above every kept key: the kept sum lies below what the fp32
    cache holds even at a shifted reference (its Z_kept reads 0).  The capture output is
    still exact, and the sparse step on unchanged inputs falls back to U / Z_full -- exact
    there, because the kept mass is negligible -- with every value finite."""
    N, d, D, bs, peak, gap = 1000, 64, 64, 64, 600, 200.0
    g = torch.Generator().manual_seed(99)
    B, H = 1, 2
    scale = 1.0 / np.sqrt(d)
    u = torch.randn(d, generator=g)
    q = u + 0.3 * torch.randn(B, H, N, d, generator=g)
    k = 0.5 * torch.randn(B, H, N, d, generator=g)
    k[:, :, peak] = gap / (scale * float(u @ u)) * u
    v = torch.randn(B, H, N, d, generator=g)
    h = tuple(x.to(torch.bfloat16) for x in (q, k, v))
    nb = -(-N // bs)
    rp, ci = _csr_without_block(B * H, nb, 4, seed=5, block=peak // bs)
    x = [t.to(cuda_device) for t in h]
    rp_d, ci_d = to_dev(rp, cuda_device), to_dev(ci, cuda_device)
    out, st = usa.rt_attn_full_capture(*x, head_dim=d, block_size=bs, scale=scale, row_ptr=rp_d, col_idx=ci_d)
    got = usa.rt_attn_sparse_reshape(*x, head_dim=d, block_size=bs, scale=scale, row_ptr=rp_d, col_idx=ci_d,
                                     stats=st)
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0
    orc = oracle.full_capture(*h, d, bs, scale, rp, ci)
    assert np.log(orc["zfull"] / orc["zkept"]).min() > 170.0
    assert (st.zkept == 0).float().mean().item() > 0.5  # most rows are beyond the range
    for t in (st.m, st.zfull, st.u):
        assert torch.isfinite(t).all()
    compare_out(out.reshape(-1, D), orc["o"], d, "capture O, masked max 200 nats up")
    compare_out(got.reshape(-1, D), oracle.sparse_reshape(*h, d, bs, scale, rp, ci, orc), d,
                "sparse step beyond the cache range, same inputs")


# ------------------------------------------------------------------ maximum size
def test_cycle_at_the_block_limit(cuda_device):
    """One mask + capture + sparse cycle at the largest supported block count (2048 blocks
    of 64 tokens, one head): the key-tile lists are at their longest and the sparse kernel's
    list buffers push it to one CTA per SM.  Mask rows, then sampled rows of the capture and
    the sparse step, against the oracle."""
    N, d, bs = 2048 * 64, 64, 64
    w = _wl(N, d, d, bs, B=1, H=1, std=1.0, seed=17, drift=0.05)
    (h0, h1), (d0, d1) = _inputs(w, cuda_device)
    keep = 16
    kw = dict(head_dim=d, block_size=bs, scale=w.scale)
    rp, ci, sc = usa.rt_build_block_mask(d0[0], d0[1], keep_blocks=keep, block_scores=True, **kw)
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0
    pq = oracle.pool_blocks(h0[0], d, bs)
    pk = oracle.pool_blocks(h0[1], d, bs)
    s64 = oracle.block_scores(pq, pk, w.scale)
    tol = score_tol(s64)
    assert np.max(np.abs(sc.double().cpu().numpy().reshape(s64.shape) - s64)) <= tol
    rp_h, ci_h = rp.cpu().numpy(), ci.cpu().numpy()
    assert check_mask(rp_h, ci_h, s64, keep, bs, 0, tol) <= 20

    out0, st = usa.rt_attn_full_capture(*d0, row_ptr=rp, col_idx=ci, **kw)
    out1 = usa.rt_attn_sparse_reshape(*d1, row_ptr=rp, col_idx=ci, stats=st, **kw)
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0
    rng = np.random.default_rng(3)
    rows = np.unique(np.concatenate([[0, 63, 64, 127, N - 129, N - 1], rng.choice(N, 90, replace=False)]))
    idx = torch.as_tensor(rows, device=cuda_device)
    orc = oracle.full_capture(*h0, d, bs, w.scale, rp_h, ci_h, rows=rows)
    orc_abs = oracle.full_capture(h0[0], h0[1], h0[2].abs(), d, bs, w.scale, rp_h, ci_h, rows=rows)["u"]
    compare_out(out0.reshape(-1, d)[idx], orc["o"], d, "capture O at the block limit")
    compare_stats(st, rows, orc, orc_abs, d, "capture stats at the block limit")
    want = oracle.sparse_reshape(*h1, d, bs, w.scale, rp_h, ci_h, orc, rows=rows)
    compare_out(out1.reshape(-1, d)[idx], want, d, "sparse O at the block limit")


# ------------------------------------------------------------------ degenerate lengths
@pytest.mark.parametrize("N,d,D,bs", [(1, 64, 64, 64), (17, 72, 80, 64), (63, 64, 64, 64), (65, 64, 64, 64),
                                      (129, 64, 64, 128), (1, 128, 128, 128)])
def test_cycle_short_sequences(cuda_device, N, d, D, bs):
    """Sequences shorter than one query tile, or one token past a block: the TMA boxes reach
    past the tensor and every tile is ragged.  Mask, capture and sparse step on every row."""
    w = _wl(N, d, D, bs, B=2, H=2, std=1.0, seed=100 + N, drift=0.05)
    (h0, h1), (d0, d1) = _inputs(w, cuda_device)
    nb = w.n_blocks
    keep = max(1, nb // 2)
    kw = dict(head_dim=d, block_size=bs, scale=w.scale)
    rp, ci = usa.rt_build_block_mask(d0[0], d0[1], keep_blocks=keep, **kw)
    out0, st = usa.rt_attn_full_capture(*d0, row_ptr=rp, col_idx=ci, **kw)
    out1 = usa.rt_attn_sparse_reshape(*d1, row_ptr=rp, col_idx=ci, stats=st, **kw)
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0
    s64 = oracle.block_scores(oracle.pool_blocks(h0[0], d, bs), oracle.pool_blocks(h0[1], d, bs), w.scale)
    rpo, cio = rp.cpu().numpy(), ci.cpu().numpy()  # checked against the oracle's selection
    check_mask(rpo, cio, s64, keep, bs, 0, score_tol(s64))
    orc = oracle.full_capture(*h0, d, bs, w.scale, rpo, cio)
    compare_out(out0.reshape(-1, D), orc["o"], d, "capture O (short)")
    want = oracle.sparse_reshape(*h1, d, bs, w.scale, rpo, cio, orc)
    compare_out(out1.reshape(-1, D), want, d, "sparse O (short)")


# ------------------------------------------------------------------ binding checks
def test_binding_rejects_mismatched_buffers(cuda_device):
    """Caller-supplied buffers of the wrong dtype, shape or device raise before any launch
    (the C ABI cannot see buffer sizes)."""
    B, H, N, d = 1, 2, 256, 64
    q = torch.zeros(B, H, N, d, dtype=torch.bfloat16, device=cuda_device)
    kw = dict(head_dim=d, block_size=64, scale=0.125)
    rp, ci = usa.rt_build_block_mask(q, q, keep_blocks=2, **kw)
    with pytest.raises(ValueError):
        usa.rt_build_block_mask(q, q, keep_blocks=2, row_ptr=rp[:-1], **kw)              # too short
    with pytest.raises(ValueError):
        usa.rt_build_block_mask(q, q, keep_blocks=2, col_idx=ci.to(torch.int64), **kw)     # dtype
    _, st = usa.rt_attn_full_capture(q, q, q, row_ptr=rp, col_idx=ci, **kw)
    with pytest.raises(ValueError):
        usa.rt_attn_full_capture(q, q, q, row_ptr=rp, col_idx=ci, out=q[:, :1], **kw)      # shape
    bad = usa.Stats(st.m, st.zfull, st.zkept, st.u[..., :32].contiguous())
    with pytest.raises(ValueError):
        usa.rt_attn_sparse_reshape(q, q, q, row_ptr=rp, col_idx=ci, stats=bad, **kw)       # U width
    with pytest.raises(ValueError):
        usa.rt_attn_sparse_reshape(q, q, q, row_ptr=rp.cpu(), col_idx=ci, stats=st, **kw)  # device
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0


# ------------------------------------------------------------------ compressed residual cache (f16 U, row scale)
def _decoded(st):
    """The statistics with U decoded to fp32 (compare_stats reads .u)."""
    return usa.Stats(st.m, st.zfull, st.zkept, st.residual())


@pytest.mark.parametrize("N,d,D,bs", CASES)
@pytest.mark.parametrize("keep_frac", [Fraction(1, 4), Fraction(1, 1)])
def test_compressed_capture_matches_oracle(cuda_device, N, d, D, bs, keep_frac):
    """The f16 cache with one power-of-two scale per row, decoded, against the oracle's U at
    the unchanged statistics tolerance; output and the other statistics as before."""
    w = _wl(N, d, D, bs, std=1.2, seed=7 * N + d)
    (h0, _), (d0, _) = _inputs(w, cuda_device)
    bh, nb = w.batch * w.heads, w.n_blocks
    keep = w.keep_blocks(keep_frac)
    rp, ci = random_csr(bh, nb, keep, seed=N)
    out, st = usa.rt_attn_full_capture(*d0, head_dim=d, block_size=bs, scale=w.scale, compressed=True,
                                       row_ptr=to_dev(rp, cuda_device), col_idx=to_dev(ci, cuda_device))
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0
    assert st.compressed and st.u.dtype == torch.float16
    orc = oracle.full_capture(*h0, d, bs, w.scale, rp, ci)
    orc_abs = oracle.full_capture(h0[0], h0[1], h0[2].abs(), d, bs, w.scale, rp, ci)["u"]
    compare_out(out.reshape(-1, D), orc["o"], d, "capture O (compressed cache)")
    compare_stats(_decoded(st), np.arange(bh * N), orc, orc_abs, d, "capture stats (compressed cache)")
    if keep == nb:
        assert torch.all(st.u == 0) and torch.all(st.u_scale == 1)


@pytest.mark.parametrize("N,d,D,bs", [(1000, 64, 64, 64), (1000, 72, 80, 128), (1000, 128, 128, 64)])
def test_compressed_cache_is_the_fp32_cache_rounded(cuda_device, N, d, D, bs):
    """Both capture variants compute the same fp32 U; the compressed one stores it as
    f16(U * 2^k) with 2^-k in u_scale and the row's largest |U| * 2^k in [2^14, 2^15):
    bit for bit, and the output and the other statistics are identical."""
    w = _wl(N, d, D, bs, std=1.2, seed=3 * N + d)
    (_, _), (d0, _) = _inputs(w, cuda_device)
    bh, nb = w.batch * w.heads, w.n_blocks
    rp, ci = random_csr(bh, nb, max(1, nb // 4), seed=N + 5)
    kw = dict(head_dim=d, block_size=bs, scale=w.scale, row_ptr=to_dev(rp, cuda_device),
              col_idx=to_dev(ci, cuda_device))
    o32, s32 = usa.rt_attn_full_capture(*d0, **kw)
    o16, s16 = usa.rt_attn_full_capture(*d0, compressed=True, **kw)
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0
    assert torch.equal(o32.view(torch.int16), o16.view(torch.int16))
    for a, b in ((s32.m, s16.m), (s32.zfull, s16.zfull), (s32.zkept, s16.zkept)):
        assert torch.equal(a, b)
    sc = s16.u_scale
    mant, _ = torch.frexp(sc)
    assert torch.all(mant == 0.5), "scales are powers of two"
    want = (s32.u / sc[..., None]).to(torch.float16)
    assert torch.equal(want.view(torch.int16), s16.u.view(torch.int16))
    amax = s16.u.float().abs().amax(-1)
    nz = s32.u.abs().amax(-1) > 0
    assert torch.all((amax[nz] >= 2.0 ** 14) & (amax[nz] <= 2.0 ** 15))


@pytest.mark.parametrize("N,d,D,bs", CASES)
def test_sparse_with_compressed_cache_matches_oracle(cuda_device, N, d, D, bs):
    """Capture with the compressed cache, then the sparse step on drifted inputs reading it:
    against the oracle's sparse step with its own fp64 statistics."""
    w = _wl(N, d, D, bs, std=1.2, seed=11 * N + d, drift=0.05)
    (h0, h1), (d0, d1) = _inputs(w, cuda_device)
    bh, nb = w.batch * w.heads, w.n_blocks
    keep = w.keep_blocks(Fraction(1, 4))
    rp, ci = random_csr(bh, nb, keep, seed=N + 1)
    kw = dict(head_dim=d, block_size=bs, scale=w.scale, row_ptr=to_dev(rp, cuda_device),
              col_idx=to_dev(ci, cuda_device))
    _, st = usa.rt_attn_full_capture(*d0, compressed=True, **kw)
    tiles = usa.rt_pair_query_blocks(d0[0], kw["row_ptr"], kw["col_idx"], head_dim=d, block_size=bs)
    out = usa.rt_attn_sparse_reshape(*d1, stats=st, tile_blocks=tiles, **kw)
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0
    st_o = oracle.full_capture(*h0, d, bs, w.scale, rp, ci)
    want = oracle.sparse_reshape(*h1, d, bs, w.scale, rp, ci, st_o)
    compare_out(out.reshape(-1, D), want, d, "sparse O (compressed cache)")
    # unchanged inputs: the sparse step reading the compressed cache recovers the capture output
    o0 = usa.rt_attn_sparse_reshape(*d0, stats=st, tile_blocks=tiles, **kw)
    torch.cuda.synchronize()
    compare_out(o0.reshape(-1, D), st_o["o"], d, "sparse on unchanged inputs (compressed cache)")


@pytest.mark.parametrize("gap", [14.0, 18.0, 30.0])
def test_compressed_capture_peaked_rows(cuda_device, gap):
    """The peaked rows with the compressed cache: each row's scale follows its own largest
    |U|, however small U is next to the row's maximum."""
    N, d, D, bs, peak = 2000, 64, 64, 64, 1500
    g = torch.Generator().manual_seed(int(gap * 10) + N + peak)
    B, H = 1, 2
    scale = 1.0 / np.sqrt(d)
    u = torch.randn(d, generator=g)
    q = (u + 0.3 * torch.randn(B, H, N, d, generator=g)).to(torch.bfloat16)
    k = 0.5 * torch.randn(B, H, N, d, generator=g)
    k[:, :, peak] = gap / (scale * float(u @ u)) * u
    k = k.to(torch.bfloat16)
    v = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    nb = -(-N // bs)
    rp, ci = _csr_with_block(B * H, nb, nb // 4, seed=N + peak, block=peak // bs)
    dq, dk, dv = (x.to(cuda_device) for x in (q, k, v))
    out, st = usa.rt_attn_full_capture(dq, dk, dv, head_dim=d, block_size=bs, scale=scale, compressed=True,
                                       row_ptr=to_dev(rp, cuda_device), col_idx=to_dev(ci, cuda_device))
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0
    orc = oracle.full_capture(q, k, v, d, bs, scale, rp, ci)
    orc_abs = oracle.full_capture(q, k, v.abs(), d, bs, scale, rp, ci)["u"]
    compare_out(out.reshape(-1, D), orc["o"], d, f"peak gap {gap:g}: capture O (compressed)")
    compare_stats(_decoded(st), np.arange(B * H * N), orc, orc_abs, d, f"peak gap {gap:g}: stats (compressed)")


# ------------------------------------------------------------------ mask from exact block masses
def mass_tol(a64):
    """Bound on |fp32 GPU block mass - fp64 oracle mass| used for tie decisions."""
    return 1e-5 * (1.0 + float(np.max(np.abs(a64))))


@pytest.mark.parametrize("N,d,D,bs", CASES)
@pytest.mark.parametrize("keep_frac", [Fraction(1, 4), Fraction(1, 1)])
def test_exact_mask_matches_oracle(cuda_device, N, d, D, bs, keep_frac):
    """Block masses from the capture pass against the oracle's fp64 softmax sums, and the
    kept sets against the oracle's selection on them (near ties as for the pooled mask)."""
    w = _wl(N, d, D, bs, std=1.3, seed=13 * N + d)
    (h0, _), (d0, _) = _inputs(w, cuda_device)
    nb = w.n_blocks
    keep = w.keep_blocks(keep_frac)
    forced = 70 if keep >= 2 else 0
    rp, ci, mass = usa.rt_build_block_mask_exact(*d0, head_dim=d, block_size=bs, scale=w.scale, keep_blocks=keep,
                                                 forced_prefix_tokens=forced, block_mass=True)
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0
    a64 = oracle.block_mass(h0[0], h0[1], d, bs, w.scale)
    tol = mass_tol(a64)
    got = mass.double().cpu().numpy().reshape(a64.shape)
    assert np.max(np.abs(got - a64)) <= tol, np.max(np.abs(got - a64))
    differ = check_mask(rp.cpu().numpy(), ci.cpu().numpy(), a64, keep, bs, forced, tol)
    assert differ <= max(1, (w.batch * w.heads * nb) // 100)


def test_exact_mask_with_caller_workspace_is_identical(cuda_device):
    """A caller workspace (filled with garbage first) gives the same masses and CSR as the
    library's pool, and a too-small one is refused."""
    N, d, D, bs = 1000, 72, 80, 64
    w = _wl(N, d, D, bs, std=1.3, seed=77)
    _, (d0, _) = _inputs(w, cuda_device)
    kw = dict(head_dim=d, block_size=bs, scale=w.scale, keep_blocks=4, forced_prefix_tokens=0, block_mass=True)
    rp, ci, mass = usa.rt_build_block_mask_exact(*d0, **kw)
    nbytes = usa.rt_exact_mask_workspace_bytes(w.batch, w.heads, N, head_dim=d, head_dim_padded=D, block_size=bs)
    ws = torch.randint(0, 256, (nbytes,), dtype=torch.uint8, device=cuda_device)
    rp2, ci2, mass2 = usa.rt_build_block_mask_exact(*d0, workspace=ws, **kw)
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0
    assert torch.equal(rp, rp2) and torch.equal(ci, ci2) and torch.equal(mass, mass2)
    with pytest.raises(usa.RtError):
        usa.rt_build_block_mask_exact(*d0, workspace=ws[:nbytes - 256], **kw)


def test_exact_mask_keeps_a_dominant_block(cuda_device):
    """One key aligned with every query: with keep = 1 every query block keeps its block,
    whatever the pooled block means say."""
    N, d, bs = 1000, 64, 64
    g = torch.Generator().manual_seed(9)
    u = torch.randn(d, generator=g)
    q = (u + 0.2 * torch.randn(1, 2, N, d, generator=g)).to(torch.bfloat16)
    k = 0.3 * torch.randn(1, 2, N, d, generator=g)
    k[:, :, 777] = 0.6 * u
    k[:, :, 768:777] -= 0.3 * u  # the block's mean points away from the queries
    k = k.to(torch.bfloat16)
    v = torch.randn(1, 2, N, d, generator=g).to(torch.bfloat16)
    rp, ci = usa.rt_build_block_mask_exact(q.to(cuda_device), k.to(cuda_device), v.to(cuda_device), head_dim=d,
                                           block_size=bs, scale=0.125, keep_blocks=1)
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0
    assert torch.all(ci == 777 // bs)
    rp_o, ci_o = oracle.build_block_mask_exact(q, k, d, bs, 0.125, 1, 0)
    assert np.array_equal(ci.cpu().numpy(), ci_o)


# ------------------------------------------------------------------ Hilbert token order
@pytest.mark.parametrize("D,d", [(64, 64), (80, 72), (128, 112)])
def test_permute_tokens_matches_oracle(cuda_device, D, d):
    """Gather and scatter by the Hilbert order equal the oracle's reindexing bit for bit and
    undo each other; an entry outside [0, N) gathers a zero row."""
    B, H, gh, gw = 2, 3, 24, 40
    N = gh * gw
    x = torch.zeros(B, H, N, D, dtype=torch.bfloat16)
    x[..., :d] = torch.randn(B, H, N, d, generator=torch.Generator().manual_seed(D)).to(torch.bfloat16)
    perm = usa.rt_hilbert_order(gh, gw)
    pd = perm.to(cuda_device)
    xd = x.to(cuda_device)
    fwd = usa.rt_permute_tokens(xd, pd, head_dim=d)
    back = usa.rt_permute_tokens(fwd, pd, inverse=True, head_dim=d)
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0
    want = oracle.permute_tokens(x, perm.numpy())
    assert torch.equal(fwd.cpu().view(torch.int16), want.view(torch.int16))
    assert torch.equal(back.cpu().view(torch.int16), x.view(torch.int16))
    bad = perm.clone()
    bad[7] = -1
    g = usa.rt_permute_tokens(xd, bad.to(cuda_device), head_dim=d)
    torch.cuda.synchronize()
    assert torch.all(g[:, :, 7] == 0) and torch.equal(g[:, :, 8].cpu(), want[:, :, 8])


@pytest.mark.parametrize("gh,gw,d,D,bs", [(32, 32, 72, 80, 64), (24, 40, 64, 64, 64), (32, 32, 72, 80, 128)])
def test_hilbert_cycle_matches_oracle(cuda_device, gh, gw, d, D, bs):
    """Q, K, V reordered along the Hilbert curve, then mask, capture and sparse step on the
    reordered tokens, the outputs mapped back: against the oracle doing the same steps."""
    N = gh * gw
    w = Workload(name="case", batch=1, heads=2, seq_len=N, head_dim=d, head_dim_padded=D, block_size=bs,
                 keep=(Fraction(1, 8),), forced_prefix_tokens=0, steps=2, capture_every=2, drift_sigma=0.05,
                 kind="iid", iid_std=1.2, seed=gh + gw + bs)
    (h0, h1), (d0, d1) = _inputs(w, cuda_device)
    perm = usa.rt_hilbert_order(gh, gw)
    pd = perm.to(cuda_device)
    p0 = [usa.rt_permute_tokens(x, pd, head_dim=d) for x in d0]
    p1 = [usa.rt_permute_tokens(x, pd, head_dim=d) for x in d1]
    kw = dict(head_dim=d, block_size=bs, scale=w.scale)
    keep = w.keep_blocks()
    rp, ci, sc = usa.rt_build_block_mask(p0[0], p0[1], keep_blocks=keep, block_scores=True, **kw)
    out0p, st = usa.rt_attn_full_capture(*p0, row_ptr=rp, col_idx=ci, **kw)
    out1p = usa.rt_attn_sparse_reshape(*p1, row_ptr=rp, col_idx=ci, stats=st, **kw)
    out0 = usa.rt_permute_tokens(out0p, pd, inverse=True, head_dim=d)
    out1 = usa.rt_permute_tokens(out1p, pd, inverse=True, head_dim=d)
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0
    # oracle: the same steps on its own reordering of the host tensors
    ph0 = [oracle.permute_tokens(x, perm.numpy()) for x in h0]
    ph1 = [oracle.permute_tokens(x, perm.numpy()) for x in h1]
    _, _, s64 = oracle.build_block_mask(ph0[0], ph0[1], d, bs, w.scale, keep, 0, return_scores=True)
    tol = score_tol(s64)
    assert np.max(np.abs(sc.double().cpu().numpy().reshape(s64.shape) - s64)) <= tol
    rp_h, ci_h = rp.cpu().numpy(), ci.cpu().numpy()
    assert check_mask(rp_h, ci_h, s64, keep, bs, 0, tol) <= 1
    orc = oracle.full_capture(*ph0, d, bs, w.scale, rp_h, ci_h)
    want1 = oracle.sparse_reshape(*ph1, d, bs, w.scale, rp_h, ci_h, orc)
    inv = np.argsort(perm.numpy())
    bh = w.batch * w.heads
    to_orig = lambda a: a.reshape(bh, N, -1)[:, inv].reshape(bh * N, -1)
    compare_out(out0.reshape(-1, D), to_orig(orc["o"]), d, "Hilbert capture O")
    compare_out(out1.reshape(-1, D), to_orig(want1), d, "Hilbert sparse O")


def test_hilbert_cycle_on_a_video_grid_with_text_prefix(cuda_device):
    """Video token layout (text tokens in front, frames of a patch grid that is not a power of
    two): the text keeps its place, each frame follows the enclosing curve; the cycle on the
    reordered tokens against the oracle doing the same steps."""
    T, F, gh, gw = 70, 3, 10, 13
    N = T + F * gh * gw
    d, D, bs = 64, 64, 64
    w = Workload(name="case", batch=1, heads=2, seq_len=N, head_dim=d, head_dim_padded=D, block_size=bs,
                 keep=(Fraction(1, 4),), forced_prefix_tokens=T, steps=2, capture_every=2, drift_sigma=0.05,
                 kind="iid", iid_std=1.2, seed=5)
    (h0, h1), (d0, d1) = _inputs(w, cuda_device)
    perm = usa.rt_hilbert_order(gh, gw, frames=F, prefix_tokens=T)
    assert np.array_equal(perm.numpy(), oracle.hilbert_order(gh, gw, frames=F, prefix=T))
    pd = perm.to(cuda_device)
    p0 = [usa.rt_permute_tokens(x, pd, head_dim=d) for x in d0]
    p1 = [usa.rt_permute_tokens(x, pd, head_dim=d) for x in d1]
    kw = dict(head_dim=d, block_size=bs, scale=w.scale)
    keep = w.keep_blocks()
    rp, ci, sc = usa.rt_build_block_mask(p0[0], p0[1], keep_blocks=keep, forced_prefix_tokens=T, block_scores=True,
                                         **kw)
    _, st = usa.rt_attn_full_capture(*p0, row_ptr=rp, col_idx=ci, **kw)
    out1 = usa.rt_permute_tokens(usa.rt_attn_sparse_reshape(*p1, row_ptr=rp, col_idx=ci, stats=st, **kw), pd,
                                 inverse=True, head_dim=d)
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0
    ph0 = [oracle.permute_tokens(x, perm.numpy()) for x in h0]
    ph1 = [oracle.permute_tokens(x, perm.numpy()) for x in h1]
    _, _, s64 = oracle.build_block_mask(ph0[0], ph0[1], d, bs, w.scale, keep, T, return_scores=True)
    tol = score_tol(s64)
    rp_h, ci_h = rp.cpu().numpy(), ci.cpu().numpy()
    assert check_mask(rp_h, ci_h, s64, keep, bs, T, tol) <= 1
    orc = oracle.full_capture(*ph0, d, bs, w.scale, rp_h, ci_h)
    want1 = oracle.sparse_reshape(*ph1, d, bs, w.scale, rp_h, ci_h, orc)
    inv = np.argsort(perm.numpy())
    compare_out(out1.reshape(-1, D), want1.reshape(2, N, d)[:, inv].reshape(2 * N, d), d, "Hilbert video sparse O")
