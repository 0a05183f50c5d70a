"""Pins of the fp64 oracle to things other than itself.

Each test checks one oracle function against an independent source: a
library routine (torch SDPA / logsumexp / softmax in fp64, numpy), brute
force on tiny inputs, or a closed form derived from the method's
definition.  A plausible slip in the oracle (a dropped term, a flipped sign
or index, a transposed operand, a wrong ratio direction) fails one of them.
"""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle


def _bf16(x):
    return torch.as_tensor(x, dtype=torch.float32).to(torch.bfloat16)


def _rand_qkv(B, H, N, d, D, std=1.0, seed=0):
    g = torch.Generator().manual_seed(seed)
    out = []
    for _ in range(3):
        x = torch.zeros(B, H, N, D, dtype=torch.bfloat16)
        x[..., :d] = (torch.randn(B, H, N, d, generator=g) * std).to(torch.bfloat16)
        out.append(x)
    return out


def _csr_from_sets(sets):
    row_ptr = [0]
    col = []
    for s in sets:
        col += sorted(s)
        row_ptr.append(len(col))
    return np.array(row_ptr, np.int32), np.array(col, np.int32)


def _block_mask_dense(row_ptr, col_idx, bh_count, n, bs):
    """Boolean [BH, N, N] token mask from a block CSR (True = kept)."""
    nb = -(-n // bs)
    m = torch.zeros(bh_count, n, n, dtype=torch.bool)
    for bh in range(bh_count):
        for qb in range(nb):
            r = bh * nb + qb
            for e in range(row_ptr[r], row_ptr[r + 1]):
                kb = col_idx[e]
                m[bh, qb * bs:(qb + 1) * bs, kb * bs:(kb + 1) * bs] = True
    return m


def _sdpa64(q, k, v, d, mask=None):
    """torch scaled_dot_product_attention in fp64 over the logical columns."""
    B, H, N, D = q.shape
    qq = q[..., :d].double().reshape(B * H, N, d)
    kk = k[..., :d].double().reshape(B * H, N, d)
    vv = v[..., :d].double().reshape(B * H, N, d)
    return torch.nn.functional.scaled_dot_product_attention(
        qq, kk, vv, attn_mask=mask, scale=1.0 / math.sqrt(d))


# ---------------------------------------------------------------- pooling
def test_pool_matches_numpy_mean_with_ragged_tail_and_pad_ignored():
    N, d, D, bs = 200, 72, 80, 64                      # last block: 8 tokens
    q, _, _ = _rand_qkv(1, 3, N, d, D)
    q[..., d:] = _bf16(7.0)                            # pad columns must not enter the mean
    got = oracle.pool_blocks(q, d, bs)
    x = q[..., :d].float().numpy().astype(np.float64).reshape(3, N, d)
    for b in range(4):
        want = x[:, b * bs:min(N, (b + 1) * bs)].mean(axis=1)
        np.testing.assert_allclose(got[:, b], want, rtol=0, atol=1e-13)
    assert got.shape == (3, 4, d)


def test_block_scores_match_numpy_matmul():
    rng = np.random.default_rng(1)
    pq, pk = rng.normal(size=(2, 5, 7)), rng.normal(size=(2, 5, 7))
    got = oracle.block_scores(pq, pk, 0.25)
    want = 0.25 * np.einsum("bqc,bkc->bqk", pq, pk)
    np.testing.assert_allclose(got, want, rtol=1e-14, atol=1e-14)
    # transposed operands would give the transpose: make sure it is not symmetric here
    assert not np.allclose(got, got.transpose(0, 2, 1))


# ---------------------------------------------------------------- selection
def _brute_topk(scores, keep, forced):
    """The unique kept set: forced blocks plus a set S of the others such that
    every member of S beats every non-member (score desc, then index asc)."""
    nkb = len(scores)
    rest = [kb for kb in range(nkb) if kb >= forced]
    def beats(a, b):
        return scores[a] > scores[b] or (scores[a] == scores[b] and a < b)
    found = []
    for S in itertools.combinations(rest, keep - forced):
        out = [y for y in rest if y not in S]
        if all(beats(x, y) for x in S for y in out):
            found.append(set(S) | set(range(forced)))
    assert len(found) == 1
    return found[0]


@pytest.mark.parametrize("keep", [1, 2, 3, 5, 8])
@pytest.mark.parametrize("forced_tokens,bs", [(0, 64), (1, 64), (130, 64), (100, 128)])
@pytest.mark.parametrize("ties", [False, True])
def test_select_equals_brute_force(keep, forced_tokens, bs, ties):
    nkb = 8
    forced = min(nkb, -(-forced_tokens // bs)) if forced_tokens > 0 else 0
    rng = np.random.default_rng(keep * 100 + forced_tokens + ties)
    rows = 12
    s = rng.integers(-2, 3, size=(rows, nkb)).astype(np.float64) if ties else rng.normal(size=(rows, nkb))
    if forced > keep:  # more forced blocks than kept ones: the input is rejected, not truncated
        with pytest.raises(RuntimeError, match="select failed"):
            oracle.select_blocks(s, keep, bs, forced_tokens)
        return
    row_ptr, col_idx = oracle.select_blocks(s, keep, bs, forced_tokens)
    assert list(row_ptr) == [r * keep for r in range(rows + 1)]
    for r in range(rows):
        got = col_idx[r * keep:(r + 1) * keep]
        assert list(got) == sorted(got), "kept blocks must be ascending"
        assert set(got) == _brute_topk(s[r], keep, forced)


def test_select_max_sum_without_ties():
    rng = np.random.default_rng(7)
    s = rng.normal(size=(20, 8))
    _, col_idx = oracle.select_blocks(s, 3, 64, 0)
    for r in range(20):
        best = max(itertools.combinations(range(8), 3), key=lambda c: s[r, list(c)].sum())
        assert set(col_idx[r * 3:(r + 1) * 3]) == set(best)


def test_select_degenerate_keeps():
    s = np.random.default_rng(3).normal(size=(4, 6))
    _, ci = oracle.select_blocks(s, 6, 64, 0)            # keep all
    assert ci.reshape(4, 6).tolist() == [list(range(6))] * 4
    _, ci = oracle.select_blocks(s, 2, 64, 100)          # keep == forced
    assert ci.reshape(4, 2).tolist() == [[0, 1]] * 4
    with pytest.raises(RuntimeError):
        oracle.select_blocks(s, 1, 64, 100)              # forced > keep is rejected


# ---------------------------------------------------------------- full attention + stats
@pytest.mark.parametrize("N,d,D,bs", [(256, 64, 64, 64), (200, 72, 80, 64), (384, 72, 80, 128)])
def test_capture_matches_torch_fp64(N, d, D, bs):
    B, H = 1, 2
    q, k, v = _rand_qkv(B, H, N, d, D, std=1.0, seed=N)
    nb = -(-N // bs)
    rng = np.random.default_rng(N)
    sets = [set(rng.choice(nb, size=max(1, nb // 3), replace=False).tolist()) for _ in range(B * H * nb)]
    row_ptr, col_idx = _csr_from_sets(sets)
    st = oracle.full_capture(q, k, v, d, bs, 1 / math.sqrt(d), row_ptr, col_idx, threads=4)

    o_ref = _sdpa64(q, k, v, d).reshape(-1, d).numpy()
    np.testing.assert_allclose(st["o"], o_ref, rtol=0, atol=1e-12)

    qq = q[..., :d].double().reshape(B * H, N, d)
    kk = k[..., :d].double().reshape(B * H, N, d)
    vv = v[..., :d].double().reshape(B * H, N, d)
    s = torch.einsum("bic,bjc->bij", qq, kk) / math.sqrt(d)
    keep = _block_mask_dense(row_ptr, col_idx, B * H, N, bs)
    np.testing.assert_allclose(st["m"], s.amax(-1).reshape(-1).numpy(), rtol=0, atol=1e-13)
    lse = torch.logsumexp(s, -1).reshape(-1).numpy()
    np.testing.assert_allclose(st["m"] + np.log(st["zfull"]), lse, rtol=0, atol=1e-12)
    lse_kept = torch.logsumexp(s.masked_fill(~keep, -math.inf), -1).reshape(-1).numpy()
    np.testing.assert_allclose(st["m"] + np.log(st["zkept"]), lse_kept, rtol=0, atol=1e-12)
    p = torch.softmax(s, -1)
    u_over_z = torch.einsum("bij,bjc->bic", p * (~keep), vv).reshape(-1, d).numpy()
    np.testing.assert_allclose(st["u"] / st["zfull"][:, None], u_over_z, rtol=0, atol=1e-12)
    assert np.all(st["zfull"] >= st["zkept"])


def test_capture_closed_forms():
    N, d, bs = 128, 64, 64
    q, k, v = _rand_qkv(1, 1, N, d, d, seed=5)
    row_ptr, col_idx = _csr_from_sets([{0}, {1}])
    v1 = torch.ones_like(v)                              # rows of softmax sum to 1
    st = oracle.full_capture(q, k, v1, d, bs, 1 / 8, row_ptr, col_idx)
    np.testing.assert_allclose(st["o"], 1.0, rtol=0, atol=1e-14)
    # U sums exactly the masked mass when v = 1
    np.testing.assert_allclose(st["u"][:, 0], st["zfull"] - st["zkept"], rtol=1e-13)
    q0 = torch.zeros_like(q)                             # uniform attention: O = mean of V
    st = oracle.full_capture(q0, k, v, d, bs, 1 / 8, row_ptr, col_idx)
    np.testing.assert_allclose(st["o"], np.broadcast_to(v[0, 0].double().mean(0).numpy(), (N, d)), atol=1e-14)
    np.testing.assert_allclose(st["zfull"], N)
    np.testing.assert_allclose(st["zkept"], bs)
    np.testing.assert_allclose(st["m"], 0.0)


def test_capture_keep_all_has_no_residual():
    N, d, bs = 192, 64, 64
    q, k, v = _rand_qkv(1, 2, N, d, d, seed=9)
    row_ptr, col_idx = _csr_from_sets([{0, 1, 2}] * 6)
    st = oracle.full_capture(q, k, v, d, bs, 1 / 8, row_ptr, col_idx)
    assert np.all(st["u"] == 0.0)
    np.testing.assert_array_equal(st["zfull"], st["zkept"])


def test_capture_rows_subset_matches_all_rows():
    N, d, bs = 256, 64, 64
    q, k, v = _rand_qkv(1, 2, N, d, d, seed=11)
    row_ptr, col_idx = _csr_from_sets([{1, 3}] * 8)
    full = oracle.full_capture(q, k, v, d, bs, 1 / 8, row_ptr, col_idx, threads=3)
    rows = np.array([0, 63, 64, 300, 511])
    sub = oracle.full_capture(q, k, v, d, bs, 1 / 8, row_ptr, col_idx, rows=rows, threads=2)
    for key in full:
        np.testing.assert_array_equal(sub[key], full[key][rows])


# ---------------------------------------------------------------- sparse step + reshape
def _sparse_case(N=256, d=72, D=80, bs=64, seed=21):
    q, k, v = _rand_qkv(1, 2, N, d, D, std=1.0, seed=seed)
    nb = -(-N // bs)
    rng = np.random.default_rng(seed)
    sets = [set(rng.choice(nb, size=2, replace=False).tolist()) for _ in range(2 * nb)]
    return q, k, v, _csr_from_sets(sets)


def test_plain_sparse_equals_sdpa_with_block_mask():
    N, d, D, bs = 200, 72, 80, 64
    q, k, v, (row_ptr, col_idx) = _sparse_case(N, d, D, bs)
    got = oracle.sparse_reshape(q, k, v, d, bs, 1 / math.sqrt(d), row_ptr, col_idx, None)
    mask = _block_mask_dense(row_ptr, col_idx, 2, N, bs)
    want = _sdpa64(q, k, v, d, mask).reshape(-1, d).numpy()
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_reshape_keep_all_equals_full_attention_of_current_inputs():
    N, d, D, bs = 256, 64, 64, 64
    q0, k0, v0 = _rand_qkv(1, 2, N, d, D, seed=1)
    q1, k1, v1 = _rand_qkv(1, 2, N, d, D, seed=2)        # arbitrary new step
    row_ptr, col_idx = _csr_from_sets([set(range(4))] * 8)
    st = oracle.full_capture(q0, k0, v0, d, bs, 1 / 8, row_ptr, col_idx)
    got = oracle.sparse_reshape(q1, k1, v1, d, bs, 1 / 8, row_ptr, col_idx, st)
    want = _sdpa64(q1, k1, v1, d).reshape(-1, d).numpy()
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_reshape_unchanged_inputs_recover_full_attention_with_max_in_masked_block():
    N, d, D, bs = 256, 72, 80, 64
    q, k, v, (row_ptr, col_idx) = _sparse_case(N, d, D, bs, seed=3)
    # plant a dominant key in a block that query block 0 of head 0 does not keep
    masked_kb = next(kb for kb in range(4) if kb not in set(col_idx[row_ptr[0]:row_ptr[1]]))
    k[0, 0, masked_kb * bs + 5, :d] = (q[0, 0, :bs, :d].float().mean(0) * 40).to(torch.bfloat16)
    st = oracle.full_capture(q, k, v, d, bs, 1 / math.sqrt(d), row_ptr, col_idx)
    got = oracle.sparse_reshape(q, k, v, d, bs, 1 / math.sqrt(d), row_ptr, col_idx, st)
    np.testing.assert_allclose(got, st["o"], rtol=0, atol=1e-12)
    # the planted key really moved the row max out of the kept set for some rows
    s_kept_max = oracle.sparse_reshape(q, k, v, d, bs, 1 / math.sqrt(d), row_ptr, col_idx, None)
    assert np.any(np.abs(s_kept_max[:bs] - st["o"][:bs]) > 1e-3)


@pytest.mark.parametrize("delta", [-40.0, 7.5, 60.0])
def test_reshape_is_independent_of_the_cache_reference(delta):
    """The cached m is only the reference the three sums share: m + delta with Z_full,
    Z_kept and U scaled by e^-delta gives the same reshaped output (the GPU cache lowers m
    on rows led by masked keys and relies on this)."""
    N, d, D, bs = 256, 64, 64, 64
    q0, k0, v0 = _rand_qkv(1, 2, N, d, D, seed=4)
    q1, k1, v1 = _rand_qkv(1, 2, N, d, D, seed=5)
    q, k, v, (row_ptr, col_idx) = _sparse_case(N, d, D, bs, seed=6)
    st = oracle.full_capture(q0, k0, v0, d, bs, 1 / 8, row_ptr, col_idx)
    f = math.exp(-delta)
    moved = {"m": st["m"] + delta, "zfull": st["zfull"] * f, "zkept": st["zkept"] * f, "u": st["u"] * f}
    want = oracle.sparse_reshape(q1, k1, v1, d, bs, 1 / 8, row_ptr, col_idx, st)
    got = oracle.sparse_reshape(q1, k1, v1, d, bs, 1 / 8, row_ptr, col_idx, moved)
    np.testing.assert_allclose(got, want, rtol=1e-11, atol=1e-12)


def test_reshape_uniform_kept_shift_closed_form():
    """Ratio reading pinned by a closed form.

    With V unchanged and every kept score of a row shifted by the same delta,
    the kept-only average is unchanged and the cached masked part is scaled
    by exp(-delta):  o = (Z_kept/Z_full) * o_kept + exp(-delta) * U / Z_full.
    """
    N, d, bs = 128, 8, 64
    g = torch.Generator().manual_seed(4)
    qrow = torch.randint(-2, 3, (d,), generator=g).float() / 4
    qrow[0] = 0.5
    q = torch.zeros(1, 1, N, d)
    q[0, 0, :] = qrow                                    # identical queries: one delta per row
    k = torch.randint(-4, 5, (1, 1, N, d), generator=g).float() / 8
    v = torch.randint(-4, 5, (1, 1, N, d), generator=g).float() / 8
    q, k, v = (x.to(torch.bfloat16) for x in (q, k, v))
    row_ptr, col_idx = _csr_from_sets([{1}, {0}])        # block 0 keeps block 1, block 1 keeps block 0
    scale = 0.5
    st = oracle.full_capture(q, k, v, d, bs, scale, row_ptr, col_idx)
    alpha = 0.25                                         # k' = k + alpha*q on every key (all blocks kept by someone)
    k1 = (k.float() + alpha * q.float()).to(torch.bfloat16)
    assert torch.equal(k1.float(), k.float() + alpha * q.float())   # exact in bf16
    delta = scale * alpha * float((qrow * qrow).sum())
    got = oracle.sparse_reshape(q, k1, v, d, bs, scale, row_ptr, col_idx, st)
    o_kept = oracle.sparse_reshape(q, k, v, d, bs, scale, row_ptr, col_idx, None)
    want = (st["zkept"] / st["zfull"])[:, None] * o_kept + math.exp(-delta) * st["u"] / st["zfull"][:, None]
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-13)
    # the additive-denominator reading would not satisfy it
    assert not np.allclose(got, st["o"], atol=1e-6)


def test_sparse_empty_row_gives_zero():
    N, d, bs = 128, 64, 64
    q, k, v = _rand_qkv(1, 1, N, d, d, seed=8)
    row_ptr, col_idx = np.array([0, 0, 1], np.int32), np.array([1], np.int32)
    got = oracle.sparse_reshape(q, k, v, d, bs, 1 / 8, row_ptr, col_idx, None)
    assert np.all(got[:bs] == 0.0)
    assert np.all(np.isfinite(got[bs:])) and np.any(got[bs:] != 0.0)


def test_mask_step_composes_pool_score_select():
    from ultra_sparse_attention_b200.workloads import WORKLOADS, base_inputs
    w = WORKLOADS["tiny"]
    q, k, _ = base_inputs(w)
    rp, ci, s = oracle.build_block_mask(q, k, w.head_dim, w.block_size, w.scale, w.keep_blocks(), 0,
                                        return_scores=True)
    x = q.float().numpy().astype(np.float64).reshape(2, 8, 64, 64).mean(2)
    y = k.float().numpy().astype(np.float64).reshape(2, 8, 64, 64).mean(2)
    np.testing.assert_allclose(s, w.scale * np.einsum("bqc,bkc->bqk", x, y), rtol=1e-12, atol=1e-15)
    for r in range(16):
        assert set(ci[2 * r:2 * r + 2]) == _brute_topk(s.reshape(16, 8)[r], 2, 0)


# ------------------------------------------------------------------ exact block masses
def _torch_block_mass(q, k, d, bs, scale):
    """fp64 torch softmax over all keys, summed over query and key blocks (ragged tail)."""
    B, H, N, _ = q.shape
    qq = q[..., :d].double().reshape(B * H, N, d)
    kk = k[..., :d].double().reshape(B * H, N, d)
    p = torch.softmax(scale * qq @ kk.transpose(1, 2), dim=-1)       # [BH, N, N]
    nb = -(-N // bs)
    blk = torch.arange(N) // bs
    a = torch.zeros(B * H, nb, N, dtype=torch.float64).index_add_(1, blk, p)   # sum query rows
    return torch.zeros(B * H, nb, nb, dtype=torch.float64).index_add_(2, blk, a).numpy()


@pytest.mark.parametrize("N,d,D,bs", [(200, 64, 64, 64), (300, 72, 80, 128), (128, 16, 64, 64)])
def test_block_mass_matches_torch_softmax(N, d, D, bs):
    q, k, _ = _rand_qkv(2, 2, N, d, D, std=1.3, seed=N + d)
    scale = 1.0 / math.sqrt(d)
    got = oracle.block_mass(q, k, d, bs, scale)
    want = _torch_block_mass(q, k, d, bs, scale)
    assert np.max(np.abs(got - want)) <= 1e-12
    # a transposed operand (masses of K attending to Q) is a different matrix
    swapped = oracle.block_mass(k, q, d, bs, scale)
    assert np.max(np.abs(swapped - got)) > 1e-3


def test_block_mass_rows_sum_to_the_block_size():
    """Every query token's probabilities sum to 1, so a query block's masses sum to its
    number of real tokens (the ragged tail block to its own count)."""
    N, bs = 1000, 64
    q, k, _ = _rand_qkv(1, 3, N, 64, 64, std=2.0, seed=5)
    a = oracle.block_mass(q, k, 64, bs, 0.125)
    rows = np.minimum(bs, N - np.arange(-(-N // bs)) * bs)
    assert np.allclose(a.sum(-1), rows[None, :], rtol=0, atol=1e-10)
    assert np.all(a >= 0)


def test_block_mass_uniform_scores_closed_form():
    """Q = 0: every score is 0, each probability 1/N, so mass = rows(qb) * cols(kb) / N."""
    N, bs = 300, 64
    q = torch.zeros(1, 2, N, 64, dtype=torch.bfloat16)
    _, k, _ = _rand_qkv(1, 2, N, 64, 64, seed=2)
    a = oracle.block_mass(q, k, 64, bs, 0.125)
    sizes = np.minimum(bs, N - np.arange(-(-N // bs)) * bs).astype(np.float64)
    want = np.outer(sizes, sizes) / N
    assert np.max(np.abs(a - want[None])) <= 1e-11  # 4096 fp64 additions of 1/N per entry


def test_exact_mask_keeps_the_block_of_a_dominant_key():
    """A key aligned with every query (a large score for all rows) puts most of each row's
    mass in its block; with keep = 1 every query block keeps exactly that block, with keep
    = all every block, and the selection equals select_blocks on the masses."""
    N, d, bs = 512, 64, 64
    g = torch.Generator().manual_seed(9)
    u = torch.randn(d, generator=g)
    q = torch.zeros(1, 1, N, d)
    q[..., :] = u + 0.2 * torch.randn(1, 1, N, d, generator=g)
    k = 0.3 * torch.randn(1, 1, N, d, generator=g)
    k[0, 0, 333] = 0.6 * u
    q, k = q.to(torch.bfloat16), k.to(torch.bfloat16)
    rp, ci, a = oracle.build_block_mask_exact(q, k, d, bs, 0.125, 1, 0, return_mass=True)
    assert list(ci) == [333 // bs] * (N // bs)
    rp_s, ci_s = oracle.select_blocks(a, 1, bs, 0)
    assert np.array_equal(ci, ci_s) and np.array_equal(rp, rp_s)
    _, ci_all = oracle.build_block_mask_exact(q, k, d, bs, 0.125, N // bs, 0)
    assert list(ci_all) == list(range(N // bs)) * (N // bs)
    _, ci_f = oracle.build_block_mask_exact(q, k, d, bs, 0.125, 2, 100)  # forced blocks 0, 1
    assert list(ci_f) == [0, 1] * (N // bs)


def test_block_mass_listed_query_blocks_match_all():
    N, bs = 700, 64
    q, k, _ = _rand_qkv(1, 2, N, 64, 64, std=1.5, seed=8)
    full = oracle.block_mass(q, k, 64, bs, 0.125)
    nb = -(-N // bs)
    ids = np.array([0, 5, nb - 1, nb, 2 * nb - 1])
    part = oracle.block_mass(q, k, 64, bs, 0.125, qblocks=ids)
    assert np.array_equal(part, full.reshape(-1, nb)[ids])


# ------------------------------------------------------------------ Hilbert token order
def test_hilbert_order_one_is_the_u_shape():
    assert oracle.hilbert_curve(1) == [(0, 0), (0, 1), (1, 1), (1, 0)]


@pytest.mark.parametrize("k", [1, 2, 3, 4, 6])
def test_hilbert_curve_is_a_continuous_bijection_filling_quadrants(k):
    cells = oracle.hilbert_curve(k)
    n = 1 << k
    assert sorted(cells) == [(x, y) for x in range(n) for y in range(n)]          # every cell once
    for (x0, y0), (x1, y1) in zip(cells, cells[1:]):
        assert abs(x1 - x0) + abs(y1 - y0) == 1                                  # 4-adjacent steps
    assert cells[0] == (0, 0) and cells[-1] == (n - 1, 0)
    s, q = n // 2, (n * n) // 4
    quads = [(0, 0), (0, s), (s, s), (s, 0)]  # lower-left, upper-left, upper-right, lower-right
    for i, (qx, qy) in enumerate(quads):
        part = cells[i * q:(i + 1) * q]
        assert all(qx <= x < qx + s and qy <= y < qy + s for x, y in part)


def test_hilbert_order_permutation_with_prefix_frames_and_ragged_grid():
    # a 3 x 5 grid inside the 8 x 8 curve, two frames, 4 text tokens in front
    perm = oracle.hilbert_order(3, 5, frames=2, prefix=4)
    assert sorted(perm.tolist()) == list(range(4 + 2 * 15))
    assert perm[:4].tolist() == [0, 1, 2, 3]
    f0, f1 = perm[4:19] - 4, perm[19:] - 19
    assert np.array_equal(f0, f1)
    # the cells keep the order they have on the enclosing curve
    curve = [y * 5 + x for x, y in oracle.hilbert_curve(3) if x < 5 and y < 3]
    assert f0.tolist() == curve
    # a power-of-two grid is the pure curve: consecutive tokens are grid neighbours
    p = oracle.hilbert_order(16, 16)
    xy = [(t % 16, t // 16) for t in p]
    assert all(abs(a[0] - b[0]) + abs(a[1] - b[1]) == 1 for a, b in zip(xy, xy[1:]))


def test_hilbert_blocks_are_compact_squares():
    """On a 64 x 64 grid every 64-token block of the Hilbert order is an 8 x 8 square
    (the locality the reordering is for), where a row-major block is a 64 x 1 line."""
    p = oracle.hilbert_order(64, 64)
    for b in range(64):
        xs = p[b * 64:(b + 1) * 64] % 64
        ys = p[b * 64:(b + 1) * 64] // 64
        assert xs.max() - xs.min() == 7 and ys.max() - ys.min() == 7


def test_permute_tokens_round_trip_and_attention_equivariance():
    """Un-permuting undoes permuting; full attention commutes with a common permutation of
    the tokens (fp64 torch SDPA), which is what lets the attention path run on the reordered
    sequence and map its output back."""
    q, k, v = _rand_qkv(1, 2, 64, 16, 16, seed=4)
    perm = oracle.hilbert_order(8, 8)
    qp = oracle.permute_tokens(q, perm)
    assert torch.equal(oracle.permute_tokens(qp, perm, inverse=True), q)
    assert torch.equal(qp[0, 1, 5], q[0, 1, perm[5]])
    kp, vp = oracle.permute_tokens(k, perm), oracle.permute_tokens(v, perm)
    o = _sdpa64(q, k, v, 16)
    op = _sdpa64(qp, kp, vp, 16)
    back = op.reshape(1, 2, 64, 16)[..., torch.as_tensor(np.argsort(perm)), :]
    assert torch.allclose(back.reshape(o.shape), o, atol=1e-13)
