"""Saving and reloading a capture step's cache (CPU: the file round trip; GPU: a
sparse step from the reloaded cache, bit for bit, and replayed on the oracle)."""
import numpy as np
import pytest
import torch

import ultra_sparse_attention_b200 as usa
from ultra_sparse_attention_b200.cache_io import load_cache, save_cache


def _fake_cache(compressed, B=1, H=2, N=300, D=80, bs=64):
    g = torch.Generator().manual_seed(3)
    nb = -(-N // bs)
    rp = torch.arange(B * H * nb + 1, dtype=torch.int32) * 2
    ci = torch.randint(0, nb, (B * H * nb * 2,), dtype=torch.int32, generator=g)
    f = lambda *s: torch.randn(*s, generator=g)
    u = f(B, H, N, D)
    st = usa.Stats(f(B, H, N), f(B, H, N).abs() + 1, f(B, H, N).abs() + 1,
                   u.to(torch.float16) if compressed else u, f(B, H, N).abs() if compressed else None)
    tiles = torch.randint(-1, nb, (B * H, -(-N // 128), 2), dtype=torch.int32, generator=g)
    return rp, ci, st, tiles


@pytest.mark.parametrize("compressed", [False, True])
def test_cache_file_round_trip(tmp_path, compressed):
    rp, ci, st, tiles = _fake_cache(compressed)
    path = tmp_path / "cache.npz"
    save_cache(path, head_dim=72, block_size=64, scale=0.125, row_ptr=rp, col_idx=ci, stats=st, tile_blocks=tiles)
    c = load_cache(path, device="cpu")
    assert c["head_dim"] == 72 and c["block_size"] == 64 and c["scale"] == 0.125 and c["shape"] == (1, 2, 300, 80)
    assert torch.equal(c["row_ptr"], rp) and torch.equal(c["col_idx"], ci) and torch.equal(c["tile_blocks"], tiles)
    s2 = c["stats"]
    assert s2.compressed == compressed
    for a, b in ((s2.m, st.m), (s2.zfull, st.zfull), (s2.zkept, st.zkept)):
        assert torch.equal(a, b)
    assert torch.equal(s2.u.view(torch.int16) if compressed else s2.u, st.u.view(torch.int16) if compressed else st.u)
    if compressed:
        assert torch.equal(s2.u_scale, st.u_scale)


def test_cache_file_without_table_and_bad_files(tmp_path):
    rp, ci, st, _ = _fake_cache(False)
    path = tmp_path / "c.npz"
    save_cache(path, head_dim=80, block_size=64, scale=0.1, row_ptr=rp, col_idx=ci, stats=st)
    assert load_cache(path, device="cpu")["tile_blocks"] is None
    with np.load(path) as z:
        bad = {k: z[k] for k in z.files}
    bad["format"] = np.array(99, np.int64)
    np.savez(tmp_path / "bad.npz", **bad)
    with pytest.raises(ValueError):
        load_cache(tmp_path / "bad.npz", device="cpu")
    bad["format"] = np.array(1, np.int64)
    bad["row_ptr"] = bad["row_ptr"][:-1]
    np.savez(tmp_path / "bad2.npz", **bad)
    with pytest.raises(ValueError):
        load_cache(tmp_path / "bad2.npz", device="cpu")


@pytest.mark.gpu
@pytest.mark.parametrize("compressed", [False, True])
def test_sparse_step_from_a_reloaded_cache(cuda_device, tmp_path, compressed):
    """Capture, save, reload, run the sparse step: the same bits as from the in-memory cache;
    the file alone replays the step on the oracle within the output tolerance."""
    import oracle
    from parity import compare_out, sample_rows
    from ultra_sparse_attention_b200.workloads import WORKLOADS, denoising_inputs
    w = WORKLOADS["image"]
    st_ = denoising_inputs(w, 2)
    h0, h1 = next(st_)[1:], next(st_)[1:]
    d0 = [x.to(cuda_device) for x in h0]
    d1 = [x.to(cuda_device) for x in h1]
    kw = dict(head_dim=w.head_dim, block_size=w.block_size, scale=w.scale)
    rp, ci = usa.rt_build_block_mask(d0[0], d0[1], keep_blocks=w.keep_blocks(), **kw)
    tiles = usa.rt_pair_query_blocks(d0[0], rp, ci, head_dim=w.head_dim, block_size=w.block_size)
    _, st = usa.rt_attn_full_capture(*d0, row_ptr=rp, col_idx=ci, compressed=compressed, **kw)
    path = tmp_path / "layer0.npz"
    save_cache(path, row_ptr=rp, col_idx=ci, stats=st, tile_blocks=tiles, **kw)
    c = load_cache(path, device=cuda_device)
    a = usa.rt_attn_sparse_reshape(*d1, row_ptr=rp, col_idx=ci, stats=st, tile_blocks=tiles, **kw)
    b = usa.rt_attn_sparse_reshape(*d1, row_ptr=c["row_ptr"], col_idx=c["col_idx"], stats=c["stats"],
                                   tile_blocks=c["tile_blocks"], head_dim=c["head_dim"],
                                   block_size=c["block_size"], scale=c["scale"])
    torch.cuda.synchronize()
    assert usa.rt_take_device_error() == 0
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    # offline replay: the oracle's sparse step from the file's statistics
    cc = load_cache(path, device="cpu")
    B, H, N, D = cc["shape"]
    rows = sample_rows(B * H, N, 128, seed=4)
    s = cc["stats"]
    u = s.residual().reshape(-1, D)[torch.as_tensor(rows)].double().numpy()[:, :w.head_dim]
    stats = {"m": s.m.reshape(-1)[rows].double().numpy(), "zfull": s.zfull.reshape(-1)[rows].double().numpy(),
             "zkept": s.zkept.reshape(-1)[rows].double().numpy(), "u": u}
    want = oracle.sparse_reshape(*h1, cc["head_dim"], cc["block_size"], cc["scale"], cc["row_ptr"].numpy(),
                                 cc["col_idx"].numpy(), stats, rows=rows)
    compare_out(b.reshape(-1, D)[torch.as_tensor(rows, device=cuda_device)], want, w.head_dim, "replayed sparse O")
