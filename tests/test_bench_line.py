"""The JSON line bench.py prints, on CPU: the keys and objects the benchmark
contract requires, and the arithmetic that ties them to the measured times.

Our arm's line is assembled from a synthetic measurement (times chosen here,
no GPU); the reference arm's line comes from a real, tiny oracle run."""
import os
import sys

import numpy as np
import pytest

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
import bench  # noqa: E402

TOP_KEYS = ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
            "scaling", "vs_baseline", "dtype", "data", "config")


class _Args:
    steps, warmup = 5, 3


def _measurement(world, with_e2e=True):
    w = bench.WORKLOADS["tiny"]
    keep = w.keep_blocks(w.keep[0])
    bh, nb = w.batch * w.heads, w.n_blocks
    row_ptr = np.arange(bh * nb + 1, dtype=np.int64) * keep
    col_idx = np.tile(np.arange(keep, dtype=np.int64), bh * nb)
    nums = bench.workload_numbers(w, keep, row_ptr, col_idx)
    e2e = {"h2d_bytes_per_step": 3 * bh * w.seq_len * w.head_dim_padded * 2,
           "d2h_bytes_per_step": bh * w.seq_len * w.head_dim_padded * 2} if with_e2e else None
    return {"w": w, "keep": keep, "keep_ratio": w.keep[0], "total_ms": 10.0, "mask_ms": 0.05, "pair_ms": 0.01,
            "capture_ms": 1.5, "sparse_ms": 0.25, "e2e": e2e, "e2e_ms": 0.4,
            "clocks": {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 12},
            "nums": nums}


@pytest.mark.parametrize("world", [1, 2])
def test_our_line_has_the_contract_keys(world):
    r = _measurement(world)
    peaks = dict(bench.FALLBACK_PEAKS)
    cpu = {"value": 0.01, "unit": bench.UNIT, "cores": 8, "kind": "oracle", "sample": "rows"}
    line = bench.build_line(_Args, r, world, peaks, "fallback", None, cpu if world == 1 else None)
    for k in TOP_KEYS:
        assert k in line, k
    assert line["metric"] == bench.METRIC and line["unit"] == bench.UNIT
    assert line["n_gpus"] == world and line["steps"] == 5 and line["warmup"] == 3
    assert line["higher_is_better"] is True and line["scaling"] == "weak"
    assert line["vs_baseline"] is None and line["data"] == "synthetic" and line["dtype"] == "bf16"
    assert line["ms_per_step"] == pytest.approx(2.0)
    assert "workload" in line["config"] and "l2" in line["config"]
    # value: dense-equivalent flops of every rank over the sparse step's time
    dense = 4.0 * 2 * 512 * 512 * 64
    assert r["nums"]["dense_flops"] == dense
    assert line["value"] == pytest.approx(world * dense / 0.25e-3 / 1e12)
    # roofline of the dominant kernel (the capture here: 1.5 ms)
    roof = line["roofline"]
    assert set(("bound", "achieved", "peak", "unit", "frac", "traffic")) <= set(roof)
    assert roof["kernel"] == "rt_attn_full_capture" and roof["bound"] == "tensor"
    assert roof["unit"] == "TFLOP/s" and roof["peak"] == peaks["bf16_tflops"]
    assert roof["achieved"] == pytest.approx(dense / 1.5e-3 / 1e12)
    assert roof["frac"] == pytest.approx(roof["achieved"] / roof["peak"])
    # executed flops of the sparse step: every query row against keep*64 keys
    assert r["nums"]["executed_flops"] == 4.0 * 64 * 2 * 512 * (r["keep"] * 64)
    assert line["executed_tflops"] == pytest.approx(r["nums"]["executed_flops"] / 0.25e-3 / 1e12)
    e2e = line["e2e"]
    assert e2e["unit"] == bench.UNIT
    assert e2e["value"] == pytest.approx(world * dense / 0.4e-3 / 1e12)
    assert e2e["h2d_bytes_per_step"] > 0 and e2e["d2h_bytes_per_step"] > 0
    assert line["gpu_launches"] == bench.LAUNCHES_PER_STEP * 5
    assert set(("sm_mhz", "sm_max_mhz", "reasons")) <= set(line["clocks"])
    if world == 1:
        cb = line["cpu_baseline"]
        assert cb["kind"] == "oracle" and cb["cores"] >= 1 and cb["sample"] and cb["unit"] == bench.UNIT
    else:
        assert line["cpu_baseline"] is None


def line_full_step(r):
    return bench.build_line(_Args, r, 1, dict(bench.FALLBACK_PEAKS), "fallback", None, None)["full_step_ms"]


def test_key_tiles_per_query_tile_counts_the_union():
    # 2 heads x 4 query blocks (block 64, N = 256): head 0 rows {0,1},{0,2},{0,1},{0,2}; head 1 all {3}
    rp = np.arange(9, dtype=np.int64) * 2
    ci = np.array([0, 1, 0, 2, 0, 1, 0, 2] + [3, 3] * 4)
    ci[9::2] = 3
    # neighbours: head 0 tiles {0,1,2} {0,1,2} -> 3, 3; head 1 {3} -> 1, 1
    assert bench.key_tiles_per_query_tile(rp, ci, None, 4, 64, 2, 256) == pytest.approx((3 + 3 + 1 + 1) / 4)
    tiles = np.array([[[0, 2], [1, 3]], [[0, 1], [2, 3]]])
    # paired: head 0 {0,1} {0,2} -> 2, 2
    assert bench.key_tiles_per_query_tile(rp, ci, tiles, 4, 64, 2, 256) == pytest.approx((2 + 2 + 1 + 1) / 4)


def test_roofline_follows_the_dominant_kernel():
    r = _measurement(1)
    r["capture_ms"], r["sparse_ms"] = 0.1, 0.5
    assert line_full_step(r) == pytest.approx(0.05 + 0.01 + 0.1)
    line = bench.build_line(_Args, r, 1, dict(bench.FALLBACK_PEAKS), "fallback", None, None)
    roof = line["roofline"]
    assert roof["kernel"] == "rt_attn_sparse_reshape"
    assert roof["achieved"] == pytest.approx(line["executed_tflops"])
    r["mask_ms"] = 1.0
    line = bench.build_line(_Args, r, 1, dict(bench.FALLBACK_PEAKS), "fallback", None, None)
    roof = line["roofline"]
    assert roof["kernel"] == "rt_build_block_mask" and roof["bound"] == "hbm" and roof["unit"] == "GB/s"
    assert roof["frac"] == pytest.approx(roof["achieved"] / bench.FALLBACK_PEAKS["hbm_gbs"])


def test_reference_line_has_the_contract_keys():
    class A:
        workload, keep, heads, cpu_rows, warmup, steps, gpus = "tiny", None, None, 32, 0, 1, 1
    line = bench.run_reference(A, 0, 1)
    for k in TOP_KEYS:
        assert k in line, k
    assert line["impl"] == "reference" and line["dtype"] == "f64" and line["value"] > 0
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1 and cb["sample"]
    assert line["e2e"] == {"value": line["value"], "unit": line["unit"], "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    assert bench.run_reference(A, 1, 2) is None


def test_sparse_roofline_and_page_claims():
    r = _measurement(1)
    peaks = dict(bench.FALLBACK_PEAKS)
    line = bench.build_line(_Args, r, 1, peaks, "fallback", None, None)
    rs = line["roofline_sparse"]
    assert rs["kernel"] == "rt_attn_sparse_reshape" and rs["bound"] == "tensor" and rs["unit"] == "TFLOP/s"
    assert rs["achieved"] == pytest.approx(r["nums"]["executed_flops"] / 0.25e-3 / 1e12)
    assert rs["frac"] == pytest.approx(rs["achieved"] / peaks["bf16_tflops"])
    assert rs["hbm_frac"] == pytest.approx(r["nums"]["sparse_bytes"] / 0.25e-3 / 1e9 / peaks["hbm_gbs"])
    claims = line["pages_claims"]
    assert len(claims) == 2 and all(c["hardware"] == "not stated" and c["source"] for c in claims)
    assert "3.1%" in claims[0]["claim"] and "95%" in claims[1]["claim"]


def test_oracle_checker_on_oracle_outputs():
    """The checker's error figures are those of bf16-rounded oracle outputs: within the
    tolerances, with no mask row differing when it is given the oracle's own CSR."""
    import torch

    import oracle
    w = bench.WORKLOADS["tiny"]
    steps = list(bench.denoising_inputs(w, 2))
    h0, h1 = steps[0][1:], steps[1][1:]
    keep = w.keep_blocks()
    d, bs, D, N = w.head_dim, w.block_size, w.head_dim_padded, w.seq_len
    rp, ci = oracle.build_block_mask(h0[0], h0[1], d, bs, w.scale, keep, 0)
    cap = oracle.full_capture(*h0, d, bs, w.scale, rp, ci)
    sp = oracle.sparse_reshape(*h1, d, bs, w.scale, rp, ci, cap)
    B, H = w.batch, w.heads

    def as_out(x):
        t = torch.zeros(B * H * N, D)
        t[:, :d] = torch.as_tensor(x, dtype=torch.float32)
        return t.to(torch.bfloat16).reshape(B, H, N, D)

    u = torch.zeros(B * H * N, D)
    u[:, :d] = torch.as_tensor(cap["u"], dtype=torch.float32)
    st = bench.OracleChecker  # the checker only reads .m .zfull .zkept .u
    stats = type("S", (), {"m": torch.as_tensor(cap["m"], dtype=torch.float32),
                           "zfull": torch.as_tensor(cap["zfull"], dtype=torch.float32),
                           "zkept": torch.as_tensor(cap["zkept"], dtype=torch.float32), "u": u})()
    res = st(rows=32).check(w, keep, h0, h1, rp, ci, as_out(cap["o"]), stats, as_out(sp))
    assert res["rows"] == 32 and res["mask_rows_differing"] == 0
    for k in ("capture_o", "sparse_o"):
        assert res[k]["max_abs_unit_scale"] <= 2 ** -8 and res[k]["mean_abs"] <= 1.5e-3
    assert res["capture_stats"]["ratio_rel"] < 1e-6 and res["capture_stats"]["u_err_over_bound"] < 0.01
