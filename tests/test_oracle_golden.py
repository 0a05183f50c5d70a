"""The oracle on hand-worked examples (tests/golden/worked_examples.json).

The examples are small enough to check on paper; their values follow from the
definitions alone (uniform scores make every exponential 1; block scores that
are exact binary fractions make the selection's ties and forced prefix
decidable by inspection), so they pin the oracle to something other than
itself.
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))
with open(os.path.join(HERE, "golden", "worked_examples.json")) as f:
    EXAMPLES = {e["name"]: e for e in json.load(f)["examples"]}


def _t(rows, shape):
    return torch.tensor(rows, dtype=torch.float32).reshape(shape["B"], shape["H"], shape["N"], shape["D"]).to(
        torch.bfloat16)


def test_uniform_scores_cycle():
    e = EXAMPLES["uniform_scores_cycle"]
    s, x = e["shape"], e["expect"]
    q, k, v = _t(e["q"], s), _t(e["k"], s), _t(e["v"], s)
    rp, ci = oracle.build_block_mask(q, k, s["d"], s["block"], s["scale"], s["keep"], s["forced_tokens"])
    assert rp.tolist() == x["row_ptr"] and ci.tolist() == x["col_idx"]
    st = oracle.full_capture(q, k, v, s["d"], s["block"], s["scale"], rp, ci)
    n = s["N"]
    np.testing.assert_allclose(st["o"], np.tile(x["capture_o"], (n, 1)), rtol=0, atol=1e-12)
    np.testing.assert_allclose(st["m"], np.full(n, x["m"]), rtol=0, atol=1e-12)
    np.testing.assert_allclose(st["zfull"], np.full(n, x["zfull"]), rtol=1e-14)
    np.testing.assert_allclose(st["zkept"], np.full(n, x["zkept"]), rtol=1e-14)
    np.testing.assert_allclose(st["u"], np.tile(x["u"], (n, 1)), rtol=1e-14)
    q1, v1 = _t(e["q_next"], s), _t(e["v_next"], s)
    o = oracle.sparse_reshape(q1, k, v1, s["d"], s["block"], s["scale"], rp, ci, st)
    np.testing.assert_allclose(o, np.tile(x["sparse_o"], (n, 1)), rtol=1e-14)
    o_plain = oracle.sparse_reshape(q1, k, v1, s["d"], s["block"], s["scale"], rp, ci, None)
    np.testing.assert_allclose(o_plain, np.tile(x["plain_o"], (n, 1)), rtol=1e-14)


def test_selection_ties_and_prefix():
    e = EXAMPLES["selection_ties_and_prefix"]
    s, x = e["shape"], e["expect"]
    q, k = _t(e["q"], s), _t(e["k"], s)
    sc = oracle.block_scores(oracle.pool_blocks(q, s["d"], s["block"]), oracle.pool_blocks(k, s["d"], s["block"]),
                             s["scale"])
    np.testing.assert_array_equal(sc.reshape(4, 4), np.array(x["scores"], dtype=np.float64))
    for key, keep in (("keep2", 2), ("keep3", 3)):
        rp, ci = oracle.build_block_mask(q, k, s["d"], s["block"], s["scale"], keep, x[key]["forced_tokens"])
        assert rp.tolist() == [r * keep for r in range(5)]
        assert ci.tolist() == x[key]["col_idx"], key
