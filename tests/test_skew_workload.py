"""The skewed-routing workload's inputs (CPU): the stored router bias and the
near-tied LM-head rows.

The workload asks for 4 hot experts holding about half of the top-6 slots and
5% of the rows with near-tied top-2 LM logits.  The bias is stored (the
workload table and tests/golden/skew_router_bias.json) so that the benchmark
builds the inputs without the oracle; these tests tie the stored value to a
fresh bisection on the oracle's router, and check the tie construction.
"""
import json
import os
import sys

import numpy as np

import oracle
from moe_decoder_speculative_b200 import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
sys.path.insert(0, GOLDEN)
import make_skew_router_bias  # noqa: E402


def test_stored_bias_matches_the_golden_file_and_a_fresh_bisection():
    rec = json.load(open(os.path.join(GOLDEN, "skew_router_bias.json")))
    w = wl.workload(4)
    assert w.hot_bias == rec["beta"]
    beta, share = make_skew_router_bias.bisect_beta(w.hot_share)
    assert beta == rec["beta"]
    assert abs(share - w.hot_share) <= 0.0025


def test_inputs_carry_the_bias_and_it_gives_the_hot_share():
    w = wl.workload(4)
    inp = wl.make_inputs(w)
    hot = wl.hot_experts(w)
    b = inp["layers"][0]["router_bias"]
    assert b.dtype == np.float32 and b.shape == (w.E,)
    assert np.all(b[hot] == np.float32(w.hot_bias)) and np.count_nonzero(b) == w.n_hot
    idx, _, _, _ = oracle.router(inp["hidden"], inp["layers"][0]["w_router"], w.k, bias=b)
    assert abs(np.isin(idx, hot).mean() - w.hot_share) <= 0.0025
    # without the bias the hot experts hold about their uniform share, 4/64 of the slots
    idx0, _, _, _ = oracle.router(inp["hidden"], inp["layers"][0]["w_router"], w.k)
    assert np.isin(idx0, hot).mean() < 0.1


def test_tied_lm_rows_copy_the_chosen_row_or_move_one_element():
    w = wl.workload(4)
    rng = np.random.default_rng(3)
    V, H = w.V, w.H
    w_lm = wl.f32_to_bf16_bits(rng.standard_normal((V, H)).astype(np.float32) * 0.02)
    am = rng.integers(0, V, size=w.T).astype(np.int32)
    w2, rows, v2s = wl.make_tied_lm_head(w, w_lm, am)
    assert len(rows) == round(w.tie_frac * w.T) and len(set(rows.tolist())) == len(rows)
    assert not np.isin(v2s, am).any()                      # v2 is a token no row chose
    changed = np.flatnonzero(np.any(w2 != w_lm, axis=1))
    assert set(changed.tolist()) == set(v2s.tolist())      # only the v2 rows change
    for i, (r, v2) in enumerate(zip(rows, v2s)):
        diff = np.flatnonzero(w2[v2] != w_lm[am[r]])
        if i % 2 == 0:
            assert diff.size == 0                          # an exact copy: an exact tie
        else:
            assert diff.size == 1
            step = int(w2[v2, diff[0]]) - int(w_lm[am[r], diff[0]])
            assert 1 <= abs(step) <= 4                     # 1-4 bf16 codes away
