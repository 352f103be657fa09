"""GPU parity of the pre-RMSNorm layer variant (mv_moe_weights.norm_gain)
against the oracle.

RMSNorm's sum of squares is reduced in another order on the GPU, so a
normalised bf16 element may differ by one unit in the last place; routing and
argmax decisions are therefore compared exactly except where the oracle's
gate gap (< 1e-3) or LM gap (< 1e-2) flags them, and the MoE output within
2e-2 x RMS, as for the plain layer.
"""
import numpy as np
import pytest
import torch

import oracle
from moe_decoder_speculative_b200 import binding as bd
from moe_decoder_speculative_b200 import workloads as wl

pytestmark = pytest.mark.gpu

GATE_GAP, LM_GAP, MOE_TOL = 1e-3, 1e-2, 2e-2


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from moe_decoder_speculative_b200 import build
    build.build()


def _np(t):
    return t.cpu().numpy()


def test_rmsnorm_matches_the_oracle_within_one_unit():
    rng = np.random.default_rng(1)
    for T, H in [(1, 1280), (128, 1280), (37, 128)]:
        x = wl.normal_bf16(np.random.SeedSequence([T, H]), (T, H), 1.5)
        g = wl.f32_to_bf16_bits(1.0 + 0.1 * rng.standard_normal(H).astype(np.float32))
        ref = wl.bf16_bits_to_f32(oracle.rmsnorm(x, g))
        got = wl.bf16_bits_to_f32(bd.bf16_from_device(bd.moe_rmsnorm(bd.bf16_to_device(x), bd.bf16_to_device(g))))
        torch.cuda.synchronize()
        assert np.all(np.abs(got - ref) <= np.abs(ref) * 2.0 ** -7)
        assert np.mean(got == ref) > 0.99


def _layers(wid, layers, norm=True):
    w = wl.workload(wid)
    inp = wl.make_inputs(w, layers=layers, norm=norm)
    return w, inp


def test_public_calls_compose_the_norm_layer_teacher_forced():
    """xn = moe_rmsnorm(h); route xn; moe_ffn_forward(xn, residual = h), per
    layer on the oracle's own h_l: routing sets and MoE output match."""
    w, inp = _layers(2, 2)
    st = oracle.moe_stack(inp["hidden"], inp["layers"], w.k, keep=True)
    shape = bd.shape_of(w)
    for l, ref in enumerate(st["layers"]):
        lw = bd.LayerWeights(inp["layers"][l])
        h = bd.bf16_to_device(ref["h_in"])
        xn = bd.moe_rmsnorm(h, lw.t["norm_gain"])
        idx, tw = bd.moe_router_topk(xn, shape, lw.t["w_router"], lw.t["router_bias"])
        ws = bd.workspace(bd.moe_ffn_workspace_size(w.T, shape))
        out = bd.moe_ffn_forward(xn, shape, lw, idx, tw, residual=h, ws=ws)
        bd.sync_status(ws)
        idx = _np(idx)
        clear = ref["gap"] >= GATE_GAP
        assert clear.mean() > 0.5
        for r in np.nonzero(clear)[0]:
            assert set(idx[r]) == set(ref["idx"][r]), (l, r)
        # the layer output on rows routed alike, against the oracle's h_{l+1}:
        # the MoE tolerance plus one bf16 unit of the rounded sum
        nxt = st["layers"][l + 1]["h_in"] if l + 1 < len(st["layers"]) else st["h"]
        ref_next = wl.bf16_bits_to_f32(nxt)
        got_next = wl.bf16_bits_to_f32(bd.bf16_from_device(out))
        rms = float(np.sqrt(np.mean(ref["m"].astype(np.float64) ** 2)))
        rows = np.nonzero(clear)[0]
        bound = MOE_TOL * rms + np.abs(ref_next[rows]) * 2.0 ** -7
        assert np.all(np.abs(got_next[rows] - ref_next[rows]) <= bound), l


@pytest.mark.parametrize("wid,layers,B,K", [(0, None, None, None), (2, 2, None, None), (4, None, None, None),
                                             (0, None, 300, 3)])
def test_verify_step_with_norm_layers(wid, layers, B, K):
    """The slab path (0, 2), the fused path without slabs (4: 512 rows) and the
    unfused path above 1,024 rows (300 x 4 rows of the small shape)."""
    import dataclasses
    w = wl.workload(wid)
    if B is not None:
        w = dataclasses.replace(w, B=B, K=K)
    inp = wl.make_inputs(w, layers=layers, norm=True)
    shape = bd.shape_of(w)
    lws = [bd.LayerWeights(l) for l in inp["layers"]]
    w_lm = bd.bf16_to_device(inp["w_lm"])
    hid = bd.bf16_to_device(inp["hidden"])
    plan = bd.VerifyPlan(shape, lws, w_lm, w.B, w.K)
    _, _, _, am0 = plan(hid, torch.zeros((w.B, max(1, w.K)), dtype=torch.int32, device="cuda"))
    drafts = wl.make_drafts(w, _np(am0))
    acc, nxt, em, am = [_np(t).copy() for t in plan(hid, torch.from_numpy(drafts).cuda())]
    plan.sync_status()
    st = oracle.verify_step(inp["hidden"], drafts, w.B, w.K, inp["layers"], w.k, inp["w_lm"])
    flag = st["lm_gap"] < LM_GAP
    for rec in st["layers"]:
        flag |= rec["gap"] < GATE_GAP
    clean = ~flag
    np.testing.assert_array_equal(am[clean], st["argmax"][clean])
    # acceptance is exact given the GPU's own argmax
    a2, n2, e2 = oracle.greedy_accept(am, drafts, w.B, w.K)
    np.testing.assert_array_equal(acc, a2)
    np.testing.assert_array_equal(nxt, n2)
    if w.V > 100000:
        assert clean.mean() > 0.5
