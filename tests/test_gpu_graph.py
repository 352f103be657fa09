"""verify_graph_*: the verify step recorded once as a CUDA graph and replayed.

A replay must give exactly what verify_step gives on the same inputs (the
graph holds the same kernels with the same arguments; the scheduling
counters are cleared inside the graph), with new inputs written into the
fixed input buffers between replays.
"""
import numpy as np
import pytest
import torch

from moe_decoder_speculative_b200 import binding as bd
from moe_decoder_speculative_b200 import workloads as wl
from parity_helpers import reference, row_flags

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from moe_decoder_speculative_b200 import build
    build.build()


def _setup(wid, layers=None):
    w = wl.workload(wid)
    inp = wl.make_inputs(w, layers=layers)
    shape = bd.shape_of(w)
    lws = [bd.LayerWeights(l) for l in inp["layers"]]
    w_lm = bd.bf16_to_device(inp["w_lm"])
    return w, inp, shape, lws, w_lm


def _np(t):
    return t.cpu().numpy().copy()


@pytest.mark.parametrize("wid,layers", [(0, None), (1, None), (2, 2), (4, None)])
def test_graph_replays_equal_eager_steps(wid, layers):
    w, inp, shape, lws, w_lm = _setup(wid, layers)
    eager = bd.VerifyPlan(shape, lws, w_lm, w.B, w.K)
    gplan = bd.VerifyPlan(shape, lws, w_lm, w.B, w.K)
    hid_buf = torch.empty((w.T, w.H), dtype=torch.bfloat16, device="cuda")
    dr_buf = torch.empty((w.B, max(1, w.K)), dtype=torch.int32, device="cuda")
    g = bd.VerifyGraph(gplan, hid_buf, dr_buf)
    for step in range(3):
        hidden = bd.bf16_to_device(wl.normal_bf16(np.random.SeedSequence([wid, 100 + step]), (w.T, w.H), w.x_std))
        _, _, _, am0 = eager(hidden, torch.zeros((w.B, max(1, w.K)), dtype=torch.int32, device="cuda"))
        drafts = torch.from_numpy(wl.make_drafts(w, _np(am0), ss=np.random.SeedSequence([wid, step]))
                                  if w.K else np.zeros((w.B, 1), np.int32)).cuda()
        ref = [_np(t) for t in eager(hidden, drafts)]
        eager.sync_status()
        hid_buf.copy_(hidden)
        dr_buf.copy_(drafts)
        got = [_np(t) for t in g()]
        g.sync_status()
        for a, b in zip(got, ref):
            np.testing.assert_array_equal(a, b)
    g.close()


@pytest.mark.parametrize("wid", [0, 1, 4])
def test_graph_matches_the_oracle(wid):
    """Graph replays against the oracle's verify step: argmax, accepted
    lengths, next and emitted tokens exact on every row of the tiny workload
    (its absolute flag thresholds flag every row, so they excuse nothing
    there), and on every unflagged row / sequence of the others."""
    w, inp, st = reference(wid)
    shape = bd.shape_of(w)
    lws = [bd.LayerWeights(l) for l in inp["layers"]]
    plan = bd.VerifyPlan(shape, lws, bd.bf16_to_device(inp["w_lm"]), w.B, w.K)
    hid = bd.bf16_to_device(inp["hidden"])
    dr = torch.from_numpy(st["drafts"]).cuda()
    g = bd.VerifyGraph(plan, hid, dr)
    for _ in range(2):
        acc, nxt, em, am = [_np(t) for t in g()]
        g.sync_status()
        ok = np.ones(w.T, bool) if wid == 0 else ~row_flags(st)
        assert ok.sum() >= 0.5 * w.T
        np.testing.assert_array_equal(am[ok], st["argmax"][ok])
        seq_ok = ok.reshape(w.B, w.K + 1).all(1)
        np.testing.assert_array_equal(acc[seq_ok], st["accepted"][seq_ok])
        np.testing.assert_array_equal(nxt[seq_ok], st["next_token"][seq_ok])
        np.testing.assert_array_equal(em[seq_ok], st["emitted"][seq_ok])
        # acceptance is exact on every sequence given the GPU's own argmax
        import oracle
        a2, n2, e2 = oracle.greedy_accept(am, st["drafts"], w.B, w.K)
        np.testing.assert_array_equal(acc, a2)
        np.testing.assert_array_equal(nxt, n2)
        np.testing.assert_array_equal(em, e2)
    g.close()


def test_graph_kernel_count_and_launch_counter():
    w, inp, shape, lws, w_lm = _setup(1)
    plan = bd.VerifyPlan(shape, lws, w_lm, w.B, w.K)
    hid = bd.bf16_to_device(inp["hidden"])
    dr = torch.zeros((w.B, w.K), dtype=torch.int32, device="cuda")
    n0 = bd.launch_count()
    plan(hid, dr)
    eager_launches = bd.launch_count() - n0
    n1 = bd.launch_count()
    g = bd.VerifyGraph(plan, hid, dr)
    assert bd.launch_count() == n1          # recording runs nothing
    assert g.kernels == eager_launches
    g()
    g()
    assert bd.launch_count() - n1 == 2 * g.kernels
    g.sync_status()


def test_graph_with_k0_is_plain_greedy():
    w, inp, shape, lws, w_lm = _setup(0)
    B = 5
    plan = bd.VerifyPlan(shape, lws, w_lm, B, 0)
    hid = bd.bf16_to_device(inp["hidden"][:B])
    g = bd.VerifyGraph(plan, hid, None)
    acc, nxt, em, am = g()
    g.sync_status()
    assert np.all(_np(acc) == 0)
    np.testing.assert_array_equal(_np(nxt), _np(am))
    ref = _np(bd.lm_head_argmax(_chain(hid, shape, lws), w_lm))
    np.testing.assert_array_equal(_np(am), ref)


def _chain(h, shape, lws):
    for lw in lws:
        idx, tw = bd.moe_router_topk(h, shape, lw.t["w_router"], lw.t["router_bias"])
        h = bd.moe_ffn_forward(h, shape, lw, idx, tw, residual=h)
    return h


def test_graph_creation_is_refused_while_profiling():
    w, inp, shape, lws, w_lm = _setup(0)
    plan = bd.VerifyPlan(shape, lws, w_lm, w.B, w.K)
    hid = bd.bf16_to_device(inp["hidden"])
    dr = torch.zeros((w.B, w.K), dtype=torch.int32, device="cuda")
    bd.profile_enable(True)
    try:
        with pytest.raises(bd.MVError) as exc:
            bd.VerifyGraph(plan, hid, dr)
        assert exc.value.status == 1   # MV_ERR_INVALID_ARG
    finally:
        bd.profile_enable(False)
        bd.profile_collect()


def test_graph_creation_checks_arguments_like_verify_step():
    w, inp, shape, lws, w_lm = _setup(0)
    plan = bd.VerifyPlan(shape, lws, w_lm, w.B, w.K)
    hid = bd.bf16_to_device(inp["hidden"])
    with pytest.raises(bd.MVError) as exc:
        bd.VerifyGraph(plan, hid, None)   # K = 3 needs drafts
    assert exc.value.status == 1
    # the thread can still record and run a valid graph afterwards
    g = bd.VerifyGraph(plan, hid, torch.zeros((w.B, w.K), dtype=torch.int32, device="cuda"))
    g()
    g.sync_status()
