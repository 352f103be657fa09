"""Failure detection on the GPU without faulting it: every device-side wait of
the library is bounded.  A 1 ns bound makes the waits of a MoE layer run out
(no copy lands that fast); the kernels give up, drain their own copies and
MMAs, free TMEM, exit, and the sticky error word reports MV_ERR_TIMEOUT.  The
context stays usable: with the default bound restored the same call gives the
oracle's result again."""
import numpy as np
import pytest
import torch

from moe_decoder_speculative_b200 import binding as bd
from moe_decoder_speculative_b200 import workloads as wl
from parity_helpers import MOE_TOL, moe_error, reference

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from moe_decoder_speculative_b200 import build
    build.build()


def test_wait_bound_runs_out_and_context_survives():
    w, inp, st = reference(1)
    shape = bd.shape_of(w)
    ref = st["layers"][0]
    lw = bd.LayerWeights(inp["layers"][0])
    x = bd.bf16_to_device(ref["h_in"])
    idx = torch.from_numpy(ref["idx"]).cuda()
    tw = torch.from_numpy(ref["w"]).cuda()
    ws = bd.workspace(bd.moe_ffn_workspace_size(w.T, shape))
    try:
        bd.set_wait_timeout_ns(1)
        bd.moe_ffn_forward(x, shape, lw, idx, tw, ws=ws)
        with pytest.raises(bd.MVError) as exc:
            bd.sync_status(ws)
        assert exc.value.status == 6  # MV_ERR_TIMEOUT
    finally:
        bd.set_wait_timeout_ns(0)   # back to the default bound
    bd.sync_status(ws)              # the word was cleared when it was read
    out = bd.moe_ffn_forward(x, shape, lw, idx, tw, ws=ws)
    bd.sync_status(ws)
    m_gpu = wl.bf16_bits_to_f32(bd.bf16_from_device(out))
    assert moe_error(m_gpu, ref["m"]) <= MOE_TOL


def test_out_of_range_expert_ids_are_reported():
    """Caller-supplied routing with an expert id outside [0, E) is skipped and
    reported as MV_ERR_INTERNAL instead of being read out of bounds."""
    w, inp, st = reference(0)
    shape = bd.shape_of(w)
    ref = st["layers"][0]
    lw = bd.LayerWeights(inp["layers"][0])
    idx = ref["idx"].copy()
    idx[3, 1] = w.E + 5
    ws = bd.workspace(bd.moe_ffn_workspace_size(w.T, shape))
    bd.moe_ffn_forward(bd.bf16_to_device(ref["h_in"]), shape, lw, torch.from_numpy(idx).cuda(),
                       torch.from_numpy(ref["w"]).cuda(), ws=ws)
    with pytest.raises(bd.MVError) as exc:
        bd.sync_status(ws)
    assert exc.value.status == 7  # MV_ERR_INTERNAL
    bd.sync_status(ws)


def test_wait_bound_runs_out_in_the_verify_step_and_context_survives():
    """The whole verify step with a 1 ns bound: the waits of its routing, GEMM
    and LM-head launches run out; the kernels drain their copies, exit and the
    step reports MV_ERR_TIMEOUT.  With the default bound restored the same
    step gives the same tokens as before."""
    w, inp, st = reference(0)
    shape = bd.shape_of(w)
    plan = bd.VerifyPlan(shape, [bd.LayerWeights(l) for l in inp["layers"]], bd.bf16_to_device(inp["w_lm"]),
                         w.B, w.K)
    hidden = bd.bf16_to_device(inp["hidden"])
    d = torch.from_numpy(st["drafts"]).cuda()
    good = [t.cpu().numpy().copy() for t in plan(hidden, d)]
    plan.sync_status()
    try:
        bd.set_wait_timeout_ns(1)
        plan(hidden, d)
        with pytest.raises(bd.MVError) as exc:
            plan.sync_status()
        assert exc.value.status == 6  # MV_ERR_TIMEOUT
    finally:
        bd.set_wait_timeout_ns(0)
    plan.sync_status()
    again = [t.cpu().numpy() for t in plan(hidden, d)]
    plan.sync_status()
    for a, b in zip(good, again):
        np.testing.assert_array_equal(a, b)
