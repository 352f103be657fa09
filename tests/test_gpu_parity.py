"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the
same seeded inputs.

Exact for indices, accepted lengths and tokens (except rows the flag rules
excuse, which are counted); MoE outputs within max-abs 2e-2 x RMS of the
oracle's.  Sizes run from the tiny workload through the full model shape.
"""
import numpy as np
import pytest
import torch

import oracle
from moe_decoder_speculative_b200 import binding as bd
from moe_decoder_speculative_b200 import workloads as wl
from parity_helpers import (GATE_GAP, LM_GAP, MOE_TOL, drift_excused, gate_flags, moe_error, reference,
                             row_flags)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from moe_decoder_speculative_b200 import build
    build.build()


def same_routing(idx_a, idx_b):
    """Rows whose selected expert SETS agree (slot order among near-equal selected
    logits is not a routing decision)."""
    return np.all(np.sort(idx_a, axis=1) == np.sort(idx_b, axis=1), axis=1)


def dev_layers(inp):
    return [bd.LayerWeights(l) for l in inp["layers"]]


def to_np(t):
    return t.cpu().numpy()


# ---------------------------------------------------------------------------
# per kernel
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("wid", [0, 1, 4])
def test_router_topk(wid):
    w, inp, st = reference(wid)
    shape = bd.shape_of(w)
    x = bd.bf16_to_device(inp["hidden"])
    lw = bd.LayerWeights(inp["layers"][0])
    idx, tw = bd.moe_router_topk(x, shape, lw.t["w_router"], lw.t["router_bias"])
    torch.cuda.synchronize()
    idx, tw = to_np(idx), to_np(tw)
    ref = st["layers"][0]
    ok = ref["gap"] >= GATE_GAP
    assert same_routing(idx, ref["idx"])[ok].all()
    same = np.all(idx == ref["idx"], axis=1)
    assert same.mean() > 0.9
    np.testing.assert_allclose(tw[same], ref["w"][same], rtol=2e-5, atol=2e-6)
    assert np.all(np.abs(tw.sum(1) - 1) < 1e-5)


@pytest.mark.parametrize("T,bias", [(1500, False), (2049, True)])
def test_router_topk_large_batch(T, bias):
    """Batches above 1024 rows route on the tensor cores (top-k in the epilogue)."""
    rng = np.random.default_rng(T)
    H, E, k = 1280, 64, 6
    x = wl.f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    wr = wl.f32_to_bf16_bits(rng.standard_normal((E, H)).astype(np.float32) * 0.02)
    b = rng.standard_normal(E).astype(np.float32) * 0.5 if bias else None
    idx_ref, w_ref, _, gap = oracle.router(x, wr, k, bias=b)
    shape = bd.MoeShape(H, E, 896, 0, k)
    idx, tw = bd.moe_router_topk(bd.bf16_to_device(x), shape, bd.bf16_to_device(wr),
                                 None if b is None else torch.from_numpy(b).cuda())
    idx, tw = to_np(idx), to_np(tw)
    ok = gap >= GATE_GAP
    assert same_routing(idx, idx_ref)[ok].all()
    same = np.all(idx == idx_ref, axis=1)
    assert same.mean() > 0.95
    np.testing.assert_allclose(tw[same], w_ref[same], rtol=2e-5, atol=2e-6)


def _router_case(T, seed):
    rng = np.random.default_rng(seed)
    H, E, k = 1280, 64, 6
    x = wl.f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    wr = wl.f32_to_bf16_bits(rng.standard_normal((E, H)).astype(np.float32) * 0.02)
    return x, wr, bd.MoeShape(H, E, 896, 0, k), k


@pytest.mark.parametrize("T", [4, 128, 700, 1500, 2049])
def test_router_rows_with_fewer_than_k_finite_logits(T):
    """Only 4 experts have finite logits (bias -inf elsewhere) under top-6: every
    row still gets 6 distinct experts, the 4 finite ones in descending order and
    then the -inf ones by id (0 and 1), with weight 0, as the oracle's stable
    ordering gives.  1 and 2 rows per routing CTA (T <= 512, T > 512), and the
    tensor-core router's epilogue top-k (T > 1024)."""
    x, wr, shape, k = _router_case(T, 100 + T)
    finite = np.array([5, 17, 40, 63])
    b = np.full(shape.E, -np.inf, np.float32)
    b[finite] = 0.0
    idx_ref, w_ref, _, _ = oracle.router(x, wr, k, bias=b)
    idx, tw = bd.moe_router_topk(bd.bf16_to_device(x), shape, bd.bf16_to_device(wr), torch.from_numpy(b).cuda())
    idx, tw = to_np(idx), to_np(tw)
    np.testing.assert_array_equal(idx_ref[:, 4:], np.tile([0, 1], (T, 1)))    # the oracle's own reading
    np.testing.assert_array_equal(idx[:, 4:], idx_ref[:, 4:])
    assert np.all(np.sort(idx[:, :4], axis=1) == finite)
    assert np.all(tw[:, 4:] == 0.0)
    same = np.all(idx == idx_ref, axis=1)
    assert same.mean() > 0.95
    np.testing.assert_allclose(tw[same], w_ref[same], rtol=2e-5, atol=2e-6)


@pytest.mark.parametrize("T", [128, 700, 1500, 2049])
def test_router_nan_logits_are_never_chosen_over_numbers(T):
    """A NaN logit (bias NaN on experts 0-9) ranks below every number: with 54
    numbers per row the routing equals the oracle's with those experts at -inf
    (CUDA-core routers up to 1024 rows, the tensor-core router beyond)."""
    x, wr, shape, k = _router_case(T, 200 + T)
    b = np.zeros(shape.E, np.float32)
    b[:10] = np.nan
    b_ref = b.copy()
    b_ref[:10] = -np.inf
    idx_ref, w_ref, _, gap = oracle.router(x, wr, k, bias=b_ref)
    idx, tw = bd.moe_router_topk(bd.bf16_to_device(x), shape, bd.bf16_to_device(wr), torch.from_numpy(b).cuda())
    idx, tw = to_np(idx), to_np(tw)
    assert idx.min() >= 10 and idx.max() < shape.E
    assert np.all(np.isfinite(tw))
    ok = gap >= GATE_GAP
    assert same_routing(idx, idx_ref)[ok].all()
    same = np.all(idx == idx_ref, axis=1)
    assert same.mean() > 0.95
    np.testing.assert_allclose(tw[same], w_ref[same], rtol=2e-5, atol=2e-6)


@pytest.mark.parametrize("T", [4, 700, 1500])
def test_router_rows_short_of_numbers_take_nan_experts_last(T):
    """Two finite logits, two -inf and sixty NaN per row under top-6: the slots
    hold the two numbers, then the -inf experts by id (30, 31), then the NaN
    experts by id (0, 1), as on the oracle; a NaN among the kept logits makes
    every weight of the row NaN on both sides (the renormalising sum is NaN).
    CUDA-core routers (4, 700 rows) and the tensor-core router (1,500 rows)."""
    x, wr, shape, k = _router_case(T, 300 + T)
    b = np.full(shape.E, np.nan, np.float32)
    b[[5, 17]] = 0.0
    b[[30, 31]] = -np.inf
    idx_ref, w_ref, _, _ = oracle.router(x, wr, k, bias=b)
    np.testing.assert_array_equal(idx_ref[:, 2:], np.tile([30, 31, 0, 1], (T, 1)))
    idx, tw = bd.moe_router_topk(bd.bf16_to_device(x), shape, bd.bf16_to_device(wr), torch.from_numpy(b).cuda())
    idx, tw = to_np(idx), to_np(tw)
    np.testing.assert_array_equal(idx[:, 2:], idx_ref[:, 2:])
    assert np.all(np.sort(idx[:, :2], axis=1) == [5, 17])
    assert np.all(np.isnan(tw)) and np.all(np.isnan(w_ref))


@pytest.mark.parametrize("T,E,k", [(16, 8, 2), (128, 64, 6), (37, 64, 6), (1, 8, 8), (1000, 256, 8)])
def test_expert_permute(T, E, k):
    rng = np.random.default_rng(T * 7 + E)
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    counts, offsets, perm, inv = bd.moe_expert_permute(torch.from_numpy(idx).cuda(), E)
    torch.cuda.synchronize()
    flat = idx.reshape(-1)
    want_perm = np.argsort(flat, kind="stable")
    np.testing.assert_array_equal(to_np(counts), np.bincount(flat, minlength=E))
    np.testing.assert_array_equal(to_np(offsets), np.concatenate([[0], np.cumsum(np.bincount(flat, minlength=E))]))
    np.testing.assert_array_equal(to_np(perm), want_perm)
    np.testing.assert_array_equal(to_np(perm)[to_np(inv)], np.arange(T * k))


@pytest.mark.parametrize("wid", [0, 1, 4])
def test_moe_ffn_teacher_forced(wid):
    """GPU MoE layer fed the oracle's input and routing, against the oracle's MoE output."""
    w, inp, st = reference(wid)
    shape = bd.shape_of(w)
    ref = st["layers"][0]
    lw = bd.LayerWeights(inp["layers"][0])
    x = bd.bf16_to_device(ref["h_in"])
    idx = torch.from_numpy(ref["idx"]).cuda()
    tw = torch.from_numpy(ref["w"]).cuda()
    out = bd.moe_ffn_forward(x, shape, lw, idx, tw)           # bf16(m)
    out_r = bd.moe_ffn_forward(x, shape, lw, idx, tw, residual=x)
    torch.cuda.synchronize()
    m_gpu = wl.bf16_bits_to_f32(bd.bf16_from_device(out))
    assert moe_error(m_gpu, ref["m"]) <= MOE_TOL
    h_gpu = wl.bf16_bits_to_f32(bd.bf16_from_device(out_r))
    h_ref = wl.bf16_bits_to_f32(st["h"] if len(st["layers"]) == 1 else st["layers"][1]["h_in"])
    assert np.max(np.abs(h_gpu - h_ref)) <= MOE_TOL * np.sqrt(np.mean(ref["m"].astype(np.float64) ** 2)) + \
        np.max(np.abs(h_ref)) * 2.0 ** -8


@pytest.mark.parametrize("wid", [0, 1, 4])
def test_lm_head_argmax(wid):
    w, inp, st = reference(wid)
    h = bd.bf16_to_device(st["h"])
    wlm = bd.bf16_to_device(inp["w_lm"])
    am = to_np(bd.lm_head_argmax(h, wlm))
    # the LM check alone: the oracle's own h, so only the LM gap excuses a row
    ok = st["lm_gap"] >= LM_GAP
    np.testing.assert_array_equal(am[ok], st["argmax"][ok])
    if "tie_rows" in inp:     # exact ties resolve to the lower index on both sides
        exact = st["lm_gap"] == 0
        np.testing.assert_array_equal(am[exact], st["argmax"][exact])


def test_lm_head_ragged_vocab_and_rows():
    """V not a multiple of the 128-row tile, T spanning a ragged N tile."""
    rng = np.random.default_rng(5)
    T, H, V = 150, 192, 1000
    h = wl.f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    wlm = wl.f32_to_bf16_bits(rng.standard_normal((V, H)).astype(np.float32) * 0.05)
    ref, _, gap = oracle.lm_head_argmax(h, wlm)
    am = to_np(bd.lm_head_argmax(bd.bf16_to_device(h), bd.bf16_to_device(wlm)))
    ok = gap >= LM_GAP
    np.testing.assert_array_equal(am[ok], ref[ok])


@pytest.mark.parametrize("T", [256, 300, 513])
def test_lm_head_pairs_ragged_vocab_and_rows(T):
    """From 256 rows the LM head runs on CTA pairs (256 tokens x 256
    vocabulary rows per unit): a vocabulary that is not a multiple of 256, a
    ragged last token tile, a reduction of 3 k-blocks (one stage half empty),
    and vocabulary rows 7 and 900 made equal to rows 3 and 500 so that exact
    ties occur and must go to the lower index."""
    rng = np.random.default_rng(50 + T)
    H, V = 192, 1000
    h = wl.f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    wlm = wl.f32_to_bf16_bits(rng.standard_normal((V, H)).astype(np.float32) * 0.05)
    wlm[7] = wlm[3]
    wlm[900] = wlm[500]
    h[:40] = wl.f32_to_bf16_bits(wl.bf16_bits_to_f32(wlm[3]) * 4.0)   # rows 3 and 7 lead, tied
    ref, _, gap = oracle.lm_head_argmax(h, wlm)
    am = to_np(bd.lm_head_argmax(bd.bf16_to_device(h), bd.bf16_to_device(wlm)))
    ok = gap >= LM_GAP
    assert ok.mean() > 0.5
    np.testing.assert_array_equal(am[ok], ref[ok])
    tied = gap == 0
    np.testing.assert_array_equal(am[tied], ref[tied])
    assert np.all(ref[:40] == 3) and np.all(am[:40] == 3)


def test_greedy_accept_exhaustive():
    rng = np.random.default_rng(6)
    for K in (0, 1, 3, 7):
        B, V = 4096, 3
        g = rng.integers(0, V, size=(B, K + 1)).astype(np.int32)
        d = rng.integers(-1, V + 1, size=(B, K)).astype(np.int32)   # includes out-of-range drafts
        acc, nxt, em = bd.greedy_accept(torch.from_numpy(g.reshape(-1)).cuda(),
                                        torch.from_numpy(d).cuda() if K else None, B, K)
        ra, rn, re = oracle.greedy_accept(g.reshape(-1), d, B, K)
        np.testing.assert_array_equal(to_np(acc), ra)
        np.testing.assert_array_equal(to_np(nxt), rn)
        np.testing.assert_array_equal(to_np(em), re)


# ---------------------------------------------------------------------------
# the whole verify step
# ---------------------------------------------------------------------------

def run_verify(w, inp, drafts):
    shape = bd.shape_of(w)
    layers = dev_layers(inp)
    plan = bd.VerifyPlan(shape, layers, bd.bf16_to_device(inp["w_lm"]), w.B, w.K)
    hidden = bd.bf16_to_device(inp["hidden"])
    d = torch.from_numpy(drafts).cuda()
    acc, nxt, em, am = plan(hidden, d)
    plan.sync_status()
    return plan, hidden, d, to_np(acc), to_np(nxt), to_np(em), to_np(am)


def check_verify(w, st, acc, nxt, em, am, exact_all=False):
    """Exact agreement of argmax, accepted lengths, next and emitted tokens
    with the oracle on every unflagged row (every sequence whose rows are all
    unflagged).  With exact_all, flagged rows must agree too: the tiny
    workload's absolute thresholds flag every row (its logits are ~1e-3 in
    size), so there the flags excuse nothing and all rows are compared."""
    flags = row_flags(st)
    ok = ~flags
    mism = am != st["argmax"]
    assert not np.any(mism & ok), f"{int(np.sum(mism & ok))} unflagged rows disagree"
    seq_ok = ok.reshape(w.B, w.K + 1).all(1)
    if exact_all:
        bad = np.flatnonzero(mism)
        assert bad.size == 0, (f"{bad.size} of {w.T} rows disagree with the oracle: rows {bad.tolist()}, "
                               f"LM gaps {st['lm_gap'][bad].tolist()}, gate gaps "
                               f"{[float(min(l['gap'][r] for l in st['layers'])) for r in bad]}")
        seq_ok = np.ones(w.B, bool)
    np.testing.assert_array_equal(acc[seq_ok], st["accepted"][seq_ok])
    np.testing.assert_array_equal(nxt[seq_ok], st["next_token"][seq_ok])
    np.testing.assert_array_equal(em[seq_ok], st["emitted"][seq_ok])
    assert np.all((acc >= 0) & (acc <= w.K))
    return {"flagged_rows": int(flags.sum()), "flagged_mismatch": int(np.sum(mism & flags)),
            "clean_seqs": int(seq_ok.sum())}


@pytest.mark.parametrize("wid", [0, 1, 4])
def test_verify_step(wid):
    w, inp, st = reference(wid)
    _, _, _, acc, nxt, em, am = run_verify(w, inp, st["drafts"])
    info = check_verify(w, st, acc, nxt, em, am, exact_all=(wid == 0))
    assert info["flagged_mismatch"] == 0 or wid != 0
    assert info["clean_seqs"] >= 0.5 * w.B


def gpu_layer_chain(w, inp, plan, hidden):
    """The GPU's own per-layer hidden states through the public per-step calls
    (bit-identical to verify_step's internals)."""
    shape = bd.shape_of(w)
    hs, idxs = [bd.bf16_from_device(hidden)], []
    h = hidden
    for lw in plan.layers:
        idx, tw = bd.moe_router_topk(h, shape, lw.t["w_router"], lw.t["router_bias"])
        h = bd.moe_ffn_forward(h, shape, lw, idx, tw, residual=h)
        idxs.append(to_np(idx))
        hs.append(bd.bf16_from_device(h))
    am = to_np(bd.lm_head_argmax(h, plan.w_lm))
    return hs, idxs, am


@pytest.mark.slow
def test_verify_step_conc32_12_layers():
    """The headline workload: 32 sequences x (K+1=4) rows through 12 layers.

    (1) Oracle-anchored: each GPU layer fed the oracle's h_l -- routing sets
        exact except rows with gate gap < 1e-3, MoE output within 2e-2 x RMS.
    (2) GPU-anchored: the oracle re-run on the GPU's own h_l at every layer --
        the GPU's routing exact except the oracle's flags on that input, the
        GPU's h_{l+1} within the MoE tolerance of bf16(h_l + m_oracle), the
        GPU's argmax exact except LM gap < 1e-2, acceptance exact.
    (3) Free-running end to end against the oracle's own 12-layer run: rows
        decided above the measured drift bound agree exactly (reported)."""
    w, inp, st = reference(2)
    plan, hidden, d, acc, nxt, em, am = run_verify(w, inp, st["drafts"])
    shape = bd.shape_of(w)
    # (1)
    for l, ref in enumerate(st["layers"]):
        x = bd.bf16_to_device(ref["h_in"])
        lw = plan.layers[l]
        idx, _ = bd.moe_router_topk(x, shape, lw.t["w_router"], lw.t["router_bias"])
        ok = ref["gap"] >= GATE_GAP
        assert same_routing(to_np(idx), ref["idx"])[ok].all(), f"layer {l} routing"
        out = bd.moe_ffn_forward(x, shape, lw, torch.from_numpy(ref["idx"]).cuda(), torch.from_numpy(ref["w"]).cuda())
        m_gpu = wl.bf16_bits_to_f32(bd.bf16_from_device(out))
        assert moe_error(m_gpu, ref["m"]) <= MOE_TOL, f"layer {l}"
    # (2)
    hs, idxs, am_chain = gpu_layer_chain(w, inp, plan, hidden)
    np.testing.assert_array_equal(am_chain, am)
    for l, lay in enumerate(inp["layers"]):
        o_idx, o_w, _, o_gap = oracle.router(hs[l], lay["w_router"], w.k, bias=lay.get("router_bias"))
        ok = o_gap >= GATE_GAP
        assert same_routing(idxs[l], o_idx)[ok].all(), f"GPU-anchored routing, layer {l}"
        o_m, _ = oracle.moe_ffn(hs[l], lay, o_idx, o_w)
        h_in = wl.bf16_bits_to_f32(hs[l]).astype(np.float64)
        dm = wl.bf16_bits_to_f32(hs[l + 1]) - h_in                       # GPU's m, seen through bf16(h + m)
        rows = same_routing(idxs[l], o_idx)
        ulp = np.abs(h_in + o_m) * 2.0 ** -8
        rms = np.sqrt(np.mean(o_m.astype(np.float64) ** 2))
        assert np.all((np.abs(dm - o_m) <= MOE_TOL * rms + ulp)[rows]), f"GPU-anchored MoE, layer {l}"
    o_am, _, o_lm_gap = oracle.lm_head_argmax(hs[-1], inp["w_lm"])
    ok = o_lm_gap >= LM_GAP
    np.testing.assert_array_equal(am[ok], o_am[ok])
    ra, rn, re = oracle.greedy_accept(am, st["drafts"], w.B, w.K)
    np.testing.assert_array_equal(acc, ra)
    np.testing.assert_array_equal(nxt, rn)
    np.testing.assert_array_equal(em, re)
    # (3)
    ex, _ = drift_excused(st, inp["w_lm"], [l["w_router"] for l in inp["layers"]], hs)
    ex |= row_flags(st)
    ok = ~ex
    for l, ref in enumerate(st["layers"]):
        assert same_routing(idxs[l], ref["idx"])[ok].all(), f"end-to-end routing, layer {l}"
    np.testing.assert_array_equal(am[ok], st["argmax"][ok])
    print(f"\nconc32: argmax agrees with the free-running oracle on {int(np.sum(am == st['argmax']))}/{w.T} rows; "
          f"{int(ok.sum())} rows decided above the drift bound, all agree")


def test_verify_step_equals_its_calls():
    """verify_step is bit-identical to router -> ffn (x L) -> lm_head_argmax -> accept."""
    w, inp, st = reference(0)
    plan, hidden, d, acc, nxt, em, am = run_verify(w, inp, st["drafts"])
    shape = bd.shape_of(w)
    h = hidden
    for lw in plan.layers:
        idx, tw = bd.moe_router_topk(h, shape, lw.t["w_router"], lw.t["router_bias"])
        h = bd.moe_ffn_forward(h, shape, lw, idx, tw, residual=h)
    am2 = bd.lm_head_argmax(h, plan.w_lm)
    a2, n2, e2 = bd.greedy_accept(am2, d, w.B, w.K)
    np.testing.assert_array_equal(to_np(am2), am)
    np.testing.assert_array_equal(to_np(a2), acc)
    np.testing.assert_array_equal(to_np(n2), nxt)
    np.testing.assert_array_equal(to_np(e2), em)


@pytest.mark.parametrize("wid", [0, 1, 4])
def test_k0_is_plain_greedy(wid):
    """Speculation off (K=0): every row is its own sequence and its next token
    is the verifier's argmax (plain greedy).  Each row's result is the
    oracle's for the same row of the workload's K>0 step (rows are
    independent), so the oracle's run of that step is the reference: exact on
    every row of the tiny workload, on every unflagged row of the others."""
    w, inp, st = reference(wid)
    B = w.T
    shape = bd.shape_of(w)
    plan = bd.VerifyPlan(shape, dev_layers(inp), bd.bf16_to_device(inp["w_lm"]), B, 0)
    acc, nxt, em, am = plan(bd.bf16_to_device(inp["hidden"]), None)
    plan.sync_status()
    acc, nxt, em, am = to_np(acc), to_np(nxt), to_np(em), to_np(am)
    ok = np.ones(B, bool) if wid == 0 else ~row_flags(st)
    assert ok.sum() >= 0.5 * B
    assert np.all(acc == 0)
    np.testing.assert_array_equal(nxt, am)
    np.testing.assert_array_equal(am[ok], st["argmax"][ok])
    np.testing.assert_array_equal(em[:, 0], nxt)


def test_batch_invariance_and_determinism():
    """A sequence's result does not depend on the other sequences in the batch,
    and repeated runs give identical bits."""
    w, inp, st = reference(1)
    wb = wl.workload(1)
    shape = bd.shape_of(wb)
    layers = dev_layers(inp)
    wlm = bd.bf16_to_device(inp["w_lm"])
    rng = np.random.default_rng(9)
    other = wl.f32_to_bf16_bits(rng.standard_normal((12, wb.H)).astype(np.float32))
    big = np.concatenate([other[:4], inp["hidden"], other[4:]])   # our sequence is number 1 of 4
    d_big = np.concatenate([rng.integers(0, wb.V, (1, 3)), st["drafts"], rng.integers(0, wb.V, (2, 3))]).astype(np.int32)
    p1 = bd.VerifyPlan(shape, layers, wlm, 1, 3)
    p4 = bd.VerifyPlan(shape, layers, wlm, 4, 3)
    r1 = [to_np(t).copy() for t in p1(bd.bf16_to_device(inp["hidden"]), torch.from_numpy(st["drafts"]).cuda())]
    r1b = [to_np(t).copy() for t in p1(bd.bf16_to_device(inp["hidden"]), torch.from_numpy(st["drafts"]).cuda())]
    r4 = [to_np(t).copy() for t in p4(bd.bf16_to_device(big), torch.from_numpy(d_big).cuda())]
    for a, b in zip(r1, r1b):
        np.testing.assert_array_equal(a, b)
    np.testing.assert_array_equal(r4[3][4:8], r1[3])       # argmax rows
    assert r4[0][1] == r1[0][0] and r4[1][1] == r1[1][0]


def test_skewed_routing_flag_path():
    """Four hot experts take about half the slots; about 5% of rows carry
    near-tied LM logits; everything unflagged is exact."""
    w, inp, st = reference(4)
    hot = wl.hot_experts(w)
    share = np.isin(st["layers"][0]["idx"], hot).mean()
    assert abs(share - 0.5) <= 0.01
    assert np.sum(st["lm_gap"] < LM_GAP) >= 0.04 * w.T
    _, _, _, acc, nxt, em, am = run_verify(w, inp, st["drafts"])
    check_verify(w, st, acc, nxt, em, am)


def test_prefill_layer_sampled_rows():
    """The 9,248-row prefill layer on the GPU; the oracle checks routing on every
    row and the MoE output on a sample of rows spread over the batch."""
    w = wl.workload(3)
    inp = wl.make_inputs(w)
    shape = bd.shape_of(w)
    x = inp["hidden"]
    lay = inp["layers"][0]
    idx_ref, w_ref, _, gap = oracle.router(x, lay["w_router"], w.k)
    lw = bd.LayerWeights(lay)
    xd = bd.bf16_to_device(x)
    idx, tw = bd.moe_router_topk(xd, shape, lw.t["w_router"], None)
    out = bd.moe_ffn_forward(xd, shape, lw, idx, tw)
    torch.cuda.synchronize()
    idx = to_np(idx)
    ok = gap >= GATE_GAP
    assert same_routing(idx, idx_ref)[ok].all()
    rows = np.unique(np.concatenate([np.arange(0, w.T, 37), [w.T - 1]]))
    rows = rows[np.all(idx[rows] == idx_ref[rows], axis=1)]
    m_ref, _ = oracle.moe_ffn(x[rows], lay, idx_ref[rows], w_ref[rows])
    m_gpu = wl.bf16_bits_to_f32(bd.bf16_from_device(out))[rows]
    assert moe_error(m_gpu, m_ref) <= MOE_TOL


def test_prefill_groups_of_every_size():
    """The prefill-sized grouped GEMM (CTA pairs, 256-token units) on 2,049
    rows whose routing is skewed by a router bias: experts with no rows, one
    row, a few rows, and several 256-token units, plus the ragged shared
    expert.  Teacher-forced (the oracle's routing given to both sides); the
    MoE output of a sample of rows spread over every group is within the
    tolerance."""
    rng = np.random.default_rng(77)
    T, H, E, k, I, Ish = 2049, 1280, 64, 6, 896, 1792
    w = wl.workload(3)
    lay = wl.make_layer(w, np.random.SeedSequence(77))
    x = wl.f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    bias = np.full(E, -30.0, np.float32)          # most experts unreachable
    bias[:8] = [4.0, 3.5, 3.0, 2.5, 2.0, 1.0, 0.0, -1.0]
    bias[8:14] = [-1.5, -2.0, -2.5, -3.0, -3.5, -4.0]   # 34, 4 and 0 rows: ragged and empty groups
    idx, tw, _, _ = oracle.router(x, lay["w_router"], k, bias=bias)
    counts = np.bincount(idx.reshape(-1), minlength=E)
    assert counts.max() > 512 and (counts == 0).any() and ((counts > 0) & (counts < 16)).any()
    shape = bd.MoeShape(H, E, I, Ish, k)
    lw = bd.LayerWeights(lay)
    out = bd.moe_ffn_forward(bd.bf16_to_device(x), shape, lw, torch.from_numpy(idx).cuda(), torch.from_numpy(tw).cuda())
    torch.cuda.synchronize()
    # rows of every touched expert, plus a stride over the batch and the last row
    rows = set(range(0, T, 41)) | {T - 1}
    for e in np.flatnonzero(counts):
        r_e = np.flatnonzero((idx == e).any(axis=1))
        rows |= {int(r_e[0]), int(r_e[-1])}
    rows = np.array(sorted(rows))
    m_ref, _ = oracle.moe_ffn(x[rows], lay, idx[rows], tw[rows])
    m_gpu = wl.bf16_bits_to_f32(bd.bf16_from_device(out))[rows]
    assert moe_error(m_gpu, m_ref) <= MOE_TOL


def _biased_reference(wid, layers, dead):
    """Oracle reference of a workload whose router bias is -30 on the `dead`
    experts in every layer, so that no row chooses them."""
    w = wl.workload(wid)
    inp = wl.make_inputs(w, layers)
    for lay in inp["layers"]:
        b = np.zeros(w.E, np.float32) if lay.get("router_bias") is None else lay["router_bias"].copy()
        b[dead] = -30.0
        lay["router_bias"] = b
    st = oracle.moe_stack(inp["hidden"], inp["layers"], w.k, keep=True)
    am, _, lm_gap = oracle.lm_head_argmax(st["h"], inp["w_lm"])
    drafts = wl.make_drafts(w, am)
    acc, nxt, em = oracle.greedy_accept(am, drafts, w.B, w.K)
    st.update(argmax=am, lm_gap=lm_gap, drafts=drafts, accepted=acc, next_token=nxt, emitted=em)
    for lay in st["layers"]:
        assert not np.isin(lay["idx"], dead).any()
    return w, inp, st


def test_verify_step_with_experts_no_row_chooses_tiny():
    """Tiny workload (16 rows, top-2 of 8 experts) with experts 0 and 5 chosen
    by no row: their groups are empty in every layer (no units, no outputs
    read by the combine).  Every row equals the oracle."""
    w, inp, st = _biased_reference(0, None, [0, 5])
    _, _, _, acc, nxt, em, am = run_verify(w, inp, st["drafts"])
    check_verify(w, st, acc, nxt, em, am, exact_all=True)


def test_verify_step_with_experts_no_row_chooses_conc32():
    """The concurrency-32 batch (128 rows, top-6 of 64) through 2 layers with
    experts 3, 17, 40 and 63 chosen by no row (empty slabs in both layers, the
    second layer's routing fused with the first layer's combine).  Unflagged
    rows equal the oracle, and the step's argmax equals the public per-layer
    calls' (router, grouped FFN, LM head) bit for bit."""
    w, inp, st = _biased_reference(2, 2, [3, 17, 40, 63])
    plan, hidden, d, acc, nxt, em, am = run_verify(w, inp, st["drafts"])
    check_verify(w, st, acc, nxt, em, am)
    _, _, am_chain = gpu_layer_chain(w, inp, plan, hidden)
    np.testing.assert_array_equal(am_chain, am)


def test_verify_step_two_layers_equals_the_per_layer_calls():
    """Concurrency-32 batch, 2 layers, no bias: the step (slab grouping inside
    the fused combine-route kernel) and the public per-layer calls give the
    same argmax bit for bit, and unflagged rows equal the oracle."""
    w, inp, st = reference(2, 2)
    plan, hidden, d, acc, nxt, em, am = run_verify(w, inp, st["drafts"])
    check_verify(w, st, acc, nxt, em, am)
    _, _, am_chain = gpu_layer_chain(w, inp, plan, hidden)
    np.testing.assert_array_equal(am_chain, am)
