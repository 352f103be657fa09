"""GPU parity of the FastMTP draft block (fastmtp_draft) and of the
draft-and-verify loop step (speculative_step) against the oracle.

Drafts are integers decided by fp32 LM logits: they must equal the oracle's
exactly at every step up to the first step whose oracle top-2 gap is below
1e-2 (after a legitimately different choice the two recursions diverge).
Step outputs h_j are bf16-rounded states: where the fp32 value before
rounding differs in its last bits (another summation order), the rounded
value may differ by one bf16 unit in the last place, 2^-8 of its magnitude,
and a step's input carries the previous step's flips.  So h_j must match
within 2e-2 x RMS plus 2^-7 of each element's magnitude up to that step.
"""
import numpy as np
import pytest
import torch

import oracle
from moe_decoder_speculative_b200 import binding as bd
from moe_decoder_speculative_b200 import workloads as wl

pytestmark = pytest.mark.gpu

LM_GAP = 1e-2
H_TOL = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from moe_decoder_speculative_b200 import build
    build.build()


def _np(t):
    return t.cpu().numpy()


def bf(a):
    return wl.f32_to_bf16_bits(np.asarray(a, np.float32))


def check_drafts(gpu_drafts, gpu_steps, ref):
    """Exact drafts and close step outputs up to each row's first flagged step."""
    K, B = ref["gaps"].shape
    checked = 0
    for b in range(B):
        for j in range(K):
            hs_g = wl.bf16_bits_to_f32(gpu_steps[j, b]) if gpu_steps is not None else None
            hs_r = wl.bf16_bits_to_f32(ref["h_steps"][j, b])
            if hs_g is not None:
                rms = float(np.sqrt(np.mean(hs_r.astype(np.float64) ** 2)))
                assert np.all(np.abs(hs_g - hs_r) <= H_TOL * rms + np.abs(hs_r) * 2.0 ** -7), (b, j)
            if ref["gaps"][j, b] < LM_GAP:
                break
            assert gpu_drafts[b, j] == ref["drafts"][b, j], (b, j)
            checked += 1
    return checked


@pytest.mark.parametrize("wid,B,K", [(0, 4, 3), (0, 7, 1), (2, 32, 3), (2, 3, 5)])
def test_fastmtp_draft_matches_the_oracle(wid, B, K):
    w = wl.workload(wid)
    draft = wl.make_draft_block(w)
    w_lm_np = wl.make_lm_head(w)
    rng = np.random.default_rng(100 + wid)
    h0 = wl.normal_bf16(np.random.SeedSequence([wid, 7]), (B, w.H), w.x_std)
    t0 = rng.integers(0, w.V, B).astype(np.int32)
    ref = oracle.fastmtp_draft(h0, t0, K, draft, w_lm_np)
    dw = bd.DraftWeights(draft)
    w_lm = bd.bf16_to_device(w_lm_np)
    ws = bd.workspace(int(bd.lib().fastmtp_draft_workspace_size(B, K, w.H, dw.I_d, w.V)))
    drafts, steps = bd.fastmtp_draft(bd.bf16_to_device(h0), torch.from_numpy(t0).cuda(), K, dw, w_lm,
                                     keep_steps=True, ws=ws)
    bd.sync_status(ws)
    checked = check_drafts(_np(drafts), bd.bf16_from_device(steps).reshape(K, B, w.H), ref)
    assert checked >= 0.5 * B * K


def test_fastmtp_draft_walks_a_permutation_exactly():
    """The oracle pin's closed form on the GPU kernels: W_proj = [0 | P],
    identity embedding rows and LM head, zero FFN: drafts pi(t), pi^2(t), ..."""
    H = V = 64
    rng = np.random.default_rng(4)
    pi = rng.permutation(V)
    P = np.zeros((V, V), np.float32)
    P[pi, np.arange(V)] = 1.0
    draft = {"w_emb": bf(np.eye(V, H) * 0.37), "g_hidden": bf(np.ones(H)), "g_embed": bf(np.ones(H)),
             "w_proj": bf(np.concatenate([np.zeros((H, H)), P], axis=1)),
             "w_gate": bf(rng.standard_normal((64, H)) * 0.1), "w_up": bf(rng.standard_normal((64, H)) * 0.1),
             "w_down": bf(np.zeros((H, 64)))}
    B, K = 6, 4
    t0 = rng.integers(0, V, B).astype(np.int32)
    h0 = bf(rng.standard_normal((B, H)))
    drafts, steps = bd.fastmtp_draft(bd.bf16_to_device(h0), torch.from_numpy(t0).cuda(), K, bd.DraftWeights(draft),
                                     bd.bf16_to_device(bf(np.eye(V, H))), keep_steps=True)
    torch.cuda.synchronize()
    expect = np.zeros((B, K), np.int32)
    t = t0.copy()
    for j in range(K):
        t = pi[t]
        expect[:, j] = t
    np.testing.assert_array_equal(_np(drafts), expect)
    st = wl.bf16_bits_to_f32(bd.bf16_from_device(steps)).reshape(K, B, H)
    for j in range(K):
        np.testing.assert_array_equal(st[j], 8.0 * np.eye(V, H)[expect[:, j]])


def test_fastmtp_draft_reports_a_bad_first_token():
    w = wl.workload(0)
    dw = bd.DraftWeights(wl.make_draft_block(w))
    w_lm = bd.bf16_to_device(wl.make_lm_head(w))
    B, K = 3, 2
    h0 = bd.bf16_to_device(wl.normal_bf16(np.random.SeedSequence(5), (B, w.H), 1.0))
    ws = bd.workspace(int(bd.lib().fastmtp_draft_workspace_size(B, K, w.H, dw.I_d, w.V)))
    bd.fastmtp_draft(h0, torch.tensor([0, w.V + 3, 1], dtype=torch.int32, device="cuda"), K, dw, w_lm, ws=ws)
    with pytest.raises(bd.MVError) as exc:
        bd.sync_status(ws)
    assert exc.value.status == 7   # MV_ERR_INTERNAL
    bd.sync_status(ws)


def _chain(h, shape, lws):
    for lw in lws:
        idx, tw = bd.moe_router_topk(h, shape, lw.t["w_router"], lw.t["router_bias"])
        h = bd.moe_ffn_forward(h, shape, lw, idx, tw, residual=h)
    return h


@pytest.mark.parametrize("wid,layers", [(0, None), (2, 2)])
def test_speculative_step_equals_verify_then_draft(wid, layers):
    """speculative_step = verify_step, then fastmtp_draft from h_L at row
    b*(K+1) + accepted[b] and the next token (bit-identical, GPU vs GPU), and
    its drafts match the oracle's loop step up to near ties."""
    w = wl.workload(wid)
    inp = wl.make_inputs(w, layers=layers)
    shape = bd.shape_of(w)
    lws = [bd.LayerWeights(l) for l in inp["layers"]]
    w_lm = bd.bf16_to_device(inp["w_lm"])
    draft = wl.make_draft_block(w)
    dw = bd.DraftWeights(draft)
    hidden = bd.bf16_to_device(inp["hidden"])
    vplan = bd.VerifyPlan(shape, lws, w_lm, w.B, w.K)
    _, _, _, am0 = vplan(hidden, torch.zeros((w.B, w.K), dtype=torch.int32, device="cuda"))
    drafts = torch.from_numpy(wl.make_drafts(w, _np(am0))).cuda()
    sp = bd.SpeculativePlan(shape, lws, w_lm, dw, w.B, w.K)
    acc, nxt, em, am, nd = [t.clone() for t in sp(hidden, drafts)]
    sp.sync_status()
    acc2, nxt2, em2, am2 = [t.clone() for t in vplan(hidden, drafts)]
    vplan.sync_status()
    for a, b in ((acc, acc2), (nxt, nxt2), (em, em2), (am, am2)):
        np.testing.assert_array_equal(_np(a), _np(b))
    hL = _chain(hidden, shape, lws)
    rows = torch.arange(w.B, device="cuda") * (w.K + 1) + acc.long()
    nd2 = bd.fastmtp_draft(hL[rows].contiguous(), nxt, w.K, dw, w_lm)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(_np(nd)[:, :w.K], _np(nd2))
    # against the oracle's draft step on the GPU's own verifier state
    ref = oracle.fastmtp_draft(bd.bf16_from_device(hL[rows].contiguous()), _np(nxt), w.K, draft, inp["w_lm"])
    check_drafts(_np(nd)[:, :w.K], None, ref)


def test_gpu_draft_and_verify_loop_is_lossless():
    """The toy decoder's speculative loop with drafts from the GPU draft block
    (speculative_step) emits exactly the GPU's plain greedy stream."""
    from test_gpu_lossless import V, H, ToyGPU, greedy
    toy = ToyGPU()
    rng = np.random.default_rng(3)
    draft = {"w_emb": bf(rng.standard_normal((V, H))), "g_hidden": bf(np.ones(H)), "g_embed": bf(np.ones(H)),
             "w_proj": bf(rng.standard_normal((H, 2 * H)) * 0.1), "w_gate": bf(rng.standard_normal((64, H)) * 0.1),
             "w_up": bf(rng.standard_normal((64, H)) * 0.1), "w_down": bf(rng.standard_normal((H, 64)) * 0.1)}
    dw = bd.DraftWeights(draft)
    B, n = 16, 100
    prompts = [list(rng.integers(0, V, size=2)) for _ in range(B)]
    ref = greedy(toy, prompts, n + 8)
    for K in (1, 3):
        sp = bd.SpeculativePlan(toy.shape, toy.layers, toy.w_lm, dw, B, K)
        seqs = [list(p) for p in prompts]
        drafts = torch.zeros((B, K), dtype=torch.int32, device="cuda")
        while min(len(s) for s in seqs) < 2 + n:
            d = _np(drafts)
            cur, prev = [], []
            for b, s in enumerate(seqs):
                cur += [s[-1]] + list(d[b])
                prev += ([s[-2], s[-1]] + list(d[b][:-1]))[:K + 1]
            acc, _, em, _, nd = sp(bd.bf16_to_device(toy.rows(cur, prev)), drafts)
            sp.sync_status()
            acc, em = _np(acc), _np(em)
            for b, s in enumerate(seqs):
                s.extend(int(t) for t in em[b][:acc[b] + 1])
            drafts = nd[:, :K].clone()
            assert np.all((_np(drafts) >= 0) & (_np(drafts) < V))
        for b in range(B):
            assert seqs[b][:2 + n] == ref[b][:2 + n]
