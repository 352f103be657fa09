"""Pins for the CPU oracle: checks against what the pages and mathematics fix.

None of these re-types the oracle's loops.  Each pins a part of the oracle to
something outside it: a closed form on structured weights, an invariant, a
special case that reduces to a textbook or library routine, brute force over
tiny inputs, or a fact the pages print.  A plausible slip in the oracle (a
dropped term, a wrong sign or index, a transposed operand, a wrong tie rule)
fails at least one test here.
"""
import itertools
import json
import os

import numpy as np
import pytest
from scipy.special import softmax

from moe_decoder_speculative_b200 import workloads as wl

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16(a):
    return wl.f32_to_bf16_bits(np.asarray(a, np.float32))


def f32(b):
    return wl.bf16_bits_to_f32(b)


def rand_bf16(rng, shape, std):
    return bf16(rng.standard_normal(shape).astype(np.float32) * std)


# ---------------------------------------------------------------------------
# Router
# ---------------------------------------------------------------------------

def test_router_one_hot_logits_are_weight_columns(oracle_mod):
    """x = e_h0 makes every logit the router column W[:, h0] (+ bias): exact."""
    rng = np.random.default_rng(1)
    H, E, k = 32, 8, 3
    wr = rand_bf16(rng, (E, H), 1.0)
    bias = rng.standard_normal(E).astype(np.float32)
    for h0 in (0, 7, H - 1):
        x = np.zeros((1, H), np.float32)
        x[0, h0] = 1.0
        for b in (None, bias):
            _, _, logits, _ = oracle_mod.router(bf16(x), wr, k, bias=b)
            want = f32(wr[:, h0]) + (0 if b is None else b)
            np.testing.assert_array_equal(logits[0], want.astype(np.float32))


def test_router_logits_match_float64_matmul(oracle_mod):
    """General x: fp32 sequential logits equal the float64 product to fp32 accuracy."""
    rng = np.random.default_rng(2)
    T, H, E = 20, 1280, 64
    x, wr = rand_bf16(rng, (T, H), 1.0), rand_bf16(rng, (E, H), 0.02)
    _, _, logits, _ = oracle_mod.router(x, wr, 6)
    ref = f32(x).astype(np.float64) @ f32(wr).astype(np.float64).T
    bound = H * 2.0 ** -24 * (np.abs(f32(x)).astype(np.float64) @ np.abs(f32(wr)).astype(np.float64).T)
    assert np.all(np.abs(logits - ref) <= bound + 1e-12)


@pytest.mark.parametrize("E,k", [(8, 2), (8, 3), (6, 6), (7, 1)])
def test_router_selection_brute_force(oracle_mod, E, k):
    """The chosen set maximises the summed logits over all C(E,k) subsets; among
    equal-sum sets the lower expert ids win; slots run in descending logit order."""
    rng = np.random.default_rng(3 + E * 10 + k)
    H = 16
    for trial in range(40):
        wr = rand_bf16(rng, (E, H), 1.0)
        if trial % 2:   # force exact ties: duplicate some expert rows
            src = rng.integers(0, E, size=E // 2)
            dst = rng.choice(E, size=E // 2, replace=False)
            wr[dst] = wr[src]
        x = rand_bf16(rng, (1, H), 1.0)
        idx, w, logits, gap = oracle_mod.router(x, wr, k)
        l = logits[0].astype(np.float64)
        best = max(itertools.combinations(range(E), k),
                   key=lambda s: (sum(l[list(s)]), [-e for e in s]))
        assert sorted(idx[0].tolist()) == list(best)
        # slot order: descending logit, ascending id on ties
        keys = [(-l[e], e) for e in idx[0]]
        assert keys == sorted(keys)
        srt = np.sort(l)[::-1]
        want_gap = np.inf if k == E else srt[k - 1] - srt[k]
        assert gap[0] == np.float32(want_gap)


def test_router_fewer_than_k_numbers_takes_the_rest_by_id(oracle_mod):
    """Reading of the selection rule on degenerate rows: numbers first (largest
    first), then -inf logits by id, then NaN logits by id; k distinct experts.
    Logits are set through the bias on a zero row, so the expected ids follow
    from the rule alone.  Weights: 0 on -inf experts when the row has numbers
    and no NaN (a NaN logit anywhere makes the softmax over all E NaN)."""
    H, E, k = 8, 8, 6
    x = np.zeros((1, H), np.float32)
    wr = np.zeros((E, H), np.float32)
    nan, inf = np.float32(np.nan), np.float32(np.inf)
    cases = [
        # bias per expert                                    expected slots
        ([-inf, 0.5, -inf, 2.0, -inf, -inf, 1.0, -inf], [3, 6, 1, 0, 2, 4]),
        ([nan, 0.5, -inf, 2.0, nan, -inf, 1.0, nan], [3, 6, 1, 2, 5, 0]),
        ([nan, nan, nan, 1.0, nan, nan, nan, nan], [3, 0, 1, 2, 4, 5]),
        ([-inf] * 8, [0, 1, 2, 3, 4, 5]),
    ]
    for b, want in cases:
        b = np.array(b, np.float32)
        idx, w, _, _ = oracle_mod.router(bf16(x), bf16(wr), k, bias=b)
        assert idx[0].tolist() == want, (b, idx[0])
        fin = np.isfinite(b[want])
        if fin.any() and not np.isnan(b).any():
            assert np.all(w[0][~fin] == 0)
            np.testing.assert_allclose(w[0][fin].sum(), 1.0, rtol=1e-6)
        elif np.isnan(b).any():
            assert np.all(np.isnan(w[0]))


def test_router_nan_logits_do_not_displace_numbers(oracle_mod):
    """With at least k numbers, NaN logits change no selection: it equals the
    one with those experts at -inf.  The weights then follow the form over the
    selected experts (the softmax over all E would be NaN)."""
    rng = np.random.default_rng(41)
    T, H, E, k = 32, 64, 16, 4
    x, wr = rand_bf16(rng, (T, H), 1.0), rand_bf16(rng, (E, H), 0.3)
    b_nan = np.zeros(E, np.float32)
    b_nan[[0, 3, 9]] = np.nan
    b_inf = b_nan.copy()
    b_inf[[0, 3, 9]] = -np.inf
    a = oracle_mod.router(x, wr, k, bias=b_nan, weight_form=1)
    c = oracle_mod.router(x, wr, k, bias=b_inf, weight_form=1)
    np.testing.assert_array_equal(a[0], c[0])
    np.testing.assert_array_equal(a[1], c[1])
    assert np.all(np.isfinite(a[1]))
    assert not np.isin(a[0], [0, 3, 9]).any()


def test_gate_weights_invariants_and_forms(oracle_mod):
    """w >= 0, sum w = 1, and the literal softmax-then-renormalise form equals
    the short form exp(l - l_max_sel) / sum_sel."""
    rng = np.random.default_rng(4)
    T, H, E, k = 64, 128, 64, 6
    x, wr = rand_bf16(rng, (T, H), 1.0), rand_bf16(rng, (E, H), 0.2)
    idx0, w0, _, _ = oracle_mod.router(x, wr, k, weight_form=0)
    idx1, w1, _, _ = oracle_mod.router(x, wr, k, weight_form=1)
    np.testing.assert_array_equal(idx0, idx1)
    assert np.all(w0 >= 0)
    assert np.all(np.abs(w0.astype(np.float64).sum(1) - 1) <= 1e-6)
    np.testing.assert_allclose(w0, w1, rtol=1e-6, atol=1e-7)
    # weights are non-increasing along the slots (slots are in logit order)
    assert np.all(np.diff(w0, axis=1) <= 1e-7)


def test_gate_k_equals_E_is_full_softmax(oracle_mod):
    rng = np.random.default_rng(5)
    T, H, E = 16, 64, 8
    x, wr = rand_bf16(rng, (T, H), 1.0), rand_bf16(rng, (E, H), 0.5)
    idx, w, logits, gap = oracle_mod.router(x, wr, E)
    assert np.all(np.isinf(gap))
    p = softmax(logits.astype(np.float64), axis=1)
    got = np.zeros_like(p)
    np.put_along_axis(got, idx, w, axis=1)
    np.testing.assert_allclose(got, p, rtol=2e-6, atol=1e-8)


def test_gate_equal_logits_give_uniform_weights(oracle_mod):
    H, E, k = 8, 8, 4
    wr = np.zeros((E, H), np.float32)
    wr[:4, 0] = 2.0     # four experts tie at the top
    wr[4:, 0] = -1.0
    x = np.zeros((1, H), np.float32)
    x[0, 0] = 1.0
    idx, w, _, gap = oracle_mod.router(bf16(x), bf16(wr), k)
    assert idx[0].tolist() == [0, 1, 2, 3]
    np.testing.assert_array_equal(w[0], np.full(k, 0.25, np.float32))
    assert gap[0] == 3.0


# ---------------------------------------------------------------------------
# Expert SwiGLU
# ---------------------------------------------------------------------------

def _silu64(g):
    return g / (1.0 + np.exp(-g))


def test_swiglu_permutation_weights_closed_form(oracle_mod):
    """With Wg, Wu selection matrices (row i picks x[pi_g(i)], x[pi_u(i)]) and Wd
    picking a[sigma(h)], the expert output is y[h] = c_d * a[sigma(h)] with
    a[i] = bf16(silu(c_g x[pi_g(i)]) * c_u x[pi_u(i)]).  I != H, so a transposed
    or mis-strided weight read lands on the wrong entries."""
    rng = np.random.default_rng(6)
    H, I = 24, 16
    cg, cu, cd = 0.5, 2.0, 0.25
    pig = rng.permutation(H)[:I]
    piu = rng.permutation(H)[:I]
    sig = rng.integers(0, I, size=H)
    wg = np.zeros((I, H), np.float32)
    wg[np.arange(I), pig] = cg
    wu = np.zeros((I, H), np.float32)
    wu[np.arange(I), piu] = cu
    wd = np.zeros((H, I), np.float32)
    wd[np.arange(H), sig] = cd
    for trial in range(20):
        x = bf16(rng.standard_normal(H) * 3)
        a, y = oracle_mod.swiglu(x, bf16(wg), bf16(wu), bf16(wd))
        xf = f32(x).astype(np.float64)
        a_want = _silu64(cg * xf[pig]) * (cu * xf[piu])
        # a is bf16: allow the one-ulp rounding flip a float-vs-double silu can cause
        assert np.all(np.abs(f32(a) - a_want) <= np.abs(a_want) * 2.0 ** -8 + 1e-30)
        np.testing.assert_array_equal(y, (cd * f32(a)[sig]).astype(np.float32))


def test_swiglu_zero_gate_gives_zero(oracle_mod):
    """silu(0) = 0: a zero gate row kills the activation whatever the up row is."""
    rng = np.random.default_rng(7)
    H, I = 16, 8
    x = rand_bf16(rng, H, 1.0)
    wg = np.zeros((I, H), np.uint16)
    wu, wd = rand_bf16(rng, (I, H), 1.0), rand_bf16(rng, (H, I), 1.0)
    a, y = oracle_mod.swiglu(x, wg, wu, wd)
    assert np.all(f32(a) == 0) and np.all(y == 0)


def test_shared_pair_equals_concatenated_expert(oracle_mod):
    """Two experts of intermediate I summed equal one expert of 2I whose gate/up
    rows and down columns are the two concatenated (the shared-expert reading)."""
    rng = np.random.default_rng(8)
    H, I = 64, 32
    x = rand_bf16(rng, H, 1.0)
    g1, u1, d1 = rand_bf16(rng, (I, H), 0.1), rand_bf16(rng, (I, H), 0.1), rand_bf16(rng, (H, I), 0.1)
    g2, u2, d2 = rand_bf16(rng, (I, H), 0.1), rand_bf16(rng, (I, H), 0.1), rand_bf16(rng, (H, I), 0.1)
    _, y1 = oracle_mod.swiglu(x, g1, u1, d1, acc_double=True)
    _, y2 = oracle_mod.swiglu(x, g2, u2, d2, acc_double=True)
    _, y12 = oracle_mod.swiglu(x, np.vstack([g1, g2]), np.vstack([u1, u2]),
                               np.hstack([d1, d2]), acc_double=True)
    np.testing.assert_allclose(y12, y1.astype(np.float64) + y2, rtol=1e-6, atol=1e-7)


# ---------------------------------------------------------------------------
# MoE layer
# ---------------------------------------------------------------------------

def _tiny_layer(rng, H, E, I, Ish, std=0.1):
    return {
        "w_router": rand_bf16(rng, (E, H), 0.3),
        "w_gate": rand_bf16(rng, (E, I, H), std), "w_up": rand_bf16(rng, (E, I, H), std),
        "w_down": rand_bf16(rng, (E, H, I), std),
        "ws_gate": rand_bf16(rng, (Ish, H), std), "ws_up": rand_bf16(rng, (Ish, H), std),
        "ws_down": rand_bf16(rng, (H, Ish), std),
    }


def _dense_mixture(x, layer, probs):
    """sum_e p_e FFN_e(x) + shared(x), in float64 with a rounded to bf16."""
    xf = f32(x).astype(np.float64)
    out = np.zeros((x.shape[0], x.shape[1]))

    def ffn(wg, wu, wd):
        g = xf @ f32(wg).astype(np.float64).T
        u = xf @ f32(wu).astype(np.float64).T
        a = f32(bf16((_silu64(g) * u).astype(np.float32))).astype(np.float64)
        return a @ f32(wd).astype(np.float64).T

    for e in range(layer["w_gate"].shape[0]):
        out += probs[:, e:e + 1] * ffn(layer["w_gate"][e], layer["w_up"][e], layer["w_down"][e])
    return out + ffn(layer["ws_gate"], layer["ws_up"], layer["ws_down"])


def test_k_equals_E_is_dense_mixture(oracle_mod):
    """Top-k with k = E reproduces the dense softmax-weighted mixture of all
    experts plus the shared expert."""
    rng = np.random.default_rng(9)
    T, H, E, I, Ish = 12, 64, 8, 32, 32
    layer = _tiny_layer(rng, H, E, I, Ish)
    x = rand_bf16(rng, (T, H), 1.0)
    idx, w, logits, _ = oracle_mod.router(x, layer["w_router"], E)
    m, _ = oracle_mod.moe_ffn(x, layer, idx, w)
    want = _dense_mixture(x, layer, softmax(logits.astype(np.float64), axis=1))
    rms = np.sqrt(np.mean(want ** 2))
    assert np.max(np.abs(m - want)) <= 2e-3 * rms


def test_moe_shared_added_with_weight_one_and_residual(oracle_mod):
    rng = np.random.default_rng(10)
    T, H, E, I, Ish, k = 8, 64, 8, 32, 64, 2
    layer = _tiny_layer(rng, H, E, I, Ish)
    x = rand_bf16(rng, (T, H), 1.0)
    idx, w, _, _ = oracle_mod.router(x, layer["w_router"], k)
    m, out_plain = oracle_mod.moe_ffn(x, layer, idx, w)
    no_shared = dict(layer, ws_gate=None, ws_up=None, ws_down=None)
    m0, _ = oracle_mod.moe_ffn(x, no_shared, idx, w)
    ysh = np.stack([oracle_mod.swiglu(x[r], layer["ws_gate"], layer["ws_up"], layer["ws_down"])[1]
                    for r in range(T)])
    np.testing.assert_allclose(m - m0, ysh, rtol=1e-5, atol=1e-6)
    # without residual out = bf16(m); with residual out = bf16(res + m)
    np.testing.assert_array_equal(out_plain, bf16(m))
    res = rand_bf16(rng, (T, H), 4.0)
    _, out_res = oracle_mod.moe_ffn(x, layer, idx, w, residual=res)
    np.testing.assert_array_equal(out_res, bf16(f32(res) + m))


def test_routed_weights_scale_expert_outputs(oracle_mod):
    """With one slot (k=1) the routed part is w * y_e; moving the weight moves it."""
    rng = np.random.default_rng(11)
    H, E, I = 32, 4, 16
    layer = _tiny_layer(rng, H, E, I, 0)
    layer.update(ws_gate=None, ws_up=None, ws_down=None)
    x = rand_bf16(rng, (1, H), 1.0)
    for e in range(E):
        _, y = oracle_mod.swiglu(x[0], layer["w_gate"][e], layer["w_up"][e], layer["w_down"][e])
        for wv in (1.0, 0.5, 0.25):
            m, _ = oracle_mod.moe_ffn(x, layer, np.array([[e]], np.int32),
                                      np.array([[wv]], np.float32))
            np.testing.assert_array_equal(m[0], (np.float32(wv) * y).astype(np.float32))


def test_zero_weight_layer_is_identity_on_residual(oracle_mod):
    rng = np.random.default_rng(12)
    T, H, E, I = 8, 64, 8, 32
    z = {k: np.zeros_like(v) for k, v in _tiny_layer(rng, H, E, I, 32).items()}
    h = rand_bf16(rng, (T, H), 1.0)
    st = oracle_mod.moe_stack(h, [z, z, z], 2)
    np.testing.assert_array_equal(st["h"], h)


def test_batch_invariance(oracle_mod):
    """A row's result is the same alone or inside a batch (rows are independent)."""
    w = wl.workload(0)
    inp = wl.make_inputs(w)
    x = inp["hidden"]
    full = oracle_mod.moe_stack(x, inp["layers"], w.k)
    for r in (0, 5, 15):
        one = oracle_mod.moe_stack(x[r:r + 1], inp["layers"], w.k)
        np.testing.assert_array_equal(one["h"][0], full["h"][r])


def test_float_oracle_within_bound_of_double(oracle_mod):
    """The fp32 oracle stays within a small multiple of the fp32 summation bound
    of its double-accumulation mode on the tiny workload."""
    w = wl.workload(0)
    inp = wl.make_inputs(w)
    a = oracle_mod.moe_stack(inp["hidden"], inp["layers"], w.k, keep=True)
    b = oracle_mod.moe_stack(inp["hidden"], inp["layers"], w.k, keep=True, acc_double=True)
    for la, lb in zip(a["layers"], b["layers"]):
        same = np.all(la["idx"] == lb["idx"], axis=1)
        assert same.mean() > 0.9
        d = np.abs(la["m"] - lb["m"])[same]
        rms = np.sqrt(np.mean(lb["m"][same].astype(np.float64) ** 2))
        assert d.max() <= 1e-4 * rms


# ---------------------------------------------------------------------------
# LM head + greedy choice
# ---------------------------------------------------------------------------

def test_lm_one_hot_picks_column_argmax(oracle_mod):
    rng = np.random.default_rng(13)
    H, V = 32, 300
    wlm = rand_bf16(rng, (V, H), 1.0)
    for h0 in (0, 3, H - 1):
        h = np.zeros((1, H), np.float32)
        h[0, h0] = 1.0
        am, zmax, gap = oracle_mod.lm_head_argmax(bf16(h), wlm)
        col = f32(wlm[:, h0]).astype(np.float64)
        assert am[0] == int(np.argmax(col))
        assert zmax[0] == col.max()
        s = np.sort(col)
        assert gap[0] == np.float32(s[-1] - s[-2])


def test_lm_random_matches_float64_argmax(oracle_mod):
    rng = np.random.default_rng(14)
    T, H, V = 64, 256, 2000
    h, wlm = rand_bf16(rng, (T, H), 1.0), rand_bf16(rng, (V, H), 0.05)
    am, zmax, gap = oracle_mod.lm_head_argmax(h, wlm)
    z = f32(h).astype(np.float64) @ f32(wlm).astype(np.float64).T
    srt = np.sort(z, axis=1)
    clear = (srt[:, -1] - srt[:, -2]) > 1e-5
    assert clear.mean() > 0.9
    np.testing.assert_array_equal(am[clear], np.argmax(z, axis=1)[clear])
    np.testing.assert_allclose(zmax, z.max(1), rtol=1e-5, atol=1e-5)


def test_lm_exact_tie_goes_to_lower_index(oracle_mod):
    """Copying a row's winning LM-head row to a lower index makes an exact tie,
    which the lower index wins with gap 0; copying it higher changes nothing."""
    rng = np.random.default_rng(15)
    T, H, V = 8, 64, 500
    h, wlm = rand_bf16(rng, (T, H), 1.0), rand_bf16(rng, (V, H), 0.05)
    am, _, _ = oracle_mod.lm_head_argmax(h, wlm)
    for r in range(T):
        g = int(am[r])
        lo = g - 1 - int(rng.integers(0, max(1, g)))  # some index below g
        if lo >= 0:
            w2 = wlm.copy()
            w2[lo] = wlm[g]
            am2, _, gap2 = oracle_mod.lm_head_argmax(h[r:r + 1], w2)
            assert am2[0] == lo and gap2[0] == 0.0
        if g + 1 < V:
            w3 = wlm.copy()
            w3[g + 1] = wlm[g]
            am3, _, gap3 = oracle_mod.lm_head_argmax(h[r:r + 1], w3)
            assert am3[0] == g and gap3[0] == 0.0
    # an all-zero head: every logit is 0, the first index wins
    am0, _, gap0 = oracle_mod.lm_head_argmax(h, np.zeros_like(wlm))
    assert np.all(am0 == 0) and np.all(gap0 == 0)


# ---------------------------------------------------------------------------
# Greedy acceptance
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("K", [0, 1, 2, 3])
def test_accept_exhaustive_small(oracle_mod, K):
    """Every (verifier choices, drafts) pair over a 3-token vocabulary: the kept
    prefix is the longest common prefix of drafts and choices; the committed
    tokens are that prefix plus the verifier's next choice."""
    V = 3
    cases_g = list(itertools.product(range(V), repeat=K + 1))
    cases_d = list(itertools.product(range(V), repeat=K))
    G = np.array([g for g in cases_g for _ in cases_d], np.int32)
    D = np.array([d for _ in cases_g for d in cases_d], np.int32).reshape(len(G), K)
    B = len(G)
    acc, nxt, em = oracle_mod.greedy_accept(G.reshape(-1), D, B, K)
    for b in range(B):
        a = len(os.path.commonprefix([list(D[b]), list(G[b][:K])]))
        assert acc[b] == a
        assert nxt[b] == G[b][a]
        assert list(em[b][:a + 1]) == list(G[b][:a + 1])
        assert np.all(em[b][a + 1:] == -1)
        assert 0 <= acc[b] <= K


def test_accept_extreme_drafters(oracle_mod):
    rng = np.random.default_rng(16)
    B, K, V = 50, 3, 1000
    g = rng.integers(0, V, size=(B, K + 1)).astype(np.int32)
    acc, nxt, _ = oracle_mod.greedy_accept(g.reshape(-1), g[:, :K].copy(), B, K)
    assert np.all(acc == K) and np.all(nxt == g[:, K])
    wrong = (g[:, :K] + 1) % V
    acc, nxt, _ = oracle_mod.greedy_accept(g.reshape(-1), wrong, B, K)
    assert np.all(acc == 0) and np.all(nxt == g[:, 0])


@pytest.mark.parametrize("p,K", [(0.576, 3), (0.9, 1), (0.3, 2)])
def test_accept_expected_commit_closed_form(oracle_mod, p, K):
    """Drafts that independently agree with probability p commit
    E[a + 1] = 1 + p + ... + p^K tokens per pass."""
    rng = np.random.default_rng(17)
    B, V = 200_000, 1 << 20
    g = rng.integers(0, V, size=(B, K + 1)).astype(np.int32)
    agree = rng.random((B, K)) < p
    d = np.where(agree, g[:, :K], (g[:, :K] + 1) % V).astype(np.int32)
    acc, _, _ = oracle_mod.greedy_accept(g.reshape(-1), d, B, K)
    want = sum(p ** j for j in range(K + 1))
    se = np.std(acc + 1) / np.sqrt(B)
    assert abs(np.mean(acc + 1) - want) < 6 * se


def test_pages_tokens_per_pass_golden():
    """The pages print K=3, 57.6% acceptance and 'up to 2.7 tokens per verifier
    pass'; reading the rate as the kept fraction of drafted tokens, one pass
    commits 1 + K * rate of them."""
    facts = json.load(open(os.path.join(GOLDEN, "model_card_facts.json")))
    per_pass = 1 + facts["drafts_K"] * facts["acceptance_rate"]
    assert round(per_pass, 1) == facts["tokens_per_verifier_pass_up_to"]
    assert 1 <= per_pass <= facts["drafts_K"] + 1


# ---------------------------------------------------------------------------
# Losslessness on a toy decoder
# ---------------------------------------------------------------------------

class ToyDecoder:
    """V=64, H=64 toy: h_t = bf16(E1[tok_t] + E2[tok_{t-1}]), two MoE layers with
    residual, LM-head argmax.  Causal: a row depends only on its own two tokens."""

    def __init__(self, oracle_mod, seed=0, V=64, H=64):
        rng = np.random.default_rng(seed)
        self.o = oracle_mod
        self.V, self.H = V, H
        self.e1 = rng.standard_normal((V, H)).astype(np.float32)
        self.e2 = rng.standard_normal((V, H)).astype(np.float32)
        self.layers = [_tiny_layer(rng, H, 4, 32, 32, std=0.2) for _ in range(2)]
        self.w_lm = rand_bf16(rng, (V, H), 0.3)

    def next_tokens(self, cur, prev):
        h = bf16(self.e1[np.asarray(cur)] + self.e2[np.asarray(prev)])
        st = self.o.moe_stack(h, self.layers, 2)
        am, _, _ = self.o.lm_head_argmax(st["h"], self.w_lm)
        return am


def _greedy(toy, prompts, n):
    seqs = [list(p) for p in prompts]
    for _ in range(n):
        nxt = toy.next_tokens([s[-1] for s in seqs], [s[-2] for s in seqs])
        for s, t in zip(seqs, nxt):
            s.append(int(t))
    return seqs


def _speculative(toy, prompts, n, K, drafter):
    seqs = [list(p) for p in prompts]
    B = len(seqs)
    passes = 0
    target = len(prompts[0]) + n
    while min(len(s) for s in seqs) < target:
        drafts = np.array([drafter(b, s, K) for b, s in enumerate(seqs)], np.int32).reshape(B, K)
        cur, prev = [], []
        for b, s in enumerate(seqs):
            toks = [s[-1]] + list(drafts[b])
            prevs = [s[-2], s[-1]] + list(drafts[b][:-1]) if K else [s[-2]]
            cur += toks
            prev += prevs[:K + 1]
        g = toy.next_tokens(cur, prev)
        acc, nxt, em = toy.o.greedy_accept(g, drafts, B, K)
        for b, s in enumerate(seqs):
            if len(s) < target:
                s.extend(int(t) for t in em[b][:acc[b] + 1])
        passes += 1
    return [s[:target] for s in seqs], passes


@pytest.mark.parametrize("K", [0, 1, 3])
@pytest.mark.parametrize("kind", ["copy0.576", "right", "wrong", "random"])
def test_speculative_loop_is_lossless(oracle_mod, K, kind):
    toy = ToyDecoder(oracle_mod)
    rng = np.random.default_rng(18)
    prompts = [list(rng.integers(0, toy.V, size=2)) for _ in range(16)]
    n = 200
    ref = _greedy(toy, prompts, n + 3 * (K + 1))

    def drafter(b, s, K):
        truth = ref[b][len(s):len(s) + K]
        truth = list(truth) + [0] * (K - len(truth))   # sequences already done
        out = []
        for t in truth:
            if kind == "right" or (kind == "copy0.576" and rng.random() < 0.576):
                out.append(t)
            elif kind == "wrong":
                out.append((t + 1) % toy.V)
            else:
                out.append(int(rng.integers(0, toy.V)))
        return out

    got, passes = _speculative(toy, prompts, n, K, drafter)
    assert got == [s[:len(got[0])] for s in ref]
    if kind == "right":
        assert passes <= -(-n // (K + 1)) + 1
    if kind == "wrong" or K == 0:
        assert passes == n


# ---------------------------------------------------------------------------
# Shape facts the pages print
# ---------------------------------------------------------------------------

def test_model_shape_matches_pages():
    facts = json.load(open(os.path.join(GOLDEN, "model_card_facts.json")))
    w = wl.workload(2)
    assert (w.H, w.E, w.k, w.V, w.L) == (facts["hidden"], facts["routed_experts"], facts["top_k"],
                                         facts["vocab"], facts["decoder_layers"])
    assert w.I_sh == facts["shared_experts"] * w.I
    assert w.T == 32 * (facts["drafts_K"] + 1)
    assert wl.workload(3).T == 8 * facts["visual_tokens_per_page_max"]
    # Active parameters per token: per layer (top-k routed + shared) SwiGLU
    # experts, the router and a 4*H^2 attention block, plus the LM head.  The
    # pages say "about 570M"; the expert intermediate of 896 lands within 2%.
    per_layer = 3 * w.H * w.I * w.k + 3 * w.H * w.I_sh + w.H * w.E + 4 * w.H * w.H
    active = w.L * per_layer + w.V * w.H
    assert abs(active / facts["active_params_per_token"] - 1) < 0.02


def test_workload_generation_is_deterministic():
    w = wl.workload(0)
    a, b = wl.make_inputs(w), wl.make_inputs(w)
    np.testing.assert_array_equal(a["hidden"], b["hidden"])
    np.testing.assert_array_equal(a["layers"][0]["w_down"], b["layers"][0]["w_down"])
    np.testing.assert_array_equal(a["w_lm"], b["w_lm"])
    x = f32(a["hidden"])
    assert abs(x.std() - 0.02) < 0.002
    # bf16 rounding of the encoder is nearest-even
    v = np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 0.0], np.float32)
    np.testing.assert_array_equal(f32(wl.f32_to_bf16_bits(v)), np.array([1.0, 1.0 + 2 ** -6, -2.5, 0.0], np.float32))
