"""Pins of the oracle's FastMTP draft block and RMSNorm (CPU).

The pages (jina-ocr-v1 model card, decoding-speed paragraph; the tldrocket
write-up, speculative paragraph) say only that the drafts come from one dense
draft block applied recursively K times.  The oracle's reading of the block
(RMSNorm of the previous hidden state and of the last token's embedding,
concatenated, projected 2H -> H, a dense SwiGLU FFN with residual, the shared
LM head's greedy choice) is pinned here by closed forms that a plausible slip
(the halves concatenated the other way round, a transposed projection, a
recursion that restarts from the first hidden state or token, a missing
residual or square root, eps outside the root) would break.
"""
import numpy as np
import pytest

from moe_decoder_speculative_b200 import workloads as wl

H = 64
V = 64


def bf(a):
    return wl.f32_to_bf16_bits(np.asarray(a, np.float32))


def f(b):
    return wl.bf16_bits_to_f32(b)


def perm_matrix(pi):
    """P with P @ e_v = e_{pi[v]}, i.e. P[pi[v], v] = 1."""
    n = len(pi)
    P = np.zeros((n, n), np.float32)
    P[pi, np.arange(n)] = 1.0
    return P


def base_block(rng, Id=64):
    """Draft weights with an all-zero FFN (y = 0) and unit gains."""
    return {
        "w_emb": bf(rng.standard_normal((V, H))),
        "g_hidden": bf(np.ones(H)),
        "g_embed": bf(np.ones(H)),
        "w_proj": bf(np.zeros((H, 2 * H))),
        "w_gate": bf(rng.standard_normal((Id, H)) * 0.1),
        "w_up": bf(rng.standard_normal((Id, H)) * 0.1),
        "w_down": bf(np.zeros((H, Id))),
    }


# ---------------------------------------------------------------- RMSNorm

@pytest.mark.parametrize("c", [3.0, 0.5, -2.0, 1024.0])
def test_rmsnorm_of_a_constant_row_is_the_gain(oracle_mod, c):
    rng = np.random.default_rng(1)
    g = bf(rng.uniform(0.5, 2.0, H))
    out = oracle_mod.rmsnorm(bf(np.full(H, c)), g)[0]
    np.testing.assert_array_equal(out, g if c > 0 else bf(-f(g)))


def test_rmsnorm_of_a_one_hot_row(oracle_mod):
    g = bf(np.linspace(0.5, 1.5, H))
    for i, s in [(0, 1.0), (17, 0.25), (63, 40.0)]:
        x = np.zeros(H, np.float32)
        x[i] = s
        out = f(oracle_mod.rmsnorm(bf(x), g)[0])
        expect = np.zeros(H, np.float32)
        expect[i] = f(bf([8.0 * f(g)[i]]))[0]  # sqrt(64) * g_i
        np.testing.assert_array_equal(out, expect)


def test_rmsnorm_eps_sits_inside_the_root_next_to_the_mean(oracle_mod):
    c, eps = 1e-3, 1e-6                     # mean(x^2) = eps: r = 1/sqrt(2 eps)
    out = f(oracle_mod.rmsnorm(bf(np.full(H, c)), bf(np.ones(H)), eps=eps)[0])
    cb = float(f(bf([c]))[0])
    np.testing.assert_array_equal(out, f(bf(np.full(H, cb / np.sqrt(cb * cb + eps)))))


def test_rmsnorm_is_scale_invariant_without_eps(oracle_mod):
    rng = np.random.default_rng(2)
    x = bf(rng.standard_normal((5, H)))
    g = bf(rng.uniform(0.5, 2.0, H))
    a = oracle_mod.rmsnorm(x, g, eps=0.0)
    for k in (-3, 4):
        np.testing.assert_array_equal(oracle_mod.rmsnorm(bf(f(x) * 2.0 ** k), g, eps=0.0), a)


def test_rmsnorm_float_within_rounding_of_double(oracle_mod):
    rng = np.random.default_rng(3)
    x = bf(rng.standard_normal((64, 1280)))
    g = bf(rng.uniform(0.5, 2.0, 1280))
    a = f(oracle_mod.rmsnorm(x, g))
    b = f(oracle_mod.rmsnorm(x, g, acc_double=True))
    # at most one bf16 ulp apart (the float sum of squares is within ~1e-6 relative)
    assert np.all(np.abs(a - b) <= np.abs(b) * 2.0 ** -7 + 1e-30)
    assert np.mean(a == b) > 0.99


# ---------------------------------------------------------------- draft block

def test_embedding_path_walks_a_permutation(oracle_mod):
    """W_proj = [0 | P], E = identity rows, W_lm = identity, FFN zero:
    z = P . RMSNorm(e_t) = 8 e_{pi(t)}, so the drafts are pi(t), pi^2(t), ...
    (the previous hidden state is ignored by the zero half)."""
    rng = np.random.default_rng(4)
    pi = rng.permutation(V)
    d = base_block(rng)
    d["w_emb"] = bf(np.eye(V, H) * 0.37)
    d["w_proj"] = bf(np.concatenate([np.zeros((H, H)), perm_matrix(pi)], axis=1))
    w_lm = bf(np.eye(V, H))
    B, K = 6, 4
    t0 = rng.integers(0, V, B).astype(np.int32)
    h0 = bf(rng.standard_normal((B, H)))
    out = oracle_mod.fastmtp_draft(h0, t0, K, d, w_lm)
    expect = np.zeros((B, K), np.int32)
    t = t0.copy()
    for j in range(K):
        t = pi[t]
        expect[:, j] = t
    np.testing.assert_array_equal(out["drafts"], expect)
    # each step's hidden state is exactly 8 e_{draft}
    for j in range(K):
        hs = f(out["h_steps"][j])
        np.testing.assert_array_equal(hs, 8.0 * np.eye(V, H)[expect[:, j]])


def test_hidden_path_recurses_on_the_blocks_own_output(oracle_mod):
    """W_proj = [Q | 0] (Q a permutation), FFN zero, W_lm = identity and
    h0 = 2 e_v: RMSNorm gives 8 e_v, z = 8 e_{sigma(v)}, and step j starts from
    step j-1's output, so the drafts are sigma(v), sigma^2(v), sigma^3(v)."""
    rng = np.random.default_rng(5)
    sigma = rng.permutation(V)
    d = base_block(rng)
    d["w_proj"] = bf(np.concatenate([perm_matrix(sigma), np.zeros((H, H))], axis=1))
    w_lm = bf(np.eye(V, H))
    B, K = 5, 3
    v = rng.integers(0, V, B)
    h0 = bf(2.0 * np.eye(V, H)[v])
    t0 = rng.integers(0, V, B).astype(np.int32)
    out = oracle_mod.fastmtp_draft(h0, t0, K, d, w_lm)
    expect = np.stack([sigma[v], sigma[sigma[v]], sigma[sigma[sigma[v]]]], axis=1)
    np.testing.assert_array_equal(out["drafts"], expect)
    np.testing.assert_array_equal(f(out["h_steps"][0]), 8.0 * np.eye(V, H)[sigma[v]])


def test_ffn_output_is_added_to_the_projection(oracle_mod):
    """W_proj = [I | 0], gate = up = down = identity, h0 = 2 e_v:
    z = 8 e_v, a = bf16(silu(8) * 8) = 64, h' = bf16(z + a) = 72 e_v, and the
    next step normalises 72 e_v back to 8 e_v, so every step gives 72 e_v."""
    rng = np.random.default_rng(6)
    d = base_block(rng, Id=H)
    d["w_proj"] = bf(np.concatenate([np.eye(H), np.zeros((H, H))], axis=1))
    d["w_gate"] = bf(np.eye(H))
    d["w_up"] = bf(np.eye(H))
    d["w_down"] = bf(np.eye(H))
    w_lm = bf(np.eye(V, H))
    B, K = 4, 3
    v = rng.integers(0, V, B)
    out = oracle_mod.fastmtp_draft(bf(2.0 * np.eye(V, H)[v]), np.zeros(B, np.int32), K, d, w_lm)
    a = float(f(bf([8.0 * 8.0 / (1.0 + np.exp(-8.0))]))[0])
    assert a == 64.0
    for j in range(K):
        np.testing.assert_array_equal(f(out["h_steps"][j]), 72.0 * np.eye(V, H)[v])
        np.testing.assert_array_equal(out["drafts"][:, j], v)


def test_gains_scale_their_own_half(oracle_mod):
    """A gain of 0.5 on the embedding half halves z on the embedding path and
    leaves the hidden path alone (the gains are not swapped)."""
    rng = np.random.default_rng(7)
    d = base_block(rng)
    d["w_emb"] = bf(np.eye(V, H))
    d["g_embed"] = bf(np.full(H, 0.5))
    d["w_proj"] = bf(np.concatenate([np.eye(H), np.eye(H)], axis=1))   # z = norm(h) + norm(e)
    w_lm = bf(np.eye(V, H))
    h0 = bf(2.0 * np.eye(V, H)[[3]])
    out = oracle_mod.fastmtp_draft(h0, np.array([9], np.int32), 1, d, w_lm)
    expect = np.zeros(H, np.float32)
    expect[3] = 8.0
    expect[9] = 4.0
    np.testing.assert_array_equal(f(out["h_steps"][0][0]), expect)
    assert out["drafts"][0, 0] == 3


def test_draft_arguments_are_checked(oracle_mod):
    rng = np.random.default_rng(8)
    d = base_block(rng)
    w_lm = bf(np.eye(V, H))
    with pytest.raises(ValueError):
        oracle_mod.fastmtp_draft(bf(np.ones((2, H))), np.array([0, V], np.int32), 2, d, w_lm)
    out = oracle_mod.fastmtp_draft(bf(np.ones((2, H))), np.array([0, 1], np.int32), 0, d, w_lm)
    assert out["drafts"].shape == (2, 0)


def test_speculative_loop_with_the_draft_block_is_lossless(oracle_mod):
    """The draft-and-verify loop (verify_step, then the draft block from the
    verifier's hidden state at the last kept row and its next token) emits
    exactly the plain greedy stream of a toy causal decoder."""
    rng = np.random.default_rng(9)
    Vt, E, k, I, Ish = 64, 8, 2, 64, 64
    layers = [{"w_router": bf(rng.standard_normal((E, H)) * 0.3),
               "w_gate": bf(rng.standard_normal((E, I, H)) * 0.2), "w_up": bf(rng.standard_normal((E, I, H)) * 0.2),
               "w_down": bf(rng.standard_normal((E, H, I)) * 0.2), "ws_gate": bf(rng.standard_normal((Ish, H)) * 0.2),
               "ws_up": bf(rng.standard_normal((Ish, H)) * 0.2), "ws_down": bf(rng.standard_normal((H, Ish)) * 0.2),
               "router_bias": None}]
    w_lm = bf(rng.standard_normal((Vt, H)) * 0.3)
    e1, e2 = rng.standard_normal((Vt, H)), rng.standard_normal((Vt, H))
    draft = {"w_emb": bf(rng.standard_normal((Vt, H))), "g_hidden": bf(np.ones(H)), "g_embed": bf(np.ones(H)),
             "w_proj": bf(rng.standard_normal((H, 2 * H)) * 0.1), "w_gate": bf(rng.standard_normal((64, H)) * 0.1),
             "w_up": bf(rng.standard_normal((64, H)) * 0.1), "w_down": bf(rng.standard_normal((H, 64)) * 0.1)}
    rows = lambda cur, prev: bf(e1[np.asarray(cur) % Vt] + e2[np.asarray(prev) % Vt])
    B, n = 8, 40
    prompts = [list(rng.integers(0, Vt, 2)) for _ in range(B)]
    greedy = [list(p) for p in prompts]
    for _ in range(n + 8):
        st = oracle_mod.verify_step(rows([s[-1] for s in greedy], [s[-2] for s in greedy]), None, B, 0, layers, k, w_lm)
        for s, t in zip(greedy, st["argmax"]):
            s.append(int(t))
    for K in (1, 3):
        seqs = [list(p) for p in prompts]
        drafts = np.zeros((B, K), np.int32)
        kept = 0
        while min(len(s) for s in seqs) < 2 + n:
            cur, prev = [], []
            for b, s in enumerate(seqs):
                cur += [s[-1]] + list(drafts[b])
                prev += ([s[-2], s[-1]] + list(drafts[b][:-1]))[:K + 1]
            st = oracle_mod.speculative_step(rows(cur, prev), drafts, B, K, layers, k, w_lm, draft)
            for b, s in enumerate(seqs):
                s.extend(int(t) for t in st["emitted"][b][:st["accepted"][b] + 1])
            kept += int(st["accepted"].sum())
            drafts = st["next_drafts"]
            assert drafts.shape == (B, K) and np.all((drafts >= 0) & (drafts < Vt))
        for b in range(B):
            assert seqs[b][:2 + n] == greedy[b][:2 + n]


# ------------------------------------------- where the loop step starts drafting

def _start_case(rng, half):
    """A verify step with no MoE layers (h_L = the input rows) whose rows are
    one-hot, row r = e_r, and an LM head that sends e_r to token pi(r), so the
    verifier's choice at row r is pi(r).  Each sequence's drafts are built to
    keep a chosen number of them.  The draft block has a zero FFN and reads
    only one half of its input: the hidden half (projection [I | 0]) or the
    embedding half ([0 | I], with one-hot embeddings E[v] = e_{sigma(v)})."""
    B, K = 4, 3
    T = B * (K + 1)
    pi = rng.permutation(V)
    sigma = rng.permutation(V)
    hidden = bf(np.eye(T, H))
    w_lm = bf(perm_matrix(pi))              # W_lm[pi[r]] = e_r
    g = pi[np.arange(T)]
    keep = np.array([2, 0, 3, 1])
    drafts = np.zeros((B, K), np.int32)
    for b in range(B):
        for i in range(K):
            d = g[b * (K + 1) + i]
            drafts[b, i] = d if i < keep[b] else (d + 1) % V
    blk = base_block(rng)
    proj = np.zeros((H, 2 * H), np.float32)
    if half == "hidden":
        proj[:, :H] = np.eye(H)
    else:
        proj[:, H:] = np.eye(H)
        blk["w_emb"] = bf(perm_matrix(sigma).T)   # E[v] = e_{sigma[v]}
    blk["w_proj"] = bf(proj)
    return B, K, pi, sigma, hidden, w_lm, drafts, keep, blk


def test_loop_step_drafts_from_the_last_kept_row(oracle_mod):
    """The draft block starts from the verifier's final hidden state at each
    sequence's last kept row, b*(K+1) + accepted[b].  With a block that reads
    only the hidden half, that row r = e_r normalises to 8 e_r, and every
    step's choice is pi(r): a start at row b*(K+1), or one past the kept row,
    gives another token."""
    rng = np.random.default_rng(31)
    B, K, pi, _, hidden, w_lm, drafts, keep, blk = _start_case(rng, "hidden")
    st = oracle_mod.speculative_step(hidden, drafts, B, K, [], 2, w_lm, blk)
    np.testing.assert_array_equal(st["accepted"], keep)
    r = np.arange(B) * (K + 1) + keep
    np.testing.assert_array_equal(st["next_drafts"], np.repeat(pi[r][:, None], K, axis=1))
    for wrong in (np.arange(B) * (K + 1), r + 1):
        assert np.any(pi[wrong] != pi[r])


def test_loop_step_drafts_from_the_verifiers_next_token(oracle_mod):
    """The first draft step embeds the verifier's next token, g at the last
    kept row: with a block that reads only the embedding half, t0 = pi(r)
    embeds to e_{sigma(pi(r))}, so the first draft is pi(sigma(pi(r))) and
    every later step walks pi o sigma once more."""
    rng = np.random.default_rng(32)
    B, K, pi, sigma, hidden, w_lm, drafts, keep, blk = _start_case(rng, "embed")
    st = oracle_mod.speculative_step(hidden, drafts, B, K, [], 2, w_lm, blk)
    r = np.arange(B) * (K + 1) + keep
    np.testing.assert_array_equal(st["next_token"], pi[r])
    t = pi[r]
    for j in range(K):
        t = pi[sigma[t]]
        np.testing.assert_array_equal(st["next_drafts"][:, j], t)
