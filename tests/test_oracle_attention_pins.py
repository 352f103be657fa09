"""Pins of the oracle's decoder self-attention and rotary positions (CPU).

The pages give the decoder's attention only one fact: a 32,768-position
limit (jina-ocr-v1 model card, architecture paragraph).  The oracle's reading
(causal multi-head attention of each verify row over its sequence's key /
value cache, scores scaled by 1/sqrt(d), softmax, weighted sum of values;
rotary positions on pairs (i, i + d/2) with base 10,000) is pinned here by
closed forms and by a brute force written with numpy / scipy, so that a
plausible slip (a missing square root in the scale, an off-by-one in the
causal bound, a transposed cache index, interleaved rotary pairs, the wrong
rotation sense) breaks a test.
"""
import numpy as np
import pytest
import scipy.special

from moe_decoder_speculative_b200 import workloads as wl


def bf(a):
    return wl.f32_to_bf16_bits(np.asarray(a, np.float32))


def f(b):
    return wl.bf16_bits_to_f32(b).astype(np.float64)


def case(rng, B=3, K=3, nh=2, d=64, L=40, ctx=(0, 7, 30), q_scale=1.0):
    q = bf(rng.standard_normal((B * (K + 1), nh * d)) * q_scale)
    kc = bf(rng.standard_normal((B, nh, L, d)))
    vc = bf(rng.standard_normal((B, nh, L, d)))
    return q, kc, vc, np.array(ctx[:B], np.int32)


def brute(q, kc, vc, ctx, K):
    """The definition with numpy / scipy, vectorised per (row, head)."""
    B, nh, L, d = kc.shape
    out = np.zeros((B * (K + 1), nh * d))
    for r in range(B * (K + 1)):
        b, j = divmod(r, K + 1)
        p = ctx[b] + j
        for h in range(nh):
            qv = f(q[r, h * d:(h + 1) * d])
            s = f(kc[b, h, :p + 1]) @ qv / np.sqrt(d)
            out[r, h * d:(h + 1) * d] = scipy.special.softmax(s) @ f(vc[b, h, :p + 1])
    return out


def test_attention_matches_a_numpy_scipy_brute_force(oracle_mod):
    rng = np.random.default_rng(1)
    K = 3
    q, kc, vc, ctx = case(rng, K=K)
    o = oracle_mod.decode_attention(q, kc, vc, ctx, K)
    np.testing.assert_allclose(o, brute(q, kc, vc, ctx, K), rtol=1e-12, atol=1e-12)


def test_one_visible_position_returns_its_value(oracle_mod):
    """ctx = 0 and K = 0: the only visible position is the row's own, so the
    softmax is exactly 1 and the output is that position's value row."""
    rng = np.random.default_rng(2)
    q, kc, vc, _ = case(rng, B=2, K=0, ctx=(0, 0))
    o = oracle_mod.decode_attention(q, kc, vc, np.zeros(2, np.int32), 0)
    nh, d = kc.shape[1], kc.shape[3]
    for b in range(2):
        np.testing.assert_array_equal(o[b].reshape(nh, d), f(vc[b, :, 0]))


def test_zero_query_averages_the_visible_values(oracle_mod):
    """q = 0 gives equal scores: the output is the mean of the values at
    positions 0..ctx+j, and nothing after them."""
    rng = np.random.default_rng(3)
    K = 3
    _, kc, vc, ctx = case(rng, K=K)
    B, nh, L, d = kc.shape
    q = np.zeros((B * (K + 1), nh * d), np.uint16)
    o = oracle_mod.decode_attention(q, kc, vc, ctx, K)
    for r in range(B * (K + 1)):
        b, j = divmod(r, K + 1)
        want = f(vc[b, :, :ctx[b] + j + 1]).mean(axis=1).reshape(-1)
        np.testing.assert_allclose(o[r], want, rtol=1e-13, atol=1e-14)


def test_scores_carry_the_inverse_square_root_scale(oracle_mod):
    """Two visible positions: the weight of position 1 is 1 / (1 + e^{s0 - s1})
    with s = q . k / sqrt(d) (a scale of 1/d or 1 gives another number)."""
    d = 64
    q = bf(np.full((1, d), 0.5))
    kc = np.zeros((1, 1, 4, d), np.uint16)
    kc[0, 0, 0] = bf(np.full(d, 0.25))
    kc[0, 0, 1] = bf(np.full(d, -0.125))
    vc = np.zeros((1, 1, 4, d), np.uint16)
    vc[0, 0, 0] = bf(np.full(d, 1.0))
    vc[0, 0, 1] = bf(np.full(d, -3.0))
    o = oracle_mod.decode_attention(q, kc, vc, np.array([1], np.int32), 0)
    s0, s1 = 0.5 * 0.25 * d / np.sqrt(d), -0.5 * 0.125 * d / np.sqrt(d)
    w1 = 1.0 / (1.0 + np.exp(s0 - s1))
    np.testing.assert_allclose(o[0], np.full(d, (1 - w1) * 1.0 + w1 * -3.0), rtol=1e-14)


def test_a_dominant_score_picks_its_cache_row(oracle_mod):
    """Row j of sequence b, head h, has the query 1000 e_i (its own dimension
    i) and meets the key e_i at one chosen visible position; every other key of
    that head is another row's e_i' or zero, so the chosen position scores
    1000 / sqrt(d) = 125 against 0 and the output is its value row.  Pins the
    [b][h][pos][d] cache indexing and that each head reads its own q slice."""
    rng = np.random.default_rng(4)
    B, K, nh, d, L = 2, 1, 3, 64, 16
    ctx = np.array([5, 9], np.int32)
    kc = np.zeros((B, nh, L, d), np.uint16)
    vc = bf(rng.standard_normal((B, nh, L, d)))
    q = np.zeros((B * (K + 1), nh * d), np.uint16)
    pick = {}
    for b in range(B):
        for h in range(nh):
            dims = rng.choice(d, size=K + 1, replace=False)
            poss = rng.choice(ctx[b] + 1, size=K + 1, replace=False)   # visible to every row of b
            for j in range(K + 1):
                r = b * (K + 1) + j
                q[r, h * d + dims[j]] = bf([1000.0])[0]
                kc[b, h, poss[j], dims[j]] = bf([1.0])[0]
                pick[(r, h)] = (b, int(poss[j]))
    o = oracle_mod.decode_attention(q, kc, vc, ctx, K)
    for (r, h), (b, pos) in pick.items():
        np.testing.assert_allclose(o[r, h * d:(h + 1) * d], f(vc[b, h, pos]), rtol=1e-15, atol=0)


def test_rows_see_exactly_their_causal_prefix(oracle_mod):
    """Row j of a sequence sees positions 0..ctx+j: changing keys or values at
    later positions (including this step's later rows) leaves it unchanged, and
    changing position ctx+j itself changes it."""
    rng = np.random.default_rng(5)
    K = 3
    q, kc, vc, ctx = case(rng, K=K)
    base = oracle_mod.decode_attention(q, kc, vc, ctx, K)
    B = len(ctx)
    for b in range(B):
        for j in range(K + 1):
            r = b * (K + 1) + j
            p = ctx[b] + j
            k2, v2 = kc.copy(), vc.copy()
            k2[b, :, p + 1:] = bf(rng.standard_normal(k2[b, :, p + 1:].shape))
            v2[b, :, p + 1:] = bf(rng.standard_normal(v2[b, :, p + 1:].shape))
            o2 = oracle_mod.decode_attention(q, k2, v2, ctx, K)
            np.testing.assert_array_equal(o2[r], base[r])
            v3 = vc.copy()
            v3[b, :, p] = bf(f(v3[b, :, p]) + 1.0)
            o3 = oracle_mod.decode_attention(q, kc, v3, ctx, K)
            assert np.all(o3[r] != base[r])


def test_attention_arguments_are_checked(oracle_mod):
    rng = np.random.default_rng(6)
    q, kc, vc, _ = case(rng, B=1, K=3, ctx=(0,))
    with pytest.raises(ValueError):
        oracle_mod.decode_attention(q, kc, vc, np.array([kc.shape[2] - 3], np.int32), 3)   # past the cache


# ---------------------------------------------------------------- rotary positions

def test_rope_at_position_zero_is_the_identity(oracle_mod):
    rng = np.random.default_rng(7)
    x = bf(rng.standard_normal((3, 2 * 64)))
    np.testing.assert_array_equal(oracle_mod.rope(x, np.zeros(3, np.int32), 2), x)


def test_rope_turns_pairs_i_and_i_plus_half(oracle_mod):
    """d = 4: e_0 at position p becomes (cos p, 0, sin p, 0) and e_2 becomes
    (-sin p, 0, cos p, 0) (pairs (0, 2) and (1, 3), the first pair at angle p),
    and e_1 turns by p / sqrt(10000) = p / 100 into (0, cos, 0, sin).
    Interleaved pairs (0, 1) or the opposite sense fail."""
    for p in (1, 3, 17):
        y0 = f(oracle_mod.rope(bf([[1, 0, 0, 0]]), np.array([p], np.int32), 1)[0])
        np.testing.assert_array_equal(y0, f(bf([np.cos(p), 0, np.sin(p), 0])))
        y1 = f(oracle_mod.rope(bf([[0, 1, 0, 0]]), np.array([p], np.int32), 1)[0])
        a = p * 10000.0 ** (-2 * 1 / 4)
        np.testing.assert_array_equal(y1, f(bf([0, np.cos(a), 0, np.sin(a)])))
        y2 = f(oracle_mod.rope(bf([[0, 0, 1, 0]]), np.array([p], np.int32), 1)[0])
        np.testing.assert_array_equal(y2, f(bf([-np.sin(p), 0, np.cos(p), 0])))   # the same turn, e_2 -> (-sin, cos)


def test_rope_scores_depend_on_the_relative_position(oracle_mod):
    """q . k after rotating q to position m and k to n depends only on m - n
    (up to the bf16 rounding of the rotated vectors), and each head rotates
    on its own."""
    rng = np.random.default_rng(8)
    d, nh = 128, 2
    q = bf(rng.standard_normal((1, nh * d)))
    k = bf(rng.standard_normal((1, nh * d)))
    for m, n in [(40, 30), (1000, 990), (32767, 32757)]:
        qm = f(oracle_mod.rope(q, np.array([m], np.int32), nh)[0])
        kn = f(oracle_mod.rope(k, np.array([n], np.int32), nh)[0])
        q10 = f(oracle_mod.rope(q, np.array([m - n], np.int32), nh)[0])
        for h in range(nh):
            sl = slice(h * d, (h + 1) * d)
            ref = q10[sl] @ f(k[0, sl])
            scale = np.linalg.norm(f(q[0, sl])) * np.linalg.norm(f(k[0, sl]))
            assert abs(qm[sl] @ kn[sl] - ref) <= 2 ** -7 * scale
