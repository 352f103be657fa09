"""GPU parity of decode_attention: the decoder's self-attention on the verify
rows over a key/value cache (jina-ocr-v1 model card, architecture paragraph:
a 32,768-position decoder; the head layout is this library's reading).

Against the oracle's float64 definition on the same seeded bf16 inputs.  The
kernel works in fp32 (products of bf16 values, online softmax) and rounds the
output to bf16 once, so an element may differ from the exact value by the
rounding (half a bf16 unit: 2^-9 of its size, a whole unit when the fp32
value sits at a rounding boundary) plus the fp32 error of sums over a few
thousand positions (~1e-6 of the values' size): the bound is
|gpu - ref| <= 2^-8 |ref| + 2^-16 max|v|.
"""
import numpy as np
import pytest
import torch

import oracle
from moe_decoder_speculative_b200 import binding as bd
from moe_decoder_speculative_b200 import workloads as wl

pytestmark = pytest.mark.gpu

HD = 128


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from moe_decoder_speculative_b200 import build
    build.build()


def make_case(seed, B, K, nh, ctx, L_max, poison=True):
    """q, k and v ~ N(0, 1) in bf16; cache positions past ctx[b] + K hold NaN
    bit patterns (poison), which must never reach a result."""
    rng = np.random.default_rng(seed)
    q = wl.f32_to_bf16_bits(rng.standard_normal((B * (K + 1), nh * HD)).astype(np.float32))
    kc = wl.f32_to_bf16_bits(rng.standard_normal((B, nh, L_max, HD)).astype(np.float32))
    vc = wl.f32_to_bf16_bits(rng.standard_normal((B, nh, L_max, HD)).astype(np.float32))
    if poison:
        for b in range(B):
            kc[b, :, ctx[b] + K + 1:] = 0x7FC1
            vc[b, :, ctx[b] + K + 1:] = 0xFFC1
    return q, kc, vc, np.asarray(ctx, np.int32)


def run_gpu(q, kc, vc, ctx, K, max_ctx):
    ws = bd.workspace(bd.decode_attention_workspace_size(kc.shape[0], K, kc.shape[1], max_ctx))
    out = bd.decode_attention(bd.bf16_to_device(q), bd.bf16_to_device(kc), bd.bf16_to_device(vc),
                              torch.from_numpy(ctx).cuda(), K, max_ctx, ws=ws)
    bd.sync_status(ws)
    return wl.bf16_bits_to_f32(bd.bf16_from_device(out)).astype(np.float64), ws


def check(got, ref, vc, ctx, K):
    vmax = 0.0
    for b in range(len(ctx)):
        vmax = max(vmax, float(np.nanmax(np.abs(wl.bf16_bits_to_f32(vc[b, :, :ctx[b] + K + 1])))))
    err = np.abs(got - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -16 * vmax
    assert np.all(np.isfinite(got))
    assert np.all(err <= bound), f"max excess {np.max(err - bound):.3g} at {np.unravel_index(np.argmax(err - bound), err.shape)}"


def test_decode_attention_conc32_rows_over_thousands_of_positions():
    """The concurrency-32 verify rows (32 sequences x K+1 = 4) and the model's
    10 heads over caches of 0 to 4,096 earlier positions (ragged, including
    lengths on split and tile boundaries), with poisoned positions past each
    sequence's rows."""
    B, K, nh = 32, 3, 10
    max_ctx = 4096
    rng = np.random.default_rng(1)
    ctx = rng.integers(0, max_ctx + 1, size=B)
    ctx[:8] = [0, 1, 508, 509, 1020, 1021, 4096, 4092]   # n_keys = 4, 5, 512, 513, 1024 (one whole split), 1025, 4100, 4096
    L_max = max_ctx + K + 1
    q, kc, vc, ctx = make_case(2, B, K, nh, ctx, L_max)
    got, _ = run_gpu(q, kc, vc, ctx, K, max_ctx)
    ref = oracle.decode_attention(q, kc, vc, ctx, K)
    check(got, ref, vc, ctx, K)


@pytest.mark.parametrize("K", [0, 1, 2, 7])
def test_decode_attention_draft_counts(K):
    """K = 0 (plain greedy: one query row), 1, 2 (three rows in a four-row
    tile) and 7 (eight rows), a few sequences and 3 heads."""
    B, nh, max_ctx = 3, 3, 1500
    ctx = np.array([0, 777, 1500])
    q, kc, vc, ctx = make_case(10 + K, B, K, nh, ctx, max_ctx + K + 1 + 37)
    got, _ = run_gpu(q, kc, vc, ctx, K, max_ctx)
    check(got, oracle.decode_attention(q, kc, vc, ctx, K), vc, ctx, K)


def test_decode_attention_is_batch_invariant_and_deterministic():
    """A sequence's rows give the same bits alone or among other sequences
    (and with another max_ctx), and a repeated call gives the same bits."""
    B, K, nh, max_ctx = 6, 3, 2, 3000
    ctx = np.array([2999, 10, 1024, 3000, 640, 1])
    L_max = max_ctx + K + 1
    q, kc, vc, ctx = make_case(20, B, K, nh, ctx, L_max)
    all_rows, _ = run_gpu(q, kc, vc, ctx, K, max_ctx)
    again, _ = run_gpu(q, kc, vc, ctx, K, max_ctx)
    np.testing.assert_array_equal(all_rows, again)
    b = 3
    one, _ = run_gpu(q[b * (K + 1):(b + 1) * (K + 1)], kc[b:b + 1], vc[b:b + 1], ctx[b:b + 1], K, int(ctx[b]))
    np.testing.assert_array_equal(one, all_rows[b * (K + 1):(b + 1) * (K + 1)])


def test_decode_attention_single_position_and_dominant_score():
    """ctx = 0, K = 0: the one visible position is the row's own, so the output
    is its value row rounded to bf16 (exact); a query 1000 e_i against the
    key e_i at one position of a long cache returns that position's value."""
    B, K, nh = 2, 0, 2
    q, kc, vc, ctx = make_case(30, B, K, nh, [0, 0], 8)
    got, _ = run_gpu(q, kc, vc, ctx, K, 0)
    for b in range(B):
        np.testing.assert_array_equal(got[b].reshape(nh, HD), wl.bf16_bits_to_f32(vc[b, :, 0]))
    B, K, nh, max_ctx = 1, 0, 1, 3000
    kc = np.zeros((B, nh, max_ctx + 1, HD), np.uint16)
    vc = wl.f32_to_bf16_bits(np.random.default_rng(31).standard_normal((B, nh, max_ctx + 1, HD)).astype(np.float32))
    q = np.zeros((1, HD), np.uint16)
    q[0, 77] = wl.f32_to_bf16_bits(np.float32([1000.0]))[0]
    kc[0, 0, 2345, 77] = wl.f32_to_bf16_bits(np.float32([1.0]))[0]
    got, _ = run_gpu(q, kc, vc, np.array([max_ctx], np.int32), K, max_ctx)
    np.testing.assert_array_equal(got[0], wl.bf16_bits_to_f32(vc[0, 0, 2345]))


def test_decode_attention_reports_a_context_length_out_of_range():
    """A ctx_len above max_ctx is not read past: that sequence's rows stay as
    they were, mv_sync_status reports MV_ERR_INTERNAL, the others are exact."""
    B, K, nh, max_ctx = 3, 1, 2, 600
    ctx = np.array([100, 600, 50])
    q, kc, vc, ctx = make_case(40, B, K, nh, ctx, max_ctx + K + 1 + 200, poison=False)
    bad = ctx.copy()
    bad[1] = 700                                       # above max_ctx (still inside the cache)
    ws = bd.workspace(bd.decode_attention_workspace_size(B, K, nh, max_ctx))
    out = torch.zeros((B * (K + 1), nh * HD), dtype=torch.bfloat16, device="cuda")
    bd.decode_attention(bd.bf16_to_device(q), bd.bf16_to_device(kc), bd.bf16_to_device(vc),
                        torch.from_numpy(bad).cuda(), K, max_ctx, out=out, ws=ws)
    with pytest.raises(bd.MVError) as exc:
        bd.sync_status(ws)
    assert exc.value.status == 7
    got = wl.bf16_bits_to_f32(bd.bf16_from_device(out)).astype(np.float64)
    assert np.all(got[(K + 1):2 * (K + 1)] == 0)
    ref = oracle.decode_attention(q, kc, vc, ctx, K)
    keep = np.r_[0:K + 1, 2 * (K + 1):3 * (K + 1)]
    check(got[keep], ref[keep], vc, ctx, K)
