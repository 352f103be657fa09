"""Host-side contracts of the later entry points, without a GPU: the RMSNorm,
the FastMTP draft block, the draft-and-verify step, the no-alloc LM head and
the CUDA-graph handle calls reject bad arguments before any CUDA call, with
the status the header documents."""
import ctypes

import pytest

from moe_decoder_speculative_b200 import binding as bd

OK, INVALID, SHAPE, MISALIGNED, WS_SMALL, CUDA = 0, 1, 2, 3, 4, 5
A = 1 << 20          # a fake, 16-byte aligned "device address" (never dereferenced on the host)
H, V, I_D = 128, 1024, 64


@pytest.fixture(scope="module")
def L():
    from moe_decoder_speculative_b200 import build
    build.build()
    return bd.lib()


def draft(I_d=I_D, aligned=True, missing=None):
    ptrs = [A] * 7
    if not aligned:
        ptrs[3] = A + 2                      # w_proj
    if missing is not None:
        ptrs[missing] = None
    return bd.DraftWeightsC(*ptrs, I_d)


def shape(Hs=H, E=8, I=64, Ish=64, k=2):
    return bd.MoeShape(Hs, E, I, Ish, k)


def test_rmsnorm_checks(L):
    assert L.moe_rmsnorm(A, -1, H, A, A + 4096, None) == INVALID
    assert L.moe_rmsnorm(A, 4, 0, A, A + 4096, None) == INVALID
    assert L.moe_rmsnorm(A, 4, 100, A, A + 4096, None) == SHAPE        # H not a multiple of 8
    assert L.moe_rmsnorm(None, 4, H, A, A + 4096, None) == INVALID
    assert L.moe_rmsnorm(A, 4, H, None, A + 4096, None) == INVALID     # gain is always needed
    assert L.moe_rmsnorm(A + 2, 4, H, A, A + 4096, None) == MISALIGNED
    assert L.moe_rmsnorm(A, 4, H, A, A, None) == INVALID               # out aliases x
    assert b"alias" in L.mv_last_error()


def test_draft_workspace_sizes(L):
    d1 = L.fastmtp_draft_workspace_size(4, 3, H, I_D, V)
    assert d1 > 0
    assert L.fastmtp_draft_workspace_size(8, 3, H, I_D, V) > d1
    assert L.fastmtp_draft_workspace_size(4, 5, H, I_D, V) > d1
    s = shape()
    v = L.verify_step_workspace_size(4, 3, ctypes.byref(s), V)
    assert L.speculative_step_workspace_size(4, 3, ctypes.byref(s), I_D, V) >= v + d1
    assert L.speculative_step_workspace_size(4, 3, None, I_D, V) == 0


def test_fastmtp_draft_checks(L):
    need = L.fastmtp_draft_workspace_size(4, 3, H, I_D, V)

    def call(B=4, K=3, Hs=H, d=None, Vs=V, ws=A, ws_bytes=need, w_lm=A, drafts=A + 8192):
        d = draft() if d is None else d
        return L.fastmtp_draft(A, A + 4096, B, K, Hs, ctypes.byref(d), w_lm, Vs, drafts, None, ws, ws_bytes, None)

    assert call(K=33) == INVALID                          # K <= 32
    assert call(B=-1) == INVALID
    assert call(d=draft(I_d=96)) == SHAPE                  # I_d a multiple of 64
    assert call(Hs=96) == SHAPE                            # H a multiple of 64
    assert call(Vs=1020) == SHAPE                          # V a multiple of 8
    assert call(d=draft(aligned=False)) == MISALIGNED
    assert call(d=draft(missing=0)) == INVALID             # w_emb
    assert call(w_lm=None) == INVALID
    assert call(drafts=None) == INVALID
    assert call(ws=None) == INVALID
    assert call(ws_bytes=need - 1) == WS_SMALL
    assert L.fastmtp_draft(A, A + 4096, 4, 3, H, None, A, V, A + 8192, None, A, need, None) == INVALID
    # nothing to draft: every check passes and nothing is launched
    assert call(B=0, drafts=None, ws_bytes=L.fastmtp_draft_workspace_size(0, 3, H, I_D, V)) == OK
    assert call(K=0, drafts=None, ws_bytes=L.fastmtp_draft_workspace_size(4, 0, H, I_D, V)) == OK


def test_speculative_step_checks(L):
    s = shape()
    w = (bd.MoeWeights * 1)(bd.MoeWeights(A, None, A, A, A, A, A, A))
    d = draft()
    need = L.speculative_step_workspace_size(4, 3, ctypes.byref(s), I_D, V)

    def call(drafts=A, next_drafts=A + 8192, ws_bytes=need, dd=d):
        return L.speculative_step(A, drafts, 4, 3, ctypes.byref(s), w, 1, A, V,
                                  None if dd is None else ctypes.byref(dd), A, A, None, None, next_drafts, A,
                                  ws_bytes, None)

    assert call(next_drafts=A) == INVALID                  # may not alias drafts
    assert call(next_drafts=None) == INVALID               # needed for K > 0
    assert call(ws_bytes=need - 1) == WS_SMALL
    assert call(dd=None) == INVALID
    assert call(dd=draft(I_d=32)) == SHAPE


def test_lm_head_argmax_noalloc_checks(L):
    assert L.lm_head_argmax_noalloc(A, -1, H, A, V, A, None) == INVALID
    assert L.lm_head_argmax_noalloc(A, 4, 100, A, V, A, None) == SHAPE
    assert L.lm_head_argmax_noalloc(A, 4, H, A, 1020, A, None) == SHAPE
    assert L.lm_head_argmax_noalloc(A, 4, H, A, V, None, None) == INVALID
    # the built-in scratch: T <= 259 rows at V = 129,280, as the header states
    big_v = 129280
    assert L.lm_head_argmax_noalloc(A, 260, 1280, A, big_v, A, None) == SHAPE
    assert b"scratch" in L.mv_last_error()
    assert L.lm_head_argmax_noalloc(A, 0, 1280, A, big_v, A, None) == OK    # nothing to launch


def test_graph_handle_calls(L):
    assert L.verify_graph_kernels(None) == -1
    assert L.verify_graph_destroy(None) == OK
    assert L.verify_graph_launch(None, None) == INVALID
    s = shape()
    w = (bd.MoeWeights * 1)(bd.MoeWeights(A, None, A, A, A, A, A, A))
    need = L.verify_step_workspace_size(4, 3, ctypes.byref(s), V)
    args = (A, A, 4, 3, ctypes.byref(s), w, 1, A, V, A, A, None, None, A, need)
    assert L.verify_graph_create(*args, None) == INVALID            # no out-parameter
    g = ctypes.c_void_p(12345)
    L.mv_profile_enable(1)
    try:
        assert L.verify_graph_create(*args, ctypes.byref(g)) == INVALID   # per-launch events cannot be recorded
        assert g.value is None                                            # the handle is cleared on failure
    finally:
        L.mv_profile_enable(0)
    bad = args[:14] + (need - 1,)
    assert L.verify_graph_create(*bad, ctypes.byref(g)) == WS_SMALL


def test_decode_attention_checks(L):
    B, K, nh, L_max, max_ctx = 2, 3, 4, 600, 512
    need = L.decode_attention_workspace_size(B, K, nh, max_ctx)
    assert need > 0
    assert L.decode_attention_workspace_size(B, K, nh, 4 * max_ctx) > need
    assert L.decode_attention_workspace_size(B, 8, nh, max_ctx) == 0          # K + 1 > 8 rows
    ok = dict(q=A, k=A, v=A, ctx=A, B=B, K=K, nh=nh, hd=128, L=L_max, mc=max_ctx, out=A, ws=A, wsb=need)

    def call(**kw):
        a = {**ok, **kw}
        return L.decode_attention(a["q"], a["k"], a["v"], a["ctx"], a["B"], a["K"], a["nh"], a["hd"], a["L"],
                                  a["mc"], a["out"], a["ws"], a["wsb"], None)

    assert call(B=-1) == INVALID
    assert call(nh=0) == INVALID
    assert call(hd=64) == SHAPE                               # head dim 128 only
    assert call(K=8) == SHAPE                                 # at most 7 drafts
    assert call(L=max_ctx + K) == INVALID                     # max_ctx + K + 1 > L_max
    assert b"L_max" in L.mv_last_error()
    assert call(q=None) == INVALID
    assert call(v=None) == INVALID
    assert call(ctx=A + 4) == MISALIGNED
    assert call(out=A + 2) == MISALIGNED
    assert call(wsb=need - 1) == WS_SMALL
    assert call(B=0, q=None, ctx=None, out=None) == OK        # nothing to do, nothing launched
