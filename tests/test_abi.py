"""The C-ABI boundary without a GPU: the library loads, exports every symbol the
header declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

from moe_decoder_speculative_b200 import binding as bd

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_verify.h")

OK, INVALID, SHAPE, MISALIGNED, WS_SMALL, CUDA = 0, 1, 2, 3, 4, 5
A = 1 << 20          # a fake, 16-byte aligned "device address" (never dereferenced on the host)


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^MV_API\s+[\w\s\*]*?\b(\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def L():
    from moe_decoder_speculative_b200 import build
    build.build()
    return bd.lib()


def test_every_declared_symbol_is_exported(L):
    syms = declared_symbols()
    assert len(syms) >= 18
    for s in syms:
        assert hasattr(L, s), f"{s} declared in moe_verify.h but not exported"
    assert sorted(bd.EXPORTED) == syms


def test_version(L):
    assert b"sm_100a" in L.mv_version()


def shape(H=128, E=8, I=64, Ish=64, k=2):
    return bd.MoeShape(H, E, I, Ish, k)


def weights(aligned=True, shared=True):
    off = 0 if aligned else 2
    w = bd.MoeWeights(A + off, None, A, A, A, A if shared else None, A if shared else None, A if shared else None)
    return w


def test_router_argument_checks(L):
    s = shape()
    st = None
    assert L.moe_router_topk(None, 4, ctypes.byref(s), A, None, A, A, st) == INVALID
    assert L.moe_router_topk(A + 4, 4, ctypes.byref(s), A, None, A, A, st) == MISALIGNED
    assert L.moe_router_topk(A, -1, ctypes.byref(s), A, None, A, A, st) == INVALID
    bad = shape(H=100)
    assert L.moe_router_topk(A, 4, ctypes.byref(bad), A, None, A, A, st) == SHAPE
    bad = shape(k=9, E=16)
    assert L.moe_router_topk(A, 4, ctypes.byref(bad), A, None, A, A, st) == SHAPE
    bad = shape(k=3, E=2)
    assert L.moe_router_topk(A, 4, ctypes.byref(bad), A, None, A, A, st) == INVALID
    assert L.moe_router_topk(A, 4, None, A, None, A, A, st) == INVALID
    assert L.moe_router_topk(A, 0, ctypes.byref(s), A, None, A, A, st) == OK   # nothing to launch
    assert b"NULL" in L.mv_last_error() or L.mv_last_error() is not None


def test_ffn_argument_checks(L):
    s = shape()
    w = weights()
    need = L.moe_ffn_workspace_size(16, ctypes.byref(s))
    assert need > 0
    assert L.moe_ffn_workspace_size(32, ctypes.byref(s)) > need
    args = lambda x=A, ws_bytes=need, wts=w, out=A + 4096: (x, 16, ctypes.byref(s), ctypes.byref(wts), A, A, None,
                                                            out, A, ws_bytes, None)
    assert L.moe_ffn_forward(*args(ws_bytes=need - 1)) == WS_SMALL
    assert L.moe_ffn_forward(*args(wts=weights(aligned=False))) == MISALIGNED
    assert L.moe_ffn_forward(*args(out=A)) == INVALID                   # out aliases x
    ns = weights(shared=False)
    assert L.moe_ffn_forward(*args(wts=ns)) == INVALID                 # shared expert pointers missing
    s0 = shape(Ish=0)
    assert L.moe_ffn_forward(A, 16, ctypes.byref(s0), ctypes.byref(ns), A, A, None, A + 4096, A,
                             L.moe_ffn_workspace_size(16, ctypes.byref(s0)), None) in (OK, CUDA)


def test_lm_and_accept_argument_checks(L):
    assert L.lm_head_argmax(A, 4, 100, A, 1024, A, A, 1 << 30, None) == SHAPE
    assert L.lm_head_argmax(A, 4, 128, A, 1020, A, A, 1 << 30, None) == SHAPE
    need = L.lm_head_workspace_size(4, 1024)
    assert L.lm_head_argmax(A, 4, 128, A, 1024, A, A, need - 1, None) == WS_SMALL
    assert L.greedy_accept(A, A, 4, 33, A, A, None, None) == INVALID     # K > 32
    assert L.greedy_accept(A, None, 4, 3, A, A, None, None) == INVALID   # drafts needed for K > 0
    assert L.greedy_accept(A, None, 0, 3, None, None, None, None) == OK  # B = 0
    assert L.greedy_accept(A + 8, A, 4, 3, A, A, None, None) == MISALIGNED


def test_verify_step_argument_checks(L):
    s = shape()
    w = (bd.MoeWeights * 2)(weights(), weights())
    need = L.verify_step_workspace_size(4, 3, ctypes.byref(s), 1024)
    assert need > L.verify_step_workspace_size(2, 3, ctypes.byref(s), 1024)
    call = lambda **kw: L.verify_step(kw.get("hidden", A), kw.get("drafts", A), kw.get("B", 4), kw.get("K", 3),
                                      ctypes.byref(s), w, kw.get("L", 2), A, kw.get("V", 1024), A, A, None, None, A,
                                      kw.get("ws", need), None)
    assert call(ws=need - 1) == WS_SMALL
    assert call(K=-1) == INVALID
    assert call(V=1001) == SHAPE
    assert call(drafts=None) == INVALID
    assert call(L=-1) == INVALID
    assert call(B=0) == OK
    # a fully valid call on a machine without a GPU fails cleanly at the first CUDA call
    import torch
    if not torch.cuda.is_available():
        assert call() == CUDA
        assert b"" != L.mv_last_error()


def test_timeout_setter_and_launch_counter(L):
    L.mv_set_wait_timeout_ns(1000)
    L.mv_set_wait_timeout_ns(0)      # back to the default
    assert L.mv_launch_count() >= 0
    assert L.mv_kernel_name(0) == b"router_topk"
    assert L.mv_kernel_name(99) is None
