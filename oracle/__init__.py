"""CPU oracle for the greedy MoE speculative-verify step (test infrastructure).

Only the tests, the package smoke check and the benchmark's CPU-baseline leg
may import this package.  The product path (the CUDA library and its Python
binding) never imports, links or executes anything here.

The arithmetic lives in ``moe_oracle.cpp`` (plain loops, sequential fp32
accumulation, optional double accumulation); this module only builds that file
with g++ and marshals numpy arrays into it.  ``verify_step`` composes the
per-step functions in the order the method runs them: for every layer the
router then the MoE FFN with residual, then the LM-head argmax, then greedy
acceptance.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "moe_oracle.cpp")
_LIB_PATH = os.path.join(_HERE, "_build", "libmoe_oracle.so")
_lib = None
_lock = threading.Lock()

CXX_FLAGS = ["-std=c++17", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
             "-shared", "-fPIC"]


def build(force: bool = False) -> str:
    """Compile the oracle shared library in-tree (seconds)."""
    os.makedirs(os.path.dirname(_LIB_PATH), exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.check_call(["g++", *CXX_FLAGS, _SRC, "-o", tmp])
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            i = ctypes.c_int
            lib.oracle_router.argtypes = [P, i, i, i, i, P, P, P, P, P, P, i, i, i]
            lib.oracle_moe_ffn.argtypes = [P, i, i, i, i, i, i, P, P, P, P, P, P, P, P, P, P, P, i, i]
            lib.oracle_swiglu.argtypes = [P, i, i, P, P, P, P, P, i]
            lib.oracle_lm_head_argmax.argtypes = [P, i, i, P, i, P, P, P, i, i]
            lib.oracle_greedy_accept.argtypes = [P, P, i, i, P, P, P]
            f32 = ctypes.c_float
            lib.oracle_rmsnorm.argtypes = [P, i, i, P, f32, P, i]
            lib.oracle_fastmtp_draft.argtypes = [P, P, i, i, i, i, i, P, P, P, P, P, P, P, P, f32, P, P, P, i, i]
            lib.oracle_rope.argtypes = [P, i, i, i, P, ctypes.c_double, P]
            lib.oracle_decode_attention.argtypes = [P, P, P, P, i, i, i, i, i, P, i]
            for f in ("oracle_router", "oracle_moe_ffn", "oracle_swiglu",
                      "oracle_lm_head_argmax", "oracle_greedy_accept", "oracle_num_threads",
                      "oracle_rmsnorm", "oracle_fastmtp_draft", "oracle_rope", "oracle_decode_attention"):
                getattr(lib, f).restype = ctypes.c_int
            _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _u16(a):
    return np.ascontiguousarray(a, dtype=np.uint16)


def num_threads() -> int:
    return int(_load().oracle_num_threads())


def router(x, w_router, k, bias=None, weight_form=0, acc_double=False, n_threads=0):
    """Top-k routing of every row of x [T][H] (bf16 bits).

    Returns (idx int32 [T][k], w fp32 [T][k], logits fp32 [T][E], gap fp32 [T])
    where gap is the k-th minus the (k+1)-th largest logit (+inf when k == E).
    """
    x, w_router = _u16(x), _u16(w_router)
    T, H = x.shape
    E = w_router.shape[0]
    idx = np.zeros((T, k), np.int32)
    w = np.zeros((T, k), np.float32)
    logits = np.zeros((T, E), np.float32)
    gap = np.zeros(T, np.float32)
    b = None if bias is None else np.ascontiguousarray(bias, dtype=np.float32)
    rc = _load().oracle_router(_p(x), T, H, E, int(k), _p(w_router), _p(b), _p(idx), _p(w),
                               _p(logits), _p(gap), int(weight_form), int(acc_double),
                               int(n_threads))
    if rc:
        raise ValueError("oracle_router: invalid arguments")
    return idx, w, logits, gap


def moe_ffn(x, layer, idx, w, residual=None, acc_double=False, n_threads=0):
    """One MoE layer given the routing.  Returns (m fp32 [T][H], out bf16 bits [T][H]).

    m is the MoE output (routed mixture plus shared expert); out = bf16(residual + m),
    or bf16(m) when residual is None.
    """
    x = _u16(x)
    T, H = x.shape
    wg, wu, wd = _u16(layer["w_gate"]), _u16(layer["w_up"]), _u16(layer["w_down"])
    E, I, _ = wg.shape
    k = idx.shape[1]
    if layer.get("ws_gate") is not None:
        sg, su, sd = _u16(layer["ws_gate"]), _u16(layer["ws_up"]), _u16(layer["ws_down"])
        Ish = sg.shape[0]
    else:
        sg = su = sd = None
        Ish = 0
    idx = np.ascontiguousarray(idx, np.int32)
    w = np.ascontiguousarray(w, np.float32)
    res = None if residual is None else _u16(residual)
    m = np.zeros((T, H), np.float32)
    out = np.zeros((T, H), np.uint16)
    rc = _load().oracle_moe_ffn(_p(x), T, H, E, I, Ish, k, _p(wg), _p(wu), _p(wd), _p(sg),
                                _p(su), _p(sd), _p(idx), _p(w), _p(res), _p(m), _p(out),
                                int(acc_double), int(n_threads))
    if rc:
        raise ValueError("oracle_moe_ffn: invalid arguments")
    return m, out


def swiglu(x_row, wg, wu, wd, acc_double=False):
    """One expert on one row: returns (a bf16 bits [I], y fp32 [H])."""
    x_row, wg, wu, wd = _u16(x_row), _u16(wg), _u16(wu), _u16(wd)
    H = x_row.shape[0]
    I = wg.shape[0]
    a = np.zeros(I, np.uint16)
    y = np.zeros(H, np.float32)
    rc = _load().oracle_swiglu(_p(x_row), H, I, _p(wg), _p(wu), _p(wd), _p(a), _p(y),
                               int(acc_double))
    if rc:
        raise ValueError("oracle_swiglu: invalid arguments")
    return a, y


def lm_head_argmax(h, w_lm, acc_double=False, n_threads=0):
    """Greedy choice per row.  Returns (argmax int32 [T], zmax fp32 [T], gap fp32 [T])."""
    h, w_lm = _u16(h), _u16(w_lm)
    T, H = h.shape
    V = w_lm.shape[0]
    am = np.zeros(T, np.int32)
    zmax = np.zeros(T, np.float32)
    gap = np.zeros(T, np.float32)
    rc = _load().oracle_lm_head_argmax(_p(h), T, H, _p(w_lm), V, _p(am), _p(zmax), _p(gap),
                                       int(acc_double), int(n_threads))
    if rc:
        raise ValueError("oracle_lm_head_argmax: invalid arguments")
    return am, zmax, gap


def greedy_accept(argmax, drafts, B, K):
    """Returns (accepted [B], next_token [B], emitted [B][K+1], -1 past the kept prefix)."""
    argmax = np.ascontiguousarray(argmax, np.int32)
    d = np.ascontiguousarray(drafts, np.int32) if K > 0 else None
    acc = np.zeros(B, np.int32)
    nxt = np.zeros(B, np.int32)
    em = np.zeros((B, K + 1), np.int32)
    rc = _load().oracle_greedy_accept(_p(argmax), _p(d), B, K, _p(acc), _p(nxt), _p(em))
    if rc:
        raise ValueError("oracle_greedy_accept: invalid arguments")
    return acc, nxt, em


def moe_stack(hidden, layers, k, acc_double=False, n_threads=0, keep=False):
    """Run the stacked MoE layers with a residual: h_{l+1} = bf16(h_l + MoE_l(x_l)).

    x_l = h_l, or, when the layer carries a "norm_gain" (the pre-RMSNorm
    variant of the decoder block), x_l = rmsnorm(h_l, norm_gain): the router
    and the experts see the normalised rows, the residual stays h_l.
    Returns a dict with the final h, and per layer the routing (idx, w), the
    6th-vs-7th logit gap and the MoE output m (when keep=True).
    """
    h = _u16(hidden)
    per_layer = []
    for layer in layers:
        g = layer.get("norm_gain")
        x = h if g is None else rmsnorm(h, g, acc_double=acc_double)
        idx, w, logits, gap = router(x, layer["w_router"], k, bias=layer.get("router_bias"),
                                     acc_double=acc_double, n_threads=n_threads)
        m, h_next = moe_ffn(x, layer, idx, w, residual=h, acc_double=acc_double,
                            n_threads=n_threads)
        rec = {"idx": idx, "w": w, "gap": gap}
        if keep:
            rec.update(h_in=h, m=m, logits=logits, x_in=x)
        per_layer.append(rec)
        h = h_next
    return {"h": h, "layers": per_layer}


def verify_step(hidden, drafts, B, K, layers, k, w_lm, acc_double=False, n_threads=0,
                keep=False):
    """The whole verify step: layers, LM-head argmax, greedy acceptance."""
    st = moe_stack(hidden, layers, k, acc_double=acc_double, n_threads=n_threads, keep=keep)
    am, zmax, lm_gap = lm_head_argmax(st["h"], w_lm, acc_double=acc_double, n_threads=n_threads)
    acc, nxt, em = greedy_accept(am, drafts, B, K)
    st.update(argmax=am, zmax=zmax, lm_gap=lm_gap, accepted=acc, next_token=nxt, emitted=em)
    return st


RMS_EPS = 1e-6   # RMSNorm epsilon of the draft block (a reading; the pages give none)

DRAFT_KEYS = ("w_emb", "g_hidden", "g_embed", "w_proj", "w_gate", "w_up", "w_down")


def rmsnorm(x, gain, eps=RMS_EPS, acc_double=False):
    """RMSNorm of every row of x [T][n] (bf16 bits): bf16((x * r) * gain),
    r = 1 / sqrt(mean(x^2) + eps).  Returns bf16 bits [T][n]."""
    x = _u16(np.atleast_2d(x))
    T, n = x.shape
    g = _u16(gain)
    out = np.zeros_like(x)
    rc = _load().oracle_rmsnorm(_p(x), T, n, _p(g), float(eps), _p(out), int(acc_double))
    if rc:
        raise ValueError("oracle_rmsnorm: invalid arguments")
    return out


def fastmtp_draft(h0, t0, K, draft, w_lm, eps=RMS_EPS, acc_double=False, n_threads=0):
    """K recursive steps of the FastMTP draft block from the verifier's last
    hidden state h0 [B][H] and next token t0 [B].  ``draft`` holds the block's
    weights (DRAFT_KEYS: w_emb [V][H], g_hidden [H], g_embed [H],
    w_proj [H][2H], w_gate [I_d][H], w_up [I_d][H], w_down [H][I_d], bf16 bits).
    Returns {"drafts" int32 [B][K], "h_steps" bf16 [K][B][H], "gaps" fp32 [K][B]}."""
    h0 = _u16(h0)
    B, H = h0.shape
    t0 = np.ascontiguousarray(t0, np.int32)
    w = {k: _u16(draft[k]) for k in DRAFT_KEYS}
    w_lm = _u16(w_lm)
    V = w_lm.shape[0]
    Id = w["w_gate"].shape[0]
    drafts = np.zeros((B, K), np.int32)
    h_steps = np.zeros((K, B, H), np.uint16)
    gaps = np.zeros((K, B), np.float32)
    rc = _load().oracle_fastmtp_draft(_p(h0), _p(t0), B, int(K), H, Id, V, *[_p(w[k]) for k in DRAFT_KEYS],
                                      _p(w_lm), float(eps), _p(drafts), _p(h_steps), _p(gaps),
                                      int(acc_double), int(n_threads))
    if rc:
        raise ValueError("oracle_fastmtp_draft: invalid arguments")
    return {"drafts": drafts, "h_steps": h_steps, "gaps": gaps}


def speculative_step(hidden, drafts, B, K, layers, k, w_lm, draft, eps=RMS_EPS, acc_double=False,
                     n_threads=0):
    """One iteration of the draft-and-verify loop: verify_step on the rows,
    then the draft block from the verifier's final hidden state at each
    sequence's last kept row (row b*(K+1) + accepted[b]) and its next token,
    giving the K drafts of the next iteration."""
    st = verify_step(hidden, drafts, B, K, layers, k, w_lm, acc_double=acc_double, n_threads=n_threads)
    rows = np.arange(B) * (K + 1) + st["accepted"]
    h0 = st["h"][rows]
    nxt = fastmtp_draft(h0, st["next_token"], K, draft, w_lm, eps=eps, acc_double=acc_double,
                        n_threads=n_threads)
    st.update(draft_h0=h0, next_drafts=nxt["drafts"], draft_h_steps=nxt["h_steps"], draft_gaps=nxt["gaps"])
    return st


ROPE_THETA = 10000.0   # rotary base of the decoder's positions (a reading; the pages give none)


def rope(x, pos, n_heads, theta=ROPE_THETA):
    """Rotary position embedding of every row of x [T][n_heads*d] (bf16 bits),
    row r at position pos[r]: pairs (i, i+d/2) of each head turn by
    pos * theta^(-2i/d).  Returns bf16 bits of the same shape."""
    x = _u16(np.atleast_2d(x))
    T, n = x.shape
    d = n // n_heads
    pos = np.ascontiguousarray(pos, np.int32)
    y = np.zeros_like(x)
    rc = _load().oracle_rope(_p(x), T, int(n_heads), d, _p(pos), float(theta), _p(y))
    if rc:
        raise ValueError("oracle_rope: invalid arguments")
    return y


def decode_attention(q, k_cache, v_cache, ctx_len, K, n_threads=0):
    """Causal self-attention of the verify rows over the key/value cache.

    q [B*(K+1)][nh*d] bf16 bits (row r = b*(K+1)+j, position ctx_len[b]+j);
    k_cache, v_cache [B][nh][L_max][d] bf16 bits, holding each sequence's
    earlier positions and this step's K+1 rows; ctx_len [B] int32.
    Returns the outputs [B*(K+1)][nh*d] in float64 (not rounded)."""
    k_cache, v_cache = _u16(k_cache), _u16(v_cache)
    B, nh, L_max, d = k_cache.shape
    q = _u16(q).reshape(B * (K + 1), nh * d)
    ctx = np.ascontiguousarray(ctx_len, np.int32)
    out = np.zeros((B * (K + 1), nh * d), np.float64)
    rc = _load().oracle_decode_attention(_p(q), _p(k_cache), _p(_u16(v_cache)), _p(ctx), B, int(K), nh, d, L_max,
                                         _p(out), int(n_threads))
    if rc:
        raise ValueError("oracle_decode_attention: invalid arguments")
    return out
