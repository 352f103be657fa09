"""Shared helpers for the GPU parity tests: oracle references of each workload,
the flag rules, and the comparisons.

Flag rules (the workloads' parity contract): a row is excused from exact
index/token agreement where the oracle's k-th vs (k+1)-th router logit gap is
below 1e-3 in any layer, or its top-2 LM logit gap is below 1e-2.  MoE
outputs must lie within max-abs 2e-2 x RMS of the oracle's MoE output.
"""
from __future__ import annotations

import functools

import numpy as np

import oracle
from moe_decoder_speculative_b200 import workloads as wl

GATE_GAP = 1e-3
LM_GAP = 1e-2
MOE_TOL = 2e-2


@functools.lru_cache(maxsize=4)
def reference(wid: int, layers: int | None = None):
    """Inputs and the oracle's verify step for a workload (cached)."""
    w = wl.workload(wid)
    inp = wl.make_inputs(w, layers)   # the skewed workload's router bias is part of the inputs
    st = oracle.moe_stack(inp["hidden"], inp["layers"], w.k, keep=True)
    if w.has_verify:
        am, zmax, lm_gap = oracle.lm_head_argmax(st["h"], inp["w_lm"])
        if w.tie_frac > 0:   # near-tied LM rows, built from the oracle's first choices
            inp["w_lm"], inp["tie_rows"], inp["tie_tokens"] = wl.make_tied_lm_head(w, inp["w_lm"], am)
            am, zmax, lm_gap = oracle.lm_head_argmax(st["h"], inp["w_lm"])
        drafts = wl.make_drafts(w, am)
        acc, nxt, em = oracle.greedy_accept(am, drafts, w.B, w.K)
        st.update(argmax=am, lm_gap=lm_gap, drafts=drafts, accepted=acc, next_token=nxt, emitted=em)
    return w, inp, st


def gate_flags(st) -> np.ndarray:
    """Rows flagged by the router gap rule in any layer."""
    f = np.zeros(len(st["h"]), bool)
    for lay in st["layers"]:
        f |= lay["gap"] < GATE_GAP
    return f


def row_flags(st) -> np.ndarray:
    f = gate_flags(st)
    if "lm_gap" in st:
        f |= st["lm_gap"] < LM_GAP
    return f


def moe_error(m_gpu: np.ndarray, m_ref: np.ndarray) -> float:
    """max |gpu - ref| / RMS(ref)."""
    rms = float(np.sqrt(np.mean(m_ref.astype(np.float64) ** 2)))
    return float(np.max(np.abs(m_gpu.astype(np.float64) - m_ref)) / rms)


def drift_excused(st, w_lm, router_ws, gpu_h):
    """Rows excused end to end by input drift.

    Through a stack of layers the GPU's hidden states drift from the oracle's by
    bf16 rounding flips (any change of fp32 summation order does this; the
    oracle's own float and double modes drift the same way).  A routing choice
    at layer l can only differ if the oracle's k-th vs (k+1)-th gap is below
    2 * max_e |dh_l . W_r[e]| (dh_l = GPU input minus oracle input, exact in
    float64), plus the fp32 allowance GATE_GAP; the LM choice likewise with the
    LM-head rows and LM_GAP.  Returns (excused rows, per-layer bound).
    """
    T = len(st["h"])
    ex = np.zeros(T, bool)
    bounds = []
    for l, lay in enumerate(st["layers"]):
        dh = wl.bf16_bits_to_f32(gpu_h[l]).astype(np.float64) - wl.bf16_bits_to_f32(lay["h_in"])
        wr = wl.bf16_bits_to_f32(router_ws[l]).astype(np.float64)
        b = np.max(np.abs(dh @ wr.T), axis=1)
        bounds.append(b)
        ex |= lay["gap"] < GATE_GAP + 2 * b
    dh = wl.bf16_bits_to_f32(gpu_h[-1]).astype(np.float64) - wl.bf16_bits_to_f32(st["h"])
    b_lm = np.zeros(T)
    wlm = wl.bf16_bits_to_f32(w_lm)
    for v0 in range(0, wlm.shape[0], 16384):
        b_lm = np.maximum(b_lm, np.max(np.abs(dh @ wlm[v0:v0 + 16384].astype(np.float64).T), axis=1))
    bounds.append(b_lm)
    ex |= st["lm_gap"] < LM_GAP + 2 * b_lm
    return ex, bounds
