"""Seeded synthetic inputs for the MoE speculative-verify step.

This module is the one piece both the CUDA path and the CPU oracle consume.  It
draws numbers and lays them out; it contains none of the method's arithmetic
(no routing, no expert math, no argmax, no acceptance).  Every tensor is drawn
from numpy's PCG64 generator under a fixed ``SeedSequence`` tree, so the same
workload id always produces the same bytes on any machine.

Shapes follow the jina-ocr-v1 model card (jina.ai/models/jina-ocr-v1),
architecture paragraph: hidden 1280, 64 routed experts plus 2 shared under
top-6 routing, a 129,280-token vocabulary, 12 decoder layers.  The routed
expert intermediate size (896) and the shared one (2 x 896 = 1792) are the
workload definitions' values; the model card gives only the expert counts.

Layout conventions (all bf16 tensors are stored as uint16 bit patterns):
  hidden      [T][H]          row r = b*(K+1) + j, j = 0 current token, 1..K drafts
  w_router    [E][H]
  w_gate      [E][I][H]       w_up the same
  w_down      [E][H][I]
  ws_gate     [I_sh][H]       ws_up the same (the two shared experts concatenated along I)
  ws_down     [H][I_sh]
  w_lm        [V][H]
  drafts      [B][K] int32
"""
from __future__ import annotations

import dataclasses
from concurrent.futures import ThreadPoolExecutor
import os

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "workload", "f32_to_bf16_bits", "bf16_bits_to_f32",
    "normal_bf16", "make_layer", "make_hidden", "make_lm_head", "make_inputs",
    "make_drafts", "hot_experts", "router_bias", "make_draft_block", "layer_seeds",
    "make_tied_lm_head",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: shapes, distributions and seeds."""
    id: int
    name: str
    H: int
    E: int
    k: int
    I: int
    I_sh: int
    V: int          # 0 = no LM head / no verify stage
    B: int          # sequences (verify) ; for prefill B = pages
    K: int          # drafts per sequence (verify); -1 = no verify stage
    L: int          # stacked MoE layers
    T_override: int = 0   # prefill: explicit row count
    x_std: float = 1.0
    w_std: float = 0.02
    p_agree: float = 0.576
    n_hot: int = 0        # skewed routing: number of hot experts
    hot_share: float = 0.0
    hot_bias: float = 0.0  # fp32 router-logit bias on the hot experts (the value the skew script stores)
    tie_frac: float = 0.0  # fraction of rows given near-tied LM logits

    @property
    def T(self) -> int:
        return self.T_override if self.T_override else self.B * (self.K + 1)

    @property
    def has_verify(self) -> bool:
        return self.K >= 0 and self.V > 0


MODEL = dict(H=1280, E=64, k=6, I=896, I_sh=1792, V=129280)

# Router-logit bias on the 4 hot experts of the skewed-routing workload: the
# value stored in tests/golden/skew_router_bias.json by the script beside it,
# which bisects it on the CPU oracle so that the hot experts take 50% of the
# top-6 slots (a CPU test re-runs that bisection and compares).
HOT_BIAS_W4 = 1.625

# The five workloads: a tiny one the oracle finishes in well under a second,
# the batch-1 interactive case, the concurrency-32 decode verify (the headline),
# the 8-page x 1,156-visual-token prefill layer, and the skewed-routing stress.
WORKLOADS = {
    0: Workload(0, "tiny_verify_h128_e8_b4_k3", H=128, E=8, k=2, I=64, I_sh=64, V=1024,
                B=4, K=3, L=1, x_std=0.02, w_std=0.02, p_agree=0.576),
    1: Workload(1, "batch1_verify_b1_k3_l1", **MODEL, B=1, K=3, L=1, p_agree=0.576),
    2: Workload(2, "conc32_verify_b32_k3_l12", **MODEL, B=32, K=3, L=12, p_agree=0.576),
    3: Workload(3, "prefill_moe_t9248_l1", H=1280, E=64, k=6, I=896, I_sh=1792, V=0,
                B=8, K=-1, L=1, T_override=8 * 1156),
    4: Workload(4, "skew_verify_b256_k1_l1", **MODEL, B=256, K=1, L=1, p_agree=0.9,
                n_hot=4, hot_share=0.5, hot_bias=HOT_BIAS_W4, tie_frac=0.05),
}


def workload(wid: int) -> Workload:
    return WORKLOADS[int(wid)]


# ----------------------------------------------------------------------------
# bf16 bit conversion (input encoding only)
# ----------------------------------------------------------------------------

def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16, nearest-even, returned as uint16 bits."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    b = a.view(np.uint32).copy()
    b += ((b >> 16) & 1) + 0x7FFF
    return (b >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


# ----------------------------------------------------------------------------
# seeded draws
# ----------------------------------------------------------------------------

_CHUNK = 1 << 22   # elements per independently-seeded chunk
_POOL = None


def _pool():
    global _POOL
    if _POOL is None:
        _POOL = ThreadPoolExecutor(max(1, min(16, os.cpu_count() or 1)))
    return _POOL


def normal_bf16(ss: np.random.SeedSequence, shape, std: float) -> np.ndarray:
    """N(0, std^2) draws rounded to bf16 bits.

    The flat tensor is cut into fixed chunks of 2^22 elements; chunk c draws from
    ``ss.spawn(n)[c]``, so the bytes do not depend on thread scheduling.
    """
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.uint16)
    nchunks = max(1, (n + _CHUNK - 1) // _CHUNK)
    kids = ss.spawn(nchunks)

    def fill(c):
        lo, hi = c * _CHUNK, min(n, (c + 1) * _CHUNK)
        g = np.random.Generator(np.random.PCG64(kids[c]))
        v = g.standard_normal(hi - lo, dtype=np.float32)
        v *= np.float32(std)
        out[lo:hi] = f32_to_bf16_bits(v)

    list(_pool().map(fill, range(nchunks)))
    return out.reshape(shape)


def _tree(wid: int):
    """Fixed seed tree: root(seed=workload id) -> [hidden, layers, lm_head, drafts, hot, ties,
    draft_block].  (Child i does not depend on how many siblings are spawned.)"""
    root = np.random.SeedSequence(int(wid))
    return root.spawn(7)


def make_layer(w: Workload, layer_ss: np.random.SeedSequence, norm: bool = False) -> dict:
    """One MoE layer's weights, all N(0, w_std^2) in bf16; with norm, also the
    gain of the pre-RMSNorm variant, norm_gain [H] ~ 1 + N(0, 0.1^2)."""
    s = layer_ss.spawn(8)
    H, E, I, Ish = w.H, w.E, w.I, w.I_sh
    d = {
        "w_router": normal_bf16(s[0], (E, H), w.w_std),
        "w_gate": normal_bf16(s[1], (E, I, H), w.w_std),
        "w_up": normal_bf16(s[2], (E, I, H), w.w_std),
        "w_down": normal_bf16(s[3], (E, H, I), w.w_std),
    }
    if Ish > 0:
        d["ws_gate"] = normal_bf16(s[4], (Ish, H), w.w_std)
        d["ws_up"] = normal_bf16(s[5], (Ish, H), w.w_std)
        d["ws_down"] = normal_bf16(s[6], (H, Ish), w.w_std)
    d["router_bias"] = None
    if norm:
        d["norm_gain"] = f32_to_bf16_bits(1.0 + bf16_bits_to_f32(normal_bf16(s[7], (H,), 0.1)))
    return d


def make_hidden(w: Workload) -> np.ndarray:
    return normal_bf16(_tree(w.id)[0], (w.T, w.H), w.x_std)


def make_draft_block(w: Workload, I_d: int | None = None) -> dict:
    """Synthetic weights of the FastMTP draft block, bf16 bits: token embedding
    w_emb [V][H] ~ N(0, 1); RMSNorm gains g_hidden, g_embed [H] ~ 1 + N(0, 0.1^2);
    projection w_proj [H][2H] and a dense SwiGLU FFN (w_gate, w_up [I_d][H],
    w_down [H][I_d]) ~ N(0, w_std^2).  I_d defaults to the shared expert's
    width I_sh."""
    s = _tree(w.id)[6].spawn(7)
    H, Id = w.H, (I_d or w.I_sh)

    def gain(ss):
        return f32_to_bf16_bits(1.0 + bf16_bits_to_f32(normal_bf16(ss, (H,), 0.1)))

    return {
        "w_emb": normal_bf16(s[0], (w.V, H), 1.0),
        "g_hidden": gain(s[1]),
        "g_embed": gain(s[2]),
        "w_proj": normal_bf16(s[3], (H, 2 * H), w.w_std),
        "w_gate": normal_bf16(s[4], (Id, H), w.w_std),
        "w_up": normal_bf16(s[5], (Id, H), w.w_std),
        "w_down": normal_bf16(s[6], (H, Id), w.w_std),
    }


def make_lm_head(w: Workload) -> np.ndarray | None:
    if w.V <= 0:
        return None
    return normal_bf16(_tree(w.id)[2], (w.V, w.H), w.w_std)


def layer_seeds(w: Workload) -> list:
    """The seed sequence of each of the workload's L layers."""
    return _tree(w.id)[1].spawn(w.L)


def make_inputs(w: Workload, layers: int | None = None, norm: bool = False) -> dict:
    """All tensors of a workload except the drafts (which need the verifier's
    argmax) and, for the skewed-routing workload, the near-tied LM-head rows
    (which need the verifier's argmax too: make_tied_lm_head).

    ``layers`` limits how many of the L layers are drawn (for partial tests); the
    layers that are drawn are the same bytes as in the full workload.  With hot
    experts, every layer's router carries the fp32 bias ``w.hot_bias`` on them.
    """
    L = w.L if layers is None else min(layers, w.L)
    layer_ss = layer_seeds(w)
    out = {
        "hidden": make_hidden(w),
        "layers": [make_layer(w, layer_ss[l], norm) for l in range(L)],
        "w_lm": make_lm_head(w),
    }
    if w.n_hot:
        out["hot_experts"] = hot_experts(w)
        out["beta"] = w.hot_bias
        for lay in out["layers"]:
            lay["router_bias"] = router_bias(w, w.hot_bias)
    return out


def make_drafts(w: Workload, verifier_argmax: np.ndarray, p: float | None = None,
                ss: np.random.SeedSequence | None = None) -> np.ndarray:
    """Draft tokens: position i of sequence b copies the verifier's argmax at row
    b*(K+1)+i with probability p, otherwise it is a uniform token id in [0, V)
    (which may, by chance, equal the argmax).

    ``verifier_argmax`` is supplied by the caller; this function only mixes it
    with seeded random draws.
    """
    p = w.p_agree if p is None else p
    ss = _tree(w.id)[3] if ss is None else ss
    g = np.random.Generator(np.random.PCG64(ss))
    B, K, V = w.B, w.K, w.V
    agree = g.random((B, K)) < p
    rand_tok = g.integers(0, V, size=(B, K), dtype=np.int64).astype(np.int32)
    am = np.asarray(verifier_argmax, dtype=np.int32).reshape(B, K + 1)
    return np.where(agree, am[:, :K], rand_tok).astype(np.int32)


def hot_experts(w: Workload) -> np.ndarray:
    """The seeded set of 'hot' experts for the skewed-routing workload."""
    g = np.random.Generator(np.random.PCG64(_tree(w.id)[4]))
    return np.sort(g.choice(w.E, size=w.n_hot, replace=False)).astype(np.int32)


def router_bias(w: Workload, beta: float) -> np.ndarray:
    """fp32 additive router bias: beta on the hot experts, 0 elsewhere."""
    b = np.zeros(w.E, dtype=np.float32)
    b[hot_experts(w)] = np.float32(beta)
    return b


def tie_rng(w: Workload) -> np.random.Generator:
    """Random stream used to choose the rows that get near-tied LM logits."""
    return np.random.Generator(np.random.PCG64(_tree(w.id)[5]))


def make_tied_lm_head(w: Workload, w_lm: np.ndarray, verifier_argmax: np.ndarray):
    """Near-tied LM-head rows for ``w.tie_frac`` of the rows (seeded).

    For each chosen row r, a token v2 that no row chose is given the LM-head
    row of r's choice g: W_lm[v2] := W_lm[g] (an exact tie of the two logits);
    for every other such row one element of W_lm[v2] is then moved by 1-4 bf16
    codes (a gap of ~1e-4).  ``verifier_argmax`` (the choices before the ties)
    is supplied by the caller; this function only copies rows and moves bit
    patterns.  Returns (the new W_lm, the chosen rows, their v2 tokens).
    """
    rng = tie_rng(w)
    g_first = np.asarray(verifier_argmax, dtype=np.int64)
    T = len(g_first)
    n = max(1, int(round(w.tie_frac * T)))
    rows = np.sort(rng.choice(T, size=n, replace=False))
    unused = np.setdiff1d(np.arange(w.V), np.unique(g_first))
    v2s = rng.choice(unused, size=n, replace=False)
    w2 = w_lm.copy()
    for i, (r, v2) in enumerate(zip(rows, v2s)):
        w2[v2] = w_lm[g_first[r]]
        if i % 2:
            while True:   # a normal, finite element: nearby codes stay same-signed and finite
                col = int(rng.integers(0, w.H))
                if 0x0100 <= (int(w2[v2, col]) & 0x7FFF) < 0x7F00:
                    break
            codes = int(rng.integers(1, 5)) * (1 if rng.random() < 0.5 else -1)
            w2[v2, col] = np.uint16(int(w2[v2, col]) + codes)
    return w2, rows, v2s
