"""ctypes binding over libmoe_verify.so (include/moe_verify.h).

Argument marshalling only: every step of the verify path runs in the
library's CUDA kernels.  Tensors are torch CUDA tensors used as plain device
memory (bf16 data may be torch.bfloat16 or any 2-byte dtype holding the bf16
bits); the stream is torch's current stream unless one is given.  There is no
CPU fallback: if the library is not built, the first call raises.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libmoe_verify.so")

MV_OK = 0
STATUS_NAMES = {0: "MV_OK", 1: "MV_ERR_INVALID_ARG", 2: "MV_ERR_UNSUPPORTED_SHAPE", 3: "MV_ERR_MISALIGNED",
                4: "MV_ERR_WORKSPACE_TOO_SMALL", 5: "MV_ERR_CUDA", 6: "MV_ERR_TIMEOUT", 7: "MV_ERR_INTERNAL"}
EXPORTED = ["moe_router_topk", "moe_expert_permute", "moe_ffn_workspace_size", "moe_ffn_forward",
            "lm_head_workspace_size", "lm_head_argmax", "greedy_accept", "verify_step_workspace_size",
            "verify_step", "mv_workspace_init", "mv_sync_status", "mv_last_error", "mv_version",
            "mv_launch_count", "mv_profile_enable", "mv_profile_collect", "mv_kernel_name",
            "mv_set_wait_timeout_ns", "lm_head_argmax_noalloc", "verify_graph_create", "verify_graph_launch",
            "verify_graph_kernels", "verify_graph_destroy", "fastmtp_draft_workspace_size", "fastmtp_draft",
            "speculative_step_workspace_size", "speculative_step", "moe_rmsnorm",
            "decode_attention_workspace_size", "decode_attention"]


class MVError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class MoeShape(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int32), ("E", ctypes.c_int32), ("I", ctypes.c_int32),
                ("I_shared", ctypes.c_int32), ("k", ctypes.c_int32)]


class MoeWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("w_router", "router_bias", "w_gate", "w_up", "w_down",
                                                "ws_gate", "ws_up", "ws_down", "norm_gain")]


DRAFT_KEYS = ("w_emb", "g_hidden", "g_embed", "w_proj", "w_gate", "w_up", "w_down")


class DraftWeightsC(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in DRAFT_KEYS] + [("I_d", ctypes.c_int32)]


_lib = None


def lib():
    """Load the shared library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m moe_decoder_speculative_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        P, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
        S, W = ctypes.POINTER(MoeShape), ctypes.POINTER(MoeWeights)
        sig = {
            "moe_router_topk": (i32, [P, i32, S, P, P, P, P, P]),
            "moe_expert_permute": (i32, [P, i32, i32, i32, P, P, P, P, P]),
            "moe_rmsnorm": (i32, [P, i32, i32, P, P, P]),
            "moe_ffn_workspace_size": (sz, [i32, S]),
            "moe_ffn_forward": (i32, [P, i32, S, W, P, P, P, P, P, sz, P]),
            "lm_head_workspace_size": (sz, [i32, i32]),
            "lm_head_argmax": (i32, [P, i32, i32, P, i32, P, P, sz, P]),
            "lm_head_argmax_noalloc": (i32, [P, i32, i32, P, i32, P, P]),
            "greedy_accept": (i32, [P, P, i32, i32, P, P, P, P]),
            "verify_step_workspace_size": (sz, [i32, i32, S, i32]),
            "verify_step": (i32, [P, P, i32, i32, S, W, i32, P, i32, P, P, P, P, P, sz, P]),
            "mv_workspace_init": (i32, [P, sz, P]),
            "mv_sync_status": (i32, [P, P]),
            "mv_last_error": (ctypes.c_char_p, []),
            "mv_version": (ctypes.c_char_p, []),
            "mv_launch_count": (ctypes.c_uint64, []),
            "mv_profile_enable": (None, [i32]),
            "mv_profile_collect": (i32, [P, P, i32]),
            "mv_kernel_name": (ctypes.c_char_p, [i32]),
            "mv_set_wait_timeout_ns": (None, [i64]),
            "verify_graph_create": (i32, [P, P, i32, i32, S, W, i32, P, i32, P, P, P, P, P, sz,
                                          ctypes.POINTER(ctypes.c_void_p)]),
            "verify_graph_launch": (i32, [P, P]),
            "verify_graph_kernels": (i32, [P]),
            "verify_graph_destroy": (i32, [P]),
            "fastmtp_draft_workspace_size": (sz, [i32, i32, i32, i32, i32]),
            "fastmtp_draft": (i32, [P, P, i32, i32, i32, ctypes.POINTER(DraftWeightsC), P, i32, P, P, P, sz, P]),
            "speculative_step_workspace_size": (sz, [i32, i32, S, i32, i32]),
            "decode_attention_workspace_size": (sz, [i32, i32, i32, i32]),
            "decode_attention": (i32, [P, P, P, P, i32, i32, i32, i32, i32, i32, P, P, sz, P]),
            "speculative_step": (i32, [P, P, i32, i32, S, W, i32, P, i32, ctypes.POINTER(DraftWeightsC), P, P, P, P,
                                       P, P, sz, P]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(status: int):
    if status != MV_OK:
        raise MVError(status, lib().mv_last_error().decode())


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _shape(H, E, I, I_shared, k):
    return MoeShape(int(H), int(E), int(I), int(I_shared), int(k))


def shape_of(w) -> MoeShape:
    """MoeShape from an object with H, E, I, I_sh, k attributes (e.g. a Workload)."""
    return _shape(w.H, w.E, w.I, w.I_sh, w.k)


# ---------------------------------------------------------------------------
# host <-> device helpers (plumbing)
# ---------------------------------------------------------------------------

def bf16_to_device(a: np.ndarray, device="cuda") -> torch.Tensor:
    """uint16 bf16 bits (numpy) -> torch.bfloat16 tensor on the device."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint16).view(np.int16))
    return t.to(device).view(torch.bfloat16)


def bf16_from_device(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


class LayerWeights:
    """Device copies of one MoE layer's weights plus the C struct pointing at them."""

    def __init__(self, layer: dict, device="cuda"):
        self.t = {}
        for n in ("w_router", "w_gate", "w_up", "w_down", "ws_gate", "ws_up", "ws_down", "norm_gain"):
            v = layer.get(n)
            self.t[n] = None if v is None else (v if isinstance(v, torch.Tensor) else bf16_to_device(v, device))
        b = layer.get("router_bias")
        self.t["router_bias"] = None if b is None else (
            b if isinstance(b, torch.Tensor) else torch.from_numpy(np.ascontiguousarray(b, np.float32)).to(device))
        self.c = MoeWeights(*[None if self.t[n] is None else self.t[n].data_ptr()
                              for n, _ in MoeWeights._fields_])


def moe_rmsnorm(x, gain, out=None, stream=None):
    """bf16((x * s) * gain) per row, s = 1 / sqrt(mean(x^2) + 1e-6) (the
    pre-RMSNorm layer variant's input)."""
    T, H = x.shape
    out = torch.empty_like(x) if out is None else out
    _check(lib().moe_rmsnorm(_p(x), T, H, _p(gain), _p(out), _stream(stream)))
    return out


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """A zero-filled device workspace (its error header starts cleared)."""
    return torch.zeros(max(int(nbytes), 1), dtype=torch.uint8, device=device)


# ---------------------------------------------------------------------------
# the C-ABI calls
# ---------------------------------------------------------------------------

def moe_router_topk(x, shape: MoeShape, w_router, router_bias=None, topk_idx=None, topk_w=None, stream=None):
    T = x.shape[0]
    dev = x.device
    if topk_idx is None:
        topk_idx = torch.empty((T, shape.k), dtype=torch.int32, device=dev)
    if topk_w is None:
        topk_w = torch.empty((T, shape.k), dtype=torch.float32, device=dev)
    _check(lib().moe_router_topk(_p(x), T, ctypes.byref(shape), _p(w_router), _p(router_bias), _p(topk_idx),
                                 _p(topk_w), _stream(stream)))
    return topk_idx, topk_w


def moe_expert_permute(topk_idx, E: int, stream=None):
    T, k = topk_idx.shape
    dev = topk_idx.device
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.empty(max(T * k, 4), dtype=torch.int32, device=dev)
    inv = torch.empty(max(T * k, 4), dtype=torch.int32, device=dev)
    _check(lib().moe_expert_permute(_p(topk_idx), T, E, k, _p(counts), _p(offsets), _p(perm), _p(inv),
                                    _stream(stream)))
    return counts, offsets, perm[:T * k], inv[:T * k]


def moe_ffn_workspace_size(T: int, shape: MoeShape) -> int:
    return int(lib().moe_ffn_workspace_size(T, ctypes.byref(shape)))


def moe_ffn_forward(x, shape: MoeShape, weights: LayerWeights, topk_idx, topk_w, residual=None, out=None,
                    ws=None, stream=None):
    T = x.shape[0]
    if out is None:
        out = torch.empty_like(x)
    if ws is None:
        ws = workspace(moe_ffn_workspace_size(T, shape), x.device)
    _check(lib().moe_ffn_forward(_p(x), T, ctypes.byref(shape), ctypes.byref(weights.c), _p(topk_idx),
                                 _p(topk_w), _p(residual), _p(out), _p(ws), ws.numel(), _stream(stream)))
    return out


def lm_head_workspace_size(T: int, V: int) -> int:
    return int(lib().lm_head_workspace_size(T, V))


def lm_head_argmax(h, w_lm, argmax=None, ws=None, stream=None):
    T, H = h.shape
    V = w_lm.shape[0]
    if argmax is None:
        argmax = torch.empty(T, dtype=torch.int32, device=h.device)
    if ws is None:
        ws = workspace(lm_head_workspace_size(T, V), h.device)
    _check(lib().lm_head_argmax(_p(h), T, H, _p(w_lm), V, _p(argmax), _p(ws), ws.numel(), _stream(stream)))
    return argmax


def lm_head_argmax_noalloc(h, w_lm, argmax=None, stream=None):
    """lm_head_argmax without a workspace: the library's built-in scratch is used."""
    T, H = h.shape
    V = w_lm.shape[0]
    if argmax is None:
        argmax = torch.empty(T, dtype=torch.int32, device=h.device)
    _check(lib().lm_head_argmax_noalloc(_p(h), T, H, _p(w_lm), V, _p(argmax), _stream(stream)))
    return argmax


def greedy_accept(argmax, drafts, B: int, K: int, emitted=True, stream=None):
    dev = argmax.device
    acc = torch.empty(B, dtype=torch.int32, device=dev)
    nxt = torch.empty(B, dtype=torch.int32, device=dev)
    em = torch.empty((B, K + 1), dtype=torch.int32, device=dev) if emitted else None
    _check(lib().greedy_accept(_p(argmax), _p(drafts) if K > 0 else None, B, K, _p(acc), _p(nxt), _p(em),
                               _stream(stream)))
    return acc, nxt, em


def decode_attention_workspace_size(B: int, K: int, n_heads: int, max_ctx: int) -> int:
    return int(lib().decode_attention_workspace_size(B, K, n_heads, max_ctx))


def decode_attention(q, k_cache, v_cache, ctx_len, K: int, max_ctx: int, out=None, ws=None, stream=None):
    """Causal self-attention of the B*(K+1) verify rows q [T][n_heads*128]
    over the cache k_cache / v_cache [B][n_heads][L_max][128] (bf16), with
    ctx_len [B] int32 earlier positions per sequence (device tensor, every
    value <= max_ctx).  Returns out [T][n_heads*128] bf16."""
    B, n_heads, L_max, head_dim = k_cache.shape
    if out is None:
        out = torch.empty((B * (K + 1), n_heads * head_dim), dtype=torch.bfloat16, device=q.device)
    if ws is None:
        ws = workspace(decode_attention_workspace_size(B, K, n_heads, max_ctx), q.device)
    _check(lib().decode_attention(_p(q), _p(k_cache), _p(v_cache), _p(ctx_len), B, K, n_heads, head_dim, L_max,
                                  max_ctx, _p(out), _p(ws), ws.numel(), _stream(stream)))
    return out


def verify_step_workspace_size(B: int, K: int, shape: MoeShape, V: int) -> int:
    return int(lib().verify_step_workspace_size(B, K, ctypes.byref(shape), V))


class VerifyPlan:
    """Keeps the C array of layer structs and a workspace for repeated verify steps."""

    def __init__(self, shape: MoeShape, layers: list, w_lm, B: int, K: int, device="cuda"):
        self.shape, self.layers, self.w_lm, self.B, self.K = shape, layers, w_lm, B, K
        self.V = w_lm.shape[0]
        arr = (MoeWeights * max(1, len(layers)))()
        for i, lw in enumerate(layers):
            arr[i] = lw.c
        self.c_layers = arr
        self.ws = workspace(verify_step_workspace_size(B, K, shape, self.V), device)
        T = B * (K + 1)
        # the per-sequence results side by side in one block (`results`), so
        # that a caller reads them back with one copy; each part starts on a
        # 16-byte boundary, as the C interface requires
        Bp = (B + 3) // 4 * 4
        self.results = torch.empty(2 * Bp + B * (K + 1), dtype=torch.int32, device=device)
        self.accepted = self.results[:B]
        self.next_token = self.results[Bp:Bp + B]
        self.emitted = self.results[2 * Bp:].view(B, K + 1)
        self.argmax = torch.empty(T, dtype=torch.int32, device=device)

    def __call__(self, hidden, drafts, stream=None):
        _check(lib().verify_step(_p(hidden), _p(drafts) if self.K > 0 else None, self.B, self.K,
                                 ctypes.byref(self.shape), self.c_layers, len(self.layers), _p(self.w_lm), self.V,
                                 _p(self.accepted), _p(self.next_token), _p(self.emitted), _p(self.argmax),
                                 _p(self.ws), self.ws.numel(), _stream(stream)))
        return self.accepted, self.next_token, self.emitted, self.argmax

    def sync_status(self, stream=None):
        sync_status(self.ws, stream)


class DraftWeights:
    """Device copies of the FastMTP draft block's weights plus the C struct."""

    def __init__(self, draft: dict, device="cuda"):
        self.t = {n: (draft[n] if isinstance(draft[n], torch.Tensor) else bf16_to_device(draft[n], device))
                  for n in DRAFT_KEYS}
        self.I_d = int(self.t["w_gate"].shape[0])
        self.c = DraftWeightsC(*[self.t[n].data_ptr() for n in DRAFT_KEYS], self.I_d)


def fastmtp_draft(h0, t0, K: int, draft: DraftWeights, w_lm, keep_steps=False, ws=None, stream=None):
    """K recursive draft-block steps from h0 [B][H] (bf16) and t0 [B] (int32).
    Returns drafts int32 [B][K] (and the step outputs bf16 [K][B][H] when
    keep_steps)."""
    B, H = h0.shape
    V = w_lm.shape[0]
    drafts = torch.empty((B, K), dtype=torch.int32, device=h0.device)
    steps = torch.empty((K, B, H), dtype=torch.bfloat16, device=h0.device) if keep_steps else None
    if ws is None:
        ws = workspace(int(lib().fastmtp_draft_workspace_size(B, K, H, draft.I_d, V)), h0.device)
    _check(lib().fastmtp_draft(_p(h0), _p(t0), B, K, H, ctypes.byref(draft.c), _p(w_lm), V, _p(drafts), _p(steps),
                               _p(ws), ws.numel(), _stream(stream)))
    return (drafts, steps) if keep_steps else drafts


class SpeculativePlan:
    """speculative_step: verify_step, then the draft block from the verifier's
    state, giving the next iteration's drafts -- one loop iteration on the GPU."""

    def __init__(self, shape: MoeShape, layers: list, w_lm, draft: DraftWeights, B: int, K: int, device="cuda"):
        self.shape, self.layers, self.w_lm, self.draft, self.B, self.K = shape, layers, w_lm, draft, B, K
        self.V = w_lm.shape[0]
        arr = (MoeWeights * max(1, len(layers)))()
        for i, lw in enumerate(layers):
            arr[i] = lw.c
        self.c_layers = arr
        n = int(lib().speculative_step_workspace_size(B, K, ctypes.byref(shape), draft.I_d, self.V))
        self.ws = workspace(n, device)
        T = B * (K + 1)
        # the per-sequence results side by side in one block (`results`), so
        # that a caller reads them back with one copy; each part starts on a
        # 16-byte boundary, as the C interface requires
        Bp = (B + 3) // 4 * 4
        self.results = torch.empty(2 * Bp + B * (K + 1), dtype=torch.int32, device=device)
        self.accepted = self.results[:B]
        self.next_token = self.results[Bp:Bp + B]
        self.emitted = self.results[2 * Bp:].view(B, K + 1)
        self.argmax = torch.empty(T, dtype=torch.int32, device=device)
        self.next_drafts = torch.empty((B, max(1, K)), dtype=torch.int32, device=device)

    def __call__(self, hidden, drafts, stream=None):
        _check(lib().speculative_step(_p(hidden), _p(drafts) if self.K > 0 else None, self.B, self.K,
                                      ctypes.byref(self.shape), self.c_layers, len(self.layers), _p(self.w_lm),
                                      self.V, ctypes.byref(self.draft.c), _p(self.accepted), _p(self.next_token),
                                      _p(self.emitted), _p(self.argmax), _p(self.next_drafts), _p(self.ws),
                                      self.ws.numel(), _stream(stream)))
        return self.accepted, self.next_token, self.emitted, self.argmax, self.next_drafts

    def sync_status(self, stream=None):
        sync_status(self.ws, stream)


class VerifyGraph:
    """A VerifyPlan's step recorded once as a CUDA graph over fixed input
    buffers (verify_graph_create); each call replays it (verify_graph_launch).
    Write the next step's rows into `hidden` and drafts into `drafts` (in
    place) before a call; the outputs are the plan's output tensors."""

    def __init__(self, plan: VerifyPlan, hidden, drafts=None):
        self.plan, self.hidden = plan, hidden
        self.drafts = drafts if plan.K > 0 else None
        h = ctypes.c_void_p()
        _check(lib().verify_graph_create(_p(hidden), _p(self.drafts), plan.B, plan.K, ctypes.byref(plan.shape),
                                         plan.c_layers, len(plan.layers), _p(plan.w_lm), plan.V, _p(plan.accepted),
                                         _p(plan.next_token), _p(plan.emitted), _p(plan.argmax), _p(plan.ws),
                                         plan.ws.numel(), ctypes.byref(h)))
        self._h = h

    @property
    def kernels(self) -> int:
        return int(lib().verify_graph_kernels(self._h))

    def __call__(self, stream=None):
        _check(lib().verify_graph_launch(self._h, _stream(stream)))
        p = self.plan
        return p.accepted, p.next_token, p.emitted, p.argmax

    def sync_status(self, stream=None):
        self.plan.sync_status(stream)

    def close(self):
        if self._h is not None and self._h.value:
            lib().verify_graph_destroy(self._h)
        self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def verify_step(hidden, drafts, B, K, shape, layers, w_lm, stream=None):
    plan = VerifyPlan(shape, layers, w_lm, B, K, hidden.device)
    return plan(hidden, drafts, stream)


def sync_status(ws, stream=None):
    _check(lib().mv_sync_status(_p(ws), _stream(stream)))


def version() -> str:
    return lib().mv_version().decode()


def launch_count() -> int:
    return int(lib().mv_launch_count())


def set_wait_timeout_ns(ns: int):
    lib().mv_set_wait_timeout_ns(int(ns))


def profile_enable(on: bool):
    lib().mv_profile_enable(1 if on else 0)


def profile_collect() -> dict:
    n = 16
    launches = (ctypes.c_int64 * n)()
    ms = (ctypes.c_double * n)()
    k = lib().mv_profile_collect(launches, ms, n)
    out = {}
    for i in range(k):
        name = lib().mv_kernel_name(i).decode()
        out[name] = {"launches": int(launches[i]), "ms": float(ms[i])}
    return out
