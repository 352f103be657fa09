#!/usr/bin/env python
"""Benchmark of the greedy MoE speculative-verify step on B200.

One step = the whole hot path over one batch: 32 sequences x (K+1 = 4) token
rows through 12 MoE layers (router top-6 of 64 routed experts + 2 shared,
SwiGLU experts, residual combine), the 129,280-token LM-head argmax and greedy
acceptance -- the concurrency-32 decode verify workload (hidden 1280, expert
intermediate 896, shared 1792).  Inputs are seeded synthetic bf16 tensors
(weights N(0, 0.02^2), hidden states N(0, 1)); drafts copy the verifier's own
argmax with probability 0.576, else a uniform token id.

Prints ONE JSON line (rank 0).  `value` = committed tokens (accepted + 1 per
sequence) per second over all ranks, device-timed with CUDA events, inputs
resident in HBM.  `e2e` = the same metric through the public API with the
step's inputs copied from pinned host memory and its results read back inside
the timed region.  Multi-GPU (torchrun): independent replicas, one batch per
rank, no collective on the data path (weak scaling); time = max over ranks.

--impl reference times the CPU oracle (test infrastructure, plain C++ loops)
on the host cores, each step a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import glob
import hashlib
import json
import os
import re
import statistics
import subprocess
import tempfile
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from moe_decoder_speculative_b200 import workloads as wl  # noqa: E402

# The workload's metric name; `value` counts committed tokens (accepted + 1 per
# sequence, the tokens a verify step emits), and `rows_per_s` the verified rows.
METRIC = "verified tokens/s per MoE verify step at 32x(K+1) rows, counted as committed tokens (accepted+1 per sequence)"
UNIT = "committed tokens/s"
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=2, help="workload id (default: concurrency-32 verify)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-prefill", action="store_true",
                    help="leave out the prefill-layer figures the default line carries")
    ap.add_argument("--layers", type=int, default=None,
                    help="run only the first N MoE layers (a smaller case for profiling; not a bench line)")
    ap.add_argument("--graph", action="store_true",
                    help="time replays of the step recorded once as a CUDA graph (verify_graph_*)")
    ap.add_argument("--latency", action="store_true",
                    help="per-step latency of one sequence (batch 1) for K = 0, 1, 3, eager and graph")
    ap.add_argument("--norm", action="store_true",
                    help="the pre-RMSNorm variant of every layer (seeded norm gains)")
    ap.add_argument("--attention", action="store_true",
                    help="the decoder self-attention over the key/value cache alone (decode_attention)")
    ap.add_argument("--spec", action="store_true",
                    help="the draft-and-verify loop step (speculative_step) and the FastMTP draft block alone")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# helpers
# ---------------------------------------------------------------------------

FALLBACK_BF16_TFLOPS = 1590.0


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        try:
            d = json.load(open(p))
            return float(d["hbm_gbs"]), "measured"
        except Exception:
            pass
    return FALLBACK_HBM_GBS, "fallback"


def measured_tensor_peaks():
    """(burst, sustained) dense bf16 TFLOP/s and their source."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        try:
            d = json.load(open(p))
            return float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
        except Exception:
            pass
    return FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def source_digest(files):
    h = hashlib.sha256()
    for f in files:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()[:16]


GEMM_SOURCES = ["moe_decoder_speculative_b200/csrc/gemm_tc.cu", "moe_decoder_speculative_b200/csrc/mv_device.cuh",
                "moe_decoder_speculative_b200/csrc/gemm_params.h"]


def ncu_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from a committed ncu summary, if the
    summary was taken on the current kernel source (else None)."""
    digest = source_digest(GEMM_SOURCES)
    pat = re.compile(r"traffic\[(\w+)\]:\s*bytes_per_launch=(\d+)\s+source=(\w+)")
    for f in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        for line in open(f):
            m = pat.search(line)
            if m and m.group(1) == kernel and m.group(3) == digest:
                return int(m.group(2))
    return None


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"moe_verify_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
            if self.gpu_id:
                cmd += ["-i", self.gpu_id]
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(cmd, stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                rows.append(parts)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows)}


def gpu_uuid(torch, dev):
    try:
        u = torch.cuda.get_device_properties(dev).uuid
        s = str(u)
        return s if s.startswith("GPU-") else "GPU-" + s
    except Exception:
        return None


# ---------------------------------------------------------------------------
# algorithmic bytes (what the method must move per launch)
# ---------------------------------------------------------------------------

def algorithmic_bytes(w, touched, T):
    """Per-launch algorithmic bytes of each kernel kind for one verify step.
    touched[l] = distinct routed experts chosen in layer l.  The grouped MoE
    GEMM streams the touched experts' gate/up/down weights and the shared
    expert once, reads the gathered and plain token rows, writes and re-reads
    the bf16 SwiGLU activations and writes the fp32 expert outputs."""
    H, I, Ish, k, V, E = w.H, w.I, w.I_sh, w.k, w.V, w.E
    n = T * k
    avg_t = float(np.mean(touched)) if len(touched) else 0.0
    act = n * I + T * Ish
    return {
        "grouped_moe_gemm": avg_t * 3 * I * H * 2 + 3 * Ish * H * 2 + (n + T) * H * 2 + 2 * act * 2 + (n + T) * H * 4,
        "lm_head_gemm_argmax": V * H * 2 + T * H * 2 + ((V + 255) // 256 * 4) * T * 8,
        "router_topk": E * H * 2 + T * H * 2 + T * k * 8,
        "expert_permute": n * 4 * 3 + n * H * 2 * 2,
        "combine_unpermute": n * H * 4 + T * H * 4 + T * H * 2 * 2 + n * 12,
        "combine_route": n * H * 4 + T * H * 4 + T * H * 2 * 2 + n * 12 + E * H * 2 + T * k * 8,
    }


def algorithmic_flops(w, T):
    """Per-launch algorithmic flops (2 per multiply-add) of the contracting
    kernels: the routed and shared SwiGLU experts, the LM head, the router."""
    H, I, Ish, k, V, E = w.H, w.I, w.I_sh, w.k, w.V, w.E
    n = T * k
    return {
        "grouped_moe_gemm": 2 * H * (3 * n * I + 3 * T * Ish),
        "lm_head_gemm_argmax": 2 * T * H * V,
        "router_topk": 2 * T * H * E,
        "combine_route": 2 * T * H * E,
    }


def kernel_roofline(avg_s, alg_bytes, alg_flops, hbm_gbs, tc_tflops):
    """The resource that binds a kernel, by its two roofline times (bytes at
    the HBM peak, flops at the bf16 tensor peak), the achieved fraction of that
    peak, and the achieved fraction of the other one."""
    gbs = alg_bytes / avg_s / 1e9
    tfs = alg_flops / avg_s / 1e12
    if alg_flops / (tc_tflops * 1e12) > alg_bytes / (hbm_gbs * 1e9):
        return {"bound": "tensor", "achieved": round(tfs, 1), "peak": tc_tflops, "unit": "TFLOP/s",
                "frac": round(tfs / tc_tflops, 4), "hbm_frac": round(gbs / hbm_gbs, 4)}
    return {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_gbs, "unit": "GB/s",
            "frac": round(gbs / hbm_gbs, 4), "tensor_frac": round(tfs / tc_tflops, 4)}


def step_algorithmic_bytes(w, touched, T):
    H, I, Ish, k, V, E = w.H, w.I, w.I_sh, w.k, w.V, w.E
    per_layer = [t * 3 * I * H * 2 + 3 * Ish * H * 2 + E * H * 2 for t in touched]
    return sum(per_layer) + V * H * 2 + 2 * T * H * 2


# ---------------------------------------------------------------------------
# CPU oracle runs (baseline leg and the reference arm)
# ---------------------------------------------------------------------------

def oracle_step(oracle, w, inp, drafts, S):
    rows = S * (w.K + 1)
    st = oracle.verify_step(inp["hidden"][:rows], drafts[:S], S, w.K, inp["layers"], w.k, inp["w_lm"])
    return int(np.sum(st["accepted"] + 1))


def oracle_single_thread(oracle):
    """Seconds of one oracle verify step on one host thread, for the tiny
    workload and the model-shape batch-1 layer.  It leaves the oracle on one
    thread, so it runs after every other oracle timing."""
    res = {}
    for wid in (0, 1):
        w = wl.workload(wid)
        inp = wl.make_inputs(w)
        drafts = np.zeros((w.B, w.K), np.int32)
        t0 = time.perf_counter()
        oracle.verify_step(inp["hidden"], drafts, w.B, w.K, inp["layers"], w.k, inp["w_lm"], n_threads=1)
        res[w.name] = round(time.perf_counter() - t0, 4)
    return res


def oracle_sample_size(oracle, w, inp, budget_s):
    """Sequences per oracle step so that one step takes about budget_s seconds."""
    t0 = time.perf_counter()
    lay = inp["layers"][0]
    x = inp["hidden"]
    idx, tw, _, _ = oracle.router(x, lay["w_router"], w.k)
    oracle.moe_ffn(x, lay, idx, tw, residual=x)
    t_layer = time.perf_counter() - t0            # one layer on all T rows
    t_full = (w.L + 6.0) * t_layer                # + LM head ~ 6 layers of work per row
    S = w.B if t_full <= budget_s else max(1, int(w.B * budget_s / t_full))
    return S, t_full


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    w = wl.workload(args.workload)
    inp = wl.make_inputs(w)
    # drafts copy the oracle's own argmax (one oracle LM pass on the final h of a short sample)
    S, t_full = oracle_sample_size(oracle, w, inp, budget_s=max(0.5, min(5.0, 150.0 / max(1, args.steps + args.warmup))))
    rows = S * (w.K + 1)
    st = oracle.verify_step(inp["hidden"][:rows], np.zeros((S, w.K), np.int32), S, w.K, inp["layers"], w.k,
                            inp["w_lm"])
    am = np.concatenate([st["argmax"], np.zeros((w.B - S) * (w.K + 1), np.int32)])
    drafts = wl.make_drafts(w, am)
    for _ in range(args.warmup):
        oracle_step(oracle, w, inp, drafts, S)
    t0 = time.perf_counter()
    committed = 0
    for _ in range(args.steps):
        committed += oracle_step(oracle, w, inp, drafts, S)
    dt = time.perf_counter() - t0
    value = committed / dt
    cores = oracle.num_threads()
    sample = f"{S} of {w.B} sequences ({rows} rows) x {w.L} layers + LM head + accept per step"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / max(1, args.steps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic", "config": {"workload": w.name, "B": w.B, "K": w.K, "rows": w.T, "layers": w.L,
                                         "sampled_sequences": S},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def reduce_over_ranks(ms, ms_e2e, committed, device):
    """Replicas report the slowest rank's device time (MAX) and the committed
    tokens of all ranks (SUM); a single process returns its own numbers."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return ms, ms_e2e, committed
    t = torch.tensor([ms, ms_e2e], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    c = torch.tensor([committed], dtype=torch.int64, device=device)
    dist.all_reduce(c, op=dist.ReduceOp.SUM)
    return float(t[0]), float(t[1]), int(c.item())


def run_ours(args):
    import torch
    import torch.distributed as dist

    from moe_decoder_speculative_b200 import binding as bd

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())

    def barrier():
        if world > 1:
            dist.barrier()

    w = wl.workload(args.workload)
    assert w.has_verify, "the benchmark times the verify step"
    side = None
    if rank == 0 and world == 1 and args.workload == 2 and not args.no_prefill and args.layers is None:
        # Figures reported beside the decode step, not part of its value, taken
        # first (their buffers are freed before the step's are made): the
        # prefill-sized MoE layer (8 pages x 1,156 visual tokens, tensor-bound)
        # and the decoder's self-attention over a 4,096-position cache (HBM-bound).
        side = {}
        with ClockSampler(gpu_uuid(torch, dev)) as pclk:
            side["prefill_layer"] = measure_prefill(3, min(args.steps, 50), args.warmup)
        side["prefill_layer"]["clocks"] = pclk.summary()
        with ClockSampler(gpu_uuid(torch, dev)) as aclk:
            side["attention"] = measure_attention(min(args.steps, 50), args.warmup)
        side["attention"]["clocks"] = aclk.summary()
        torch.cuda.empty_cache()
    inp = wl.make_inputs(w, layers=args.layers, norm=args.norm)
    if rank > 0:   # each replica verifies its own batch of sequences
        inp["hidden"] = wl.normal_bf16(np.random.SeedSequence([w.id, rank]), (w.T, w.H), w.x_std)
    shape = bd.shape_of(w)
    layers = [bd.LayerWeights(l, dev) for l in inp["layers"]]
    w_lm = bd.bf16_to_device(inp["w_lm"], dev)
    hidden = bd.bf16_to_device(inp["hidden"], dev)
    plan = bd.VerifyPlan(shape, layers, w_lm, w.B, w.K, dev)
    T = w.T

    # drafts: the verifier's own argmax (one untimed pass) copied with probability p_agree
    zero = torch.zeros((w.B, w.K), dtype=torch.int32, device=dev)
    _, _, _, am = plan(hidden, zero)
    tie_rows = 0
    if w.tie_frac > 0:
        # near-tied LM-head rows built from this first pass's choices, then a second pass
        w_lm_np, rows_t, _ = wl.make_tied_lm_head(w, inp["w_lm"], am.cpu().numpy())
        tie_rows = len(rows_t)
        w_lm = bd.bf16_to_device(w_lm_np, dev)
        plan = bd.VerifyPlan(shape, layers, w_lm, w.B, w.K, dev)
        _, _, _, am = plan(hidden, zero)
    drafts_np = wl.make_drafts(w, am.cpu().numpy())
    drafts = torch.from_numpy(drafts_np).to(dev)

    # touched experts per layer (for the algorithmic byte count) and the hot
    # experts' share of the routing slots, via the public per-step calls
    touched, hot_share = [], []
    hot = torch.from_numpy(wl.hot_experts(w)).to(dev) if w.n_hot else None
    h = hidden
    for lw in layers:
        idx, tw = bd.moe_router_topk(h, shape, lw.t["w_router"], lw.t["router_bias"])
        touched.append(int(torch.unique(idx).numel()))
        if hot is not None:
            hot_share.append(round(float(torch.isin(idx, hot).float().mean().item()), 4))
        h = bd.moe_ffn_forward(h, shape, lw, idx, tw, residual=h)
    plan.sync_status()

    stream = torch.cuda.current_stream()
    step = lambda: plan(hidden, drafts)
    graph = None
    if args.graph:   # the step recorded once; replays read the same (resident) input buffers
        graph = bd.VerifyGraph(plan, hidden, drafts)
        step = graph
    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()
    acc, _, _, _ = step()
    committed_per_step = int((acc + 1).sum().item())

    with ClockSampler(gpu_uuid(torch, dev)) as clocks:
        # ---- headline: device-timed K steps, inputs resident ----
        barrier()
        torch.cuda.synchronize()
        n0 = bd.launch_count()
        ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize()
        barrier()
        launches = bd.launch_count() - n0
        ms = ev0.elapsed_time(ev1)
        plan.sync_status()

        # ---- per-kernel durations: the same K steps with an event pair around every launch ----
        barrier()
        torch.cuda.synchronize()
        bd.profile_enable(True)
        ev2, ev3 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev2.record(stream)
        for _ in range(args.steps):
            plan(hidden, drafts)
        ev3.record(stream)
        torch.cuda.synchronize()
        bd.profile_enable(False)
        kern = bd.profile_collect()
        ms_instr = ev2.elapsed_time(ev3)
        barrier()

        # ---- end to end through the public API with host buffers ----
        # Every step copies its inputs (hidden rows, drafts) from pinned host
        # memory and reads its results (accepted, next token, emitted) back,
        # all inside the timed region.  Two plans (same weights, their own
        # workspaces and result blocks) and two input buffers alternate: after
        # step i a copy stream reads step i's results back in one copy of its
        # plan's contiguous result block and then brings in step i+2's inputs,
        # while step i+1 computes; step i+2 waits for both copies.
        hid_h = torch.from_numpy(inp["hidden"].view(np.int16)).pin_memory()
        dr_h = torch.from_numpy(drafts_np).pin_memory()
        hid_d = [torch.empty_like(hid_h, device=dev) for _ in range(2)]
        dr_d = [torch.empty_like(dr_h, device=dev) for _ in range(2)]
        plans = [plan, bd.VerifyPlan(shape, layers, w_lm, w.B, w.K, dev)]
        if args.graph:
            e2e_graph = [bd.VerifyGraph(plans[i], hid_d[i].view(torch.bfloat16), dr_d[i]) for i in range(2)]
            e2e_step = lambda i: e2e_graph[i]()
        else:
            e2e_graph = None
            e2e_step = lambda i: plans[i](hid_d[i].view(torch.bfloat16), dr_d[i])
        res_h = [torch.empty_like(plan.results, device="cpu").pin_memory() for _ in range(2)]
        copy_stream = torch.cuda.Stream(device=dev)
        in_ready = [torch.cuda.Event() for _ in range(2)]
        step_done = [torch.cuda.Event() for _ in range(2)]

        def h2d(b):  # inputs into buffer b (the copy stream has waited for their last reader)
            with torch.cuda.stream(copy_stream):
                hid_d[b].copy_(hid_h, non_blocking=True)
                dr_d[b].copy_(dr_h, non_blocking=True)
                in_ready[b].record(copy_stream)

        for b in range(2):  # untimed: the second plan's first steps
            h2d(b)
            stream.wait_event(in_ready[b])
            e2e_step(b)
        plans[1].sync_status()
        barrier()
        torch.cuda.synchronize()
        ev4, ev5 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ev4.record(stream)
        copy_stream.wait_stream(stream)
        for b in range(min(2, args.steps)):
            h2d(b)
        for i in range(args.steps):
            b = i % 2
            stream.wait_event(in_ready[b])
            e2e_step(b)
            step_done[b].record(stream)
            with torch.cuda.stream(copy_stream):
                copy_stream.wait_event(step_done[b])
                res_h[b].copy_(plans[b].results, non_blocking=True)
            if i + 2 < args.steps:
                h2d(b)
        stream.wait_stream(copy_stream)
        ev5.record(stream)
        torch.cuda.synchronize()
        ms_e2e = ev4.elapsed_time(ev5)
        barrier()
    clk = clocks.summary()

    ms, ms_e2e, committed_all = reduce_over_ranks(ms, ms_e2e, committed_per_step, dev)

    K = args.steps
    value = committed_all * K / (ms / 1e3)
    e2e_value = committed_all * K / (ms_e2e / 1e3)
    peak, peak_kind = measured_peaks()
    tc_burst, tc_sustained, _ = measured_tensor_peaks()
    alg = algorithmic_bytes(w, touched, T)
    flops = algorithmic_flops(w, T)
    kernels = {}
    for name, d in kern.items():
        if d["launches"] == 0:
            continue
        avg_s = d["ms"] / d["launches"] / 1e3
        entry = {"launches": d["launches"], "avg_us": round(avg_s * 1e6, 3),
                 "share": round(d["ms"] / max(1e-9, sum(x["ms"] for x in kern.values())), 4)}
        if name in alg:
            entry["alg_bytes"] = int(alg[name])
            entry["gbs"] = round(alg[name] / avg_s / 1e9, 1)
        if name in flops:
            entry["tflops"] = round(flops[name] / avg_s / 1e12, 1)
        kernels[name] = entry
    dom = max(kernels, key=lambda n: kern[n]["ms"])
    dom_avg_s = kern[dom]["ms"] / kern[dom]["launches"] / 1e3
    # a kernel timed alone by events: the burst tensor peak
    dom_roof = kernel_roofline(dom_avg_s, alg[dom], flops.get(dom, 0), peak, tc_burst)
    traffic = ncu_traffic(dom)
    step_bytes = step_algorithmic_bytes(w, touched, T)
    step_flops = sum(flops[n] * kern[n]["launches"] for n in flops if n in kern) / max(1, args.steps)
    out = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K, "warmup": args.warmup,
        "ms_per_step": ms / K, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": f"synthetic (seeded bf16 weights N(0,0.02^2), hidden N(0,1); drafts copy the "
                                  f"verifier argmax w.p. {w.p_agree})",
        "config": {"workload": w.name, "B": w.B, "K": w.K, "rows": T, "layers": len(layers), "H": w.H, "E": w.E,
                   "top_k": w.k, "I": w.I, "I_shared": w.I_sh, "V": w.V,
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "launch": "CUDA graph replay (verify_graph_launch)" if args.graph else "eager (verify_step)",
                   "layer": "pre-RMSNorm variant" if args.norm else "residual, no norm",
                   "l2": f"weights ({step_bytes / 1e9:.2f} GB per step) larger than L2: no flush needed"},
        "rows_per_s": world * T * K / (ms / 1e3),
        "committed_per_step": committed_all,
        "step_roofline": {"alg_bytes": int(step_bytes), "achieved_gbs": round(step_bytes / (ms / K / 1e3) / 1e9, 1),
                          "peak_gbs": peak, "frac": round(step_bytes / (ms / K / 1e3) / 1e9 / peak, 4),
                          "alg_flops": int(step_flops),
                          "tensor_frac": round(step_flops / (ms / K / 1e3) / 1e12 / tc_sustained, 4)},
        "roofline": {"kernel": dom, **dom_roof, "peak_source": peak_kind,
                     "traffic": traffic, "alg_bytes_per_launch": int(alg[dom]),
                     "alg_flops_per_launch": int(flops.get(dom, 0))},
        "kernels": kernels,
        "instrumented_ms_per_step": ms_instr / K,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": int(hid_h.numel() * 2 + dr_h.numel() * 4),
                "d2h_bytes_per_step": int(res_h[0].numel() * 4)},
        "gpu_launches": int(launches),
        "clocks": clk,
        "touched_experts": touched,
    }
    if w.n_hot:
        out["skew"] = {"hot_experts": wl.hot_experts(w).tolist(), "router_bias": w.hot_bias,
                       "hot_share_of_slots": hot_share, "tied_lm_rows": tie_rows}

    if side is not None:
        out.update(side)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        oracle.build()
        S, _ = oracle_sample_size(oracle, w, inp, budget_s=20.0)
        t0 = time.perf_counter()
        committed = oracle_step(oracle, w, inp, drafts_np, S)
        dt = time.perf_counter() - t0
        out["cpu_baseline"] = {"value": committed / dt, "unit": UNIT, "cores": oracle.num_threads(),
                               "kind": "oracle",
                               "sample": f"{S} of {w.B} sequences ({S * (w.K + 1)} rows) x {w.L} layers + LM head + "
                                         f"accept, one pass, {dt:.1f} s"}
        out["cpu_baseline"]["single_thread_s_per_step"] = oracle_single_thread(oracle)
    if rank == 0:
        print(json.dumps(out))
    plan = plans = graph = e2e_graph = step = e2e_step = None
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_latency(args):
    """One sequence (batch 1): host-to-result latency of one verify step for
    K = 0, 1, 3 drafts, launched eagerly (verify_step) or as a replay of the
    recorded step (verify_graph_launch).  Each step's device time runs from
    an event recorded before the launch call to one recorded after it, with
    the host synchronised after every step, so launch overhead counts.
    Committed tokens per second = the mean committed tokens per step (drafts
    copy the verifier's own argmax w.p. p, fresh drafts every step) over the
    median step latency."""
    import dataclasses

    import torch

    from moe_decoder_speculative_b200 import binding as bd

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    base = wl.workload(args.workload if args.workload != 2 else 1)
    assert base.has_verify and base.B == 1, "the latency table is for a batch-1 verify workload"
    layers_n = args.layers if args.layers else base.L
    base = dataclasses.replace(base, L=max(base.L, layers_n))   # layer l has the same bytes at any depth
    inp0 = wl.make_inputs(base, layers=layers_n)
    shape = bd.shape_of(base)
    layers = [bd.LayerWeights(l, dev) for l in inp0["layers"]]
    w_lm = bd.bf16_to_device(inp0["w_lm"], dev)
    stream = torch.cuda.current_stream()
    n_steps = max(50, args.steps)
    rows = []
    for K in (0, 1, 3):
        w = dataclasses.replace(base, K=K)
        hidden = bd.bf16_to_device(wl.make_hidden(w), dev)
        plan = bd.VerifyPlan(shape, layers, w_lm, 1, K, dev)
        _, _, _, am = plan(hidden, torch.zeros((1, max(1, K)), dtype=torch.int32, device=dev))
        am = am.cpu().numpy()
        sets = [torch.from_numpy(wl.make_drafts(w, am, ss=np.random.SeedSequence([w.id, K, i]))
                                 if K else np.zeros((1, 1), np.int32)).to(dev) for i in range(n_steps)]
        dr_buf = torch.zeros((1, max(1, K)), dtype=torch.int32, device=dev)
        graph = bd.VerifyGraph(plan, hidden, dr_buf)
        for mode in ("eager", "graph"):
            def one(i):
                if mode == "eager":
                    return plan(hidden, sets[i])
                dr_buf.copy_(sets[i])
                return graph()
            for i in range(max(3, args.warmup)):
                one(i % n_steps)
            torch.cuda.synchronize()
            times, committed = [], 0
            for i in range(n_steps):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                acc, _, _, _ = one(i)
                e1.record(stream)
                e1.synchronize()
                times.append(e0.elapsed_time(e1))
                committed += int(acc[0].item()) + 1
            plan.sync_status()
            lat = float(np.median(times))
            row = {"K": K, "launch": mode, "latency_us": round(lat * 1e3, 2),
                   "p90_us": round(float(np.percentile(times, 90)) * 1e3, 2),
                   "committed_per_step": round(committed / n_steps, 4),
                   "committed_tok_s": round(committed / n_steps / (lat / 1e3), 1),
                   "kernels_per_step": graph.kernels}
            if mode == "eager":   # per-kernel device time of the same steps, one event pair per launch
                bd.profile_enable(True)
                for i in range(n_steps):
                    one(i)
                torch.cuda.synchronize()
                bd.profile_enable(False)
                kern = bd.profile_collect()
                row["kernels_us"] = {k: round(1e3 * v["ms"] / v["launches"], 2) for k, v in kern.items()
                                     if v["launches"]}
            rows.append(row)
        graph.close()
    best = max(rows, key=lambda r: r["committed_tok_s"])
    print(json.dumps({
        "metric": "batch-1 verify latency and committed tokens/s by draft count", "value": best["committed_tok_s"],
        "unit": "tokens/s", "n_gpus": 1, "steps": n_steps, "warmup": args.warmup, "higher_is_better": True,
        "dtype": "bf16", "data": "synthetic (seeded weights; drafts copy the verifier argmax w.p. 0.576)",
        "config": {"workload": base.name, "B": 1, "layers": layers_n, "H": base.H, "E": base.E, "V": base.V},
        "best": best, "table": rows}))
    return 0


def draft_step_bytes(w, B, I_d):
    """Algorithmic bytes of one FastMTP draft step for B rows: the projection,
    the dense SwiGLU and the LM head weights once, the embedding rows, and the
    bf16 rows in and out of each GEMM."""
    H, V = w.H, w.V
    weights = 2 * H * H * 2 + 3 * I_d * H * 2 + V * H * 2
    rows = B * (2 * H * 2 + H * 2 * 4 + I_d * 2 * 2 + H * 2)   # u, z (w+r twice), a (w+r), h'
    return weights + rows + B * H * 2


def run_spec(args):
    """speculative_step on the concurrency-32 workload: one draft-and-verify
    loop iteration (verify_step, then K FastMTP draft-block steps from the
    verifier's state) with inputs resident, and fastmtp_draft alone.  The
    draft block's weights are synthetic, so its drafts rarely match the
    verifier (the committed tokens per iteration are reported as measured)."""
    import torch

    from moe_decoder_speculative_b200 import binding as bd

    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    w = wl.workload(args.workload)
    assert w.has_verify, "a verify workload"
    inp = wl.make_inputs(w, layers=args.layers)
    shape = bd.shape_of(w)
    layers = [bd.LayerWeights(l, dev) for l in inp["layers"]]
    w_lm = bd.bf16_to_device(inp["w_lm"], dev)
    hidden = bd.bf16_to_device(inp["hidden"], dev)
    dw = bd.DraftWeights(wl.make_draft_block(w), dev)
    vplan = bd.VerifyPlan(shape, layers, w_lm, w.B, w.K, dev)
    _, _, _, am = vplan(hidden, torch.zeros((w.B, w.K), dtype=torch.int32, device=dev))
    drafts = torch.from_numpy(wl.make_drafts(w, am.cpu().numpy())).to(dev)
    sp = bd.SpeculativePlan(shape, layers, w_lm, dw, w.B, w.K, dev)
    h0 = hidden[:: w.K + 1].contiguous()
    t0 = am[:: w.K + 1].contiguous()
    dws = bd.workspace(int(bd.lib().fastmtp_draft_workspace_size(w.B, w.K, w.H, dw.I_d, w.V)), dev)
    stream = torch.cuda.current_stream()

    def timed(fn, n):
        for _ in range(max(3, args.warmup)):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n0 = bd.launch_count()
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n, (bd.launch_count() - n0) // n

    n = max(20, args.steps)
    with ClockSampler(gpu_uuid(torch, dev)) as clocks:
        ms_spec, l_spec = timed(lambda: sp(hidden, drafts), n)
        ms_verify, l_verify = timed(lambda: vplan(hidden, drafts), n)
        ms_draft, l_draft = timed(lambda: bd.fastmtp_draft(h0, t0, w.K, dw, w_lm, ws=dws), n)
        bd.profile_enable(True)
        for _ in range(n):
            sp(hidden, drafts)
        torch.cuda.synchronize()
        bd.profile_enable(False)
        kern = bd.profile_collect()
    sp.sync_status()
    bd.sync_status(dws)
    acc = sp.accepted.cpu().numpy()
    nd = sp.next_drafts.cpu().numpy()
    step_bytes = draft_step_bytes(w, w.B, dw.I_d)
    peak, peak_kind = measured_peaks()
    kernels = {k: {"launches": v["launches"], "avg_us": round(1e3 * v["ms"] / v["launches"], 2)}
               for k, v in kern.items() if v["launches"]}
    d_gemm = kern.get("draft_block_gemm", {"ms": 0, "launches": 1})
    d_lm = kern.get("draft_lm_head_argmax", {"ms": 0, "launches": 1})
    draft_bytes = w.K * step_bytes
    print(json.dumps({
        "metric": "draft-and-verify loop iteration (speculative_step) at 32 sequences x K=3",
        "value": ms_spec * 1e3, "unit": "us per iteration", "higher_is_better": False, "n_gpus": 1,
        "steps": n, "warmup": args.warmup, "dtype": "bf16",
        "data": "synthetic (seeded weights; draft block weights random, so its drafts rarely match)",
        "config": {"workload": w.name, "B": w.B, "K": w.K, "layers": len(layers), "I_d": dw.I_d},
        "verify_us": ms_verify * 1e3, "draft_us": ms_draft * 1e3,
        "launches": {"speculative_step": l_spec, "verify_step": l_verify, "fastmtp_draft": l_draft},
        "draft_roofline": {"bound": "hbm", "alg_bytes": int(draft_bytes),
                           "achieved_gbs": round(draft_bytes / (ms_draft / 1e3) / 1e9, 1), "peak_gbs": peak,
                           "frac": round(draft_bytes / (ms_draft / 1e3) / 1e9 / peak, 4), "peak_source": peak_kind},
        "draft_kernels": {"draft_block_gemm_gbs": round((2 * w.H * w.H * 2 + 3 * dw.I_d * w.H * 2) /
                                                        (d_gemm["ms"] / d_gemm["launches"] / 1e3) / 1e9, 1)
                          if d_gemm["ms"] else None,
                          "draft_lm_gbs": round(w.V * w.H * 2 / (d_lm["ms"] / d_lm["launches"] / 1e3) / 1e9, 1)
                          if d_lm["ms"] else None},
        "kernels": kernels, "committed_per_iteration": int((acc + 1).sum()),
        "next_drafts_valid": bool(np.all((nd >= 0) & (nd < w.V))), "clocks": clocks.summary(),
    }))
    return 0


def measure_prefill(wid, steps, warmup):
    """The prefill-sized MoE layer (routing + grouped SwiGLU experts + combine
    over 8 pages x 1,156 visual tokens), device-timed with CUDA events: the
    layer's time and rows/s, and the grouped GEMM's TFLOP/s against the bf16
    tensor peak (burst: a sub-millisecond kernel timed alone by events)."""
    import torch

    from moe_decoder_speculative_b200 import binding as bd

    w = wl.workload(wid)
    inp = wl.make_inputs(w, layers=1)
    shape = bd.shape_of(w)
    lw = bd.LayerWeights(inp["layers"][0])
    x = bd.bf16_to_device(inp["hidden"])
    T = w.T
    ws = bd.workspace(bd.moe_ffn_workspace_size(T, shape))
    idx = torch.empty((T, w.k), dtype=torch.int32, device="cuda")
    tw = torch.empty((T, w.k), dtype=torch.float32, device="cuda")
    out = torch.empty_like(x)

    def step():
        bd.moe_router_topk(x, shape, lw.t["w_router"], lw.t["router_bias"], idx, tw)
        bd.moe_ffn_forward(x, shape, lw, idx, tw, residual=x, out=out, ws=ws)

    for _ in range(max(3, warmup)):
        step()
    torch.cuda.synchronize()
    bd.sync_status(ws)
    touched = int(torch.unique(idx).numel())
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n0 = bd.launch_count()
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    launches = bd.launch_count() - n0
    ms = e0.elapsed_time(e1)
    # per-kernel event times: at most 20 steps (longer event-bracketed passes
    # read 6-8 % high on every prefill kernel while the uninstrumented layer
    # time stays the same)
    bd.profile_enable(True)
    for _ in range(min(steps, 20)):
        step()
    torch.cuda.synchronize()
    bd.profile_enable(False)
    kern = bd.profile_collect()
    bd.sync_status(ws)
    gemm_flops = T * (w.k * 3 * 2 * w.H * w.I + 3 * 2 * w.H * w.I_sh)
    layer_flops = gemm_flops + T * 2 * w.H * w.E
    g = kern.get("grouped_moe_gemm", {"launches": 0, "ms": 0.0})
    gemm_s = g["ms"] / max(1, g["launches"]) / 1e3
    burst, sustained, src = measured_tensor_peaks()
    achieved = gemm_flops / gemm_s / 1e12 if gemm_s > 0 else None
    layer_s = ms / steps / 1e3
    return {
        "workload": w.name, "rows": T, "touched_experts": touched, "ms_per_layer": ms / steps,
        "rows_per_s": T / layer_s, "launches": int(launches),
        "layer_tflops": round(layer_flops / layer_s / 1e12, 1),
        "layer_frac_of_burst": round(layer_flops / layer_s / 1e12 / burst, 4),
        "gemm": {"kernel": "grouped_moe_gemm", "bound": "tensor", "avg_us": round(gemm_s * 1e6, 2),
                 "achieved": round(achieved, 1) if achieved else None, "unit": "TFLOP/s",
                 "peak": burst, "frac": round(achieved / burst, 4) if achieved else None,
                 "peak_sustained": sustained, "frac_of_sustained": round(achieved / sustained, 4) if achieved else None,
                 "peak_source": src, "alg_flops_per_launch": gemm_flops},
        "kernels": {k: {"launches": v["launches"], "avg_us": round(1e3 * v["ms"] / max(1, v["launches"]), 2)}
                    for k, v in kern.items() if v["launches"]},
    }


def measure_attention(steps, warmup, B=32, K=3, n_heads=10, max_ctx=4096):
    """The decoder's self-attention on the verify rows (decode_attention):
    32 sequences x (K+1 = 4) rows, 10 heads of 128, each sequence with 4,096
    cached positions (about 2 pages of 1,156 visual tokens plus their output
    tokens).  HBM-bound: the algorithmic bytes are the visible keys and values
    once, the queries in and the outputs out; inputs (0.67 GB) exceed L2."""
    import torch

    from moe_decoder_speculative_b200 import binding as bd

    HD = 128
    L_max = max_ctx + K + 1
    g = torch.Generator(device="cuda").manual_seed(7)
    q = torch.randn((B * (K + 1), n_heads * HD), device="cuda", generator=g).to(torch.bfloat16)
    kc = torch.randn((B, n_heads, L_max, HD), device="cuda", generator=g).to(torch.bfloat16)
    vc = torch.randn((B, n_heads, L_max, HD), device="cuda", generator=g).to(torch.bfloat16)
    ctx = torch.full((B,), max_ctx, dtype=torch.int32, device="cuda")
    ws = bd.workspace(bd.decode_attention_workspace_size(B, K, n_heads, max_ctx))
    out = torch.empty_like(q)
    for _ in range(max(3, warmup)):
        bd.decode_attention(q, kc, vc, ctx, K, max_ctx, out=out, ws=ws)
    torch.cuda.synchronize()
    bd.sync_status(ws)
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    bd.profile_enable(True)
    e0.record(stream)
    for _ in range(steps):
        bd.decode_attention(q, kc, vc, ctx, K, max_ctx, out=out, ws=ws)
    e1.record(stream)
    torch.cuda.synchronize()
    bd.profile_enable(False)
    kern = bd.profile_collect().get("decode_attention", {"launches": 0, "ms": 0.0})
    bd.sync_status(ws)
    alg = B * n_heads * (max_ctx + K + 1) * HD * 2 * 2 + 2 * q.numel() * 2
    avg_s = kern["ms"] / max(1, kern["launches"]) / 1e3
    peak, src = measured_peaks()
    gbs = alg / avg_s / 1e9 if avg_s > 0 else None
    del q, kc, vc, out, ws
    torch.cuda.empty_cache()
    return {"kernel": "decode_attention", "B": B, "K": K, "n_heads": n_heads, "head_dim": HD,
            "cached_positions": max_ctx, "avg_us": round(avg_s * 1e6, 2), "ms_per_call": e0.elapsed_time(e1) / steps,
            "alg_bytes_per_launch": int(alg), "bound": "hbm", "achieved": round(gbs, 1) if gbs else None,
            "unit": "GB/s", "peak": peak, "peak_source": src, "frac": round(gbs / peak, 4) if gbs else None}


def run_prefill(args):
    """The prefill layer as its own bench line (rows/s)."""
    import torch

    torch.cuda.set_device(0)
    w = wl.workload(args.workload)
    with ClockSampler(gpu_uuid(torch, torch.device("cuda", 0))) as clocks:
        r = measure_prefill(args.workload, args.steps, args.warmup)
    K = args.steps
    print(json.dumps({
        "metric": "prefill MoE layer rows/s (8 pages x 1,156 visual tokens)", "value": r["rows_per_s"],
        "unit": "rows/s", "n_gpus": 1, "steps": K, "warmup": args.warmup, "ms_per_step": r["ms_per_layer"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "rows": w.T, "H": w.H, "E": w.E, "top_k": w.k, "I": w.I, "I_shared": w.I_sh,
                   "touched_experts": r["touched_experts"],
                   "l2": "weights + activations (0.5 GB) larger than L2: no flush needed"},
        "layer_tflops": r["layer_tflops"], "layer_frac_of_burst": r["layer_frac_of_burst"],
        "roofline": r["gemm"], "kernels": r["kernels"],
        "gpu_launches": r["launches"], "clocks": clocks.summary(),
    }))
    return 0


def run_attention(args):
    """The decoder's self-attention on the verify rows as its own bench line."""
    import torch

    torch.cuda.set_device(0)
    with ClockSampler(gpu_uuid(torch, torch.device("cuda", 0))) as clocks:
        r = measure_attention(args.steps, args.warmup)
    print(json.dumps({
        "metric": "decode self-attention of the verify rows over the key/value cache, GB/s", "value": r["achieved"],
        "unit": "GB/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_per_call"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "attention_b32_k3_h10x128_ctx4096", "B": r["B"], "K": r["K"], "n_heads": r["n_heads"],
                   "head_dim": r["head_dim"], "cached_positions": r["cached_positions"],
                   "l2": "cache (0.67 GB) larger than L2: no flush needed"},
        "roofline": {k: r[k] for k in ("kernel", "bound", "achieved", "peak", "unit", "frac", "peak_source",
                                       "alg_bytes_per_launch")},
        "clocks": clocks.summary(),
    }))
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.attention:
        return run_attention(args)
    if args.latency:
        return run_latency(args)
    if args.spec:
        return run_spec(args)
    if not wl.workload(args.workload).has_verify:
        return run_prefill(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
