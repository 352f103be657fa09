"""bench.py's roofline bookkeeping (CPU): algorithmic flops in closed form, and
each kernel reported against the resource its two roofline times say binds it
(bytes at the HBM peak against flops at the bf16 tensor peak)."""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402
from moe_decoder_speculative_b200 import workloads as wl  # noqa: E402

HBM, TC = 6552.6, 1659.7


def test_flops_closed_forms():
    w = wl.workload(2)
    T = 128
    f = bench.algorithmic_flops(w, T)
    # every row: k routed experts and the shared one, each three H x I contractions
    assert f["grouped_moe_gemm"] == T * (w.k * 6 * w.H * w.I + 6 * w.H * w.I_sh)
    assert f["lm_head_gemm_argmax"] == 2 * T * w.H * w.V
    assert f["router_topk"] == 2 * T * w.H * w.E


def test_fractions_at_the_peaks():
    r = bench.kernel_roofline(1e-3, HBM * 1e6, 0, HBM, TC)  # the peak's bytes in 1 ms
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["frac"] == 1.0 and r["tensor_frac"] == 0
    r = bench.kernel_roofline(1e-3, 0, TC * 1e9, HBM, TC)   # the peak's flops in 1 ms
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s" and r["frac"] == 1.0 and r["hbm_frac"] == 0


def test_lm_head_binds_on_hbm_at_128_rows_and_on_the_tensor_cores_at_512():
    """The LM head streams 331 MB at any row count; its flops grow with the rows
    and pass the HBM time between the two workloads (ridge ~253 flops/byte)."""
    w = wl.workload(2)
    for T, want in [(128, "hbm"), (512, "tensor")]:
        b = bench.algorithmic_bytes(w, [64], T)["lm_head_gemm_argmax"]
        f = bench.algorithmic_flops(w, T)["lm_head_gemm_argmax"]
        assert bench.kernel_roofline(100e-6, b, f, HBM, TC)["bound"] == want


def test_decode_moe_gemm_binds_on_hbm():
    w = wl.workload(2)
    b = bench.algorithmic_bytes(w, [64], 128)["grouped_moe_gemm"]
    f = bench.algorithmic_flops(w, 128)["grouped_moe_gemm"]
    r = bench.kernel_roofline(76.6e-6, b, f, HBM, TC)
    assert r["bound"] == "hbm" and 0.9 < r["frac"] < 0.95 and r["tensor_frac"] < 0.1
