"""lm_head_argmax_noalloc: the LM-head greedy choice for callers that cannot
allocate device memory.

Such callers (code inside a host framework that owns every device
allocation, or latency-critical threads that may not take cudaMalloc's locks
and implicit synchronisation) pass only inputs and outputs; the scratch is the
library's built-in 4 MiB device array.  The test calls the entry point
through the C ABI twice in a row and checks each result against the
workspace-based lm_head_argmax on the same inputs (argmax indices: exact)
and against the CPU oracle on the rows whose top-2 gap is not near-tied.
This file is collected last, and it holds no state from other tests: it
passes alone in a fresh process as well as after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

from moe_decoder_speculative_b200 import binding as bd
from moe_decoder_speculative_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from moe_decoder_speculative_b200 import build
    build.build()


def _call_noalloc(h, w_lm, out):
    T, H = h.shape
    V = w_lm.shape[0]
    L = bd.lib()
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.lm_head_argmax_noalloc(ctypes.c_void_p(h.data_ptr()), T, H, ctypes.c_void_p(w_lm.data_ptr()), V,
                                    ctypes.c_void_p(out.data_ptr()), stream)


@pytest.mark.parametrize("T", [5, 128, 259])
def test_noalloc_matches_workspace_entry_point_and_oracle_twice(T):
    """Two calls in a row at the model's vocabulary: 5 rows (the narrow
    16-row token tiles), 128 rows (the concurrency-32 verify rows, 128-row
    token tiles) and 259 rows (the largest size the 4 MiB scratch holds at
    V = 129,280).  Each call's argmax equals the workspace entry point's on
    every row and the CPU oracle's on every row whose top-2 logit gap is at
    least 1e-2."""
    import oracle
    rng = np.random.default_rng(11 + T)
    H, V = 1280, 129280
    h_np = wl.f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32))
    w_np = wl.f32_to_bf16_bits(rng.standard_normal((V, H)).astype(np.float32) * 0.02)
    h = bd.bf16_to_device(h_np)
    w_lm = bd.bf16_to_device(w_np)
    ref = bd.lm_head_argmax(h, w_lm).cpu().numpy()
    o_am, _, o_gap = oracle.lm_head_argmax(h_np, w_np)
    ok = o_gap >= 1e-2
    assert ok.mean() > 0.5
    for _ in range(2):
        out = torch.full((T,), -7, dtype=torch.int32, device="cuda")
        assert _call_noalloc(h, w_lm, out) == bd.MV_OK, bd.lib().mv_last_error()
        got = out.cpu().numpy()
        np.testing.assert_array_equal(got, ref)
        np.testing.assert_array_equal(got[ok], o_am[ok])
        assert np.all((got >= 0) & (got < V))


def test_noalloc_rejects_sizes_beyond_its_scratch():
    T, H, V = 260, 1280, 129280          # 2020 keys x 260 rows x 8 B + 4352 B > 4 MiB (259 rows fit)
    h = torch.zeros((T, H), dtype=torch.bfloat16, device="cuda")
    w_lm = torch.zeros((8, H), dtype=torch.bfloat16, device="cuda")   # never read: the size check comes first
    out = torch.zeros(T, dtype=torch.int32, device="cuda")
    L = bd.lib()
    st = L.lm_head_argmax_noalloc(ctypes.c_void_p(h.data_ptr()), T, H, ctypes.c_void_p(w_lm.data_ptr()), V,
                                  ctypes.c_void_p(out.data_ptr()), None)
    assert st == 2   # MV_ERR_UNSUPPORTED_SHAPE
    assert b"no-alloc scratch" in L.mv_last_error()
