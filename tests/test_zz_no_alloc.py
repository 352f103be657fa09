"""lm_head_argmax_noalloc: the LM-head greedy choice for callers that cannot
allocate device memory.

Such callers (code inside a host framework that owns every device
allocation, or latency-critical threads that may not take cudaMalloc's locks
and implicit synchronisation) pass only inputs and outputs; the scratch is the
library's built-in 4 MiB device array.  The test calls the entry point
through the C ABI twice in a row and checks each result against the
workspace-based lm_head_argmax on the same inputs (argmax indices: exact).
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


def test_noalloc_matches_workspace_entry_point_twice():
    rng = np.random.default_rng(11)
    T, H, V = 128, 1280, 129280          # the concurrency-32 verify rows and the model's vocabulary
    h = bd.bf16_to_device(wl.f32_to_bf16_bits(rng.standard_normal((T, H)).astype(np.float32)))
    w_lm = bd.bf16_to_device(wl.f32_to_bf16_bits(rng.standard_normal((V, H)).astype(np.float32) * 0.02))
    ref = bd.lm_head_argmax(h, w_lm).cpu().numpy()
    for _ in range(2):
        out = torch.full((T,), -7, dtype=torch.int32, device="cuda")
        assert _call_noalloc(h, w_lm, out) == bd.MV_OK, bd.lib().mv_last_error()
        got = out.cpu().numpy()
        np.testing.assert_array_equal(got, ref)
        assert np.all((got >= 0) & (got < V))


def test_noalloc_rejects_sizes_beyond_its_scratch():
    T, H, V = 300, 1280, 129280          # 2020 keys x 300 rows x 8 B > 4 MiB
    h = torch.zeros((T, H), dtype=torch.bfloat16, device="cuda")
    w_lm = torch.zeros((8, H), dtype=torch.bfloat16, device="cuda")   # never read: the size check comes first
    out = torch.zeros(T, dtype=torch.int32, device="cuda")
    L = bd.lib()
    st = L.lm_head_argmax_noalloc(ctypes.c_void_p(h.data_ptr()), T, H, ctypes.c_void_p(w_lm.data_ptr()), V,
                                  ctypes.c_void_p(out.data_ptr()), None)
    assert st == 2   # MV_ERR_UNSUPPORTED_SHAPE
    assert b"no-alloc scratch" in L.mv_last_error()
