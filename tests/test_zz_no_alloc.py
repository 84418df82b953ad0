"""The allocation-free dense GEMM entry point (dg_fp8_gemm_nt_noalloc), through the C ABI.

It exists for callers that may not allocate device memory during a call (for example code running under a
global-mode stream capture, where allocation calls are refused, or engines whose memory manager owns all of
device memory).  It must give the same results as dg_fp8_gemm_nt; two calls in a row on different inputs check
that the shared static buffer holds nothing stale from the previous call.  This file is collected last.
"""
import ctypes

import pytest
import torch

import synth
from _helpers import assert_close, bf16_to_f64

pytestmark = pytest.mark.gpu


def _call(fn, t, out, p):
    P = ctypes.c_void_p
    return fn(P(t["a"].data_ptr()), P(t["sfa"].data_ptr()), P(t["b"].data_ptr()), P(t["sfb"].data_ptr()),
              P(out.data_ptr()), p.M, p.N, p.K, P(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("M,N,K", [(512, 2048, 1024), (300, 7168, 384), (4096, 7168, 7168)])
def test_noalloc_matches_allocating_entry_point_on_two_calls(M, N, K):
    import moe_grouped_gemm_03_b200 as dg

    L = dg.lib()
    for call, seed in enumerate((M + 1, M + 2)):  # two calls in a row, different inputs and scales
        p = synth.make_dense(M, N, K, seed=seed)
        t = synth.to_torch(p)
        ref = torch.empty(M, N, dtype=torch.bfloat16, device="cuda")
        assert _call(L.dg_fp8_gemm_nt, t, ref, p) == 0, dg.last_error()
        out = torch.full((M, N), float("nan"), dtype=torch.bfloat16, device="cuda")
        assert _call(L.dg_fp8_gemm_nt_noalloc, t, out, p) == 0, dg.last_error()
        dg.check_device_error()
        assert_close(bf16_to_f64(out), bf16_to_f64(ref), f"call {call} of {M}x{N}x{K}")


def test_noalloc_rejects_shapes_beyond_its_buffer():
    import moe_grouped_gemm_03_b200 as dg

    L = dg.lib()
    small = torch.empty(4096, dtype=torch.uint8, device="cuda")  # never read: the call is rejected first
    P = ctypes.c_void_p
    ptr = P(small.data_ptr())
    rc = L.dg_fp8_gemm_nt_noalloc(ptr, ptr, ptr, ptr, ptr, 1 << 20, 7168, 65536,
                                  P(torch.cuda.current_stream().cuda_stream))
    assert rc == -3 and "16777216" in dg.last_error()
