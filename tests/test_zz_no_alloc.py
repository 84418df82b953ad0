"""The allocation-free dense GEMM entry point (dg_fp8_gemm_nt_noalloc), through the C ABI.

It exists for callers that may not allocate device memory during a call (for example code running under a
global-mode stream capture, where allocation calls are refused, or engines whose memory manager owns all of
device memory).  It runs the same kernels on the same tile plan as dg_fp8_gemm_nt, with its packed scales in a
fixed buffer instead of per-call scratch, so its results must equal dg_fp8_gemm_nt's bit for bit; one call is also
checked against the oracle.  Calls in a row on different inputs and scales, a large call followed by a small one
included, check that the shared buffer holds nothing stale from an earlier call.  This file is collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synth
from _helpers import assert_close, bf16_to_f64

pytestmark = pytest.mark.gpu


def _call(fn, t, out, p):
    P = ctypes.c_void_p
    return fn(P(t["a"].data_ptr()), P(t["sfa"].data_ptr()), P(t["b"].data_ptr()), P(t["sfb"].data_ptr()),
              P(out.data_ptr()), p.M, p.N, p.K, P(torch.cuda.current_stream().cuda_stream))


def _both(p):
    """(allocation-free result, dg_fp8_gemm_nt result) on the same inputs, D pre-filled with NaN bits."""
    import moe_grouped_gemm_03_b200 as dg

    L = dg.lib()
    t = synth.to_torch(p)
    out = torch.full((p.M, p.N), float("nan"), dtype=torch.bfloat16, device="cuda")
    assert _call(L.dg_fp8_gemm_nt_noalloc, t, out, p) == 0, dg.last_error()
    ref = torch.full((p.M, p.N), float("nan"), dtype=torch.bfloat16, device="cuda")
    assert _call(L.dg_fp8_gemm_nt, t, ref, p) == 0, dg.last_error()
    dg.check_device_error()
    return out, ref


def _rescaled(p, ja, jb):
    """The same problem with every A scale multiplied by 2^ja and every B scale by 2^jb (still powers of two)."""
    p.sfa = (p.sfa * np.float32(2.0 ** ja)).astype(np.float32)
    p.sfb = (p.sfb * np.float32(2.0 ** jb)).astype(np.float32)
    return p


# (128, 256, 512) is a short call (one kernel, no buffer); the others pack their scales into the buffer
@pytest.mark.parametrize("M,N,K", [(512, 2048, 2560), (300, 7168, 2304), (4096, 7168, 7168), (128, 256, 512)])
def test_noalloc_equals_allocating_entry_point_bit_for_bit_on_two_calls(M, N, K):
    for call, seed in enumerate((M + 1, M + 2)):  # two calls in a row, different inputs and scales
        p = synth.make_dense(M, N, K, seed=seed)
        out, ref = _both(p)
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), f"call {call} of {M}x{N}x{K}"


def test_noalloc_large_then_small_call_matches_oracle():
    """A large call fills much of the shared buffer; the small call after it, with other scales, must read only its
    own packed scales: bit-identical to dg_fp8_gemm_nt and within the tolerance of the oracle."""
    big = _rescaled(synth.make_dense(2048, 7168, 4096, seed=31), 2, -3)
    out, ref = _both(big)
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), "large call"
    small = _rescaled(synth.make_dense(300, 640, 2560, seed=32), -4, 5)  # (K > 2048: packed into the buffer)
    out, ref = _both(small)
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16)), "small call after the large one"
    assert_close(bf16_to_f64(out), oracle.problem_full(small).reshape(small.M, small.N), "small call vs oracle")


def test_noalloc_rejects_shapes_beyond_its_buffer():
    import moe_grouped_gemm_03_b200 as dg

    L = dg.lib()
    small = torch.empty(4096, dtype=torch.uint8, device="cuda")  # never read: the call is rejected first
    P = ctypes.c_void_p
    ptr = P(small.data_ptr())
    rc = L.dg_fp8_gemm_nt_noalloc(ptr, ptr, ptr, ptr, ptr, 1 << 20, 7168, 65536,
                                  P(torch.cuda.current_stream().cuda_stream))
    assert rc == -3 and "16777216" in dg.last_error()
