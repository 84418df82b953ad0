"""The entry points under CUDA graph capture: a captured call replays to the eager result, and replays read the
inputs' current contents (nothing is baked into the graph but pointers and shapes).

Each call enqueues a scale pre-pass and the GEMM as its programmatic dependent, with stream-ordered scratch
(the allocation-free dense call uses its fixed buffer instead), so capture turns them into kernel nodes with a
programmatic edge and memory nodes.
"""
import numpy as np
import pytest
import torch

import synth
from _helpers import run_problem

pytestmark = pytest.mark.gpu


def _capture(fn):
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()  # warm-up on the side stream (first-call setup happens outside the capture)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            fn()
    torch.cuda.current_stream().wait_stream(s)
    return g


@pytest.mark.parametrize("make", [
    lambda: synth.make_dense(384, 1024, 512, seed=31),
    lambda: synth.make_contiguous([200, 77, 384], 1024, 512, seed=32),
    lambda: synth.make_masked(6, 256, 768, 512, seed=33, expected_m=128),
    lambda: synth.make_nopad([130, 0, 257], 512, 256, seed=34),
    lambda: synth.make_contiguous_nn([129, 300], 512, 384, seed=35),
    lambda: synth.make_k_grouped([128, 384], 200, 512, seed=36, with_c=False),
    lambda: synth.make_contiguous_w4a8([129, 300], 512, 256, seed=38),
], ids=["dense", "contiguous", "masked", "nopad", "nn", "k_grouped", "w4a8"])
def test_captured_call_replays_to_eager_result(make):
    import moe_grouped_gemm_03_b200 as dg

    p = make()
    t = synth.to_torch(p)
    eager = run_problem(p, tensors=t).clone()
    dg.check_device_error()
    out = torch.empty_like(eager)
    out.view(torch.int16).fill_(-1)
    graph = _capture(lambda: run_problem(p, tensors=t, out=out))
    graph.replay()
    torch.cuda.synchronize()
    dg.check_device_error()
    assert torch.equal(out.view(torch.int16), eager.view(torch.int16))
    # new operand values through the same graph: a replay reads the inputs' current contents
    t["a"].copy_(torch.roll(t["a"], shifts=1, dims=0))
    eager2 = run_problem(p, tensors=t).clone()
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), eager2.view(torch.int16))
    assert not torch.equal(eager2.view(torch.int16), eager.view(torch.int16))


def test_captured_noalloc_call_replays():
    import moe_grouped_gemm_03_b200 as dg

    p = synth.make_dense(256, 512, 512, seed=37)
    t = synth.to_torch(p)
    eager = torch.empty(p.out_shape(), dtype=torch.bfloat16, device="cuda")
    dg.fp8_gemm_nt_noalloc((t["a"], t["sfa"]), (t["b"], t["sfb"]), eager)
    out = torch.empty_like(eager)
    graph = _capture(lambda: dg.fp8_gemm_nt_noalloc((t["a"], t["sfa"]), (t["b"], t["sfb"]), out))
    graph.replay()
    torch.cuda.synchronize()
    dg.check_device_error()
    assert torch.equal(out, eager)
