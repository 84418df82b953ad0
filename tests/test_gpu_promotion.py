"""The fp32 scale-promotion path (any finite fp32 scales) and the power-of-two check of the block-scaled path.

With promotion on, every bf16-output call runs plain e4m3 MMAs into one tensor-memory buffer per 128-K block
and the epilogue warps accumulate buffer * sfa * sfb in fp32; the results must match the oracle, which takes
the scales as given (fp64).  With promotion off (the default), scales must be powers of two: the scale
pre-pass reports any other scale the call reads as DG_ERR_BAD_SCALE, and ignores the scales of rows the call
does not own.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from _helpers import assert_close, bf16_to_f64, run_problem, untouched_rows_ok

pytestmark = pytest.mark.gpu


@pytest.fixture
def promotion():
    import moe_grouped_gemm_03_b200 as dg

    assert dg.set_fp32_scale_promotion(True)
    yield
    dg.set_fp32_scale_promotion(False)


@pytest.fixture(params=[0, 1], ids=["single", "pairs"])
def policy(request):
    import moe_grouped_gemm_03_b200 as dg

    dg.set_cta_pair_policy(request.param)
    yield request.param
    dg.set_cta_pair_policy(-1)


def _full_check(p):
    import moe_grouped_gemm_03_b200 as dg

    out = run_problem(p)
    dg.check_device_error()
    ref = oracle.problem_full(p).reshape(-1, p.N)
    got = bf16_to_f64(out).reshape(-1, p.N)
    valid = ~np.isnan(ref[:, 0])
    assert_close(got[valid], ref[valid], p.name)
    assert untouched_rows_ok(out, valid), "rows outside the groups were written"


CASES = {
    "dense": lambda: synth.make_dense(300, 272, 640, seed=51),  # ragged M and N, five K blocks
    "dense_one_row": lambda: synth.make_dense(1, 16, 128, seed=52),
    "contiguous": lambda: synth.make_contiguous([200, 0, 77, 384], 512, 384, seed=53),
    "masked": lambda: synth.make_masked(5, 200, 384, 512, masked_m=[0, 1, 128, 200, 77], seed=54, expected_m=100),
    "nopad": lambda: synth.make_nopad([130, 0, 257, 5], 256, 256, seed=55, extra_rows=9),
    "nn": lambda: synth.make_contiguous_nn([129, 300], 400, 384, seed=56),
}


@pytest.mark.parametrize("name", list(CASES))
def test_promotion_matches_the_oracle_on_fp32_scales(name, promotion, policy):
    _full_check(synth.with_fp32_scales(CASES[name](), seed=len(name)))


@pytest.mark.parametrize("name", ["dense", "contiguous", "masked"])
def test_promotion_on_power_of_two_scales(name, promotion, policy):
    _full_check(CASES[name]())


def test_promotion_noalloc_call(promotion):
    import moe_grouped_gemm_03_b200 as dg

    p = synth.with_fp32_scales(synth.make_dense(256, 384, 512, seed=57), seed=57)
    t = synth.to_torch(p)
    out = torch.empty(p.out_shape(), dtype=torch.bfloat16, device="cuda")
    dg.fp8_gemm_nt_noalloc((t["a"], t["sfa"]), (t["b"], t["sfb"]), out)
    dg.check_device_error()
    assert_close(bf16_to_f64(out), oracle.problem_full(p), p.name)


def test_promotion_full_size_dense_sampled_rows(promotion):
    """The dense 4096 x 7168 x 7168 workload with fp32 scales, checked on every 256-row window's edges and
    middle rows (all columns)."""
    import moe_grouped_gemm_03_b200 as dg

    p = synth.with_fp32_scales(synth.make_config(2), seed=2)
    out = run_problem(p)
    dg.check_device_error()
    rows = np.unique(np.concatenate([np.arange(0, p.M, 256), np.arange(127, p.M, 256), np.arange(255, p.M, 256),
                                     np.random.default_rng(2).choice(p.M, 64, replace=False)]))
    ref = oracle.problem_rows(p, rows)
    assert_close(bf16_to_f64(out[torch.from_numpy(rows).cuda()]), ref, p.name)


def test_block_scaled_path_reports_non_power_of_two_scales():
    import moe_grouped_gemm_03_b200 as dg

    assert not dg.get_fp32_scale_promotion()
    p = synth.with_fp32_scales(synth.make_dense(128, 256, 256, seed=58), seed=58)
    run_problem(p)
    with pytest.raises(dg.DGError) as e:
        dg.check_device_error()
    assert e.value.status == -7
    dg.check_device_error()  # the word was cleared


def test_scales_of_rows_the_call_does_not_own_are_not_checked():
    """Padding rows (contiguous) and rows past masked_m (masked) may hold any scale: no error, exact results."""
    import moe_grouped_gemm_03_b200 as dg

    p = synth.make_contiguous([100, 300], 256, 384, seed=59)
    p.sfa[:, np.nonzero(p.m_indices < 0)[0]] = 0.3
    _full_check(p)
    q = synth.make_masked(3, 256, 256, 256, masked_m=[10, 0, 256], seed=60, expected_m=128)
    q.sfa[0, :, 10:256] = 0.3
    q.sfa[1, :, :256] = 0.7
    _full_check(q)
    dg.check_device_error()


def test_promotion_refuses_the_k_grouped_and_w4a8_calls(promotion):
    import moe_grouped_gemm_03_b200 as dg

    with pytest.raises(dg.DGError) as e:
        run_problem(synth.make_k_grouped([128, 256], 128, 256, seed=61, with_c=False))
    assert e.value.status == -3
    with pytest.raises(dg.DGError) as e:
        run_problem(synth.make_contiguous_w4a8([129, 40], 256, 256, seed=62))
    assert e.value.status == -3
