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
    # more than a wave of 128-wide pair tiles (two waves on 74 pairs), every call kind's row tables in play
    "dense_waves": lambda: synth.make_dense(1200, 2048, 640, seed=71),
    "contiguous_waves": lambda: synth.make_contiguous([600, 500], 2048, 512, seed=72),
    "masked_waves": lambda: synth.make_masked(5, 200, 2048, 512, masked_m=[0, 1, 128, 200, 77], seed=73, expected_m=100),
    "nn_waves": lambda: synth.make_contiguous_nn([600, 500], 2048, 384, seed=74),
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


@pytest.mark.parametrize("K", [256, 2176], ids=["one_kernel", "pre_pass"])
def test_block_scaled_path_reports_non_power_of_two_scales(K):
    """Both ways a dense call runs with promotion off check the scales: the short call's single kernel (the
    promotion GEMM's epilogue) and the scale pre-pass of the block-scaled GEMM."""
    import moe_grouped_gemm_03_b200 as dg

    assert not dg.get_fp32_scale_promotion()
    p = synth.with_fp32_scales(synth.make_dense(128, 256, K, seed=58), seed=58)
    run_problem(p)
    with pytest.raises(dg.DGError) as e:
        dg.check_device_error()
    assert e.value.status == -7
    dg.check_device_error()  # the word was cleared


def test_short_dense_call_reads_a_zero_scale_as_the_smallest_exponent():
    """A zero scale is valid on both dense paths (the exponent code 0, 2^-127): no error is raised."""
    import moe_grouped_gemm_03_b200 as dg

    for K in (256, 2176):
        p = synth.make_dense(128, 256, K, seed=59)
        p.sfa[:, 5] = 0.0
        p.sfb[0, 1, 0] = 0.0  # column block 1, K block 0
        out = run_problem(p)
        dg.check_device_error()
        got = bf16_to_f64(out)
        assert np.all(np.abs(got[5]) < 1e-20)  # row 5: every product scaled by 2^-127 (about 6e-39)
        ref = oracle.problem_full(p).reshape(p.M, p.N)
        assert_close(got, ref, p.name)


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


def _k_grouped(p, c_mode, sfb=None):
    """Runs a K-grouped problem; c_mode 'none', 'separate' (C in its own tensor) or 'inplace' (D holds C)."""
    import moe_grouped_gemm_03_b200 as dg

    t = synth.to_torch(p)
    out = torch.full(p.out_shape(), float("nan"), dtype=torch.float32, device="cuda")
    c = None
    if c_mode == "separate":
        c = t["c"]
    elif c_mode == "inplace":
        out.copy_(t["c"])
        c = out
    dg.k_grouped_fp8_gemm_nt_contiguous((t["a"], t["sfa"]), (t["b"], t["sfb"] if sfb is None else sfb), out,
                                        p.counts.tolist(), t["ks"], c)
    dg.check_device_error()
    return out.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("ks,M,N", [
    ([128, 256, 384], 256, 512),
    ([0, 128, 640], 200, 272),    # an empty K range, M and N tails (N not a multiple of the 64-wide tile)
    ([384, 128, 256, 0, 128], 300, 1040),
    ([128], 1, 16),               # one row, narrowest N
])
@pytest.mark.parametrize("c_mode", ["none", "separate", "inplace"])
def test_promotion_k_grouped_matches_the_oracle_on_fp32_scales(ks, M, N, c_mode, promotion, policy):
    """Per-column B scales (one per row of B and K block), each group contracting only its own K blocks, fp32 D
    stored or added; the fp32 output holds the tight bound of the block-scaled K-grouped path."""
    p = synth.with_fp32_scales(synth.make_k_grouped(ks, M, N, seed=sum(ks) + M + N + 7, with_c=c_mode != "none"),
                               seed=M + N)
    got = _k_grouped(p, c_mode)
    ref = oracle.problem_full(p)
    assert_close(got.reshape(-1, N), ref.reshape(-1, N), p.name)
    rms = float(np.sqrt((ref * ref).mean()))
    assert np.abs(got - ref).max() <= 1e-4 * rms + 1e-5 * np.abs(ref).max()


def test_promotion_k_grouped_full_size_sampled(promotion):
    """The K-grouped weight-gradient workload (workload 3's token counts as K extents) with fp32 scales, checked
    on sampled rows of every group."""
    p = synth.with_fp32_scales(synth.make_config(8), seed=8)
    got = _k_grouped(p, "none")
    rng = np.random.default_rng(8)
    rows = np.unique(np.concatenate([[0, p.M - 1], rng.choice(p.M, 24, replace=False)]))
    flat = (np.arange(p.G)[:, None] * p.M + rows[None, :]).ravel()  # rows of the flattened [G * M, N] output
    ref = oracle.problem_rows(p, flat)
    assert_close(got.reshape(-1, p.N)[flat], ref, p.name)


def test_promotion_k_grouped_needs_16_byte_aligned_sfb(promotion):
    import moe_grouped_gemm_03_b200 as dg

    p = synth.with_fp32_scales(synth.make_k_grouped([128, 256], 128, 256, seed=61, with_c=False), seed=61)
    t = synth.to_torch(p)
    flat = torch.zeros(t["sfb"].numel() + 1, dtype=torch.float32, device="cuda")
    shifted = flat[1:].view(t["sfb"].shape)  # 4-byte aligned, not 16
    shifted.copy_(t["sfb"])
    with pytest.raises(dg.DGError) as e:
        _k_grouped(p, "none", sfb=shifted)
    assert e.value.status == -2


W4A8_CASES = {
    "contiguous": lambda: synth.make_contiguous_w4a8([0, 1, 127, 128, 129, 300], 512, 256, seed=63),
    "contiguous_tails": lambda: synth.make_contiguous_w4a8([513, 7, 260], 4112, 384, seed=64),
    "masked": lambda: synth.make_masked_w4a8(5, 200, 256, 512, masked_m=[0, 1, 128, 200, 77], seed=65,
                                             expected_m=100),
    "masked_wide": lambda: synth.make_masked_w4a8(3, 256, 7168, 256, masked_m=[256, 0, 129], seed=66,
                                                  expected_m=128),
}


@pytest.mark.parametrize("name", list(W4A8_CASES))
def test_promotion_w4a8_matches_the_oracle_on_fp32_scales(name, promotion, policy):
    """E2M1 B with one fp32 scale per (row of B, 32-K sub-block): each 32-K MMA writes its own partial, which the
    epilogue scales by sfa(m, kb) * sfb(g, j, n)."""
    _full_check(synth.with_fp32_scales(W4A8_CASES[name](), seed=len(name) + 3))


def test_promotion_w4a8_on_power_of_two_scales(promotion):
    _full_check(W4A8_CASES["contiguous"]())
