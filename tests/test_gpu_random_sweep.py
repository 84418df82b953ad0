"""A seeded sweep of random shapes through every entry point, each output checked against the oracle.

Shapes are drawn to land on tile edges and just past them: row counts near multiples of 128 and 256 (and 0),
N a multiple of 16 that is seldom a multiple of the tile width, K from one to twelve 128-blocks, group
counts from 1 to 8, and the CTA-pair policy drawn as well. The single-CTA and pair paths, the window tables and
the per-CTA tile lists meet combinations that the fixed cases do not. Two larger cases put more row windows in
the dense and K-grouped launches than one raster group holds (the tile order then has several groups and a
narrower last one); they are checked on sampled rows from every window. A second sweep runs random draws with
fp32 (non-power-of-two) scales through the fp32 promotion path of every call kind.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from _helpers import assert_close, bf16_to_f64, run_problem, untouched_rows_ok

pytestmark = pytest.mark.gpu

KINDS = ["dense", "contiguous", "masked", "nopad", "contiguous_nn", "k_grouped", "contiguous_w4a8", "masked_w4a8"]
EDGE_ROWS = [0, 1, 2, 127, 128, 129, 255, 256, 257, 383, 384, 385]


def _rows(rng, lo=0, hi=520):
    if rng.random() < 0.5:
        return int(rng.choice([r for r in EDGE_ROWS if lo <= r <= hi]))
    return int(rng.integers(lo, hi + 1))


def _draw(case):
    rng = np.random.default_rng(7000 + case)
    kind = KINDS[case % len(KINDS)]
    N = 16 * int(rng.integers(1, 65))  # 16 .. 1024
    K = 128 * int(rng.integers(1, 13))  # 128 .. 1536
    G = int(rng.integers(1, 9))
    seed = 9000 + case
    name = f"sweep{case}-{kind}"
    if kind == "dense":
        return synth.make_dense(max(1, _rows(rng, 1, 700)), N, K, seed=seed, name=name)
    if kind in ("contiguous", "contiguous_nn", "contiguous_w4a8"):
        counts = [_rows(rng) for _ in range(G)]
        if sum(counts) == 0:
            counts[0] = 1
        make = {"contiguous": synth.make_contiguous, "contiguous_nn": synth.make_contiguous_nn,
                "contiguous_w4a8": synth.make_contiguous_w4a8}[kind]
        return make(counts, N, K, seed=seed, name=name)
    if kind == "nopad":
        counts = [_rows(rng) for _ in range(G)]
        return synth.make_nopad(counts, N, K, seed=seed, extra_rows=int(rng.integers(0, 20)), name=name)
    if kind in ("masked", "masked_w4a8"):
        M_max = int(rng.choice([64, 128, 200, 256, 384]))
        mm = [int(rng.integers(0, M_max + 1)) if rng.random() < 0.7 else int(rng.choice([0, M_max])) for _ in range(G)]
        em = int(rng.integers(1, M_max + 1))
        make = synth.make_masked if kind == "masked" else synth.make_masked_w4a8
        return make(G, M_max, N, K, masked_m=mm, seed=seed, expected_m=em, name=name)
    ks = [128 * int(rng.integers(0, 7)) for _ in range(G)]
    if sum(ks) == 0:
        ks[0] = 128
    return synth.make_k_grouped(ks, max(1, _rows(rng, 1, 600)), N, seed=seed, with_c=bool(rng.random() < 0.5),
                                name=name)


@pytest.mark.parametrize("case", range(48))
def test_random_shape(case):
    import moe_grouped_gemm_03_b200 as dg

    p = _draw(case)
    policy, swap = (int(v) for v in np.random.default_rng(case).choice([-1, 0, 1], size=2))
    dg.set_cta_pair_policy(policy)
    dg.set_swap_policy(swap)
    try:
        out = run_problem(p)
        dg.check_device_error()
    finally:
        dg.set_cta_pair_policy(-1)
        dg.set_swap_policy(-1)
    ref = oracle.problem_full(p).reshape(-1, p.N)
    got = bf16_to_f64(out).reshape(-1, p.N)
    valid = ~np.isnan(ref[:, 0])
    assert_close(got[valid], ref[valid], f"{p.name} policy {policy} swap {swap}")
    assert untouched_rows_ok(out, valid), f"{p.name}: rows outside the groups were written"


@pytest.mark.parametrize("case", range(24))
def test_random_shape_fp32_promotion(case):
    """The same draws with every scale given its own fp32 mantissa (no power of two left) and fp32 scale promotion
    on: each call kind's promotion epilogue -- one B scale per 128-column block, per column and K block (K-grouped,
    fp32 D), per column and 32-K sub-block (W4A8) -- against the oracle on random shapes and CTA policies."""
    import moe_grouped_gemm_03_b200 as dg

    p = synth.with_fp32_scales(_draw(100 + case), seed=case)
    policy = int(np.random.default_rng(500 + case).choice([-1, 0, 1]))
    dg.set_cta_pair_policy(policy)
    dg.set_fp32_scale_promotion(True)
    try:
        out = run_problem(p)
        dg.check_device_error()
    finally:
        dg.set_cta_pair_policy(-1)
        dg.set_fp32_scale_promotion(False)
    ref = oracle.problem_full(p).reshape(-1, p.N)
    got = bf16_to_f64(out).reshape(-1, p.N)
    valid = ~np.isnan(ref[:, 0])
    assert_close(got[valid], ref[valid], f"{p.name} (fp32 scales, promotion) policy {policy}")
    assert untouched_rows_ok(out, valid), f"{p.name}: rows outside the groups were written"


def _window_rows(M, window=256):
    """First, middle and last row of every 256-row window (and the last row of M)."""
    rows = []
    for w0 in range(0, M, window):
        rows += [w0, min(M - 1, w0 + 131), min(M - 1, w0 + window - 1)]
    return np.unique(np.array(rows + [M - 1]))


def test_dense_with_several_raster_groups():
    """M = 16500 rows and K = 4096: 65 pair windows, more than one raster group of row windows holds."""
    import moe_grouped_gemm_03_b200 as dg

    p = synth.make_dense(16500, 272, 4096, seed=77, name="dense 16500x272x4096")
    out = run_problem(p)
    dg.check_device_error()
    rows = _window_rows(p.M)
    ref = oracle.problem_rows(p, rows)
    assert_close(bf16_to_f64(out[torch.from_numpy(rows).cuda()]), ref, p.name)


def test_k_grouped_with_several_raster_groups():
    """Two groups of K = 4096 over M = 16400 rows: each group's 65 windows span more than one raster group."""
    import moe_grouped_gemm_03_b200 as dg

    p = synth.make_k_grouped([4096, 4096], 16400, 144, seed=78, with_c=False, name="k-grouped 2x4096 M=16400")
    out = run_problem(p)
    dg.check_device_error()
    base = _window_rows(p.M)
    rows = np.concatenate([base, p.M + base])  # rows of D flattened over the groups
    ref = oracle.problem_rows(p, rows)
    got = out.reshape(-1, p.N)[torch.from_numpy(rows).cuda()]
    assert_close(got.cpu().numpy().astype(np.float64), ref, p.name)
