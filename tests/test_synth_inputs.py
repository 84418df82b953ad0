"""The seeded generator: exact power-of-two scale choice, e4m3 range, layouts and the workload facts."""
import numpy as np
import pytest
import torch

import synth


def test_scale_exponent_is_smallest_power_of_two_covering_amax():
    amax = np.array([448.0, 448.0001, 447.99, 1.0, 0.875 * 2 ** -3, 3.5, 1e-30, 7e4, 0.0], np.float32)
    e = synth.pow2_scale_exponent(amax)
    for x, ei in zip(amax.astype(np.float64), e):
        if x == 0:
            assert ei == 0
            continue
        assert x <= 448.0 * 2.0 ** ei
        assert x > 448.0 * 2.0 ** (ei - 1)


def test_exact_tie_takes_the_lower_exponent():
    # amax == 448 * 2**e exactly -> that e (ceil(log2) of an exact power of two)
    assert list(synth.pow2_scale_exponent(np.array([448.0, 224.0, 896.0], np.float32))) == [0, -1, 1]


def test_quantised_values_within_range_and_round_to_nearest_even():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((64, 256), dtype=np.float32)
    codes, s = synth.quantize_rows(x)
    deq = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    assert np.isfinite(deq).all() and np.abs(deq).max() <= 448
    amax_q = np.abs(deq.reshape(64, 2, 128)).max(axis=2)
    assert (amax_q > 224 * 0.9).all()  # every block uses the top binade of e4m3
    # each code is the nearest e4m3 value of x/s
    xs = x / np.repeat(s, 128, axis=1)
    err = np.abs(deq - xs)
    assert (err <= np.abs(xs) * 2 ** -4 + 2 ** -10).all()


def test_workload_facts():
    rng = np.random.default_rng(0)
    assert list(rng.integers(1024, 8192, endpoint=True, size=8)) == [7122, 5590, 4688, 2958, 3230, 1317, 1563,
                                                                        1142]
    rng = np.random.default_rng(0)
    mm = rng.integers(0, 256, endpoint=True, size=32)
    assert mm.sum() == 4319 and (mm == 0).sum() == 1 and sum((int(x) + 127) // 128 for x in mm) == 52
    z = synth.zipf_counts(65536, 64, 1.2)
    assert z.sum() == 65536 and z.max() == 19170 and z.min() == 130 and (np.diff(z) <= 0).all()
    assert sum(synth.align_up(int(c), 128) for c in z) == 70016


def test_contiguous_layout():
    p = synth.make_contiguous([3, 128, 129], N=128, K=128, seed=1)
    assert p.rows == 128 + 128 + 256
    mi = p.m_indices
    assert (mi[:3] == 0).all() and (mi[3:128] == -1).all() and (mi[128:256] == 1).all()
    assert (mi[256:385] == 2).all() and (mi[385:] == -1).all()
    assert p.sfa.shape == (1, 512) and p.sfb.shape == (3, 1, 1)
    # garbage rows carry NaN codes
    assert (p.a[3:128, 0] == 0x7F).all()


def test_nopad_layout():
    p = synth.make_nopad([3, 0, 130], N=128, K=256, seed=1, extra_rows=5)
    assert p.rows == 138 and p.sfa.shape == (2, 140) and p.sfb.shape == (3, 1, 2)
    np.testing.assert_array_equal(p.valid_rows(), np.arange(133))
    np.testing.assert_array_equal(p.row_groups(np.array([0, 2, 3, 132])), [0, 0, 2, 2])
    assert (p.a[133:, 0] == 0x7F).all() and p.flops() == 2 * 133 * 128 * 256


def test_contiguous_nn_layout():
    p = synth.make_contiguous_nn([3, 129], N=256, K=384, seed=1)
    q = synth.make_contiguous([3, 129], N=256, K=384, seed=1)
    assert p.b.shape == (2, 384, 256) and p.sfb.shape == (2, 3, 2)
    assert np.array_equal(p.b, q.b.transpose(0, 2, 1)) and np.array_equal(p.sfb, q.sfb.transpose(0, 2, 1))
    assert np.array_equal(p.a, q.a) and np.array_equal(p.m_indices, q.m_indices)


def test_k_grouped_layout():
    p = synth.make_k_grouped([128, 0, 256], M=10, N=20, seed=1)
    assert p.a.shape == (10, 384) and p.b.shape == (20, 384) and p.sfa.shape == (3, 12) and p.sfb.shape == (3, 20)
    assert p.c.shape == (3, 10, 20) and p.out_shape() == (3, 10, 20)
    assert p.flops() == 2 * 10 * 20 * 384


def test_e2m1_quantisation():
    """The B quantiser of the W4A8 inputs: smallest power-of-two scale with amax <= 6 * scale, round to nearest
    on the E2M1 grid with ties to the even code."""
    np.testing.assert_array_equal(synth.pow2_scale_exponent_e2m1(np.array([6.0, 6.01, 3.0, 0.0, 12.0])), [0, 1, -1, 0, 1])
    np.testing.assert_array_equal(synth._to_e2m1_codes(np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, -6.0])),
                                  [0, 2, 2, 4, 4, 6, 6, 15])
    p = synth.make_contiguous_w4a8([3, 129], N=64, K=256, seed=1)
    assert p.b.shape == (2, 64, 128) and p.sfb.shape == (2, 8, 64)


def test_masked_layout():
    p = synth.make_masked(G=2, M_max=10, N=128, K=256, masked_m=[0, 10], seed=1)
    assert p.a.shape == (20, 256) and p.sfa.shape == (2, 2, 12) and p.sfb.shape == (2, 1, 2)
    assert (p.a[:10, 0] == 0x7F).all()
    assert len(p.valid_rows()) == 10 and p.flops() == 2 * 10 * 128 * 256


def test_seeded_determinism():
    a = synth.make_dense(16, 128, 256, seed=3)
    b = synth.make_dense(16, 128, 256, seed=3)
    assert np.array_equal(a.a, b.a) and np.array_equal(a.b, b.b) and np.array_equal(a.sfa, b.sfa)


def test_with_fp32_scales_gives_each_block_its_own_mantissa():
    base = synth.make_contiguous([130, 0, 257], 272, 384, seed=5)
    p = synth.with_fp32_scales(synth.make_contiguous([130, 0, 257], 272, 384, seed=5), seed=5)
    again = synth.with_fp32_scales(synth.make_contiguous([130, 0, 257], 272, 384, seed=5), seed=5)
    assert np.array_equal(p.a, base.a) and np.array_equal(p.b, base.b)  # codes unchanged
    for new, old in ((p.sfa, base.sfa), (p.sfb, base.sfb)):
        ratio = new.astype(np.float64) / old
        assert ((ratio >= 1.0) & (ratio < 2.0)).all()
        mantissa = new.view(np.uint32) & 0x7FFFFF
        assert (mantissa != 0).mean() > 0.99  # (almost) no power of two left
    assert np.array_equal(p.sfa, again.sfa) and np.array_equal(p.sfb, again.sfb)  # seeded


def test_workload_10_is_workload_2_with_fp32_scales():
    w2, w10 = synth.make_config(2), synth.make_config(10)
    assert (w10.kind, w10.M, w10.N, w10.K) == ("dense", 4096, 7168, 7168)
    assert np.array_equal(w10.a, w2.a) and np.array_equal(w10.b, w2.b)
    for s10, s2 in ((w10.sfa, w2.sfa), (w10.sfb, w2.sfb)):
        ratio = s10.astype(np.float64) / s2
        assert ((ratio >= 1.0) & (ratio < 2.0)).all()
    assert ((w10.sfb.view(np.uint32) & 0x7FFFFF) != 0).all()  # no B scale is a power of two
