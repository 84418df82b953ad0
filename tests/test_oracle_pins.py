"""Pins of the CPU oracle against facts that do not come from the oracle itself.

* e4m3 decode: all 256 codes against torch's float8_e4m3fn -> float32 conversion, plus the special values
  of the OCP E4M3 format.
* contraction: brute force on integer-valued operands against exact int64 matrix products; with unit
  scales it reduces to numpy.matmul in float64.
* scales: the blockwise definition equals dequantise-then-matmul, and scaling one block's scale by 2**j
  scales exactly that block's contribution (scale linearity).
* grouping: contiguous and masked results equal per-group dense products; rows that no group owns are
  left untouched.
"""
import numpy as np
import pytest
import torch

import oracle
import synth


def torch_decode(codes):
    t = torch.from_numpy(np.ascontiguousarray(codes, np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float32).double().numpy()


def test_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    mine = oracle.decode_e4m3(codes)
    ref = torch_decode(codes)
    nan = np.isnan(ref)
    assert (np.isnan(mine) == nan).all()
    assert nan.sum() == 2  # S.1111.111 only
    np.testing.assert_array_equal(mine[~nan], ref[~nan])
    # signed zero
    assert np.signbit(mine[0x80]) and not np.signbit(mine[0x00])


@pytest.mark.parametrize("code,value", [
    (0x00, 0.0), (0x01, 2.0 ** -9), (0x07, 7 * 2.0 ** -9), (0x08, 2.0 ** -6), (0x38, 1.0),
    (0x7E, 448.0), (0xFE, -448.0), (0x40, 2.0), (0x3C, 1.5), (0xB8, -1.0)])
def test_decode_special_values(code, value):
    assert oracle.decode_e4m3(np.array([code], np.uint8))[0] == value


def test_decode_nan_codes():
    assert np.isnan(oracle.decode_e4m3(np.array([0x7F, 0xFF], np.uint8))).all()


def _codes_for_values(values):
    """e4m3 codes of exactly representable values (via torch's encoder, independent of the oracle)."""
    t = torch.tensor(values, dtype=torch.float32).to(torch.float8_e4m3fn)
    back = t.to(torch.float32).numpy()
    assert np.array_equal(back, np.asarray(values, np.float32))
    return t.view(torch.uint8).numpy()


@pytest.mark.parametrize("M,N", [(1, 1), (3, 5), (8, 8), (2, 128), (128, 7), (128, 128)])
@pytest.mark.parametrize("K", [128, 256])
def test_bruteforce_integer_operands(M, N, K):
    rng = np.random.default_rng(M * 1000 + N * 10 + K)
    ia = rng.integers(-8, 9, size=(M, K))
    ib = rng.integers(-8, 9, size=(N, K))
    a = _codes_for_values(ia.astype(np.float32))
    b = _codes_for_values(ib.astype(np.float32))
    sfa = np.ones((K // 128, synth.tma_aligned_rows(M)), np.float32)
    sfb = np.ones(((N + 127) // 128, K // 128), np.float32)
    got = oracle.fp8_gemm_nt(a, sfa, b, sfb)
    exact = ia.astype(np.int64) @ ib.astype(np.int64).T
    np.testing.assert_array_equal(got, exact.astype(np.float64))


def test_fp32_scales_against_exact_rational_arithmetic():
    """Arbitrary fp32 scales (no powers of two) on integer-valued operands: the oracle's fp64 result equals the
    exact rational value of sum_kb sfa * sfb * (integer dot product), computed with fractions.Fraction, to
    within fp64 rounding of the sum."""
    from fractions import Fraction

    rng = np.random.default_rng(11)
    M, N, K = 3, 130, 384  # two 128-column scale blocks (the second ragged), three K blocks
    nkb, nnb = K // 128, 2
    ia = rng.integers(-8, 9, size=(M, K))
    ib = rng.integers(-8, 9, size=(N, K))
    a = _codes_for_values(ia.astype(np.float32))
    b = _codes_for_values(ib.astype(np.float32))
    sfa = rng.uniform(0.01, 3.0, size=(nkb, synth.tma_aligned_rows(M))).astype(np.float32)
    sfb = rng.uniform(0.01, 3.0, size=(nnb, nkb)).astype(np.float32)
    got = oracle.fp8_gemm_nt(a, sfa, b, sfb)
    for m in range(M):
        for n in range(N):
            exact, mag = Fraction(0), 0.0
            for kb in range(nkb):
                dot = int(ia[m, 128 * kb:128 * (kb + 1)] @ ib[n, 128 * kb:128 * (kb + 1)])
                term = Fraction(float(sfa[kb, m])) * Fraction(float(sfb[n // 128, kb])) * dot
                exact += term
                mag += abs(float(term))
            assert abs(got[m, n] - float(exact)) <= 1e-15 * (mag + 1.0), (m, n)


def _random_finite_codes(rng, shape):
    c = rng.integers(0, 256, size=shape, dtype=np.uint8)
    return np.where((c & 0x7F) == 0x7F, c ^ 0x01, c).astype(np.uint8)


def test_unit_scales_reduce_to_numpy_matmul():
    rng = np.random.default_rng(1)
    M, N, K = 37, 200, 384
    a = _random_finite_codes(rng, (M, K))
    b = _random_finite_codes(rng, (N, K))
    got = oracle.fp8_gemm_nt(a, np.ones((K // 128, 40), np.float32), b, np.ones((2, K // 128), np.float32))
    ref = torch_decode(a) @ torch_decode(b).T
    np.testing.assert_allclose(got, ref, rtol=1e-13, atol=0)


@pytest.mark.parametrize("scales", ["pow2", "fp32"])
def test_blockwise_definition_equals_dequantise_then_matmul(scales):
    """With arbitrary power-of-two (or arbitrary fp32) scales the blockwise sum equals the matmul of the
    dequantised operands."""
    rng = np.random.default_rng(2)
    M, N, K = 19, 300, 512  # N not a multiple of 128: ragged last scale block
    nkb = K // 128
    a = _random_finite_codes(rng, (M, K))
    b = _random_finite_codes(rng, (N, K))
    sfa = np.ldexp(1.0, rng.integers(-6, 7, size=(nkb, 20))).astype(np.float32)
    sfb = np.ldexp(1.0, rng.integers(-6, 7, size=(3, nkb))).astype(np.float32)
    if scales == "fp32":
        sfa = (sfa * rng.uniform(1, 2, size=sfa.shape)).astype(np.float32)
        sfb = (sfb * rng.uniform(1, 2, size=sfb.shape)).astype(np.float32)
    got = oracle.fp8_gemm_nt(a, sfa, b, sfb)
    A = torch_decode(a) * np.repeat(sfa[:, :M].T, 128, axis=1)
    sb_full = np.repeat(np.repeat(sfb, 128, axis=0)[:N], 128, axis=1)
    B = torch_decode(b) * sb_full
    # fp64 rounding of the two summation orders, bounded by the sum of the products' magnitudes (with fp32 scales a
    # dequantised product carries up to 56 significant bits, so cancelling sums differ by more than 1e-12 relative)
    mag = np.abs(A) @ np.abs(B).T
    assert (np.abs(got - A @ B.T) <= 1e-13 * mag + 1e-12).all()


def test_dropped_or_misindexed_scale_is_detected():
    """Sanity of the pin above: a transposed sfb index would change the result (so the pin can fail)."""
    rng = np.random.default_rng(3)
    M, N, K = 4, 256, 256
    a = _random_finite_codes(rng, (M, K))
    b = _random_finite_codes(rng, (N, K))
    sfa = np.ones((2, 4), np.float32)
    sfb = np.array([[1.0, 2.0], [4.0, 8.0]], np.float32)
    good = oracle.fp8_gemm_nt(a, sfa, b, sfb)
    wrong = oracle.fp8_gemm_nt(a, sfa, b, np.ascontiguousarray(sfb.T))
    assert not np.allclose(good, wrong)


@pytest.mark.parametrize("which", ["sfa", "sfb"])
def test_scale_linearity(which):
    rng = np.random.default_rng(4)
    M, N, K = 9, 256, 384
    nkb = K // 128
    a = _random_finite_codes(rng, (M, K))
    b = _random_finite_codes(rng, (N, K))
    sfa = np.ldexp(1.0, rng.integers(-3, 4, size=(nkb, 12))).astype(np.float32)
    sfb = np.ldexp(1.0, rng.integers(-3, 4, size=(2, nkb))).astype(np.float32)
    base = oracle.fp8_gemm_nt(a, sfa, b, sfb)
    j, kb = 5, 1
    Ad, Bd = torch_decode(a), torch_decode(b)
    if which == "sfa":
        m = 4
        sfa2 = sfa.copy()
        sfa2[kb, m] *= 2.0 ** j
        got = oracle.fp8_gemm_nt(a, sfa2, b, sfb)
        block = Ad[m, kb * 128:(kb + 1) * 128] @ Bd[:, kb * 128:(kb + 1) * 128].T  # [N]
        contrib = sfa[kb, m] * np.repeat(sfb[:, kb], 128)[:N] * block
        expect = base.copy()
        expect[m] += (2.0 ** j - 1.0) * contrib
        np.testing.assert_array_equal(np.delete(got, m, 0), np.delete(base, m, 0))
        np.testing.assert_allclose(got, expect, rtol=1e-13, atol=1e-10)
    else:
        nb = 1
        sfb2 = sfb.copy()
        sfb2[nb, kb] *= 2.0 ** j
        got = oracle.fp8_gemm_nt(a, sfa, b, sfb2)
        cols = slice(nb * 128, (nb + 1) * 128)
        block = Ad[:, kb * 128:(kb + 1) * 128] @ Bd[cols, kb * 128:(kb + 1) * 128].T  # [M, 128]
        contrib = sfa[kb, :M][:, None] * sfb[nb, kb] * block
        expect = base.copy()
        expect[:, cols] += (2.0 ** j - 1.0) * contrib
        np.testing.assert_array_equal(got[:, :128], base[:, :128])
        np.testing.assert_allclose(got, expect, rtol=1e-13, atol=1e-10)


def test_whole_row_power_of_two_scaling_is_exact():
    rng = np.random.default_rng(5)
    p = synth.make_dense(8, 128, 256, seed=5)
    base = oracle.problem_full(p)
    p.sfa[:, 3] *= 8.0
    got = oracle.problem_full(p)
    np.testing.assert_array_equal(got[3], 8.0 * base[3])


def test_contiguous_equals_per_group_dense():
    p = synth.make_contiguous([130, 1, 256, 0, 77], N=256, K=256, seed=6)
    full = oracle.problem_full(p)
    starts = np.concatenate([[0], np.cumsum([synth.align_up(int(c), 128) for c in p.counts])])
    for g in range(p.G):
        s, c = starts[g], int(p.counts[g])
        dense = oracle.fp8_gemm_nt(p.a[s:s + c], np.ascontiguousarray(p.sfa[:, s:s + c + 4]), p.b[g], p.sfb[g])
        np.testing.assert_array_equal(full[s:s + c], dense)
        assert np.isnan(full[s + c:starts[g + 1]]).all()  # padding rows untouched


def test_masked_equals_per_group_dense_and_leaves_rows_untouched():
    p = synth.make_masked(G=4, M_max=136, N=128, K=256, masked_m=[0, 136, 5, 128], seed=7)
    full = oracle.problem_full(p)
    for g in range(p.G):
        mm = int(p.masked_m[g])
        rows = p.a[g * p.M:g * p.M + mm]
        dense = oracle.fp8_gemm_nt(rows, np.ascontiguousarray(p.sfa[g][:, :synth.tma_aligned_rows(max(mm, 1))]),
                                   p.b[g], p.sfb[g]) if mm else np.zeros((0, p.N))
        np.testing.assert_array_equal(full[g, :mm], dense)
        assert np.isnan(full[g, mm:]).all()


def test_nopad_equals_per_group_dense_and_leaves_tail_untouched():
    """No-padding layout: group g's rows off_g .. off_g + counts[g] - 1 equal a dense GEMM of exactly those rows
    with B_g; a zero-count group owns no row; rows past the sum of the counts stay untouched."""
    counts = [130, 1, 0, 256, 77]
    p = synth.make_nopad(counts, N=256, K=256, seed=16, extra_rows=9)
    full = oracle.problem_full(p)
    off = np.concatenate([[0], np.cumsum(counts)])
    for g, c in enumerate(counts):
        if c == 0:
            continue
        s = off[g]
        sfa = np.ascontiguousarray(p.sfa[:, s:s + synth.tma_aligned_rows(c)])
        dense = oracle.fp8_gemm_nt(p.a[s:s + c], sfa, p.b[g], p.sfb[g])
        np.testing.assert_array_equal(full[s:s + c], dense)
    assert np.isnan(full[off[-1]:]).all() and not np.isnan(full[:off[-1]]).any()


def test_nopad_equals_contiguous_layout_of_the_same_rows():
    """The same tokens in the padded contiguous layout give the same products row for row."""
    counts = [3, 129, 128, 0, 200]
    q = synth.make_nopad(counts, N=128, K=256, seed=17)
    padded = [synth.align_up(c, 128) for c in counts]
    starts = np.concatenate([[0], np.cumsum(padded)])
    M_total = int(starts[-1])
    a = np.zeros((M_total, q.K), np.uint8)
    sfa = np.ones((q.K // 128, synth.tma_aligned_rows(M_total)), np.float32)
    m_indices = np.full(M_total, -1, np.int32)
    src = 0
    for g, c in enumerate(counts):
        a[starts[g]:starts[g] + c] = q.a[src:src + c]
        sfa[:, starts[g]:starts[g] + c] = q.sfa[:, src:src + c]
        m_indices[starts[g]:starts[g] + c] = g
        src += c
    contig = oracle.m_grouped_fp8_gemm_nt_contiguous(a, sfa, q.b, q.sfb, m_indices)
    nopad = oracle.problem_full(q)
    src = 0
    for g, c in enumerate(counts):
        np.testing.assert_array_equal(nopad[src:src + c], contig[starts[g]:starts[g] + c])
        src += c


def test_nn_unit_scales_equal_matmul_of_k_by_n_b():
    """NN orientation: with unit scales the product is decode(A) @ decode(B_g) with B_g read as [K, N] (a
    transposed reading fails this for N != K)."""
    p = synth.make_contiguous_nn([3, 130], N=256, K=384, seed=19)
    p.sfa[:] = 1.0
    p.sfb[:] = 1.0
    full = oracle.problem_full(p)
    starts = [0, 128]
    for g, c in enumerate(p.counts):
        s, c = starts[g], int(c)
        want = oracle.decode_e4m3(p.a[s:s + c]) @ oracle.decode_e4m3(p.b[g])
        np.testing.assert_allclose(full[s:s + c], want, rtol=0, atol=0)


def test_nn_block_scale_orientation():
    """Doubling B's scale block (kb=1, nb=0) of the NN layout changes exactly output columns 0..127 of that
    group, by exactly that K block's contribution."""
    p = synth.make_contiguous_nn([130], N=256, K=384, seed=20)
    base = oracle.problem_full(p)
    p.sfb[0, 1, 0] *= 2.0
    moved = oracle.problem_full(p)
    rows = np.arange(130)
    assert np.array_equal(moved[rows, 128:], base[rows, 128:])
    a = oracle.decode_e4m3(p.a[:130, 128:256]) * p.sfa[1, :130, None]
    b = oracle.decode_e4m3(p.b[0, 128:256, :128])  # K block 1, columns 0..127
    contribution = (a @ b) * (p.sfb[0, 1, 0] / 2.0)
    np.testing.assert_allclose(moved[rows, :128] - base[rows, :128], contribution, rtol=1e-12, atol=1e-9)


def test_k_grouped_equals_dense_products_of_each_k_segment():
    """With B's row scales constant over each 128-row block, group g's K-grouped output equals C_g plus the
    (separately pinned) dense block-scaled oracle on group g's K segment; an empty segment leaves C_g."""
    ks = [256, 0, 384, 128]
    p = synth.make_k_grouped(ks, M=136, N=256, seed=21)
    nb = (p.N + 127) // 128
    blocks = np.ones((nb, p.K // 128), np.float32)
    for kb in range(p.K // 128):
        for j in range(nb):
            blocks[j, kb] = p.sfb[kb, 128 * j]
            p.sfb[kb, 128 * j:128 * (j + 1)] = blocks[j, kb]
    full = oracle.problem_full(p)
    k0 = 0
    for g, k in enumerate(ks):
        if k == 0:
            np.testing.assert_array_equal(full[g], p.c[g])
            continue
        seg = slice(k0, k0 + k)
        sfa = np.ascontiguousarray(p.sfa[k0 // 128:(k0 + k) // 128])
        dense = oracle.fp8_gemm_nt(np.ascontiguousarray(p.a[:, seg]), sfa, np.ascontiguousarray(p.b[:, seg]),
                                   np.ascontiguousarray(blocks[:, k0 // 128:(k0 + k) // 128]))
        np.testing.assert_allclose(full[g], p.c[g] + dense, rtol=1e-13, atol=1e-10)
        k0 += k


def test_k_grouped_row_scale_moves_one_column_of_one_group():
    """Doubling B's scale of row n in K block kb changes only column n of the group whose segment holds kb,
    by exactly that block's contribution; without C an empty group's output is zero."""
    p = synth.make_k_grouped([128, 256, 0], M=64, N=200, seed=22, with_c=False)
    base = oracle.problem_full(p)
    assert (base[2] == 0).all()
    kb, n = 2, 77  # K block 2 lies in group 1 (blocks 1..2)
    p.sfb[kb, n] *= 2.0
    moved = oracle.problem_full(p)
    diff = moved - base
    mask = np.zeros_like(diff, bool)
    mask[1, :, n] = True
    assert (diff[~mask] == 0).all()
    blk = slice(128 * kb, 128 * kb + 128)
    a = oracle.decode_e4m3(p.a[:, blk]) * p.sfa[kb, :64][:, None]
    contribution = a @ oracle.decode_e4m3(p.b[n, blk]) * (p.sfb[kb, n] / 2.0)
    np.testing.assert_allclose(diff[1, :, n], contribution, rtol=1e-12, atol=1e-9)


def test_k_grouped_fp32_scales_against_exact_rational_arithmetic():
    """K-grouped with arbitrary fp32 scales (one per row and K block on both sides) on integer-valued operands:
    D_g[m][n] equals the exact rational sum over group g's K blocks of sfa(kb, m) * sfb(kb, n) * (integer dot
    product), to within fp64 rounding of the sum; an empty group gives zero.  (The oracle scales each element
    before the dot product, so its rounding is bounded by the sum of the elements' magnitudes.)"""
    from fractions import Fraction

    rng = np.random.default_rng(26)
    ks = [256, 0, 128]
    p = synth.make_k_grouped(ks, M=3, N=20, seed=26, with_c=False)
    ia = rng.integers(-8, 9, size=(p.M, p.K))
    ib = rng.integers(-8, 9, size=(p.N, p.K))
    p.a = _codes_for_values(ia.astype(np.float32))
    p.b = _codes_for_values(ib.astype(np.float32))
    p.sfa = rng.uniform(0.01, 3.0, size=p.sfa.shape).astype(np.float32)
    p.sfb = rng.uniform(0.01, 3.0, size=p.sfb.shape).astype(np.float32)
    got = oracle.problem_full(p)
    assert (got[1] == 0).all()
    first = [0, 2, 2]  # each group's first 128-K block
    for g, k in enumerate(ks):
        for m in range(p.M):
            for n in range(p.N):
                exact, mag = Fraction(0), 0.0
                for kb in range(first[g], first[g] + k // 128):
                    blk = slice(128 * kb, 128 * (kb + 1))
                    dot = int(ia[m, blk] @ ib[n, blk])
                    scale = Fraction(float(p.sfa[kb, m])) * Fraction(float(p.sfb[kb, n]))
                    exact += scale * dot
                    mag += float(scale) * float(np.abs(ia[m, blk] * ib[n, blk]).sum())
                assert abs(got[g, m, n] - float(exact)) <= 4e-16 * (mag + 1.0), (g, m, n)


def test_w4a8_fp32_scales_against_exact_rational_arithmetic():
    """W4A8 with arbitrary fp32 scales (A per row and 128-K block, B per row and 32-K sub-block) on integer
    e4m3 A and E2M1-grid B: each owned row equals the exact rational sum over K blocks kb and their four 32-K
    sub-blocks j of sfa(kb, m) * sfb(g, 4kb + j, n) * (integer dot product of the sub-block), to within fp64
    rounding of the sum."""
    from fractions import Fraction

    rng = np.random.default_rng(27)
    p = synth.make_contiguous_w4a8([2, 130], N=20, K=256, seed=27)
    grid = np.array([0, 1, 2, 3, 4, 6, -1, -2, -3, -4, -6])
    codes_of = {0: 0, 1: 2, 2: 4, 3: 5, 4: 6, 6: 7, -1: 10, -2: 12, -3: 13, -4: 14, -6: 15}
    ia = rng.integers(-8, 9, size=(p.rows, p.K))
    ib = rng.choice(grid, size=(p.G, p.N, p.K))
    p.a = _codes_for_values(ia.astype(np.float32))
    p.b = synth.pack_e2m1(np.vectorize(codes_of.get)(ib).astype(np.uint8))
    p.sfa = rng.uniform(0.01, 3.0, size=p.sfa.shape).astype(np.float32)
    p.sfb = rng.uniform(0.01, 3.0, size=p.sfb.shape).astype(np.float32)
    full = oracle.problem_full(p)
    for g, start in enumerate([0, 128]):
        for m in range(start, start + int(p.counts[g])):
            for n in range(0, p.N, 3):
                exact, mag = Fraction(0), 0.0
                for kb in range(p.K // 128):
                    for j in range(4):
                        sub = slice(128 * kb + 32 * j, 128 * kb + 32 * (j + 1))
                        dot = int(ia[m, sub] @ ib[g, n, sub])
                        term = Fraction(float(p.sfa[kb, m])) * Fraction(float(p.sfb[g, 4 * kb + j, n])) * dot
                        exact += term
                        mag += abs(float(term))
                assert abs(full[m, n] - float(exact)) <= 1e-15 * (mag + 1.0), (g, m, n)


def test_e2m1_decode_matches_the_format_table():
    """All 16 E2M1 codes against the element table of the OCP Microscaling (MX) v1.0 specification (FP4 E2M1:
    +-0, 0.5, 1, 1.5, 2, 3, 4, 6 in code order, sign in bit 3)."""
    table = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    want = np.array(table + [-v for v in table])
    np.testing.assert_array_equal(oracle.decode_e2m1(np.arange(16)), want)
    # packing: element 2i in the low nibble
    np.testing.assert_array_equal(oracle.unpack_e2m1(np.array([[0x21, 0xF7]], np.uint8)), [[1, 2, 7, 15]])


def test_w4a8_bruteforce_integer_operands():
    """Integer-valued e4m3 A times E2M1 B (values -6..6 on the E2M1 grid) with unit scales equals the exact
    integer product (a misplaced nibble, sub-block or group fails it)."""
    rng = np.random.default_rng(23)
    p = synth.make_contiguous_w4a8([3, 130], N=48, K=256, seed=23)
    grid = np.array([0, 1, 2, 3, 4, 6, -1, -2, -3, -4, -6])
    codes_of = {0: 0, 1: 2, 2: 4, 3: 5, 4: 6, 6: 7, -1: 10, -2: 12, -3: 13, -4: 14, -6: 15}
    ia = rng.integers(-8, 9, size=(p.rows, p.K))
    ib = rng.choice(grid, size=(p.G, p.N, p.K))
    p.a = _codes_for_values(ia.astype(np.float32))
    p.b = synth.pack_e2m1(np.vectorize(codes_of.get)(ib).astype(np.uint8))
    p.sfa[:] = 1.0
    p.sfb[:] = 1.0
    full = oracle.problem_full(p)
    for g, start in enumerate([0, 128]):
        c = int(p.counts[g])
        exact = ia[start:start + c].astype(np.int64) @ ib[g].astype(np.int64).T
        np.testing.assert_array_equal(full[start:start + c], exact.astype(np.float64))


def test_w4a8_sub_block_scale_moves_one_column():
    """Doubling B's scale of row n in one 32-K sub-block changes only column n of that group's rows, by exactly
    that sub-block's contribution (scaled by A's 128-K block scale)."""
    p = synth.make_contiguous_w4a8([130], N=64, K=256, seed=24)
    base = oracle.problem_full(p)
    j, n = 5, 17  # sub-block 5 = K 160..191, inside 128-K block 1
    p.sfb[0, j, n] *= 2.0
    moved = oracle.problem_full(p)
    rows = np.arange(130)
    diff = moved[rows] - base[rows]
    others = np.ones(p.N, bool)
    others[n] = False
    assert (diff[:, others] == 0).all()
    sub = slice(32 * j, 32 * j + 32)
    a = oracle.decode_e4m3(p.a[:130, sub]) * p.sfa[1, :130][:, None]
    b = oracle.decode_e2m1(oracle.unpack_e2m1(p.b[0, n]))[sub]
    np.testing.assert_allclose(diff[:, n], (a @ b) * (p.sfb[0, j, n] / 2.0), rtol=1e-12, atol=1e-9)


def test_masked_w4a8_equals_contiguous_w4a8_of_the_same_rows():
    """The masked W4A8 layout's owned rows equal the (separately pinned) contiguous W4A8 product of the same
    rows, scales and B."""
    q = synth.make_masked_w4a8(3, 128, 64, 256, masked_m=[128, 5, 0], seed=25)
    c = synth.make_contiguous_w4a8([128, 128, 128], 64, 256, seed=25)
    c.a = q.a.copy()
    c.sfa = np.concatenate([q.sfa[g][:, :128] for g in range(3)], axis=1)
    c.b, c.sfb = q.b.copy(), q.sfb.copy()
    c.m_indices = np.repeat(np.arange(3, dtype=np.int32), 128)
    full_q = oracle.problem_full(q).reshape(-1, 64)
    full_c = oracle.problem_full(c)
    rows = q.valid_rows()
    np.testing.assert_array_equal(full_q[rows], full_c[rows])
    assert np.isnan(full_q[np.setdiff1d(np.arange(384), rows)]).all()


def test_library_call_shapes_agree_with_problem_driver():
    p = synth.make_masked(G=3, M_max=64, N=128, K=128, masked_m=[3, 64, 0], seed=8)
    a = p.a.reshape(p.G, p.M, p.K)
    got = oracle.m_grouped_fp8_gemm_nt_masked(a, p.sfa, p.b, p.sfb, p.masked_m)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(oracle.problem_full(p)))
    np.testing.assert_array_equal(np.nan_to_num(got), np.nan_to_num(oracle.problem_full(p)))
    q = synth.make_contiguous([5, 200], N=128, K=128, seed=9)
    got = oracle.m_grouped_fp8_gemm_nt_contiguous(q.a, q.sfa, q.b, q.sfb, q.m_indices)
    np.testing.assert_array_equal(np.nan_to_num(got), np.nan_to_num(oracle.problem_full(q)))
    r = synth.make_nopad([7, 0, 140], N=128, K=128, seed=10, extra_rows=3)
    got = oracle.m_grouped_fp8_gemm_nt_nopad(r.a, r.sfa, r.b, r.sfb, r.counts)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(oracle.problem_full(r)))
    np.testing.assert_array_equal(np.nan_to_num(got), np.nan_to_num(oracle.problem_full(r)))
    n = synth.make_contiguous_nn([9, 130], N=128, K=256, seed=11)
    got = oracle.m_grouped_fp8_gemm_nn_contiguous(n.a, n.sfa, n.b, n.sfb, n.m_indices)
    np.testing.assert_array_equal(np.nan_to_num(got), np.nan_to_num(oracle.problem_full(n)))
