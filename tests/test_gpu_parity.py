"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the same seeded inputs.

Tolerance (per element, over the rows the GEMM owns): |gpu - ref| <= 2^-7 |ref| + 1e-2 rms(ref), and the
global similarity calc_diff = 1 - 2<x,y>/(|x|^2+|y|^2) < 1e-3.  Rows the GEMM does not own must keep the
sentinel bits pre-filled in D.
"""
import numpy as np
import pytest
import torch

import oracle
import synth
from _helpers import assert_close, bf16_to_f64, run_problem, untouched_rows_ok

pytestmark = pytest.mark.gpu


@pytest.fixture(params=[0, 1], ids=["single_cta", "cta_pair"])
def policy(request):
    import moe_grouped_gemm_03_b200 as dg

    dg.set_cta_pair_policy(request.param)
    yield request.param
    dg.set_cta_pair_policy(-1)


@pytest.fixture(params=[0, 1], ids=["unswapped", "swapped"])
def swap(request):
    """Tiles with the operands in their own order, or swapped (B's rows on the MMA's M side, tokens on N)."""
    import moe_grouped_gemm_03_b200 as dg

    dg.set_swap_policy(request.param)
    yield request.param
    dg.set_swap_policy(-1)


def _full_check(p):
    out = run_problem(p)
    import moe_grouped_gemm_03_b200 as dg

    dg.check_device_error()
    ref = oracle.problem_full(p).reshape(-1, p.N)
    got = bf16_to_f64(out).reshape(-1, p.N)
    valid = ~np.isnan(ref[:, 0])
    assert_close(got[valid], ref[valid], p.name)
    assert untouched_rows_ok(out, valid), "rows outside the groups were written"
    return out


def test_pair_and_single_paths_agree():
    """Single-CTA 128-row tiles and 2-CTA 256-row tiles give the same products (within fp32 ordering)."""
    import moe_grouped_gemm_03_b200 as dg

    p = synth.make_contiguous([300, 129, 640, 1], 1024, 1024, seed=21)
    outs = []
    for pol in (0, 1):
        dg.set_cta_pair_policy(pol)
        outs.append(run_problem(p).clone())
    dg.set_cta_pair_policy(-1)
    valid = np.zeros(p.rows, bool)
    valid[p.valid_rows()] = True
    sel = torch.from_numpy(valid).cuda()
    assert_close(bf16_to_f64(outs[1][sel]), bf16_to_f64(outs[0][sel]), "pair vs single")


def test_config1_dense_small():
    _full_check(synth.make_config(1))


@pytest.mark.parametrize("M,N,K", [
    # short calls (K <= 2048, 2MNK <= 2^34): one kernel, the promotion GEMM on power-of-two scales
    (1, 16, 128),        # one row, narrowest N
    (128, 128, 128),     # one tile, one K block
    (300, 608, 384),     # ragged M tail, N not a multiple of any tile width
    (129, 4096, 256),    # M tail of one row over many N tiles
    (1000, 2048, 1024),  # several waves of tiles
    (64, 7168, 512),     # N=7168
    # longer K: the scale pre-pass and the block-scaled GEMM
    (1, 16, 2176),
    (300, 608, 2304),
    (129, 4096, 2560),
    (1000, 2048, 2176),  # several waves of tiles
    (64, 7168, 4096),    # N=7168 (224-wide tiles)
])
def test_dense_shapes(M, N, K, policy):
    _full_check(synth.make_dense(M, N, K, seed=M + N + K))


@pytest.mark.parametrize("counts,N,K", [
    ([0, 1, 127, 128, 129, 300], 512, 256),
    ([513, 7, 260], 4096, 384),
    ([1], 16, 128),
    ([129, 1, 130, 255, 256, 257, 3], 640, 256),  # odd block counts: 256-row windows straddle groups
    ([128] * 9, 256, 128),                        # nine one-block groups: every pair window holds two groups
])
def test_contiguous_shapes(counts, N, K, policy, swap):
    _full_check(synth.make_contiguous(counts, N, K, seed=sum(counts) + N))


def test_contiguous_beyond_the_swapped_tables(policy):
    """More 128-row blocks (1105) than the device tables of the swapped-operand tiles hold (1024): the call runs
    the unswapped 128- or 256-row windows instead."""
    _full_check(synth.make_contiguous([15000, 1, 129, 30000, 95000, 127, 256, 255, 70], 256, 128, seed=77))


@pytest.mark.parametrize("G,M_max,N,K,mm", [
    (5, 200, 256, 512, [0, 1, 128, 200, 77]),
    (3, 256, 7168, 256, [256, 0, 129]),
    (4, 64, 160, 128, [64, 63, 0, 1]),
    (40, 128, 384, 256, None),
    # groups cut into several token chunks (a chunk holds at most 224 tokens; 1000 -> 5 chunks of 208 rows),
    # N not a multiple of 256, a partial scale group along K (5 K blocks)
    (6, 700, 304, 640, [700, 225, 224, 449, 15, 0]),
    (2, 1000, 7168, 256, [1000, 31]),
])
def test_masked_shapes(G, M_max, N, K, mm, policy, swap):
    _full_check(synth.make_masked(G, M_max, N, K, masked_m=mm, seed=G + M_max, expected_m=M_max // 2))


@pytest.mark.parametrize("counts,N,K", [
    ([0, 1, 127, 128, 129, 300], 512, 256),
    ([513, 7, 260], 4096, 384),
    ([1], 16, 128),
    ([129, 1, 130, 255, 256, 257, 3], 640, 256),
])
def test_contiguous_nn_shapes(counts, N, K, policy, swap):
    _full_check(synth.make_contiguous_nn(counts, N, K, seed=sum(counts) + N))


def test_nn_equals_nt_on_the_transposed_b(policy):
    """The NN call on B [G, K, N] and the NT call on the same B stored [G, N, K] give bit-identical outputs."""
    nn = synth.make_contiguous_nn([200, 77, 384], 1040, 512, seed=22)
    nt = synth.make_contiguous([200, 77, 384], 1040, 512, seed=22)
    a = run_problem(nn).clone()
    b = run_problem(nt)
    import moe_grouped_gemm_03_b200 as dg

    dg.check_device_error()
    valid = torch.from_numpy(nt.m_indices >= 0).cuda()
    assert torch.equal(a[valid], b[valid])


def _run_k_grouped(p, c_mode):
    """c_mode: 'none' (D = products), 'separate' (C in its own tensor) or 'inplace' (D holds C on entry)."""
    import moe_grouped_gemm_03_b200 as dg

    t = synth.to_torch(p)
    out = torch.full(p.out_shape(), float("nan"), dtype=torch.float32, device="cuda")
    c = None
    if c_mode == "separate":
        c = t["c"]
    elif c_mode == "inplace":
        out.copy_(t["c"])
        c = out
    dg.k_grouped_fp8_gemm_nt_contiguous((t["a"], t["sfa"]), (t["b"], t["sfb"]), out, p.counts.tolist(), t["ks"], c)
    dg.check_device_error()
    return out.cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("ks,M,N", [
    ([128, 256, 384], 256, 512),
    ([0, 128, 640], 200, 272),    # an empty K range, M and N tails
    ([512] * 4, 136, 1040),
    ([128], 1, 16),               # one row, narrowest N
    ([384, 128], 1000, 2048),     # several waves of tiles
])
@pytest.mark.parametrize("c_mode", ["none", "separate", "inplace"])
def test_k_grouped_shapes(ks, M, N, c_mode, policy):
    p = synth.make_k_grouped(ks, M, N, seed=sum(ks) + M + N, with_c=c_mode != "none")
    got = _run_k_grouped(p, c_mode)
    ref = oracle.problem_full(p)
    assert_close(got.reshape(-1, N), ref.reshape(-1, N), p.name)
    # fp32 output: far tighter than the bf16 tolerance (fp32 accumulation over at most 640 products per group)
    rms = float(np.sqrt((ref * ref).mean()))
    assert np.abs(got - ref).max() <= 1e-4 * rms + 1e-5 * np.abs(ref).max()


@pytest.mark.parametrize("counts,N,K", [
    ([0, 1, 127, 128, 129, 300], 512, 256),
    ([513, 7, 260], 4096, 384),
    ([1], 16, 128),
    ([129, 1, 130, 255, 256, 257, 3], 640, 256),
    ([300, 200], 7168, 1024),
])
def test_contiguous_w4a8_shapes(counts, N, K, policy):
    _full_check(synth.make_contiguous_w4a8(counts, N, K, seed=sum(counts) + N + 4))


@pytest.mark.parametrize("G,M_max,N,K,mm", [
    (5, 200, 256, 512, [0, 1, 128, 200, 77]),
    (3, 256, 7168, 256, [256, 0, 129]),
    (40, 128, 384, 256, None),
])
def test_masked_w4a8_shapes(G, M_max, N, K, mm, policy):
    _full_check(synth.make_masked_w4a8(G, M_max, N, K, masked_m=mm, seed=G + M_max + 4, expected_m=M_max // 2))


@pytest.fixture
def alignment_256():
    import moe_grouped_gemm_03_b200 as dg

    dg.set_m_alignment_for_contiguous_layout(256)
    yield 256
    dg.set_m_alignment_for_contiguous_layout(128)


@pytest.mark.parametrize("counts,N,K", [
    ([0, 1, 127, 128, 129, 300], 512, 256),
    ([129, 1, 130, 255, 256, 257, 3], 640, 384),
    ([256] * 5, 256, 128),
])
def test_contiguous_alignment_256(counts, N, K, policy, alignment_256, swap):
    """Segments padded to 256 rows (the optional alignment): every 256-row window holds one group."""
    _full_check(synth.make_contiguous(counts, N, K, seed=sum(counts) + 256, alignment=256))


@pytest.mark.parametrize("counts,N,K,extra", [
    ([0, 1, 127, 128, 129, 300], 512, 256, 0),
    ([513, 7, 260], 4096, 384, 5),
    ([1], 16, 128, 0),
    ([129, 1, 130, 255, 256, 257, 3], 640, 256, 131),  # groups start at any row; a tail no group owns
    ([37] * 40, 384, 256, 0),                          # forty small groups: every window is partial
    ([0, 0, 0], 256, 128, 40),                         # no group owns a row: nothing is written
])
def test_nopad_shapes(counts, N, K, extra, policy, swap):
    _full_check(synth.make_nopad(counts, N, K, seed=sum(counts) + N + extra, extra_rows=extra))


def test_nopad_counts_past_m_total_are_clipped_and_reported(policy, swap):
    """Counts summing past M_total: the rows up to M_total are computed as the clipped layout says, and the
    device error word reports it; a negative count owns no row."""
    import moe_grouped_gemm_03_b200 as dg

    p = synth.make_nopad([100, 50], 256, 256, seed=15)
    t = synth.to_torch(p)
    t["counts"].copy_(torch.tensor([100, 80], dtype=torch.int32))
    out = run_problem(p, tensors=t)
    with pytest.raises(dg.DGError) as e:
        dg.check_device_error()
    assert e.value.status == -6
    assert_close(bf16_to_f64(out), oracle.problem_full(p), "clipped counts")
    q = synth.make_nopad([0, 64], 256, 256, seed=16)
    tq = synth.to_torch(q)
    tq["counts"].copy_(torch.tensor([-5, 64], dtype=torch.int32))
    out = run_problem(q, tensors=tq)
    with pytest.raises(dg.DGError):
        dg.check_device_error()
    assert_close(bf16_to_f64(out), oracle.problem_full(q), "negative count")


def test_nopad_equals_contiguous_call_on_the_padded_layout(policy):
    """The same tokens through the no-padding and the contiguous entry points give bit-identical rows."""
    import moe_grouped_gemm_03_b200 as dg

    counts = [200, 77, 384, 1]
    q = synth.make_nopad(counts, 1024, 512, seed=18)
    out_np = run_problem(q)
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
    t = synth.to_torch(q)
    out_c = torch.empty(M_total, q.N, dtype=torch.bfloat16, device="cuda")
    dg.m_grouped_fp8_gemm_nt_contiguous((torch.from_numpy(a).cuda(), torch.from_numpy(sfa).cuda()),
                                        (t["b"], t["sfb"]), out_c, torch.from_numpy(m_indices).cuda())
    dg.check_device_error()
    src = 0
    for g, c in enumerate(counts):
        assert torch.equal(out_np[src:src + c], out_c[starts[g]:starts[g] + c]), f"group {g}"
        src += c


def test_masked_all_groups_empty_writes_nothing(policy, swap):
    p = synth.make_masked(3, 128, 256, 256, masked_m=[0, 0, 0], seed=1)
    out = run_problem(p)
    assert untouched_rows_ok(out, np.zeros(3 * 128, bool))


def test_row_power_of_two_scaling_is_bitwise(policy):
    """D(2^j sfa[row]) == 2^j D(sfa[row]) bit for bit (power-of-two scaling is exact in fp32 and bf16)."""
    p = synth.make_dense(256, 512, 512, seed=11)
    base = run_problem(p).clone()
    rows = [0, 5, 130, 255]
    p.sfa[:, rows] *= 8.0
    got = run_problem(p)
    torch.testing.assert_close(got[rows].float(), 8.0 * base[rows].float(), rtol=0, atol=0)
    other = [r for r in range(256) if r not in rows]
    assert torch.equal(got[other], base[other])


def test_contiguous_groups_equal_dense_calls(policy):
    p = synth.make_contiguous([200, 77, 384], 1024, 512, seed=12)
    out = run_problem(p)
    import moe_grouped_gemm_03_b200 as dg

    t = synth.to_torch(p)
    start = 0
    for g, c in enumerate(p.counts):
        seg = synth.align_up(int(c), 128)
        rows = slice(start, start + seg)
        sfa = torch.from_numpy(np.ascontiguousarray(p.sfa[:, rows])).cuda()
        d = torch.empty(seg, p.N, dtype=torch.bfloat16, device="cuda")
        dg.fp8_gemm_nt((t["a"][rows].contiguous(), sfa), (t["b"][g].contiguous(), t["sfb"][g].contiguous()), d)
        a = bf16_to_f64(out[start:start + int(c)])
        b = bf16_to_f64(d[:int(c)])
        assert_close(a, b, f"group {g}")
        start += seg


def test_bad_group_id_is_reported_and_skipped(policy, swap):
    import moe_grouped_gemm_03_b200 as dg

    p = synth.make_contiguous([128, 128], 256, 256, seed=13)
    t = synth.to_torch(p)
    t["m_indices"][128:256] = 7  # group 7 does not exist (G = 2)
    out = run_problem(p, tensors=t)
    with pytest.raises(dg.DGError) as e:
        dg.check_device_error()
    assert e.value.status == -6
    valid = np.zeros(256, bool)
    valid[:128] = True
    assert untouched_rows_ok(out, valid)
    ref = oracle.problem_full(p)[:128]
    assert_close(bf16_to_f64(out[:128]), ref, "group 0 next to a bad group")
    dg.check_device_error()  # the word was cleared


def test_expected_m_does_not_change_results():
    p = synth.make_masked(8, 256, 7168, 256, seed=14)
    out1 = run_problem(p).clone()
    p.expected_m = 1
    out2 = run_problem(p)
    valid = np.zeros(8 * 256, bool)
    valid[p.valid_rows()] = True
    a = out1.reshape(-1, p.N)[torch.from_numpy(valid).cuda()]
    b = out2.reshape(-1, p.N)[torch.from_numpy(valid).cuda()]
    assert_close(bf16_to_f64(a), bf16_to_f64(b), "expected_m")


def test_contiguous_many_groups_takes_the_single_cta_path():
    """3000 one-block groups: more 128-row blocks than the pair window table holds (2048), so the call falls back
    to single-CTA tiles; group ids above 2^11 exercise the tile list's group field.  Sampled rows vs the oracle."""
    import moe_grouped_gemm_03_b200 as dg

    rng = np.random.default_rng(41)
    counts = rng.integers(1, 129, size=3000)
    p = synth.make_contiguous(counts, 32, 128, seed=41)
    out = run_problem(p)
    dg.check_device_error()
    valid = p.valid_rows()
    rows = np.unique(np.concatenate([valid[:200], valid[-200:], rng.choice(valid, 400, replace=False)]))
    ref = oracle.problem_rows(p, rows)
    assert_close(bf16_to_f64(out[torch.from_numpy(rows).cuda()]), ref, "3000 groups")
    mask = np.zeros(p.rows, bool)
    mask[valid] = True
    assert untouched_rows_ok(out, mask)


def test_masked_and_nopad_at_the_group_limit(policy, swap):
    """1024 groups, the most the masked and no-padding calls accept."""
    import moe_grouped_gemm_03_b200 as dg

    rng = np.random.default_rng(42)
    mm = rng.integers(0, 65, size=1024)
    _full_check(synth.make_masked(1024, 64, 128, 128, masked_m=mm, seed=42, expected_m=32))
    q = synth.make_nopad(rng.integers(0, 40, size=1024), 128, 128, seed=43, extra_rows=7)
    _full_check(q)
    dg.check_device_error()
