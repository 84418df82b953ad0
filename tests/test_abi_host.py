"""C-ABI checks that need no GPU: the library loads, exports every declared symbol, its host arithmetic
matches the pages' worked example, and bad arguments return error codes before anything is launched."""
import ctypes
import os
import subprocess

import pytest

import moe_grouped_gemm_03_b200 as dg

HERE = os.path.dirname(os.path.abspath(__file__))
L = dg.lib()


def test_every_declared_symbol_is_exported():
    names = dg.header_symbols()
    assert len(names) >= 11
    out = subprocess.run(["nm", "-D", "--defined-only", dg.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        getattr(L, n)  # resolvable through ctypes


def test_alignment_and_tma_size():
    assert dg.get_m_alignment_for_contiguous_layout() == 128
    assert dg.get_tma_aligned_size(1, 4) == 4
    assert dg.get_tma_aligned_size(4096, 4) == 4096
    assert dg.get_tma_aligned_size(4319, 4) == 4320
    assert dg.get_tma_aligned_size(17, 1) == 32
    assert dg.get_tma_aligned_size(5, 0) == -1


def test_tile_count_worked_example():
    rows = [ln.split() for ln in open(os.path.join(HERE, "golden", "sm_utilisation_example.txt"))
            if ln.strip() and not ln.startswith("#")]
    assert rows
    for M, N, bm, bn, tiles in rows:
        assert dg.num_tiles(int(M), int(N), int(bm), int(bn)) == int(tiles)


def test_block_n_choice_avoids_wave_quantisation_on_148_sms():
    # dense 4096 x 7168: 32 M blocks; 224-wide tiles give 1024 tiles = 6.92 waves of 148
    assert dg.select_block_n(32, 7168, 148) == 224
    # a single 128-row block of a 256-wide output: two 128-wide tiles beat one ragged 224 + 32
    assert dg.select_block_n(1, 256, 148) == 128
    for mb, n in [(1, 16), (7, 4096), (547, 7168), (220, 4096)]:
        assert dg.select_block_n(mb, n, 148) in (128, 160, 192, 224)


def test_num_sms_cap_roundtrip():
    try:
        dg.set_num_sms(100)
        assert dg.get_num_sms() in (100,) or dg.get_num_sms() < 100
    finally:
        dg.set_num_sms(0)


def _call_dense(a=1, sfa=1, b=1, sfb=1, d=1, M=128, N=256, K=512):
    P = ctypes.c_void_p
    return L.dg_fp8_gemm_nt(P(a * 256), P(sfa * 256), P(b * 256), P(sfb * 256), P(d * 256), M, N, K, None)


@pytest.mark.parametrize("kw,code", [
    (dict(a=0), -1), (dict(d=0), -1), (dict(K=100), -2), (dict(K=0), -1), (dict(N=8), -2), (dict(N=0), -1),
    (dict(M=-1), -1)])
def test_dense_validation(kw, code):
    assert _call_dense(**kw) == code
    assert dg.last_error()


def test_dense_misaligned_pointer():
    P = ctypes.c_void_p
    assert L.dg_fp8_gemm_nt(P(256 + 8), P(256), P(256), P(256), P(256), 128, 256, 512, None) == -2


def test_dense_empty_is_noop_without_device():
    assert _call_dense(M=0) == 0


def test_grouped_validation():
    P = ctypes.c_void_p
    ok = dict(a=P(256), sfa=P(256), b=P(256), sfb=P(256), d=P(256))
    # contiguous: G < 1, M_total not a multiple of 128, null m_indices
    assert L.dg_m_grouped_fp8_gemm_nt_contiguous(*ok.values(), P(256), 256, 256, 512, 0, None) == -1
    assert L.dg_m_grouped_fp8_gemm_nt_contiguous(*ok.values(), P(256), 200, 256, 512, 2, None) == -2
    assert L.dg_m_grouped_fp8_gemm_nt_contiguous(*ok.values(), None, 256, 256, 512, 2, None) == -1
    assert L.dg_m_grouped_fp8_gemm_nt_contiguous(*ok.values(), P(258), 256, 256, 512, 2, None) == -2
    assert L.dg_m_grouped_fp8_gemm_nt_contiguous(*ok.values(), P(256), 0, 256, 512, 2, None) == 0
    # masked: G out of range, M_max < 1, null masked_m
    assert L.dg_m_grouped_fp8_gemm_nt_masked(*ok.values(), P(256), 0, 256, 256, 512, 128, None) == -1
    assert L.dg_m_grouped_fp8_gemm_nt_masked(*ok.values(), P(256), 1025, 256, 256, 512, 128, None) == -1
    assert L.dg_m_grouped_fp8_gemm_nt_masked(*ok.values(), P(256), 4, 0, 256, 512, 128, None) == -1
    assert L.dg_m_grouped_fp8_gemm_nt_masked(*ok.values(), None, 4, 256, 256, 512, 128, None) == -1
    assert L.dg_m_grouped_fp8_gemm_nt_masked(*ok.values(), P(256), 4, 256, 250, 512, 128, None) == -2


def test_debug_wait_limit_range():
    """The wait-limit testing aid accepts 0 (default) or 1 ms .. 2 s, and needs no device."""
    assert L.dg_debug_bounded_wait(ctypes.c_ulonglong(5), 0) == -1
    assert L.dg_debug_bounded_wait(ctypes.c_ulonglong(3_000_000_000), 0) == -1
    assert L.dg_debug_bounded_wait(ctypes.c_ulonglong(1_000_000), 0) == 0
    assert L.dg_debug_bounded_wait(ctypes.c_ulonglong(0), 0) == 0


def test_contiguous_alignment_setting():
    """128 (default) or 256 per the pages; other values are refused; M_total is validated against it."""
    import moe_grouped_gemm_03_b200 as dg

    P = ctypes.c_void_p
    ok = dict(a=P(256), sfa=P(256), b=P(256), sfb=P(256), d=P(256))
    assert L.dg_get_m_alignment_for_contiguous_layout() == 128
    assert L.dg_set_m_alignment_for_contiguous_layout(64) == -1
    assert L.dg_set_m_alignment_for_contiguous_layout(384) == -1
    assert L.dg_get_m_alignment_for_contiguous_layout() == 128
    try:
        assert dg.set_m_alignment_for_contiguous_layout(256) == 256
        assert dg.get_m_alignment_for_contiguous_layout() == 256
        assert dg.get_mk_alignment_for_contiguous_layout() == 256  # the MATE name, same value
        # 384 rows are 128-aligned but not 256-aligned
        assert L.dg_m_grouped_fp8_gemm_nt_contiguous(*ok.values(), P(256), 384, 256, 512, 2, None) == -2
        assert L.dg_m_grouped_fp8_gemm_nt_contiguous(*ok.values(), P(256), 0, 256, 512, 2, None) == 0
    finally:
        assert dg.set_m_alignment_for_contiguous_layout(128) == 128
    assert L.dg_m_grouped_fp8_gemm_nt_contiguous(*ok.values(), P(256), 200, 256, 512, 2, None) == -2


def test_fp32_scale_promotion_setting_roundtrip():
    assert dg.get_fp32_scale_promotion() is False  # power-of-two scales (UE8M0) by default
    try:
        assert L.dg_set_fp32_scale_promotion(7) == 1  # any nonzero value switches it on
        assert dg.get_fp32_scale_promotion() is True
        # argument checks still come first on the promotion path (nothing is launched)
        z = ctypes.c_void_p(16)
        assert L.dg_fp8_gemm_nt(z, z, z, z, z, 128, 256, 100, None) == -2
        assert L.dg_fp8_gemm_nt(z, z, z, z, z, 0, 256, 128, None) == 0  # empty: a no-op, no device needed
    finally:
        assert dg.set_fp32_scale_promotion(False) is False
    assert L.dg_get_fp32_scale_promotion() == 0


def test_status_names_cover_the_header():
    import re

    text = open(dg.HEADER_PATH).read()
    declared = {int(v): name for name, v in re.findall(r"\b(DG_(?:OK|ERR_[A-Z_]+))\s*=\s*(-?\d+)", text)}
    assert declared[0] == "DG_OK" and declared[-7] == "DG_ERR_BAD_SCALE"
    assert declared == dg.STATUS_NAMES


def test_mn_major_tma_aligned_scale_layout():
    import numpy as np
    import torch

    import synth

    sf = torch.arange(1, 1 + 13 * 3, dtype=torch.float32).reshape(13, 3)  # [M, K/128], M = 13 -> aligned 16
    out = dg.get_mn_major_tma_aligned_tensor(sf)
    assert out.shape == (3, 16) and out.is_contiguous() and out.dtype == torch.float32
    assert torch.equal(out[:, :13], sf.t()) and torch.equal(out[:, 13:], torch.ones(3, 3))
    g = torch.rand(2, 5, 4)
    og = dg.get_col_major_tma_aligned_tensor(g)
    assert og.shape == (2, 4, 8) and torch.equal(og[:, :, :5], g.transpose(1, 2))
    # the generator's dense-call sfa is exactly this layout of its per-row scales
    p = synth.make_dense(37, 128, 384, seed=3)
    per_row = torch.from_numpy(np.ascontiguousarray(p.sfa[:, :37].T))
    assert torch.equal(dg.get_mn_major_tma_aligned_tensor(per_row), torch.from_numpy(p.sfa))
