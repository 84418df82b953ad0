"""Shared test helpers: run a synth.Problem through the library, compare with the oracle."""
import numpy as np
import torch

SENTINEL_BITS = 0xFFFF  # a bf16 NaN pattern pre-filled in D: rows the GEMM does not own must keep it


def run_problem(p, tensors=None, out=None, stream=None):
    import moe_grouped_gemm_03_b200 as dg
    import synth

    t = tensors if tensors is not None else synth.to_torch(p)
    if out is None:
        dtype = torch.float32 if p.kind == "k_grouped" else torch.bfloat16
        out = torch.empty(p.out_shape(), dtype=dtype, device="cuda")
        out.view(torch.int16).fill_(-1)  # 0xFFFF (a NaN in either type)
    if p.kind == "k_grouped":  # C, when the problem has one, is passed as a separate tensor
        dg.k_grouped_fp8_gemm_nt_contiguous((t["a"], t["sfa"]), (t["b"], t["sfb"]), out, p.counts.tolist(),
                                            t["ks"], t.get("c"))
        return out
    if p.kind == "dense":
        dg.fp8_gemm_nt((t["a"], t["sfa"]), (t["b"], t["sfb"]), out)
    elif p.kind == "contiguous":
        dg.m_grouped_fp8_gemm_nt_contiguous((t["a"], t["sfa"]), (t["b"], t["sfb"]), out, t["m_indices"])
    elif p.kind == "masked_w4a8":
        dg.m_grouped_fp8_fp4_gemm_nt_masked((t["a"], t["sfa"]), (t["b"], t["sfb"]), out, t["masked_m"], p.expected_m)
    elif p.kind == "contiguous_w4a8":
        dg.m_grouped_fp8_fp4_gemm_nt_contiguous((t["a"], t["sfa"]), (t["b"], t["sfb"]), out, t["m_indices"])
    elif p.kind == "contiguous_nn":
        dg.m_grouped_fp8_gemm_nn_contiguous((t["a"], t["sfa"]), (t["b"], t["sfb"]), out, t["m_indices"])
    elif p.kind == "nopad":
        dg.m_grouped_fp8_gemm_nt_nopad((t["a"], t["sfa"]), (t["b"], t["sfb"]), out, t["counts"])
    else:
        dg.m_grouped_fp8_gemm_nt_masked((t["a"], t["sfa"]), (t["b"], t["sfb"]), out, t["masked_m"], p.expected_m)
    return out


def bf16_to_f64(out: torch.Tensor) -> np.ndarray:
    return out.float().cpu().numpy().astype(np.float64)


def calc_diff(x: np.ndarray, y: np.ndarray) -> float:
    """1 - 2<x,y> / (|x|^2 + |y|^2), in float64 (the global similarity measure of the tolerance)."""
    x = x.astype(np.float64).ravel()
    y = y.astype(np.float64).ravel()
    den = (x * x).sum() + (y * y).sum()
    return 0.0 if den == 0 else float(1.0 - 2.0 * (x * y).sum() / den)


def assert_close(gpu: np.ndarray, ref: np.ndarray, what: str = ""):
    """Per element |gpu - ref| <= 2^-7 |ref| + 1e-2 rms(ref), and calc_diff < 1e-3."""
    assert gpu.shape == ref.shape
    assert np.isfinite(gpu).all(), f"{what}: non-finite GPU values"
    rms = float(np.sqrt((ref * ref).mean())) if ref.size else 0.0
    bound = 2.0 ** -7 * np.abs(ref) + 1e-2 * rms
    err = np.abs(gpu - ref)
    bad = err > bound
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} elements out of tolerance; first at {tuple(i)}: "
                             f"gpu={gpu[tuple(i)]} ref={ref[tuple(i)]} bound={bound[tuple(i)]}")
    d = calc_diff(gpu, ref)
    assert d < 1e-3, f"{what}: calc_diff {d}"


def untouched_rows_ok(out: torch.Tensor, rows_mask: np.ndarray) -> bool:
    """True if every row where rows_mask is False still holds the sentinel bits."""
    bits = out.view(torch.int16).reshape(rows_mask.shape[0], -1).cpu().numpy().view(np.uint16)
    keep = ~rows_mask
    return bool((bits[keep] == SENTINEL_BITS).all())
