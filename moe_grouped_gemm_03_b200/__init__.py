"""B200 (sm_100a) FP8 NT GEMM with fine-grained scaling: dense, M-grouped contiguous and M-grouped masked.

Thin ctypes binding over ``libdg.so`` (the C ABI in ``include/dg.h``).  This module only marshals
arguments: it checks dtypes/shapes of the torch tensors, passes raw device pointers and the current CUDA
stream, and turns a negative status into ``DGError``.  Every step of the GEMM runs in the library's CUDA
kernels; there is no fallback of any kind.

Operands follow the NT convention of the DeepGEMM family ("Interfaces / Notices" of the DeepGEMM-for-PPU
README): ``lhs = (a, sfa)`` with ``a`` [M, K] e4m3 and ``sfa`` fp32 [K/128, tma_aligned(M)] (MN-major, one
scale per row and 128-K block); ``rhs = (b, sfb)`` with ``b`` [N, K] e4m3 (grouped: [G, N, K]) and ``sfb``
fp32 [ceil(N/128), K/128] (grouped: [G, ...]), one scale per 128x128 block.  Scales must be powers of two
unless ``set_fp32_scale_promotion(True)`` is in force (any finite fp32 scales, promoted per 128-K block).
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional, Tuple

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdg.so")
HEADER_PATH = os.path.join(os.path.dirname(_HERE), "include", "dg.h")

DG_OK = 0
STATUS_NAMES = {0: "DG_OK", -1: "DG_ERR_INVALID_ARG", -2: "DG_ERR_ALIGNMENT", -3: "DG_ERR_UNSUPPORTED",
                -4: "DG_ERR_CUDA", -5: "DG_ERR_DEVICE_TIMEOUT", -6: "DG_ERR_BAD_GROUP",
                -7: "DG_ERR_BAD_SCALE"}


class DGError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m moe_grouped_gemm_03_b200.build` "
                      "(or __graft_entry__.build()); there is no non-CUDA implementation")

_lib = ctypes.CDLL(LIB_PATH)
_P = ctypes.c_void_p
_I = ctypes.c_int
_LL = ctypes.c_longlong

_SIGNATURES = {
    "dg_get_m_alignment_for_contiguous_layout": (_I, []),
    "dg_set_m_alignment_for_contiguous_layout": (_I, [_I]),
    "dg_get_tma_aligned_size": (_I, [_I, _I]),
    "dg_set_num_sms": (_I, [_I]),
    "dg_get_num_sms": (_I, []),
    "dg_num_tiles": (_LL, [_LL, _LL, _I, _I]),
    "dg_select_block_n": (_I, [_LL, _I, _I]),
    "dg_fp8_gemm_nt": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _P]),
    "dg_m_grouped_fp8_gemm_nt_contiguous": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "dg_m_grouped_fp8_gemm_nt_masked": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "dg_m_grouped_fp8_gemm_nt_nopad": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "dg_m_grouped_fp8_gemm_nn_contiguous": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "dg_m_grouped_fp8_fp4_gemm_nt_contiguous": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "dg_m_grouped_fp8_fp4_gemm_nt_masked": (_I, [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _P]),
    "dg_k_grouped_fp8_gemm_nt_contiguous": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _P]),
    "dg_fp8_gemm_nt_noalloc": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _P]),
    "dg_set_cta_pair_policy": (_I, [_I]),
    "dg_set_swap_policy": (_I, [_I]),
    "dg_set_fp32_scale_promotion": (_I, [_I]),
    "dg_get_fp32_scale_promotion": (_I, []),
    "dg_debug_bounded_wait": (_I, [ctypes.c_ulonglong, _I]),
    "dg_debug_clock_record": (_I, [_I]),
    "dg_debug_clock_read": (_I, [_P, _I]),
    "dg_last_error": (ctypes.c_char_p, []),
    "dg_check_device_error": (_I, [_P]),
}
for _name, (_res, _args) in _SIGNATURES.items():
    _fn = getattr(_lib, _name)
    _fn.restype = _res
    _fn.argtypes = _args


def lib() -> ctypes.CDLL:
    """The loaded C library (raw entry points with the names of include/dg.h)."""
    return _lib


def header_symbols():
    """Names of the functions include/dg.h declares."""
    with open(HEADER_PATH) as f:
        return re.findall(r"^DG_EXPORT[^(]*?\b(dg_\w+)\(", f.read(), flags=re.M)


def last_error() -> str:
    return _lib.dg_last_error().decode()


def _check(status: int):
    if status != DG_OK:
        raise DGError(status, last_error())


def _ptr(t) -> int:
    return 0 if t is None else t.data_ptr()


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


_FP8_TYPES = (torch.uint8, torch.float8_e4m3fn)


def _need(cond: bool, what) -> None:
    """Raise DG_ERR_INVALID_ARG when cond is false; `what` is the message or a callable that builds it (messages
    are only formatted on failure, which keeps a passing check cheap)."""
    if not cond:
        raise DGError(-1, what() if callable(what) else what)


def _check_operand(name, t, dims, dtypes):
    if isinstance(t, torch.Tensor) and t.dim() == dims and t.dtype in dtypes and t.is_cuda and t.is_contiguous():
        return
    _need(isinstance(t, torch.Tensor), lambda: f"{name} must be a torch.Tensor")
    _need(t.dim() == dims, lambda: f"{name} must have {dims} dims, got {tuple(t.shape)}")
    _need(t.dtype in dtypes, lambda: f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    _need(t.is_contiguous(), lambda: f"{name} must be contiguous")
    _need(t.is_cuda, lambda: f"{name} must be a CUDA tensor")


# ------------------------------------------------------------------------------------------------ utilities
def get_m_alignment_for_contiguous_layout() -> int:
    return _lib.dg_get_m_alignment_for_contiguous_layout()


def get_mk_alignment_for_contiguous_layout() -> int:
    """The MATE wrapper's name for get_m_alignment_for_contiguous_layout (same value)."""
    return _lib.dg_get_m_alignment_for_contiguous_layout()


def set_m_alignment_for_contiguous_layout(alignment: int) -> int:
    """128 (default) or 256: the per-segment M padding the contiguous calls expect from here on."""
    rc = _lib.dg_set_m_alignment_for_contiguous_layout(int(alignment))
    _check(rc if rc < 0 else DG_OK)
    return rc


def get_tma_aligned_size(mn: int, element_size: int) -> int:
    return _lib.dg_get_tma_aligned_size(mn, element_size)


def get_mn_major_tma_aligned_tensor(sf: torch.Tensor) -> torch.Tensor:
    """Per-row scales [M, K/128] (masked layout: [G, M, K/128]) -> the layout the GEMMs take for sfa: fp32,
    MN-major and TMA-aligned, [K/128, tma_aligned(M)] (or [G, K/128, tma_aligned(M)]), contiguous, on the same
    device; the padding columns hold 1.0.  ("Utilities" and "Notices" of the DeepGEMM-for-PPU README: the LHS
    scale factor tensor is TMA-aligned and transposed.)  Input preparation by a tensor copy, outside any GEMM
    call."""
    _need(isinstance(sf, torch.Tensor) and sf.dim() in (2, 3), "sf must be a [M, K/128] or [G, M, K/128] tensor")
    x = sf.unsqueeze(0) if sf.dim() == 2 else sf
    G, M, nkb = x.shape
    out = torch.ones((G, nkb, get_tma_aligned_size(M, 4)), dtype=torch.float32, device=sf.device)
    out[:, :, :M] = x.transpose(1, 2)
    return out[0] if sf.dim() == 2 else out


get_col_major_tma_aligned_tensor = get_mn_major_tma_aligned_tensor  # the pages' other name for it


def set_num_sms(n: int) -> int:
    return _lib.dg_set_num_sms(n)


def get_num_sms() -> int:
    return _lib.dg_get_num_sms()


def num_tiles(M: int, N: int, block_m: int, block_n: int) -> int:
    return _lib.dg_num_tiles(M, N, block_m, block_n)


def select_block_n(num_m_blocks: int, N: int, num_sms: int) -> int:
    return _lib.dg_select_block_n(num_m_blocks, N, num_sms)


def set_cta_pair_policy(policy: int) -> int:
    """-1: library decides; 0: single-CTA 128-row tiles only; 1: 2-CTA 256-row tiles wherever possible."""
    return _lib.dg_set_cta_pair_policy(policy)


def set_swap_policy(policy: int) -> int:
    """-1: library decides; 0: never; 1: swapped operands (B's rows on the MMA's M side, a group's tokens on its
    N side) wherever supported."""
    return _lib.dg_set_swap_policy(policy)


def set_fp32_scale_promotion(enable: bool) -> bool:
    """False (default): scales must be powers of two (applied as UE8M0 exponents by the block-scaled MMA; others
    are reported as DG_ERR_BAD_SCALE by check_device_error).  True: any finite fp32 scales, applied by fp32
    promotion of every 128-K block's partial product (W4A8: of every 32-K sub-block's), on every call."""
    return bool(_lib.dg_set_fp32_scale_promotion(1 if enable else 0))


def get_fp32_scale_promotion() -> bool:
    return bool(_lib.dg_get_fp32_scale_promotion())


def debug_bounded_wait(limit_ns: int = 0, drop_first_stage: bool = False) -> None:
    """Testing aid: set the in-kernel wait limit (0 = default 2 s) and, optionally, make the next GEMM launch
    leave one operand stage unloaded so a wait runs out and DG_ERR_DEVICE_TIMEOUT is recorded."""
    _check(_lib.dg_debug_bounded_wait(int(limit_ns), 1 if drop_first_stage else 0))


def debug_clock_record(enable: bool) -> None:
    """Measurement aid: while on, every GEMM launch's first CTA adds its SM cycles and nanoseconds to a per-device
    accumulator (dg_debug_clock_record)."""
    _lib.dg_debug_clock_record(1 if enable else 0)


def debug_clock_read(reset: bool = True):
    """(cycles, nanoseconds, launches) recorded on the current device since the last reset (dg_debug_clock_read);
    cycles / nanoseconds is the mean SM clock of those launches in GHz."""
    out = (ctypes.c_ulonglong * 3)()
    _check(_lib.dg_debug_clock_read(ctypes.cast(out, _P), 1 if reset else 0))
    return int(out[0]), int(out[1]), int(out[2])


def check_device_error(stream=None) -> None:
    """Synchronise the stream and raise if a kernel recorded a device-side error since the last check."""
    s = _stream() if stream is None else stream
    _check(_lib.dg_check_device_error(s))


# ------------------------------------------------------------------------------------------------ GEMMs
def fp8_gemm_nt(lhs: Tuple[torch.Tensor, torch.Tensor], rhs: Tuple[torch.Tensor, torch.Tensor],
                out: torch.Tensor) -> None:
    """out[M, N] = bf16(lhs @ rhs^T) with fine-grained scales (dense)."""
    a, sfa = lhs
    b, sfb = rhs
    _check_operand("a", a, 2, _FP8_TYPES)
    _check_operand("b", b, 2, _FP8_TYPES)
    _check_operand("sfa", sfa, 2, (torch.float32,))
    _check_operand("sfb", sfb, 2, (torch.float32,))
    _check_operand("out", out, 2, (torch.bfloat16,))
    M, K = a.shape
    N = b.shape[0]
    _need(b.shape[1] == K and tuple(out.shape) == (M, N), "shape mismatch between a, b and out")
    _need(sfa.shape == (K // 128, get_tma_aligned_size(M, 4)), lambda: f"sfa must be [{K // 128}, {get_tma_aligned_size(M, 4)}]")
    _need(sfb.shape == ((N + 127) // 128, K // 128), "sfb must be [ceil(N/128), K/128]")
    _check(_lib.dg_fp8_gemm_nt(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(out), M, N, K, _stream()))


def fp8_gemm_nt_noalloc(lhs: Tuple[torch.Tensor, torch.Tensor], rhs: Tuple[torch.Tensor, torch.Tensor],
                        out: torch.Tensor) -> None:
    """Same as fp8_gemm_nt but allocates no device memory: the packed scales go to the library's fixed 16 MiB
    buffer (for callers that may not allocate during the call, e.g. under a global-mode stream capture).
    Calls overlapping on the GPU share that buffer and race; calls on one stream are safe."""
    a, sfa = lhs
    b, sfb = rhs
    _check_operand("a", a, 2, _FP8_TYPES)
    _check_operand("b", b, 2, _FP8_TYPES)
    _check_operand("sfa", sfa, 2, (torch.float32,))
    _check_operand("sfb", sfb, 2, (torch.float32,))
    _check_operand("out", out, 2, (torch.bfloat16,))
    M, K = a.shape
    N = b.shape[0]
    _need(b.shape[1] == K and tuple(out.shape) == (M, N), "shape mismatch between a, b and out")
    _need(sfa.shape == (K // 128, get_tma_aligned_size(M, 4)), lambda: f"sfa must be [{K // 128}, {get_tma_aligned_size(M, 4)}]")
    _need(sfb.shape == ((N + 127) // 128, K // 128), "sfb must be [ceil(N/128), K/128]")
    _check(_lib.dg_fp8_gemm_nt_noalloc(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(out), M, N, K, _stream()))


def m_grouped_fp8_gemm_nt_contiguous(lhs, rhs, out: torch.Tensor, m_indices: torch.Tensor) -> None:
    """Contiguous layout: out[m] = lhs[m] @ rhs[m_indices[m]]^T; rows with m_indices == -1 are untouched."""
    a, sfa = lhs
    b, sfb = rhs
    _check_operand("a", a, 2, _FP8_TYPES)
    _check_operand("b", b, 3, _FP8_TYPES)
    _check_operand("sfa", sfa, 2, (torch.float32,))
    _check_operand("sfb", sfb, 3, (torch.float32,))
    _check_operand("out", out, 2, (torch.bfloat16,))
    _check_operand("m_indices", m_indices, 1, (torch.int32,))
    M, K = a.shape
    G, N, _ = b.shape
    _need(b.shape[2] == K and tuple(out.shape) == (M, N) and m_indices.shape[0] == M, "shape mismatch")
    _need(sfa.shape == (K // 128, get_tma_aligned_size(M, 4)), "sfa must be [K/128, tma_aligned(M)]")
    _need(sfb.shape == (G, (N + 127) // 128, K // 128), "sfb must be [G, ceil(N/128), K/128]")
    _check(_lib.dg_m_grouped_fp8_gemm_nt_contiguous(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(out),
                                                    _ptr(m_indices), M, N, K, G, _stream()))


def m_grouped_fp8_gemm_nt_masked(lhs, rhs, out: torch.Tensor, masked_m: torch.Tensor, expected_m: int) -> None:
    """Masked layout: out[g, :masked_m[g]] = lhs[g, :masked_m[g]] @ rhs[g]^T; other rows are untouched."""
    a, sfa = lhs
    b, sfb = rhs
    _check_operand("a", a, 3, _FP8_TYPES)
    _check_operand("b", b, 3, _FP8_TYPES)
    _check_operand("sfa", sfa, 3, (torch.float32,))
    _check_operand("sfb", sfb, 3, (torch.float32,))
    _check_operand("out", out, 3, (torch.bfloat16,))
    _check_operand("masked_m", masked_m, 1, (torch.int32,))
    G, M_max, K = a.shape
    N = b.shape[1]
    _need(b.shape[0] == G and b.shape[2] == K and tuple(out.shape) == (G, M_max, N) and masked_m.shape[0] == G,
          "shape mismatch")
    _need(sfa.shape == (G, K // 128, get_tma_aligned_size(M_max, 4)), "sfa must be [G, K/128, tma_aligned(M_max)]")
    _need(sfb.shape == (G, (N + 127) // 128, K // 128), "sfb must be [G, ceil(N/128), K/128]")
    _check(_lib.dg_m_grouped_fp8_gemm_nt_masked(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(out), _ptr(masked_m),
                                                G, M_max, N, K, int(expected_m), _stream()))


def m_grouped_fp8_gemm_nn_contiguous(lhs, rhs, out: torch.Tensor, m_indices: torch.Tensor) -> None:
    """Contiguous layout with rhs = (b [G, K, N], sfb [G, K/128, ceil(N/128)]): out = lhs @ rhs[g] per group."""
    a, sfa = lhs
    b, sfb = rhs
    _check_operand("a", a, 2, _FP8_TYPES)
    _check_operand("b", b, 3, _FP8_TYPES)
    _check_operand("sfa", sfa, 2, (torch.float32,))
    _check_operand("sfb", sfb, 3, (torch.float32,))
    _check_operand("out", out, 2, (torch.bfloat16,))
    _check_operand("m_indices", m_indices, 1, (torch.int32,))
    M, K = a.shape
    G, _, N = b.shape
    _need(b.shape[1] == K and tuple(out.shape) == (M, N) and m_indices.shape[0] == M, "shape mismatch")
    _need(sfa.shape == (K // 128, get_tma_aligned_size(M, 4)), "sfa must be [K/128, tma_aligned(M)]")
    _need(sfb.shape == (G, K // 128, (N + 127) // 128), "sfb must be [G, K/128, ceil(N/128)]")
    _check(_lib.dg_m_grouped_fp8_gemm_nn_contiguous(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(out),
                                                    _ptr(m_indices), M, N, K, G, _stream()))


def k_grouped_fp8_gemm_nt_contiguous(lhs, rhs, out: torch.Tensor, ks, ks_tensor: torch.Tensor,
                                     c: Optional[torch.Tensor] = None) -> None:
    """K-grouped (recipe (1, 1, 128)): lhs = (a [M, sum ks], sfa [sum ks/128, tma_aligned(M)]), rhs = (b [N, sum ks],
    sfb [sum ks/128, tma_aligned(N)]); out fp32 [G, M, N] = c + per-group products (c None, another tensor, or out)."""
    a, sfa = lhs
    b, sfb = rhs
    _check_operand("a", a, 2, _FP8_TYPES)
    _check_operand("b", b, 2, _FP8_TYPES)
    _check_operand("sfa", sfa, 2, (torch.float32,))
    _check_operand("sfb", sfb, 2, (torch.float32,))
    _check_operand("out", out, 3, (torch.float32,))
    _check_operand("ks_tensor", ks_tensor, 1, (torch.int32,))
    ks = [int(k) for k in ks]
    G = len(ks)
    M, Kt = a.shape
    N = b.shape[0]
    _need(b.shape[1] == Kt and sum(ks) == Kt and tuple(out.shape) == (G, M, N) and ks_tensor.shape[0] == G,
          "shape mismatch")
    _need(sfa.shape == (Kt // 128, get_tma_aligned_size(M, 4)), "sfa must be [sum ks/128, tma_aligned(M)]")
    _need(sfb.shape == (Kt // 128, get_tma_aligned_size(N, 4)), "sfb must be [sum ks/128, tma_aligned(N)]")
    if c is not None:
        _check_operand("c", c, 3, (torch.float32,))
        _need(tuple(c.shape) == (G, M, N), "c must be [G, M, N]")
    ks_host = (ctypes.c_int * G)(*ks)
    _check(_lib.dg_k_grouped_fp8_gemm_nt_contiguous(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(out), _ptr(c),
                                                    ctypes.cast(ks_host, ctypes.c_void_p), _ptr(ks_tensor), G, M,
                                                    N, _stream()))


def m_grouped_fp8_fp4_gemm_nt_contiguous(lhs, rhs, out: torch.Tensor, m_indices: torch.Tensor) -> None:
    """W4A8 contiguous layout: rhs = (b packed E2M1 uint8 [G, N, K/2], sfb [G, K/32, tma_aligned(N)]), one B
    scale per (row, 32-K block); lhs and out as for m_grouped_fp8_gemm_nt_contiguous."""
    a, sfa = lhs
    b, sfb = rhs
    _check_operand("a", a, 2, _FP8_TYPES)
    _check_operand("b", b, 3, (torch.uint8,))
    _check_operand("sfa", sfa, 2, (torch.float32,))
    _check_operand("sfb", sfb, 3, (torch.float32,))
    _check_operand("out", out, 2, (torch.bfloat16,))
    _check_operand("m_indices", m_indices, 1, (torch.int32,))
    M, K = a.shape
    G, N, half_k = b.shape
    _need(half_k * 2 == K and tuple(out.shape) == (M, N) and m_indices.shape[0] == M, "shape mismatch")
    _need(sfa.shape == (K // 128, get_tma_aligned_size(M, 4)), "sfa must be [K/128, tma_aligned(M)]")
    _need(sfb.shape == (G, K // 32, get_tma_aligned_size(N, 4)), "sfb must be [G, K/32, tma_aligned(N)]")
    _check(_lib.dg_m_grouped_fp8_fp4_gemm_nt_contiguous(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(out),
                                                        _ptr(m_indices), M, N, K, G, _stream()))


def m_grouped_fp8_fp4_gemm_nt_masked(lhs, rhs, out: torch.Tensor, masked_m: torch.Tensor, expected_m: int) -> None:
    """W4A8 masked layout: rhs = (b packed E2M1 uint8 [G, N, K/2], sfb [G, K/32, tma_aligned(N)]); lhs, out and
    masked_m as for m_grouped_fp8_gemm_nt_masked."""
    a, sfa = lhs
    b, sfb = rhs
    _check_operand("a", a, 3, _FP8_TYPES)
    _check_operand("b", b, 3, (torch.uint8,))
    _check_operand("sfa", sfa, 3, (torch.float32,))
    _check_operand("sfb", sfb, 3, (torch.float32,))
    _check_operand("out", out, 3, (torch.bfloat16,))
    _check_operand("masked_m", masked_m, 1, (torch.int32,))
    G, M_max, K = a.shape
    N = b.shape[1]
    _need(b.shape[0] == G and b.shape[2] * 2 == K and tuple(out.shape) == (G, M_max, N) and masked_m.shape[0] == G,
          "shape mismatch")
    _need(sfa.shape == (G, K // 128, get_tma_aligned_size(M_max, 4)), "sfa must be [G, K/128, tma_aligned(M_max)]")
    _need(sfb.shape == (G, K // 32, get_tma_aligned_size(N, 4)), "sfb must be [G, K/32, tma_aligned(N)]")
    _check(_lib.dg_m_grouped_fp8_fp4_gemm_nt_masked(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(out), _ptr(masked_m),
                                                    G, M_max, N, K, int(expected_m), _stream()))


def m_grouped_fp8_gemm_nt_nopad(lhs, rhs, out: torch.Tensor, counts: torch.Tensor) -> None:
    """No-padding layout: group g's rows are off_g .. off_g + counts[g] - 1 (off_g = sum of the earlier counts);
    out rows of group g = lhs rows of group g @ rhs[g]^T; rows past sum(counts) are untouched."""
    a, sfa = lhs
    b, sfb = rhs
    _check_operand("a", a, 2, _FP8_TYPES)
    _check_operand("b", b, 3, _FP8_TYPES)
    _check_operand("sfa", sfa, 2, (torch.float32,))
    _check_operand("sfb", sfb, 3, (torch.float32,))
    _check_operand("out", out, 2, (torch.bfloat16,))
    _check_operand("counts", counts, 1, (torch.int32,))
    M, K = a.shape
    G, N, _ = b.shape
    _need(b.shape[2] == K and tuple(out.shape) == (M, N) and counts.shape[0] == G, "shape mismatch")
    _need(sfa.shape[0] == K // 128 and sfa.shape[1] == get_tma_aligned_size(M, 4),
          "sfa must be [K/128, tma_aligned(M_total)]")
    _need(sfb.shape == (G, (N + 127) // 128, K // 128), "sfb must be [G, ceil(N/128), K/128]")
    _check(_lib.dg_m_grouped_fp8_gemm_nt_nopad(_ptr(a), _ptr(sfa), _ptr(b), _ptr(sfb), _ptr(out), _ptr(counts),
                                               M, N, K, G, _stream()))


__all__ = [
    "DGError", "fp8_gemm_nt", "fp8_gemm_nt_noalloc", "m_grouped_fp8_gemm_nt_contiguous", "m_grouped_fp8_gemm_nt_masked",
    "m_grouped_fp8_gemm_nt_nopad", "m_grouped_fp8_gemm_nn_contiguous", "k_grouped_fp8_gemm_nt_contiguous",
    "m_grouped_fp8_fp4_gemm_nt_contiguous", "m_grouped_fp8_fp4_gemm_nt_masked",
    "get_m_alignment_for_contiguous_layout", "set_m_alignment_for_contiguous_layout", "get_tma_aligned_size", "set_num_sms", "get_num_sms", "num_tiles",
    "select_block_n", "set_cta_pair_policy", "check_device_error", "lib", "header_symbols", "last_error",
]
