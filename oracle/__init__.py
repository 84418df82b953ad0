"""CPU oracle for the FP8 NT GEMM family -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline / reference legs of ``bench.py`` may
import this package.  It shares no code with the CUDA library and the library never calls it.

The arithmetic lives in ``oracle.c`` (plain C, OpenMP over rows, double accumulation): the definition

    ref[m, n] = sum_kb sfa(m, kb) * sfb(g, n // 128, kb) * sum_{k in block kb} dec(a[m, k]) * dec(b_g[n, k])

("FP8 GEMM kernels with fine-grained scaling", DeepGEMM-for-PPU README, "Interfaces": the NT dense GEMM
gemm_fp8_fp8_bf16_nt, the contiguous- and masked-layout grouped GEMMs; recipe (1, 128, 128) from the MATE
deep_gemm wrapper API list).  This module only selects rows and marshals pointers.

Grouped layouts (same README, "Grouped GEMMs (contiguous layout)" / "(masked layout)"):
* contiguous: row m belongs to group m_indices[m]; rows with m_indices == -1 are padding and produce nothing.
* masked: group g owns rows 0 .. masked_m[g]-1 of its [M_max, K] slab; the other rows produce nothing.
* NN (MATE docs, 0.2.7 additions, `m_grouped_fp8_gemm_nn_contiguous`): the contiguous layout with each group's
  B stored [K, N]; the product is the same contraction, D[m, n] = sum_k A[m, k] B_g[k, n], with B's 128x128
  block scales stored [K/128, ceil(N/128)].  The oracle reads B_g[k, n] as the NT definition's b_g[n, k].
* K-grouped (MATE docs, 0.2.7 additions, `k_grouped_fp8_gemm_nt_contiguous`, recipe (1, 1, 128)): A [M, sum K]
  and B [N, sum K], both K-major, with the groups' K segments concatenated; one scale per (row, 128-K block) on
  both sides; D_g[m, n] = C_g[m, n] + sum over the 128-K blocks kb of group g of
  sfa(m, kb) * sfb(n, kb) * sum_{k in kb} dec(a[m, k]) * dec(b[n, k]).  Computed here with numpy in float64,
  one 128-K block at a time (each block's sum of 128 products of e4m3 values is exact in float64).
* W4A8 (MATE docs, 0.2.7 additions: e4m3 A with packed E2M1 FP4 B, recipe_a (1, 128), recipe_b (1, 32)): the
  contiguous layout with B_g stored as 4-bit E2M1 codes packed two per byte (element 2i in the low nibble) and
  one B scale per (row n, 32-K block): D[m, n] = sum over 128-K blocks kb of sfa(m, kb) * sum over its four
  32-K sub-blocks j of sfb(g, 4 kb + j, n) * sum_{k in the sub-block} dec(a[m, k]) * dec2(b_g[n, k]).
  Computed with numpy in float64 one 32-K block at a time (each block's sum is exact in float64).
* no padding (same README, "Grouped GEMMs (nopad layout)"): the groups' rows are concatenated in group order
  with no alignment; group g owns rows off_g .. off_g + counts[g] - 1 with off_g = counts[0] + ... +
  counts[g-1]; rows past the sum of the counts produce nothing.
Rows that produce nothing are returned as NaN (the "left untouched" sentinel).
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i64 = ctypes.c_int64
        L.oracle_e4m3_decode.restype = ctypes.c_double
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_decode_array.argtypes = [P, i64, P]
        L.oracle_gemm_rows.argtypes = [P, P, P, i64, P, i64, P, i64, P, P, i64, i64, i64, P]
        L.oracle_num_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(x: np.ndarray):
    return ctypes.c_void_p(x.ctypes.data)


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def decode_e4m3(codes) -> np.ndarray:
    """OCP E4M3 codes (uint8) -> float64 values."""
    c = np.ascontiguousarray(codes, dtype=np.uint8)
    out = np.empty(c.shape, np.float64)
    lib().oracle_e4m3_decode_array(_ptr(c), c.size, _ptr(out))
    return out


def decode_e2m1(codes) -> np.ndarray:
    """4-bit OCP E2M1 codes (0..15) -> float64: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0;
    exponent 0 is subnormal (0 or 0.5); no Inf or NaN codes."""
    c = np.asarray(codes, np.int64)
    sign = np.where(c & 8, -1.0, 1.0)
    e = (c >> 1) & 3
    m = c & 1
    mag = np.where(e == 0, 0.5 * m, np.ldexp(1.0 + 0.5 * m, e - 1))
    return sign * mag


def unpack_e2m1(packed) -> np.ndarray:
    """Bytes [..., K/2] -> 4-bit codes [..., K]: element 2i from the low nibble of byte i, 2i + 1 from the high."""
    b = np.asarray(packed, np.uint8)
    out = np.empty(b.shape[:-1] + (2 * b.shape[-1],), np.uint8)
    out[..., 0::2] = b & 0x0F
    out[..., 1::2] = b >> 4
    return out


def w4a8_rows(p, rows) -> np.ndarray:
    """Rows of a W4A8 ``synth.Problem`` (contiguous or masked; rows of groups only)."""
    rows = np.asarray(rows, np.int64)
    groups = p.row_groups(rows)
    out = np.zeros((len(rows), p.N))
    for g in np.unique(groups):
        sel = groups == g
        r = rows[sel]
        bdec = decode_e2m1(unpack_e2m1(p.b[g]))  # [N, K]
        adec = decode_e4m3(p.a[r])                # [rows, K]
        acc = np.zeros((len(r), p.N))
        for kb in range(p.K // 128):
            blk = np.zeros((len(r), p.N))
            for j in range(4):
                sub = slice(128 * kb + 32 * j, 128 * kb + 32 * j + 32)
                blk += (adec[:, sub] @ bdec[:, sub].T) * p.sfb[g, 4 * kb + j, :p.N][None, :]
            sa = p.sfa[g, kb, r - g * p.M] if p.kind == "masked_w4a8" else p.sfa[kb, r]
            acc += blk * sa[:, None]
        out[sel] = acc
    return out


def gemm_rows(a, sfa_row_off, sfa_kb_stride, sfa, b, sfb, rows, groups, N, K) -> np.ndarray:
    """Raw entry: listed rows of the fine-grained-scaled product, double [len(rows), N]."""
    a = np.ascontiguousarray(a, np.uint8)
    sfa = np.ascontiguousarray(sfa, np.float32)
    b = np.ascontiguousarray(b, np.uint8)
    sfb = np.ascontiguousarray(sfb, np.float32)
    rows = np.ascontiguousarray(rows, np.int64)
    groups = np.ascontiguousarray(groups, np.int32)
    off = np.ascontiguousarray(sfa_row_off, np.int64)
    assert K % 128 == 0 and a.shape[-1] == K
    n_rows = len(rows)
    out = np.empty((n_rows, N), np.float64)
    if n_rows == 0 or N == 0:
        return out
    G = b.shape[0] if b.ndim == 3 else 1
    assert rows.min() >= 0 and rows.max() < a.shape[0]
    assert groups.min() >= 0 and groups.max() < G
    nnb = (N + 127) // 128
    b_group_stride = N * K
    sfb_group_stride = nnb * (K // 128)
    assert sfb.size == G * sfb_group_stride and b.size == G * b_group_stride
    assert off.max() + (K // 128 - 1) * sfa_kb_stride < sfa.size
    lib().oracle_gemm_rows(_ptr(a), _ptr(sfa), _ptr(off), sfa_kb_stride, _ptr(b), b_group_stride, _ptr(sfb),
                           sfb_group_stride, _ptr(rows), _ptr(groups), n_rows, N, K, _ptr(out))
    return out


def problem_rows(p, rows) -> np.ndarray:
    """Selected global rows of a ``synth.Problem`` (rows must be rows the GEMM produces)."""
    rows = np.asarray(rows, np.int64)
    if p.kind == "k_grouped":  # rows of the flattened [G * M, N] output
        out = np.zeros((len(rows), p.N))
        for g in np.unique(rows // p.M):
            sel = rows // p.M == g
            out[sel] = k_grouped_rows(p, int(g), rows[sel] - g * p.M)
        return out
    groups = p.row_groups(rows)
    if p.kind in ("contiguous_w4a8", "masked_w4a8"):
        return w4a8_rows(p, rows)
    if p.kind == "contiguous_nn":
        # B_g[k, n] is the definition's b_g[n, k]; sfb_g[kb, nb] its s_b(g, nb, kb)
        b = np.ascontiguousarray(p.b.transpose(0, 2, 1))
        sfb = np.ascontiguousarray(p.sfb.transpose(0, 2, 1))
        return gemm_rows(p.a, rows, p.sfa.shape[1], p.sfa, b, sfb, rows, groups, p.N, p.K)
    if p.kind == "masked":
        Ma = p.sfa.shape[2]
        nkb = p.sfa.shape[1]
        g = rows // p.M
        off = g * nkb * Ma + (rows - g * p.M)
        kb_stride = Ma
    else:
        kb_stride = p.sfa.shape[1]
        off = rows
    return gemm_rows(p.a, off, kb_stride, p.sfa, p.b, p.sfb, rows, groups, p.N, p.K)


def k_grouped_rows(p, g, rows) -> np.ndarray:
    """Rows ``rows`` (of M) of group g's output of a K-grouped ``synth.Problem`` (C added when present)."""
    rows = np.asarray(rows, np.int64)
    ks = np.asarray(p.counts, np.int64)
    kb0 = int(ks[:g].sum()) // 128
    out = np.zeros((len(rows), p.N)) if p.c is None else p.c[g][rows].astype(np.float64)
    for kb in range(kb0, kb0 + int(ks[g]) // 128):
        blk = slice(128 * kb, 128 * kb + 128)
        a = decode_e4m3(p.a[rows, blk]) * p.sfa[kb, rows][:, None]
        b = decode_e4m3(p.b[:, blk]) * p.sfb[kb, :p.N][:, None]
        out += a @ b.T
    return out


def problem_full(p) -> np.ndarray:
    """The whole output of a ``synth.Problem`` in its output shape; rows that produce nothing are NaN."""
    if p.kind == "k_grouped":
        return np.stack([k_grouped_rows(p, g, np.arange(p.M)) for g in range(p.G)])
    rows = p.valid_rows()
    out = np.full((p.rows, p.N), np.nan, np.float64)
    out[rows] = problem_rows(p, rows)
    return out.reshape(p.out_shape())


# ----- convenience entry points in the library's own call shapes ---------------------------------------

def fp8_gemm_nt(a, sfa, b, sfb):
    """Dense: a [M,K] codes, sfa [K/128, >=M] MN-major, b [N,K] codes, sfb [ceil(N/128), K/128]."""
    M, K = a.shape
    N = b.shape[0]
    rows = np.arange(M, dtype=np.int64)
    return gemm_rows(a, rows, sfa.shape[1], sfa, b.reshape(1, N, K), sfb.reshape(1, *sfb.shape), rows,
                     np.zeros(M, np.int32), N, K)


def m_grouped_fp8_gemm_nt_contiguous(a, sfa, b, sfb, m_indices):
    """a [M_total,K], sfa [K/128, >=M_total], b [G,N,K], sfb [G, ceil(N/128), K/128], m_indices [M_total]."""
    M, K = a.shape
    G, N, _ = b.shape
    rows = np.nonzero(np.asarray(m_indices) >= 0)[0].astype(np.int64)
    out = np.full((M, N), np.nan)
    out[rows] = gemm_rows(a, rows, sfa.shape[1], sfa, b, sfb, rows, np.asarray(m_indices)[rows], N, K)
    return out


def m_grouped_fp8_gemm_nt_masked(a, sfa, b, sfb, masked_m):
    """a [G,M_max,K], sfa [G, K/128, >=M_max], b [G,N,K], sfb [G, ceil(N/128), K/128], masked_m [G]."""
    G, M_max, K = a.shape
    N = b.shape[1]
    nkb, Ma = sfa.shape[1], sfa.shape[2]
    rows = np.concatenate([g * M_max + np.arange(int(masked_m[g])) for g in range(G)]).astype(np.int64)
    g = rows // M_max
    out = np.full((G * M_max, N), np.nan)
    out[rows] = gemm_rows(a.reshape(G * M_max, K), g * nkb * Ma + rows - g * M_max, Ma, sfa, b, sfb, rows, g, N, K)
    return out.reshape(G, M_max, N)


def m_grouped_fp8_gemm_nt_nopad(a, sfa, b, sfb, counts):
    """a [M_total,K], sfa [K/128, >=M_total], b [G,N,K], sfb [G, ceil(N/128), K/128], counts [G]
    (sum(counts) <= M_total)."""
    M, K = a.shape
    G, N, _ = b.shape
    counts = np.asarray(counts, np.int64)
    off = np.concatenate([[0], np.cumsum(counts)[:-1]])
    rows = np.concatenate([off[g] + np.arange(counts[g]) for g in range(G)]).astype(np.int64)
    groups = np.concatenate([np.full(counts[g], g) for g in range(G)]).astype(np.int32)
    out = np.full((M, N), np.nan)
    if len(rows):
        out[rows] = gemm_rows(a, rows, sfa.shape[1], sfa, b, sfb, rows, groups, N, K)
    return out


def m_grouped_fp8_gemm_nn_contiguous(a, sfa, b, sfb, m_indices):
    """a [M_total,K], sfa [K/128, >=M_total], b [G,K,N], sfb [G, K/128, ceil(N/128)], m_indices [M_total]."""
    return m_grouped_fp8_gemm_nt_contiguous(a, sfa, np.ascontiguousarray(np.transpose(b, (0, 2, 1))),
                                            np.ascontiguousarray(np.transpose(sfb, (0, 2, 1))), m_indices)
