"""Seeded synthetic inputs for the FP8 NT GEMM family (dense, M-grouped contiguous, M-grouped masked).

This module only *prepares inputs*: it draws fp32 N(0,1) data from ``numpy.random.default_rng(seed)``,
quantises it to OCP e4m3 with power-of-two (UE8M0-representable) scales, and builds the grouping metadata
(``m_indices`` / ``masked_m`` / per-group ``counts``).  It holds none of the GEMM arithmetic.  Both the CPU oracle and the CUDA
path consume what it returns, and neither is imported here.

Recipe (fine-grained scaling, "FP8 GEMM kernels with fine-grained scaling", DeepGEMM-for-PPU README,
"Interfaces / Notices" and the scaling recipe (1, 128, 128) named by the MATE deep_gemm wrapper API list):

* A [rows, K]: one scale per (row, 128-K block); B [N, K] per group: one scale per 128x128 block.
* scale s = 2**e with e the smallest integer such that amax <= 448 * 2**e (= 2**ceil(log2(amax / 448))),
  computed exactly from the binary exponent of amax; amax == 0 gives s = 1.
* q = e4m3_RNE(x / s) (torch's fp32 -> float8_e4m3fn cast, round-to-nearest-even; |x / s| <= 448).
* sfa is stored MN-major ("LHS scale TMA-aligned and transposed"): [K/128][align4(rows)] fp32
  (masked: [G][K/128][align4(M_max)]).  sfb is [G][ceil(N/128)][K/128] fp32.
* Rows that no group owns (contiguous padding, masked rows >= masked_m[g], no-padding rows past the sum of
  the counts) hold garbage: random bytes, e4m3 NaN codes included, with random power-of-two scales.
* No-padding layout ("Grouped GEMMs (nopad layout)"): the groups' rows are concatenated in group order with
  no alignment; group g owns rows off_g .. off_g + counts[g] - 1, off_g = counts[0] + ... + counts[g-1].

Draw order per problem: group sizes (or masked_m) -> A fp32 -> B fp32 (group by group) -> garbage.
"""
from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import numpy as np

E4M3_MAX = 448.0
SCALE_BLOCK = 128  # K (and B's N) extent of one scale block
M_ALIGNMENT = 128  # per-segment padding of the contiguous layout


def align_up(x: int, a: int) -> int:
    return (x + a - 1) // a * a


def tma_aligned_rows(rows: int) -> int:
    """Row extent of the MN-major fp32 scale array: padded to a 16-byte multiple (4 floats)."""
    return align_up(rows, 4)


@dataclasses.dataclass
class Problem:
    """One GEMM problem in the layouts the library takes.

    kind       'dense' | 'contiguous' | 'masked' | 'nopad' | 'contiguous_nn' | 'k_grouped' | 'contiguous_w4a8' |
               'masked_w4a8'
    a          uint8 e4m3 codes, [rows, K]; masked: [G * M_max, K] (= [G, M_max, K] flattened)
    sfa        fp32, dense/contiguous [K/128, align4(rows)]; masked [G, K/128, align4(M_max)]
    b          uint8 e4m3 codes, [G, N, K] (G = 1 for dense); contiguous_nn: [G, K, N]; contiguous_w4a8: packed
               E2M1 codes [G, N, K/2] (element 2i in the low nibble of byte i)
    sfb        fp32, [G, ceil(N/128), K/128]; contiguous_nn: [G, K/128, ceil(N/128)]; contiguous_w4a8: one scale
               per (row, 32-K block), [G, K/32, align4(N)] (recipe (1, 32))
    m_indices  int32 [rows] (contiguous only): group id of each row, -1 for padding rows
    masked_m   int32 [G] (masked only): number of valid rows of each group
    counts     int32 [G]: contiguous -- valid rows per group (metadata); nopad -- the call's per-group row counts;
               k_grouped -- the groups' K extents (multiples of 128)
    k_grouped  a [M, sum K] and b [N, sum K] (both K-major, the groups' K segments concatenated); sfa
               [sum K / 128, align4(M)] and sfb [sum K / 128, align4(N)] (one scale per row and 128-K block,
               recipe (1, 1, 128)); c fp32 [G, M, N] or None; output fp32 [G, M, N]
    """

    kind: str
    M: int  # dense: M; contiguous: M_total (padded); masked: M_max; nopad: M_total (>= sum of counts)
    N: int
    K: int
    G: int
    a: np.ndarray
    sfa: np.ndarray
    b: np.ndarray
    sfb: np.ndarray
    m_indices: Optional[np.ndarray] = None
    masked_m: Optional[np.ndarray] = None
    expected_m: int = 0
    counts: Optional[np.ndarray] = None  # contiguous: valid rows per group
    name: str = ""
    c: Optional[np.ndarray] = None  # k_grouped: the accumulator input

    @property
    def rows(self) -> int:
        """Rows of the flattened output (= rows of ``a`` except for K-grouped problems, G x M)."""
        return self.G * self.M if self.kind == "k_grouped" else self.a.shape[0]

    def valid_rows(self) -> np.ndarray:
        """Global row indices (into ``a`` / the flattened output) that the GEMM must produce."""
        if self.kind == "k_grouped":
            return np.arange(self.G * self.M, dtype=np.int64)  # rows of the flattened [G * M, N] output
        if self.kind == "dense":
            return np.arange(self.M, dtype=np.int64)
        if self.kind in ("contiguous", "contiguous_nn", "contiguous_w4a8"):
            return np.nonzero(self.m_indices >= 0)[0].astype(np.int64)
        if self.kind == "nopad":
            return np.arange(int(np.sum(self.counts, dtype=np.int64)), dtype=np.int64)
        out = [g * self.M + np.arange(int(self.masked_m[g]), dtype=np.int64) for g in range(self.G)]
        return np.concatenate(out) if out else np.zeros(0, np.int64)

    def row_groups(self, rows: np.ndarray) -> np.ndarray:
        if self.kind == "k_grouped":
            return (rows // self.M).astype(np.int32)
        if self.kind == "dense":
            return np.zeros(len(rows), np.int32)
        if self.kind in ("contiguous", "contiguous_nn", "contiguous_w4a8"):
            return self.m_indices[rows].astype(np.int32)
        if self.kind == "nopad":
            ends = np.cumsum(np.asarray(self.counts, np.int64))
            return np.searchsorted(ends, rows, side="right").astype(np.int32)
        return (rows // self.M).astype(np.int32)

    def flops(self) -> int:
        if self.kind == "k_grouped":  # each group contracts its own K segment
            return 2 * self.M * self.N * self.K
        return 2 * int(len(self.valid_rows())) * self.N * self.K

    def out_shape(self):
        if self.kind == "k_grouped":
            return (self.G, self.M, self.N)
        if self.kind in ("masked", "masked_w4a8"):
            return (self.G, self.M, self.N)
        return (self.rows, self.N)


# ----------------------------------------------------------------------------------------------
# quantisation (input preparation)
# ----------------------------------------------------------------------------------------------

def pow2_scale_exponent(amax: np.ndarray) -> np.ndarray:
    """Smallest integer e with amax <= 448 * 2**e, exactly (amax >= 0, fp32).  amax == 0 -> 0.

    With amax = f * 2**ea (frexp, f in [0.5, 1)) and 448 = 0.875 * 2**9:
    amax <= 0.875 * 2**(9 + e)  <=>  e >= ea - 9 when f <= 0.875, else e >= ea - 8.
    """
    f, ea = np.frexp(amax.astype(np.float64))
    e = ea.astype(np.int64) - 9 + (f > 0.875).astype(np.int64)
    return np.where(amax > 0, e, 0)


E2M1_MAX = 6.0
# magnitudes of the E2M1 codes 0..7 (OCP MX format: 1 sign, 2 exponent (bias 1), 1 mantissa bit, no Inf/NaN)
_E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def pow2_scale_exponent_e2m1(amax: np.ndarray) -> np.ndarray:
    """Smallest integer e with amax <= 6 * 2**e, exactly; amax == 0 -> 0.  With amax = f * 2**ea (f in [0.5, 1))
    and 6 = 0.75 * 2**3: e >= ea - 3 when f <= 0.75, else e >= ea - 2."""
    f, ea = np.frexp(amax.astype(np.float64))
    e = ea.astype(np.int64) - 3 + (f > 0.75).astype(np.int64)
    return np.where(amax > 0, e, 0)


def _to_e2m1_codes(y: np.ndarray) -> np.ndarray:
    """|y| <= 6 -> 4-bit E2M1 codes (uint8 0..15), round to nearest, ties to the even code (mantissa bit 0)."""
    mag = np.abs(np.asarray(y, np.float64))
    hi = np.clip(np.searchsorted(_E2M1_MAGNITUDES, mag, side="left"), 0, 7)
    lo = np.clip(hi - 1, 0, 7)
    d_lo = mag - _E2M1_MAGNITUDES[lo]
    d_hi = _E2M1_MAGNITUDES[hi] - mag
    code = np.where(d_lo < d_hi, lo, np.where(d_hi < d_lo, hi, np.where(lo % 2 == 0, lo, hi)))
    return (code | np.where(np.signbit(y) & (code != 0), 8, 0)).astype(np.uint8)


def quantize_rows_e2m1(x: np.ndarray):
    """x fp32 [R, K] -> (codes uint8 [R, K] in 0..15, scales fp32 [R, K/32]), one scale per (row, 32-K block)."""
    R, K = x.shape
    assert K % 32 == 0
    xb = x.reshape(R, K // 32, 32)
    e = pow2_scale_exponent_e2m1(np.abs(xb).max(axis=2))
    q = np.ldexp(xb.astype(np.float64), -e[:, :, None])
    return _to_e2m1_codes(q.reshape(R, K)), np.ldexp(np.ones_like(e, dtype=np.float32), e).astype(np.float32)


def pack_e2m1(codes: np.ndarray) -> np.ndarray:
    """4-bit codes [..., K] -> bytes [..., K/2]: element 2i in the low nibble, 2i + 1 in the high nibble."""
    c = np.asarray(codes, np.uint8)
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def _to_e4m3_codes(x: np.ndarray) -> np.ndarray:
    import torch

    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def quantize_rows(x: np.ndarray):
    """x fp32 [R, K] -> (codes uint8 [R, K], scales fp32 [R, K/128]) with one scale per (row, 128-K block)."""
    R, K = x.shape
    assert K % SCALE_BLOCK == 0
    nkb = K // SCALE_BLOCK
    xb = x.reshape(R, nkb, SCALE_BLOCK)
    e = pow2_scale_exponent(np.abs(xb).max(axis=2))  # [R, nkb]
    q = np.ldexp(xb, -e[:, :, None]).astype(np.float32, copy=False)  # exact: a power-of-two scaling
    codes = _to_e4m3_codes(q.reshape(R, K))
    return codes, np.ldexp(np.ones_like(e, dtype=np.float32), e).astype(np.float32)


def quantize_blocks(x: np.ndarray):
    """x fp32 [N, K] -> (codes uint8 [N, K], scales fp32 [ceil(N/128), K/128]), one scale per 128x128 block."""
    N, K = x.shape
    assert K % SCALE_BLOCK == 0
    nkb = K // SCALE_BLOCK
    nnb = (N + SCALE_BLOCK - 1) // SCALE_BLOCK
    pad = nnb * SCALE_BLOCK - N
    xp = np.pad(x, ((0, pad), (0, 0))) if pad else x
    xb = xp.reshape(nnb, SCALE_BLOCK, nkb, SCALE_BLOCK)
    e = pow2_scale_exponent(np.abs(xb).max(axis=(1, 3)))  # [nnb, nkb]
    q = np.ldexp(xb, -e[:, None, :, None]).astype(np.float32, copy=False).reshape(nnb * SCALE_BLOCK, K)[:N]
    return _to_e4m3_codes(q), np.ldexp(np.ones_like(e, dtype=np.float32), e).astype(np.float32)


def _garbage_rows(rng: np.random.Generator, codes: np.ndarray, sfa_t: np.ndarray, rows: np.ndarray):
    """Fill rows that no group owns with random bytes (NaN codes included) and random 2**j scales."""
    if len(rows) == 0:
        return
    K = codes.shape[1]
    junk = rng.integers(0, 256, size=(len(rows), K), dtype=np.uint8)
    junk[:, 0] = 0x7F  # make sure every garbage row carries an e4m3 NaN code
    codes[rows] = junk
    nkb = sfa_t.shape[0]
    sfa_t[:, rows] = np.ldexp(1.0, rng.integers(-10, 11, size=(nkb, len(rows)))).astype(np.float32)


def _draw_normal(rng: np.random.Generator, shape) -> np.ndarray:
    return rng.standard_normal(size=shape, dtype=np.float32)


def _quantize_b(rng: np.random.Generator, G: int, N: int, K: int):
    nkb = K // SCALE_BLOCK
    nnb = (N + SCALE_BLOCK - 1) // SCALE_BLOCK
    b = np.empty((G, N, K), np.uint8)
    sfb = np.empty((G, nnb, nkb), np.float32)
    for g in range(G):
        b[g], sfb[g] = quantize_blocks(_draw_normal(rng, (N, K)))
    return b, sfb


# ----------------------------------------------------------------------------------------------
# problem builders
# ----------------------------------------------------------------------------------------------

def make_dense(M: int, N: int, K: int, seed: int = 0, name: str = "") -> Problem:
    rng = np.random.default_rng(seed)
    codes, s = quantize_rows(_draw_normal(rng, (M, K)))
    Ma = tma_aligned_rows(M)
    sfa = np.ones((K // SCALE_BLOCK, Ma), np.float32)
    sfa[:, :M] = s.T
    b, sfb = _quantize_b(rng, 1, N, K)
    return Problem("dense", M, N, K, 1, codes, sfa, b, sfb, name=name or f"dense M={M} N={N} K={K}")


def make_contiguous(counts: Sequence[int], N: int, K: int, seed: int = 0, name: str = "",
                    rng: Optional[np.random.Generator] = None, alignment: int = M_ALIGNMENT) -> Problem:
    """Groups' token segments concatenated along M, each padded to ``alignment`` rows (padding: -1)."""
    rng = rng if rng is not None else np.random.default_rng(seed)
    counts = np.asarray(counts, np.int64)
    G = len(counts)
    padded = np.array([align_up(int(c), alignment) for c in counts], np.int64)
    M_total = int(padded.sum())
    m_indices = np.full(M_total, -1, np.int32)
    starts = np.concatenate([[0], np.cumsum(padded)[:-1]]).astype(np.int64)
    for g in range(G):
        m_indices[starts[g]:starts[g] + counts[g]] = g
    valid = np.nonzero(m_indices >= 0)[0]
    invalid = np.nonzero(m_indices < 0)[0]
    codes = np.zeros((M_total, K), np.uint8)
    Ma = tma_aligned_rows(M_total)
    sfa = np.ones((K // SCALE_BLOCK, Ma), np.float32)
    qa, s = quantize_rows(_draw_normal(rng, (len(valid), K)))
    codes[valid] = qa
    sfa[:, valid] = s.T
    b, sfb = _quantize_b(rng, G, N, K)
    _garbage_rows(rng, codes, sfa, invalid)
    return Problem("contiguous", M_total, N, K, G, codes, sfa, b, sfb, m_indices=m_indices,
                   counts=counts.astype(np.int32), name=name or f"contiguous G={G} N={N} K={K}")


def make_contiguous_nn(counts: Sequence[int], N: int, K: int, seed: int = 0, name: str = "",
                       rng: Optional[np.random.Generator] = None) -> Problem:
    """The contiguous layout with B in the NN orientation: the same draws as ``make_contiguous``, with each
    group's B stored [K, N] (N contiguous) and its 128x128 block scales [K/128, ceil(N/128)]."""
    p = make_contiguous(counts, N, K, seed=seed, rng=rng)
    p.kind = "contiguous_nn"
    p.b = np.ascontiguousarray(p.b.transpose(0, 2, 1))
    p.sfb = np.ascontiguousarray(p.sfb.transpose(0, 2, 1))
    p.name = name or f"contiguous NN G={p.G} N={N} K={K}"
    return p


def make_k_grouped(ks: Sequence[int], M: int, N: int, seed: int = 0, with_c: bool = True, name: str = "",
                   rng: Optional[np.random.Generator] = None) -> Problem:
    """K-grouped operands: A [M, sum K] and B [N, sum K] with one scale per (row, 128-K block) (recipe
    (1, 1, 128)); group g contracts its own K segment.  c ~ N(0, 1) fp32 [G, M, N] when ``with_c``."""
    rng = rng if rng is not None else np.random.default_rng(seed)
    ks = np.asarray(ks, np.int64)
    assert (ks >= 0).all() and (ks % SCALE_BLOCK == 0).all()
    G, Kt = len(ks), int(ks.sum())
    a, sa = quantize_rows(_draw_normal(rng, (M, Kt)))
    b, sb = quantize_rows(_draw_normal(rng, (N, Kt)))
    sfa = np.ones((Kt // SCALE_BLOCK, tma_aligned_rows(M)), np.float32)
    sfa[:, :M] = sa.T
    sfb = np.ones((Kt // SCALE_BLOCK, tma_aligned_rows(N)), np.float32)
    sfb[:, :N] = sb.T
    c = _draw_normal(rng, (G, M, N)) if with_c else None
    return Problem("k_grouped", M, N, Kt, G, a, sfa, b, sfb, counts=ks.astype(np.int32), c=c,
                   name=name or f"k-grouped G={G} M={M} N={N}")


def make_contiguous_w4a8(counts: Sequence[int], N: int, K: int, seed: int = 0, name: str = "",
                         rng: Optional[np.random.Generator] = None) -> Problem:
    """The contiguous layout with B in E2M1 (FP4, packed two per byte) and one B scale per (row, 32-K block);
    A as in ``make_contiguous`` (e4m3, one scale per (row, 128-K block))."""
    rng = rng if rng is not None else np.random.default_rng(seed)
    p = make_contiguous(counts, N, K, rng=rng)
    G = p.G
    b = np.empty((G, N, K // 2), np.uint8)
    sfb = np.ones((G, K // 32, tma_aligned_rows(N)), np.float32)
    for g in range(G):
        codes, sb = quantize_rows_e2m1(_draw_normal(rng, (N, K)))
        b[g] = pack_e2m1(codes)
        sfb[g, :, :N] = sb.T
    p.kind = "contiguous_w4a8"
    p.b, p.sfb = b, sfb
    p.name = name or f"contiguous W4A8 G={G} N={N} K={K}"
    return p


def make_masked_w4a8(G: int, M_max: int, N: int, K: int, masked_m: Optional[Sequence[int]] = None, seed: int = 0,
                     expected_m: int = 0, name: str = "") -> Problem:
    """The masked layout with B in E2M1 and one B scale per (row, 32-K block), as ``make_contiguous_w4a8``."""
    p = make_masked(G, M_max, N, K, masked_m=masked_m, seed=seed, expected_m=expected_m)
    rng = np.random.default_rng(seed + 1)
    b = np.empty((G, N, K // 2), np.uint8)
    sfb = np.ones((G, K // 32, tma_aligned_rows(N)), np.float32)
    for g in range(G):
        codes, sb = quantize_rows_e2m1(_draw_normal(rng, (N, K)))
        b[g] = pack_e2m1(codes)
        sfb[g, :, :N] = sb.T
    p.kind = "masked_w4a8"
    p.b, p.sfb = b, sfb
    p.name = name or f"masked W4A8 G={G} M_max={M_max} N={N} K={K}"
    return p


def make_nopad(counts: Sequence[int], N: int, K: int, seed: int = 0, extra_rows: int = 0, name: str = "",
               rng: Optional[np.random.Generator] = None) -> Problem:
    """Groups' rows concatenated with no padding, then ``extra_rows`` rows that no group owns (garbage)."""
    rng = rng if rng is not None else np.random.default_rng(seed)
    counts = np.asarray(counts, np.int64)
    assert (counts >= 0).all()
    G = len(counts)
    valid = int(counts.sum())
    M_total = valid + int(extra_rows)
    codes = np.zeros((M_total, K), np.uint8)
    sfa = np.ones((K // SCALE_BLOCK, tma_aligned_rows(max(M_total, 1))), np.float32)
    qa, s = quantize_rows(_draw_normal(rng, (valid, K)))
    codes[:valid] = qa
    sfa[:, :valid] = s.T
    b, sfb = _quantize_b(rng, G, N, K)
    _garbage_rows(rng, codes, sfa, np.arange(valid, M_total))
    return Problem("nopad", M_total, N, K, G, codes, sfa, b, sfb, counts=counts.astype(np.int32),
                   name=name or f"nopad G={G} N={N} K={K}")


def make_masked(G: int, M_max: int, N: int, K: int, masked_m: Optional[Sequence[int]] = None,
                seed: int = 0, expected_m: int = 0, name: str = "") -> Problem:
    """[G, M_max, K] activations; rows >= masked_m[g] of each group are garbage and must stay unwritten.
    masked_m, when not given, is drawn uniformly from [0, M_max] (inclusive)."""
    rng = np.random.default_rng(seed)
    if masked_m is None:
        masked_m = rng.integers(0, M_max, endpoint=True, size=G)
    masked_m = np.asarray(masked_m, np.int32)
    assert masked_m.shape == (G,) and (masked_m >= 0).all() and (masked_m <= M_max).all()
    nkb = K // SCALE_BLOCK
    codes, s = quantize_rows(_draw_normal(rng, (G * M_max, K)))
    Ma = tma_aligned_rows(M_max)
    sfa = np.ones((G, nkb, Ma), np.float32)
    sfa[:, :, :M_max] = s.reshape(G, M_max, nkb).transpose(0, 2, 1)
    b, sfb = _quantize_b(rng, G, N, K)
    for g in range(G):
        rows = np.arange(int(masked_m[g]), M_max)
        view = codes[g * M_max:(g + 1) * M_max]
        _garbage_rows(rng, view, sfa[g], rows)
    return Problem("masked", M_max, N, K, G, codes, sfa, b, sfb, masked_m=masked_m,
                   expected_m=expected_m or M_max, name=name or f"masked G={G} M_max={M_max} N={N} K={K}")


def with_fp32_scales(p: Problem, seed: int = 0) -> Problem:
    """The same problem with every A and B scale multiplied by its own seeded factor drawn uniformly from [1, 2)
    (fp32): scales that are no longer powers of two (each 128-K block and 128x128 block gets its own mantissa).
    The e4m3 codes are unchanged.  Input for the fp32 scale-promotion path."""
    rng = np.random.default_rng(seed + 0x5CA1E)
    p.sfa = (p.sfa * rng.uniform(1.0, 2.0, size=p.sfa.shape)).astype(np.float32)
    p.sfb = (p.sfb * rng.uniform(1.0, 2.0, size=p.sfb.shape)).astype(np.float32)
    p.name = p.name + " (fp32 scales)"
    return p


def zipf_counts(total: int, G: int, s: float) -> np.ndarray:
    """Deterministic Zipf(s) split of ``total`` tokens over G groups: w_g = (g+1)^-s, floor(total * w / sum w)
    plus largest-remainder rounding so that the counts sum to ``total`` (ties go to the lower group id)."""
    w = (np.arange(1, G + 1, dtype=np.float64)) ** (-s)
    exact = total * w / w.sum()
    counts = np.floor(exact).astype(np.int64)
    rem = total - int(counts.sum())
    order = np.argsort(-(exact - counts), kind="stable")
    counts[order[:rem]] += 1
    return counts


# The five workloads (all seed 0); 6: workload 5's token split in the no-padding layout; 7: workload 3 with B
# in the NN orientation; 8: workload 3's token counts as the K extents of a K-grouped (weight-gradient) GEMM;
# 9: workload 3 with B in E2M1 (W4A8).
WORKLOAD_NAMES = {
    1: "dense FP8 NT GEMM M=128 N=256 K=512",
    2: "dense FP8 NT GEMM M=4096 N=7168 K=7168",
    3: "M-grouped contiguous FP8 GEMM G=8 N=4096 K=7168, tokens U[1024,8192] per group",
    4: "M-grouped masked FP8 GEMM G=32 M_max=256 N=7168 K=2048, masked_m U[0,256], expected_m=128",
    5: "M-grouped contiguous FP8 GEMM G=64 N=7168 K=2048, Zipf(1.2) split of 65536 tokens",
    6: "M-grouped no-padding FP8 GEMM G=64 N=7168 K=2048, Zipf(1.2) split of 65536 tokens",
    7: "M-grouped contiguous FP8 NN GEMM (B [G, K, N]) G=8 N=4096 K=7168, tokens U[1024,8192] per group",
    8: "K-grouped FP8 NT GEMM, fp32 D_g = A_g B_g^T, G=8 M=4096 N=7168, K_g = tokens U[1024,8192] rounded up to 128",
    9: "M-grouped contiguous W4A8 GEMM (e4m3 A x E2M1 B) G=8 N=4096 K=7168, tokens U[1024,8192] per group",
    10: "dense FP8 NT GEMM M=4096 N=7168 K=7168 with fp32 (non-power-of-two) scales",
}


def make_config(i: int, seed: int = 0) -> Problem:
    if i == 1:
        return make_dense(128, 256, 512, seed, name=WORKLOAD_NAMES[1])
    if i == 2:
        return make_dense(4096, 7168, 7168, seed, name=WORKLOAD_NAMES[2])
    if i == 3:
        rng = np.random.default_rng(seed)
        counts = rng.integers(1024, 8192, endpoint=True, size=8)
        return make_contiguous(counts, 4096, 7168, rng=rng, name=WORKLOAD_NAMES[3])
    if i == 4:
        return make_masked(32, 256, 7168, 2048, seed=seed, expected_m=128, name=WORKLOAD_NAMES[4])
    if i == 5:
        rng = np.random.default_rng(seed)
        return make_contiguous(zipf_counts(65536, 64, 1.2), 7168, 2048, rng=rng, name=WORKLOAD_NAMES[5])
    if i == 9:
        rng = np.random.default_rng(seed)
        counts = rng.integers(1024, 8192, endpoint=True, size=8)
        return make_contiguous_w4a8(counts, 4096, 7168, rng=rng, name=WORKLOAD_NAMES[9])
    if i == 8:
        rng = np.random.default_rng(seed)
        counts = rng.integers(1024, 8192, endpoint=True, size=8)
        return make_k_grouped([align_up(int(c), SCALE_BLOCK) for c in counts], 4096, 7168, rng=rng, with_c=False,
                              name=WORKLOAD_NAMES[8])
    if i == 7:
        rng = np.random.default_rng(seed)
        counts = rng.integers(1024, 8192, endpoint=True, size=8)
        return make_contiguous_nn(counts, 4096, 7168, rng=rng, name=WORKLOAD_NAMES[7])
    if i == 6:
        rng = np.random.default_rng(seed)
        return make_nopad(zipf_counts(65536, 64, 1.2), 7168, 2048, rng=rng, name=WORKLOAD_NAMES[6])
    if i == 10:
        p = with_fp32_scales(make_dense(4096, 7168, 7168, seed), seed)
        p.name = WORKLOAD_NAMES[10]
        return p
    raise ValueError(f"unknown config {i}")


def to_torch(p: Problem, device="cuda"):
    """Device copies of a problem's arrays in the library's call layout (no arithmetic)."""
    import torch

    def t(x):
        return torch.from_numpy(np.ascontiguousarray(x)).to(device)

    out = {"a": t(p.a), "sfa": t(p.sfa), "b": t(p.b), "sfb": t(p.sfb)}
    if p.kind == "dense":
        out["b"] = out["b"].view(p.N, p.K)
        out["sfb"] = out["sfb"].view(p.sfb.shape[1], p.sfb.shape[2])
    if p.kind in ("masked", "masked_w4a8"):
        out["a"] = out["a"].view(p.G, p.M, p.K)
        out["masked_m"] = t(p.masked_m)
    if p.kind in ("contiguous", "contiguous_nn", "contiguous_w4a8"):
        out["m_indices"] = t(p.m_indices)
    if p.kind == "nopad":
        out["counts"] = t(p.counts)
    if p.kind == "k_grouped":
        out["ks"] = t(p.counts)
        if p.c is not None:
            out["c"] = t(p.c)
    return out
