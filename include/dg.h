/*
 * dg.h -- C ABI of the B200 (sm_100a) FP8 NT GEMM library with fine-grained scaling.
 *
 * The operation ("FP8 GEMM kernels with fine-grained scaling", DeepGEMM-for-PPU README, "Interfaces"):
 *
 *     D[m][n] = bf16_RNE( sum_kb sfa(m, kb) * sfb(g, n/128, kb) * sum_{k in block kb} A[m][k] * B_g[n][k] )
 *
 * A and B are OCP e4m3 ("e4m3fn") codes, one byte per element.  A has one scale per (row, 128-K block)
 * and B one scale per 128x128 block (the (1, 128, 128) recipe of the MATE deep_gemm wrapper API list).
 * Only the NT form exists: A is [M, K] and B is [N, K], both K-major ("non-transposed LHS, transposed
 * RHS", README "Notices").  Accumulation is fp32 on the tensor cores.
 *
 * Scale layouts (README "Notices": the LHS scale is TMA-aligned and transposed):
 *   sfa  fp32, MN-major: [K/128][ld] with ld = dg_get_tma_aligned_size(rows, 4) (rows rounded up to a
 *        multiple of 4 so every K block's column starts on 16 bytes).  Masked layout: [G][K/128][ld(M_max)].
 *   sfb  fp32, [G][ceil(N/128)][K/128] (G = 1 for the dense call).
 * Scale values.  By default every scale must be a power of two in [2^-126, 2^127] (a UE8M0 value): the
 * block-scaled tensor-core MMA applies the scales as exponents.  The scale pre-pass checks every scale the
 * call reads (the A scales of rows the call owns, all B scales) and reports one with a sign, mantissa bits,
 * Inf or NaN as DG_ERR_BAD_SCALE through dg_check_device_error(); the results of that call are then wrong.
 * A zero scale is taken as 2^-127.  After dg_set_fp32_scale_promotion(1) every call takes any finite fp32
 * scales: every 128-K block's partial product (W4A8: every 32-K sub-block's) is multiplied by sfa * sfb and
 * added in fp32 (the "promotion operations" of the DeepGEMM-for-PPU README, "Optimizations"), at a lower speed.
 *
 * Common conventions
 *   - All array arguments are device pointers owned by the caller.  The library keeps no reference after the
 *     call returns; its only per-call memory is stream-ordered scratch (packed scales, the NN call's transposed
 *     B) taken from and returned to a device memory pool on `stream` (dg_fp8_gemm_nt_noalloc takes none).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default stream).  m_indices and
 *     masked_m are read only on the device, so the host never synchronises.
 *   - Arguments are validated before anything is launched; a bad argument returns a negative dg_status,
 *     launches nothing and sets the message returned by dg_last_error().
 *   - Rows the GEMM does not own are never written: contiguous rows with m_indices == -1, masked rows
 *     with index >= masked_m[g] (all of D[g] when masked_m[g] == 0).
 *   - Pointer alignment: a, b, d, sfa, sfb 16-byte aligned; m_indices, masked_m 4-byte aligned.
 *   - Shapes: K % 128 == 0, N % 16 == 0, N, K > 0, all extents below 2^31 elements per dimension.
 *   - Device-side faults are not expected.  Every wait inside the kernel is bounded; a kernel that gives
 *     up records a code that dg_check_device_error() returns (DG_ERR_DEVICE_TIMEOUT, DG_ERR_BAD_GROUP or
 *     DG_ERR_BAD_SCALE).
 *   - Settings (dg_set_m_alignment_for_contiguous_layout, dg_set_num_sms, dg_set_cta_pair_policy, dg_set_swap_policy,
 *     dg_set_fp32_scale_promotion, dg_debug_bounded_wait, dg_debug_clock_record) are process-wide, not
 *     per thread or per stream.  Setting one while another thread calls the library is defined (each value is
 *     an atomic) but that call sees whichever value was in force when it read it, so two users of one process
 *     that want different settings must serialise their calls.  The M alignment also changes how every
 *     later contiguous call's M_total is validated.
 *   - The first call on a device, and the first call of each kernel configuration (tile width, CTA pair or
 *     single CTA, layout) on it, does one-time set-up that is not a stream operation: device attribute
 *     queries, symbol address look-ups, the kernel's shared-memory attribute and its cluster occupancy.  Make
 *     one eager call of each shape class before capturing a stream into a CUDA graph.
 */
#ifndef DG_H_
#define DG_H_

#if defined(__GNUC__)
#define DG_EXPORT __attribute__((visibility("default")))
#else
#define DG_EXPORT
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *dg_stream_t; /* same type as cudaStream_t */

typedef enum {
    DG_OK = 0,
    DG_ERR_INVALID_ARG = -1,   /* null pointer, bad extent, bad group count */
    DG_ERR_ALIGNMENT = -2,     /* pointer or extent not aligned as required */
    DG_ERR_UNSUPPORTED = -3,   /* device is not sm_100, or a shape outside the supported set */
    DG_ERR_CUDA = -4,          /* a CUDA runtime/driver call failed */
    DG_ERR_DEVICE_TIMEOUT = -5,/* (device error word) a bounded wait inside the kernel ran out */
    DG_ERR_BAD_GROUP = -6,     /* (device error word) a group id outside [-1, G), masked_m outside [0, M_max],
                                  or no-padding counts that are negative or sum past M_total */
    DG_ERR_BAD_SCALE = -7      /* (device error word) a scale read by a block-scaled call is not a power of two */
} dg_status;

/* Per-segment M padding of the contiguous layout: each group's rows start on a multiple of this (128 unless
 * set to 256).  README "Grouped GEMMs (contiguous layout)": segments are aligned to the GEMM M block size;
 * MATE docs "Contiguous Grouped GEMM Alignment": the alignment is 128 by default, 256 on request, nothing else. */
DG_EXPORT int dg_get_m_alignment_for_contiguous_layout(void);

/* Sets that alignment for the contiguous calls that follow (process-wide, see "Common conventions").  128 or 256; returns the value set, or DG_ERR_INVALID_ARG (nothing changes) for any other value.
 * With 256 every group owns whole 256-row windows, so the 2-CTA tiles never straddle two groups; results do
 * not depend on the alignment, only M_total's validation does (M_total % alignment == 0). */
DG_EXPORT int dg_set_m_alignment_for_contiguous_layout(int alignment);

/* Rows rounded up so that `mn` elements of `elem_bytes` bytes fill whole 16-byte units (README
 * "Utilities": get_tma_aligned_size).  Returns -1 for a non-positive elem_bytes. */
DG_EXPORT int dg_get_tma_aligned_size(int mn, int elem_bytes);

/* Cap on the persistent grid (README "Utilities": set_num_sms / get_num_sms).  n <= 0 restores the
 * default (every SM of the current device).  Returns the value now in force, or a negative status. */
DG_EXPORT int dg_set_num_sms(int n);
DG_EXPORT int dg_get_num_sms(void);

/* Output tiles of an M x N problem with block_m x block_n tiles: ceil(M/block_m) * ceil(N/block_n).
 * README "Unaligned block sizes": M=256, N=7168 gives 112 tiles at 128x128 and 128 tiles at 128x112. */
DG_EXPORT long long dg_num_tiles(long long M, long long N, int block_m, int block_n);

/* The N tile the library picks for `num_m_blocks` 128-row single-CTA tiles of an N-wide output on `num_sms`
 * SMs: the candidate (224, 192, 160, 128) minimising waves x (128 + BN), the operand rows a CTA loads per K
 * block (README "Unaligned block sizes": wave quantisation on the SM count). */
DG_EXPORT int dg_select_block_n(long long num_m_blocks, int N, int num_sms);

/* Dense NT GEMM (README "Normal dense GEMMs", gemm_fp8_fp8_bf16_nt).
 *   a [M][K] e4m3, sfa [K/128][ld(M)] fp32, b [N][K] e4m3, sfb [ceil(N/128)][K/128] fp32,
 *   d [M][N] bf16 row-major (written in full).  M == 0 is a no-op.
 *   Short calls (K <= 2048 and 2*M*N*K <= 2^34) launch one kernel instead of the scale pre-pass and the
 *   block-scaled GEMM: the fp32-promotion GEMM, which reads the scales directly and still requires them to be
 *   powers of two (DG_ERR_BAD_SCALE), reading a zero scale as 2^-127.  Results agree with the block-scaled path
 *   within the tolerance of fp32 accumulation, not bit for bit. */
DG_EXPORT int dg_fp8_gemm_nt(const void *a, const float *sfa, const void *b, const float *sfb, void *d,
                   int M, int N, int K, dg_stream_t stream);

/* M-grouped GEMM, contiguous layout (README "Grouped GEMMs (contiguous layout)").
 *   a [M_total][K] e4m3 (group segments concatenated, each padded to dg_get_m_alignment...()),
 *   sfa [K/128][ld(M_total)], b [G][N][K] e4m3, sfb [G][ceil(N/128)][K/128],
 *   m_indices int32 [M_total] on the device: the group of each row, -1 for a padding row.  Every
 *   128-row block must hold one group (its first row decides; a block whose first row is -1 is skipped),
 *   d [M_total][N] bf16: rows with m_indices == -1 are left untouched.
 *   M_total % dg_get_m_alignment_for_contiguous_layout() == 0, 1 <= G <= 65534. */
DG_EXPORT int dg_m_grouped_fp8_gemm_nt_contiguous(const void *a, const float *sfa, const void *b, const float *sfb,
                                        void *d, const int *m_indices, int M_total, int N, int K, int G,
                                        dg_stream_t stream);

/* M-grouped GEMM, masked layout (README "Grouped GEMMs (masked layout)").
 *   a [G][M_max][K] e4m3, sfa [G][K/128][ld(M_max)], b [G][N][K] e4m3, sfb [G][ceil(N/128)][K/128],
 *   masked_m int32 [G] on the device: rows 0..masked_m[g]-1 of group g are computed,
 *   d [G][M_max][N] bf16: rows >= masked_m[g] are left untouched.
 *   expected_m: the caller's guess of a typical masked_m, used only to pick the tile shape; results do
 *   not depend on it.  1 <= G <= 1024. */
DG_EXPORT int dg_m_grouped_fp8_gemm_nt_masked(const void *a, const float *sfa, const void *b, const float *sfb,
                                    void *d, const int *masked_m, int G, int M_max, int N, int K,
                                    int expected_m, dg_stream_t stream);

/* M-grouped GEMM, contiguous layout with B in the NN orientation (MATE docs, 0.2.7 additions,
 * `m_grouped_fp8_gemm_nn_contiguous`: B is [num_groups, K, N]; recipe (1, 128, 128) only).
 *   Same as dg_m_grouped_fp8_gemm_nt_contiguous except
 *   b [G][K][N] e4m3 (N contiguous) and sfb [G][K/128][ceil(N/128)] (B's 128x128 block scales in B's
 *   orientation): D[m][n] = sum_k A[m][k] * B_g[k][n] with the block scales as in the NT call.
 *   With swapped-operand tiles (dg_set_swap_policy; used whenever the policy allows and M_total / 128 <= 1024) the
 *   kernel reads B in place: each K block of 128 of B's columns is loaded as an MN-major tile (128 K-rows of 128
 *   bytes).  Otherwise the library transposes B into stream-ordered scratch of G*N*K bytes (one HBM read and write
 *   of B) and runs the NT kernel on it; the scratch is released in stream order when the call's work is done. */
DG_EXPORT int dg_m_grouped_fp8_gemm_nn_contiguous(const void *a, const float *sfa, const void *b, const float *sfb,
                                        void *d, const int *m_indices, int M_total, int N, int K, int G,
                                        dg_stream_t stream);

/* M-grouped GEMM, contiguous layout, W4A8: e4m3 A times E2M1 (FP4) B (MATE docs, 0.2.7 additions,
 * `m_grouped_fp8_fp4_gemm_nt_contiguous`: "FP8 E4M3 A plus packed E2M1 FP4 B", recipe_a (1, 128), recipe_b (1, 32)).
 *   Same as dg_m_grouped_fp8_gemm_nt_contiguous except
 *   b [G][N][K/2] bytes: E2M1 codes (sign, 2 exponent bits with bias 1, 1 mantissa bit) packed two per byte, code
 *     k in the low nibble of byte k/2 when k is even, the high nibble when odd; 32-byte aligned;
 *   sfb [G][K/32][ld(N)] fp32, MN-major: one power-of-two scale per (row n, 32-K block):
 *   D[m][n] = sum over 128-K blocks kb of sfa(m, kb) * sum over its four 32-K sub-blocks j of sfb(g, 4 kb + j, n)
 *             * sum_{k in the sub-block} A[m][k] * B_g[n][k].
 *   Scales must be powers of two (others: DG_ERR_BAD_SCALE) unless fp32 scale promotion is on
 *   (dg_set_fp32_scale_promotion), which takes any finite scales and then needs sfb 16-byte aligned. */
DG_EXPORT int dg_m_grouped_fp8_fp4_gemm_nt_contiguous(const void *a, const float *sfa, const void *b,
                                            const float *sfb, void *d, const int *m_indices, int M_total, int N, int K,
                                            int G, dg_stream_t stream);

/* M-grouped GEMM, masked layout, W4A8 (`m_grouped_fp8_fp4_gemm_nt_masked`, same page): as
 * dg_m_grouped_fp8_gemm_nt_masked except b [G][N][K/2] bytes of packed E2M1 codes (32-byte aligned) and
 * sfb [G][K/32][ld(N)] fp32, one scale per (row n, 32-K block), as in dg_m_grouped_fp8_fp4_gemm_nt_contiguous
 * (powers of two, or any finite scales with sfb 16-byte aligned while fp32 scale promotion is on). */
DG_EXPORT int dg_m_grouped_fp8_fp4_gemm_nt_masked(const void *a, const float *sfa, const void *b, const float *sfb,
                                        void *d, const int *masked_m, int G, int M_max, int N, int K, int expected_m,
                                        dg_stream_t stream);

/* K-grouped GEMM (MATE docs, 0.2.7 additions, `k_grouped_fp8_gemm_nt_contiguous`: recipe (1, 1, 128), host K
 * extents, C accumulated into D), e.g. the per-expert weight gradient of an MoE layer.
 *   a [M][sum ks] e4m3 and b [N][sum ks] e4m3, both K-major, the groups' K segments concatenated in group order;
 *   sfa [sum ks / 128][ld(M)] and sfb [sum ks / 128][ld(N)] fp32: one scale per (row, 128-K block), MN-major;
 *   ks: G host ints, each a multiple of 128 (0 allowed); ks_device: the same G values on the device (the kernel
 *   reads these; they must equal ks);
 *   d fp32 [G][M][N]:  D_g = C_g + sum over group g's 128-K blocks kb of sfa(m, kb) * sfb(n, kb) *
 *   sum_{k in kb} A[m][k] * B[n][k].  c: NULL (D_g = the sum), another [G][M][N] fp32 buffer (copied into d
 *   first), or d itself (accumulate in place).  A group with ks = 0 gives D_g = C_g (0 without C).
 *   1 <= G <= 1024, N % 16 == 0, 16-byte aligned a, b, c, d.  Device values of ks_device that are negative or
 *   not multiples of 128 are reported by dg_check_device_error() as DG_ERR_BAD_GROUP.  Scales must be powers of
 *   two (others: DG_ERR_BAD_SCALE) unless fp32 scale promotion is on, which takes any finite scales and then
 *   needs sfb 16-byte aligned (else DG_ERR_ALIGNMENT). */
DG_EXPORT int dg_k_grouped_fp8_gemm_nt_contiguous(const void *a, const float *sfa, const void *b, const float *sfb,
                                        float *d, const float *c, const int *ks, const int *ks_device, int G, int M,
                                        int N, dg_stream_t stream);

/* M-grouped GEMM, no-padding layout (README "Grouped GEMMs (nopad layout)": a per-group token count replaces
 * the alignment of each group's rows to the M block).
 *   a [M_total][K] e4m3: group g's rows are off_g .. off_g + counts[g] - 1, off_g = counts[0] + ... +
 *     counts[g-1] (groups in order, no gaps, no alignment); rows from sum(counts) to M_total - 1 belong to no
 *     group.  sfa [K/128][ld(M_total)] (as for the dense call), b [G][N][K] e4m3, sfb [G][ceil(N/128)][K/128].
 *   counts int32 [G] on the device; the host never reads it.
 *   d [M_total][N] bf16: rows no group owns are left untouched.
 *   Negative counts count as 0; counts whose sum exceeds M_total are clipped at row M_total.  Both are
 *   reported by dg_check_device_error() as DG_ERR_BAD_GROUP.  1 <= G <= 1024; M_total has no alignment
 *   requirement (0 launches nothing). */
DG_EXPORT int dg_m_grouped_fp8_gemm_nt_nopad(const void *a, const float *sfa, const void *b, const float *sfb,
                                   void *d, const int *counts, int M_total, int N, int K, int G, dg_stream_t stream);

/* Dense NT GEMM that allocates no device memory (the pages have no counterpart: it exists for callers of this
 * library).  Same arguments, layouts, validation and results as dg_fp8_gemm_nt.  dg_fp8_gemm_nt takes a small
 * stream-ordered scratch buffer per call for its packed scale factors; callers that may not allocate during the
 * call -- code running under a global-mode stream capture, where allocation calls are refused, or engines whose
 * own memory manager owns all of device memory -- use this entry point instead, which puts the packed scales in a
 * fixed 16 MiB buffer that lives as long as the library is loaded (every device that loads the library holds
 * one).  It never calls cudaMalloc, cudaFree or any allocating routine.
 *   - Limit: the packed scales take at most (ceil(M/128) + 2*ceil(N/BN)) * ceil(K/512) * 512 bytes (BN is the
 *     chosen tile width, 128..224); a shape needing more than 16 MiB returns DG_ERR_UNSUPPORTED and launches
 *     nothing (M = N = K = 16384 needs about 4.5 MB).  Short calls (one kernel, see dg_fp8_gemm_nt) and calls
 *     with fp32 scale promotion on read the caller's scales directly and use no buffer at all (no limit).
 *   - The first call on each device looks up the buffer's device address with that device current, and the
 *     first call of each tile configuration does the one-time kernel set-up listed under "Common conventions";
 *     make one eager call of the same shape class on each device before any stream capture.
 *   - All calls share the buffer and each call rewrites every word it uses: calls whose work overlaps on the GPU
 *     (unordered streams) race; calls ordered on one stream are safe. */
DG_EXPORT int dg_fp8_gemm_nt_noalloc(const void *a, const float *sfa, const void *b, const float *sfb, void *d,
                                     int M, int N, int K, dg_stream_t stream);

/* Scale handling for the next calls on any thread ("promotion operations", DeepGEMM-for-PPU README,
 * "Optimizations"; the wrapper's disable_ue8m0_cast option).  0 (default): scales must be powers of two and are
 * applied by the block-scaled MMA (kind::mxf8f6f4, UE8M0 scales in tensor memory).  1: any finite fp32 scales;
 * every call then runs plain kind::f8f6f4 MMAs into one tensor-memory buffer per 128-K block, and the epilogue
 * warps accumulate buffer * sfa(m, kb) * sfb in fp32 registers (the scales are read from the caller's arrays, no
 * scale pre-pass):
 *   - e4m3 B (dense, allocation-free, contiguous, masked, no-padding, NN): 128-column tiles, sfb(g, n/128, kb);
 *   - K-grouped: 128-column tiles, the per-column sfb(n, kb), fp32 D stored or added as without promotion;
 *   - W4A8 (E2M1 B): 64-column tiles, one buffer per 32-K sub-block j, sfb(g, j, n).
 * The calls with per-column B scales (K-grouped, W4A8) need sfb 16-byte aligned (else DG_ERR_ALIGNMENT).
 * Returns the setting now in force. */
DG_EXPORT int dg_set_fp32_scale_promotion(int enable);
DG_EXPORT int dg_get_fp32_scale_promotion(void);

/* Tile-shape policy for the next calls on any thread: -1 (default) lets the library choose between one
 * CTA per 128-row tile and CTA pairs (2-CTA clusters, tcgen05 cta_group::2) computing 256-row tiles;
 * 0 forces single CTAs; 1 uses pairs wherever the layout allows.  Results agree within the tolerance of
 * fp32 accumulation either way.  Returns the policy now in force.  (README "Optimizations": larger block
 * sizes up to 256x256.) */
DG_EXPORT int dg_set_cta_pair_policy(int policy);

/* Operand order of the grouped tiles for the next calls on any thread: -1 (default) lets the library choose, 0
 * never swaps, 1 swaps wherever supported.  Swapped operands put B's rows (D's columns) on the tensor core's M
 * side and a group's tokens (D's rows) on its N side, which the MMA sizes per tile in steps of 16, so a group of
 * m tokens costs ceil(m / 16) * 16 rows of MMA work instead of whole 128- or 256-row windows; each tile covers
 * 256 (CTA pair) or 128 columns of D and up to 224 of one group's tokens.  Supported for the masked, no-padding
 * and contiguous FP8 calls (the contiguous ones while M_total / 128 <= 1024) with block-scaled (power-of-two)
 * scales.  The library swaps the masked calls and the NN call, and the no-padding and contiguous calls whose groups
 * hold at most 512 rows on average or whose N fills 256-wide tiles better than the unswapped tile width.  Results
 * agree within the tolerance of fp32 accumulation either way.  Returns the policy
 * now in force.  (README "Grouped GEMMs (masked layout)": decode-time groups of a few tokens.) */
DG_EXPORT int dg_set_swap_policy(int policy);

/* Testing aid for the bounded waits (no counterpart in the method; it exists so that the timeout path can be
 * exercised without faulting or hanging a GPU).
 *   limit_ns          limit of every mbarrier wait inside the GEMM kernel: 0 restores the default of 2 s,
 *                     otherwise 1e6 .. 2e9 ns.  Stays in force for every later launch.
 *   drop_first_stage  non-zero: the NEXT GEMM launch only (any entry point) leaves the first operand stage of its
 *                     first CTA (or CTA pair) unloaded, so that CTA's tensor-core thread waits for data that never
 *                     comes.  Its wait runs out after limit_ns, the CTA abandons its tiles (their rows of D are
 *                     left unwritten), the other CTAs finish, and dg_check_device_error() returns
 *                     DG_ERR_DEVICE_TIMEOUT.  The CUDA context stays usable.
 * Process-wide (see "Common conventions"); call it between launches.  Returns DG_OK or DG_ERR_INVALID_ARG. */
DG_EXPORT int dg_debug_bounded_wait(unsigned long long limit_ns, int drop_first_stage);

/* Measurement aid (no counterpart in the method; it exists so that a benchmark can state the SM clock its GEMM
 * launches actually ran at, which under the board's power limit is below the maximum clock).
 *   dg_debug_clock_record(1): every later GEMM launch (any entry point, any device) makes its first CTA add
 *     the SM clock cycles (clock64) and the nanoseconds (globaltimer) it spent from start to exit, and 1, to a
 *     per-device accumulator of three 64-bit counters; 0 switches it off (the default).  Returns the setting.
 *   dg_debug_clock_read(out, reset): synchronises the current device, copies its three counters (cycles,
 *     nanoseconds, launches) to the host array out[3] and, when reset != 0, clears them.  The mean SM clock of
 *     the recorded launches is out[0] / out[1] GHz.  Returns DG_OK, DG_ERR_INVALID_ARG or DG_ERR_CUDA. */
DG_EXPORT int dg_debug_clock_record(int enable);
DG_EXPORT int dg_debug_clock_read(unsigned long long *out, int reset);

/* Message for the last non-OK status returned on this thread ("" if none). */
DG_EXPORT const char *dg_last_error(void);

/* Synchronises `stream`, then returns and clears the device error word of the current device:
 * DG_OK, DG_ERR_DEVICE_TIMEOUT, DG_ERR_BAD_GROUP or DG_ERR_BAD_SCALE (DG_ERR_CUDA if the synchronisation
 * failed).  The first error recorded since the last check wins. */
DG_EXPORT int dg_check_device_error(dg_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* DG_H_ */
