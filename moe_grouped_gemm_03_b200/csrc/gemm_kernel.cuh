// Persistent, warp-specialised FP8 NT GEMM with fine-grained scaling for sm_100a.
//
//   D[m][n] = bf16( sum_kb sfa(m,kb) * sfb(g, n/128, kb) * sum_{k in kb} A[m][k] * B_g[n][k] )
//
// ("FP8 GEMM kernels with fine-grained scaling", DeepGEMM-for-PPU README: "Interfaces" for the three
// call shapes, "Optimizations" for persistent warp specialisation, the unified block scheduler, larger
// blocks and unaligned block sizes.)
//
// The per-128-K scale promotion runs inside the tensor core: the MMA is tcgen05.mma kind::mxf8f6f4 with
// block scaling (one UE8M0 scale per 32 K elements and row/column).  The fp32 power-of-two scales are packed
// beforehand (scale_pack.cuh) into 32-bit words holding the UE8M0 bytes of four consecutive 128-K blocks,
// already in the shared-memory layout tcgen05.cp reads; the MMAs of K block kb select byte kb % 4 through
// the scale-factor ids of the instruction descriptor for all four 32-wide K sub-blocks, which applies the
// 1x128 / 128x128 recipe exactly.
//
// Cfg::PROMO (any finite fp32 scales): the promotion runs in the epilogue warps instead.  Plain kind::f8f6f4
// MMAs write each 128-K block's partial product into its own TMEM buffer (two partial stages of KPS buffers),
// and the epilogue warps accumulate partial * sfa * sfb in fp32 registers, reading the caller's fp32 scales
// directly (no pre-pass): 128-wide tiles with one B scale per 128-column block, or (Cfg::PCOL) 64-wide tiles
// with one B scale per column -- per K block for the K-grouped call (fp32 D), per 32-K sub-block for E2M1 B,
// whose four 32-K MMAs per K block then write four partials.  The host also runs short dense calls on power-of-two
// scales through the 128-wide promotion kernel, with the scale check of the block-scaled path.
//
// CTAS = 1: one CTA computes a 128 x BN output tile.  CTAS = 2: a cluster of two CTAs (a CTA pair) computes
// a 256 x BN tile with tcgen05.mma.cta_group::2: each CTA loads its own 128 rows of A and its own BN/2 rows
// of B (no multicast), the leader CTA issues the MMAs, and each CTA's TMEM holds its 128 rows of D.  All
// cross-CTA data arrives by TMA whose byte counts complete the leader's barrier.
//
// Per CTA, 192 threads:
//   warp 0      TMA producer: per pipeline stage KPS 128-K blocks of A [128 x 128 B] and B [BN/CTAS x 128 B]
//               (128-byte swizzle) and, at the first stage of each group of four K blocks, the packed scale
//               atoms of the group (SFA of this CTA's rows, SFB of the whole tile; none with PROMO).
//   warp 1      TMEM owner (both CTAs) and MMA issuer (one thread of the leader CTA): copies a group's scale
//               atoms shared -> TMEM (tcgen05.cp), then issues four tcgen05.mma (K = 32 each) per 128-K
//               block into one of two TMEM accumulators (BN fp32 columns).
//   warps 2..5  epilogue: TMEM -> registers -> bf16 (RNE) -> global, only for rows the GEMM owns, while the
//               MMA already fills the other accumulator with the next tile (with PROMO: the fp32 promotion of
//               each partial product, then the same bf16 stores).
//
// Tile scheduler (every role walks the same sequence): windows of 128*CTAS rows x BN columns handed
// round-robin to the persistent CTAs (pairs); dense and K-grouped tiles go down the windows first inside raster
// groups of windows (see raster_tile), the other layouts across the columns first.
//   dense       ceil(M / 128*CTAS) windows.
//   contiguous  CTAS = 1: M_total/128 blocks, group = m_indices[first row], -1 skips the block.
//               CTAS = 2: 256-row windows starting at each group's first block (two blocks of one group; the
//               last window of a group with an odd block count computes, and does not store, one block of
//               the next rows).  The window list is built on the device at kernel start.
//   masked      per group ceil(masked_m[g] / 128*CTAS) windows, counted on the device, so the host never
//               needs masked_m.
//   no padding  the same per-group windows over the groups' row counts, each group starting at the sum of
//               the earlier counts (no alignment); rows past a group's count are computed and not stored.
// Each CTA decodes its tile sequence once at kernel start (all threads, into a shared-memory list), so no
// role pays a decode -- a binary search and global loads of m_indices -- per tile.
//
// Every mbarrier wait is bounded: after WAIT_LIMIT_NS the waiting thread raises a CTA-wide abort flag and
// records ERR_TIMEOUT in the device error word; every role then leaves its loop, the producer waits (bounded)
// for its loads in flight, the MMA thread waits (bounded) for its tensor-core work, and TMEM is released.
#pragma once
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace dg {

enum : int { MODE_DENSE = 0, MODE_CONTIGUOUS = 1, MODE_MASKED = 2, MODE_NOPAD = 3, MODE_KGROUPED = 4 };
// output: bf16 D (the M-grouped and dense calls), fp32 D written, or fp32 D += the product (K-grouped call)
enum : int { OUT_BF16 = 0, OUT_F32_STORE = 1, OUT_F32_ADD = 2 };

constexpr int BLOCK_M = 128;  // rows per CTA
constexpr int BLOCK_K = 128;  // = the scale block along K
constexpr int MMA_K = 32;     // K of one kind::mxf8f6f4 MMA
constexpr int SF_GROUP = 4;   // 128-K blocks whose scales share one 32-bit word (one byte each)
constexpr int SF_ATOM_WORDS = 128;  // a packed scale atom: 128 rows x one 32-bit word (512 bytes)
constexpr int NUM_THREADS = 192;
constexpr int EPI_WARP0 = 2;        // epilogue warps 2..5 (TMEM lane quarter = warp % 4)
constexpr int MAX_MASKED_GROUPS = 1024;
constexpr int MAX_PAIR_WINDOWS = 2048;  // contiguous layout with CTA pairs: at most 2048 256-row windows
constexpr int TILE_LIST_CAP = 1024;     // tiles per CTA decoded up front (further tiles are decoded on the fly)
constexpr int EPI_CHUNK_BYTES = 32 * 32 * 2;  // one epilogue staging chunk: 32 rows x 32 bf16 columns
constexpr int TMEM_COLS = 512;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;  // default limit of any single wait: 2 s
constexpr int SMEM_LIMIT = 232448;                  // 227 KB of dynamic shared memory per CTA

// device error word codes
constexpr unsigned ERR_TIMEOUT = 1u;
constexpr unsigned ERR_BAD_GROUP = 2u;
constexpr unsigned ERR_BAD_SCALE = 3u;  // a scale the block-scaled MMA cannot represent (not a power of two)

struct GemmParams {
    int mode;
    int M;             // dense: M; contiguous / no padding: M_total; masked: M_max; K-grouped: M
    int out_mode;      // OUT_*
    int N, K, G;
    int num_windows;   // dense / contiguous: windows (128- or 256-row); K-grouped: G x windows of M;
                       // masked / no padding: unused
    int num_n_blocks;  // ceil(N / BN)
    int num_sf_groups; // ceil(K / (128 * SF_GROUP)); K-grouped: the sum over groups of ceil(K_g / (128 * SF_GROUP))
    int sfa_blocks;    // 128-row blocks per group of the packed SFA (masked layout; swapped operands: of B's rows)
    int swap_chunks;   // swapped operands: token chunks (all groups) the packed token-side scales have room for
    int raster_bands;  // dense / K-grouped: row windows per raster group (the tile order); 0: columns first
    __nv_bfloat16 *d;
    float *d32;        // fp32 output (out_mode != OUT_BF16): [G][M][N]
    const int *m_indices;
    const int *masked_m;  // masked: masked_m; no padding: the groups' row counts; K-grouped: the groups' K extents
    unsigned *err;
    unsigned long long wait_limit_ns;  // limit of any single wait
    int skip_first_load;               // test hook: the first CTA (pair) never loads stage 0
    // fp32 scale promotion (Cfg::PROMO): the caller's scales, read by the epilogue warps
    const float *sfa32;  // MN-major [K/128][sfa_ld] (masked: [G][K/128][sfa_ld])
    // Cfg::PCOL = false: scale of (group g, 128-column block nb, K block kb) at g * sfb_sg + nb * sfb_sn + kb * sfb_sk;
    // Cfg::PCOL: one scale per column n (K-grouped: per K block kb of the whole K range; W4A8: per 32-K sub-block
    // j) at g * sfb_sg + kb (or j) * sfb_sk + n, the address of each 4 columns 16-byte aligned
    const float *sfb32;
    int sfa_ld;
    int sfb_sg, sfb_sn, sfb_sk;
    // 1: the scales must be powers of two (the block-scaled calls' rule, applied by the promotion GEMM when a dense
    // call runs as one kernel): each one read is checked (ERR_BAD_SCALE) and a zero scale is read as 2^-127
    int check_scales;
    // measurement aid (null: off): CTA 0 adds its SM cycles, nanoseconds and 1 to clock_acc[0..2] at exit
    unsigned long long *clock_acc;
};

template <int BN_, int CTAS_, int KPS_, bool BF4_ = false, bool PROMO_ = false, bool SWAP_ = false,
          bool BNN_ = false, bool PCOL_ = false>
struct Cfg {
    static constexpr int BN = BN_;
    static constexpr int CTAS = CTAS_;
    static constexpr int KPS = KPS_;                              // 128-K blocks per pipeline stage
    // B in E2M1 (W4A8): B's smem tiles keep the e4m3 footprint (TMA stages 4-bit codes one byte each) and B has
    // one scale per (row, 32-K block), i.e. one 4-byte scale word per row per 128-K block, so a stage carries
    // the B scale atoms of each of its K blocks (A's atom still packs SF_GROUP K blocks)
    static constexpr bool BF4 = BF4_;
    // fp32 scale promotion: plain kind::f8f6f4 MMAs write each 128-K block's partial product to its own TMEM
    // buffer (two partial stages of KPS blocks, 2 * KPS * BN columns), and the epilogue warps accumulate
    // partial * sfa * sfb in registers.  No scale atoms travel with the stages.  e4m3 B: BN = 128, a tile's
    // columns are exactly one 128-column block of B's scales (K-grouped: 64 columns of per-column scales).  E2M1 B
    // (one scale per column and 32-K sub-block): each of a K block's four 32-K MMAs writes its own partial
    // (PSUB = 4), so BN = 64 and one K block per stage fill the 512 TMEM columns.
    static constexpr bool PROMO = PROMO_;
    static constexpr int PSUB = PROMO && BF4_ ? 4 : 1;  // partial buffers per 128-K block
    // promotion with one B scale per column (the K-grouped calls' configuration, fp32 D; E2M1 B always): the
    // epilogue stages each partial stage's column scales in shared memory
    static constexpr bool PCOL = PROMO && (PCOL_ || BF4_);
    // Swapped operands (masked layout): the MMA's M side runs over B's rows (D's columns, TILE_M per tile) and
    // its N side over up to BN of one group's tokens (D's rows).  The A-side tile of shared memory then holds 128
    // rows of B and the B-side tile up to BN/CTAS tokens of A; the MMA's N is set per tile to the tile's token
    // count rounded up to 16, so a group is padded to 16 rows instead of TILE_M.  Same buffers, barriers and
    // TMEM layout as the unswapped configuration.
    static constexpr bool SWAP = SWAP_;
    // With swapped operands, B in the NN orientation ([G][K][N], N contiguous): each K block of the M-side tile is
    // loaded as 128 K-rows of 128 N-bytes, an MN-major operand (the 128-byte swizzle atom of 8 K-rows x 128 B), so
    // no transposed copy of B is made.
    static constexpr bool BNN = BNN_;
    static constexpr int SFB_KB = BF4 ? KPS : 1;                  // K blocks whose B scale atoms a stage holds
    static constexpr int TILE_M = BLOCK_M * CTAS;
    static constexpr int B_ROWS = BN / CTAS;                      // B rows this CTA loads
    static constexpr int SFB_ATOMS = (BN + 127) / 128;            // 128-row scale atoms covering BN rows
    static constexpr int A_BYTES1 = BLOCK_M * BLOCK_K;            // one K block of A (e4m3: 1 byte each)
    static constexpr int B_BYTES1 = B_ROWS * BLOCK_K;             // one K block of this CTA's B rows
    // transaction bytes of that load: an E2M1 box counts its packed bytes (half a byte per code), although
    // shared memory receives one byte per code
    static constexpr int B_TX1 = BF4_ ? B_ROWS * BLOCK_K / 2 : B_BYTES1;
    static constexpr int A_BYTES = KPS * A_BYTES1;                // per stage
    static constexpr int B_BYTES = KPS * B_BYTES1;
    static constexpr int SF_BYTES = PROMO ? 0 : (1 + SFB_KB * SFB_ATOMS) * SF_ATOM_WORDS * 4;  // SFA + SFB atoms
    static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SF_BYTES;
    static constexpr int SF_COLS = 4 + 4 * SFB_KB * SFB_ATOMS;    // TMEM columns of one scale slot
    static constexpr int SF_TMEM_BASE = 2 * BN;                   // after the two accumulators
    // scale slots in TMEM, used round-robin by successive scale groups (not by stages)
    static constexpr int SF_SLOTS_FIT = (TMEM_COLS - SF_TMEM_BASE) / SF_COLS;
    static constexpr int SF_SLOTS = SF_SLOTS_FIT > 4 ? 4 : SF_SLOTS_FIT;
    // window prefix (masked / no padding: G + 1 entries, then the groups' first rows) or pair windows
    static constexpr int TABLE_INTS =
        MAX_PAIR_WINDOWS + 1 > 2 * (MAX_MASKED_GROUPS + 1) ? MAX_PAIR_WINDOWS + 1 : 2 * (MAX_MASKED_GROUPS + 1);
    static constexpr int EPI_BYTES = 4 * 2 * EPI_CHUNK_BYTES;    // per epilogue warp: two staging chunks
    // promotion with per-column B scales: per epilogue warp, two partial stages' worth (KPS * PSUB rows of BN)
    static constexpr int PSB_FLOATS = KPS * PSUB * BN;
    static constexpr int PSB_BYTES = PCOL ? 4 * 2 * PSB_FLOATS * 4 : 0;
    static constexpr int FIXED_BYTES = EPI_BYTES + PSB_BYTES + 4 * TABLE_INTS + 4 * MAX_MASKED_GROUPS + 2 * MAX_MASKED_GROUPS + 16 +
                                       8 * TILE_LIST_CAP + 16 + 8 * 16 + 1024;
    static constexpr int STAGES_FIT = (SMEM_LIMIT - FIXED_BYTES - 8 * 2 * 8) / STAGE_BYTES;
    static constexpr int STAGES_MAX = STAGES_FIT;
    static constexpr int STAGES = STAGES_MAX > 8 ? 8 : STAGES_MAX;
    static constexpr int NUM_BARRIERS = 2 * STAGES + 5;
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
    static constexpr int OFF_SF = OFF_B + STAGES * B_BYTES;
    static constexpr int OFF_EPI = OFF_SF + STAGES * SF_BYTES;    // 1024-aligned (64-byte swizzle atoms)
    static constexpr int OFF_PSB = OFF_EPI + EPI_BYTES;
    static constexpr int OFF_BAR = OFF_PSB + PSB_BYTES;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARRIERS * 8;   // tmem base, abort flag
    static constexpr int OFF_PREFIX = OFF_MISC + 16;               // int[TABLE_INTS]
    static constexpr int OFF_MM = OFF_PREFIX + 4 * TABLE_INTS;     // masked: clamped masked_m
    static constexpr int OFF_RG = OFF_MM + 4 * MAX_MASKED_GROUPS;  // short[]: group of each run (contiguous, swapped)
    static constexpr int OFF_TILES = (OFF_RG + 2 * MAX_MASKED_GROUPS + 15) / 16 * 16;  // uint2[TILE_LIST_CAP]
    static constexpr int SMEM_BYTES = OFF_TILES + 8 * TILE_LIST_CAP + 1024;     // + alignment slack
    static_assert(CTAS == 1 || CTAS == 2, "single CTA or CTA pair");
    static_assert(!PROMO || ((BF4 ? BN == 64 && KPS == 1 : (BN == 128 || (PCOL && BN == 64))) &&
                             2 * KPS * PSUB * BN <= TMEM_COLS),
                  "promotion: 128-wide tiles (e4m3 B; 64 with per-column scales) or 64-wide tiles of one K block "
                  "(E2M1 B)");
    static_assert(!PCOL || (PSB_FLOATS % 64 == 0 && OFF_PSB % 16 == 0), "per-column scale staging");
    static_assert(!PCOL_ || PROMO_, "per-column B scales are a promotion variant");
    static_assert(!SWAP || (!PROMO && !BF4 && BN % 16 == 0), "swapped operands: block-scaled e4m3 only");
    static_assert(!BNN || SWAP, "B in the NN orientation is read through swapped operands");
    static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "BN must be a multiple of 32 in [32, 256]");
    static_assert(B_ROWS % 8 == 0, "B tile rows must fill whole 8-row swizzle atoms");
    static_assert(STAGES >= 3, "pipeline too shallow");
    static_assert(SF_SLOTS >= 2 && SF_TMEM_BASE + SF_SLOTS * SF_COLS <= TMEM_COLS, "TMEM budget");
    static_assert(SMEM_BYTES <= SMEM_LIMIT, "shared memory budget");
    static_assert(A_BYTES1 % 1024 == 0 && B_BYTES1 % 1024 == 0, "swizzle atoms need 1024-byte alignment");
    static_assert(SF_GROUP % KPS == 0, "a stage must not straddle a scale group");
    static_assert(OFF_A % 1024 == 0 && OFF_B % 1024 == 0 && OFF_SF % 512 == 0 && OFF_EPI % 512 == 0, "TMA buffers");
    static_assert(OFF_BAR % 8 == 0 && OFF_MISC % 8 == 0, "mbarriers need 8-byte alignment");
    static_assert(OFF_PREFIX % 4 == 0 && OFF_MM % 4 == 0 && OFF_TILES % 16 == 0, "tables");
};

struct Tile {
    int row0;        // first row of the window in A / D (flattened [rows, K] / [rows, N])
    int local_row0;  // first row of the window inside its group (masked) or = row0
    int n0;
    int nb;
    int g;
};

struct SharedCtl {
    volatile int *abort;
    const int *prefix;   // masked / no padding: window prefix per group; contiguous pairs: first block of each
                         // window; K-grouped: first packed scale group of each group; swapped operands: chunk
                         // prefix per group (contiguous: per run)
    const int *mm;       // masked / no padding: the groups' clamped row counts; K-grouped: 128-K blocks per group;
                         // contiguous with swapped operands: rows of each run
    const int *off;      // no padding: first row of each group; K-grouped: first 128-K block of each group;
                         // contiguous with swapped operands: first row of each run
    const short *gblk;   // contiguous pairs, kernel prologue only: group of each 128-row block
    const short *rg;     // contiguous with swapped operands: group of each run
    int ntab;            // entries of prefix / mm / off: G, or the runs (contiguous with swapped operands)
};

__device__ __forceinline__ void raise_error(unsigned *err, unsigned code) { atomicCAS(err, 0u, code); }

// Nonzero unless the scale's fp32 bits are ones the exponent code represents exactly: +0 (taken as 2^-127) or
// a positive normal power of two (no sign, no mantissa bits, not Inf / NaN).
__device__ __forceinline__ uint32_t ue8m0_inexact_bits(uint32_t b) {
    return (b & 0x807FFFFFu) | (((b >> 23) & 0xFFu) == 0xFFu ? 1u : 0u);
}
constexpr uint32_t UE8M0_ZERO_F32_BITS = 0x00400000u;  // 2^-127 (fp32 subnormal): the value of exponent code 0

// Slow path of the bounded mbarrier wait.  false = gave up (this CTA is aborting).
__device__ __noinline__ bool wait_bounded_slow(uint64_t *bar, uint32_t parity, volatile int *abort, unsigned *err,
                                               uint64_t limit) {
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait_sleep(bar, parity, 100000u)) return true;
        if ((it & 3u) == 0) {
            if (*abort) return false;
            if (global_timer_ns() - t0 > limit) {
                *abort = 1;
                raise_error(err, ERR_TIMEOUT);
                return false;
            }
        }
    }
}

__device__ __forceinline__ bool wait_bounded(uint64_t *bar, uint32_t parity, volatile int *abort, unsigned *err,
                                             uint64_t limit) {
    if (mbar_try_wait(bar, parity)) return true;
    return wait_bounded_slow(bar, parity, abort, err, limit);
}

// Whole-warp wait: lane 0 waits, the outcome is broadcast, and the warp leaves converged (the callers
// follow with .sync.aligned tcgen05 instructions).
__device__ __forceinline__ bool warp_wait_bounded(uint64_t *bar, uint32_t parity, volatile int *abort,
                                                  unsigned *err, uint64_t limit, int lane) {
    int ok = 1;
    if (lane == 0) ok = wait_bounded(bar, parity, abort, err, limit) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

// A group id read from m_indices: -1 for padding; ids >= G are reported and treated as padding.
__device__ __forceinline__ int checked_group(const GemmParams &p, int g) {
    if (g >= p.G) {
        raise_error(p.err, ERR_BAD_GROUP);
        return -1;
    }
    return g < 0 ? -1 : g;
}

__device__ __forceinline__ int group_of_block(const GemmParams &p, int block) {
    const int row = block * BLOCK_M;
    if (row >= p.M) return -1;
    return checked_group(p, __ldg(p.m_indices + row));
}

// largest i in [0, n) with table[i] <= v, given table[0] <= v < table[n]
__device__ __forceinline__ int upper_index(const int *table, int n, int v) {
    int lo = 0, hi = n;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (table[mid] <= v) lo = mid; else hi = mid;
    }
    return lo;
}

// Order of the tiles of a grid of `windows` row windows x `nblocks` column blocks: tile t -> (window, *nb).
// The windows are cut into raster groups of `bands` consecutive windows; inside a group the tiles walk down
// the windows first, then across the columns, so the CTAs running at one time share a few B column blocks
// and the group's A rows, which stay in L2 while the group's columns are swept.  bands <= 0: columns first.
__device__ __forceinline__ int raster_tile(int t, int windows, int nblocks, int bands, int &nb) {
    if (bands <= 0) {
        const int w = t / nblocks;
        nb = t - w * nblocks;
        return w;
    }
    const int span = bands * nblocks;  // tiles of one full raster group
    const int grp = t / span;
    const int w0 = grp * bands;
    const int gm = min(bands, windows - w0);  // the last group may be narrower
    const int local = t - grp * span;
    nb = local / gm;
    return w0 + (local - nb * gm);
}

// Swapped operands: a group of m tokens is cut into ceil(m / bn) chunks of equal size, rounded up to 16 rows (the
// MMA's N granularity), so no chunk exceeds bn.  Rows of one chunk: chunk_rows(m, bn); the last may hold fewer.
__host__ __device__ __forceinline__ int chunk_rows(int m, int bn) {
    if (m <= 0) return bn;
    const int chunks = (m + bn - 1) / bn;
    return ((m + chunks - 1) / chunks + 15) & ~15;
}

template <class C>
__device__ __forceinline__ bool decode_tile(const GemmParams &p, const SharedCtl &ctl, int t, Tile &ti) {
    if (p.mode == MODE_DENSE) {
        const int w = raster_tile(t, p.num_windows, p.num_n_blocks, p.raster_bands, ti.nb);
        ti.n0 = ti.nb * C::BN;
        ti.g = 0;
        ti.row0 = ti.local_row0 = w * C::TILE_M;
        return true;
    }
    if (p.mode == MODE_KGROUPED) {  // every group covers all M rows; a group's tiles are consecutive
        const int per_group = p.num_windows / p.G;
        const int group_tiles = per_group * p.num_n_blocks;
        ti.g = t / group_tiles;
        const int w = raster_tile(t - ti.g * group_tiles, per_group, p.num_n_blocks, p.raster_bands, ti.nb);
        ti.n0 = ti.nb * C::BN;
        ti.row0 = ti.local_row0 = w * C::TILE_M;
        return true;
    }
    const int w = t / p.num_n_blocks;  // window-tile index
    ti.nb = t - w * p.num_n_blocks;
    ti.n0 = ti.nb * (C::SWAP ? C::TILE_M : C::BN);
    if constexpr (C::SWAP) {  // window w = one chunk of one group's (contiguous: one run's) tokens
        const int g = upper_index(ctl.prefix, ctl.ntab, w);
        ti.g = g;
        ti.local_row0 = (w - ctl.prefix[g]) * chunk_rows(ctl.mm[g], C::BN);
        ti.row0 = (p.mode == MODE_MASKED ? g * p.M : ctl.off[g]) + ti.local_row0;
        return true;
    }
    if (p.mode == MODE_CONTIGUOUS) {
        if constexpr (C::CTAS == 1) {
            ti.row0 = ti.local_row0 = w * BLOCK_M;
            ti.g = group_of_block(p, w);
            return ti.g >= 0;
        } else {
            const int b0 = ctl.prefix[w];  // first block of the window
            ti.row0 = ti.local_row0 = b0 * BLOCK_M;
            ti.g = ctl.gblk ? ctl.gblk[b0] : group_of_block(p, b0);  // the staged table exists only in the prologue
            return ti.g >= 0;
        }
    }
    const int g = upper_index(ctl.prefix, p.G, w);
    ti.g = g;
    ti.local_row0 = (w - ctl.prefix[g]) * C::TILE_M;
    ti.row0 = (p.mode == MODE_MASKED ? g * p.M : ctl.off[g]) + ti.local_row0;
    return true;
}

// A decoded tile packed into 8 bytes: row0, then (g + 1) in the low 16 bits and nb in the high 16 bits
// (g + 1 = 0 marks a tile that computes nothing).  local_row0 = row0 - (the group's first row) for the masked
// and no-padding layouts, else row0.
__device__ __forceinline__ uint2 pack_tile(bool valid, const Tile &ti) {
    return make_uint2(static_cast<uint32_t>(ti.row0),
                      (valid ? static_cast<uint32_t>(ti.g + 1) : 0u) | (static_cast<uint32_t>(ti.nb) << 16));
}

template <class C>
__device__ __forceinline__ bool unpack_tile(const GemmParams &p, const SharedCtl &ctl, uint2 e, Tile &ti) {
    const int g1 = static_cast<int>(e.y & 0xFFFFu);
    if (g1 == 0) return false;
    ti.g = g1 - 1;
    ti.nb = static_cast<int>(e.y >> 16);
    ti.n0 = ti.nb * (C::SWAP ? C::TILE_M : C::BN);
    ti.row0 = static_cast<int>(e.x);
    if (p.mode == MODE_MASKED)
        ti.local_row0 = ti.row0 - ti.g * p.M;
    else if (p.mode == MODE_NOPAD || (C::SWAP && p.mode == MODE_CONTIGUOUS))
        ti.local_row0 = ti.row0 - ctl.off[ti.g];
    else
        ti.local_row0 = ti.row0;
    return true;
}

// Warp-wide exclusive prefix sum of one int per lane; *total receives the sum over the warp.
__device__ __forceinline__ int warp_exclusive_sum(int v, int lane, int *total) {
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += u;
    }
    *total = __shfl_sync(0xffffffffu, incl, 31);
    return incl - v;
}

// Masked layout (one warp, after mm[] holds the clamped masked_m): prefix[g] = windows of groups before g,
// prefix[G] = all windows.
// Window prefix of the groups' row counts: prefix[g] = ceil(mm[0] / tile_m) + ... + ceil(mm[g-1] / tile_m),
// prefix[G] = the total (one warp; lane l scans a contiguous chunk of groups).
__device__ void build_window_prefix(int G, int tile_m, const int *mm, int *prefix, int lane) {
    const int chunk = (G + 31) / 32;
    const int begin = min(lane * chunk, G), end = min(begin + chunk, G);
    int local = 0;
    for (int g = begin; g < end; ++g) local += (mm[g] + tile_m - 1) / tile_m;
    int total;
    int run = warp_exclusive_sum(local, lane, &total);
    for (int g = begin; g < end; ++g) {
        prefix[g] = run;
        run += (mm[g] + tile_m - 1) / tile_m;
    }
    if (lane == 0) prefix[G] = total;
}

// No-padding layout: the groups' first rows off[g] = counts[0] + ... + counts[g-1] (a 64-bit running sum), and
// the counts (already >= 0) clamped so that every group ends by row M; rows past M are reported and dropped.
// One warp, the same chunking as build_window_prefix.
__device__ void build_group_rows(int G, int M, int *mm, int *off, unsigned *err, int lane) {
    const int chunk = (G + 31) / 32;
    const int begin = min(lane * chunk, G), end = min(begin + chunk, G);
    long long local = 0;
    for (int g = begin; g < end; ++g) local += mm[g];
    long long incl = local;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const long long u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
    }
    long long run = incl - local;
    for (int g = begin; g < end; ++g) {
        const long long c = mm[g];
        const int start = static_cast<int>(run < M ? run : M);
        int kept = static_cast<int>(c);
        if (run + c > M) {
            kept = M - start;
            if (err) raise_error(err, ERR_BAD_GROUP);
        }
        off[g] = start;
        mm[g] = kept;
        run += c;
    }
}

// Contiguous layout with CTA pairs (one warp, after gblk[] holds each 128-row block's group or -1): the
// 256-row windows start at each group's first block and advance by two blocks inside the group's run, so a
// window never spans two groups except the last window of a run with an odd number of blocks, whose second
// half computes rows it does not store.  list[0..n) = first block of each window, list[MAX_PAIR_WINDOWS] = n.
__device__ void build_pair_windows(int num_blocks, const short *gblk, int *list, int lane) {
    const int chunk = (num_blocks + 31) / 32;
    const int begin = min(lane * chunk, num_blocks), end = min(begin + chunk, num_blocks);
    auto run_head = [&](int b) { return gblk[b] >= 0 && (b == 0 || gblk[b - 1] != gblk[b]); };
    // the last run head at or before each chunk's start (inclusive max-scan of run heads)
    int last = -1;
    for (int b = begin; b < end; ++b)
        if (run_head(b)) last = b;
    int carried = last;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, carried, off);
        if (lane >= off) carried = max(carried, u);
    }
    int head = __shfl_up_sync(0xffffffffu, carried, 1);
    if (lane == 0) head = -1;
    int count = 0;
    for (int b = begin, h = head; b < end; ++b) {
        if (run_head(b)) h = b;
        if (gblk[b] >= 0 && ((b - h) & 1) == 0) ++count;
    }
    int total;
    int pos = warp_exclusive_sum(count, lane, &total);
    for (int b = begin, h = head; b < end; ++b) {
        if (run_head(b)) h = b;
        if (gblk[b] >= 0 && ((b - h) & 1) == 0 && pos < MAX_PAIR_WINDOWS) list[pos++] = b;
    }
    if (lane == 0) list[MAX_PAIR_WINDOWS] = min(total, MAX_PAIR_WINDOWS);
}

// Contiguous layout with swapped operands, step 1 (one warp; gblk[b] = the group of 128-row block b or -1): runs of
// consecutive blocks of one group.  off[r] = run r's first block, mm[r] = its last block, rg[r] = its group, in row
// order; returns the run count (at most num_blocks).
__device__ int build_run_heads(int num_blocks, const short *gblk, int *off, int *mm, short *rg, int lane) {
    const int chunk = (num_blocks + 31) / 32;
    const int begin = min(lane * chunk, num_blocks), end = min(begin + chunk, num_blocks);
    auto head = [&](int b) { return gblk[b] >= 0 && (b == 0 || gblk[b - 1] != gblk[b]); };
    auto tail = [&](int b) { return gblk[b] >= 0 && (b + 1 == num_blocks || gblk[b + 1] != gblk[b]); };
    int nh = 0, nt = 0;
    for (int b = begin; b < end; ++b) {
        nh += head(b) ? 1 : 0;
        nt += tail(b) ? 1 : 0;
    }
    int runs, tails;
    int ph = warp_exclusive_sum(nh, lane, &runs);
    int pt = warp_exclusive_sum(nt, lane, &tails);
    for (int b = begin; b < end; ++b) {
        if (head(b)) {
            off[ph] = b;
            rg[ph] = gblk[b];
            ++ph;
        }
        if (tail(b)) mm[pt++] = b;
    }
    return runs;
}

// Step 2 (warp `warp` of `nwarps`, after step 1): run r's rows go from its first block's first row to the last row
// of its last block that belongs to its group (the layout pads a segment at its end); off[r] becomes that first row
// and mm[r] the row count.  Rows inside the run that belong to no group are computed and never stored.
__device__ void finish_runs(const int *m_indices, int M, int runs, int *off, int *mm, const short *rg, int warp,
                            int nwarps, int lane) {
    for (int r = warp; r < runs; r += nwarps) {
        const int last_blk = mm[r], first_blk = off[r], g = rg[r];
        const int base = last_blk * BLOCK_M;
        int v[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int row = base + 32 * j + lane;
            v[j] = row < M ? __ldg(m_indices + row) : -1;
        }
        int last = 0;  // the block's first row belongs to g, so some row does
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const unsigned bal = __ballot_sync(0xffffffffu, v[j] == g);
            if (bal) last = 32 * j + 31 - __clz(bal);
        }
        __syncwarp();
        if (lane == 0) {
            off[r] = first_blk * BLOCK_M;
            mm[r] = (last_blk - first_blk) * BLOCK_M + last + 1;
        }
    }
}

template <class C>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    fp8_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                    const __grid_constant__ CUtensorMap tmap_sfa, const __grid_constant__ CUtensorMap tmap_sfb,
                    const __grid_constant__ CUtensorMap tmap_d, const GemmParams p) {
    constexpr int BN = C::BN;
    constexpr int STAGES = C::STAGES;
    constexpr int CTAS = C::CTAS;
    constexpr bool PAIR = CTAS == 2;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem + C::OFF_A;
    uint8_t *sB = smem + C::OFF_B;
    uint8_t *sSF = smem + C::OFF_SF;
    uint8_t *sEpi = smem + C::OFF_EPI;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *full = bars;                  // [STAGES] stage landed (the leader's counts both CTAs' bytes)
    uint64_t *empty = bars + STAGES;        // [STAGES] MMAs done with the stage (both CTAs, by commit)
    uint64_t *tmem_full = bars + 2 * STAGES;  // [2]
    uint64_t *tmem_empty = tmem_full + 2;   // [2] (the leader's counts the epilogue warps of both CTAs)
    uint64_t *drain = tmem_empty + 2;       // [1]
    uint32_t *s_tmem_base = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *s_abort = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    int *s_prefix = reinterpret_cast<int *>(smem + C::OFF_PREFIX);
    int *s_mm = reinterpret_cast<int *>(smem + C::OFF_MM);
    int *s_off = s_prefix + (MAX_MASKED_GROUPS + 1);  // no padding: the groups' first rows
    uint2 *s_tiles = reinterpret_cast<uint2 *>(smem + C::OFF_TILES);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const uint32_t rank = PAIR ? cluster_cta_rank() : 0u;
    const int cluster_id = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
    const int num_clusters = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
    const bool clock_rec = p.clock_acc != nullptr && blockIdx.x == 0 && threadIdx.x == 0;
    const unsigned long long clk0 = clock_rec ? clock64() : 0ull, ns0 = clock_rec ? global_timer_ns() : 0ull;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);  // armed by the leader's producer with every byte of the stage
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tmem_full[i], 1);
            mbar_init(&tmem_empty[i], 4 * CTAS);  // one arrival per epilogue warp of each CTA
        }
        mbar_init(drain, 1);
        *s_abort = 0;
        mbar_init_fence();
        fence_proxy_async_smem();
        tma_prefetch_desc(&tmap_a);
        tma_prefetch_desc(&tmap_b);
        tma_prefetch_desc(&tmap_sfa);
        tma_prefetch_desc(&tmap_sfb);
        tma_prefetch_desc(&tmap_d);
    }
    if (warp == 1) {
        tmem_alloc<CTAS>(s_tmem_base, TMEM_COLS);
        tmem_relinquish<CTAS>();
    }
    // Scheduler tables.  Loads first, by all threads (independent loads in flight together), into shared
    // memory: masked_m, or the group of every 128-row block (staged in the A ring, unused until the producer
    // starts); then one warp scans them.
    const bool pair_contig = PAIR && p.mode == MODE_CONTIGUOUS && !C::SWAP;
    const bool swap_contig = C::SWAP && p.mode == MODE_CONTIGUOUS;
    short *s_gblk = reinterpret_cast<short *>(sA);
    short *s_rg = reinterpret_cast<short *>(smem + C::OFF_RG);
    int *s_ntab = reinterpret_cast<int *>(smem + C::OFF_MISC + 8);
    const int num_blocks = p.M / BLOCK_M;
    if (p.mode == MODE_MASKED || p.mode == MODE_NOPAD) {
        for (int g = threadIdx.x; g < p.G; g += NUM_THREADS) {
            int m = __ldg(p.masked_m + g);
            if (m < 0 || (p.mode == MODE_MASKED && m > p.M)) {
                raise_error(p.err, ERR_BAD_GROUP);
                m = m < 0 ? 0 : p.M;
            }
            s_mm[g] = m;
        }
    } else if (p.mode == MODE_KGROUPED) {
        for (int g = threadIdx.x; g < p.G; g += NUM_THREADS) {
            const int k = __ldg(p.masked_m + g);  // a K extent: a non-negative multiple of 128
            if (k < 0 || k % BLOCK_K) raise_error(p.err, ERR_BAD_GROUP);
            s_mm[g] = k < 0 ? 0 : k / BLOCK_K;
        }
    } else if (pair_contig || swap_contig) {
        // several independent loads in flight per thread (m_indices is usually cold in L2 here)
        constexpr int U = 8;
        for (int b0 = threadIdx.x; b0 < num_blocks; b0 += NUM_THREADS * U) {
            int g[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int b = b0 + u * NUM_THREADS;
                g[u] = b < num_blocks ? __ldg(p.m_indices + static_cast<size_t>(b) * BLOCK_M) : -1;
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int b = b0 + u * NUM_THREADS;
                if (b < num_blocks) s_gblk[b] = static_cast<short>(checked_group(p, g[u]));
            }
        }
    }
    __syncthreads();
    if (warp == EPI_WARP0) {
        if (p.mode == MODE_NOPAD) {
            build_group_rows(p.G, p.M, s_mm, s_off, p.err, lane);
            __syncwarp();
        }
        if (p.mode == MODE_KGROUPED) {
            // each group's first 128-K block (clipped to K) and first packed scale group (SF_GROUP blocks each)
            build_group_rows(p.G, p.K / BLOCK_K, s_mm, s_off, p.err, lane);
            __syncwarp();
            build_window_prefix(p.G, SF_GROUP, s_mm, s_prefix, lane);
        } else if (p.mode == MODE_MASKED || p.mode == MODE_NOPAD) {
            build_window_prefix(p.G, C::SWAP ? C::BN : C::TILE_M, s_mm, s_prefix, lane);
        } else if (pair_contig) {
            build_pair_windows(num_blocks, s_gblk, s_prefix, lane);
        } else if (swap_contig) {
            const int runs = build_run_heads(num_blocks, s_gblk, s_off, s_mm, s_rg, lane);
            if (lane == 0) *s_ntab = runs;
        }
        if (!swap_contig && lane == 0) *s_ntab = p.G;
    }
    if (swap_contig) {  // the runs' row ranges (every warp), then their chunk prefix
        __syncthreads();
        finish_runs(p.m_indices, p.M, *s_ntab, s_off, s_mm, s_rg, warp, NUM_THREADS / 32, lane);
        __syncthreads();
        if (warp == EPI_WARP0) build_window_prefix(*s_ntab, C::BN, s_mm, s_prefix, lane);
    }
    tc_fence_before_sync();
    __syncthreads();
    if constexpr (PAIR) cluster_sync();  // the peer's barriers exist before any cross-CTA signal
    tc_fence_after_sync();
    const uint32_t tmem_base = *s_tmem_base;

    const int ntab = *s_ntab;
    const SharedCtl ctl{s_abort, s_prefix, s_mm, s_off, s_gblk, s_rg, ntab};
    const int nkb = p.K / BLOCK_K;
    int total_windows;
    if (p.mode == MODE_MASKED || p.mode == MODE_NOPAD || swap_contig)
        total_windows = s_prefix[ntab];
    else if (pair_contig)
        total_windows = s_prefix[MAX_PAIR_WINDOWS];
    else
        total_windows = p.num_windows;
    const int total_tiles = total_windows * p.num_n_blocks;
    const int my_rows = BLOCK_M * static_cast<int>(rank);  // offset of this CTA's rows inside the window

    // This CTA's (pair's) tile sequence t = cluster_id + k * num_clusters, decoded once by all threads; every
    // role then reads tile k with one shared-memory load instead of decoding it (which can take global loads).
    const int my_tiles = total_tiles > cluster_id ? (total_tiles - cluster_id + num_clusters - 1) / num_clusters : 0;
    for (int k = threadIdx.x; k < min(my_tiles, TILE_LIST_CAP); k += NUM_THREADS) {
        Tile ti;
        const bool valid = decode_tile<C>(p, ctl, cluster_id + k * num_clusters, ti);
        s_tiles[k] = pack_tile(valid, ti);
    }
    __syncthreads();
    const SharedCtl ctl_main{s_abort, s_prefix, s_mm, s_off, nullptr, s_rg, ntab};  // the A ring holds operands now
    auto tile_at = [&](int k, Tile &ti) -> bool {
        if (k < TILE_LIST_CAP) return unpack_tile<C>(p, ctl_main, s_tiles[k], ti);
        return decode_tile<C>(p, ctl_main, cluster_id + k * num_clusters, ti);
    };

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            uint32_t armed = 0, armed_ph = 0;  // stages armed at least once / parity of their last arming
            bool ok = true;
            const uint32_t full_leader0 = PAIR ? map_shared_rank(smem_u32(&full[0]), 0) : 0u;
            // The packed scale atoms come from the pre-pass launched just before this kernel.  The first STAGES
            // stages' operand loads go out before waiting for it; their scale loads follow once it has finished
            // (their barriers are armed with the scale bytes up front, so no stage completes without them).
            auto load_scales = [&](int st, int ya, int yb) {
                uint8_t *sf_dst = sSF + st * C::SF_BYTES;
                if constexpr (PAIR) {
                    const uint32_t leader_full = full_leader0 + 8u * static_cast<uint32_t>(st);
                    tma_load_2d_pair(sf_dst, &tmap_sfa, leader_full, 0, ya);
                    tma_load_2d_pair(sf_dst + SF_ATOM_WORDS * 4, &tmap_sfb, leader_full, 0, yb);
                } else {
                    tma_load_2d(sf_dst, &tmap_sfa, &full[st], 0, ya);
                    tma_load_2d(sf_dst + SF_ATOM_WORDS * 4, &tmap_sfb, &full[st], 0, yb);
                }
            };
            bool scales_ready = false;
            int n_deferred = 0, issued = 0;
            int def_stage[8], def_ya[8], def_yb[8];
            static_assert(STAGES <= 8, "deferred scale loads are kept for at most 8 stages");
            auto wait_for_scales = [&]() {
                if (scales_ready) return;
                grid_dependency_wait();
                scales_ready = true;
                for (int i = 0; i < n_deferred; ++i) load_scales(def_stage[i], def_ya[i], def_yb[i]);
                n_deferred = 0;
            };
            // test hook: the first CTA (pair) starts its ring at stage 1, so stage 0 is never armed or loaded and
            // the tensor-core thread's first wait runs out
            if (p.skip_first_load && cluster_id == 0) s = 1;
            for (int k = 0; k < my_tiles && ok; ++k) {
                Tile ti;
                if (!tile_at(k, ti)) continue;
                // K-grouped: one B for all groups, each group contracts its own range of 128-K blocks and owns
                // its own packed scale groups
                const bool kgrouped = p.mode == MODE_KGROUPED;
                const int gb = kgrouped ? 0 : ti.g;                       // B's group
                const int tile_nkb = kgrouped ? ctl_main.mm[ti.g] : nkb;  // 128-K blocks of this tile
                const int kbase = kgrouped ? ctl_main.off[ti.g] : 0;      // its first 128-K block
                const int qbase = kgrouped ? ctl_main.prefix[ti.g] : 0;   // its first packed scale group
                int arow, brow, sfa_y0, sfb_y0;  // rows loaded through tmap_a / tmap_b, first scale atoms
                int a_k_rows = 0;  // B in the NN orientation: the first K row of the group in tmap_a (rows G*K)
                if constexpr (C::SWAP) {
                    // tmap_a covers B's rows (the MMA's M side), tmap_b the tokens (its N side); this CTA brings
                    // its 128 rows of B and its half of the tile's tokens (the MMA's N rounded to 16, split in two)
                    const int m = ctl_main.mm[ti.g];
                    const int cs = chunk_rows(m, C::BN);
                    const int nmma = (min(cs, m - ti.local_row0) + 15) & ~15;
                    const int gB = swap_contig ? ctl_main.rg[ti.g] : ti.g;  // (contiguous: ti.g is a run)
                    arow = gB * p.N + ti.n0 + my_rows;
                    a_k_rows = gB * p.K;
                    brow = ti.row0 + static_cast<int>(rank) * (nmma / CTAS);
                    // packed scale atoms: B side [g][128-row block of B][group] (every row of an atom holds the
                    // block's scale), token side [chunk][group][atom] over all groups' chunks in order
                    sfa_y0 = (gB * p.sfa_blocks + (ti.n0 + my_rows) / BLOCK_M) * p.num_sf_groups;
                    sfb_y0 = (ctl_main.prefix[ti.g] + ti.local_row0 / cs) * p.num_sf_groups * C::SFB_ATOMS;
                } else {
                    arow = ti.row0 + my_rows;
                    brow = gb * p.N + ti.n0 + static_cast<int>(rank) * C::B_ROWS;
                    // packed scale atoms: SFA [block][group], SFB [g][n block][group][atom]
                    // (no padding: atoms of each group's windows, CTAS blocks per window, after the earlier groups')
                    int sfa_block = (ti.local_row0 + my_rows) / BLOCK_M;
                    if (p.mode == MODE_MASKED)
                        sfa_block += ti.g * p.sfa_blocks;
                    else if (p.mode == MODE_NOPAD)
                        sfa_block += CTAS * ctl_main.prefix[ti.g];
                    else
                        sfa_block = (ti.row0 + my_rows) / BLOCK_M;
                    sfa_y0 = sfa_block * p.num_sf_groups + qbase;
                    // B scale words along K per tile: one per scale group, or (FP4 B) one per 128-K block
                    const int sfb_words = C::BF4 ? nkb : p.num_sf_groups;
                    sfb_y0 = ((gb * p.num_n_blocks + ti.nb) * sfb_words + qbase) * C::SFB_ATOMS;
                }
                for (int kb0 = 0; kb0 < tile_nkb; kb0 += C::KPS) {
                    // this stage carries scale atoms (the promotion path reads fp32 scales directly)
                    const bool group_start = !C::PROMO && (C::BF4 || kb0 % SF_GROUP == 0);
                    if (issued == STAGES) wait_for_scales();  // the ring is full: the MMAs need the scales now
                    if (!wait_bounded(&empty[s], ph ^ 1u, s_abort, p.err, p.wait_limit_ns)) { ok = false; break; }
                    uint8_t *a_dst = sA + s * C::A_BYTES;
                    uint8_t *b_dst = sB + s * C::B_BYTES;
                    const int q = kb0 / SF_GROUP;
                    const int nk = min(C::KPS, tile_nkb - kb0);  // K blocks in this stage
                    const uint32_t bytes =
                        static_cast<uint32_t>(nk * (C::A_BYTES1 + C::B_TX1) + (group_start ? C::SF_BYTES : 0));
                    if constexpr (PAIR) {
                        // Only the leader arms the barrier (with both CTAs' bytes); the peer's loads just count
                        // their bytes on it.  A peer load may land before the leader arms the phase: the
                        // transaction count dips below zero but the phase cannot complete before the arrival.
                        const uint32_t leader_full = full_leader0 + 8u * static_cast<uint32_t>(s);
                        if (rank == 0) mbar_arrive_expect_tx(&full[s], CTAS * bytes);
                        for (int i = 0; i < nk; ++i) {
                            const int x = (kbase + kb0 + i) * BLOCK_K;
                            if constexpr (C::BNN)  // 128 N columns x 128 K rows of B [G*K][N]
                                tma_load_2d_pair(a_dst + i * C::A_BYTES1, &tmap_a, leader_full, ti.n0 + my_rows,
                                                 a_k_rows + x);
                            else
                                tma_load_2d_pair(a_dst + i * C::A_BYTES1, &tmap_a, leader_full, x, arow);
                            tma_load_2d_pair(b_dst + i * C::B_BYTES1, &tmap_b, leader_full, x, brow);
                        }
                    } else {
                        mbar_arrive_expect_tx(&full[s], bytes);
                        for (int i = 0; i < nk; ++i) {
                            const int x = (kbase + kb0 + i) * BLOCK_K;
                            if constexpr (C::BNN)
                                tma_load_2d(a_dst + i * C::A_BYTES1, &tmap_a, &full[s], ti.n0, a_k_rows + x);
                            else
                                tma_load_2d(a_dst + i * C::A_BYTES1, &tmap_a, &full[s], x, arow);
                            tma_load_2d(b_dst + i * C::B_BYTES1, &tmap_b, &full[s], x, brow);
                        }
                    }
                    if (group_start) {
                        const int qb = C::BF4 ? kb0 : q;  // the stage's first B scale word
                        if (scales_ready) {
                            load_scales(s, sfa_y0 + q, sfb_y0 + qb * C::SFB_ATOMS);
                        } else {
                            def_stage[n_deferred] = s;
                            def_ya[n_deferred] = sfa_y0 + q;
                            def_yb[n_deferred] = sfb_y0 + qb * C::SFB_ATOMS;
                            ++n_deferred;
                        }
                    }
                    ++issued;
                    armed |= 1u << s;
                    armed_ph = (armed_ph & ~(1u << s)) | (ph << s);
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                }
            }
            wait_for_scales();  // (also after an abort: every armed stage gets all its bytes)
            if (!PAIR || rank == 0) {
                // let the loads still in flight land before shared memory goes away, also when a consumer gave
                // up on them (in a pair the bytes of both CTAs are counted on the leader's barrier; the final
                // cluster barrier holds the peer).  On the normal path every armed phase has completed already.
                for (int i = 0; i < STAGES; ++i) {
                    if (!(armed >> i & 1u)) continue;
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(&full[i], (armed_ph >> i) & 1u) && global_timer_ns() - t0 < p.wait_limit_ns) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer (leader CTA)
        if (C::PROMO && lane == 0 && rank == 0) {
            // fp32 scale promotion: each 128-K block's partial product goes to its own TMEM buffer of the current
            // partial stage (KPS buffers of BN columns; E2M1 B: each 32-K MMA to its own, KPS * PSUB buffers); the
            // epilogue warps release a partial stage once they have read it, so the MMAs run up to two stages
            // ahead of the promotion
            constexpr uint32_t IDESC_P = idesc_f8f6f4_e4m3(C::TILE_M, BN, C::BF4);
            int s = 0;
            uint32_t ph = 0;
            int pb = 0;  // partial stage
            uint32_t pb_ph = 0;
            bool ok = true;
            for (int k = 0; k < my_tiles && ok; ++k) {
                Tile ti;
                if (!tile_at(k, ti)) continue;
                // (K-grouped: the group's own K blocks; none: no stage, the epilogue writes zeros or nothing)
                const int tile_nkb = p.mode == MODE_KGROUPED ? ctl_main.mm[ti.g] : nkb;
                for (int kb0 = 0; kb0 < tile_nkb; kb0 += C::KPS) {
                    const int nk = min(C::KPS, tile_nkb - kb0);
                    if (!wait_bounded(&full[s], ph, s_abort, p.err, p.wait_limit_ns)) { ok = false; break; }
                    if (!wait_bounded(&tmem_empty[pb], pb_ph ^ 1u, s_abort, p.err, p.wait_limit_ns)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t a_stage = smem_u32(sA + s * C::A_BYTES);
                    const uint32_t b_stage = smem_u32(sB + s * C::B_BYTES);
                    for (int i = 0; i < nk; ++i) {
#pragma unroll
                        for (int kk = 0; kk < BLOCK_K / MMA_K; ++kk) {
                            // partial (pb * KPS + i) * PSUB + sub: the K block's, or (PSUB = 4) this 32-K slice's
                            const int part = (pb * C::KPS + i) * C::PSUB + (C::PSUB > 1 ? kk : 0);
                            tc_mma_f8<CTAS>(tmem_base + static_cast<uint32_t>(part * BN),
                                            sdesc_kmajor_sw128(a_stage + i * C::A_BYTES1 + kk * MMA_K),
                                            sdesc_kmajor_sw128(b_stage + i * C::B_BYTES1 + kk * MMA_K), IDESC_P,
                                            C::PSUB > 1 ? 0u : static_cast<uint32_t>(kk != 0));
                        }
                    }
                    tc_commit<CTAS>(&empty[s]);
                    tc_commit<CTAS>(&tmem_full[pb]);
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                    pb ^= 1;
                    if (pb == 0) pb_ph ^= 1u;
                }
            }
            tc_commit<CTAS>(drain);
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < p.wait_limit_ns) {
            }
        } else if (!C::PROMO && lane == 0 && rank == 0) {
            // (swapped operands: N is the tile's token count rounded up to 16, set per tile below)
            // (B in the NN orientation: the M-side operand is MN-major, bit 15 of the instruction descriptor)
            constexpr uint32_t IDESC = idesc_mxf8_e4m3(C::TILE_M, C::SWAP ? 0 : BN, C::BF4) | (C::BNN ? 1u << 15 : 0u);
            int s = 0;
            uint32_t ph = 0;
            int acc = 0;
            uint32_t acc_ph = 0;
            int sf_slot = 0;  // TMEM scale slot of the next scale group
            bool ok = true;
            for (int k = 0; k < my_tiles && ok; ++k) {
                Tile ti;
                if (!tile_at(k, ti)) continue;
                if (!wait_bounded(&tmem_empty[acc], acc_ph ^ 1u, s_abort, p.err, p.wait_limit_ns)) break;
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
                uint32_t sf_tmem = 0;
                uint32_t idesc_n = 0;  // N / 8 in bits 17..22 (swapped operands only)
                if constexpr (C::SWAP) {
                    const int m = ctl_main.mm[ti.g];
                    const int nmma = (min(chunk_rows(m, BN), m - ti.local_row0) + 15) & ~15;
                    idesc_n = static_cast<uint32_t>(nmma >> 3) << 17;
                }
                // (K-grouped: a group with no K blocks issues no MMA; its epilogue writes zeros or nothing)
                const int tile_nkb = p.mode == MODE_KGROUPED ? ctl_main.mm[ti.g] : nkb;
                for (int kb0 = 0; kb0 < tile_nkb; kb0 += C::KPS) {
                    const int nk = min(C::KPS, tile_nkb - kb0);
                    if (!wait_bounded(&full[s], ph, s_abort, p.err, p.wait_limit_ns)) { ok = false; break; }
                    tc_fence_after_sync();
                    if (C::BF4 || kb0 % SF_GROUP == 0) {
                        // the group's (FP4 B: the stage's) scales into the next TMEM slot (the slot's previous
                        // readers, SF_SLOTS slots back, were issued earlier and the tensor pipe runs in order)
                        sf_tmem = tmem_base + static_cast<uint32_t>(C::SF_TMEM_BASE + sf_slot * C::SF_COLS);
                        if (++sf_slot == C::SF_SLOTS) sf_slot = 0;
                        const uint32_t sf_smem = smem_u32(sSF + s * C::SF_BYTES);
                        tc_cp_32x128b_warpx4<CTAS>(sf_tmem, sdesc_rows16_noswizzle(sf_smem));
#pragma unroll
                        for (int a = 0; a < C::SFB_KB * C::SFB_ATOMS; ++a)
                            tc_cp_32x128b_warpx4<CTAS>(sf_tmem + 4 + 4 * a,
                                                       sdesc_rows16_noswizzle(sf_smem + 512 + 512 * a));
                    }
                    const uint32_t a_stage = smem_u32(sA + s * C::A_BYTES);
                    const uint32_t b_stage = smem_u32(sB + s * C::B_BYTES);
                    for (int i = 0; i < nk; ++i) {
                        const int kb = kb0 + i;
                        const uint32_t sub = static_cast<uint32_t>(kb % SF_GROUP);  // byte of the packed scales
                        const uint32_t a_base = a_stage + i * C::A_BYTES1;
                        const uint32_t b_base = b_stage + i * C::B_BYTES1;
                        // B's scales: the group's word (byte kb % 4) or, FP4 B, this K block's word in the slot,
                        // whose byte k is the scale of the 32-K sub-block the k-th MMA contracts
                        const uint32_t sf_b = sf_tmem + 4 + (C::BF4 ? static_cast<uint32_t>(4 * C::SFB_ATOMS * i) : 0u);
#pragma unroll
                        for (int k = 0; k < BLOCK_K / MMA_K; ++k) {
                            const uint32_t b_byte = C::BF4 ? static_cast<uint32_t>(k) : sub;
                            const uint32_t idesc = IDESC | idesc_n | (sub << 29) | (b_byte << 4);
                            // K step of an MN-major tile: 32 K-rows of 128 bytes
                            const uint64_t a_desc = C::BNN ? sdesc_mnmajor_sw128(a_base + k * MMA_K * 128)
                                                           : sdesc_kmajor_sw128(a_base + k * MMA_K);
                            tc_mma_mxf8<CTAS>(d_tmem, a_desc, sdesc_kmajor_sw128(b_base + k * MMA_K), idesc, sf_tmem,
                                              sf_b, (kb | k) != 0);
                        }
                    }
                    tc_commit<CTAS>(&empty[s]);
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                }
                if (!ok) break;
                tc_commit<CTAS>(&tmem_full[acc]);
                acc ^= 1;
                if (acc == 0) acc_ph ^= 1u;
            }
            // all tensor-core work of the pair must be complete before TMEM is released
            tc_commit<CTAS>(drain);
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < p.wait_limit_ns) {
            }
        }
    } else {
        // ---------------------------------------------------------------- epilogue (warps 2..5)
        // Each warp owns 32 rows (its TMEM lane quarter).  A 32-column chunk is converted to bf16 and, when all
        // 32 rows belong to the call, staged in shared memory (64-byte rows, 16-byte chunks XOR-swizzled by
        // (row / 2) % 4, the layout of a 64-byte-swizzle TMA box) and written by one TMA tensor store; rows and
        // columns outside D are clipped by the store.  Warps with rows the call must not write store their
        // owned rows directly.
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        const uint32_t tmem_empty_leader0 = PAIR ? map_shared_rank(smem_u32(&tmem_empty[0]), 0) : 0u;
        uint8_t *stage_buf = sEpi + (warp - EPI_WARP0) * 2 * EPI_CHUNK_BYTES;
        int acc = 0;
        uint32_t acc_ph = 0;
        int chunk_count = 0;  // chunks this warp has staged (selects the staging buffer)
        // Does this lane's row of the tile belong to the call (the rows D may be written at)?
        auto row_owned = [&](const Tile &ti, int row, int r_local) -> bool {
            if (p.mode == MODE_DENSE) return row < p.M;
            if (p.mode == MODE_CONTIGUOUS) return row < p.M && __ldg(p.m_indices + row) == ti.g;
            return ti.local_row0 + r_local < ctl.mm[ti.g];
        };
        // One 32-column bf16 chunk of this lane's row (h: 16 packed pairs): staged and written by one TMA tensor
        // store when all 32 rows of the warp belong to the call (tma_ok), else stored by the owning lanes.
        auto emit_bf16 = [&](const Tile &ti, int row, int c, const uint32_t(&h)[16], bool tma_ok, bool valid) {
            if (tma_ok) {
                uint8_t *buf = stage_buf + (chunk_count & 1) * EPI_CHUNK_BYTES;
                if (chunk_count >= 2) {
                    if (lane == 0) bulk_wait_group_read<1>();  // the store that last used buf has read it
                    __syncwarp();
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int sw = j ^ ((lane >> 1) & 3);
                    *reinterpret_cast<uint4 *>(buf + lane * 64 + sw * 16) =
                        make_uint4(h[4 * j], h[4 * j + 1], h[4 * j + 2], h[4 * j + 3]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&tmap_d, buf, ti.n0 + 32 * c, ti.row0 + my_rows + 32 * q);
                    bulk_commit_group();
                }
                ++chunk_count;
            } else if (valid) {
                __nv_bfloat16 *out = p.d + static_cast<size_t>(row) * p.N + ti.n0;
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int col = ti.n0 + 32 * c + 8 * j;
                    if (col < p.N)
                        *reinterpret_cast<uint4 *>(out + 32 * c + 8 * j) =
                            make_uint4(h[4 * j], h[4 * j + 1], h[4 * j + 2], h[4 * j + 3]);
                }
            }
        };
        // One 32-column fp32 chunk of this lane's row into D [G][M][N] (K-grouped calls): two 16-column halves
        // (64-byte rows, the swizzled staging of the bf16 chunks), each stored or added by one TMA operation on the
        // 3-D map, which clips rows past M.
        auto emit_f32 = [&](const Tile &ti, int c, const uint32_t(&r)[32]) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint8_t *buf = stage_buf + (chunk_count & 1) * EPI_CHUNK_BYTES;
                if (chunk_count >= 2) {
                    if (lane == 0) bulk_wait_group_read<1>();  // the store that last used buf has read it
                    __syncwarp();
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int sw = j ^ ((lane >> 1) & 3);
                    *reinterpret_cast<uint4 *>(buf + lane * 64 + sw * 16) =
                        make_uint4(r[16 * h + 4 * j], r[16 * h + 4 * j + 1], r[16 * h + 4 * j + 2],
                                   r[16 * h + 4 * j + 3]);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    const int x = ti.n0 + 32 * c + 16 * h, y = ti.row0 + my_rows + 32 * q;
                    if (p.out_mode == OUT_F32_ADD)
                        tma_reduce_add_3d(&tmap_d, buf, x, y, ti.g);
                    else
                        tma_store_3d(&tmap_d, buf, x, y, ti.g);
                    bulk_commit_group();
                }
                ++chunk_count;
            }
        };
        int pb = 0;  // promotion: the partial stage read next
        uint32_t pb_ph = 0;
        // this warp's two staging buffers of per-column B scales (promotion with sfb_cols)
        float *psb = reinterpret_cast<float *>(smem + C::OFF_PSB) + (warp - EPI_WARP0) * 2 * C::PSB_FLOATS;
        int psb_stage = 0;  // partial stages read with per-column scales (selects the staging buffer)
        // fp32 scale promotion of one tile: this lane's row accumulates partial * sfa[row, kb] * sfb over the tile's
        // K blocks in registers, then it is written as bf16 (or, K-grouped, fp32).  B's scale is either one per
        // 128-column block and K block (BN = 128: one value per partial, read by every lane), or one per column
        // (K-grouped: per K block; E2M1 B: per 32-K sub-block, one partial each).  Per-column scales are copied
        // into this warp's staging buffer one partial stage ahead and read back four columns at a time; the
        // per-row A scales (and the per-block B scale) are loaded into registers one stage ahead.  false = gave up.
        auto promote_tile = [&](const Tile &ti) -> bool {
            const int r_local = my_rows + 32 * q + lane;
            const int row = ti.row0 + r_local;
            constexpr bool kgrouped = C::PCOL && !C::BF4;  // (the K-grouped calls' configuration)
            const int tile_nkb = kgrouped ? ctl.mm[ti.g] : nkb;  // K blocks of this tile
            const int kbase = kgrouped ? ctl.off[ti.g] : 0;      // its first K block in the scale arrays
            constexpr bool col_scales = C::PCOL;
            bool row_in;          // the row exists in the A scale array (rows past it read no scale)
            long long sa_base;    // element of (row, K block 0); K block kb at sa_base + kb * sfa_ld
            if (p.mode == MODE_MASKED) {
                const int lrow = ti.local_row0 + r_local;
                row_in = lrow < p.M;
                sa_base = static_cast<long long>(ti.g) * nkb * p.sfa_ld + lrow;
            } else {
                row_in = row < p.M;
                sa_base = row;
            }
            const float *sfb_t = p.sfb32 + static_cast<long long>(ti.g) * p.sfb_sg +
                                 (col_scales ? static_cast<long long>(ti.n0)
                                             : static_cast<long long>(ti.n0 / 128) * p.sfb_sn);
            float acc_r[BN];
#pragma unroll
            for (int j = 0; j < BN; ++j) acc_r[j] = 0.f;
            float sa_n[C::KPS], sb_n[C::KPS];
            auto load_scales = [&](int kb0) {
#pragma unroll
                for (int i = 0; i < C::KPS; ++i) {
                    const int kb = kb0 + i;
                    const bool in = kb < tile_nkb;
                    const long long kg = kbase + kb;
                    sa_n[i] = (in && row_in) ? __ldg(p.sfa32 + sa_base + kg * p.sfa_ld) : 0.f;
                    sb_n[i] = (in && !col_scales) ? __ldg(sfb_t + kg * p.sfb_sk) : 0.f;
                    if (!col_scales && p.check_scales) {
                        const uint32_t ba = __float_as_uint(sa_n[i]), bb = __float_as_uint(sb_n[i]);
                        if (ue8m0_inexact_bits(ba) | ue8m0_inexact_bits(bb)) raise_error(p.err, ERR_BAD_SCALE);
                        if (ba == 0u) sa_n[i] = __uint_as_float(UE8M0_ZERO_F32_BITS);
                        if (bb == 0u) sb_n[i] = __uint_as_float(UE8M0_ZERO_F32_BITS);
                    }
                }
            };
            // the per-column scales of the partial stage starting at K block kb0: KPS * PSUB rows of BN columns
            // (row i = the scale row PSUB * (kbase + kb0) + i), 16 bytes per copy; rows past the tile's K blocks
            // and columns past N are zero-filled
            auto fetch_cols = [&](int kb0, int buf) {
                float *dst = psb + buf * C::PSB_FLOATS;
                constexpr int Q = BN / 4;                 // 16-byte copies per row
                constexpr int F4 = C::PSB_FLOATS / 4;     // and per stage
#pragma unroll
                for (int u = 0; u < (F4 + 31) / 32; ++u) {
                    const int f = lane + 32 * u;
                    if (F4 % 32 != 0 && f >= F4) break;
                    const int i = f / Q, c4 = f % Q;
                    const bool in = kb0 + i / C::PSUB < tile_nkb && ti.n0 + 4 * c4 < p.N;
                    const float *src =
                        sfb_t + static_cast<long long>(C::PSUB * (kbase + kb0) + i) * p.sfb_sk + 4 * c4;
                    cp_async_16(dst + 4 * f, in ? src : p.sfb32, in ? 16u : 0u);
                }
                cp_async_commit();
            };
            load_scales(0);
            if constexpr (col_scales) {
                if (tile_nkb > 0) fetch_cols(0, psb_stage & 1);
            }
            for (int kb0 = 0; kb0 < tile_nkb; kb0 += C::KPS) {
                const int nk = min(C::KPS, tile_nkb - kb0);
                const float *sbs = psb + (psb_stage & 1) * C::PSB_FLOATS;
                if constexpr (col_scales) {
                    if (kb0 + C::KPS < tile_nkb) {
                        __syncwarp();  // every lane is done with the other buffer (read two stages back)
                        fetch_cols(kb0 + C::KPS, (psb_stage + 1) & 1);
                        cp_async_wait<1>();
                    } else {
                        cp_async_wait<0>();
                    }
                    __syncwarp();  // this stage's copies by every lane are visible
                }
                if (!warp_wait_bounded(&tmem_full[pb], pb_ph, s_abort, p.err, p.wait_limit_ns, lane)) {
                    if constexpr (col_scales) cp_async_wait<0>();
                    return false;
                }
                tc_fence_after_sync();
                const uint32_t t_part = tmem_base + (static_cast<uint32_t>(32 * q) << 16) +
                                        static_cast<uint32_t>(pb * C::KPS * C::PSUB * BN);
                if constexpr (col_scales) {
#pragma unroll
                    for (int i = 0; i < C::KPS * C::PSUB; ++i) {
                        if (i / C::PSUB < nk) {
                            const float sa = sa_n[i / C::PSUB];
                            const float4 *sb4 = reinterpret_cast<const float4 *>(sbs + i * BN);
                            static_assert(BN == 64, "per-column promotion reads a partial as two 32-column loads");
                            uint32_t r[2][32];  // both halves of the partial in flight at once
                            tmem_ld_32x32b_x32(t_part + static_cast<uint32_t>(i * BN), r[0]);
                            tmem_ld_32x32b_x32(t_part + static_cast<uint32_t>(i * BN + 32), r[1]);
                            tmem_ld_wait_regs(r[0]);
                            tmem_ld_wait_regs(r[1]);
#pragma unroll
                            for (int c = 0; c < 2; ++c) {
#pragma unroll
                                for (int j = 0; j < 8; ++j) {
                                    const float4 v = lds_f32x4(sb4 + 8 * c + j);  // the same address in every lane
                                    const int o = 32 * c + 4 * j;
                                    // acc += (partial * sfb) * sfa, two columns per instruction
                                    float t0, t1, t2, t3;
                                    mul_f32x2(t0, t1, __uint_as_float(r[c][4 * j]), __uint_as_float(r[c][4 * j + 1]),
                                              v.x, v.y);
                                    mul_f32x2(t2, t3, __uint_as_float(r[c][4 * j + 2]),
                                              __uint_as_float(r[c][4 * j + 3]), v.z, v.w);
                                    fma_f32x2(acc_r[o], acc_r[o + 1], t0, t1, sa, sa);
                                    fma_f32x2(acc_r[o + 2], acc_r[o + 3], t2, t3, sa, sa);
                                }
                            }
                        }
                    }
                } else {
                    float sc[C::KPS];
#pragma unroll
                    for (int i = 0; i < C::KPS; ++i) sc[i] = sa_n[i] * sb_n[i];
#pragma unroll
                    for (int i = 0; i < C::KPS; ++i) {
                        if (i < nk) {
#pragma unroll
                            for (int c = 0; c < BN / 32; c += 2) {
                                uint32_t r0[32], r1[32];
                                tmem_ld_32x32b_x32(t_part + static_cast<uint32_t>(i * BN + 32 * c), r0);
                                tmem_ld_32x32b_x32(t_part + static_cast<uint32_t>(i * BN + 32 * c + 32), r1);
                                tmem_ld_wait_regs(r0);
                                tmem_ld_wait_regs(r1);
#pragma unroll
                                for (int j = 0; j < 32; j += 2) {  // acc += partial * (sfa * sfb), two columns at once
                                    fma_f32x2(acc_r[32 * c + j], acc_r[32 * c + j + 1], __uint_as_float(r0[j]),
                                              __uint_as_float(r0[j + 1]), sc[i], sc[i]);
                                    fma_f32x2(acc_r[32 * c + 32 + j], acc_r[32 * c + 33 + j], __uint_as_float(r1[j]),
                                              __uint_as_float(r1[j + 1]), sc[i], sc[i]);
                                }
                            }
                        }
                    }
                }
                // the partial stage has been read: the MMAs may overwrite it
                tc_fence_before_sync();
                __syncwarp();
                if (lane == 0) {
                    if constexpr (PAIR)
                        mbar_arrive_remote(tmem_empty_leader0 + 8u * static_cast<uint32_t>(pb));
                    else
                        mbar_arrive(&tmem_empty[pb]);
                }
                pb ^= 1;
                if (pb == 0) pb_ph ^= 1u;
                if constexpr (col_scales) ++psb_stage;
                if (kb0 + C::KPS < tile_nkb) load_scales(kb0 + C::KPS);
            }
            if constexpr (kgrouped) {  // fp32 D
                const int halves = tile_nkb == 0 && p.out_mode == OUT_F32_ADD ? 0 : BN / 16;  // (adding zeros)
#pragma unroll
                for (int hc = 0; hc < BN / 16; ++hc) {  // 16-column halves, straight from the accumulators
                    if (hc >= halves) break;
                    uint8_t *buf = stage_buf + (chunk_count & 1) * EPI_CHUNK_BYTES;
                    if (chunk_count >= 2) {
                        if (lane == 0) bulk_wait_group_read<1>();  // the store that last used buf has read it
                        __syncwarp();
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int sw = j ^ ((lane >> 1) & 3);
                        const float *v = acc_r + 16 * hc + 4 * j;
                        *reinterpret_cast<float4 *>(buf + lane * 64 + sw * 16) = make_float4(v[0], v[1], v[2], v[3]);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        const int x = ti.n0 + 16 * hc, y = ti.row0 + my_rows + 32 * q;
                        if (p.out_mode == OUT_F32_ADD)
                            tma_reduce_add_3d(&tmap_d, buf, x, y, ti.g);
                        else
                            tma_store_3d(&tmap_d, buf, x, y, ti.g);
                        bulk_commit_group();
                    }
                    ++chunk_count;
                }
            } else {
                const bool valid = row_owned(ti, row, r_local);
                const bool tma_ok = p.mode == MODE_DENSE || __all_sync(0xffffffffu, valid);
#pragma unroll
                for (int c = 0; c < BN / 32; ++c) {
                    uint32_t h[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        __nv_bfloat162 v = __floats2bfloat162_rn(acc_r[32 * c + 2 * j], acc_r[32 * c + 2 * j + 1]);
                        h[j] = *reinterpret_cast<uint32_t *>(&v);
                    }
                    emit_bf16(ti, row, c, h, tma_ok, valid);
                }
            }
            return true;
        };
        bool promo_ok = true;
        for (int k = 0; k < my_tiles && promo_ok; ++k) {
            Tile ti;
            if (!tile_at(k, ti)) continue;
            if constexpr (C::PROMO) {
                promo_ok = promote_tile(ti);
                continue;
            }
            if (!warp_wait_bounded(&tmem_full[acc], acc_ph, s_abort, p.err, p.wait_limit_ns, lane)) break;
            tc_fence_after_sync();
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(acc * BN);
            if constexpr (C::SWAP) {
                // Swapped operands: TMEM lane = a column of D (this CTA's rows of B), TMEM column j = the tile's
                // token j (row row0 + j of D).  Each 32-token chunk is converted to bf16, turned around with one
                // exchange between neighbouring lanes (a lane then holds two adjacent columns of one token row),
                // staged as 32 token rows of 64 bytes (the 64-byte-swizzle box layout) and written by one TMA
                // store when all 32 tokens belong to the call; the chunk with the tile's last tokens is stored by
                // the lanes, row by row.
                const int m = ctl.mm[ti.g];
                const int cnt = min(chunk_rows(m, BN), m - ti.local_row0);
                const int gB = swap_contig ? ctl.rg[ti.g] : ti.g;
                const int col0 = ti.n0 + my_rows + 32 * q;  // this warp's first column of D
                const bool odd = (lane & 1) != 0;
                const int pair_col = col0 + (lane & ~1);    // first of the two columns of this lane's words
                const int cb = 2 * (lane & ~1);             // their byte offset in a 64-byte token row
#pragma unroll 1
                for (int c = 0; c < (cnt + 31) / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(t_row + 32 * c, r);
                    tmem_ld_wait_regs(r);
                    // w[i]: token row 2i (even lane) or 2i + 1 (odd lane), columns pair_col and pair_col + 1
                    uint32_t w[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        __nv_bfloat162 v =
                            __floats2bfloat162_rn(__uint_as_float(r[2 * i]), __uint_as_float(r[2 * i + 1]));
                        const uint32_t own = *reinterpret_cast<uint32_t *>(&v);  // this column, tokens 2i, 2i + 1
                        const uint32_t other = __shfl_xor_sync(0xffffffffu, own, 1);
                        w[i] = odd ? ((other >> 16) | (own & 0xFFFF0000u)) : ((own & 0xFFFFu) | (other << 16));
                    }
                    const int tok0 = 32 * c;
                    // token rows of this chunk the call owns (contiguous: m_indices[row] == the group)
                    unsigned own;
                    if (swap_contig) {
                        const int row = ti.row0 + tok0 + lane;
                        own = __ballot_sync(0xffffffffu, tok0 + lane < cnt && row < p.M && __ldg(p.m_indices + row) == gB);
                    } else {
                        own = tok0 + 32 <= cnt ? 0xffffffffu : (1u << (cnt - tok0)) - 1u;
                    }
                    if (own == 0xffffffffu) {
                        uint8_t *buf = stage_buf + (chunk_count & 1) * EPI_CHUNK_BYTES;
                        if (chunk_count >= 2) {
                            if (lane == 0) bulk_wait_group_read<1>();  // the store that last used buf has read it
                            __syncwarp();
                        }
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int tr = 2 * i + (odd ? 1 : 0);
                            const int sw = (cb >> 4) ^ ((tr >> 1) & 3);
                            *reinterpret_cast<uint32_t *>(buf + tr * 64 + sw * 16 + (cb & 15)) = w[i];
                        }
                        fence_proxy_async_smem();
                        __syncwarp();
                        if (lane == 0) {
                            tma_store_2d(&tmap_d, buf, col0, ti.row0 + tok0);
                            bulk_commit_group();
                        }
                        ++chunk_count;
                    } else if (pair_col < p.N) {
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int t = 2 * i + (odd ? 1 : 0);
                            if ((own >> t) & 1u)
                                *reinterpret_cast<uint32_t *>(p.d + static_cast<size_t>(ti.row0 + tok0 + t) * p.N +
                                                              pair_col) = w[i];
                        }
                    }
                }
            } else if (p.out_mode != OUT_BF16) {
                // fp32 D [G][M][N] (K-grouped): per 32-column TMEM load, two TMA stores or adds of 16 columns
                const bool no_k = ctl.mm[ti.g] == 0;  // an empty K range: the accumulator holds nothing
                if (!(no_k && p.out_mode == OUT_F32_ADD)) {  // (adding zeros)
#pragma unroll 1
                    for (int c = 0; c < BN / 32; ++c) {
                        uint32_t r[32];
                        tmem_ld_32x32b_x32(t_row + 32 * c, r);
                        tmem_ld_wait_regs(r);
                        if (no_k) {
#pragma unroll
                            for (int j = 0; j < 32; ++j) r[j] = 0u;
                        }
                        emit_f32(ti, c, r);
                    }
                }
            } else {
                const int r_local = my_rows + 32 * q + lane;
                const int row = ti.row0 + r_local;
                const bool valid = row_owned(ti, row, r_local);
                // dense rows past M lie outside D and are clipped by the store
                const bool tma_ok = p.mode == MODE_DENSE || __all_sync(0xffffffffu, valid);
#pragma unroll 1
                for (int c = 0; c < BN / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld_32x32b_x32(t_row + 32 * c, r);
                    tmem_ld_wait_regs(r);
                    uint32_t h[16];
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        __nv_bfloat162 v =
                            __floats2bfloat162_rn(__uint_as_float(r[2 * j]), __uint_as_float(r[2 * j + 1]));
                        h[j] = *reinterpret_cast<uint32_t *>(&v);
                    }
                    emit_bf16(ti, row, c, h, tma_ok, valid);
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) {
                if constexpr (PAIR)
                    mbar_arrive_remote(tmem_empty_leader0 + 8u * static_cast<uint32_t>(acc));
                else
                    mbar_arrive(&tmem_empty[acc]);
            }
            acc ^= 1;
            if (acc == 0) acc_ph ^= 1u;
        }
        if (lane == 0) bulk_wait_group_all();  // the tensor stores finish before the CTA's shared memory goes away
        __syncwarp();
    }

    tc_fence_before_sync();
    __syncthreads();
    if constexpr (PAIR) cluster_sync();  // neither CTA leaves while the pair may still touch its memory
    if (clock_rec) {
        atomicAdd(p.clock_acc, static_cast<unsigned long long>(clock64()) - clk0);
        atomicAdd(p.clock_acc + 1, global_timer_ns() - ns0);
        atomicAdd(p.clock_acc + 2, 1ull);
    }
    if (warp == 1) {
        __syncwarp();
        tc_fence_after_sync();
        tmem_dealloc<CTAS>(tmem_base, TMEM_COLS);
    }
}

}  // namespace dg
