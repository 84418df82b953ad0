// Scale-factor pre-pass: fp32 power-of-two scales -> packed UE8M0 atoms in the layout tcgen05.cp reads.
//
// An atom is 128 rows x one 32-bit word (512 bytes).  Byte i of a row's word is the UE8M0 code (the fp32
// exponent field) of the row's scale for K block 4q + i of scale group q.  Inside an atom, row r sits at
// word (r % 32) * 4 + r / 32: tcgen05.cp .32x128b hands lane l the 16 bytes of rows l, l+32, l+64, l+96,
// i.e. TMEM column c of the scale slot holds rows 32c .. 32c+31, which is where the block-scaled MMA reads
// the scale of row (or column) 32c + lane.
//
//   SFA atoms: [128-row block][group]       block over A's rows (masked: G x blocks-per-group; no padding:
//                                           the blocks of each group's windows, 128*CTAS rows per window,
//                                           after the earlier groups', starting at the group's first row)
//   SFB atoms: [g][N tile][group][atom a]   rows a*128 .. a*128+127 of the BN-wide N tile (tile-aligned,
//                                           so a tile whose start is not a multiple of 128 still gets one
//                                           word per output column in the right TMEM lane)
// Swapped operands (masked layout; the MMA's M side runs over B's rows, its N side over a group's tokens):
//   B-side atoms:     [g][128-row block of B][group]   every row holds the 128x128 block's scale
//   token-side atoms: [chunk][group][atom a]           rows a*128 .. a*128+127 of the chunk's tokens, the
//                                                      chunks of all groups in order (group g's first chunk
//                                                      is the sum of the earlier groups' chunk counts)
// Entries past the problem (rows >= the scale extent, K blocks >= K/128, columns >= N) hold 0x7F (2^0).
#pragma once
#include <cstdint>

#include "gemm_kernel.cuh"

namespace dg {

struct PackParams {
    int mode;             // the GEMM's layout (MODE_*)
    const int *counts;    // no padding: the groups' row counts (device)
    int tile_m;           // no padding: rows per window (128 * CTAS)
    // SFA: fp32 MN-major [K/128][ld] (masked: [G][K/128][ld])
    const float *sfa;
    int sfa_ld;
    int rows_per_group;   // masked: M_max; otherwise the row extent (M or M_total)
    int blocks_per_group; // 128-row blocks per group (masked) or in total (no padding: an upper bound)
    int sfa_groups;       // G for masked, 1 otherwise
    // SFB: fp32 [G][ceil(N/128)][K/128], or [G][K/128][ceil(N/128)] when sfb_kn (B in the NN orientation)
    const float *sfb;
    int sfb_kn;
    int sfb_ld;           // K-grouped: row extent of the MN-major SFB [K/128][sfb_ld]; FP4 B: of [G][K/32][sfb_ld]
    int sfb_fp4;          // B in E2M1: one scale per (row, 32-K block); a B word holds a 128-K block's four
    int sfb_kwords;       // B scale words along K per (group, N tile): num_sf_groups, or K/128 when sfb_fp4
    int N, G, bn, n_tiles, sfb_atoms;
    int nkb, num_sf_groups;
    const int *m_indices; // contiguous: row -> group (-1 = padding); only rows of a group have their scales checked
    unsigned *err;        // device error word: ERR_BAD_SCALE for a scale the call reads that is not a power of two
    int swap;             // swapped operands (masked layout): sfa_out holds B's atoms, sfb_out the tokens'
    int b_blocks;         // swapped: 128-row blocks of B per group in sfa_out (past N: 2^0)
    int chunks;           // swapped: token chunks sfb_out has room for (chunk size chunk_rows(group rows, bn))
    uint32_t *sfa_out;    // [sfa_groups * blocks_per_group][num_sf_groups][128]
    uint32_t *sfb_out;    // [G][n_tiles][num_sf_groups][sfb_atoms][128]
    long long sfa_words, sfb_words;
};

// (ue8m0_inexact_bits, shared with the promotion GEMM's scale check, is in gemm_kernel.cuh)
constexpr uint32_t ONE_F32_BITS = 0x3F800000u;  // 1.0f: the code 0x7F written for entries past the problem

// Most threads per block of the pre-pass (the host launches at most one block per SM).
constexpr int PACK_THREADS = 1024;

// One warp per atom: lane l builds the words of rows l, l+32, l+64, l+96 (words 4l .. 4l+3) and writes them
// with one 16-byte store, so an atom is one coalesced 512-byte write.  (Swapped operands' B-side atoms, one word
// repeated in every row, are built 32 to a warp: one round of scale loads for all of them.)
__global__ void __launch_bounds__(PACK_THREADS) pack_scales_kernel(const PackParams p) {
    grid_launch_dependents();  // the GEMM may start its prologue; it waits for this grid before reading
    // The group tables, as the GEMM derives them.  No padding: clamped row counts, first rows, window prefix.
    // K-grouped: 128-K blocks per group, first 128-K block, prefix of packed scale groups (SF_GROUP blocks).
    // Contiguous layout with swapped operands: the runs of blocks of one group (s_cnt: rows, s_off: first row,
    // s_rg: group), built as the GEMM builds them.
    __shared__ int s_cnt[MAX_MASKED_GROUPS], s_off[MAX_MASKED_GROUPS + 1], s_wpre[MAX_MASKED_GROUPS + 1];
    __shared__ short s_rg[MAX_MASKED_GROUPS], s_gb[MAX_MASKED_GROUPS];
    __shared__ int s_runs;
    const bool nopad = p.mode == MODE_NOPAD, kgrouped = p.mode == MODE_KGROUPED;
    const bool swap_contig = p.swap && p.mode == MODE_CONTIGUOUS;
    int ntab = p.G;  // entries of the tables
    if (swap_contig) {
        const int num_blocks = p.rows_per_group / 128;  // (at most MAX_MASKED_GROUPS: checked by the host)
        for (int b = threadIdx.x; b < num_blocks; b += blockDim.x) {
            const int g = __ldg(p.m_indices + static_cast<size_t>(b) * 128);
            s_gb[b] = static_cast<short>(g >= 0 && g < p.G ? g : -1);
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            const int runs = build_run_heads(num_blocks, s_gb, s_off, s_cnt, s_rg, threadIdx.x);
            if (threadIdx.x == 0) s_runs = runs;
        }
        __syncthreads();
        ntab = s_runs;
        finish_runs(p.m_indices, p.rows_per_group, ntab, s_off, s_cnt, s_rg, threadIdx.x >> 5, blockDim.x >> 5,
                    threadIdx.x & 31);
        __syncthreads();
        if (threadIdx.x < 32) build_window_prefix(ntab, p.bn, s_cnt, s_wpre, threadIdx.x);
        __syncthreads();
    } else if (nopad || kgrouped || p.swap) {
        for (int g = threadIdx.x; g < p.G; g += blockDim.x) {
            const int c = __ldg(p.counts + g);
            s_cnt[g] = c < 0 ? 0 : (kgrouped ? c / 128 : (p.mode == MODE_MASKED ? min(c, p.rows_per_group) : c));
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            if (p.mode != MODE_MASKED)
                build_group_rows(p.G, kgrouped ? p.nkb : p.rows_per_group, s_cnt, s_off, nullptr, threadIdx.x);
            __syncwarp();
            // chunks (swapped operands), windows (no padding) or packed scale groups (K-grouped) per group
            build_window_prefix(p.G, p.swap ? p.bn : (kgrouped ? SF_GROUP : p.tile_m), s_cnt, s_wpre, threadIdx.x);
        }
        __syncthreads();
    }
    // the 128-K blocks of packed scale group q: first block and how many exist (K-grouped: q counts the groups'
    // scale groups one after another, each group's starting at its own first block)
    auto k_blocks = [&](int q, int &kb_first, int &kb_count) {
        if (!kgrouped) {
            kb_first = SF_GROUP * q;
            kb_count = p.nkb - kb_first;
        } else if (q < s_wpre[p.G]) {
            const int g = upper_index(s_wpre, p.G, q);
            const int local = SF_GROUP * (q - s_wpre[g]);
            kb_first = s_off[g] + local;
            kb_count = s_cnt[g] - local;
        } else {
            kb_first = 0;
            kb_count = 0;  // past the last scale group: never read
        }
    };
    const long long sfa_atoms = p.sfa_words / SF_ATOM_WORDS;
    const long long total = sfa_atoms + p.sfb_words / SF_ATOM_WORDS;
    const int lane = threadIdx.x & 31;
    const int warps_per_block = blockDim.x >> 5;
    const long long num_warps = static_cast<long long>(gridDim.x) * warps_per_block;
    const int nnb128 = (p.N + 127) / 128;
    uint32_t bad_bits = 0;  // nonzero once this lane read a scale the block-scaled MMA cannot represent
    // Work items of the warps.  Swapped operands: first the B-side atoms 32 at a time (each holds one word, the
    // same in all 128 rows: lane l builds the word of the batch's atom l, then the warp writes the 32 atoms), then
    // the token-side atoms one each.  Otherwise the A-side atoms one each, then the B-side atoms: 32 at a time when
    // B has one scale per 128 x 128 block (an atom's 128 rows then hold at most two words, those of the two
    // blocks it meets), else (K-grouped, E2M1 B: a scale per row) one each.
    const long long b_batches = p.swap ? (sfa_atoms + 31) / 32 : 0;
    const bool sfb_batched = !p.swap && !kgrouped && !p.sfb_fp4;
    const long long sfb_total = total - sfa_atoms;
    const long long items = p.swap ? b_batches + sfb_total : (sfb_batched ? sfa_atoms + (sfb_total + 31) / 32 : total);
    // (item i goes to warp i / gridDim.x of block i % gridDim.x: the B-side batches, 16 KB of stores each, spread
    // over all SMs instead of filling the first blocks, and the blocks finish at about the same time)
    for (long long item = static_cast<long long>(threadIdx.x >> 5) * gridDim.x + blockIdx.x; item < items;
         item += num_warps) {
        if (sfb_batched && item >= sfa_atoms) {  // 32 B-side atoms [G][n_tiles][num_sf_groups][sfb_atoms]
            const long long first_b = (item - sfa_atoms) * 32;
            const long long b = first_b + lane;  // this lane's atom
            constexpr uint32_t PAST_N = 0x7F7F7F7Fu;  // rows past N: 2^0 in all four bytes
            uint32_t w0 = PAST_N, w1 = PAST_N;        // words of the atom's first 128-row block and the next
            int n_first = 0;                          // the atom's first row of B
            if (b < sfb_total) {
                const int a = static_cast<int>(b % p.sfb_atoms);
                long long rest = b / p.sfb_atoms;
                const int q = static_cast<int>(rest % p.sfb_kwords);
                rest /= p.sfb_kwords;
                const int nt = static_cast<int>(rest % p.n_tiles);
                const long long g = rest / p.n_tiles;
                n_first = nt * p.bn + a * 128;
                const int blk0 = n_first / 128;
                const int n_end = min(p.N, n_first + 128);  // the atom's rows below N: n_first .. n_end - 1
                int kb_first, kb_count;
                k_blocks(q, kb_first, kb_count);
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int blk = blk0 + h;
                    if (blk * 128 >= n_end || (h == 1 && n_first % 128 == 0)) continue;  // no row of the atom in it
                    // [G][N/128][K/128], or [G][K/128][N/128] for B in the NN orientation
                    const float *base = p.sfb_kn ? p.sfb + g * p.nkb * nnb128 + blk : p.sfb + (g * nnb128 + blk) * p.nkb;
                    const size_t stride_kb = p.sfb_kn ? static_cast<size_t>(nnb128) : 1;
                    uint32_t wv = 0;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int kb = kb_first + i;
                        const uint32_t bits = i < kb_count ? __float_as_uint(__ldg(base + kb * stride_kb)) : ONE_F32_BITS;
                        wv |= ((bits >> 23) & 0xFFu) << (8 * i);
                        bad_bits |= ue8m0_inexact_bits(bits);
                    }
                    (h == 0 ? w0 : w1) = wv;
                }
            }
#pragma unroll 2
            for (int i = 0; i < 32; ++i) {
                const uint32_t x0 = __shfl_sync(0xffffffffu, w0, i), x1 = __shfl_sync(0xffffffffu, w1, i);
                const int nf = __shfl_sync(0xffffffffu, n_first, i);
                if (first_b + i >= sfb_total) break;  // (the same for every lane)
                uint32_t word[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int n = nf + lane + 32 * j;
                    word[j] = n >= p.N ? PAST_N : (n / 128 == nf / 128 ? x0 : x1);
                }
                *reinterpret_cast<uint4 *>(p.sfb_out + (first_b + i) * SF_ATOM_WORDS + 4 * lane) =
                    make_uint4(word[0], word[1], word[2], word[3]);
            }
            continue;
        }
        if (p.swap && item < b_batches) {  // B side: the block scales of 128 rows of B
            const long long atom = item * 32 + lane;
            uint32_t wv = 0;
            if (atom < sfa_atoms) {
                const int q = static_cast<int>(atom % p.num_sf_groups);
                const long long rest = atom / p.num_sf_groups;
                const int blk = static_cast<int>(rest % p.b_blocks);
                const long long g = rest / p.b_blocks;
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int kb = SF_GROUP * q + i;
                    const bool in = blk < nnb128 && kb < p.nkb;
                    // [G][N/128][K/128], or [G][K/128][N/128] for B in the NN orientation
                    const long long idx = p.sfb_kn ? (g * p.nkb + kb) * nnb128 + blk : (g * nnb128 + blk) * p.nkb + kb;
                    const uint32_t bits = in ? __float_as_uint(__ldg(p.sfb + idx)) : ONE_F32_BITS;
                    wv |= ((bits >> 23) & 0xFFu) << (8 * i);
                    if (in) bad_bits |= ue8m0_inexact_bits(bits);
                }
            }
            const long long n_here = sfa_atoms - item * 32;  // atoms of this batch (32 except the last)
#pragma unroll 4
            for (int i = 0; i < 32; ++i) {
                const uint32_t w = __shfl_sync(0xffffffffu, wv, i);
                if (i < n_here)
                    *reinterpret_cast<uint4 *>(p.sfa_out + (item * 32 + i) * SF_ATOM_WORDS + 4 * lane) =
                        make_uint4(w, w, w, w);
            }
            continue;
        }
        const long long atom = p.swap ? sfa_atoms + (item - b_batches) : item;
        uint32_t word[4] = {0u, 0u, 0u, 0u};
        uint32_t *dst;
        if (p.swap) {
            {  // token side: the per-row scales of 256 tokens of one chunk of one group
                const long long b = atom - sfa_atoms;
                const int b32 = static_cast<int>(b);  // (token-side atoms: chunks x scale groups x 2, far below 2^31)
                const int a = b32 % p.sfb_atoms;
                const int rest = b32 / p.sfb_atoms;
                const int q = rest % p.num_sf_groups;
                const int w = rest / p.num_sf_groups;  // chunk over all groups (runs)
                if (w >= s_wpre[ntab]) continue;  // past the last chunk: never read
                const int g = upper_index(s_wpre, ntab, w);  // group, or run (contiguous)
                const int m = s_cnt[g];
                const int cs = chunk_rows(m, p.bn);
                const int c = w - s_wpre[g];
                const long long first = p.mode == MODE_MASKED ? 0 : s_off[g];  // the group's first token row
                const int gid = swap_contig ? s_rg[g] : g;
                const float *base = p.sfa + (p.mode == MODE_MASKED ? static_cast<long long>(g) * p.nkb * p.sfa_ld : 0);
                // all sixteen loads (four rows x four K blocks) first, then the words
                long long tok[4];
                bool in[4], check[4];
                uint32_t bits[4][4];
                int grp[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int r = a * 128 + lane + 32 * j;
                    const long long local = static_cast<long long>(c) * cs + r;  // token within the group
                    tok[j] = first + local;
                    in[j] = tok[j] < p.sfa_ld;
                    check[j] = in[j] && local < m && r < cs;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int kb = SF_GROUP * q + i;
                        bits[j][i] = (in[j] && kb < p.nkb)
                                         ? __float_as_uint(__ldg(base + static_cast<size_t>(kb) * p.sfa_ld + tok[j]))
                                         : ONE_F32_BITS;
                    }
                    grp[j] = swap_contig && check[j] ? __ldg(p.m_indices + tok[j]) : gid;
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    // scales of rows the call owns are checked (contiguous: rows whose m_indices is the group)
                    const bool chk = check[j] && grp[j] == gid;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        word[j] |= ((bits[j][i] >> 23) & 0xFFu) << (8 * i);
                        if (chk && SF_GROUP * q + i < p.nkb) bad_bits |= ue8m0_inexact_bits(bits[j][i]);
                    }
                }
                dst = p.sfb_out + b * SF_ATOM_WORDS;
            }
        } else if (atom < sfa_atoms) {
            const int q = static_cast<int>(atom % p.num_sf_groups);
            const long long block = atom / p.num_sf_groups;
            long long group_base = 0;  // masked: the group's scale array
            int first = 0, rows = 0;   // the block's first row in the scale array, rows of it that exist
            if (nopad) {
                const int per_window = p.tile_m / 128;
                const long long window = block / per_window;
                if (window < s_wpre[p.G]) {  // (blocks past the last window are never read)
                    const int g = upper_index(s_wpre, p.G, static_cast<int>(window));
                    const int local = static_cast<int>(block - static_cast<long long>(per_window) * s_wpre[g]) * 128;
                    first = s_off[g] + local;
                    rows = s_cnt[g] - local;
                }
            } else {
                const int g = static_cast<int>(block / p.blocks_per_group);
                group_base = static_cast<long long>(g) * p.nkb * p.sfa_ld;
                first = static_cast<int>(block % p.blocks_per_group) * 128;
                rows = p.rows_per_group - first;
            }
            const float *base = p.sfa + group_base;
            int kb_first, kb_count;
            k_blocks(q, kb_first, kb_count);
            // rows whose scales the call uses: masked, below the group's masked_m; contiguous, rows of a group
            int owned = rows;
            if (p.mode == MODE_MASKED) {
                const int m = __ldg(p.counts + block / p.blocks_per_group);
                owned = min(max(m, 0), p.rows_per_group) - first;
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int r = lane + 32 * j;
                const int row = first + r;
                const bool in = r < rows && row < p.sfa_ld;
                const bool check =
                    in && r < owned && (p.mode != MODE_CONTIGUOUS || __ldg(p.m_indices + row) >= 0);
                uint32_t bits[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int kb = kb_first + i;
                    bits[i] = (in && i < kb_count)
                                  ? __float_as_uint(__ldg(base + static_cast<size_t>(kb) * p.sfa_ld + row))
                                  : ONE_F32_BITS;
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    word[j] |= ((bits[i] >> 23) & 0xFFu) << (8 * i);
                    if (check) bad_bits |= ue8m0_inexact_bits(bits[i]);
                }
            }
            dst = p.sfa_out + atom * SF_ATOM_WORDS;
        } else {
            const long long b = atom - sfa_atoms;
            const int a = static_cast<int>(b % p.sfb_atoms);
            long long rest = b / p.sfb_atoms;
            const int q = static_cast<int>(rest % p.sfb_kwords);
            rest /= p.sfb_kwords;
            const int nt = static_cast<int>(rest % p.n_tiles);
            const int g = static_cast<int>(rest / p.n_tiles);
            int kb_first, kb_count;
            k_blocks(q, kb_first, kb_count);
            if (p.sfb_fp4) {  // the word of 128-K block q: bytes i = its 32-K sub-blocks 4q + i
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int n = nt * p.bn + a * 128 + lane + 32 * j;
                    const float *base = p.sfb + static_cast<size_t>(g) * (4 * p.nkb) * p.sfb_ld + n;
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const uint32_t bits = (n < p.N && q < p.nkb)
                                                  ? __float_as_uint(__ldg(base + static_cast<size_t>(4 * q + i) * p.sfb_ld))
                                                  : ONE_F32_BITS;
                        word[j] |= ((bits >> 23) & 0xFFu) << (8 * i);
                        bad_bits |= ue8m0_inexact_bits(bits);
                    }
                }
                dst = p.sfb_out + b * SF_ATOM_WORDS;
                *reinterpret_cast<uint4 *>(dst + 4 * lane) = make_uint4(word[0], word[1], word[2], word[3]);
                continue;
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int n = nt * p.bn + a * 128 + lane + 32 * j;
                // SFB element of column n and K block kb sits at base + kb * stride_kb: 128x128 blocks
                // [G][N/128][K/128] or, NN, [G][K/128][N/128]; K-grouped: one scale per row n, [K/128][sfb_ld]
                size_t stride_kb;
                const float *base;
                if (kgrouped) {
                    stride_kb = static_cast<size_t>(p.sfb_ld);
                    base = p.sfb + n;
                } else if (p.sfb_kn) {
                    stride_kb = static_cast<size_t>(nnb128);
                    base = p.sfb + static_cast<size_t>(g) * p.nkb * nnb128 + n / 128;
                } else {
                    stride_kb = 1;
                    base = p.sfb + (static_cast<size_t>(g) * nnb128 + n / 128) * p.nkb;
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int kb = kb_first + i;
                    const uint32_t bits =
                        (n < p.N && i < kb_count) ? __float_as_uint(__ldg(base + kb * stride_kb)) : ONE_F32_BITS;
                    word[j] |= ((bits >> 23) & 0xFFu) << (8 * i);
                    bad_bits |= ue8m0_inexact_bits(bits);
                }
            }
            dst = p.sfb_out + b * SF_ATOM_WORDS;
        }
        *reinterpret_cast<uint4 *>(dst + 4 * lane) = make_uint4(word[0], word[1], word[2], word[3]);
    }
    if (__any_sync(0xffffffffu, bad_bits != 0) && lane == 0) raise_error(p.err, ERR_BAD_SCALE);
}

}  // namespace dg
