// Scale-factor pre-pass: fp32 power-of-two scales -> packed UE8M0 atoms in the layout tcgen05.cp reads.
//
// An atom is 128 rows x one 32-bit word (512 bytes).  Byte i of a row's word is the UE8M0 code (the fp32
// exponent field) of the row's scale for K block 4q + i of scale group q.  Inside an atom, row r sits at
// word (r % 32) * 4 + r / 32: tcgen05.cp .32x128b hands lane l the 16 bytes of rows l, l+32, l+64, l+96,
// i.e. TMEM column c of the scale slot holds rows 32c .. 32c+31, which is where the block-scaled MMA reads
// the scale of row (or column) 32c + lane.
//
//   SFA atoms: [128-row block][group]       block over A's rows (masked: G x blocks-per-group)
//   SFB atoms: [g][N tile][group][atom a]   rows a*128 .. a*128+127 of the BN-wide N tile (tile-aligned,
//                                           so a tile whose start is not a multiple of 128 still gets one
//                                           word per output column in the right TMEM lane)
// Entries past the problem (rows >= the scale extent, K blocks >= K/128, columns >= N) hold 0x7F (2^0).
#pragma once
#include <cstdint>

#include "gemm_kernel.cuh"

namespace dg {

struct PackParams {
    // SFA: fp32 MN-major [K/128][ld] (masked: [G][K/128][ld])
    const float *sfa;
    int sfa_ld;
    int rows_per_group;   // masked: M_max; otherwise the row extent (M or M_total)
    int blocks_per_group; // 128-row blocks per group (masked) or in total
    int sfa_groups;       // G for masked, 1 otherwise
    // SFB: fp32 [G][ceil(N/128)][K/128]
    const float *sfb;
    int N, G, bn, n_tiles, sfb_atoms;
    int nkb, num_sf_groups;
    uint32_t *sfa_out;    // [sfa_groups * blocks_per_group][num_sf_groups][128]
    uint32_t *sfb_out;    // [G][n_tiles][num_sf_groups][sfb_atoms][128]
    long long sfa_words, sfb_words;
};

__device__ __forceinline__ uint32_t ue8m0_code(float s) { return (__float_as_uint(s) >> 23) & 0xFFu; }

__global__ void __launch_bounds__(256) pack_scales_kernel(const PackParams p) {
    grid_launch_dependents();  // the GEMM may start its prologue; it waits for this grid before reading
    const long long total = p.sfa_words + p.sfb_words;
    const int nnb128 = (p.N + 127) / 128;
    for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
         idx += static_cast<long long>(gridDim.x) * blockDim.x) {
        const int w = static_cast<int>(idx % SF_ATOM_WORDS);
        const int r = (w >> 2) + 32 * (w & 3);  // atom row stored at word w
        uint32_t word = 0;
        if (idx < p.sfa_words) {
            const long long atom = idx / SF_ATOM_WORDS;
            const int q = static_cast<int>(atom % p.num_sf_groups);
            const long long block = atom / p.num_sf_groups;
            const int g = static_cast<int>(block / p.blocks_per_group);
            const int lb = static_cast<int>(block % p.blocks_per_group);
            const int row = lb * 128 + r;
            const float *base = p.sfa + static_cast<size_t>(g) * p.nkb * p.sfa_ld;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int kb = 4 * q + i;
                const uint32_t code = (row < p.sfa_ld && row < p.rows_per_group && kb < p.nkb)
                                          ? ue8m0_code(__ldg(base + static_cast<size_t>(kb) * p.sfa_ld + row))
                                          : 0x7Fu;
                word |= code << (8 * i);
            }
            p.sfa_out[idx] = word;
        } else {
            const long long j = idx - p.sfa_words;
            long long atom = j / SF_ATOM_WORDS;
            const int a = static_cast<int>(atom % p.sfb_atoms);
            atom /= p.sfb_atoms;
            const int q = static_cast<int>(atom % p.num_sf_groups);
            atom /= p.num_sf_groups;
            const int nt = static_cast<int>(atom % p.n_tiles);
            const int g = static_cast<int>(atom / p.n_tiles);
            const int n = nt * p.bn + a * 128 + r;
            const float *base = p.sfb + (static_cast<size_t>(g) * nnb128 + n / 128) * p.nkb;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int kb = 4 * q + i;
                const uint32_t code = (n < p.N && kb < p.nkb) ? ue8m0_code(__ldg(base + kb)) : 0x7Fu;
                word |= code << (8 * i);
            }
            p.sfb_out[j] = word;
        }
    }
}

}  // namespace dg
