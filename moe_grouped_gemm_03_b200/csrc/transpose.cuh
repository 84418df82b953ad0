// Byte transpose of B from the NN orientation [G][K][N] (N contiguous) to the K-major [G][N][K] the GEMM's
// operand loads take.  HBM-bound: every byte is read once and written once, both as 16-byte accesses that
// cover 128 contiguous bytes per row of a 128 x 128 tile; the tile turns around in shared memory.
#pragma once
#include <cstdint>

namespace dg {

constexpr int TRANSPOSE_TILE = 128;     // tile edge (bytes = e4m3 elements)
constexpr int TRANSPOSE_THREADS = 256;

// Requirements (checked by the host): K % 128 == 0, N % 16 == 0, 16-byte aligned src and dst.  A tile past N
// reads nothing there and writes nothing there.
//
// Shared-memory layout: tile row k (128 bytes = eight 16-byte vectors along n) keeps vector j at slot
// j ^ ((k / 16) % 8).  The load phase stores whole 16-byte vectors (a warp covers four rows: conflict-free);
// in the write phase lane l of warp c reads word 4c + l / 8 (four n columns) of the sixteen rows
// 16 (l % 8) .. +15, and the XOR spreads the eight row groups over all 32 banks (conflict-free), then turns
// that 16 x 4 byte block around in registers (byte permutes) into four 16-byte runs along k, one per n column.
// Eight lanes together write 128 contiguous bytes of one output row.
__device__ __forceinline__ void transpose4x4_bytes(uint32_t a, uint32_t b, uint32_t c, uint32_t d, uint32_t &o0,
                                                   uint32_t &o1, uint32_t &o2, uint32_t &o3) {
    const uint32_t ab_lo = __byte_perm(a, b, 0x5140);  // a0 b0 a1 b1
    const uint32_t ab_hi = __byte_perm(a, b, 0x7362);  // a2 b2 a3 b3
    const uint32_t cd_lo = __byte_perm(c, d, 0x5140);  // c0 d0 c1 d1
    const uint32_t cd_hi = __byte_perm(c, d, 0x7362);  // c2 d2 c3 d3
    o0 = __byte_perm(ab_lo, cd_lo, 0x5410);            // a0 b0 c0 d0
    o1 = __byte_perm(ab_lo, cd_lo, 0x7632);            // a1 b1 c1 d1
    o2 = __byte_perm(ab_hi, cd_hi, 0x5410);            // a2 b2 c2 d2
    o3 = __byte_perm(ab_hi, cd_hi, 0x7632);            // a3 b3 c3 d3
}

__global__ void __launch_bounds__(TRANSPOSE_THREADS) transpose_kn_to_nk_kernel(const uint8_t *__restrict__ src,
                                                                                uint8_t *__restrict__ dst, int G,
                                                                                int K, int N) {
    constexpr int T = TRANSPOSE_TILE;
    constexpr int VECS = T / 16;  // 16-byte vectors per tile row
    static_assert(T == 128 && TRANSPOSE_THREADS == 256, "one 16 x 4 byte block per thread in the write phase");
    __shared__ __align__(16) uint4 tile[T][VECS];
    const int tiles_n = (N + T - 1) / T, tiles_k = K / T;
    const long long total = static_cast<long long>(G) * tiles_k * tiles_n;
    // This thread's four 16-byte vectors of a tile: vector i = threadIdx.x + r * THREADS, row i / VECS, column
    // 16 * (i % VECS).  The next tile's loads are issued before the current tile is written out, so every
    // thread keeps reads in flight while it stores.
    constexpr int PER_THREAD = T * VECS / TRANSPOSE_THREADS;
    static_assert(T * VECS % TRANSPOSE_THREADS == 0, "whole vectors per thread");
    uint4 x[PER_THREAD];
    auto load_tile = [&](long long t) {
        const int tn = static_cast<int>(t % tiles_n);
        const long long rest = t / tiles_n;
        const int tk = static_cast<int>(rest % tiles_k);
        const int g = static_cast<int>(rest / tiles_k);
        const int n0 = tn * T, k0 = tk * T;
        const uint8_t *s = src + (static_cast<size_t>(g) * K + k0) * N + n0;
#pragma unroll
        for (int r = 0; r < PER_THREAD; ++r) {
            const int i = threadIdx.x + r * TRANSPOSE_THREADS;
            const int row = i / VECS, v = i % VECS;  // row = k offset, v = 16-byte vector along n
            x[r] = make_uint4(0u, 0u, 0u, 0u);
            if (n0 + 16 * v < N) x[r] = *reinterpret_cast<const uint4 *>(s + static_cast<size_t>(row) * N + 16 * v);
        }
    };
    const int lane = threadIdx.x & 31;
    const int kb = lane & 7;                              // this thread's 16 rows: 16 kb .. 16 kb + 15
    const int word = 4 * (threadIdx.x >> 5) + (lane >> 3);  // its four n columns: 4 word .. 4 word + 3
    const int slot = (word >> 2) ^ kb;                    // the vector holding that word in all 16 rows
    const uint32_t *t32 = reinterpret_cast<const uint32_t *>(&tile[0][0]);
    long long t = blockIdx.x;
    if (t < total) load_tile(t);
    for (; t < total; t += gridDim.x) {
        const int tn = static_cast<int>(t % tiles_n);
        const long long rest = t / tiles_n;
        const int tk = static_cast<int>(rest % tiles_k);
        const int g = static_cast<int>(rest / tiles_k);
        const int n0 = tn * T, k0 = tk * T;
#pragma unroll
        for (int r = 0; r < PER_THREAD; ++r) {
            const int i = threadIdx.x + r * TRANSPOSE_THREADS;
            const int row = i / VECS;
            tile[row][(i % VECS) ^ ((row >> 4) & 7)] = x[r];
        }
        __syncthreads();
        if (t + gridDim.x < total) load_tile(t + gridDim.x);
        uint32_t w[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) w[r] = t32[(16 * kb + r) * (T / 4) + 4 * slot + (word & 3)];
        uint32_t o[4][4];  // o[j][q]: n column 4 word + j, k bytes 16 kb + 4q .. +3
#pragma unroll
        for (int q = 0; q < 4; ++q)
            transpose4x4_bytes(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3], o[0][q], o[1][q], o[2][q], o[3][q]);
        uint8_t *d = dst + (static_cast<size_t>(g) * N + n0) * K + k0;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int n = 4 * word + j;
            if (n0 + n < N)
                *reinterpret_cast<uint4 *>(d + static_cast<size_t>(n) * K + 16 * kb) =
                    make_uint4(o[j][0], o[j][1], o[j][2], o[j][3]);
        }
        __syncthreads();
    }
}

}  // namespace dg
