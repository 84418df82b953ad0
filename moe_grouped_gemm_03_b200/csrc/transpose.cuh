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
__global__ void __launch_bounds__(TRANSPOSE_THREADS) transpose_kn_to_nk_kernel(const uint8_t *__restrict__ src,
                                                                                uint8_t *__restrict__ dst, int G,
                                                                                int K, int N) {
    constexpr int T = TRANSPOSE_TILE;
    constexpr int VECS = T / 16;  // 16-byte vectors per tile row
    // rows padded by 4 bytes so the column reads of the write phase spread over the banks
    __shared__ __align__(16) uint8_t tile[T][T + 4];
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
            uint32_t *t32 = reinterpret_cast<uint32_t *>(&tile[i / VECS][16 * (i % VECS)]);  // 4-byte aligned
            t32[0] = x[r].x;
            t32[1] = x[r].y;
            t32[2] = x[r].z;
            t32[3] = x[r].w;
        }
        __syncthreads();
        if (t + gridDim.x < total) load_tile(t + gridDim.x);
        uint8_t *d = dst + (static_cast<size_t>(g) * N + n0) * K + k0;
        for (int i = threadIdx.x; i < T * VECS; i += TRANSPOSE_THREADS) {
            const int n = i / VECS, v = i % VECS;  // n = output row (n offset), v = 16-byte vector along k
            if (n0 + n >= N) continue;
            uint32_t w[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t y = 0;
#pragma unroll
                for (int b = 0; b < 4; ++b) y |= static_cast<uint32_t>(tile[16 * v + 4 * q + b][n]) << (8 * b);
                w[q] = y;
            }
            *reinterpret_cast<uint4 *>(d + static_cast<size_t>(n) * K + 16 * v) = make_uint4(w[0], w[1], w[2], w[3]);
        }
        __syncthreads();
    }
}

}  // namespace dg
