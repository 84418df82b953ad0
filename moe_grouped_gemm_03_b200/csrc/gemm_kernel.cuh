// Persistent, warp-specialised FP8 NT GEMM with fine-grained scaling for sm_100a.
//
//   D[m][n] = bf16( sum_kb sfa(m,kb) * sfb(g, n/128, kb) * sum_{k in kb} A[m][k] * B_g[n][k] )
//
// ("FP8 GEMM kernels with fine-grained scaling", DeepGEMM-for-PPU README: "Interfaces" for the three
// call shapes, "Optimizations" for persistent warp specialisation and the unified block scheduler.)
//
// One CTA per SM, 256 threads:
//   warp 0      TMA producer: A tile [128 x 128 B] and B tile [BN x 128 B] per 128-K block into a
//               STAGES-deep shared-memory ring (128-byte swizzle).
//   warp 1      TMEM owner and MMA issuer (one thread): per 128-K block, copies the block's scale factors
//               shared -> TMEM (tcgen05.cp) and issues four tcgen05.mma kind::mxf8f6f4 (K = 32 each) into
//               one of two TMEM accumulators (128 lanes x BN fp32 columns).
//   warp 2      scale-factor packer: turns the fp32 power-of-two scales of the block into UE8M0 bytes
//               (the fp32 exponent field) laid out the way tcgen05.cp / the block-scaled MMA read them.
//               The 128-K scale is repeated in the four byte slots of each 32-bit word, i.e. once per
//               32-wide K sub-block, so the MMA's per-32 scaling applies the 1x128 / 128x128 recipe
//               exactly and the per-K-block promotion happens inside the tensor core.
//   warps 4..7  epilogue: TMEM -> registers -> bf16 (RNE) -> global, only for rows the GEMM owns, while
//               the MMA warp already fills the other accumulator with the next tile.
//
// Tile scheduler (all roles walk the same sequence): tiles are 128-row M blocks x BN-column N blocks,
// N fastest, handed round-robin to the persistent CTAs.
//   dense       ceil(M/128) M blocks.
//   contiguous  M_total/128 M blocks; the group of a block is m_indices[first row]; -1 skips the block.
//   masked      per group ceil(masked_m[g]/128) M blocks, counted on the device (prefix in shared memory),
//               so the host never needs masked_m.
//
// Every mbarrier wait is bounded: after WAIT_LIMIT_NS the waiting thread raises a CTA-wide abort flag and
// records ERR_TIMEOUT in the device error word; all roles then leave their loops, the MMA warp waits (again
// bounded) for its tensor-core work to drain, and TMEM is freed before the CTA exits.
#pragma once
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace dg {

enum : int { MODE_DENSE = 0, MODE_CONTIGUOUS = 1, MODE_MASKED = 2 };

constexpr int BLOCK_M = 128;
constexpr int BLOCK_K = 128;  // = the scale block along K
constexpr int MMA_K = 32;     // K of one kind::mxf8f6f4 MMA
constexpr int NUM_THREADS = 256;
constexpr int MAX_MASKED_GROUPS = 1024;
constexpr int SFB_KB_REGS = 4;  // K blocks of SFB held per lane: K <= 32 * 4 * 128 = 16384 on the fast path
constexpr int TMEM_COLS = 512;
constexpr uint64_t WAIT_LIMIT_NS = 2000000000ull;  // 2 s for any single wait
constexpr int SMEM_LIMIT = 232448;                  // 227 KB of dynamic shared memory per CTA

// device error word codes
constexpr unsigned ERR_TIMEOUT = 1u;
constexpr unsigned ERR_BAD_GROUP = 2u;

struct GemmParams {
    int mode;
    int M;             // dense: M; contiguous: M_total; masked: M_max
    int N, K, G;
    int num_m_blocks;  // dense / contiguous: total; masked: per group (ceil(M_max/128))
    int num_n_blocks;
    int sfa_ld;        // sfa floats per K block (the MN-major row extent)
    const float *sfa;
    const float *sfb;
    __nv_bfloat16 *d;
    const int *m_indices;
    const int *masked_m;
    unsigned *err;
};

template <int BN_, int STAGES_>
struct Cfg {
    static constexpr int BN = BN_;
    static constexpr int STAGES = STAGES_;
    static constexpr int SFB_ATOMS = (BN + 127) / 128;            // 128-row scale atoms covering BN rows
    static constexpr int A_BYTES = BLOCK_M * BLOCK_K;             // e4m3: 1 byte per element
    static constexpr int B_BYTES = BN * BLOCK_K;
    static constexpr int SF_WORDS = 128 + 128 * SFB_ATOMS;        // 32-bit words per stage (SFA, then SFB)
    static constexpr int SFA_RAW_BYTES = BLOCK_M * 4;             // fp32 SFA slice of a stage, by TMA
    static constexpr int SF_COLS = 4 + 4 * SFB_ATOMS;             // TMEM columns per stage's scales
    static constexpr int SF_TMEM_BASE = 2 * BN;                   // after the two accumulators
    static constexpr int NUM_BARRIERS = 3 * STAGES + 5;
    static constexpr int OFF_A = 0;
    static constexpr int OFF_B = OFF_A + STAGES * A_BYTES;
    static constexpr int OFF_SF = OFF_B + STAGES * B_BYTES;
    static constexpr int OFF_SFA_RAW = OFF_SF + STAGES * SF_WORDS * 4;
    static constexpr int OFF_BAR = OFF_SFA_RAW + STAGES * SFA_RAW_BYTES;
    static constexpr int OFF_MISC = OFF_BAR + NUM_BARRIERS * 8;   // tmem base, abort flag
    static constexpr int OFF_PREFIX = OFF_MISC + 16;               // masked: int[G+1] block prefix
    static constexpr int OFF_MM = OFF_PREFIX + 4 * (MAX_MASKED_GROUPS + 1);  // masked: clamped masked_m
    static constexpr int SMEM_BYTES = OFF_MM + 4 * MAX_MASKED_GROUPS + 1024;  // + alignment slack
    static_assert(BN % 32 == 0 && BN >= 32 && BN <= 256, "BN must be a multiple of 32 in [32, 256]");
    static_assert(SF_TMEM_BASE + STAGES * SF_COLS <= TMEM_COLS, "TMEM budget");
    static_assert(SMEM_BYTES <= SMEM_LIMIT, "shared memory budget");
    static_assert(A_BYTES % 1024 == 0 && B_BYTES % 1024 == 0, "swizzle atoms need 1024-byte alignment");
};

struct Tile {
    int row0;        // first row in A / D (flattened [rows, K] / [rows, N])
    int local_row0;  // first row inside its group (masked) or = row0
    int n0;
    int g;
};

struct SharedCtl {
    volatile int *abort;
    const int *prefix;
    const int *mm;
};

__device__ __forceinline__ void raise_error(unsigned *err, unsigned code) { atomicCAS(err, 0u, code); }

// Slow path of the bounded mbarrier wait.  false = gave up (this CTA is aborting).
__device__ __noinline__ bool wait_bounded_slow(uint64_t *bar, uint32_t parity, volatile int *abort, unsigned *err) {
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 15u) == 0) {
            if (*abort) return false;
            if (global_timer_ns() - t0 > WAIT_LIMIT_NS) {
                *abort = 1;
                raise_error(err, ERR_TIMEOUT);
                return false;
            }
        }
    }
}

__device__ __forceinline__ bool wait_bounded(uint64_t *bar, uint32_t parity, volatile int *abort, unsigned *err) {
    if (mbar_try_wait(bar, parity)) return true;
    return wait_bounded_slow(bar, parity, abort, err);
}

// Whole-warp wait: lane 0 waits, the verdict is broadcast, and the warp leaves converged (the callers
// follow with .sync.aligned tcgen05 instructions or shared-memory writes guarded by the barrier).
__device__ __forceinline__ bool warp_wait_bounded(uint64_t *bar, uint32_t parity, volatile int *abort,
                                                  unsigned *err, int lane) {
    int ok = 1;
    if (lane == 0) ok = wait_bounded(bar, parity, abort, err) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

template <int BN>
__device__ __forceinline__ bool decode_tile(const GemmParams &p, const SharedCtl &ctl, int t, Tile &ti) {
    const int mb_lin = t / p.num_n_blocks;
    const int nb = t - mb_lin * p.num_n_blocks;
    ti.n0 = nb * BN;
    if (p.mode == MODE_DENSE) {
        ti.g = 0;
        ti.row0 = ti.local_row0 = mb_lin * BLOCK_M;
        return true;
    }
    if (p.mode == MODE_CONTIGUOUS) {
        ti.row0 = ti.local_row0 = mb_lin * BLOCK_M;
        const int g = __ldg(p.m_indices + ti.row0);
        if (g < 0) return false;
        if (g >= p.G) {
            raise_error(p.err, ERR_BAD_GROUP);
            return false;
        }
        ti.g = g;
        return true;
    }
    // masked: largest g with prefix[g] <= mb_lin (prefix[G] > mb_lin by construction)
    int lo = 0, hi = p.G;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (ctl.prefix[mid] <= mb_lin) lo = mid; else hi = mid;
    }
    ti.g = lo;
    ti.local_row0 = (mb_lin - ctl.prefix[lo]) * BLOCK_M;
    ti.row0 = lo * p.M + ti.local_row0;
    return true;
}

__device__ __forceinline__ uint32_t ue8m0_x4(float s) {
    // the biased exponent of a power-of-two fp32 is its UE8M0 code; repeat it in all four byte slots
    return ((__float_as_uint(s) >> 23) & 0xFFu) * 0x01010101u;
}

template <class C>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    fp8_gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                    const __grid_constant__ CUtensorMap tmap_sfa, const GemmParams p) {
    constexpr int BN = C::BN;
    constexpr int STAGES = C::STAGES;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *sA = smem + C::OFF_A;
    uint8_t *sB = smem + C::OFF_B;
    uint32_t *sSF = reinterpret_cast<uint32_t *>(smem + C::OFF_SF);
    float *sSFA_raw = reinterpret_cast<float *>(smem + C::OFF_SFA_RAW);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
    uint64_t *full_tma = bars;
    uint64_t *full_sf = bars + STAGES;
    uint64_t *empty = bars + 2 * STAGES;
    uint64_t *tmem_full = bars + 3 * STAGES;   // [2]
    uint64_t *tmem_empty = tmem_full + 2;      // [2]
    uint64_t *drain = tmem_empty + 2;          // [1]
    uint32_t *s_tmem_base = reinterpret_cast<uint32_t *>(smem + C::OFF_MISC);
    volatile int *s_abort = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
    int *s_prefix = reinterpret_cast<int *>(smem + C::OFF_PREFIX);
    int *s_mm = reinterpret_cast<int *>(smem + C::OFF_MM);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full_tma[s], 1);
            mbar_init(&full_sf[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(&tmem_full[i], 1);
            mbar_init(&tmem_empty[i], 4);  // one arrival per epilogue warp
        }
        mbar_init(drain, 1);
        *s_abort = 0;
        mbar_init_fence();
        fence_proxy_async_smem();
        tma_prefetch_desc(&tmap_a);
        tma_prefetch_desc(&tmap_b);
        tma_prefetch_desc(&tmap_sfa);
    }
    if (warp == 1) {
        tmem_alloc(s_tmem_base, TMEM_COLS);
        tmem_relinquish();
    }
    if (warp == 2 && p.mode == MODE_MASKED) {
        // per-group M-block counts and their exclusive prefix; lane l owns groups [l*chunk, (l+1)*chunk)
        const int chunk = (p.G + 31) / 32;
        const int g_begin = min(lane * chunk, p.G), g_end = min(g_begin + chunk, p.G);
        int local = 0;
        for (int g = g_begin; g < g_end; ++g) {
            int m = __ldg(p.masked_m + g);
            if (m < 0 || m > p.M) {
                raise_error(p.err, ERR_BAD_GROUP);
                m = m < 0 ? 0 : p.M;
            }
            s_mm[g] = m;
            local += (m + BLOCK_M - 1) / BLOCK_M;
        }
        int incl = local;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += v;
        }
        int run = incl - local;
        for (int g = g_begin; g < g_end; ++g) {
            s_prefix[g] = run;
            run += (s_mm[g] + BLOCK_M - 1) / BLOCK_M;
        }
        if (lane == 31) s_prefix[p.G] = incl;
    }
    tc_fence_before_sync();
    __syncthreads();
    tc_fence_after_sync();
    const uint32_t tmem_base = *s_tmem_base;

    const SharedCtl ctl{s_abort, s_prefix, s_mm};
    const int nkb = p.K / BLOCK_K;
    const int total_tiles = (p.mode == MODE_MASKED ? s_prefix[p.G] : p.num_m_blocks) * p.num_n_blocks;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            uint32_t armed = 0, armed_ph = 0;  // stages armed at least once / parity of their last arming
            bool ok = true;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
                Tile ti;
                if (!decode_tile<BN>(p, ctl, t, ti)) continue;
                const int brow = ti.g * p.N + ti.n0;
                const int sfa_row = p.mode == MODE_MASKED ? ti.g * nkb : 0;
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!wait_bounded(&empty[s], ph ^ 1u, s_abort, p.err)) { ok = false; break; }
                    mbar_arrive_expect_tx(&full_tma[s], C::A_BYTES + C::B_BYTES + C::SFA_RAW_BYTES);
                    tma_load_2d(sA + s * C::A_BYTES, &tmap_a, &full_tma[s], kb * BLOCK_K, ti.row0);
                    tma_load_2d(sB + s * C::B_BYTES, &tmap_b, &full_tma[s], kb * BLOCK_K, brow);
                    tma_load_2d(sSFA_raw + s * BLOCK_M, &tmap_sfa, &full_tma[s], ti.local_row0, sfa_row + kb);
                    armed |= 1u << s;
                    armed_ph = (armed_ph & ~(1u << s)) | (ph << s);
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                }
            }
            if (!ok) {
                // let every load still in flight land before the CTA's shared memory goes away
                for (int i = 0; i < STAGES; ++i) {
                    if (!(armed >> i & 1u)) continue;
                    const uint64_t t0 = global_timer_ns();
                    while (!mbar_try_wait(&full_tma[i], (armed_ph >> i) & 1u) &&
                           global_timer_ns() - t0 < WAIT_LIMIT_NS) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t IDESC = idesc_mxf8_e4m3(BLOCK_M, BN);
            int s = 0;
            uint32_t ph = 0;
            int acc = 0;
            uint32_t acc_ph = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
                Tile ti;
                if (!decode_tile<BN>(p, ctl, t, ti)) continue;
                if (!wait_bounded(&tmem_empty[acc], acc_ph ^ 1u, s_abort, p.err)) break;
                tc_fence_after_sync();
                const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
                for (int kb = 0; kb < nkb; ++kb) {
                    if (!wait_bounded(&full_tma[s], ph, s_abort, p.err) ||
                        !wait_bounded(&full_sf[s], ph, s_abort, p.err)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after_sync();
                    const uint32_t sf_tmem = tmem_base + static_cast<uint32_t>(C::SF_TMEM_BASE + s * C::SF_COLS);
                    const uint32_t sf_smem = smem_u32(sSF + s * C::SF_WORDS);
                    tc_cp_32x128b_warpx4(sf_tmem, sdesc_rows16_noswizzle(sf_smem));
#pragma unroll
                    for (int a = 0; a < C::SFB_ATOMS; ++a)
                        tc_cp_32x128b_warpx4(sf_tmem + 4 + 4 * a, sdesc_rows16_noswizzle(sf_smem + 512 + 512 * a));
                    const uint32_t a_base = smem_u32(sA + s * C::A_BYTES);
                    const uint32_t b_base = smem_u32(sB + s * C::B_BYTES);
#pragma unroll
                    for (int k = 0; k < BLOCK_K / MMA_K; ++k) {
                        tc_mma_mxf8(d_tmem, sdesc_kmajor_sw128(a_base + k * MMA_K), sdesc_kmajor_sw128(b_base + k * MMA_K),
                                    IDESC, sf_tmem, sf_tmem + 4, (kb | k) != 0);
                    }
                    tc_commit(&empty[s]);
                    if (++s == STAGES) { s = 0; ph ^= 1u; }
                }
                if (!ok) break;
                tc_commit(&tmem_full[acc]);
                acc ^= 1;
                if (acc == 0) acc_ph ^= 1u;
            }
            // all tensor-core work of this CTA must be complete before TMEM is released
            tc_commit(drain);
            const uint64_t t0 = global_timer_ns();
            while (!mbar_try_wait(drain, 0) && global_timer_ns() - t0 < WAIT_LIMIT_NS) {
            }
        }
    } else if (warp == 2) {
        // ---------------------------------------------------------------- scale-factor packer
        // SFA arrives with the stage (fp32 slice by TMA).  SFB: the tile's <= 3 scale rows x K blocks are
        // held in registers (lane l holds K blocks l, l+32, ...), loaded one tile ahead so the global
        // latency hides behind the current tile.
        int s = 0;
        uint32_t ph = 0;
        const int nnb128 = (p.N + 127) / 128;
        const bool sfb_in_regs = nkb <= 32 * SFB_KB_REGS;
        float cur[3][SFB_KB_REGS], nxt[3][SFB_KB_REGS];
        auto load_sfb = [&](const Tile &ti, float (&v)[3][SFB_KB_REGS]) {
            const float *sfb_g = p.sfb + static_cast<size_t>(ti.g) * nnb128 * nkb;
            const int nb0 = ti.n0 >> 7;
#pragma unroll
            for (int j = 0; j < 3; ++j)
#pragma unroll
                for (int i = 0; i < SFB_KB_REGS; ++i) {
                    const int kb = lane + 32 * i;
                    v[j][i] = (nb0 + j < nnb128 && kb < nkb) ? __ldg(sfb_g + (nb0 + j) * nkb + kb) : 1.f;
                }
        };
        auto next_valid = [&](int &t, Tile &ti) {
            for (; t < total_tiles; t += gridDim.x)
                if (decode_tile<BN>(p, ctl, t, ti)) return true;
            return false;
        };
        int t = blockIdx.x;
        Tile ti;
        bool have = next_valid(t, ti);
        if (have && sfb_in_regs) load_sfb(ti, cur);
        bool ok = true;
        while (have && ok) {
            int t2 = t + gridDim.x;
            Tile tn;
            const bool have2 = next_valid(t2, tn);
            if (have2 && sfb_in_regs) load_sfb(tn, nxt);
            const float *sfb_g = p.sfb + static_cast<size_t>(ti.g) * nnb128 * nkb;
            const int nb0 = ti.n0 >> 7;
            for (int kb = 0; kb < nkb; ++kb) {
                float sb[3];
                if (sfb_in_regs) {
                    const int reg = kb >> 5, src = kb & 31;
#pragma unroll
                    for (int j = 0; j < 3; ++j) {
                        float x = cur[j][0];
#pragma unroll
                        for (int i = 1; i < SFB_KB_REGS; ++i) x = reg == i ? cur[j][i] : x;
                        sb[j] = __shfl_sync(0xffffffffu, x, src);
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 3; ++j)
                        sb[j] = nb0 + j < nnb128 ? __ldg(sfb_g + (nb0 + j) * nkb + kb) : 1.f;
                }
                if (!warp_wait_bounded(&full_tma[s], ph, s_abort, p.err, lane)) { ok = false; break; }
                const float4 va = reinterpret_cast<const float4 *>(sSFA_raw + s * BLOCK_M)[lane];
                uint32_t *w = sSF + s * C::SF_WORDS;
                // tcgen05.cp 32x128b source: word (r % 32) * 4 + r / 32 holds row r of a 128-row atom
                const int r0 = 4 * lane;
                w[((r0 + 0) & 31) * 4 + ((r0 + 0) >> 5)] = ue8m0_x4(va.x);
                w[((r0 + 1) & 31) * 4 + ((r0 + 1) >> 5)] = ue8m0_x4(va.y);
                w[((r0 + 2) & 31) * 4 + ((r0 + 2) >> 5)] = ue8m0_x4(va.z);
                w[((r0 + 3) & 31) * 4 + ((r0 + 3) >> 5)] = ue8m0_x4(va.w);
#pragma unroll
                for (int j = 0; j < C::SFB_ATOMS * 4; ++j) {
                    const int r = lane + 32 * j;                        // row inside the BN tile
                    const int which = ((ti.n0 + r) >> 7) - nb0;         // 0, 1 or 2
                    const float v = which == 0 ? sb[0] : (which == 1 ? sb[1] : sb[2]);
                    w[128 + (r >> 7) * 128 + (r & 31) * 4 + ((r >> 5) & 3)] = ue8m0_x4(v);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&full_sf[s]);
                if (++s == STAGES) { s = 0; ph ^= 1u; }
            }
            if (sfb_in_regs) {
#pragma unroll
                for (int j = 0; j < 3; ++j)
#pragma unroll
                    for (int i = 0; i < SFB_KB_REGS; ++i) cur[j][i] = nxt[j][i];
            }
            ti = tn;
            t = t2;
            have = have2;
        }
    } else if (warp >= 4) {
        // ---------------------------------------------------------------- epilogue
        const int q = warp & 3;  // TMEM lane quarter this warp may access
        int acc = 0;
        uint32_t acc_ph = 0;
        for (int t = blockIdx.x; t < total_tiles; t += gridDim.x) {
            Tile ti;
            if (!decode_tile<BN>(p, ctl, t, ti)) continue;
            if (!warp_wait_bounded(&tmem_full[acc], acc_ph, s_abort, p.err, lane)) break;
            tc_fence_after_sync();
            const int r_local = 32 * q + lane;
            const int row = ti.row0 + r_local;
            bool valid;
            if (p.mode == MODE_DENSE)
                valid = row < p.M;
            else if (p.mode == MODE_CONTIGUOUS)
                valid = __ldg(p.m_indices + row) >= 0;
            else
                valid = ti.local_row0 + r_local < ctl.mm[ti.g];
            __nv_bfloat16 *out = p.d + static_cast<size_t>(row) * p.N + ti.n0;
            const uint32_t t_row = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + static_cast<uint32_t>(acc * BN);
#pragma unroll 1
            for (int c = 0; c < BN / 32; ++c) {
                uint32_t r[32];
                tmem_ld_32x32b_x32(t_row + 32 * c, r);
                tmem_ld_wait_regs(r);
                if (valid) {
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int col = ti.n0 + 32 * c + 8 * j;
                        if (col < p.N) {
                            uint4 v;
                            __nv_bfloat162 h0 = __floats2bfloat162_rn(__uint_as_float(r[8 * j + 0]), __uint_as_float(r[8 * j + 1]));
                            __nv_bfloat162 h1 = __floats2bfloat162_rn(__uint_as_float(r[8 * j + 2]), __uint_as_float(r[8 * j + 3]));
                            __nv_bfloat162 h2 = __floats2bfloat162_rn(__uint_as_float(r[8 * j + 4]), __uint_as_float(r[8 * j + 5]));
                            __nv_bfloat162 h3 = __floats2bfloat162_rn(__uint_as_float(r[8 * j + 6]), __uint_as_float(r[8 * j + 7]));
                            v.x = *reinterpret_cast<uint32_t *>(&h0);
                            v.y = *reinterpret_cast<uint32_t *>(&h1);
                            v.z = *reinterpret_cast<uint32_t *>(&h2);
                            v.w = *reinterpret_cast<uint32_t *>(&h3);
                            *reinterpret_cast<uint4 *>(out + 32 * c + 8 * j) = v;
                        }
                    }
                }
            }
            tc_fence_before_sync();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tmem_empty[acc]);
            acc ^= 1;
            if (acc == 0) acc_ph ^= 1u;
        }
    }

    tc_fence_before_sync();
    __syncthreads();
    if (warp == 1) {
        __syncwarp();
        tc_fence_after_sync();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

}  // namespace dg
