// Host side of the C ABI declared in include/dg.h: argument validation, tile-shape choice, TMA
// descriptors and the launch of the persistent sm_100a kernel on the caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <cstdlib>
#include <mutex>
#include <string>

#include "dg.h"
#include "gemm_kernel.cuh"
#include "scale_pack.cuh"
#include "transpose.cuh"

namespace {

thread_local std::string g_last_error;
std::atomic<int> g_num_sms_cap{0};  // 0: every SM of the device

__device__ unsigned g_device_error_word;  // first device-side error code since the last check
// measurement aid (dg_debug_clock_record): SM cycles, nanoseconds and launches summed over recorded launches
__device__ unsigned long long g_clock_acc[3];

int fail(int code, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char *what) {
    return fail(DG_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

struct DeviceInfo {
    int device = -1;
    int num_sms = 0;
    int major = 0, minor = 0;
};

int device_info(DeviceInfo &info) {
    cudaError_t e = cudaGetDevice(&info.device);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    // the attributes of a device do not change: queried once per device
    static DeviceInfo cache[64];
    if (info.device >= 0 && info.device < 64 && cache[info.device].device == info.device) {
        info = cache[info.device];
        return DG_OK;
    }
    if ((e = cudaDeviceGetAttribute(&info.num_sms, cudaDevAttrMultiProcessorCount, info.device)) != cudaSuccess)
        return cuda_fail(e, "cudaDeviceGetAttribute(SM count)");
    if ((e = cudaDeviceGetAttribute(&info.major, cudaDevAttrComputeCapabilityMajor, info.device)) != cudaSuccess)
        return cuda_fail(e, "cudaDeviceGetAttribute(major)");
    if ((e = cudaDeviceGetAttribute(&info.minor, cudaDevAttrComputeCapabilityMinor, info.device)) != cudaSuccess)
        return cuda_fail(e, "cudaDeviceGetAttribute(minor)");
    if (info.major != 10 || info.minor != 0)
        return fail(DG_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a only", info.device,
                    info.major, info.minor);
    if (info.device >= 0 && info.device < 64) cache[info.device] = info;
    return DG_OK;
}

int effective_sms(const DeviceInfo &info) {
    const int cap = g_num_sms_cap.load(std::memory_order_relaxed);
    return (cap > 0 && cap < info.num_sms) ? cap : info.num_sms;
}

// ----------------------------------------------------------------------------------------------- TMA
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

int get_encode_fn(EncodeTiledFn &fn) {
    static EncodeTiledFn cached = nullptr;
    if (!cached) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !p)
            return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
        cached = reinterpret_cast<EncodeTiledFn>(p);
    }
    fn = cached;
    return DG_OK;
}

// Row-major byte matrix [rows][K] (K-major e4m3 operand), boxes of box_rows x 128 bytes, 128-byte swizzle.
// A or B, e4m3 K-major [rows][K]: boxes of one 128-K block (128 bytes) x `box_rows` rows with the 128-byte
// swizzle (one swizzle atom per 8 rows), the layout the MMA's shared-memory descriptors expect.
int make_operand_map(CUtensorMap &map, const void *base, long long rows, int K, int box_rows) {
    EncodeTiledFn encode;
    if (int rc = get_encode_fn(encode)) return rc;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(dg::BLOCK_K), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return DG_OK;
}

// B in E2M1, packed two codes per byte [rows][K/2]: the TMA's 16 x 4-bit type with 16-byte alignment stages each
// 16 codes as 8 bytes followed by an 8-byte gap, so a box of 128 codes x `box_rows` rows fills 128-byte rows,
// the footprint and 128-byte swizzle of an e4m3 box, which is how the MMA reads an E2M1 operand.  Requires a
// 32-byte aligned base and K % 64 == 0 (the row stride K/2 a multiple of 32 bytes).
int make_operand_map_fp4(CUtensorMap &map, const void *base, long long rows, int K, int box_rows) {
    EncodeTiledFn encode;
    if (int rc = get_encode_fn(encode)) return rc;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(dg::BLOCK_K), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<void *>(base), dims, strides, box,
                        estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled (E2M1) failed (%d)", static_cast<int>(r));
    return DG_OK;
}

// B in the NN orientation, e4m3 [rows = G*K][N] (N contiguous): boxes of 128 columns x 128 K-rows with the 128-byte
// swizzle, an MN-major operand tile of one 128-K block (8 K-rows per 1024-byte swizzle atom).
int make_operand_map_nn(CUtensorMap &map, const void *base, long long rows, int N) {
    EncodeTiledFn encode;
    if (int rc = get_encode_fn(encode)) return rc;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(N)};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(dg::BLOCK_M), static_cast<cuuint32_t>(dg::BLOCK_K)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void *>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled (NN operand) failed (%d)", static_cast<int>(r));
    return DG_OK;
}

// D, bf16 row-major [rows][N]: boxes of 32 rows x 32 columns (64-byte rows) with the 64-byte swizzle, the
// layout the epilogue stages each chunk in.
int make_output_map(CUtensorMap &map, void *base, long long rows, int N) {
    EncodeTiledFn encode;
    if (int rc = get_encode_fn(encode)) return rc;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(N) * 2};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled (output) failed (%d)", static_cast<int>(r));
    return DG_OK;
}

// D fp32 [G][M][N] (K-grouped calls): a 3-D map so a box never crosses from one group's M rows into the next;
// boxes of 32 rows x 16 columns (64-byte rows) with the 64-byte swizzle, like the bf16 chunks.
int make_output_map_f32(CUtensorMap &map, float *base, int G, int M, int N) {
    EncodeTiledFn encode;
    if (int rc = get_encode_fn(encode)) return rc;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M), static_cast<cuuint64_t>(G)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(N) * 4, static_cast<cuuint64_t>(M) * N * 4};
    cuuint32_t box[3] = {16, 32, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled (fp32 output) failed (%d)", static_cast<int>(r));
    return DG_OK;
}

// Packed scale atoms: rows of 128 32-bit words (512 bytes), boxes of `box_rows` atoms, no swizzle.
int make_atom_map(CUtensorMap &map, const uint32_t *base, long long atoms, int box_rows) {
    EncodeTiledFn encode;
    if (int rc = get_encode_fn(encode)) return rc;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(dg::SF_ATOM_WORDS), static_cast<cuuint64_t>(atoms)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(dg::SF_ATOM_WORDS) * 4};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(dg::SF_ATOM_WORDS), static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = encode(&map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t *>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return fail(DG_ERR_CUDA, "cuTensorMapEncodeTiled (scales) failed (%d)", static_cast<int>(r));
    return DG_OK;
}

// Stream-ordered scratch for the packed scales, from a pool this library owns (one per device) that keeps
// freed memory for reuse, so steady-state calls do not reach the driver's allocator.
int scratch_pool(int device, cudaMemPool_t &pool) {
    static std::mutex mu;
    static cudaMemPool_t pools[64] = {};
    std::lock_guard<std::mutex> lock(mu);
    if (device < 0 || device >= 64) return fail(DG_ERR_UNSUPPORTED, "device index %d out of range", device);
    if (!pools[device]) {
        cudaMemPoolProps props = {};
        props.allocType = cudaMemAllocationTypePinned;
        props.location.type = cudaMemLocationTypeDevice;
        props.location.id = device;
        cudaError_t e = cudaMemPoolCreate(&pools[device], &props);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemPoolCreate");
        uint64_t keep = ~0ull;
        cudaMemPoolSetAttribute(pools[device], cudaMemPoolAttrReleaseThreshold, &keep);
    }
    pool = pools[device];
    return DG_OK;
}

}  // namespace

// ------------------------------------------------------------------------------------------------------------
// The fixed scratch buffer of the allocation-free dense GEMM (dg_fp8_gemm_nt_noalloc)
//
// Some callers may not allocate device memory at all during a call: code that runs while a stream is being
// captured in the global capture mode (where allocation calls are refused), engines whose memory manager owns
// every byte of HBM, or real-time paths that cannot afford an allocator call. For them the packed scales go to a
// fixed buffer that exists for the lifetime of the library instead of the per-call pool allocation. All calls
// share the buffer, so calls whose work overlaps on the GPU (different streams, no ordering between them) race on
// it; calls on one stream are ordered and safe.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB of packed scale atoms
static __device__ __align__(256) uint32_t g_noalloc_scratch[kNoAllocScratchBytes / 4];

// Device address of the static buffer, looked up once per device with that device current.  In host code the
// name g_noalloc_scratch is only a host-side stand-in for the symbol, never a device address.
int noalloc_scratch(int device, uint32_t **out) {
    static std::mutex mu;
    static uint32_t *ptrs[64] = {};
    std::lock_guard<std::mutex> lock(mu);
    if (device < 0 || device >= 64) return fail(DG_ERR_UNSUPPORTED, "device index %d out of range", device);
    if (!ptrs[device]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress (static scale buffer)");
        ptrs[device] = static_cast<uint32_t *>(p);
    }
    *out = ptrs[device];
    return DG_OK;
}

}  // namespace

namespace {

// ----------------------------------------------------------------------------------------------- launch
// Process-wide settings (atomics: reading one while another thread sets it is defined, but a call sees whichever
// value was in force when it read it).
std::atomic<int> g_m_alignment{dg::BLOCK_M};  // contiguous layout: per-segment M padding (128 or 256)
std::atomic<int> g_pair_policy{-1};  // -1: library decides; 0: single CTAs only; 1: CTA pairs whenever supported
std::atomic<bool> g_fp32_promotion{false};  // true: any fp32 scales, applied by promotion; false: powers of two
std::atomic<unsigned long long> g_wait_limit_ns{dg::WAIT_LIMIT_NS};  // limit of every in-kernel wait
std::atomic<bool> g_drop_first_stage{false};  // testing aid: the next GEMM launch leaves one stage unloaded
std::atomic<bool> g_clock_record{false};      // measurement aid: launches add their clock record
std::atomic<int> g_swap_policy{-1};  // -1: library decides; 0: never swapped operands; 1: wherever supported

// Device address of a __device__ symbol of this library (given by its host-side stand-in) on the current
// device, looked up once per device with that device current.
void *symbol_address(const void *symbol, void *(&cache)[64]) {
    int device = 0;
    if (cudaGetDevice(&device) != cudaSuccess) return nullptr;
    if (device >= 0 && device < 64 && cache[device]) return cache[device];
    void *p = nullptr;
    if (cudaGetSymbolAddress(&p, symbol) != cudaSuccess) return nullptr;
    if (device >= 0 && device < 64) cache[device] = p;
    return p;
}

unsigned long long *clock_accumulator() {
    static void *cache[64] = {nullptr};
    return static_cast<unsigned long long *>(symbol_address(g_clock_acc, cache));
}

// Per-launch settings: the wait limit, the dropped stage (one launch only) and the clock record.
void apply_wait_settings(dg::GemmParams &p) {
    p.wait_limit_ns = g_wait_limit_ns.load();
    p.skip_first_load = g_drop_first_stage.exchange(false) ? 1 : 0;
    p.clock_acc = g_clock_record.load() ? clock_accumulator() : nullptr;
}

struct ScaleArgs {
    const float *sfa;
    int sfa_ld;
    const float *sfb;
    bool sfb_kn = false;  // SFB stored [G][K/128][ceil(N/128)] (B in the NN orientation)
    bool sfb_fp4 = false; // B in E2M1 (packed two per byte) with SFB [G][K/32][sfb_ld]
    bool fixed_scratch = false;  // packed scales in the library's fixed buffer (no allocation) instead of the pool
    bool single_kernel = false;  // power-of-two scales applied by the promotion GEMM (one launch, no pre-pass)
    bool swap = false;    // masked layout with swapped operands (B's rows on the MMA's M side, tokens on its N side)
    int sfb_ld = 0;       // K-grouped: one scale per row of B, [K/128][sfb_ld]; FP4 B: [G][K/32][sfb_ld]
};

// Launch of the scale pre-pass: one warp per work item (an atom, or 32 B-side atoms of the swapped-operand
// layout), spread over every SM (one block each), so that every SM is
// free for the GEMM (a programmatic dependent) at about the same time.  An SM running a pre-pass block takes no
// GEMM CTA until that block is done (the pre-pass keeps the default shared-memory carveout).
int launch_pack(const dg::PackParams &pk, int device, cudaStream_t stream) {
    // warp work items: one per atom, except the B-side atoms of one scale per 128 x 128 block of B (the swapped
    // layout's, and the others' unless K-grouped or E2M1), built 32 to a warp
    const long long sfa_atoms = pk.sfa_words / dg::SF_ATOM_WORDS, sfb_atoms = pk.sfb_words / dg::SF_ATOM_WORDS;
    const bool sfb_batched = !pk.swap && pk.mode != dg::MODE_KGROUPED && !pk.sfb_fp4;
    const long long atoms = pk.swap ? (sfa_atoms + 31) / 32 + sfb_atoms
                                    : sfa_atoms + (sfb_batched ? (sfb_atoms + 31) / 32 : sfb_atoms);
    constexpr long long kMaxWarps = dg::PACK_THREADS / 32;
    DeviceInfo info;  // (cached per device)
    const int sms = device_info(info) == DG_OK && info.device == device && info.num_sms > 0 ? info.num_sms : 1;
    long long blocks = atoms < sms ? atoms : sms;
    if (blocks < 1) blocks = 1;
    long long warps = (atoms + blocks - 1) / blocks;
    if (warps > kMaxWarps) warps = kMaxWarps;
    if (warps < 1) warps = 1;
    dg::pack_scales_kernel<<<static_cast<unsigned>(blocks), static_cast<unsigned>(32 * warps), 0, stream>>>(pk);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "scale pack launch");
    return DG_OK;
}

template <int BN, int CTAS, int KPS, bool BF4 = false, bool SWAP = false, bool BNN = false>
int launch_cfg(const void *a, long long a_rows, const void *b, long long b_rows, const ScaleArgs &sc, dg::GemmParams p,
               int grid, int device, cudaStream_t stream) {
    using C = dg::Cfg<BN, CTAS, KPS, BF4, false, SWAP, BNN>;
    // ---- packed scale atoms (pre-pass)
    const int nkb = p.K / dg::BLOCK_K;
    dg::PackParams pk{};
    pk.sfa = sc.sfa;
    pk.sfa_ld = sc.sfa_ld;
    pk.sfb = sc.sfb;
    pk.sfb_kn = sc.sfb_kn ? 1 : 0;
    pk.sfb_ld = sc.sfb_ld;
    pk.N = p.N;
    pk.G = p.G;
    pk.bn = BN;
    pk.n_tiles = p.num_n_blocks;
    pk.sfb_atoms = C::SFB_ATOMS;
    pk.nkb = nkb;
    pk.num_sf_groups = p.num_sf_groups;
    pk.sfb_kwords = p.num_sf_groups;
    if (BF4) {  // B scale words: one per 128-K block
        pk.sfb_fp4 = 1;
        pk.sfb_kwords = nkb;
    }
    pk.mode = p.mode;
    pk.counts = p.masked_m;
    pk.m_indices = p.m_indices;
    pk.err = p.err;
    pk.tile_m = C::TILE_M;
    if (p.mode == dg::MODE_MASKED) {
        pk.rows_per_group = p.M;
        pk.blocks_per_group = p.sfa_blocks;
        pk.sfa_groups = p.G;
    } else if (p.mode == dg::MODE_NOPAD) {
        // every group's windows, at most ceil(M_total / TILE_M) + G of them, CTAS blocks each
        pk.rows_per_group = p.M;
        pk.blocks_per_group = CTAS * ((p.M + C::TILE_M - 1) / C::TILE_M + p.G);
        pk.sfa_groups = 1;
    } else {  // dense, contiguous, K-grouped (the groups share A's rows)
        pk.rows_per_group = p.M;
        pk.blocks_per_group = (p.M + dg::BLOCK_M - 1) / dg::BLOCK_M;
        pk.sfa_groups = 1;
    }
    long long sfa_atoms = static_cast<long long>(pk.sfa_groups) * pk.blocks_per_group * p.num_sf_groups;
    const long long b_groups = p.mode == dg::MODE_KGROUPED ? 1 : p.G;  // K-grouped: one B for all groups
    long long sfb_atoms = b_groups * p.num_n_blocks * pk.sfb_kwords * C::SFB_ATOMS;
    if (SWAP) {  // B-side atoms per 128-row block of B, token-side atoms per chunk (all groups' chunks in order)
        pk.swap = 1;
        pk.b_blocks = p.sfa_blocks;
        pk.chunks = p.swap_chunks;
        pk.rows_per_group = p.M;
        sfa_atoms = static_cast<long long>(p.G) * p.sfa_blocks * p.num_sf_groups;
        sfb_atoms = static_cast<long long>(p.swap_chunks) * p.num_sf_groups * C::SFB_ATOMS;
    }
    pk.sfa_words = sfa_atoms * dg::SF_ATOM_WORDS;
    pk.sfb_words = sfb_atoms * dg::SF_ATOM_WORDS;
    const size_t need = static_cast<size_t>(pk.sfa_words + pk.sfb_words) * 4;
    void *scratch = nullptr;
    cudaError_t e;
    if (sc.fixed_scratch) {  // calls no allocator: every word of both regions is rewritten by the pre-pass
        if (need > kNoAllocScratchBytes)
            return fail(DG_ERR_UNSUPPORTED,
                        "the packed scales of this shape need %zu bytes; the allocation-free call has a fixed %zu-byte "
                        "buffer (use dg_fp8_gemm_nt)",
                        need, kNoAllocScratchBytes);
        uint32_t *fixed = nullptr;
        if (int rc = noalloc_scratch(device, &fixed)) return rc;
        scratch = fixed;
    } else {
        cudaMemPool_t pool;
        if (int rc = scratch_pool(device, pool)) return rc;
        if ((e = cudaMallocFromPoolAsync(&scratch, need, pool, stream)) != cudaSuccess)
            return cuda_fail(e, "cudaMallocFromPoolAsync (packed scales)");
    }
    pk.sfa_out = static_cast<uint32_t *>(scratch);
    pk.sfb_out = pk.sfa_out + pk.sfa_words;
    int rc = DG_OK;
    do {
        // ---- tensor maps (all host work is done before the two launches, so they reach the GPU back to back)
        CUtensorMap ta, tb, tsfa, tsfb, td;
        if (p.out_mode == dg::OUT_BF16)
            rc = make_output_map(td, p.d, a_rows, p.N);
        else
            rc = make_output_map_f32(td, p.d32, p.G, p.M, p.N);
        if (rc) break;
        // (swapped operands: the 128-row boxes of the MMA's M side come from B, the N side's from A)
        if (BNN)  // (b_rows = G * K rows of N bytes)
            rc = make_operand_map_nn(ta, b, b_rows, p.N);
        else
            rc = make_operand_map(ta, SWAP ? b : a, SWAP ? b_rows : a_rows, p.K, dg::BLOCK_M);
        if (rc) break;
        if (BF4)
            rc = make_operand_map_fp4(tb, b, b_rows, p.K, C::B_ROWS);
        else
            rc = make_operand_map(tb, SWAP ? a : b, SWAP ? a_rows : b_rows, p.K, C::B_ROWS);
        if (rc) break;
        if ((rc = make_atom_map(tsfa, pk.sfa_out, sfa_atoms, 1))) break;
        if ((rc = make_atom_map(tsfb, pk.sfb_out, sfb_atoms, C::SFB_KB * C::SFB_ATOMS))) break;
        // ---- the GEMM, as a programmatic dependent of the pre-pass
        auto kernel = dg::fp8_gemm_kernel<C>;
        static bool smem_set[64] = {false};  // per instantiation and device: the attribute persists
        if (!(device >= 0 && device < 64 && smem_set[device])) {
            if ((e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES)) !=
                cudaSuccess) {
                rc = cuda_fail(e, "cudaFuncSetAttribute");
                break;
            }
            if (device >= 0 && device < 64) smem_set[device] = true;
        }
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(grid * CTAS), 1, 1);
        cfg.blockDim = dim3(dg::NUM_THREADS, 1, 1);
        cfg.dynamicSmemBytes = C::SMEM_BYTES;
        cfg.stream = stream;
        cudaLaunchAttribute attr[2];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = CTAS;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[1].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 2;
        if (CTAS > 1) {
            // a persistent grid larger than the co-resident clusters would only queue behind itself
            static int max_clusters[64] = {0};
            int &cached = max_clusters[device & 63];
            if (cached == 0) {
                int n = 0;
                if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n <= 0) {
                    cudaGetLastError();
                    n = grid;
                }
                cached = n;
            }
            if (grid > cached) cfg.gridDim.x = static_cast<unsigned>(cached * CTAS);
        }
        static const bool debug = getenv("DG_DEBUG") && getenv("DG_DEBUG")[0] == '1';
        if (debug)
            fprintf(stderr, "[dg] mode=%d%s M=%d N=%d K=%d G=%d BN=%d stages=%d x %d ctas=%d grid=%u smem=%d windows=%d"
                            " raster=%d scratch=%lld B\n",
                    p.mode, SWAP ? " (swapped operands)" : "", p.M, p.N, p.K, p.G, BN, C::STAGES, KPS, CTAS,
                    cfg.gridDim.x, C::SMEM_BYTES, p.num_windows, p.raster_bands, (pk.sfa_words + pk.sfb_words) * 4);
        apply_wait_settings(p);
        if ((rc = launch_pack(pk, device, stream))) break;
        if ((e = cudaLaunchKernelEx(&cfg, kernel, ta, tb, tsfa, tsfb, td, p)) != cudaSuccess) {
            rc = cuda_fail(e, "kernel launch");
            break;
        }
    } while (false);
    if (!sc.fixed_scratch) {
        const cudaError_t ef = cudaFreeAsync(scratch, stream);
        if (rc == DG_OK && ef != cudaSuccess) rc = cuda_fail(ef, "cudaFreeAsync (packed scales)");
    }
    return rc;
}

// The fp32 scale-promotion GEMM (any finite fp32 scales): plain kind::f8f6f4 MMAs, the epilogue warps read the
// caller's scales directly, so there is no pre-pass and no scratch.  e4m3 B: 128-wide tiles (one 128-column
// block of B's scales); K-grouped (per-column B scales, fp32 D): 64-wide tiles, which keep the accumulators and
// the fp32 epilogue within the registers; E2M1 B: 64-wide tiles, one partial per 32-K MMA.
// The launch is an ordinary stream-ordered one (the kernel's first loads may not run ahead of the previous
// kernel on the stream).
template <int BN, int CTAS, int KPS, bool BF4, bool PCOL = false>
int launch_promo(const void *a, long long a_rows, const void *b, long long b_rows, const ScaleArgs &sc,
                 dg::GemmParams p, int grid, int device, cudaStream_t stream) {
    using C = dg::Cfg<BN, CTAS, KPS, BF4, true, false, false, PCOL>;
    const int nkb = p.K / dg::BLOCK_K;
    const int nnb = (p.N + 127) / 128;
    p.sfa32 = sc.sfa;
    p.sfa_ld = sc.sfa_ld;
    p.sfb32 = sc.sfb;
    if (BF4) {  // [G][K/32][sfb_ld]: per column and 32-K sub-block
        p.sfb_sg = static_cast<int>(static_cast<long long>(p.K / 32) * sc.sfb_ld);
        p.sfb_sk = sc.sfb_ld;
    } else if (PCOL) {  // K-grouped, [sum ks / 128][sfb_ld]: per column and K block, one B for all groups
        p.sfb_sg = 0;
        p.sfb_sk = sc.sfb_ld;
    } else {
        p.sfb_sg = nkb * nnb;
        p.sfb_sn = sc.sfb_kn ? 1 : nkb;  // NN: [G][K/128][ceil(N/128)]; NT: [G][ceil(N/128)][K/128]
        p.sfb_sk = sc.sfb_kn ? nnb : 1;
    }
    CUtensorMap ta, tb, td;
    int rc;
    if (p.out_mode == dg::OUT_BF16)
        rc = make_output_map(td, p.d, a_rows, p.N);
    else
        rc = make_output_map_f32(td, p.d32, p.G, p.M, p.N);
    if (rc) return rc;
    if ((rc = make_operand_map(ta, a, a_rows, p.K, dg::BLOCK_M))) return rc;
    if (BF4)
        rc = make_operand_map_fp4(tb, b, b_rows, p.K, C::B_ROWS);
    else
        rc = make_operand_map(tb, b, b_rows, p.K, C::B_ROWS);
    if (rc) return rc;
    auto kernel = dg::fp8_gemm_kernel<C>;
    cudaError_t e;
    static bool smem_set[64] = {false};
    if (!(device >= 0 && device < 64 && smem_set[device])) {
        if ((e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES)) !=
            cudaSuccess)
            return cuda_fail(e, "cudaFuncSetAttribute");
        if (device >= 0 && device < 64) smem_set[device] = true;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid * CTAS), 1, 1);
    cfg.blockDim = dim3(dg::NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = C::SMEM_BYTES;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CTAS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (CTAS > 1) {
        static int max_clusters[64] = {0};
        int &cached = max_clusters[device & 63];
        if (cached == 0) {
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess || n <= 0) {
                cudaGetLastError();
                n = grid;
            }
            cached = n;
        }
        if (grid > cached) cfg.gridDim.x = static_cast<unsigned>(cached * CTAS);
    }
    static const bool debug = getenv("DG_DEBUG") && getenv("DG_DEBUG")[0] == '1';
    if (debug)
        fprintf(stderr, "[dg] fp32 promotion: mode=%d M=%d N=%d K=%d G=%d BN=%d stages=%d x %d ctas=%d grid=%u smem=%d\n",
                p.mode, p.M, p.N, p.K, p.G, BN, C::STAGES, C::KPS, CTAS, cfg.gridDim.x, C::SMEM_BYTES);
    apply_wait_settings(p);
    // the kernel takes five maps; the two scale-atom maps are unused on this path
    if ((e = cudaLaunchKernelEx(&cfg, kernel, ta, tb, ta, ta, td, p)) != cudaSuccess)
        return cuda_fail(e, "kernel launch");
    return DG_OK;
}

// Tile widths the library is built with, and the pipeline depth each fits in 227 KB of shared memory and
// 512 TMEM columns (two BN-wide accumulators plus one scale slot per stage).
constexpr int kCandidateBN[] = {224, 192, 160, 128};

template <bool BF4>
int launch_bn_t(int bn, int ctas, const void *a, long long a_rows, const void *b, long long b_rows,
                const ScaleArgs &sc, const dg::GemmParams &p, int grid, int device, cudaStream_t stream) {
    if (ctas == 2) {
        switch (bn) {
            case 224: return launch_cfg<224, 2, 2, BF4>(a, a_rows, b, b_rows, sc, p, grid, device, stream);
            case 192: return launch_cfg<192, 2, 2, BF4>(a, a_rows, b, b_rows, sc, p, grid, device, stream);
            case 160: return launch_cfg<160, 2, 2, BF4>(a, a_rows, b, b_rows, sc, p, grid, device, stream);
            case 128: return launch_cfg<128, 2, 2, BF4>(a, a_rows, b, b_rows, sc, p, grid, device, stream);
            default: break;
        }
    } else {
        switch (bn) {
            case 224: return launch_cfg<224, 1, 1, BF4>(a, a_rows, b, b_rows, sc, p, grid, device, stream);
            case 192: return launch_cfg<192, 1, 1, BF4>(a, a_rows, b, b_rows, sc, p, grid, device, stream);
            case 160: return launch_cfg<160, 1, 1, BF4>(a, a_rows, b, b_rows, sc, p, grid, device, stream);
            case 128: return launch_cfg<128, 1, 1, BF4>(a, a_rows, b, b_rows, sc, p, grid, device, stream);
            default: break;
        }
    }
    return fail(DG_ERR_UNSUPPORTED, "no kernel instantiated for BN=%d with %d CTA(s) per tile", bn, ctas);
}

// B e4m3, or (sc.sfb_fp4) B in E2M1 with 1x32 scales
int launch_bn(int bn, int ctas, const void *a, long long a_rows, const void *b, long long b_rows,
              const ScaleArgs &sc, const dg::GemmParams &p, int grid, int device, cudaStream_t stream) {
    if (sc.sfb_fp4) return launch_bn_t<true>(bn, ctas, a, a_rows, b, b_rows, sc, p, grid, device, stream);
    return launch_bn_t<false>(bn, ctas, a, a_rows, b, b_rows, sc, p, grid, device, stream);
}

// Tile width for `windows` row windows (128 rows per CTA, `ctas` CTAs per tile) of an N-wide output on
// `units` SMs or SM pairs.  The persistent kernel is bound by the operand bytes each CTA pulls per K block
// (128 A rows + BN/ctas B rows), so a pass costs about waves x (128 + BN/ctas); wider tiles win unless they
// add a wave (README "Unaligned block sizes": wave quantisation on the SM count).
int select_block_n(long long windows, int N, int units, int ctas) {
    if (units <= 0) units = 1;
    if (windows <= 0) windows = 1;
    int best = kCandidateBN[0];
    long long best_cost = -1;
    for (int bn : kCandidateBN) {
        const long long tiles = windows * ((N + bn - 1) / bn);
        const long long waves = (tiles + units - 1) / units;
        const long long cost = waves * (dg::BLOCK_M + bn / ctas);
        if (best_cost < 0 || cost < best_cost) {
            best_cost = cost;
            best = bn;
        }
    }
    return best;
}

// Tile order of the dense and K-grouped layouts: raster groups of this many row windows, swept down the windows
// first.  The CTAs running at one time then share a few B column blocks, and the group's A rows (at most about
// kRasterBytes, so they stay in the 126 MB L2 beside the B blocks in flight and the D tiles written back) serve
// every column block of the group.  On the dense 4096 x 7168 x 7168 GEMM this order measured 2.7% faster than
// sweeping the columns first, which re-streams all of B every ~2 windows.
constexpr long long kRasterBytes = 40ll << 20;
int raster_bands(const dg::GemmParams &p, int ctas) {
    const long long windows = p.mode == dg::MODE_KGROUPED ? p.num_windows / p.G : p.num_windows;
    const long long k = p.mode == dg::MODE_KGROUPED ? p.K / p.G : p.K;  // a group's mean K extent
    const long long window_bytes = static_cast<long long>(dg::BLOCK_M) * ctas * (k > 0 ? k : 1);
    long long bands = kRasterBytes / window_bytes;
    if (bands > windows) bands = windows;
    return static_cast<int>(bands < 1 ? 1 : bands);
}

// Shape and launch: picks single CTAs or CTA pairs, the tile width, and the persistent grid.
//   sel1 / sel2:     128-row / 256-row windows the tile shape is chosen for (a hint for the masked layout)
//   bound1 / bound2: the most 128-row / 256-row tiles the device may find (sizes the grid)
//   windows1/2:      the kernel's window count (dense, contiguous); unused for the masked layout
struct Plan {
    long long sel1, sel2, bound1, bound2, windows1, windows2;
    bool pair_supported;
};

int plan_and_launch(dg::GemmParams p, const DeviceInfo &info, const Plan &plan, const void *a, long long a_rows,
                    const void *b, long long b_rows, const ScaleArgs &sc, cudaStream_t stream) {
    const int sms = effective_sms(info);
    bool pair = plan.pair_supported && sms >= 2;
    const int policy = g_pair_policy.load();
    if (policy == 0) pair = false;
    if (policy < 0 && pair) {
        // pairs pay once there is at least a wave of them
        const int bn = select_block_n(plan.sel2, p.N, sms / 2, 2);
        pair = plan.sel2 * ((p.N + bn - 1) / bn) >= sms / 2;
    }
    const int units = pair ? sms / 2 : sms;
    const bool promotion = g_fp32_promotion.load();
    if (promotion || sc.single_kernel) {
        p.check_scales = promotion ? 0 : 1;
        // per-column B scales (K-grouped, E2M1 B) are copied 16 bytes at a time
        if ((sc.sfb_fp4 || p.mode == dg::MODE_KGROUPED) && !aligned(sc.sfb, 16))
            return fail(DG_ERR_ALIGNMENT, "with fp32 scale promotion, sfb must be 16-byte aligned");
        const int bn = sc.sfb_fp4 || p.mode == dg::MODE_KGROUPED ? 64 : 128;  // (per-column scales: 64 wide)
        p.num_n_blocks = (p.N + bn - 1) / bn;
        const bool device_windows = p.mode == dg::MODE_MASKED || p.mode == dg::MODE_NOPAD;
        p.num_windows = static_cast<int>(device_windows ? 0 : (pair ? plan.windows2 : plan.windows1));
        if (p.mode == dg::MODE_DENSE || p.mode == dg::MODE_KGROUPED) p.raster_bands = raster_bands(p, pair ? 2 : 1);
        const long long tiles = (pair ? plan.bound2 : plan.bound1) * p.num_n_blocks;
        const int grid = static_cast<int>(tiles < units ? tiles : units);
        if (grid <= 0) return DG_OK;
        // (a single CTA fits more stages of one K block)
        if (sc.sfb_fp4) {
            if (pair) return launch_promo<64, 2, 1, true>(a, a_rows, b, b_rows, sc, p, grid, info.device, stream);
            return launch_promo<64, 1, 1, true>(a, a_rows, b, b_rows, sc, p, grid, info.device, stream);
        }
        if (p.mode == dg::MODE_KGROUPED) {
            if (pair) return launch_promo<64, 2, 2, false, true>(a, a_rows, b, b_rows, sc, p, grid, info.device, stream);
            return launch_promo<64, 1, 1, false, true>(a, a_rows, b, b_rows, sc, p, grid, info.device, stream);
        }
        if (pair) return launch_promo<128, 2, 2, false>(a, a_rows, b, b_rows, sc, p, grid, info.device, stream);
        return launch_promo<128, 1, 1, false>(a, a_rows, b, b_rows, sc, p, grid, info.device, stream);
    }
    int bn = select_block_n(pair ? plan.sel2 : plan.sel1, p.N, units, pair ? 2 : 1);
    static const int forced_bn = getenv("DG_BLOCK_N") ? atoi(getenv("DG_BLOCK_N")) : 0;  // tuning override
    if (forced_bn > 0) bn = forced_bn;
    p.num_n_blocks = (p.N + bn - 1) / bn;
    const bool device_windows = p.mode == dg::MODE_MASKED || p.mode == dg::MODE_NOPAD;  // counted by the kernel
    p.num_windows = static_cast<int>(device_windows ? 0 : (pair ? plan.windows2 : plan.windows1));
    if (p.num_sf_groups == 0)  // (the K-grouped call counts its groups' scale groups itself)
        p.num_sf_groups = (p.K / dg::BLOCK_K + dg::SF_GROUP - 1) / dg::SF_GROUP;
    if (p.mode == dg::MODE_DENSE || p.mode == dg::MODE_KGROUPED)
        p.raster_bands = raster_bands(p, pair ? 2 : 1);
    const long long tiles = (pair ? plan.bound2 : plan.bound1) * p.num_n_blocks;
    const int grid = static_cast<int>(tiles < units ? tiles : units);
    if (grid <= 0) return DG_OK;
    return launch_bn(bn, pair ? 2 : 1, a, a_rows, b, b_rows, sc, p, grid, info.device, stream);
}

unsigned *device_error_word() {
    static void *cache[64] = {nullptr};  // the symbol's address on each device, looked up once
    return static_cast<unsigned *>(symbol_address(&g_device_error_word, cache));
}

int check_common(const void *a, const float *sfa, const void *b, const float *sfb, const void *d, long long N,
                 long long K) {
    if (!a || !sfa || !b || !sfb || !d) return fail(DG_ERR_INVALID_ARG, "null pointer argument");
    if (N <= 0 || K <= 0) return fail(DG_ERR_INVALID_ARG, "N=%lld and K=%lld must be positive", N, K);
    if (K % 128) return fail(DG_ERR_ALIGNMENT, "K=%lld must be a multiple of 128", K);
    if (N % 16) return fail(DG_ERR_ALIGNMENT, "N=%lld must be a multiple of 16", N);
    if (!aligned(a, 16) || !aligned(b, 16) || !aligned(d, 16) || !aligned(sfa, 16) || !aligned(sfb, 16))
        return fail(DG_ERR_ALIGNMENT, "a, b, d, sfa and sfb must be 16-byte aligned");
    return DG_OK;
}

}  // namespace


namespace {

// Swapped operands (masked, no-padding and contiguous layouts, e4m3 B, block-scaled): tiles of TILE_M rows of B
// (D's columns) x one chunk of at most kSwapTokens of a group's tokens (D's rows), the MMA's N set per tile to the
// chunk's rows rounded up to 16, so a group of m tokens costs ceil(m / 16) * 16 rows of MMA work instead of whole
// 128-row windows.  hint_chunks: the chunks the caller expects (picks single CTAs or pairs); max_chunks: the most the
// device can find (sizes the grid and the packed scales).
constexpr int kSwapTokens = 224;
constexpr int kSwapDefaultRows = 512;  // contiguous / no padding: swapped by default up to this mean group size

int select_block_n(long long windows, int N, int units, int ctas);

// The library's default for the contiguous and no-padding layouts (measured, interleaved in one process): the
// swapped tiles pay where groups are small (a group costs its rows rounded up to 16 instead of whole 256-row
// windows) or where the unswapped plan's tile width leaves part of its last column block empty and 256-wide swapped
// tiles do not (N = 4096: 19 blocks of 224 columns hold 4256; 0.984 of the unswapped time on G=8, K=7168).  With
// large groups and N a multiple of both widths they measured 1.03-1.04x slower (G=64, N=7168, K=2048: every group
// ends in a partial chunk, and a tile loads its whole 224-token box whatever its width).
bool swap_by_default(long long M_total, int G, int N, int sms) {
    if (M_total <= static_cast<long long>(G) * kSwapDefaultRows) return true;
    const long long windows = (M_total + 2 * dg::BLOCK_M - 1) / (2 * dg::BLOCK_M);
    const int bn = select_block_n(windows, N, sms / 2 > 0 ? sms / 2 : 1, 2);
    const double unswapped = static_cast<double>(N) / (static_cast<double>((N + bn - 1) / bn) * bn);
    const double swapped = static_cast<double>(N) / (static_cast<double>((N + 255) / 256) * 256);
    return swapped >= unswapped + 0.02;
}

// Swapped operands for this call?  by_default: the library's own choice for the layout and shape.
bool swap_enabled(bool by_default) {
    if (g_fp32_promotion.load()) return false;
    const int policy = g_swap_policy.load();
    return policy < 0 ? by_default : policy > 0;
}

int launch_swapped(dg::GemmParams p, const DeviceInfo &info, const void *a, long long a_rows, const void *b,
                   long long b_rows, ScaleArgs sc, long long hint_chunks, long long max_chunks, cudaStream_t stream,
                   bool b_nn = false) {
    const int sms = effective_sms(info);
    const int policy = g_pair_policy.load();
    bool pair = sms >= 2 && policy != 0;
    if (pair && policy < 0)  // pairs pay once there is at least a wave of them
        pair = hint_chunks * ((p.N + 2 * dg::BLOCK_M - 1) / (2 * dg::BLOCK_M)) >= sms / 2;
    const int tile_m = pair ? 2 * dg::BLOCK_M : dg::BLOCK_M;
    p.num_n_blocks = (p.N + tile_m - 1) / tile_m;
    p.sfa_blocks = p.num_n_blocks * (pair ? 2 : 1);
    if (max_chunks > 0x7fffffffLL / 16) return fail(DG_ERR_INVALID_ARG, "too many token chunks");
    p.swap_chunks = static_cast<int>(max_chunks);
    p.num_windows = 0;
    p.num_sf_groups = (p.K / dg::BLOCK_K + dg::SF_GROUP - 1) / dg::SF_GROUP;
    sc.swap = true;
    const long long tiles = max_chunks * p.num_n_blocks;
    const int units = pair ? sms / 2 : sms;
    const int grid = static_cast<int>(tiles < units ? tiles : units);
    if (grid <= 0) return DG_OK;
    if (b_nn) {  // B [G][K][N] read as MN-major tiles, no transposed copy
        if (pair)
            return launch_cfg<kSwapTokens, 2, 2, false, true, true>(a, a_rows, b, b_rows, sc, p, grid, info.device, stream);
        return launch_cfg<kSwapTokens, 1, 1, false, true, true>(a, a_rows, b, b_rows, sc, p, grid, info.device, stream);
    }
    if (pair) return launch_cfg<kSwapTokens, 2, 2, false, true>(a, a_rows, b, b_rows, sc, p, grid, info.device, stream);
    return launch_cfg<kSwapTokens, 1, 1, false, true>(a, a_rows, b, b_rows, sc, p, grid, info.device, stream);
}

int check_contiguous(const void *a, const float *sfa, const void *b, const float *sfb, const void *d,
                     const int *m_indices, int M_total, int N, int K, int G) {
    if (int rc = check_common(a, sfa, b, sfb, d, N, K)) return rc;
    if (!m_indices) return fail(DG_ERR_INVALID_ARG, "m_indices is null");
    if (!aligned(m_indices, 4)) return fail(DG_ERR_ALIGNMENT, "m_indices must be 4-byte aligned");
    if (G < 1 || G > 65534) return fail(DG_ERR_INVALID_ARG, "G=%d must be in [1, 65534]", G);
    if (M_total < 0) return fail(DG_ERR_INVALID_ARG, "M_total=%d must be non-negative", M_total);
    const int alignment = g_m_alignment.load();
    if (M_total % alignment)
        return fail(DG_ERR_ALIGNMENT, "M_total=%d must be a multiple of %d", M_total, alignment);
    if (static_cast<long long>(G) * N > 0x7fffffffLL) return fail(DG_ERR_INVALID_ARG, "G*N exceeds 2^31");
    return DG_OK;
}

// The contiguous GEMM on checked arguments (M_total > 0); `sfb_kn` selects the NN orientation of SFB.
int launch_contiguous(const void *a, const float *sfa, const void *b, const float *sfb, void *d,
                      const int *m_indices, int M_total, int N, int K, int G, bool sfb_kn, const DeviceInfo &info,
                      cudaStream_t stream, bool b_fp4 = false, bool b_nn = false) {
    dg::GemmParams p{};
    p.mode = dg::MODE_CONTIGUOUS;
    p.M = M_total; p.N = N; p.K = K; p.G = G;
    ScaleArgs sc{sfa, dg_get_tma_aligned_size(M_total, 4), sfb};
    sc.sfb_kn = sfb_kn;
    sc.sfb_fp4 = b_fp4;
    if (b_fp4) sc.sfb_ld = dg_get_tma_aligned_size(N, 4);
    p.d = static_cast<__nv_bfloat16 *>(d);
    p.m_indices = m_indices;
    p.err = device_error_word();
    if (!p.err) return fail(DG_ERR_CUDA, "device error word is not available");
    const long long w1 = M_total / dg::BLOCK_M, w2 = (w1 + 1) / 2;
    // Swapped operands while the device's tables hold every 128-row block: runs of blocks of one group, each cut
    // into token chunks; at most ceil(M_total / kSwapTokens) full chunks plus one partial chunk per run.
    // b_nn: B is [G][K][N], read directly by the swapped tiles (the caller has checked they apply)
    if (b_nn || (!b_fp4 && swap_enabled(swap_by_default(M_total, G, N, effective_sms(info))) &&
                 w1 <= dg::MAX_MASKED_GROUPS)) {
        const long long full = (M_total + kSwapTokens - 1) / kSwapTokens;
        return launch_swapped(p, info, a, M_total, b, static_cast<long long>(G) * (b_nn ? K : N), sc,
                              full + (G < w1 ? G : w1) / 2, full + w1, stream, b_nn);
    }
    // a 256-row window holds at most two tiles (its halves may belong to two groups)
    const long long bound = w2 + (w2 < G ? w2 : G);
    // pairs need the device-built window list to fit (at most NB/2 + G/2 windows) and group ids below 2^15
    const bool pair_ok = (w1 + G) / 2 + 1 <= dg::MAX_PAIR_WINDOWS && G <= 32767;
    const Plan plan{w1, w2, w1, bound, w1, w2, pair_ok};
    return plan_and_launch(p, info, plan, a, M_total, b, static_cast<long long>(G) * N, sc, stream);
}

}  // namespace

namespace {

// Dense calls this short run as one kernel -- the promotion GEMM, reading the caller's scales -- instead of the
// scale pre-pass and the block-scaled GEMM: their time is then mostly the second launch and the GEMM's wait for
// the pre-pass (about 6 us), which the promotion's costlier per-K-block epilogue does not spend back while K is
// short.  Measured on B200 (L2 flushed between calls, CUDA events), one kernel / two: 0.66 at 128 x 256 x 512,
// 0.85-0.88 from 0.5 to 8.6 GFLOP with K <= 2048, 0.92 at 1024 x 4096 x 2048; 1.05-1.10 with K = 7168 and 1.29 at
// 2048 x 4096 x 4096.  The scales must still be powers of two: the promotion epilogue checks each one it reads
// (DG_ERR_BAD_SCALE) and reads a zero scale as 2^-127, as the block-scaled path does.
constexpr int kSingleKernelMaxK = 2048;
constexpr long long kSingleKernelMaxFlops = 1ll << 34;
bool dense_single_kernel(long long M, long long N, long long K) {
    return K <= kSingleKernelMaxK && 2 * M * N * K <= kSingleKernelMaxFlops;
}

// The dense calls; `fixed_scratch`: the packed scales go to the library's fixed buffer (no allocation).
int dense_call(const void *a, const float *sfa, const void *b, const float *sfb, void *d, int M, int N, int K,
               dg_stream_t stream, bool fixed_scratch) {
    if (M < 0) return fail(DG_ERR_INVALID_ARG, "M=%d must be non-negative", M);
    if (int rc = check_common(a, sfa, b, sfb, d, N, K)) return rc;
    if (M == 0) return DG_OK;
    DeviceInfo info;
    if (int rc = device_info(info)) return rc;
    dg::GemmParams p{};
    p.mode = dg::MODE_DENSE;
    p.M = M; p.N = N; p.K = K; p.G = 1;
    ScaleArgs sc{sfa, dg_get_tma_aligned_size(M, 4), sfb};
    sc.fixed_scratch = fixed_scratch;
    sc.single_kernel = dense_single_kernel(M, N, K);
    p.d = static_cast<__nv_bfloat16 *>(d);
    p.err = device_error_word();
    if (!p.err) return fail(DG_ERR_CUDA, "device error word is not available");
    const long long w1 = (M + dg::BLOCK_M - 1) / dg::BLOCK_M, w2 = (M + 2 * dg::BLOCK_M - 1) / (2 * dg::BLOCK_M);
    const Plan plan{w1, w2, w1, w2, w1, w2, true};
    return plan_and_launch(p, info, plan, a, M, b, N, sc, reinterpret_cast<cudaStream_t>(stream));
}

}  // namespace

namespace {

// The masked calls: B e4m3, or (b_fp4) B in E2M1 with one scale per (row, 32-K block).
int masked_call(const void *a, const float *sfa, const void *b, const float *sfb, void *d, const int *masked_m,
                int G, int M_max, int N, int K, int expected_m, dg_stream_t stream, bool b_fp4) {
    if (int rc = check_common(a, sfa, b, sfb, d, N, K)) return rc;
    if (!masked_m) return fail(DG_ERR_INVALID_ARG, "masked_m is null");
    if (!aligned(masked_m, 4)) return fail(DG_ERR_ALIGNMENT, "masked_m must be 4-byte aligned");
    if (G < 1 || G > dg::MAX_MASKED_GROUPS)
        return fail(DG_ERR_INVALID_ARG, "G=%d must be in [1, %d]", G, dg::MAX_MASKED_GROUPS);
    if (M_max < 1) return fail(DG_ERR_INVALID_ARG, "M_max=%d must be positive", M_max);
    if (static_cast<long long>(G) * M_max > 0x7fffffffLL || static_cast<long long>(G) * N > 0x7fffffffLL)
        return fail(DG_ERR_INVALID_ARG, "G*M_max or G*N exceeds 2^31");
    DeviceInfo info;
    if (int rc = device_info(info)) return rc;
    dg::GemmParams p{};
    p.mode = dg::MODE_MASKED;
    p.M = M_max; p.N = N; p.K = K; p.G = G;
    ScaleArgs sc{sfa, dg_get_tma_aligned_size(M_max, 4), sfb};
    sc.sfb_fp4 = b_fp4;
    if (b_fp4) sc.sfb_ld = dg_get_tma_aligned_size(N, 4);
    p.sfa_blocks = (M_max + dg::BLOCK_M - 1) / dg::BLOCK_M;
    p.d = static_cast<__nv_bfloat16 *>(d);
    p.masked_m = masked_m;
    p.err = device_error_word();
    if (!p.err) return fail(DG_ERR_CUDA, "device error word is not available");
    const int hint = expected_m > 0 && expected_m < M_max ? expected_m : M_max;
    if (!b_fp4 && swap_enabled(true)) {
        const long long per = (M_max + kSwapTokens - 1) / kSwapTokens, hint_per = (hint + kSwapTokens - 1) / kSwapTokens;
        return launch_swapped(p, info, a, static_cast<long long>(G) * M_max, b, static_cast<long long>(G) * N, sc,
                              G * hint_per, G * per, reinterpret_cast<cudaStream_t>(stream));
    }
    // tile shape from the caller's hint; the grid from the most tiles masked_m could ask for
    const long long h1 = static_cast<long long>(G) * ((hint + dg::BLOCK_M - 1) / dg::BLOCK_M);
    const long long h2 = static_cast<long long>(G) * ((hint + 2 * dg::BLOCK_M - 1) / (2 * dg::BLOCK_M));
    const long long max1 = static_cast<long long>(G) * ((M_max + dg::BLOCK_M - 1) / dg::BLOCK_M);
    const long long max2 = static_cast<long long>(G) * ((M_max + 2 * dg::BLOCK_M - 1) / (2 * dg::BLOCK_M));
    const Plan plan{h1, h2, max1, max2, 0, 0, true};
    return plan_and_launch(p, info, plan, a, static_cast<long long>(G) * M_max, b, static_cast<long long>(G) * N, sc,
                           reinterpret_cast<cudaStream_t>(stream));
}

}  // namespace

extern "C" {

int dg_get_m_alignment_for_contiguous_layout(void) { return g_m_alignment.load(); }

int dg_set_m_alignment_for_contiguous_layout(int alignment) {
    if (alignment != 128 && alignment != 256)
        return fail(DG_ERR_INVALID_ARG, "alignment=%d must be 128 or 256", alignment);
    g_m_alignment.store(alignment);
    return alignment;
}

int dg_get_tma_aligned_size(int mn, int elem_bytes) {
    if (elem_bytes <= 0) return -1;
    const int per16 = 16 / elem_bytes > 0 ? 16 / elem_bytes : 1;
    return (mn + per16 - 1) / per16 * per16;
}

int dg_set_num_sms(int n) {
    g_num_sms_cap.store(n > 0 ? n : 0);
    return dg_get_num_sms();
}

int dg_get_num_sms(void) {
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
        cudaGetLastError();
        return g_num_sms_cap.load();  // no device: report the cap alone
    }
    const int cap = g_num_sms_cap.load();
    return (cap > 0 && cap < sms) ? cap : sms;
}

long long dg_num_tiles(long long M, long long N, int block_m, int block_n) {
    if (M <= 0 || N <= 0 || block_m <= 0 || block_n <= 0) return 0;
    return ((M + block_m - 1) / block_m) * ((N + block_n - 1) / block_n);
}

int dg_select_block_n(long long num_m_blocks, int N, int num_sms) { return select_block_n(num_m_blocks, N, num_sms, 1); }

const char *dg_last_error(void) { return g_last_error.c_str(); }

int dg_check_device_error(dg_stream_t stream) {
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    unsigned word = 0, zero = 0;
    if ((e = cudaMemcpyFromSymbol(&word, g_device_error_word, sizeof(word))) != cudaSuccess)
        return cuda_fail(e, "reading the device error word");
    if ((e = cudaMemcpyToSymbol(g_device_error_word, &zero, sizeof(zero))) != cudaSuccess)
        return cuda_fail(e, "clearing the device error word");
    if (word == dg::ERR_TIMEOUT) return fail(DG_ERR_DEVICE_TIMEOUT, "a bounded wait inside the kernel ran out");
    if (word == dg::ERR_BAD_GROUP)
        return fail(DG_ERR_BAD_GROUP, "a group id or masked_m value was out of range; those rows were skipped");
    if (word == dg::ERR_BAD_SCALE)
        return fail(DG_ERR_BAD_SCALE,
                    "a scale was not a power of two; the block-scaled path applies only the exponent "
                    "(dg_set_fp32_scale_promotion(1) takes any fp32 scales)");
    if (word != 0) return fail(DG_ERR_CUDA, "unknown device error word %u", word);
    return DG_OK;
}

int dg_fp8_gemm_nt(const void *a, const float *sfa, const void *b, const float *sfb, void *d, int M, int N, int K,
                   dg_stream_t stream) {
    return dense_call(a, sfa, b, sfb, d, M, N, K, stream, false);
}


int dg_m_grouped_fp8_gemm_nt_contiguous(const void *a, const float *sfa, const void *b, const float *sfb, void *d,
                                        const int *m_indices, int M_total, int N, int K, int G, dg_stream_t stream) {
    if (int rc = check_contiguous(a, sfa, b, sfb, d, m_indices, M_total, N, K, G)) return rc;
    if (M_total == 0) return DG_OK;
    DeviceInfo info;
    if (int rc = device_info(info)) return rc;
    return launch_contiguous(a, sfa, b, sfb, d, m_indices, M_total, N, K, G, false, info,
                             reinterpret_cast<cudaStream_t>(stream));
}

int dg_m_grouped_fp8_fp4_gemm_nt_contiguous(const void *a, const float *sfa, const void *b, const float *sfb,
                                            void *d, const int *m_indices, int M_total, int N, int K, int G,
                                            dg_stream_t stream) {
    if (int rc = check_contiguous(a, sfa, b, sfb, d, m_indices, M_total, N, K, G)) return rc;
    if (!aligned(b, 32)) return fail(DG_ERR_ALIGNMENT, "b (packed E2M1) must be 32-byte aligned");
    if (M_total == 0) return DG_OK;
    DeviceInfo info;
    if (int rc = device_info(info)) return rc;
    return launch_contiguous(a, sfa, b, sfb, d, m_indices, M_total, N, K, G, false, info,
                             reinterpret_cast<cudaStream_t>(stream), true);
}

int dg_m_grouped_fp8_gemm_nn_contiguous(const void *a, const float *sfa, const void *b, const float *sfb, void *d,
                                        const int *m_indices, int M_total, int N, int K, int G, dg_stream_t stream) {
    if (int rc = check_contiguous(a, sfa, b, sfb, d, m_indices, M_total, N, K, G)) return rc;
    if (M_total == 0) return DG_OK;
    DeviceInfo info;
    if (int rc = device_info(info)) return rc;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // Swapped-operand tiles read B [G][K][N] as MN-major tiles: no transposed copy
    if (swap_enabled(true) && M_total / dg::BLOCK_M <= dg::MAX_MASKED_GROUPS)
        return launch_contiguous(a, sfa, b, sfb, d, m_indices, M_total, N, K, G, true, info, s, false, true);
    // Otherwise B [G][K][N] -> K-major [G][N][K] in stream-ordered scratch, then the NT path
    cudaMemPool_t pool;
    if (int rc = scratch_pool(info.device, pool)) return rc;
    const size_t bytes = static_cast<size_t>(G) * N * K;
    void *bt = nullptr;
    cudaError_t e = cudaMallocFromPoolAsync(&bt, bytes, pool, s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMallocFromPoolAsync (B transposed)");
    const long long tiles = static_cast<long long>(G) * (K / dg::TRANSPOSE_TILE) *
                            ((N + dg::TRANSPOSE_TILE - 1) / dg::TRANSPOSE_TILE);
    const long long cap = 8LL * info.num_sms;
    dg::transpose_kn_to_nk_kernel<<<static_cast<unsigned>(tiles < cap ? tiles : cap), dg::TRANSPOSE_THREADS, 0, s>>>(
        static_cast<const uint8_t *>(b), static_cast<uint8_t *>(bt), G, K, N);
    int rc = DG_OK;
    if ((e = cudaGetLastError()) != cudaSuccess) rc = cuda_fail(e, "transpose launch");
    if (rc == DG_OK) rc = launch_contiguous(a, sfa, bt, sfb, d, m_indices, M_total, N, K, G, true, info, s);
    const cudaError_t ef = cudaFreeAsync(bt, s);
    if (rc == DG_OK && ef != cudaSuccess) rc = cuda_fail(ef, "cudaFreeAsync (B transposed)");
    return rc;
}

int dg_m_grouped_fp8_gemm_nt_masked(const void *a, const float *sfa, const void *b, const float *sfb, void *d,
                                    const int *masked_m, int G, int M_max, int N, int K, int expected_m,
                                    dg_stream_t stream) {
    return masked_call(a, sfa, b, sfb, d, masked_m, G, M_max, N, K, expected_m, stream, false);
}

int dg_m_grouped_fp8_fp4_gemm_nt_masked(const void *a, const float *sfa, const void *b, const float *sfb, void *d,
                                        const int *masked_m, int G, int M_max, int N, int K, int expected_m,
                                        dg_stream_t stream) {
    if (b && !aligned(b, 32)) return fail(DG_ERR_ALIGNMENT, "b (packed E2M1) must be 32-byte aligned");
    return masked_call(a, sfa, b, sfb, d, masked_m, G, M_max, N, K, expected_m, stream, true);
}


int dg_debug_bounded_wait(unsigned long long limit_ns, int drop_first_stage) {
    if (limit_ns != 0 && (limit_ns < 1000000ull || limit_ns > dg::WAIT_LIMIT_NS))
        return fail(DG_ERR_INVALID_ARG, "limit_ns=%llu must be 0 or within [1 ms, 2 s]", limit_ns);
    g_wait_limit_ns.store(limit_ns == 0 ? dg::WAIT_LIMIT_NS : limit_ns);
    g_drop_first_stage.store(drop_first_stage != 0);
    return DG_OK;
}

int dg_debug_clock_record(int enable) {
    g_clock_record.store(enable != 0);
    return enable != 0 ? 1 : 0;
}

int dg_debug_clock_read(unsigned long long *out, int reset) {
    if (!out) return fail(DG_ERR_INVALID_ARG, "out is null");
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
    if ((e = cudaMemcpyFromSymbol(out, g_clock_acc, sizeof(g_clock_acc))) != cudaSuccess)
        return cuda_fail(e, "reading the clock record");
    if (reset) {
        const unsigned long long zero[3] = {0, 0, 0};
        if ((e = cudaMemcpyToSymbol(g_clock_acc, zero, sizeof(zero))) != cudaSuccess)
            return cuda_fail(e, "clearing the clock record");
    }
    return DG_OK;
}

int dg_m_grouped_fp8_gemm_nt_nopad(const void *a, const float *sfa, const void *b, const float *sfb, void *d,
                                   const int *counts, int M_total, int N, int K, int G, dg_stream_t stream) {
    if (int rc = check_common(a, sfa, b, sfb, d, N, K)) return rc;
    if (!counts) return fail(DG_ERR_INVALID_ARG, "counts is null");
    if (!aligned(counts, 4)) return fail(DG_ERR_ALIGNMENT, "counts must be 4-byte aligned");
    if (G < 1 || G > dg::MAX_MASKED_GROUPS)
        return fail(DG_ERR_INVALID_ARG, "G=%d must be in [1, %d]", G, dg::MAX_MASKED_GROUPS);
    if (M_total < 0) return fail(DG_ERR_INVALID_ARG, "M_total=%d must be non-negative", M_total);
    if (static_cast<long long>(G) * N > 0x7fffffffLL) return fail(DG_ERR_INVALID_ARG, "G*N exceeds 2^31");
    if (M_total == 0) return DG_OK;
    DeviceInfo info;
    if (int rc = device_info(info)) return rc;
    dg::GemmParams p{};
    p.mode = dg::MODE_NOPAD;
    p.M = M_total; p.N = N; p.K = K; p.G = G;
    ScaleArgs sc{sfa, dg_get_tma_aligned_size(M_total, 4), sfb};
    p.d = static_cast<__nv_bfloat16 *>(d);
    p.masked_m = counts;
    p.err = device_error_word();
    if (!p.err) return fail(DG_ERR_CUDA, "device error word is not available");
    // chunks: each group adds at most one partial chunk to ceil(M_total / kSwapTokens) (by default only for small
    // groups, as for the contiguous layout)
    if (swap_enabled(swap_by_default(M_total, G, N, effective_sms(info)))) {
        const long long full = (M_total + kSwapTokens - 1) / kSwapTokens;
        return launch_swapped(p, info, a, M_total, b, static_cast<long long>(G) * N, sc, full + G / 2, full + G,
                              reinterpret_cast<cudaStream_t>(stream));
    }
    // Windows: each group adds at most one partial window to ceil(M_total / rows per window); the tile shape
    // is chosen for half a partial window per group.
    const long long w1 = (M_total + dg::BLOCK_M - 1) / dg::BLOCK_M, w2 = (M_total + 2 * dg::BLOCK_M - 1) / (2 * dg::BLOCK_M);
    const Plan plan{w1 + G / 2, w2 + G / 2, w1 + G, w2 + G, 0, 0, true};
    return plan_and_launch(p, info, plan, a, M_total, b, static_cast<long long>(G) * N, sc,
                           reinterpret_cast<cudaStream_t>(stream));
}

int dg_k_grouped_fp8_gemm_nt_contiguous(const void *a, const float *sfa, const void *b, const float *sfb, float *d,
                                        const float *c, const int *ks, const int *ks_device, int G, int M, int N,
                                        dg_stream_t stream) {
    if (!a || !sfa || !b || !sfb || !d || !ks || !ks_device) return fail(DG_ERR_INVALID_ARG, "null pointer argument");
    if (G < 1 || G > dg::MAX_MASKED_GROUPS)
        return fail(DG_ERR_INVALID_ARG, "G=%d must be in [1, %d]", G, dg::MAX_MASKED_GROUPS);
    if (M < 0 || N <= 0) return fail(DG_ERR_INVALID_ARG, "M=%d must be non-negative and N=%d positive", M, N);
    if (N % 16) return fail(DG_ERR_ALIGNMENT, "N=%d must be a multiple of 16", N);
    if (!aligned(a, 16) || !aligned(b, 16) || !aligned(d, 16) || (c && !aligned(c, 16)))
        return fail(DG_ERR_ALIGNMENT, "a, b, c and d must be 16-byte aligned");
    if (!aligned(sfa, 4) || !aligned(sfb, 4) || !aligned(ks_device, 4))
        return fail(DG_ERR_ALIGNMENT, "sfa, sfb and ks_device must be 4-byte aligned");
    long long K_total = 0, sf_groups = 0;
    for (int g = 0; g < G; ++g) {
        if (ks[g] < 0 || ks[g] % dg::BLOCK_K)
            return fail(DG_ERR_ALIGNMENT, "ks[%d]=%d must be a non-negative multiple of %d", g, ks[g], dg::BLOCK_K);
        K_total += ks[g];
        sf_groups += (ks[g] / dg::BLOCK_K + dg::SF_GROUP - 1) / dg::SF_GROUP;
    }
    if (K_total > 0x7fffff80LL) return fail(DG_ERR_INVALID_ARG, "the sum of ks exceeds 2^31");
    if (static_cast<long long>(G) * M * N > 0x7fffffffLL) return fail(DG_ERR_INVALID_ARG, "G*M*N exceeds 2^31");
    if (M == 0) return DG_OK;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const size_t d_bytes = static_cast<size_t>(G) * M * N * sizeof(float);
    // D = C + sum: a separate C is copied into D first and the products are added to D in place
    cudaError_t e;
    if (c && c != d && (e = cudaMemcpyAsync(d, c, d_bytes, cudaMemcpyDeviceToDevice, s)) != cudaSuccess)
        return cuda_fail(e, "cudaMemcpyAsync (C into D)");
    if (K_total == 0) {  // nothing to add
        if (!c && (e = cudaMemsetAsync(d, 0, d_bytes, s)) != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync (D)");
        return DG_OK;
    }
    DeviceInfo info;
    if (int rc = device_info(info)) return rc;
    dg::GemmParams p{};
    p.mode = dg::MODE_KGROUPED;
    p.out_mode = c ? dg::OUT_F32_ADD : dg::OUT_F32_STORE;
    p.M = M; p.N = N; p.K = static_cast<int>(K_total); p.G = G;
    p.num_sf_groups = static_cast<int>(sf_groups);
    p.d32 = d;
    p.masked_m = ks_device;
    p.err = device_error_word();
    if (!p.err) return fail(DG_ERR_CUDA, "device error word is not available");
    ScaleArgs sc{sfa, dg_get_tma_aligned_size(M, 4), sfb};
    sc.sfb_ld = dg_get_tma_aligned_size(N, 4);
    // every group covers all M rows: G x ceil(M / rows per window) windows
    const long long w1 = static_cast<long long>(G) * ((M + dg::BLOCK_M - 1) / dg::BLOCK_M);
    const long long w2 = static_cast<long long>(G) * ((M + 2 * dg::BLOCK_M - 1) / (2 * dg::BLOCK_M));
    const Plan plan{w1, w2, w1, w2, w1, w2, true};
    return plan_and_launch(p, info, plan, a, M, b, N, sc, s);
}

int dg_set_fp32_scale_promotion(int enable) {
    g_fp32_promotion.store(enable != 0);
    return enable != 0 ? 1 : 0;
}

int dg_get_fp32_scale_promotion(void) { return g_fp32_promotion.load() ? 1 : 0; }

int dg_set_swap_policy(int policy) {
    const int v = policy < 0 ? -1 : (policy > 0 ? 1 : 0);
    g_swap_policy.store(v);
    return v;
}

int dg_set_cta_pair_policy(int policy) {
    const int v = policy < 0 ? -1 : (policy > 0 ? 1 : 0);
    g_pair_policy.store(v);
    return v;
}

int dg_fp8_gemm_nt_noalloc(const void *a, const float *sfa, const void *b, const float *sfb, void *d, int M, int N,
                           int K, dg_stream_t stream) {
    return dense_call(a, sfa, b, sfb, d, M, N, K, stream, true);
}

}  // extern "C"
