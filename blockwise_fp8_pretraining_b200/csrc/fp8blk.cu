// C ABI of the blockwise-E4M3 FP8 linear-layer library (see include/fp8blk.h
// for the contract of every entry point).  Host code here only checks
// arguments, builds TMA tensor maps and launches kernels on the caller's
// stream; it never allocates or synchronizes (except fp8_get_error /
// fp8_clear_error, which read or reset the device error word).
#include <cudaTypedefs.h>

#include <atomic>
#include <cstdint>
#include <cstdio>
#include <cstring>

#include "../../include/fp8blk.h"
#include "gemm.cuh"
#include "quantize.cuh"

static_assert(fp8blk::kErrTimeout == static_cast<unsigned int>(FP8_ERR_TIMEOUT),
              "device time-out code must match the C ABI");

namespace {

// Launch with programmatic stream serialization: the kernel may begin
// launching while the preceding kernel of the stream finishes; it waits for
// that kernel's results in griddep_wait before touching global memory.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, args...);
}


using namespace fp8blk;

constexpr uint64_t kDefaultWaitNs = 2000000000ull;
std::atomic<uint64_t> g_wait_ns{kDefaultWaitNs};

// Test only (fp8_selftest_stall_next): bit 0 arms the next GEMM launch,
// bit 1 the next tile-quantizer launch, to over-state one barrier's bytes.
std::atomic<int> g_stall_next{0};
constexpr uint32_t kStallBytes = 16;

inline uint32_t take_stall(int bit) {
    return (g_stall_next.fetch_and(~bit) & bit) ? kStallBytes : 0u;
}

constexpr int kMaxDevices = 64;
std::atomic<int> g_sm_count[kMaxDevices];
std::atomic<int> g_gemm_attr_done[kMaxDevices];
std::atomic<int> g_gemm_pairs[kMaxDevices][12];  // co-resident CTA pairs per kernel variant

constexpr int64_t kMaxDim = (int64_t(1) << 31) - 1;

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Text of the last CUDA failure this thread saw (for fp8_last_cuda_error).
thread_local char g_detail[256] = "";

fp8_status cuda_fail(const char* where, cudaError_t e) {
    snprintf(g_detail, sizeof g_detail, "%s: %s (%d)", where, cudaGetErrorString(e), static_cast<int>(e));
    return FP8_ERR_CUDA;
}

inline fp8_status last_launch_status(const char* where) {
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? FP8_OK : cuda_fail(where, e);
}

fp8_status current_device(int* dev) {
    const cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess) return cuda_fail("cudaGetDevice", e);
    if (*dev < 0 || *dev >= kMaxDevices) return cuda_fail("device ordinal out of range", cudaErrorInvalidDevice);
    return FP8_OK;
}

fp8_status sm_count(int dev, int* out) {
    int n = g_sm_count[dev].load(std::memory_order_relaxed);
    if (n <= 0) {
        const cudaError_t e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail("cudaDeviceGetAttribute", e);
        g_sm_count[dev].store(n, std::memory_order_relaxed);
    }
    *out = n;
    return FP8_OK;
}

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static std::atomic<void*> fn{nullptr};
    void* f = fn.load(std::memory_order_acquire);
    if (!f) {
        cudaDriverEntryPointQueryResult q;
        const cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q);
        if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !f) {
            snprintf(g_detail, sizeof g_detail, "cudaGetDriverEntryPoint(cuTensorMapEncodeTiled): %s, query %d",
                     cudaGetErrorString(e), static_cast<int>(q));
            return nullptr;
        }
        fn.store(f, std::memory_order_release);
    }
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
}

// Row-major [rows, cols] byte matrix, boxes of box_rows x 128 bytes in the
// 128-byte swizzle the MMA descriptors expect; out-of-range rows read as 0.
fp8_status make_operand_map(CUtensorMap* map, const uint8_t* base, int64_t rows, int64_t cols,
                            int box_rows) {
    auto enc = tensor_map_encoder();
    if (!enc) return FP8_ERR_CUDA;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols)};
    cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estride[2] = {1u, 1u};
    CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(base), dims, strides,
                     box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        snprintf(g_detail, sizeof g_detail, "cuTensorMapEncodeTiled: CUresult %d", static_cast<int>(r));
        return FP8_ERR_CUDA;
    }
    return FP8_OK;
}

// Row-major [rows, cols] GEMM output, boxes of 32 rows x 128 bytes (64 BF16
// or 32 FP32 columns) in the 128-byte swizzle of the epilogue's staging
// buffers.
fp8_status make_output_map(CUtensorMap* map, void* base, int64_t rows, int64_t cols, bool f32) {
    auto enc = tensor_map_encoder();
    if (!enc) return FP8_ERR_CUDA;
    const int esize = f32 ? 4 : 2;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * esize};
    cuuint32_t box[2] = {static_cast<cuuint32_t>(128 / esize), 32u};
    cuuint32_t estride[2] = {1u, 1u};
    CUresult r = enc(map, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims,
                     strides, box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                     CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        snprintf(g_detail, sizeof g_detail, "cuTensorMapEncodeTiled(output): CUresult %d", static_cast<int>(r));
        return FP8_ERR_CUDA;
    }
    return FP8_OK;
}

// 2-D row-major map with a box of box_x (inner) by box_y elements.
fp8_status make_map_2d(CUtensorMap* map, CUtensorMapDataType type, int elem_bytes, const void* base,
                       int64_t rows, int64_t cols, uint32_t box_x, uint32_t box_y,
                       CUtensorMapSwizzle swizzle, const char* what) {
    auto enc = tensor_map_encoder();
    if (!enc) return FP8_ERR_CUDA;
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * elem_bytes};
    cuuint32_t box[2] = {box_x, box_y};
    cuuint32_t estride[2] = {1u, 1u};
    CUresult r = enc(map, type, 2, const_cast<void*>(base), dims, strides, box, estride,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, swizzle, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        snprintf(g_detail, sizeof g_detail, "cuTensorMapEncodeTiled(%s): CUresult %d", what, static_cast<int>(r));
        return FP8_ERR_CUDA;
    }
    return FP8_OK;
}

std::atomic<int> g_tile_attr_done[kMaxDevices];

// Persistent 128 x 128 tile quantizer (column-wise, both, weight blocks;
// with kProdSwiglu the SwiGLU product of a gate_up activation [rows, 2 *
// cols], with kProdNorm the RMSNorm output of x given r and gamma).
template <int MODE, int PROD>
fp8_status launch_tile_quant(const void* x, int64_t rows, int64_t cols, uint8_t* q, float* s_row,
                             uint8_t* qT, float* s_col, cudaStream_t stream, const float* norm_r = nullptr,
                             const void* norm_gamma = nullptr) {
    constexpr bool SWIGLU = PROD == kProdSwiglu;
    using L = tile::Layout<SWIGLU>;
    int dev = 0, sms = 0;
    fp8_status st = current_device(&dev);
    if (st != FP8_OK) return st;
    if ((st = sm_count(dev, &sms)) != FP8_OK) return st;
    const int flag = 1 << (MODE + 4 * PROD);
    if ((g_tile_attr_done[dev].load(std::memory_order_relaxed) & flag) == 0) {
        const cudaError_t e = cudaFuncSetAttribute(quant_tile_kernel<MODE, PROD>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   L::SMEM_BYTES);
        if (e != cudaSuccess) return cuda_fail("cudaFuncSetAttribute(quantize)", e);
        g_tile_attr_done[dev].fetch_or(flag, std::memory_order_relaxed);
    }
    CUtensorMap mx, mq, mqt;
    if ((st = make_map_2d(&mx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, x, rows, SWIGLU ? 2 * cols : cols, 64, 128,
                          CU_TENSOR_MAP_SWIZZLE_128B, "quantize input")) != FP8_OK)
        return st;
    // Unused maps still need a valid encoding: point them at an output.
    const void* qbase = q ? static_cast<const void*>(q) : static_cast<const void*>(qT);
    const void* qtbase = qT ? static_cast<const void*>(qT) : static_cast<const void*>(q);
    if ((st = make_map_2d(&mq, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, qbase, q ? rows : cols, q ? cols : rows,
                          128, 128, CU_TENSOR_MAP_SWIZZLE_128B, "row codes")) != FP8_OK)
        return st;
    if ((st = make_map_2d(&mqt, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, qtbase, qT ? cols : rows, qT ? rows : cols,
                          128, 128, CU_TENSOR_MAP_SWIZZLE_128B, "transposed codes")) != FP8_OK)
        return st;
    const int64_t tiles = (rows / 128) * (cols / 128);
    const int64_t cap = static_cast<int64_t>(L::BLOCKS_PER_SM) * sms;
    const unsigned grid = static_cast<unsigned>(tiles < cap ? tiles : cap);
    const cudaError_t e = launch_pdl(quant_tile_kernel<MODE, PROD>, dim3(grid), dim3(tile::THREADS),
                                     L::SMEM_BYTES, stream, mx, mq, mqt, rows, cols, s_row, s_col,
                                     qT != nullptr ? 1 : 0, g_wait_ns.load(std::memory_order_relaxed),
                                     take_stall(2), norm_r, static_cast<const __nv_bfloat16*>(norm_gamma));
    if (e != cudaSuccess) return cuda_fail("tile quantize launch", e);
    return last_launch_status("tile quantize launch");
}

// Workspace of the split schedule for `pairs` CTA pairs: FP32 partial sums
// [pairs][2][EPI_WARPS][32][32][4], then one flag per pair, CTA, warp and lane.
constexpr size_t kPartialFloatsPerPair = size_t(2) * gemm::EPI_WARPS * 128 * 32;
inline size_t gemm_workspace_bytes(int pairs) {
    const size_t partial = size_t(pairs) * kPartialFloatsPerPair * sizeof(float);
    const size_t flags = size_t(pairs) * 2 * gemm::EPI_WARPS * 32 * sizeof(int);
    return (partial + flags + 255) / 256 * 256;
}

// Whole tiles round-robin for all waves but the last two when the last wave
// would leave more than 5% of the pairs idle, a tile has at least 32 slabs
// and each pair has at least g_split_min_units (tile, slab) units of work;
// those tiles are then cut into ranges of slabs of equal length, one per
// pair.  (Measured on B200: handing partial sums over costs a few
// microseconds per launch, more than the idle pairs cost with 16 slabs per
// tile or with under about 150 units per pair.)
constexpr int kMinSplitSlabs = 32;
constexpr int64_t kDefaultSplitMinUnits = FP8_GEMM_SPLIT_MIN_WORK_DEFAULT;
std::atomic<int64_t> g_split_min_units{kDefaultSplitMinUnits};
inline int dp_tiles_for(int64_t tiles, int pairs, int num_kb) {
    const int64_t waves = (tiles + pairs - 1) / pairs;
    if (num_kb < kMinSplitSlabs || tiles >= waves * pairs * 95 / 100 ||
        tiles * num_kb < g_split_min_units.load(std::memory_order_relaxed) * pairs)
        return static_cast<int>(tiles);
    const int64_t full = tiles / pairs;
    return static_cast<int>(full >= 1 ? (full - 1) * pairs : 0);
}

// One-time set-up of a GEMM kernel variant on a device: its shared-memory
// limit, and how many CTA pairs can be resident at once (the persistent grid
// must not exceed it, or the last pairs would wait for a second wave).
template <int SCALE, int OUT, bool SPLIT>
fp8_status gemm_pairs(int dev, int sms, int* pairs_out) {
    constexpr int variant = SCALE + 2 * OUT + 6 * (SPLIT ? 1 : 0);
    const int flag = 1 << variant;
    if ((g_gemm_attr_done[dev].load(std::memory_order_relaxed) & flag) == 0) {
        cudaError_t e = cudaFuncSetAttribute(gemm::gemm_kernel<SCALE, OUT, SPLIT>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             gemm::SMEM_BYTES);
        if (e != cudaSuccess) return cuda_fail("cudaFuncSetAttribute(gemm)", e);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(sms & ~1), 1, 1);
        cfg.blockDim = dim3(gemm::THREADS, 1, 1);
        cfg.dynamicSmemBytes = gemm::SMEM_BYTES;
        int pairs = 0;
        e = cudaOccupancyMaxActiveClusters(&pairs, gemm::gemm_kernel<SCALE, OUT, SPLIT>, &cfg);
        if (e != cudaSuccess) return cuda_fail("cudaOccupancyMaxActiveClusters(gemm)", e);
        if (pairs <= 0) return cuda_fail("gemm kernel cannot be resident", cudaErrorInvalidConfiguration);
        g_gemm_pairs[dev][variant].store(pairs, std::memory_order_relaxed);
        g_gemm_attr_done[dev].fetch_or(flag, std::memory_order_relaxed);
    }
    *pairs_out = g_gemm_pairs[dev][variant].load(std::memory_order_relaxed);
    return FP8_OK;
}

// Shared launcher of the GEMMs.  A: [M_out, Kc] codes, B: [N_out, Kc]
// codes, both K-major; scales described by `p`; out: [M_out, N_out] BF16, or
// FP32 added to in place (OUT == kOutAccF32).  Launches the split-schedule
// variant of the kernel only when the schedule splits tiles: the plain
// variant's promotion loop carries nothing for it.
template <int SCALE, int OUT>
fp8_status launch_gemm(const uint8_t* a, const uint8_t* b, void* out, gemm::Params p, void* workspace,
                       size_t workspace_bytes, cudaStream_t stream) {
    int dev = 0, sms = 0;
    fp8_status st = current_device(&dev);
    if (st != FP8_OK) return st;
    if ((st = sm_count(dev, &sms)) != FP8_OK) return st;
    int max_pairs = 0, split_pairs = 0;
    if ((st = gemm_pairs<SCALE, OUT, false>(dev, sms, &max_pairs)) != FP8_OK) return st;

    CUtensorMap ma, mb, mc;
    if ((st = make_operand_map(&ma, a, p.M, p.K, gemm::BM)) != FP8_OK) return st;
    if ((st = make_operand_map(&mb, b, p.N, p.K, gemm::BN / 2)) != FP8_OK) return st;
    // (main-gradient mode writes through p.out_f32; the map still needs a
    // valid encoding)
    if ((st = make_output_map(&mc, out, OUT == gemm::kOutAccF32Shards ? (p.shard_rows > 32 ? p.shard_rows : 32) : p.M, p.N,
                              OUT != gemm::kOutBf16)) != FP8_OK)
        return st;
    if (OUT == gemm::kOutAccF32) p.out_f32 = static_cast<float*>(out);

    p.tiles_m = static_cast<int>((p.M + 2 * gemm::BM - 1) / (2 * gemm::BM));
    p.tiles_n = static_cast<int>((p.N + gemm::BN - 1) / gemm::BN);
    p.wait_ns = g_wait_ns.load(std::memory_order_relaxed);
    p.stall_tx = take_stall(1);
    const int64_t tiles = static_cast<int64_t>(p.tiles_m) * p.tiles_n;
    p.dp_tiles = static_cast<int>(tiles);
    p.ws_partial = nullptr;
    p.ws_flags = nullptr;
    if (workspace && workspace_bytes >= gemm_workspace_bytes(max_pairs))
        p.dp_tiles = dp_tiles_for(tiles, max_pairs, p.K / gemm::BK);
    if (p.dp_tiles < tiles) {
        // Same resources as the plain variant, so the same residency; a
        // smaller answer would leave pairs whose partial sums never arrive.
        if ((st = gemm_pairs<SCALE, OUT, true>(dev, sms, &split_pairs)) != FP8_OK) return st;
        if (split_pairs < max_pairs) p.dp_tiles = static_cast<int>(tiles);
    }
    cudaError_t e;
    if (p.dp_tiles < tiles) {
        p.ws_partial = static_cast<float*>(workspace);
        p.ws_flags = reinterpret_cast<int*>(static_cast<uint8_t*>(workspace) +
                                            size_t(max_pairs) * kPartialFloatsPerPair * sizeof(float));
        e = launch_pdl(gemm::gemm_kernel<SCALE, OUT, true>, dim3(2 * max_pairs), dim3(gemm::THREADS),
                       gemm::SMEM_BYTES, stream, ma, mb, mc, p);
    } else {
        const int grid_pairs = static_cast<int>(tiles < max_pairs ? tiles : max_pairs);
        e = launch_pdl(gemm::gemm_kernel<SCALE, OUT, false>, dim3(2 * grid_pairs), dim3(gemm::THREADS),
                       gemm::SMEM_BYTES, stream, ma, mb, mc, p);
    }
    if (e != cudaSuccess) return cuda_fail("gemm launch", e);
    return last_launch_status("gemm launch");
}

// wgrad: dW [N, K] over M tokens; A = dY^T codes [N, M], B = X^T codes [K, M].
gemm::Params wgrad_params(const float* sdyT, const float* sxT, int64_t N, int64_t K, int64_t M) {
    gemm::Params p{};
    p.sa = sdyT;
    p.sa_ld = N;                 // sdyT [M/128, N]
    p.sb = sxT;
    p.sb_ld = K;                 // sxT [M/128, K]
    p.M = static_cast<int>(N);
    p.N = static_cast<int>(K);
    p.K = static_cast<int>(M);
    return p;
}

bool dims_ok_gemm(int64_t M, int64_t N, int64_t K, bool m_positive) {
    if (M < 0 || N <= 0 || K <= 0) return false;
    if (m_positive && M == 0) return false;
    if (M % 128 || N % 128 || K % 128) return false;
    if (M > kMaxDim || N > kMaxDim || K > kMaxDim) return false;
    if (static_cast<int64_t>((M + 255) / 256) * ((N + gemm::BN - 1) / gemm::BN) > kMaxDim) return false;
    return true;
}

// Scratch of fp8_block_gemm_wgrad_static_ws: the split schedule's workspace
// as a file-scope device array, for callers that cannot allocate device
// memory.  Every GPU that loads the library holds it until the process
// exits; it starts zeroed (module load) and every call clears the flags it
// needs zeroed.
constexpr size_t kStaticWsBytes = size_t(24) << 20;     // 24 MiB: up to 94 CTA pairs
static __device__ __align__(256) uint8_t g_static_ws[kStaticWsBytes];
std::atomic<void*> g_static_ws_ptr[kMaxDevices];         // its device address, per device
std::atomic<int> g_static_ws_pairs[kMaxDevices];         // resident GEMM CTA pairs, per device

}  // namespace

extern "C" {

fp8_status fp8_quantize_act_1x128(const void* x_bf16, int64_t rows, int64_t cols, int mode,
                                  uint8_t* q_row, float* s_row, uint8_t* q_colT, float* s_col,
                                  void* stream) {
    if (mode != FP8_ROWWISE && mode != FP8_COLWISE && mode != FP8_BOTH) return FP8_ERR_MODE;
    if (rows < 0 || cols < 0 || cols % 128 != 0 || rows > kMaxDim || cols > kMaxDim)
        return FP8_ERR_SHAPE;
    if ((mode & FP8_COLWISE) && rows % 128 != 0) return FP8_ERR_SHAPE;
    if (rows == 0 || cols == 0) return FP8_OK;
    if (!x_bf16) return FP8_ERR_NULL;
    if ((mode & FP8_ROWWISE) && (!q_row || !s_row)) return FP8_ERR_NULL;
    if ((mode & FP8_COLWISE) && (!q_colT || !s_col)) return FP8_ERR_NULL;
    if (!aligned16(x_bf16)) return FP8_ERR_ALIGN;
    if ((mode & FP8_ROWWISE) && (!aligned16(q_row) || !aligned16(s_row))) return FP8_ERR_ALIGN;
    if ((mode & FP8_COLWISE) && (!aligned16(q_colT) || !aligned16(s_col))) return FP8_ERR_ALIGN;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const uint4* x = static_cast<const uint4*>(x_bf16);
    if (mode == FP8_ROWWISE) {
        int dev = 0, sms = 0;
        fp8_status st = current_device(&dev);
        if (st != FP8_OK) return st;
        if ((st = sm_count(dev, &sms)) != FP8_OK) return st;
        constexpr int kUnroll = 4;
        const int64_t groups = cols / 128;
        const int64_t units = rows * groups;
        const int64_t warps_needed = (units + 2 * kUnroll - 1) / (2 * kUnroll);
        int64_t blocks = (warps_needed + 7) / 8;
        const int64_t cap = static_cast<int64_t>(sms) * 8;
        if (blocks > cap) blocks = cap;
        const cudaError_t e = launch_pdl(quant_rowwise_kernel<kUnroll>, dim3(static_cast<unsigned>(blocks)),
                                         dim3(256), 0, s, x, units, rows, groups,
                                         reinterpret_cast<uint2*>(q_row), s_row);
        if (e != cudaSuccess) return cuda_fail("row-wise quantize launch", e);
        return last_launch_status("row-wise quantize launch");
    }
    if (mode == FP8_COLWISE)
        return launch_tile_quant<kTileColwise, kProdPlain>(x_bf16, rows, cols, nullptr, nullptr, q_colT, s_col, s);
    return launch_tile_quant<kTileBoth, kProdPlain>(x_bf16, rows, cols, q_row, s_row, q_colT, s_col, s);
}

fp8_status fp8_swiglu_quantize_1x128(const void* gate_up_bf16, int64_t rows, int64_t ffn, int mode,
                                     uint8_t* q_row, float* s_row, uint8_t* q_colT, float* s_col,
                                     void* stream) {
    if (mode != FP8_ROWWISE && mode != FP8_COLWISE && mode != FP8_BOTH) return FP8_ERR_MODE;
    if (rows < 0 || ffn < 0 || rows % 128 || ffn % 128 || rows > kMaxDim || ffn > kMaxDim / 2)
        return FP8_ERR_SHAPE;
    if (rows == 0 || ffn == 0) return FP8_OK;
    if (!gate_up_bf16) return FP8_ERR_NULL;
    if ((mode & FP8_ROWWISE) && (!q_row || !s_row)) return FP8_ERR_NULL;
    if ((mode & FP8_COLWISE) && (!q_colT || !s_col)) return FP8_ERR_NULL;
    if (!aligned16(gate_up_bf16)) return FP8_ERR_ALIGN;
    if ((mode & FP8_ROWWISE) && (!aligned16(q_row) || !aligned16(s_row))) return FP8_ERR_ALIGN;
    if ((mode & FP8_COLWISE) && (!aligned16(q_colT) || !aligned16(s_col))) return FP8_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (mode == FP8_ROWWISE)
        return launch_tile_quant<kTileRowwise, kProdSwiglu>(gate_up_bf16, rows, ffn, q_row, s_row, nullptr, nullptr, s);
    if (mode == FP8_COLWISE)
        return launch_tile_quant<kTileColwise, kProdSwiglu>(gate_up_bf16, rows, ffn, nullptr, nullptr, q_colT, s_col, s);
    return launch_tile_quant<kTileBoth, kProdSwiglu>(gate_up_bf16, rows, ffn, q_row, s_row, q_colT, s_col, s);
}

fp8_status fp8_rmsnorm_rstd(const void* x_bf16, int64_t rows, int64_t cols, float eps, float* rstd,
                            void* stream) {
    if (rows < 0 || cols < 0 || cols % 8 || rows > kMaxDim || cols > kMaxDim) return FP8_ERR_SHAPE;
    if (!(eps >= 0.0f) || eps > 3.0e38f) return FP8_ERR_SHAPE;
    if (rows == 0 || cols == 0) return FP8_OK;
    if (!x_bf16 || !rstd) return FP8_ERR_NULL;
    if (!aligned16(x_bf16) || !aligned16(rstd)) return FP8_ERR_ALIGN;
    const unsigned grid = static_cast<unsigned>((rows + 7) / 8);
    const cudaError_t e = launch_pdl(rmsnorm_rstd_kernel, dim3(grid), dim3(256), 0, static_cast<cudaStream_t>(stream),
                                     static_cast<const uint4*>(x_bf16), rows, cols, eps, rstd);
    if (e != cudaSuccess) return cuda_fail("rmsnorm rstd launch", e);
    return last_launch_status("rmsnorm rstd launch");
}

fp8_status fp8_rmsnorm_quantize_1x128(const void* x_bf16, int64_t rows, int64_t cols, const float* rstd,
                                      const void* gamma_bf16, int mode, uint8_t* q_row, float* s_row,
                                      uint8_t* q_colT, float* s_col, void* stream) {
    if (mode != FP8_ROWWISE && mode != FP8_COLWISE && mode != FP8_BOTH) return FP8_ERR_MODE;
    if (rows < 0 || cols < 0 || rows % 128 || cols % 128 || rows > kMaxDim || cols > kMaxDim)
        return FP8_ERR_SHAPE;
    if (rows == 0 || cols == 0) return FP8_OK;
    if (!x_bf16 || !rstd || !gamma_bf16) return FP8_ERR_NULL;
    if ((mode & FP8_ROWWISE) && (!q_row || !s_row)) return FP8_ERR_NULL;
    if ((mode & FP8_COLWISE) && (!q_colT || !s_col)) return FP8_ERR_NULL;
    if (!aligned16(x_bf16) || !aligned16(rstd) || !aligned16(gamma_bf16)) return FP8_ERR_ALIGN;
    if ((mode & FP8_ROWWISE) && (!aligned16(q_row) || !aligned16(s_row))) return FP8_ERR_ALIGN;
    if ((mode & FP8_COLWISE) && (!aligned16(q_colT) || !aligned16(s_col))) return FP8_ERR_ALIGN;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (mode == FP8_ROWWISE)
        return launch_tile_quant<kTileRowwise, kProdNorm>(x_bf16, rows, cols, q_row, s_row, nullptr, nullptr, s,
                                                          rstd, gamma_bf16);
    if (mode == FP8_COLWISE)
        return launch_tile_quant<kTileColwise, kProdNorm>(x_bf16, rows, cols, nullptr, nullptr, q_colT, s_col, s,
                                                          rstd, gamma_bf16);
    return launch_tile_quant<kTileBoth, kProdNorm>(x_bf16, rows, cols, q_row, s_row, q_colT, s_col, s, rstd,
                                                   gamma_bf16);
}

fp8_status fp8_quantize_weight_128x128(const void* w_bf16, int64_t n, int64_t k, uint8_t* wq,
                                       float* sw, uint8_t* wqT, void* stream) {
    if (n < 0 || k < 0 || n % 128 || k % 128 || n > kMaxDim || k > kMaxDim) return FP8_ERR_SHAPE;
    if (n == 0 || k == 0) return FP8_OK;
    if (!w_bf16 || !wq || !sw) return FP8_ERR_NULL;
    if (!aligned16(w_bf16) || !aligned16(wq) || !aligned16(sw) || (wqT && !aligned16(wqT)))
        return FP8_ERR_ALIGN;
    return launch_tile_quant<kTileWeight, kProdPlain>(w_bf16, n, k, wq, nullptr, wqT, sw,
                                          static_cast<cudaStream_t>(stream));
}

fp8_status fp8_block_gemm_fprop(const uint8_t* xq, const float* sx, const uint8_t* wq,
                                const float* sw, void* y_bf16, int64_t M, int64_t N, int64_t K,
                                void* workspace, size_t workspace_bytes, void* stream) {
    if (!dims_ok_gemm(M, N, K, false) || K > FP8_MAX_CONTRACTION_FPROP) return FP8_ERR_SHAPE;
    if (M == 0) return FP8_OK;
    if (!xq || !sx || !wq || !sw || !y_bf16) return FP8_ERR_NULL;
    if (!aligned16(xq) || !aligned16(sx) || !aligned16(wq) || !aligned16(sw) || !aligned16(y_bf16) ||
        !aligned16(workspace))
        return FP8_ERR_ALIGN;
    gemm::Params p{};
    p.sa = sx;
    p.sa_ld = M;                 // sx [K/128, M]
    p.sb = sw;
    p.sb_sn = K / 128;           // sw [N/128, K/128]
    p.sb_sk = 1;
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    return launch_gemm<gemm::kScaleRowBlock, gemm::kOutBf16>(xq, wq, y_bf16, p, workspace, workspace_bytes,
                                                             static_cast<cudaStream_t>(stream));
}

fp8_status fp8_block_gemm_dgrad(const uint8_t* dyq, const float* sdy, const uint8_t* wqT,
                                const float* sw, void* dx_bf16, int64_t M, int64_t N, int64_t K,
                                void* workspace, size_t workspace_bytes, void* stream) {
    if (!dims_ok_gemm(M, K, N, false) || N > FP8_MAX_CONTRACTION_FPROP) return FP8_ERR_SHAPE;
    if (M == 0) return FP8_OK;
    if (!dyq || !sdy || !wqT || !sw || !dx_bf16) return FP8_ERR_NULL;
    if (!aligned16(dyq) || !aligned16(sdy) || !aligned16(wqT) || !aligned16(sw) || !aligned16(dx_bf16) ||
        !aligned16(workspace))
        return FP8_ERR_ALIGN;
    gemm::Params p{};
    p.sa = sdy;
    p.sa_ld = M;                 // sdy [N/128, M]
    p.sb = sw;                   // s_b(output block kb, slab nb) = sw[nb][kb]
    p.sb_sn = 1;
    p.sb_sk = K / 128;
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(K);
    p.K = static_cast<int>(N);
    return launch_gemm<gemm::kScaleRowBlock, gemm::kOutBf16>(dyq, wqT, dx_bf16, p, workspace, workspace_bytes,
                                                             static_cast<cudaStream_t>(stream));
}

fp8_status fp8_block_gemm_wgrad(const uint8_t* dyqT, const float* sdyT, const uint8_t* xqT,
                                const float* sxT, void* dw_bf16, int64_t N, int64_t K, int64_t M,
                                void* workspace, size_t workspace_bytes, void* stream) {
    if (!dims_ok_gemm(N, K, M, true)) return FP8_ERR_SHAPE;
    if (!dyqT || !sdyT || !xqT || !sxT || !dw_bf16) return FP8_ERR_NULL;
    if (!aligned16(dyqT) || !aligned16(sdyT) || !aligned16(xqT) || !aligned16(sxT) || !aligned16(dw_bf16) ||
        !aligned16(workspace))
        return FP8_ERR_ALIGN;
    return launch_gemm<gemm::kScaleOuter, gemm::kOutBf16>(dyqT, xqT, dw_bf16, wgrad_params(sdyT, sxT, N, K, M),
                                                          workspace, workspace_bytes, static_cast<cudaStream_t>(stream));
}

fp8_status fp8_block_gemm_wgrad_accum_f32(const uint8_t* dyqT, const float* sdyT, const uint8_t* xqT,
                                          const float* sxT, float* dw_f32, int64_t N, int64_t K, int64_t M,
                                          void* workspace, size_t workspace_bytes, void* stream) {
    if (!dims_ok_gemm(N, K, M, true)) return FP8_ERR_SHAPE;
    if (!dyqT || !sdyT || !xqT || !sxT || !dw_f32) return FP8_ERR_NULL;
    if (!aligned16(dyqT) || !aligned16(sdyT) || !aligned16(xqT) || !aligned16(sxT) || !aligned16(dw_f32) ||
        !aligned16(workspace))
        return FP8_ERR_ALIGN;
    return launch_gemm<gemm::kScaleOuter, gemm::kOutAccF32>(dyqT, xqT, dw_f32, wgrad_params(sdyT, sxT, N, K, M),
                                                            workspace, workspace_bytes,
                                                            static_cast<cudaStream_t>(stream));
}

fp8_status fp8_block_gemm_wgrad_reduce_scatter_f32(const uint8_t* dyqT, const float* sdyT, const uint8_t* xqT,
                                                  const float* sxT, float* const* dw_shards, int nranks,
                                                  int64_t N, int64_t K, int64_t M, void* workspace,
                                                  size_t workspace_bytes, void* stream) {
    if (!dims_ok_gemm(N, K, M, true)) return FP8_ERR_SHAPE;
    if (nranks < 1 || nranks > gemm::kMaxShards || N % nranks) return FP8_ERR_SHAPE;
    if (!dyqT || !sdyT || !xqT || !sxT || !dw_shards) return FP8_ERR_NULL;
    if (!aligned16(dyqT) || !aligned16(sdyT) || !aligned16(xqT) || !aligned16(sxT) || !aligned16(workspace))
        return FP8_ERR_ALIGN;
    gemm::Params p = wgrad_params(sdyT, sxT, N, K, M);
    for (int q = 0; q < nranks; ++q) {
        if (!dw_shards[q]) return FP8_ERR_NULL;
        if (!aligned16(dw_shards[q])) return FP8_ERR_ALIGN;
        p.shards[q] = dw_shards[q];
    }
    p.shard_rows = N / nranks;
    return launch_gemm<gemm::kScaleOuter, gemm::kOutAccF32Shards>(dyqT, xqT, dw_shards[0], p, workspace,
                                                                  workspace_bytes, static_cast<cudaStream_t>(stream));
}

fp8_status fp8_block_gemm_wgrad_static_ws(const uint8_t* dyqT, const float* sdyT, const uint8_t* xqT,
                                          const float* sxT, void* dw_bf16, int64_t N, int64_t K, int64_t M,
                                          void* stream) {
    if (!dims_ok_gemm(N, K, M, true)) return FP8_ERR_SHAPE;
    if (!dyqT || !sdyT || !xqT || !sxT || !dw_bf16) return FP8_ERR_NULL;
    if (!aligned16(dyqT) || !aligned16(sdyT) || !aligned16(xqT) || !aligned16(sxT) || !aligned16(dw_bf16))
        return FP8_ERR_ALIGN;
    int dev = 0;
    fp8_status st = current_device(&dev);
    if (st != FP8_OK) return st;
    void* ws = g_static_ws_ptr[dev].load(std::memory_order_acquire);
    if (!ws) {
        // Set-up, once per device, with that device current: the array's
        // device address (the host-side name is only a stand-in for it) and
        // the number of CTA pairs, which sizes the part of it in use.
        void* ptr = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&ptr, g_static_ws);
        if (e != cudaSuccess || !ptr) return cuda_fail("cudaGetSymbolAddress(static GEMM workspace)", e);
        int sms = 0, pairs = 0;
        if ((st = sm_count(dev, &sms)) != FP8_OK) return st;
        if ((st = gemm_pairs<gemm::kScaleOuter, gemm::kOutBf16, false>(dev, sms, &pairs)) != FP8_OK) return st;
        g_static_ws_pairs[dev].store(pairs, std::memory_order_relaxed);
        g_static_ws_ptr[dev].store(ptr, std::memory_order_release);
        ws = ptr;
    }
    const int pairs = g_static_ws_pairs[dev].load(std::memory_order_relaxed);
    const size_t need = gemm_workspace_bytes(pairs);
    if (need > kStaticWsBytes) {
        snprintf(g_detail, sizeof g_detail,
                 "this GPU's GEMM workspace needs %zu bytes, more than the %zu-byte static one", need,
                 kStaticWsBytes);
        return FP8_ERR_SHAPE;
    }
    // The flags must be zero when a call starts; a call that timed out can
    // leave some set, so they are cleared every time (a memset, not an
    // allocation).
    const size_t flags_off = size_t(pairs) * kPartialFloatsPerPair * sizeof(float);
    const size_t flags_bytes = size_t(pairs) * 2 * gemm::EPI_WARPS * 32 * sizeof(int);
    const cudaError_t e =
        cudaMemsetAsync(static_cast<uint8_t*>(ws) + flags_off, 0, flags_bytes, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail("cudaMemsetAsync(static GEMM workspace flags)", e);
    return launch_gemm<gemm::kScaleOuter, gemm::kOutBf16>(dyqT, xqT, dw_bf16, wgrad_params(sdyT, sxT, N, K, M), ws,
                                                          kStaticWsBytes, static_cast<cudaStream_t>(stream));
}

fp8_status fp8_gemm_workspace_bytes(size_t* bytes) {
    if (!bytes) return FP8_ERR_NULL;
    int dev = 0;
    fp8_status st = current_device(&dev);
    if (st != FP8_OK) return st;
    // Resident CTA pairs of the GEMM kernels (all variants share one shape).
    int sms = 0, pairs = 0;
    if ((st = sm_count(dev, &sms)) != FP8_OK) return st;
    if ((st = gemm_pairs<gemm::kScaleRowBlock, gemm::kOutBf16, false>(dev, sms, &pairs)) != FP8_OK) return st;
    *bytes = gemm_workspace_bytes(pairs);
    return FP8_OK;
}

fp8_status fp8_get_error(void) {
    unsigned int v = 0;
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail("cudaDeviceSynchronize", e);
    e = cudaMemcpyFromSymbol(&v, fp8blk::g_error_word, sizeof v);
    if (e != cudaSuccess) return cuda_fail("cudaMemcpyFromSymbol", e);
    return static_cast<fp8_status>(v);
}

fp8_status fp8_clear_error(void) {
    const unsigned int zero = 0;
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail("cudaDeviceSynchronize", e);
    e = cudaMemcpyToSymbol(fp8blk::g_error_word, &zero, sizeof zero);
    if (e != cudaSuccess) return cuda_fail("cudaMemcpyToSymbol", e);
    return FP8_OK;
}

const char* fp8_last_cuda_error(void) { return g_detail; }

fp8_status fp8_set_gemm_split_min_work(int64_t units_per_pair) {
    if (units_per_pair < 0) return FP8_ERR_SHAPE;
    g_split_min_units.store(units_per_pair, std::memory_order_relaxed);
    return FP8_OK;
}

fp8_status fp8_set_wait_timeout_ns(uint64_t ns) {
    g_wait_ns.store(ns ? ns : kDefaultWaitNs, std::memory_order_relaxed);
    return FP8_OK;
}

const char* fp8_status_string(fp8_status status) {
    switch (status) {
        case FP8_OK: return "ok";
        case FP8_ERR_NULL: return "a required pointer is NULL";
        case FP8_ERR_SHAPE: return "unsupported shape";
        case FP8_ERR_ALIGN: return "pointer not 16-byte aligned";
        case FP8_ERR_MODE: return "unknown mode";
        case FP8_ERR_CUDA: return "CUDA call or kernel launch failed";
        case FP8_ERR_TIMEOUT: return "a bounded device wait timed out";
    }
    return "unknown status";
}

fp8_status fp8_cast_e4m3_scaled(const float* x, float scale, uint8_t* q, int64_t n, void* stream) {
    if (n < 0) return FP8_ERR_SHAPE;
    if (n == 0) return FP8_OK;
    if (!x || !q) return FP8_ERR_NULL;
    const int64_t blocks = (n + 255) / 256;
    if (blocks > kMaxDim) return FP8_ERR_SHAPE;
    cast_e4m3_scaled_kernel<<<static_cast<unsigned>(blocks), 256, 0, static_cast<cudaStream_t>(stream)>>>(
        x, scale, q, n);
    return last_launch_status("cast launch");
}

fp8_status fp8_selftest_division(unsigned long long* result, void* stream) {
    if (!result) return FP8_ERR_NULL;
    if (!aligned16(result)) return FP8_ERR_ALIGN;
    division_selftest_kernel<<<0x7F7F, 256, 0, static_cast<cudaStream_t>(stream)>>>(result);
    return last_launch_status("division self-test launch");
}

fp8_status fp8_selftest_silu_bf16(uint16_t* out, void* stream) {
    if (!out) return FP8_ERR_NULL;
    if (!aligned16(out)) return FP8_ERR_ALIGN;
    silu_selftest_kernel<<<256, 256, 0, static_cast<cudaStream_t>(stream)>>>(out);
    return last_launch_status("silu self-test launch");
}

fp8_status fp8_selftest_gemm_schedule(int64_t M, int64_t N, int64_t K, int pairs, int split, int32_t* segs,
                                      int64_t max_segs, int64_t* nsegs) {
    if (!segs || !nsegs) return FP8_ERR_NULL;
    if (M <= 0 || N <= 0 || K <= 0 || M % 128 || N % 128 || K % 128 || pairs <= 0 || max_segs < 0 ||
        M > kMaxDim || N > kMaxDim || K > kMaxDim)
        return FP8_ERR_SHAPE;
    gemm::Params p{};
    p.M = static_cast<int>(M);
    p.N = static_cast<int>(N);
    p.K = static_cast<int>(K);
    p.tiles_m = static_cast<int>((M + 2 * gemm::BM - 1) / (2 * gemm::BM));
    p.tiles_n = static_cast<int>((N + gemm::BN - 1) / gemm::BN);
    const int64_t tiles = static_cast<int64_t>(p.tiles_m) * p.tiles_n;
    p.dp_tiles = split ? dp_tiles_for(tiles, pairs, p.K / gemm::BK) : static_cast<int>(tiles);
    const int npairs = p.dp_tiles < tiles ? pairs : static_cast<int>(tiles < pairs ? tiles : pairs);
    const bool split_launch = p.dp_tiles < tiles;
    const int num_kb = p.K / gemm::BK;
    int64_t n = 0;
    for (int q = 0; q < npairs; ++q) {
        gemm::Seg sg;
        for (int idx = 0; split_launch ? gemm::segment<true>(p, q, npairs, idx, sg)
                                       : gemm::segment<false>(p, q, npairs, idx, sg);
             ++idx) {
            if (n >= max_segs) return FP8_ERR_SHAPE;
            int32_t* row = segs + 5 * n;
            row[0] = q;
            row[1] = sg.tile;
            row[2] = sg.kb0;
            row[3] = sg.kb1;
            // the pairs whose partial sums a finalizing segment adds: the
            // first and one past the last (equal when none)
            int32_t first = 0, last = 0;
            if (sg.kb0 == 0 && sg.kb1 < num_kb) {
                const int64_t tile_end =
                    static_cast<int64_t>(sg.tile + 1) * num_kb - static_cast<int64_t>(p.dp_tiles) * num_kb;
                first = q + 1;
                last = q + 1;
                for (int r = q + 1; r < npairs && gemm::split_range_begin(p, r, npairs) < tile_end; ++r)
                    last = r + 1;
            }
            row[4] = (first << 16) | last;
            ++n;
        }
    }
    *nsegs = n;
    return FP8_OK;
}

fp8_status fp8_selftest_stall_next(int which) {
    if (which < 1 || which > 3) return FP8_ERR_MODE;
    g_stall_next.fetch_or(which);
    return FP8_OK;
}

fp8_status fp8_selftest_wait_timeout(void* stream) {
    wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
        g_wait_ns.load(std::memory_order_relaxed), static_cast<unsigned int>(FP8_ERR_TIMEOUT));
    return last_launch_status("wait self-test launch");
}

}  // extern "C"
