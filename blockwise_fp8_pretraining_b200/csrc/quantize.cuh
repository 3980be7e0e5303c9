// Blockwise E4M3 quantizers (HBM-bound).
//
// Definition (fixed by this library; the Puro-2B model card's training-setup
// paragraph names only "blockwise E4M3"): per group, amax = max |x|,
// s = amax / 448 in IEEE float32, code = E4M3FN round-to-nearest-even of the
// IEEE float32 quotient x / s with saturation at +-448, sign kept; s == 0
// gives code 0.
//
//   quant_rowwise_kernel : 1x128 groups along rows.  Each half-warp owns one
//                          group per step (16 lanes x 16 bytes), reduces amax
//                          with 4 shuffles and writes 8 code bytes per lane.
//   quant_tile_kernel    : persistent, 128 x 128 tiles fed by TMA into a
//                          double buffer, for groups along columns (tokens)
//                          with transposed output, for both groupings from
//                          one read, and for 128x128 weight blocks (+
//                          transposed codes); codes leave by TMA stores.
#pragma once

#include <cuda_bf16.h>

#include "ptx.cuh"
#include "rmsnorm.cuh"
#include "swiglu.cuh"

namespace fp8blk {

constexpr int kGroup = 128;

// |x| maximum over the 8 bf16 values of a 16-byte chunk.
__device__ __forceinline__ float amax8(const uint4& v) {
    float a = fmaxf(fabsf(bf16_lo(v.x)), fabsf(bf16_hi(v.x)));
    a = fmaxf(a, fmaxf(fabsf(bf16_lo(v.y)), fabsf(bf16_hi(v.y))));
    a = fmaxf(a, fmaxf(fabsf(bf16_lo(v.z)), fabsf(bf16_hi(v.z))));
    a = fmaxf(a, fmaxf(fabsf(bf16_lo(v.w)), fabsf(bf16_hi(v.w))));
    return a;
}

__device__ __forceinline__ float group_scale(float amax) { return __fdiv_rn(amax, 448.0f); }

// x / s correctly rounded (IEEE float32, round-to-nearest-even) for one
// divisor s shared by a whole group, without a division per element.
// Markstein's scheme (P. Markstein, "Computation of elementary functions on
// the IBM RISC System/6000 processor", IBM J. Res. Dev. 34(1), 1990): with
// r = RN(1/s) and q0 = RN(x r), the remainder e = x - s q0 is exact in one
// FMA and RN(q0 + e r) is the correctly rounded quotient.  The remainder is
// exact only while it stays a normal float, so divisors outside
// [2^-100, 2^100] (groups of tiny or huge bf16 values) take the IEEE
// division instead.  The remainder is formed negated, e' = s q0 - x, and
// the result as q0 - e' r: the same values, and the signed zeros come out
// right (for x = -0: q0 = -0, e' = +0, -e' r + q0 = -0).  An exhaustive GPU
// check (fp8_selftest_division) compares the E4M3 codes and the quotient
// bits of both paths for every (bf16 amax, bf16 x) pair a group can hold.
struct Quotient {
    float s, r;
    bool fast;
    __device__ __forceinline__ explicit Quotient(float s_) : s(s_), r(0.0f) {
#ifdef __CUDA_ARCH__
        r = __frcp_rn(s_);
#endif
        fast = (s_ >= 0x1p-100f) && (s_ <= 0x1p100f);
    }
    // With the reciprocal RN(1/s) already at hand.
    __device__ __forceinline__ Quotient(float s_, float r_)
        : s(s_), r(r_), fast((s_ >= 0x1p-100f) && (s_ <= 0x1p100f)) {}
    __device__ __forceinline__ float operator()(float x) const {
        if (!fast) return __fdiv_rn(x, s);
        const float q0 = x * r;
        const float e = fmaf(s, q0, -x);       // -(x - s q0), exact
        return fmaf(-e, r, q0);
    }
};

// Codes of two values of a group (s > 0): quotient, then E4M3 RNE.
__device__ __forceinline__ uint32_t code2(float lo, float hi, const Quotient& q) {
    return cvt_e4m3x2(q(lo), q(hi));
}

// Codes of the 8 bf16 values of a chunk, packed in memory order.
__device__ __forceinline__ uint2 encode8(const uint4& v, float s) {
    if (s == 0.0f) return make_uint2(0u, 0u);
    const Quotient q(s);
    uint2 r;
    r.x = code2(bf16_lo(v.x), bf16_hi(v.x), q) | (code2(bf16_lo(v.y), bf16_hi(v.y), q) << 16);
    r.y = code2(bf16_lo(v.z), bf16_hi(v.z), q) | (code2(bf16_lo(v.w), bf16_hi(v.w), q) << 16);
    return r;
}

// The two bf16 of a 32-bit word (memory order: low half first) as floats.
__device__ __forceinline__ float2 unpack_bf16x2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

// max |x| over the 8 bf16 of a chunk, with packed bf16 min/max (exact).
__device__ __forceinline__ float amax8_packed(const uint4& v) {
    __nv_bfloat162 m = __habs2(*reinterpret_cast<const __nv_bfloat162*>(&v.x));
    m = __hmax2(m, __habs2(*reinterpret_cast<const __nv_bfloat162*>(&v.y)));
    m = __hmax2(m, __habs2(*reinterpret_cast<const __nv_bfloat162*>(&v.z)));
    m = __hmax2(m, __habs2(*reinterpret_cast<const __nv_bfloat162*>(&v.w)));
    const uint32_t u = *reinterpret_cast<const uint32_t*>(&m);
    return fmaxf(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
}

// Quotients of two values by two group scales at once (the Quotient scheme
// above on FP32x2 pairs); both scales must be in the fast range.
struct QuotientPair {
    float2 r, s2;
    __device__ __forceinline__ QuotientPair(const Quotient& a, const Quotient& b)
        : r(make_float2(a.r, b.r)), s2(make_float2(a.s, b.s)) {}
    __device__ __forceinline__ QuotientPair(float s0, float r0, float s1, float r1)
        : r(make_float2(r0, r1)), s2(make_float2(s0, s1)) {}
    // E4M3 codes of the two bf16 of w (first in the low byte).
    __device__ __forceinline__ uint32_t codes(uint32_t w) const {
        const float2 x = unpack_bf16x2(w);
        const float2 q0 = __fmul2_rn(x, r);
        const float2 e = __ffma2_rn(s2, q0, make_float2(-x.x, -x.y));   // s q0 - x
        const float2 q = __ffma2_rn(make_float2(-e.x, -e.y), r, q0);    // q0 - e r
        return cvt_e4m3x2(q.x, q.y);
    }
};

// Codes of the two bf16 of w with scales s0 (low) and s1 (high), any
// scales (zero gives code 0; scales outside the fast range divide).
__device__ __noinline__ uint32_t codes_pair_general(uint32_t w, const Quotient& a, const Quotient& b) {
    const float2 x = unpack_bf16x2(w);
    const float q0 = (a.s == 0.0f) ? 0.0f : a(x.x);
    const float q1 = (b.s == 0.0f) ? 0.0f : b(x.y);
    return cvt_e4m3x2(q0, q1);
}

__device__ __forceinline__ float halfwarp_max(float a) {
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 8));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 4));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
    a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
    return a;
}

// ------------------------------------------------------------- row-wise 1x128

// x: [rows, cols] bf16 as 16-byte chunks; a group ("unit") u covers elements
// [128u, 128u + 128), i.e. row u / groups, group u % groups.
template <int UNROLL>
__global__ void __launch_bounds__(256) quant_rowwise_kernel(const uint4* __restrict__ x,
                                                            int64_t units, int64_t rows,
                                                            int64_t groups,
                                                            uint2* __restrict__ q,
                                                            float* __restrict__ s) {
    const int lane = threadIdx.x & 31;
    const int sub = lane & 15;
    const int half = lane >> 4;
    const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
    griddep_wait();                    // inputs of the preceding kernel are complete
    for (int64_t base = warp * (2 * UNROLL); base < units; base += nwarps * (2 * UNROLL)) {
        uint4 v[UNROLL];
#pragma unroll
        for (int i = 0; i < UNROLL; ++i) {
            const int64_t u = base + 2 * i + half;
            v[i] = (u < units) ? __ldg(x + u * 16 + sub) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int i = 0; i < UNROLL; ++i) {
            const int64_t u = base + 2 * i + half;
            const float sc = group_scale(halfwarp_max(amax8(v[i])));
            if (u < units) {
                q[u * 16 + sub] = encode8(v[i], sc);
                if (sub == 0) {
                    const int64_t r = u / groups;
                    s[(u - r * groups) * rows + r] = sc;
                }
            }
        }
    }
}

// ---------------------------------------------------------------- 128x128 tiles

// kTileRowwise is used with the SwiGLU and RMSNorm input stages only;
// plain row-wise groups have the lighter quant_rowwise_kernel.
enum TileMode : int { kTileColwise = 0, kTileBoth = 1, kTileWeight = 2, kTileRowwise = 3 };
// What the tile kernel quantizes: its input as it is, the SwiGLU product of
// a gate_up activation, or the RMSNorm output y of its input (with r per
// row and gamma per column given).
enum TileProducer : int { kProdPlain = 0, kProdSwiglu = 1, kProdNorm = 2 };

namespace tile {
constexpr int THREADS = 256;
constexpr int BOX_BYTES = kGroup * 128;              // 128 rows x 64 bf16, 128-byte swizzle
constexpr int OUT_BYTES = kGroup * kGroup;           // one tile of codes
// Shared-memory layout.  Plain tiles: two tile buffers, separate staging of
// the two code tiles, two blocks per SM.  SWIGLU: one buffer holding the
// gate tile (two boxes) and then the up tile (two boxes); h is written over
// the gate tile, and the up tile, dead once h is formed, stages the codes;
// three blocks per SM overlap each other's loads.
template <bool SWIGLU>
struct Layout {
    static constexpr int NBUF = SWIGLU ? 1 : 2;
    static constexpr int IN_BYTES = (SWIGLU ? 4 : 2) * BOX_BYTES;
    static constexpr int OFF_IN0 = 0;
    static constexpr int OFF_IN1 = OFF_IN0 + (NBUF - 1) * IN_BYTES;
    static constexpr int OFF_ROW = SWIGLU ? 2 * BOX_BYTES : OFF_IN1 + IN_BYTES;   // row-layout codes
    static constexpr int OFF_COL = OFF_ROW + OUT_BYTES;         // transposed codes, 128-byte swizzle
    static constexpr int OFF_RED = SWIGLU ? IN_BYTES : OFF_COL + OUT_BYTES;   // 4 x 128 partial maxima
    static constexpr int OFF_COLS = OFF_RED + 4 * kGroup * 4;   // 128 column scales, then reciprocals
    static constexpr int OFF_BARS = OFF_COLS + 2 * kGroup * 4;
    static constexpr int SMEM_BYTES = OFF_BARS + 2 * 8 + 16 + 1024;   // + alignment slack
    static constexpr int BLOCKS_PER_SM = SWIGLU ? 3 : 2;
    static_assert(OFF_COL + OUT_BYTES <= (SWIGLU ? IN_BYTES : OFF_RED), "staging inside its region");
    static_assert(OFF_ROW % 1024 == 0 && OFF_COL % 1024 == 0 && BOX_BYTES % 1024 == 0,
                  "swizzled tiles must be 1024-byte aligned");
    static_assert(BLOCKS_PER_SM * SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

// Byte offset of 16-byte chunk `chunk` of row `r` in a 128-byte-swizzled
// tile of 128-byte rows (the TMA 128B swizzle pattern).
__device__ __forceinline__ int sw128(int r, int chunk) { return r * 128 + ((chunk ^ (r & 7)) << 4); }
}  // namespace tile

// Persistent quantizer of 128 x 128 bf16 tiles, two tile buffers per block
// fed by TMA, outputs staged in shared memory and written by TMA stores.
//   kTileColwise : groups along columns (tokens): s_col[rows/128, cols],
//                  codes q_colT[cols, rows]
//   kTileBoth    : the above plus groups along rows: q_row[rows, cols],
//                  s_row[cols/128, rows], from the same read
//   kTileWeight  : 128 x 128 blocks: q_row = codes [rows, cols], s_col =
//                  block scales [rows/128, cols/128], transposed codes
//                  through tmQT when has_qT
//   kTileRowwise : groups along rows only (SwiGLU and RMSNorm producers)
// SWIGLU: the quantized tensor is h = bf16(bf16(silu(gate)) * up) of a
// gate_up activation [rows, 2 * cols] (gate = columns [0, cols), up =
// [cols, 2 * cols)); each tile buffer receives the gate and the up tile of
// the same position, and h is formed in place before the passes.
// Maps (all 128-byte swizzle): tmX bf16 [rows, cols] (SWIGLU: [rows,
//   2 * cols]), box 64 x 128; tmQ u8 [rows, cols], box 128 x 128; tmQT u8
//   [cols, rows], box 128 x 128.
// Row pass: lanes l and l + 16 of warp w share row 16 w + l % 16, 64 columns each.
// Column pass: thread owns columns 2p, 2p+1 over the 32 rows of quarter qq.
template <int MODE, int PROD>
__global__ void __launch_bounds__(tile::THREADS, tile::Layout<PROD == kProdSwiglu>::BLOCKS_PER_SM)
    quant_tile_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmQT, int64_t rows, int64_t cols,
                      float* __restrict__ s_row, float* __restrict__ s_col, int has_qT,
                      uint64_t wait_ns, uint32_t stall_tx, const float* __restrict__ norm_r,
                      const __nv_bfloat16* __restrict__ norm_gamma) {
    constexpr bool SWIGLU = PROD == kProdSwiglu;
    using L = tile::Layout<SWIGLU>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_u32(smem);
    float* red = reinterpret_cast<float*>(smem + L::OFF_RED);
    const uint32_t bar0 = sbase + L::OFF_BARS;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::OFF_BARS + 16);

    const int t = threadIdx.x;
    const int lane = t & 31;
    const int warp = t >> 5;
    const int64_t tiles_c = cols / kGroup;
    const int64_t total = (rows / kGroup) * tiles_c;
    const bool want_rows = (MODE != kTileColwise);
    const bool want_cols = (MODE == kTileColwise || MODE == kTileBoth) || (MODE == kTileWeight && has_qT);

    // stall_tx (test only, 0 normally): extra bytes the block's first load
    // barrier expects, so that its wait runs out
    auto issue_load = [&](int64_t tl, int j) {
        const uint32_t dst = sbase + (j ? L::OFF_IN1 : L::OFF_IN0);
        const int32_t x = static_cast<int32_t>((tl % tiles_c) * kGroup);
        const int32_t y = static_cast<int32_t>((tl / tiles_c) * kGroup);
        mbar_arrive_expect_tx(bar0 + 8 * j, L::IN_BYTES + (tl == blockIdx.x ? stall_tx : 0u));
        tma_load_2d(dst, &tmX, x, y, bar0 + 8 * j);
        tma_load_2d(dst + tile::BOX_BYTES, &tmX, x + 64, y, bar0 + 8 * j);
        if (SWIGLU) {                  // the up tile, cols columns to the right
            const int32_t xu = x + static_cast<int32_t>(cols);
            tma_load_2d(dst + 2 * tile::BOX_BYTES, &tmX, xu, y, bar0 + 8 * j);
            tma_load_2d(dst + 3 * tile::BOX_BYTES, &tmX, xu + 64, y, bar0 + 8 * j);
        }
    };

    if (t == 0) {                      // set-up that reads nothing the preceding kernel writes
        mbar_init(bar0, 1);
        mbar_init(bar0 + 8, 1);
        *abort_flag = 0;
        fence_barrier_init();
        prefetch_tensormap(&tmX);
        prefetch_tensormap(&tmQ);
        prefetch_tensormap(&tmQT);
    }
    griddep_wait();                    // inputs of the preceding kernel are complete
    if (t == 0) {
        for (int j = 0; j < L::NBUF; ++j) {
            const int64_t tl = blockIdx.x + static_cast<int64_t>(j) * gridDim.x;
            if (tl < total) issue_load(tl, j);
        }
    }
    __syncthreads();

    // The two passes run side by side in two groups of four warps.
    // Row group (warps 0-3): thread t owns row t of the tile and all 128 of
    //   its columns (16 chunks of 8 bf16 in registers), so a 1x128 group needs
    //   no exchange with other threads.
    // Column group (warps 4-7): warp 4 + cw, lane l owns columns 2 l and
    //   2 l + 1 of box (cw & 1) over rows 64 (cw >> 1) .. + 63, read as one
    //   bf16 pair per row; a warp reads whole 128-byte rows of its box (no
    //   bank conflicts).  The two row halves of a column combine their maxima
    //   through shared memory and one named barrier of the column group.
    //   Codes pack along the tokens directly (four rows per word).
    const bool row_group = warp < 4;
    const int cw = warp - 4;
    const int cbox = cw & 1, chalf = cw >> 1;
    const int cpair = cbox * 32 + lane;            // column pair within the tile
    // Byte offset in a tile buffer of row 64 chalf + 8 i + u (u = 0..7) of
    // the column thread's pair is coff[u] + 1024 i: the swizzle depends on
    // the row only through r % 8.
    int coff[8];
#pragma unroll
    for (int u = 0; u < 8; ++u)
        coff[u] = cbox * tile::BOX_BYTES + (64 * chalf + u) * 128 + (((lane >> 2) ^ u) << 4) + (lane & 3) * 4;
    uint32_t* colx = reinterpret_cast<uint32_t*>(smem + L::OFF_COLS);   // [2 halves][64 pairs] partial maxima

    int i = 0;
    for (int64_t tl = blockIdx.x; tl < total; tl += gridDim.x, ++i) {
        const int b = i % L::NBUF;
        const int64_t tr = tl / tiles_c, tc = tl - tr * tiles_c;
        const int64_t r0 = tr * kGroup, c0 = tc * kGroup;
        const uint8_t* tin = smem + (b ? L::OFF_IN1 : L::OFF_IN0);
        bool ok = mbar_wait(bar0 + 8 * b, (i / L::NBUF) & 1, abort_flag, wait_ns, kErrTimeout);
        if (t == 0) bulk_wait_group_read0();         // previous tile's stores have read the staging
        if (__syncthreads_or(!ok)) break;

        if (SWIGLU) {
            // ---- h over the gate tile (same swizzled layout as the up tile).
            // Thread t forms chunks t + 256 j (8 elements each).  Elements
            // whose silu rounding the FP32 path cannot decide (a fraction of
            // a percent) keep their g and a bit in slow_bits; afterwards each
            // warp deals its own out to its lanes for the FP64 path, so the
            // hot loop has no call in it and no lane runs FP64 alone.
            uint8_t* gbuf = smem + (b ? L::OFF_IN1 : L::OFF_IN0);
            uint64_t slow_bits = 0;              // bit 8 j + e: element e of chunk t + 256 j
#pragma unroll 2
            for (int j = 0; j < 2 * tile::BOX_BYTES / 16 / tile::THREADS; ++j) {
                const int c = t + j * tile::THREADS;
                const uint4 g = *reinterpret_cast<const uint4*>(gbuf + 16 * c);
                const uint4 u = *reinterpret_cast<const uint4*>(gbuf + 2 * tile::BOX_BYTES + 16 * c);
                uint32_t slow = 0;
                *reinterpret_cast<uint4*>(gbuf + 16 * c) = swiglu8_fast(g, u, slow);
                slow_bits |= static_cast<uint64_t>(slow) << (8 * j);
            }
            __syncwarp();
            const int cnt = __popcll(slow_bits);
            int off = cnt;                       // inclusive, then exclusive, scan over the lanes
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int v = __shfl_up_sync(0xffffffffu, off, d);
                if (lane >= d) off += v;
            }
            const int n_slow = __shfl_sync(0xffffffffu, off, 31);
            off -= cnt;
            for (int base = 0; base < n_slow; base += 32) {
                const int k = base + lane;
                int owner = 0;                   // the last lane whose range starts at or before k
#pragma unroll
                for (int step = 16; step > 0; step >>= 1) {
                    const int o = __shfl_sync(0xffffffffu, off, owner + step);
                    if (o <= k) owner += step;
                }
                const uint32_t m_lo = __shfl_sync(0xffffffffu, static_cast<uint32_t>(slow_bits), owner);
                const uint32_t m_hi = __shfl_sync(0xffffffffu, static_cast<uint32_t>(slow_bits >> 32), owner);
                const int r = k - __shfl_sync(0xffffffffu, off, owner);
                if (k < n_slow) {
                    uint64_t m = (static_cast<uint64_t>(m_hi) << 32) | m_lo;
                    for (int i2 = 0; i2 < r; ++i2) m &= m - 1;     // drop the owner's first r elements
                    const int bit = __ffsll(static_cast<long long>(m)) - 1;
                    const int c = warp * 32 + owner + (bit >> 3) * tile::THREADS;
                    swiglu_fix(reinterpret_cast<uint16_t*>(gbuf),
                               reinterpret_cast<const uint16_t*>(gbuf + 2 * tile::BOX_BYTES), 8 * c + (bit & 7));
                }
            }
            __syncthreads();
        }

        if (PROD == kProdNorm) {
            // ---- y = bf16(gamma * bf16(x * r)) over the tile, in place.
            // Chunk c of the buffer: box c / 1024, row (c / 8) % 128, and
            // 16-byte chunk (c % 8) ^ (row % 8) of that box row.
            uint8_t* xbuf = smem + (b ? L::OFF_IN1 : L::OFF_IN0);
#pragma unroll 2
            for (int j = 0; j < 2 * tile::BOX_BYTES / 16 / tile::THREADS; ++j) {
                const int c = t + j * tile::THREADS;
                const int row = (c >> 3) & 127;
                const int col = (c >> 10) * 64 + (((c & 7) ^ (row & 7)) << 3);
                const float rr = __ldg(norm_r + r0 + row);
                const uint4 gv = __ldg(reinterpret_cast<const uint4*>(norm_gamma + c0 + col));
                *reinterpret_cast<uint4*>(xbuf + 16 * c) = rmsnorm8(*reinterpret_cast<const uint4*>(xbuf + 16 * c), rr, gv);
            }
            __syncthreads();
        }

        // In weight mode both groups need the block's scale: the row group's
        // warp maxima meet at named barrier 2 (all 256 threads; each group
        // reaches it from its own branch).
        if (row_group) {
            // ---- row pass: codes of the thread's row into the row-layout staging
            uint4 v[16];                 // the row: chunk k of box k / 8 at chunk k % 8
            float sc = 0.0f;
            if (want_rows || MODE == kTileWeight) {
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    v[k] = *reinterpret_cast<const uint4*>(tin + (k >> 3) * tile::BOX_BYTES + t * 128 +
                                                           (((k & 7) ^ (t & 7)) << 4));
                float m[4];
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    m[q] = fmaxf(fmaxf(amax8_packed(v[4 * q]), amax8_packed(v[4 * q + 1])),
                                 fmaxf(amax8_packed(v[4 * q + 2]), amax8_packed(v[4 * q + 3])));
                float a = fmaxf(fmaxf(m[0], m[1]), fmaxf(m[2], m[3]));
                if (MODE == kTileWeight) {
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
                    if (lane == 0) red[warp] = a;
                    named_bar_sync(2, tile::THREADS);
                    sc = group_scale(fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3])));
                    if (t == 0) s_col[tr * tiles_c + tc] = sc;
                } else {
                    sc = group_scale(a);
                    s_row[tc * rows + r0 + t] = sc;
                }
            }
            if (want_rows) {
                uint8_t* orow = smem + L::OFF_ROW + t * 128;
                const Quotient q(sc);
                if (q.fast) {
                    const QuotientPair qp(q, q);
#pragma unroll
                    for (int j = 0; j < 8; ++j) {       // output chunk j: input chunks 2j, 2j+1
                        const uint4 x0 = v[2 * j], x1 = v[2 * j + 1];
                        const uint4 o = make_uint4(qp.codes(x0.x) | (qp.codes(x0.y) << 16),
                                                   qp.codes(x0.z) | (qp.codes(x0.w) << 16),
                                                   qp.codes(x1.x) | (qp.codes(x1.y) << 16),
                                                   qp.codes(x1.z) | (qp.codes(x1.w) << 16));
                        *reinterpret_cast<uint4*>(orow + ((j ^ (t & 7)) << 4)) = o;
                    }
                } else {
#pragma unroll
                    for (int j = 0; j < 8; ++j) {
                        const uint4 x0 = v[2 * j], x1 = v[2 * j + 1];
                        const uint4 o = make_uint4(
                            codes_pair_general(x0.x, q, q) | (codes_pair_general(x0.y, q, q) << 16),
                            codes_pair_general(x0.z, q, q) | (codes_pair_general(x0.w, q, q) << 16),
                            codes_pair_general(x1.x, q, q) | (codes_pair_general(x1.y, q, q) << 16),
                            codes_pair_general(x1.z, q, q) | (codes_pair_general(x1.w, q, q) << 16));
                        *reinterpret_cast<uint4*>(orow + ((j ^ (t & 7)) << 4)) = o;
                    }
                }
            }
        } else {
            // ---- column pass: codes of the two columns along the tokens
            float s0 = 0.0f, s1 = 0.0f;
            if (MODE == kTileWeight) {
                named_bar_sync(2, tile::THREADS);
                s0 = s1 = group_scale(fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3])));
            }
            uint32_t w[64];              // the pair's two values of row 64 chalf + rr
            if (want_cols) {
#pragma unroll
                for (int rr = 0; rr < 64; ++rr)
                    w[rr] = *reinterpret_cast<const uint32_t*>(tin + coff[rr & 7] + (rr >> 3) * 1024);
            }
            if (MODE != kTileWeight && want_cols) {
                __nv_bfloat162 mq[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) mq[u] = __float2bfloat162_rn(0.0f);
#pragma unroll
                for (int rr = 0; rr < 64; ++rr)
                    mq[rr & 3] = __hmax2(mq[rr & 3], __habs2(*reinterpret_cast<const __nv_bfloat162*>(&w[rr])));
                const __nv_bfloat162 m2 = __hmax2(__hmax2(mq[0], mq[1]), __hmax2(mq[2], mq[3]));
                colx[chalf * 64 + cpair] = *reinterpret_cast<const uint32_t*>(&m2);
                named_bar_sync(1, 128);             // the other row half's maxima are in
                const uint32_t other = colx[(chalf ^ 1) * 64 + cpair];
                const __nv_bfloat162 mm = __hmax2(m2, *reinterpret_cast<const __nv_bfloat162*>(&other));
                const uint32_t mu = *reinterpret_cast<const uint32_t*>(&mm);
                s0 = group_scale(__uint_as_float(mu << 16));
                s1 = group_scale(__uint_as_float(mu & 0xFFFF0000u));
                if (chalf == 0) *reinterpret_cast<float2*>(s_col + tr * cols + c0 + 2 * cpair) = make_float2(s0, s1);
            }
            if (want_cols) {
                const Quotient q0(s0), q1(s1);
                const bool fast = q0.fast && q1.fast;
                const QuotientPair qa(q0, q0), qb(q1, q1);
                uint8_t* ocol = smem + L::OFF_COL;
                const int ca = 2 * cpair, cb2 = 2 * cpair + 1;   // the two columns = rows of the transposed tile
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    // words 4j .. 4j+3 of each column: rows 16 j + 4 k .. + 3, first row lowest
                    uint32_t oa[4], ob[4];
#pragma unroll
                    for (int k = 0; k < 4; ++k) {
                        const int r = 16 * j + 4 * k;
                        const uint32_t w0 = w[r], w1 = w[r + 1], w2 = w[r + 2], w3 = w[r + 3];
                        const uint32_t la = (w0 & 0xFFFFu) | (w1 << 16), lb = (w2 & 0xFFFFu) | (w3 << 16);
                        const uint32_t ha = (w0 >> 16) | (w1 & 0xFFFF0000u), hb = (w2 >> 16) | (w3 & 0xFFFF0000u);
                        if (fast) {
                            oa[k] = qa.codes(la) | (qa.codes(lb) << 16);
                            ob[k] = qb.codes(ha) | (qb.codes(hb) << 16);
                        } else {
                            oa[k] = codes_pair_general(la, q0, q0) | (codes_pair_general(lb, q0, q0) << 16);
                            ob[k] = codes_pair_general(ha, q1, q1) | (codes_pair_general(hb, q1, q1) << 16);
                        }
                    }
                    const int chunk = 4 * chalf + j;
                    *reinterpret_cast<uint4*>(ocol + ca * 128 + ((chunk ^ (ca & 7)) << 4)) =
                        make_uint4(oa[0], oa[1], oa[2], oa[3]);
                    *reinterpret_cast<uint4*>(ocol + cb2 * 128 + ((chunk ^ (cb2 & 7)) << 4)) =
                        make_uint4(ob[0], ob[1], ob[2], ob[3]);
                }
            }
        }

        // ---- stores of both code tiles, then the load NBUF tiles ahead
        fence_proxy_async_shared();
        __syncthreads();
        if (t == 0) {
            if (want_rows)
                tma_store_2d(&tmQ, sbase + L::OFF_ROW, static_cast<int32_t>(c0), static_cast<int32_t>(r0));
            if (want_cols)
                tma_store_2d(&tmQT, sbase + L::OFF_COL, static_cast<int32_t>(r0), static_cast<int32_t>(c0));
            bulk_commit_group();
            const int64_t nxt = tl + L::NBUF * static_cast<int64_t>(gridDim.x);
            if (nxt < total) {
                if (SWIGLU) bulk_wait_group_read0();    // the codes are staged in the buffer's up half
                issue_load(nxt, b);
            }
        }
    }
    griddep_launch_dependents();
    if (t == 0) {
        if (*abort_flag) {
            // let loads already requested land before the block exits
            for (int j = 0; j < L::NBUF; ++j) {
                const int64_t tl = blockIdx.x + static_cast<int64_t>(i + j) * gridDim.x;
                if (tl < total)
                    drain_wait(bar0 + 8 * ((i + j) % L::NBUF), ((i + j) / L::NBUF) & 1, wait_ns);
            }
        }
        bulk_wait_group0();
    }
}

// ---------------------------------------------------------------- test support

__global__ void cast_e4m3_scaled_kernel(const float* __restrict__ x, float scale,
                                        uint8_t* __restrict__ q, int64_t n) {
    const int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    if (i < n) q[i] = (scale == 0.0f) ? 0 : static_cast<uint8_t>(cvt_e4m3x2(__fdiv_rn(x[i], scale), 0.0f) & 0xFFu);
}

// Every positive finite bf16 amax (one block each) against every bf16 x with
// |x| <= amax: E4M3 code and quotient bits of the group path (Quotient)
// versus the IEEE division.  result[0] += code mismatches, result[1] = first
// code mismatch (amax bits << 16 | x bits), result[2] += quotient-bit
// mismatches with |x / s| >= 2^-12 (where a code can be nonzero), result[3]
// = first such mismatch, result[4] += quotient-bit mismatches below 2^-12.
__global__ void __launch_bounds__(256) division_selftest_kernel(unsigned long long* result) {
    const uint32_t abits = blockIdx.x + 1u;                 // 0x0001 .. 0x7F7F
    const float amax = __uint_as_float(abits << 16);
    const float s = group_scale(amax);
    const Quotient q(s);
    unsigned long long bad_code = 0, bad_bits = 0, bad_tiny = 0;
    uint32_t first = 0, first_bits = 0;
    for (uint32_t xb = threadIdx.x; xb < 65536u; xb += blockDim.x) {
        const float x = __uint_as_float(xb << 16);
        if (!(fabsf(x) <= amax)) continue;
        const float fast = q(x);
        const float ref = __fdiv_rn(x, s);
        if ((cvt_e4m3x2(fast, 0.0f) & 0xFFu) != (cvt_e4m3x2(ref, 0.0f) & 0xFFu)) {
            if (bad_code == 0) first = (abits << 16) | xb;
            ++bad_code;
        }
        if (__float_as_uint(fast) != __float_as_uint(ref)) {
            if (fabsf(ref) >= 0x1p-12f) {
                if (bad_bits == 0) first_bits = (abits << 16) | xb;
                ++bad_bits;
            } else {
                ++bad_tiny;
            }
        }
    }
    if (bad_code && atomicAdd(&result[0], bad_code) == 0) result[1] = first;
    if (bad_bits && atomicAdd(&result[2], bad_bits) == 0) result[3] = first_bits;
    if (bad_tiny) atomicAdd(&result[4], bad_tiny);
}

// A wait on a barrier that nothing completes: runs into the time limit.
__global__ void wait_timeout_kernel(uint64_t limit_ns, unsigned int code) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bar), 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, &abort_flag, limit_ns, code);
    __syncthreads();
}

}  // namespace fp8blk
