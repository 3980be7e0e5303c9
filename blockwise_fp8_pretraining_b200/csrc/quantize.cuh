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
//   quant_tile_kernel    : 128 x 128 tiles staged in shared memory, for
//                          groups along columns (tokens) with transposed
//                          output, for both groupings from one read, and for
//                          128x128 weight blocks (+ transposed codes).
#pragma once

#include "ptx.cuh"

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
// division instead.  copysign keeps the sign of -0 / s.  An exhaustive GPU
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
    __device__ __forceinline__ float operator()(float x) const {
        if (!fast) return __fdiv_rn(x, s);
        const float q0 = x * r;
        const float e = fmaf(-s, q0, x);
        return copysignf(fmaf(e, r, q0), x);
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

enum TileMode : int { kTileColwise = 0, kTileBoth = 1, kTileWeight = 2 };

// One 128 x 128 bf16 tile per block of 256 threads.
//   kTileColwise : s_col[rows/128, cols], q_colT[cols, rows]
//   kTileBoth    : the above plus q_row[rows, cols], s_row[cols/128, rows]
//   kTileWeight  : q_row = codes [rows, cols], s_col = block scales
//                  [rows/128, cols/128], q_colT = transposed codes or NULL
template <int MODE>
__global__ void __launch_bounds__(256, 3) quant_tile_kernel(const uint4* __restrict__ x,
                                                         int64_t rows, int64_t cols,
                                                         uint8_t* __restrict__ q_row,
                                                         float* __restrict__ s_row,
                                                         uint8_t* __restrict__ q_colT,
                                                         float* __restrict__ s_col) {
    __shared__ __align__(16) uint32_t tile[kGroup][kGroup / 2];  // bf16 pairs, 32 KB
    __shared__ float red[8][kGroup];

    const int t = threadIdx.x;
    const int lane = t & 31;
    const int warp = t >> 5;
    const int64_t tiles_c = cols / kGroup;
    const int64_t tr = blockIdx.x / tiles_c;
    const int64_t tc = blockIdx.x - tr * tiles_c;
    const int64_t r0 = tr * kGroup;
    const int64_t c0 = tc * kGroup;

    // Load: thread t owns 16-byte chunk (t % 16) of rows t/16 + 16 i.
    const int chunk = t & 15;
    const int rbase = t >> 4;
    uint4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const int64_t row = r0 + rbase + 16 * i;
        v[i] = __ldg(x + (row * cols + c0) / 8 + chunk);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
        *reinterpret_cast<uint4*>(&tile[rbase + 16 * i][chunk * 4]) = v[i];

    // Row-group amax (16 lanes share a row).
    float ramax[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) ramax[i] = halfwarp_max(amax8(v[i]));

    float block_scale = 0.0f;
    if (MODE == kTileWeight) {
        float a = 0.0f;
#pragma unroll
        for (int i = 0; i < 8; ++i) a = fmaxf(a, ramax[i]);
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 16));
        if (lane == 0) red[0][warp] = a;
    }
    __syncthreads();
    if (MODE == kTileWeight) {
        float a = red[0][0];
#pragma unroll
        for (int w = 1; w < 8; ++w) a = fmaxf(a, red[0][w]);
        block_scale = group_scale(a);
    }

    // Row-layout outputs.
    if (MODE == kTileBoth || MODE == kTileWeight) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int64_t row = r0 + rbase + 16 * i;
            const float sc = (MODE == kTileWeight) ? block_scale : group_scale(ramax[i]);
            *reinterpret_cast<uint2*>(q_row + row * cols + c0 + chunk * 8) = encode8(v[i], sc);
            if (MODE == kTileBoth && chunk == 0) s_row[tc * rows + row] = sc;
        }
        if (MODE == kTileWeight && t == 0) s_col[tr * tiles_c + tc] = block_scale;
    }

    if (MODE == kTileWeight && q_colT == nullptr) return;

    // Column pass: thread owns column pair p (cols 2p, 2p+1) over the 32 rows
    // of quarter qq.
    const int p = t & 63;
    const int qq = t >> 6;
    uint32_t w[32];
    float m0 = 0.0f, m1 = 0.0f;
#pragma unroll
    for (int rr = 0; rr < 32; ++rr) {
        w[rr] = tile[qq * 32 + rr][p];
        m0 = fmaxf(m0, fabsf(bf16_lo(w[rr])));
        m1 = fmaxf(m1, fabsf(bf16_hi(w[rr])));
    }
    float s0 = block_scale, s1 = block_scale;
    if (MODE != kTileWeight) {
        __syncthreads();   // red[] reuse
        red[qq][2 * p] = m0;
        red[qq][2 * p + 1] = m1;
        __syncthreads();
        float a0 = fmaxf(fmaxf(red[0][2 * p], red[1][2 * p]), fmaxf(red[2][2 * p], red[3][2 * p]));
        float a1 = fmaxf(fmaxf(red[0][2 * p + 1], red[1][2 * p + 1]),
                         fmaxf(red[2][2 * p + 1], red[3][2 * p + 1]));
        s0 = group_scale(a0);
        s1 = group_scale(a1);
        if (qq == 0)
            *reinterpret_cast<float2*>(s_col + tr * cols + c0 + 2 * p) = make_float2(s0, s1);
    }

    // Transposed codes: 32 consecutive tokens of columns 2p and 2p+1.
    uint32_t b0[8], b1[8];
    const Quotient q0(s0), q1(s1);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
        const uint32_t wa = w[4 * j], wb = w[4 * j + 1], wc = w[4 * j + 2], wd = w[4 * j + 3];
        if (s0 == 0.0f) {
            b0[j] = 0u;
        } else {
            b0[j] = code2(bf16_lo(wa), bf16_lo(wb), q0) | (code2(bf16_lo(wc), bf16_lo(wd), q0) << 16);
        }
        if (s1 == 0.0f) {
            b1[j] = 0u;
        } else {
            b1[j] = code2(bf16_hi(wa), bf16_hi(wb), q1) | (code2(bf16_hi(wc), bf16_hi(wd), q1) << 16);
        }
    }
    uint8_t* dst0 = q_colT + (c0 + 2 * p) * rows + r0 + qq * 32;
    uint8_t* dst1 = dst0 + rows;
    reinterpret_cast<uint4*>(dst0)[0] = make_uint4(b0[0], b0[1], b0[2], b0[3]);
    reinterpret_cast<uint4*>(dst0)[1] = make_uint4(b0[4], b0[5], b0[6], b0[7]);
    reinterpret_cast<uint4*>(dst1)[0] = make_uint4(b1[0], b1[1], b1[2], b1[3]);
    reinterpret_cast<uint4*>(dst1)[1] = make_uint4(b1[4], b1[5], b1[6], b1[7]);
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
