// RMSNorm for the fused norm quantizer: the input of the Qwen3-1.7B
// configuration's attention and feed-forward blocks (Puro-2B-Base model
// card, model property table; exported as Qwen3ForCausalLM) is
//
//   r    = 1 / sqrt(mean_k x[k]^2 + eps)          per row, in FP32
//   y[k] = bf16(gamma[k] * bf16(fp32(x[k] * r)))  each rounding to nearest even
//
// (normalize in FP32, round to BF16, scale by the BF16 weight), and the
// linear layers quantize y.  The fused quantizer applies the second line to
// each tile as it arrives and quantizes the result, so y is never written.
// r comes from rmsnorm_rstd_kernel (or from the caller): given the same r,
// the codes equal those of quantizing the unfused y bit for bit.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

#include "ptx.cuh"
#include "swiglu.cuh"

namespace fp8blk {

// r per row of x [rows, cols] (cols a multiple of 8): one warp per row;
// the squares of bfloat16 values are exact in FP64 and their sum is taken
// in FP64 (relative error below 2^-40 for these lengths, so r, rounded once
// from FP64 to FP32, is the correctly rounded value except within that
// distance of a rounding midpoint, where it may be its neighbour).
__global__ void __launch_bounds__(256) rmsnorm_rstd_kernel(const uint4* __restrict__ x, int64_t rows,
                                                           int64_t cols, float eps, float* __restrict__ r) {
    griddep_wait();
    const int lane = threadIdx.x & 31;
    const int64_t row = static_cast<int64_t>(blockIdx.x) * 8 + (threadIdx.x >> 5);
    if (row < rows) {
        const uint4* xr = x + row * (cols / 8);
        double sum = 0.0;
#pragma unroll 8
        for (int64_t c = lane; c < cols / 8; c += 32) {
            const uint4 v = __ldg(xr + c);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const double a = __uint_as_float(w[i] << 16), b = __uint_as_float(w[i] & 0xFFFF0000u);
                sum = fma(a, a, sum);
                sum = fma(b, b, sum);
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
        if (lane == 0) r[row] = static_cast<float>(1.0 / sqrt(sum / static_cast<double>(cols) + static_cast<double>(eps)));
    }
    griddep_launch_dependents();
}

// y for the 8 elements of one 16-byte chunk: x the chunk, r its row's r,
// g the 8 matching gamma values.
__device__ __forceinline__ uint4 rmsnorm8(const uint4& x, float r, const uint4& g) {
    const uint32_t* xw = reinterpret_cast<const uint32_t*>(&x);
    const uint32_t* gw = reinterpret_cast<const uint32_t*>(&g);
    uint32_t out[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float t0 = __fmul_rn(__uint_as_float(xw[i] << 16), r);
        const float t1 = __fmul_rn(__uint_as_float(xw[i] & 0xFFFF0000u), r);
        const __nv_bfloat162 tb = __floats2bfloat162_rn(t0, t1);
        const uint32_t tw = *reinterpret_cast<const uint32_t*>(&tb);
        out[i] = bf16_product(__uint_as_float(gw[i] << 16), __uint_as_float(tw << 16)) |
                 (bf16_product(__uint_as_float(gw[i] & 0xFFFF0000u), __uint_as_float(tw & 0xFFFF0000u)) << 16);
    }
    return make_uint4(out[0], out[1], out[2], out[3]);
}

}  // namespace fp8blk
