// SwiGLU product in BF16 for the fused producer of the down projection's
// input: h = bf16(bf16(silu(g)) * u), each rounding to nearest even.
//
// The feed-forward block of the Qwen3-1.7B configuration (Puro-2B-Base model
// card, model property table) is a gated SiLU unit, H = silu(gate) * up, and
// activations stay in BF16 (model card, training-setup paragraph), so the
// unfused path rounds silu(g) to BF16 and then the product.  The fused
// quantizer computes h in shared memory from the gate_up tile and quantizes
// it without writing H to memory; its codes must equal those of quantizing
// the unfused H, so both roundings have to be the correctly rounded ones.
//
// silu(g) for a bfloat16 g is rounded once, correctly, to bfloat16:
//   * 2^-20 <= |g| <= 80: FP32 evaluation g / (1 + e) with e = __expf(-g)
//     and the fast division __fdividef.  __expf is within 2 + 1.173 |g|
//     units in the last place (CUDA's documented bound for the intrinsic),
//     __fdividef within 2, and 1 + e rounds once, so the quotient is within
//     (5 + 1.173 |g|) * 2^-23 of silu(g), relative; a float32 unit in the
//     last place at the result is at least 2^-24 of it, so the error is
//     below 2 (5 + 1.173 |g|) < 12 + 3 |g| units.  When the FP32 value lies
//     further than that (plus a margin of 8) from every bfloat16 rounding
//     midpoint, it rounds like the exact value.  Otherwise (a fraction of a
//     percent of inputs) the element is evaluated in FP64.
//   * |g| < 2^-30: silu(g) = g/2 + g^2/4 + O(g^4).  g/2 is exact, and the
//     positive g^2/4 term, far below a float32 unit at g/2, only decides
//     the rounding when g/2 is a bfloat16 midpoint: the result is g/2 nudged
//     by one float32 unit towards +infinity, then rounded.
//   * elsewhere FP64 evaluation; from 2^-30 to 200 silu(g) stays more than
//     2e-9 (relative) away from every bfloat16 midpoint, far above FP64's
//     error, and beyond 200 the FP64 quotient gives g itself (g > 0) or a
//     value far below the smallest bfloat16 (g < 0).
// An exhaustive check over all 65,536 inputs (fp8_selftest_silu_bf16)
// compares this function with the oracle's correctly rounded silu.
//
// The product of two bfloat16 values has at most 16 significant bits, so it
// is exact in FP32 unless it falls below 2^-126; there it is formed in FP64
// (exact) and rounded to bfloat16 directly.
#pragma once

#include <cuda_bf16.h>

#include <cstdint>

namespace fp8blk {

__device__ __forceinline__ uint32_t bf16_rne_bits(float v) {
    const __nv_bfloat16 b = __float2bfloat16_rn(v);
    return static_cast<uint32_t>(*reinterpret_cast<const uint16_t*>(&b));
}

// Nearest bfloat16 (ties to even) of a double, through float32 rounded to
// odd: truncation toward zero with the last bit set when inexact keeps the
// information a later rounding needs, since float32 carries 16 more bits
// than bfloat16 across the whole exponent range (subnormals included).
__device__ __forceinline__ uint32_t bf16_rne_bits_from_double(double d) {
    float f = __double2float_rz(d);
    if (static_cast<double>(f) != d) f = __uint_as_float(__float_as_uint(f) | 1u);
    return bf16_rne_bits(f);
}

// Correctly rounded bfloat16 silu of a bfloat16 g (given widened to float).
__device__ __noinline__ uint32_t silu_bf16_slow(float g) {
    const float ag = fabsf(g);
    if (ag < 0x1p-30f) {
        if (g == 0.0f) return __float_as_uint(g) >> 16;           // +-0
        const float hi = 0.5f * g;                                 // exact
        const uint32_t b = __float_as_uint(hi) + (g > 0.0f ? 1u : 0xFFFFFFFFu);
        return bf16_rne_bits(__uint_as_float(b));
    }
    const double gd = static_cast<double>(g);
    return bf16_rne_bits_from_double(gd / (1.0 + exp(-gd)));
}

__device__ __forceinline__ uint32_t silu_bf16(float g) {
    const float ag = fabsf(g);
    if (ag >= 0x1p-20f && ag <= 80.0f) {
        const float q = __fdividef(g, 1.0f + __expf(-g));
        // units in the last place: 23 + 3 floor|g| >= 12 + 3|g| + 8
        const int32_t margin = 23 + 3 * static_cast<int32_t>(ag);
        const int32_t from_mid = static_cast<int32_t>(__float_as_uint(q) & 0xFFFFu) - 0x8000;
        if (from_mid > margin || from_mid < -margin) return bf16_rne_bits(q);
    }
    return silu_bf16_slow(g);
}

// h = bf16(s * u) for bfloat16 s and u (widened to float).
__device__ __forceinline__ uint32_t bf16_product(float s, float u) {
    const float p = s * u;                                       // exact unless tiny
    if (fabsf(p) < 0x1p-126f && p != 0.0f)
        return bf16_rne_bits_from_double(static_cast<double>(s) * static_cast<double>(u));
    return bf16_rne_bits(p);
}

// The 8 h values of one 16-byte chunk of gate and the matching chunk of up.
__device__ __forceinline__ uint4 swiglu8(const uint4& g, const uint4& u) {
    const uint32_t* gw = reinterpret_cast<const uint32_t*>(&g);
    const uint32_t* uw = reinterpret_cast<const uint32_t*>(&u);
    uint32_t out[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float g0 = __uint_as_float(gw[i] << 16), g1 = __uint_as_float(gw[i] & 0xFFFF0000u);
        const float u0 = __uint_as_float(uw[i] << 16), u1 = __uint_as_float(uw[i] & 0xFFFF0000u);
        const float s0 = __uint_as_float(silu_bf16(g0) << 16), s1 = __uint_as_float(silu_bf16(g1) << 16);
        out[i] = bf16_product(s0, u0) | (bf16_product(s1, u1) << 16);
    }
    return make_uint4(out[0], out[1], out[2], out[3]);
}

// Test support: silu of every bfloat16 bit pattern.
__global__ void silu_selftest_kernel(uint16_t* __restrict__ out) {
    const uint32_t i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < 65536u) out[i] = static_cast<uint16_t>(silu_bf16(__uint_as_float(i << 16)));
}

}  // namespace fp8blk
