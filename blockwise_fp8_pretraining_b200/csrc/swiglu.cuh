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
//     more than 23 + 3 floor|g| units (that bound plus a margin of 8) from
//     every bfloat16 rounding midpoint, it rounds like the exact value.
//     Otherwise (a fraction of a percent of inputs) the element is
//     evaluated in FP64; the fused producer collects such elements and
//     evaluates them after the tile's pass, spread over a warp's lanes.
//   * |g| < 2^-30: silu(g) = g/2 + g^2/4 + O(g^4).  g/2 is exact, and the
//     positive g^2/4 term, far below a float32 unit at g/2, only decides
//     the rounding when g/2 is a bfloat16 midpoint: the result is g/2 nudged
//     by one float32 unit towards +infinity, then rounded.
//   * 200 <= |g|: silu(g) is g itself to within e^-200 (relative), and g
//     is a bfloat16 value, so the result is g (g > 0); for g < 0 it is
//     below 200 e^-200, far below half the smallest bfloat16, so -0.
//   * elsewhere FP64 evaluation with exp_fp64 (relative error below
//     2^-46); from 2^-30 to 200 silu(g) stays more than 2e-9 (relative)
//     away from every bfloat16 midpoint, so it rounds like the exact value.
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

// e^x in FP64 for |x| < 200, within 2^-46 (relative).  Cody and Waite's
// reduction x = n ln2 + r, n = rint(x log2 e), |r| <= ln2 / 2 (+ rounding),
// with ln 2 split in two so that n * kLn2Hi is exact for |n| < 2^12; e^r by
// its Taylor polynomial of degree 11 (the omitted terms are below
// 0.35^12 / 12! < 7e-15 of it), then times 2^n (a normal double here).
// The constants are ln 2, log2 e and 1/k!, rounded to double.
__device__ __forceinline__ double exp_fp64(double x) {
    constexpr double kLog2e = 0x1.71547652b82fep+0;
    constexpr double kLn2Hi = 0x1.62e42fefa3000p-1;     // ln 2, first 40 bits
    constexpr double kLn2Lo = 0x1.3de6af278ece6p-42;    // ln 2 - kLn2Hi
    const double n = rint(x * kLog2e);
    const double r = fma(-n, kLn2Lo, fma(-n, kLn2Hi, x));
    double p = 0x1.ae64567f544e4p-26;                   // 1/11!
    p = fma(p, r, 0x1.27e4fb7789f5cp-22);               // 1/10!
    p = fma(p, r, 0x1.71de3a556c734p-19);               // 1/9!
    p = fma(p, r, 0x1.a01a01a01a01ap-16);               // 1/8!
    p = fma(p, r, 0x1.a01a01a01a01ap-13);               // 1/7!
    p = fma(p, r, 0x1.6c16c16c16c17p-10);               // 1/6!
    p = fma(p, r, 0x1.1111111111111p-7);                // 1/5!
    p = fma(p, r, 0x1.5555555555555p-5);                // 1/4!
    p = fma(p, r, 0x1.5555555555555p-3);                // 1/3!
    p = fma(p, r, 0.5);
    p = fma(p, r, 1.0);
    p = fma(p, r, 1.0);
    return p * __longlong_as_double(static_cast<long long>(static_cast<int>(n) + 1023) << 52);
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
    if (ag >= 200.0f) return g > 0.0f ? __float_as_uint(g) >> 16 : 0x8000u;
    const double gd = static_cast<double>(g);
    return bf16_rne_bits_from_double(gd / (1.0 + exp_fp64(-gd)));
}

// The FP32 fast path alone: true, with the bits, when it decides the
// rounding; false when the element needs silu_bf16_slow.
__device__ __forceinline__ bool silu_bf16_fast(float g, uint32_t& bits) {
    // 2^-20 <= |g| <= 80, compared on the bit pattern of |g|
    const uint32_t ab = __float_as_uint(g) & 0x7FFFFFFFu;
    if (ab - 0x35800000u <= 0x42A00000u - 0x35800000u) {
        const float q = __fdividef(g, 1.0f + __expf(-g));
        bits = bf16_rne_bits(q);
        // decided unless the low 16 bits lie within `margin` units of the
        // midpoint 0x8000
        const uint32_t margin = 23u + 3u * static_cast<uint32_t>(__uint_as_float(ab));
        return (__float_as_uint(q) & 0xFFFFu) - (0x8000u - margin) > 2u * margin;
    }
    return false;
}

__device__ __forceinline__ uint32_t silu_bf16(float g) {
    uint32_t bits;
    return silu_bf16_fast(g, bits) ? bits : silu_bf16_slow(g);
}

// h = bf16(s * u) for bfloat16 s and u (widened to float).
__device__ __forceinline__ uint32_t bf16_product(float s, float u) {
    const float p = s * u;                                       // exact unless tiny
    if (fabsf(p) < 0x1p-126f && p != 0.0f)
        return bf16_rne_bits_from_double(static_cast<double>(s) * static_cast<double>(u));
    return bf16_rne_bits(p);
}

// The 8 h values of one chunk where the fast path decides silu's rounding;
// an element it cannot decide keeps its g, and bit e of `slow` is set for
// element e (h of it is then formed by swiglu_fix).  A warp leaves such
// elements for later instead of running the FP64 path with one lane busy.
__device__ __forceinline__ uint4 swiglu8_fast(const uint4& g, const uint4& u, uint32_t& slow) {
    const uint32_t* gw = reinterpret_cast<const uint32_t*>(&g);
    const uint32_t* uw = reinterpret_cast<const uint32_t*>(&u);
    uint32_t out[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float g0 = __uint_as_float(gw[i] << 16), g1 = __uint_as_float(gw[i] & 0xFFFF0000u);
        const float u0 = __uint_as_float(uw[i] << 16), u1 = __uint_as_float(uw[i] & 0xFFFF0000u);
        uint32_t s0, s1;
        const bool f0 = silu_bf16_fast(g0, s0), f1 = silu_bf16_fast(g1, s1);
        const uint32_t h0 = f0 ? bf16_product(__uint_as_float(s0 << 16), u0) : (gw[i] & 0xFFFFu);
        const uint32_t h1 = f1 ? bf16_product(__uint_as_float(s1 << 16), u1) : (gw[i] >> 16);
        slow |= (f0 ? 0u : 1u << (2 * i)) | (f1 ? 0u : 2u << (2 * i));
        out[i] = h0 | (h1 << 16);
    }
    return make_uint4(out[0], out[1], out[2], out[3]);
}

// h of element `el` (bfloat16 index) of a tile whose gate values sit at
// hg (where h goes) and whose up values sit at hu, through the FP64 path.
__device__ __noinline__ void swiglu_fix(uint16_t* hg, const uint16_t* hu, int el) {
    const float g = __uint_as_float(static_cast<uint32_t>(hg[el]) << 16);
    const float u = __uint_as_float(static_cast<uint32_t>(hu[el]) << 16);
    hg[el] = static_cast<uint16_t>(bf16_product(__uint_as_float(silu_bf16_slow(g) << 16), u));
}

// Test support: silu of every bfloat16 bit pattern.
__global__ void silu_selftest_kernel(uint16_t* __restrict__ out) {
    const uint32_t i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i < 65536u) out[i] = static_cast<uint16_t>(silu_bf16(__uint_as_float(i << 16)));
}

}  // namespace fp8blk
