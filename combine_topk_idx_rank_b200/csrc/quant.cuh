// Quantisation arithmetic shared by the pack and routing kernels: FP8 e4m3 /
// int8 codes of x / scale with scale = max(amax, 1e-4) / qmax (IEEE division),
// optionally rounded up to a power of two; MXFP4 (E2M1 with the OCP MX shared
// scale); UE8M0 scale bytes.  See pack.cu for where each form is used.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp4.h>
#include <cuda_fp8.h>
#include <stdint.h>

#include "ep_internal.cuh"

#ifndef EP_PACK_IEEE_DIV
#define EP_PACK_IEEE_DIV 0     // 1: every quotient x / scale by the IEEE division
#endif
#ifndef EP_QUANT_PAIRED
#define EP_QUANT_PAIRED 1      // 1: the corrected quotients on packed fp32 pairs
#endif

namespace ep {
namespace {

constexpr int kQuantFp8 = 1, kQuantInt8 = 2, kQuantMxfp4 = 3;

__device__ __forceinline__ float pow2_ceil_bits(float s) {
    // s > 0 and normal: keep the exponent if the mantissa is zero, else bump it
    const uint32_t u = __float_as_uint(s);
    const uint32_t bumped = (u & 0xff800000u) + ((u & 0x007fffffu) ? 0x00800000u : 0u);
    return __uint_as_float(bumped);
}

// Quotients x / s rounded to nearest even.  With r = RN(1/s), y = RN(x r) is
// within one ulp of x / s, the remainder x - s y is exact in one fused
// multiply-add, and the corrected y + r (x - s y) rounds to RN(x / s)
// (Markstein's theorem on division with a fused multiply-add, IBM J. Res.
// Develop. 34(1), 1990) -- provided nothing underflows: x and x / s must stay
// well above the smallest normal.  So the corrected product is used when all
// 16 inputs satisfy |x| >= max(2^-100, 2^-100 s); otherwise (a zero, a tiny
// value, a NaN, or an infinite s) all 16 take the IEEE division.  Over every
// pair of a bf16 x and a bf16 group maximum (scale = max(amax, 1e-4) / 448 or
// / 127), the rule gives the same bits as the IEEE division.
template <bool FAST>
__device__ __forceinline__ void divide16(const float (&f)[16], float s, float (&v)[16]) {
    if constexpr (!FAST || EP_PACK_IEEE_DIV) {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = __fdiv_rn(f[i], s);
        return;
    }
    const float floor_ = fmaxf(0x1p-100f, __fmul_rn(0x1p-100f, s));
    const float r = __frcp_rn(s);
    bool fast = true;
#pragma unroll
    for (int i = 0; i < 16; ++i) fast &= fabsf(f[i]) >= floor_;
#if EP_QUANT_PAIRED
    // the same three correctly rounded operations on pairs of lanes (packed
    // fp32 x2 arithmetic of sm_100): y = x r, e = y (-s) + x, v = e r + y
    uint64_t r2, ns2;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r2) : "f"(r), "f"(r));
    asm("mov.b64 %0, {%1, %2};" : "=l"(ns2) : "f"(-s), "f"(-s));
#pragma unroll
    for (int i = 0; i < 16; i += 2) {
        uint64_t x2, y2, e2, v2;
        asm("mov.b64 %0, {%1, %2};" : "=l"(x2) : "f"(f[i]), "f"(f[i + 1]));
        asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(y2) : "l"(x2), "l"(r2));
        asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(e2) : "l"(y2), "l"(ns2), "l"(x2));
        asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(v2) : "l"(e2), "l"(r2), "l"(y2));
        asm("mov.b64 {%0, %1}, %2;" : "=f"(v[i]), "=f"(v[i + 1]) : "l"(v2));
    }
#else
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const float y = __fmul_rn(f[i], r);
        v[i] = __fmaf_rn(__fmaf_rn(-y, s, f[i]), r, y);
    }
#endif
    if (!fast) {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = __fdiv_rn(f[i], s);
    }
}

// 16 channels -> 16 FP8 e4m3 (RNE, saturating) or int8 (RNE, clamped to
// +-127) codes of x / s.  FAST: quotients by the rule of divide16 (the
// per-token kernel, capped at 64 registers, keeps the plain IEEE division).
template <int QUANT, bool FAST = true>
__device__ __forceinline__ uint4 quant16(const float (&f)[16], float s) {
    float v[16];
    divide16<FAST>(f, s, v);
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        if constexpr (QUANT == kQuantFp8) {
            const __nv_fp8x2_storage_t lo =
                __nv_cvt_float2_to_fp8x2(make_float2(v[4 * i], v[4 * i + 1]), __NV_SATFINITE, __NV_E4M3);
            const __nv_fp8x2_storage_t hi =
                __nv_cvt_float2_to_fp8x2(make_float2(v[4 * i + 2], v[4 * i + 3]), __NV_SATFINITE, __NV_E4M3);
            w[i] = (uint32_t)lo | ((uint32_t)hi << 16);
        } else {
            uint32_t b = 0;
#pragma unroll
            for (int j = 0; j < 4; ++j)
                b |= (uint32_t)(max(-127, min(127, __float2int_rn(v[4 * i + j]))) & 0xff) << (8 * j);
            w[i] = b;
        }
    }
    return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ void unpack16(uint4 lo, uint4 hi, float (&f)[16]) {
    f[0] = bf16lo(lo.x); f[1] = bf16hi(lo.x); f[2] = bf16lo(lo.y); f[3] = bf16hi(lo.y);
    f[4] = bf16lo(lo.z); f[5] = bf16hi(lo.z); f[6] = bf16lo(lo.w); f[7] = bf16hi(lo.w);
    f[8] = bf16lo(hi.x); f[9] = bf16hi(hi.x); f[10] = bf16lo(hi.y); f[11] = bf16hi(hi.y);
    f[12] = bf16lo(hi.z); f[13] = bf16hi(hi.z); f[14] = bf16lo(hi.w); f[15] = bf16hi(hi.w);
}

__device__ __forceinline__ float amax16(const float (&f)[16]) {
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 16; ++i) m = fmaxf(m, fabsf(f[i]));
    return m;
}

// MXFP4 shared scale of a 32-channel group: 2^(floor(log2 amax) - 2), 2 being
// the largest exponent of E2M1 (the OCP MX conversion); amax floored at 1e-4.
__device__ __forceinline__ float mx_scale(float amax) {
    const uint32_t biased = (__float_as_uint(fmaxf(amax, 1e-4f)) >> 23) & 0xffu;
    return __uint_as_float((biased - 2u) << 23);
}

// UE8M0 byte of a positive power of two: its biased exponent.
__device__ __forceinline__ uint8_t ue8m0_of(float s) { return (uint8_t)((__float_as_uint(s) >> 23) & 0xffu); }

// 16 channels -> 16 E2M1 codes, two per byte (even channel in the low nibble).
__device__ __forceinline__ uint2 quant16_fp4(const float (&f)[16], float s) {
    float v[16];
    divide16<true>(f, s, v);
    uint32_t w[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        w[h] = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const __nv_fp4x2_storage_t b = __nv_cvt_float2_to_fp4x2(
                make_float2(v[8 * h + 2 * i], v[8 * h + 2 * i + 1]), __NV_E2M1, cudaRoundNearest);
            w[h] |= (uint32_t)b << (8 * i);
        }
    }
    return make_uint2(w[0], w[1]);
}

__device__ __forceinline__ float finish_scale(float amax, float qmax, int round_scale) {
    const float s = __fdiv_rn(fmaxf(amax, 1e-4f), qmax);
    return round_scale ? pow2_ceil_bits(s) : s;
}

}  // namespace
}  // namespace ep
