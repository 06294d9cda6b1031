// kivi_decode_ops.cuh -- device helpers shared by the decode kernels: PTX
// wrappers for mbarriers and bulk copies, paired fp32 arithmetic, the exact
// code-to-float extraction tricks, RoPE angle reduction and warp reductions.
// Internal to the CUDA library.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "kivi_common.cuh"

#ifndef KIVI_SCALAR_F32
#define KIVI_SCALAR_F32 0
#endif

namespace kivi {

constexpr unsigned FULL = 0xffffffffu;
constexpr float kRescaleSlack = 8.0f;
constexpr int kWaitLimit = 1 << 22;
// ---- PTX wrappers ----------------------------------------------------------
__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint32_t bar, int count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes,
                                         uint32_t bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}
// Lane 0 of the calling warp arms `bar` for `bytes` and starts one bulk copy
// of `bytes` into it; the other lanes skip both under a predicate (no branch).
__device__ __forceinline__ void lane0_expect_copy(int lane, uint32_t bar, uint32_t dst, const void *src,
                                                  uint32_t bytes, uint32_t expect)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.eq.u32 p, %0, 0;\n\t"
        "@p mbarrier.arrive.expect_tx.shared::cta.b64 _, [%1], %5;\n\t"
        "@p cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%2], [%3], %4, [%1];\n\t}"
        ::"r"(lane), "r"(bar), "r"(dst), "l"(src), "r"(bytes), "r"(expect)
        : "memory");
}
__device__ __forceinline__ void lane0_copy(int lane, uint32_t bar, uint32_t dst, const void *src,
                                           uint32_t bytes)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.eq.u32 p, %0, 0;\n\t"
        "@p cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%2], [%3], %4, [%1];\n\t}"
        ::"r"(lane), "r"(bar), "r"(dst), "l"(src), "r"(bytes)
        : "memory");
}
__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c)
{
#if KIVI_SCALAR_F32
    return make_float2(fmaf(a.x, b.x, c.x), fmaf(a.y, b.y, c.y));
#endif
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b)
{
#if KIVI_SCALAR_F32
    return make_float2(__fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y));
#endif
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// ---- code extraction ---------------------------------------------------------
// Code pair i of a word (split-pair layout): first code at bits 2i of w,
// second at bits 2i of w16 = w >> 16.  OR-ing the field into the mantissa of
// 2^23 (`magic`, a runtime register so that the mask stays an immediate) gives
// 2^23 + c*2^(2i) exactly; adding `neg` = (-2^23, -2^23) leaves
// (c_first 2^(2i), c_second 2^(2i)).  One logic op per code; the power of two
// is folded into the scales (the pre-RoPE key path uses this conversion,
// since it dequantizes explicitly).
__device__ __forceinline__ float2 code_pair(uint32_t w, uint32_t w16, int i, uint32_t magic,
                                            float2 neg)
{
    const uint32_t msk = 3u << (2 * i);
    uint32_t a, b;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(a) : "r"(w), "r"(msk), "r"(magic));
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(b) : "r"(w16), "r"(msk), "r"(magic));
    return fadd2(make_float2(__uint_as_float(a), __uint_as_float(b)), neg);
}
// 2^-2i, the inverse of pair i's shift.
__device__ __forceinline__ float pair_scale(int i) { return __uint_as_float((uint32_t)(127 - 2 * i) << 23); }
// 2^e for -126 <= e <= 127.
__device__ __forceinline__ float pow2i(int e) { return __uint_as_float((uint32_t)(127 + e) << 23); }

// Keys, fast path: AND-ing pair i's field out of the word (or of the word
// shifted right by 16) leaves the fp32 denormal c * 2^(2i-149).  Multiplying
// by q'' = q' * 2^(kKexp-2i) gives q' c 2^(kKexp-149) with no conversion
// step; one logic op per code and one fp32x2 FMA per pair.
constexpr int kKexp = 64;
constexpr float kKunscale = 0x1p85f;   // 2^(149 - kKexp)
__device__ __forceinline__ float kq_scale(int i) { return pow2i(kKexp - 2 * i); }

// Values: AND-ing 0x00030003 << 2j out of a word leaves two f16 subnormals
// c * 2^(2j-24) in its halves (j <= 3; pairs 4..7 are read from the word
// shifted right by 8).  They multiply an f16 token weight in a mixed-precision
// FMA (exact f16 products, fp32 accumulation).  HA/HB pick the halves.
template <int HA, int HB>
__device__ __forceinline__ float hfma_f32(uint32_t a, uint32_t b, float c)
{
    float d;
    if constexpr (HA == 0 && HB == 0)
        asm("{\n\t.reg .b16 a0, a1, b0, b1;\n\tmov.b32 {a0, a1}, %1;\n\tmov.b32 {b0, b1}, %2;\n\t"
            "fma.rn.f32.f16 %0, a0, b0, %3;\n\t}" : "=f"(d) : "r"(a), "r"(b), "f"(c));
    else if constexpr (HA == 1 && HB == 0)
        asm("{\n\t.reg .b16 a0, a1, b0, b1;\n\tmov.b32 {a0, a1}, %1;\n\tmov.b32 {b0, b1}, %2;\n\t"
            "fma.rn.f32.f16 %0, a1, b0, %3;\n\t}" : "=f"(d) : "r"(a), "r"(b), "f"(c));
    else if constexpr (HA == 0 && HB == 1)
        asm("{\n\t.reg .b16 a0, a1, b0, b1;\n\tmov.b32 {a0, a1}, %1;\n\tmov.b32 {b0, b1}, %2;\n\t"
            "fma.rn.f32.f16 %0, a0, b1, %3;\n\t}" : "=f"(d) : "r"(a), "r"(b), "f"(c));
    else
        asm("{\n\t.reg .b16 a0, a1, b0, b1;\n\tmov.b32 {a0, a1}, %1;\n\tmov.b32 {b0, b1}, %2;\n\t"
            "fma.rn.f32.f16 %0, a1, b1, %3;\n\t}" : "=f"(d) : "r"(a), "r"(b), "f"(c));
    return d;
}
// Token weights are kept near 2^6 on the first group (room for the 2^8 of
// softmax slack below the f16 limit) and scaled down when one would pass 2^15.
constexpr int kVTargetExp = 6;
constexpr float kVLimit = 32768.0f;

// Values with four query heads per kv head (head_dim 128): the code part runs
// as fp32x2 FMAs, half the issue slots of one mixed FMA per code.  Token
// weights stay fp32, b = p s 2^kVexp: with p <= 2^8 (softmax slack) and
// s <= 65504 they stay below 2^124, and a code AND-ed out of its word is the
// fp32 denormal c 2^(2m-149), so each product b c 2^(2m-149) is exact and
// normal for every weight p s >= 2^(-77-2m): no per-head exponent tracking.
constexpr int kVexp = 100;
template <int D, int HG>
constexpr bool values_f32() { return HG == 4 && D == 128; }

// RoPE angles.  (sin a, cos a) of an fp32 angle 0 <= a < 2^17 * 2pi: a is
// reduced modulo 2pi by the method of Cody and Waite ("Software Manual for the
// Elementary Functions", 1980) with 2pi split in four parts, P1 = 101/16,
// P2 = -15/512 and P3 = -75/2^22 of at most 7 significant bits (each k*P_i
// exact in fp32 for k = rint(a/2pi) < 2^17, and each partial difference
// exact) and P4 = fl(2pi - P1 - P2 - P3).  The reduced angle is within 2^-22
// of the exact one; the hardware sine and cosine of it add at most 2^-21.4.
// Positions are limited accordingly when a pre-RoPE cache is created.
__device__ __forceinline__ void rope_sincos(float a, float *sn, float *cn)
{
    const float k = __fadd_rn(__fmaf_rn(a, 0.15915494f, 12582912.0f), -12582912.0f);
    float r = __fmaf_rn(-k, 6.3125f, a);
    r = __fmaf_rn(-k, -0.029296875f, r);
    r = __fmaf_rn(-k, __uint_as_float(0xb7960000u), r);
    r = __fmaf_rn(-k, __uint_as_float(0x338885a3u), r);
    *sn = __sinf(r);
    *cn = __cosf(r);
}

template <int DT>
__device__ __forceinline__ float to_f(uint16_t b)
{
    if constexpr (DT == 1) return __uint_as_float((uint32_t)b << 16);
    else return __half2float(__ushort_as_half(b));
}
__device__ __forceinline__ float f16f(uint16_t b) { return __half2float(__ushort_as_half(b)); }

__device__ __forceinline__ float warp_sum(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(FULL, x, o);
    return x;
}
// Reduce-scatter of N per-lane values: at each level (lane offset OFF, OFF/2,
// ...) a lane keeps half of its values and adds its partner's copy of them,
// until one value is left, that of index h = the lane's bits OFF, OFF/2, ...
// (most significant first), summed over those lanes.
template <int N, int OFF>
__device__ __forceinline__ float reduce_scatter(const float (&v)[N], int lane)
{
    if constexpr (N == 1) {
        return v[0];
    } else {
        const bool up = lane & OFF;
        float nv[N / 2];
#pragma unroll
        for (int i = 0; i < N / 2; ++i) {
            const float keep = up ? v[N / 2 + i] : v[i];
            const float send = up ? v[i] : v[N / 2 + i];
            nv[i] = keep + __shfl_xor_sync(FULL, send, OFF);
        }
        return reduce_scatter<N / 2, OFF / 2>(nv, lane);
    }
}
// out[h] = sum over the warp of v[h], for every h, in every lane (N a power
// of two up to 16): a reduce-scatter, the rest of the butterfly, a gather.
template <int N>
__device__ __forceinline__ void warp_sum_n(const float (&v)[N], float (&out)[N], int lane)
{
    if constexpr (N == 1) {
        out[0] = warp_sum(v[0]);
    } else {
        constexpr int LOG = N == 2 ? 1 : N == 4 ? 2 : N == 8 ? 3 : 4;
        float x = reduce_scatter<N, 16>(v, lane);
#pragma unroll
        for (int o = 16 >> LOG; o > 0; o >>= 1) x += __shfl_xor_sync(FULL, x, o);
#pragma unroll
        for (int h = 0; h < N; ++h) out[h] = __shfl_sync(FULL, x, h << (5 - LOG));
    }
}

__device__ __forceinline__ float warp_max(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(FULL, x, o));
    return x;
}

}  // namespace kivi
