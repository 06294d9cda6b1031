// kivi_diag.cu -- quantize-dequantize under the groupings the KIVI pages compare
// (kivi_fake_quant): keys per channel or per token, values per token or per
// channel, asymmetric min/max codes or symmetric absmax codes, 1 to 8 bits,
// optionally dense-and-sparse (each group's largest-magnitude element kept
// exactly).
//
// Sources: "KIVI Quantization Secures Llama-2 Accuracy at Two Bits",
// paragraphs 2-3 (reconstruction and attention-output errors of per-token and
// per-channel grouping for keys and for values); record
// kv-efficiency/kivi-2bit-llama2-13b-mha-4k, "Quality" field (the naive
// symmetric per-token 2-bit baseline); KVQuant summary, "Per-Vector
// Dense-and-Sparse Quantization".  At 2 bits the asymmetric groupings are the
// KIVI codec itself (zero = group min, scale = (max - min)/3, both stored as
// fp16, code = rint((x - zero)/scale) clamped).
//
// The work is elementwise with a group reduction and its roofline is HBM: 2
// bytes read and 4 written per element (2 read when only the error is asked
// for).  The division-exact code keeps it near the issue limit as well.
//   - Per token: a lane owns one 16-byte vector (8 channels) of a row; a group
//     of G channels is G/8 adjacent lanes, reduced with xor shuffles.
//   - Per channel: a lane owns 4 adjacent channels of one group of G tokens;
//     it reads the G rows twice (min/max, then codes), the second time from
//     L1/L2, so DRAM sees each byte once.
// Each warp takes whole chunks of one matrix, so the squared error of a chunk
// is one warp reduction and one fp64 atomic add.
//
// The arithmetic is kept off the half-rate integer/compare pipe where it can
// be: group minima and maxima are taken on packed pairs of the 16-bit inputs
// (min/max of representable values is exact in any format), and inputs enter
// fp32 arithmetic through mixed-precision FMAs (x * 1 - c with a 16-bit x and
// fp32 c, one rounding, the same as the fp32 subtraction of the widened x).
#include <cstdint>

#include <cuda_runtime.h>

#include "../../include/kivi.h"
#include "kivi_common.cuh"
#include "kivi_internal.h"

namespace kivi {
namespace {

constexpr unsigned kFull = 0xffffffffu;
constexpr int kFqThreads = 256;
constexpr int kTokenUnitsPerLane = 16;  // per-token chunk: 32 lanes x 16 vectors
constexpr int kTokenBatch = 4;          // vectors in flight per lane
constexpr int kChannelUnitsPerLane = 1; // per-channel chunk: 32 column strips
constexpr int kRowBatch = 8;            // rows in flight per lane (per channel)

struct FqParams {
    const uint16_t *x;    // [N][T][D]
    float *xhat;          // [N][T][D] or null
    double *sq_err;       // [N] or null
    long long N, T;
    int D, G;
    int lpg;              // per token: lanes per group
    long long units;      // units per matrix
    long long chunks;     // chunks per matrix
    long long items;      // N * chunks
    Magic div_chunks;     // division by chunks
    Magic div_pieces;     // division by D/4 (per-channel units per token group)
    float L;              // top code (asymmetric) or largest magnitude code (symmetric)
};

__device__ __forceinline__ uint4 load16(const uint16_t *p)
{
    return __ldg(reinterpret_cast<const uint4 *>(p));
}

__device__ __forceinline__ uint2 load8(const uint16_t *p)
{
    return __ldg(reinterpret_cast<const uint2 *>(p));
}

// Elementwise min / max of two packed pairs of 16-bit inputs.
template <int DT>
__device__ __forceinline__ uint32_t min2(uint32_t a, uint32_t b)
{
    uint32_t d;
    if constexpr (DT == KIVI_BF16)
        asm("min.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    else
        asm("min.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

template <int DT>
__device__ __forceinline__ uint32_t max2(uint32_t a, uint32_t b)
{
    uint32_t d;
    if constexpr (DT == KIVI_BF16)
        asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    else
        asm("max.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// fp32 value of half H of a packed pair (exact).
template <int DT, int H>
__device__ __forceinline__ float widen(uint32_t w)
{
    if constexpr (DT == KIVI_BF16)
        return __uint_as_float(H ? (w & 0xffff0000u) : (w << 16));
    else
        return __half2float(__ushort_as_half((unsigned short)(H ? (w >> 16) : (w & 0xffffu))));
}

// fl(x - c) for x = half H of w: a mixed-precision FMA x * 1 + (-c), rounded
// once, so equal to the fp32 subtraction of the widened x.
template <int DT, int H>
__device__ __forceinline__ float sub_from(uint32_t w, float c)
{
    float d;
    const float nc = -c;
    if constexpr (DT == KIVI_BF16) {
        if constexpr (H == 0)
            asm("{\n\t.reg .b16 lo, hi, one;\n\tmov.b32 {lo, hi}, %1;\n\tmov.b16 one, 0x3F80;\n\t"
                "fma.rn.f32.bf16 %0, lo, one, %2;\n\t}" : "=f"(d) : "r"(w), "f"(nc));
        else
            asm("{\n\t.reg .b16 lo, hi, one;\n\tmov.b32 {lo, hi}, %1;\n\tmov.b16 one, 0x3F80;\n\t"
                "fma.rn.f32.bf16 %0, hi, one, %2;\n\t}" : "=f"(d) : "r"(w), "f"(nc));
    } else {
        if constexpr (H == 0)
            asm("{\n\t.reg .b16 lo, hi, one;\n\tmov.b32 {lo, hi}, %1;\n\tmov.b16 one, 0x3C00;\n\t"
                "fma.rn.f32.f16 %0, lo, one, %2;\n\t}" : "=f"(d) : "r"(w), "f"(nc));
        else
            asm("{\n\t.reg .b16 lo, hi, one;\n\tmov.b32 {lo, hi}, %1;\n\tmov.b16 one, 0x3C00;\n\t"
                "fma.rn.f32.f16 %0, hi, one, %2;\n\t}" : "=f"(d) : "r"(w), "f"(nc));
    }
    return d;
}

template <int DT>
__device__ __forceinline__ float sub_from_h(uint32_t w, int h, float c)
{
    return h ? sub_from<DT, 1>(w, c) : sub_from<DT, 0>(w, c);
}

// max(0, min(1, a*b + c)), one rounding: positive exactly when a*b + c > 0.
__device__ __forceinline__ float fma_sat(float a, float b, float c)
{
    float d;
    asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// fp16 rounding of a non-negative scale or of a zero, written back as fp32,
// with a stored zero of either sign read as +0.
__device__ __forceinline__ float to_f16_plus0(float v)
{
    const unsigned short b = __half_as_ushort(__float2half_rn(v));
    return (b & 0x7fffu) ? __half2float(__ushort_as_half(b)) : 0.0f;
}

// Group parameters from the group minimum a and maximum b: asymmetric (s, z);
// symmetric s from the largest magnitude max(-a, b), z = 0.  rs is the
// correctly rounded reciprocal of s, or 0 when s == 0 (every code is then 0).
template <bool SYM>
__device__ __forceinline__ void group_params(float a, float b, float L, float &s, float &z,
                                             float &rs)
{
    if (SYM) {
        s = to_f16_plus0(__fdiv_rn(fmaxf(-a, b), L));
        z = 0.0f;
    } else {
        s = to_f16_plus0(__fdiv_rn(__fsub_rn(b, a), L));
        z = to_f16_plus0(a);
    }
    rs = s == 0.0f ? 0.0f : __frcp_rn(s);
}

// Dequantizes the NE = 2*NW elements of the packed words w[], element e
// (half e%2 of word e/2) with group parameters (s, z, rs)[e * STRIDE].  The
// code is rint(RN(d/s)) clamped to [lo, L], with d = x - z (asymmetric) or x
// (symmetric); a zero scale gives code 0 (rs = 0 makes the quotient 0).
//
// EXACT takes RN(d/s) by IEEE division.  Otherwise the quotient is q =
// RN(d * rs), checked with Ziv's rounding test (A. Ziv, "Fast evaluation of
// elementary mathematical functions with correctly rounded last bit", ACM TOMS
// 17(3), 1991): with rs = RN(1/s), q is within 1.5 ulp of d/s and RN(d/s)
// within 0.5 ulp, so rint(q) and rint(RN(d/s)) can differ only if q lies within
// 2 ulp (at most 2^-15 below 256) of a half-integer, and not at all when the
// residual d - q*s is 0 (one FMA rounds it once, so it reads 0 only when q*s
// equals d: no underflow is possible for q near a half-integer).  `near` becomes positive when some
// q lies that close (|q - rint(q)| > 0.5 - 2^-13, tested as
// 2^14 |q - rint(q)| - 8190 > 0) with a nonzero residual; the caller then
// redoes the elements EXACT.
// Clamping before rounding is exact because rint commutes with clamping to
// integer bounds, and rounding adds and subtracts 1.5 * 2^23, which rounds
// |y| <= 2^22 to the nearest integer, ties to even (and gives +0, never -0,
// for the zero code).
//
// With ERR, e2 gains the squared errors (x - x_hat)^2 of the NE elements, each
// difference rounded to fp32, squared and summed in fp32 (fused).  With OUT,
// the elements flagged in `sparse` (bit e) are a group's exactly kept element:
// x_hat = x, no error.
template <int DT, bool SYM, bool ERR, bool OUT, bool EXACT, int STRIDE, int NW>
__device__ __forceinline__ void fq_words(const uint32_t (&w)[NW], const float *s, const float *z,
                                         const float *rs, float L, float (&h)[2 * NW], float &e2,
                                         float &near, unsigned sparse = 0u)
{
    constexpr int NE = 2 * NW;
    constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
    const float lo = SYM ? -L - 1.0f : 0.0f;
#pragma unroll
    for (int e = 0; e < NE; ++e) {
        const int k = e * STRIDE;
        const float d = sub_from_h<DT>(w[e / 2], e & 1, z[k]);
        float y, q = 0.0f;
        if (EXACT) {
            y = s[k] == 0.0f ? 0.0f : fminf(fmaxf(__fdiv_rn(d, s[k]), lo), L);
        } else {
            q = __fmul_rn(d, rs[k]);
            y = fminf(fmaxf(q, lo), L);
        }
        const float r = __fsub_rn(__fadd_rn(y, kRound), kRound);
        // near grows when y is within the window AND q * s != d (an exact
        // quotient, q = d/s, is its own correctly rounded value and needs no
        // redo; bf16 and fp16 inputs hit exact half-integers often).  Both
        // factors are saturated to [0, 1] and, when positive, at least 2^-23.
        if (!EXACT)
            near = __fmaf_rn(fma_sat(fabsf(__fsub_rn(y, r)), 16384.0f, -8190.0f),
                             fma_sat(fabsf(__fmaf_rn(-q, s[k], d)), 0x1p126f, 0.0f), near);
        h[e] = SYM ? __fmul_rn(r, s[k]) : __fmaf_rn(r, s[k], z[k]);
        const bool keep = OUT && ((sparse >> e) & 1u);
        if (keep) h[e] = (e & 1) ? widen<DT, 1>(w[e / 2]) : widen<DT, 0>(w[e / 2]);
        if (ERR && !keep) {
            const float df = sub_from_h<DT>(w[e / 2], e & 1, h[e]);
            e2 = __fmaf_rn(df, df, e2);
        }
    }
}

__device__ __forceinline__ void flush_err(const FqParams &p, long long n, double acc, int lane)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(kFull, acc, o);
    if (lane == 0) atomicAdd(p.sq_err + n, acc);
}

__device__ __forceinline__ void store8(float *dst, const float (&h)[8])
{
    float4 *d4 = reinterpret_cast<float4 *>(dst);
    d4[0] = make_float4(h[0], h[1], h[2], h[3]);
    d4[1] = make_float4(h[4], h[5], h[6], h[7]);
}

// ---- per token: groups of G consecutive channels of one row -----------------
// A lane owns one 16-byte vector (8 channels) of a row; a group of G channels
// is G/8 adjacent lanes, reduced with xor shuffles.  A vector with a quotient
// near a rounding boundary is redone exactly.  With OUT the group's element of
// largest |x| (the first on ties) is kept exactly and the statistics skip it.
template <int DT, bool SYM, bool ERR, bool OUT>
__global__ void __launch_bounds__(kFqThreads, 4) fq_token_kernel(const FqParams p)
{
    const int lane = threadIdx.x & 31;
    const long long warp0 = ((long long)blockIdx.x * kFqThreads + threadIdx.x) >> 5;
    const long long nwarps = ((long long)gridDim.x * kFqThreads) >> 5;
    constexpr int kChunk = 32 * kTokenUnitsPerLane;
    const float inf = __int_as_float(0x7f800000);
    for (long long item = warp0; item < p.items; item += nwarps) {
        const long long n = div_floor(item, p.div_chunks);
        const long long u0 = (item - n * p.chunks) * kChunk;
        const uint16_t *xm = p.x + n * p.T * p.D;
        float *xo = p.xhat ? p.xhat + n * p.T * p.D : nullptr;
        double acc = 0.0;
#pragma unroll 1
        for (int it = 0; it < kTokenUnitsPerLane; it += kTokenBatch) {
            if (u0 + it * 32 >= p.units) break;
            uint4 v[kTokenBatch];
#pragma unroll
            for (int b = 0; b < kTokenBatch; ++b) {
                const long long u = u0 + (it + b) * 32 + lane;
                if (u < p.units) v[b] = load16(xm + u * 8);
            }
#pragma unroll
            for (int b = 0; b < kTokenBatch; ++b) {
                const long long u = u0 + (it + b) * 32 + lane;
                const bool act = u < p.units;
                const uint32_t w[4] = {v[b].x, v[b].y, v[b].z, v[b].w};
                // Inactive lanes form whole groups (a matrix holds whole
                // groups), so their neutral statistics reach no active group.
                float a = inf, c = -inf;
                unsigned sparse = 0u;
                if (OUT) {
                    // (largest |x|, its element index in the group), first on ties
                    const int base = (lane % p.lpg) * 8;
                    float xv[8];
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        xv[i] = (i & 1) ? widen<DT, 1>(w[i / 2]) : widen<DT, 0>(w[i / 2]);
                    float am = -1.0f;
                    int ai = 0x7fffffff;
                    if (act) {
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            if (fabsf(xv[i]) > am) {
                                am = fabsf(xv[i]);
                                ai = base + i;
                            }
                    }
                    for (int o = 1; o < p.lpg; o <<= 1) {
                        const float om = __shfl_xor_sync(kFull, am, o);
                        const int oi = __shfl_xor_sync(kFull, ai, o);
                        if (om > am || (om == am && oi < ai)) {
                            am = om;
                            ai = oi;
                        }
                    }
                    if (act) {
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            if (base + i != ai) {
                                a = fminf(a, xv[i]);
                                c = fmaxf(c, xv[i]);
                            }
                        if (ai >= base && ai < base + 8) sparse = 1u << (ai - base);
                    }
                } else if (act) {
                    const uint32_t mn = min2<DT>(min2<DT>(w[0], w[1]), min2<DT>(w[2], w[3]));
                    const uint32_t mx = max2<DT>(max2<DT>(w[0], w[1]), max2<DT>(w[2], w[3]));
                    a = fminf(widen<DT, 0>(mn), widen<DT, 1>(mn));
                    c = fmaxf(widen<DT, 0>(mx), widen<DT, 1>(mx));
                }
                for (int o = 1; o < p.lpg; o <<= 1) {
                    a = fminf(a, __shfl_xor_sync(kFull, a, o));
                    c = fmaxf(c, __shfl_xor_sync(kFull, c, o));
                }
                if (!act) continue;
                float sc, z, rs, h[8], e2 = 0.0f, near = 0.0f;
                group_params<SYM>(a, c, p.L, sc, z, rs);
                fq_words<DT, SYM, ERR, OUT, false, 0, 4>(w, &sc, &z, &rs, p.L, h, e2, near, sparse);
                if (near > 0.0f) {
                    e2 = 0.0f;
                    fq_words<DT, SYM, ERR, OUT, true, 0, 4>(w, &sc, &z, &rs, p.L, h, e2, near, sparse);
                }
                if (ERR) acc += (double)e2;
                if (xo) store8(xo + u * 8, h);
            }
        }
        if (ERR) flush_err(p, n, acc, lane);
    }
}

// ---- per channel: groups of G consecutive tokens of one channel ---------------
// A lane owns 4 adjacent channels (one 8-byte piece of a row) of one group; a
// unit is (token group g, piece c) of one matrix, unit = g*(D/4) + c.  A row
// with a quotient near a rounding boundary is redone exactly.  With OUT each
// channel's element of largest |x| (the first row on ties) is kept exactly; it
// is the first occurrence of the group's maximum or minimum, so the statistics
// of the others are the runner-up maximum or minimum.
template <int DT, bool SYM, bool ERR, bool OUT>
__global__ void __launch_bounds__(kFqThreads, 3) fq_channel_kernel(const FqParams p)
{
    const int lane = threadIdx.x & 31;
    const long long warp0 = ((long long)blockIdx.x * kFqThreads + threadIdx.x) >> 5;
    const long long nwarps = ((long long)gridDim.x * kFqThreads) >> 5;
    constexpr int kChunk = 32 * kChannelUnitsPerLane;
    const int pieces = p.D / 4;
    for (long long item = warp0; item < p.items; item += nwarps) {
        const long long n = div_floor(item, p.div_chunks);
        const long long u0 = (item - n * p.chunks) * kChunk;
        double acc = 0.0;
#pragma unroll 1
        for (int it = 0; it < kChannelUnitsPerLane; ++it) {
            const long long u = u0 + it * 32 + lane;
            if (u >= p.units) continue;
            const long long g = div_floor(u, p.div_pieces);
            const int col = (int)(u - g * pieces) * 4;
            const long long row0 = n * p.T + g * p.G;
            const uint16_t *src = p.x + row0 * p.D + col;
            const uint2 first = load8(src);
            float sc[4], z[4], rs[4];
            int orow[4] = {-1, -1, -1, -1};
            if (OUT) {
                const uint32_t f[2] = {first.x, first.y};
                float mx1[4], mx2[4], mn1[4], mn2[4];
                int imx[4], imn[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    mx1[e] = mn1[e] = (e & 1) ? widen<DT, 1>(f[e / 2]) : widen<DT, 0>(f[e / 2]);
                    mx2[e] = -__int_as_float(0x7f800000);
                    mn2[e] = __int_as_float(0x7f800000);
                    imx[e] = imn[e] = 0;
                }
#pragma unroll 1
                for (int t0 = 1; t0 < p.G; t0 += kRowBatch) {
                    uint2 rb[kRowBatch];
#pragma unroll
                    for (int b = 0; b < kRowBatch; ++b)
                        if (t0 + b < p.G) rb[b] = load8(src + (long long)(t0 + b) * p.D);
#pragma unroll
                    for (int b = 0; b < kRowBatch; ++b) {
                        if (t0 + b >= p.G) break;
                        const int t = t0 + b;  // rows in order: first occurrences win
                        const uint32_t g2[2] = {rb[b].x, rb[b].y};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float v = (e & 1) ? widen<DT, 1>(g2[e / 2]) : widen<DT, 0>(g2[e / 2]);
                            const bool up = v > mx1[e], dn = v < mn1[e];
                            mx2[e] = up ? mx1[e] : fmaxf(mx2[e], v);
                            mx1[e] = up ? v : mx1[e];
                            imx[e] = up ? t : imx[e];
                            mn2[e] = dn ? mn1[e] : fminf(mn2[e], v);
                            mn1[e] = dn ? v : mn1[e];
                            imn[e] = dn ? t : imn[e];
                        }
                    }
                }
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float am = fabsf(mx1[e]), an = fabsf(mn1[e]);
                    orow[e] = am > an ? imx[e] : an > am ? imn[e] : min(imx[e], imn[e]);
                    const float dmx = orow[e] == imx[e] ? mx2[e] : mx1[e];
                    const float dmn = orow[e] == imn[e] ? mn2[e] : mn1[e];
                    group_params<SYM>(dmn, dmx, p.L, sc[e], z[e], rs[e]);
                }
            } else {
            uint32_t mn[2] = {first.x, first.y}, mx[2] = {first.x, first.y};
#pragma unroll 1
            for (int t0 = 1; t0 < p.G; t0 += kRowBatch) {
                uint2 v[kRowBatch];
#pragma unroll
                for (int b = 0; b < kRowBatch; ++b)
                    if (t0 + b < p.G) v[b] = load8(src + (long long)(t0 + b) * p.D);
#pragma unroll
                for (int b = 0; b < kRowBatch; ++b) {
                    if (t0 + b < p.G) {
                        mn[0] = min2<DT>(mn[0], v[b].x);
                        mn[1] = min2<DT>(mn[1], v[b].y);
                        mx[0] = max2<DT>(mx[0], v[b].x);
                        mx[1] = max2<DT>(mx[1], v[b].y);
                    }
                }
            }
            group_params<SYM>(widen<DT, 0>(mn[0]), widen<DT, 0>(mx[0]), p.L, sc[0], z[0], rs[0]);
            group_params<SYM>(widen<DT, 1>(mn[0]), widen<DT, 1>(mx[0]), p.L, sc[1], z[1], rs[1]);
            group_params<SYM>(widen<DT, 0>(mn[1]), widen<DT, 0>(mx[1]), p.L, sc[2], z[2], rs[2]);
            group_params<SYM>(widen<DT, 1>(mn[1]), widen<DT, 1>(mx[1]), p.L, sc[3], z[3], rs[3]);
            }
            float *dst = p.xhat ? p.xhat + row0 * p.D + col : nullptr;
            float e2 = 0.0f;
#pragma unroll 1
            for (int t0 = 0; t0 < p.G; t0 += kRowBatch) {
                uint2 v[kRowBatch];
#pragma unroll
                for (int b = 0; b < kRowBatch; ++b)
                    if (t0 + b < p.G) v[b] = load8(src + (long long)(t0 + b) * p.D);
#pragma unroll
                for (int b = 0; b < kRowBatch; ++b) {
                    if (t0 + b < p.G) {
                        const uint32_t w[2] = {v[b].x, v[b].y};
                        float h[4], e2r = 0.0f, near = 0.0f;
                        unsigned sparse = 0u;
                        if (OUT) {
                            const int t = t0 + b;
                            sparse = (orow[0] == t ? 1u : 0u) | (orow[1] == t ? 2u : 0u) |
                                     (orow[2] == t ? 4u : 0u) | (orow[3] == t ? 8u : 0u);
                        }
                        fq_words<DT, SYM, ERR, OUT, false, 1, 2>(w, sc, z, rs, p.L, h, e2r, near, sparse);
                        if (near > 0.0f) {
                            e2r = 0.0f;
                            fq_words<DT, SYM, ERR, OUT, true, 1, 2>(w, sc, z, rs, p.L, h, e2r, near,
                                                                    sparse);
                        }
                        if (dst)
                            *reinterpret_cast<float4 *>(dst + (long long)(t0 + b) * p.D) =
                                make_float4(h[0], h[1], h[2], h[3]);
                        if (ERR) {
                            e2 += e2r;
                            if (b & 1) {  // runs of two rows (8 elements)
                                acc += (double)e2;
                                e2 = 0.0f;
                            }
                        }
                    }
                }
            }
            if (ERR) acc += (double)e2;
        }
        if (ERR) flush_err(p, n, acc, lane);
    }
}

template <int DT, bool SYM, bool ERR, bool OUT>
cudaError_t launch_fq(int axis, const FqParams &p, cudaStream_t st)
{
    const long long warps_per_cta = kFqThreads / 32;
    long long grid = (p.items + warps_per_cta - 1) / warps_per_cta;
    const long long cap = (long long)num_sms() * (2048 / kFqThreads);
    if (grid > cap) grid = cap;
    if (axis == KIVI_AXIS_PER_TOKEN)
        fq_token_kernel<DT, SYM, ERR, OUT><<<(unsigned)grid, kFqThreads, 0, st>>>(p);
    else
        fq_channel_kernel<DT, SYM, ERR, OUT><<<(unsigned)grid, kFqThreads, 0, st>>>(p);
    return cudaGetLastError();
}

template <int DT, bool SYM>
cudaError_t launch_fq(int axis, int outlier, const FqParams &p, cudaStream_t st)
{
    if (outlier)
        return p.sq_err ? launch_fq<DT, SYM, true, true>(axis, p, st)
                        : launch_fq<DT, SYM, false, true>(axis, p, st);
    return p.sq_err ? launch_fq<DT, SYM, true, false>(axis, p, st)
                    : launch_fq<DT, SYM, false, false>(axis, p, st);
}

}  // namespace
}  // namespace kivi

using namespace kivi;

extern "C" kivi_status kivi_fake_quant(const void *x, kivi_dtype dtype, long long N, long long T,
                                       int D, int axis, int G, int bits, int symmetric,
                                       int outlier, float *xhat, double *sq_err, void *stream)
{
    if (!x || (!xhat && !sq_err)) return KIVI_ERR_ARG;
    if (((uintptr_t)x & 15u) || ((uintptr_t)xhat & 15u) || ((uintptr_t)sq_err & 7u))
        return KIVI_ERR_ARG;
    if (dtype != KIVI_F16 && dtype != KIVI_BF16) return KIVI_ERR_ARG;
    if (N < 1 || T < 1 || D < 8 || D % 8 != 0 || G < 1) return KIVI_ERR_ARG;
    if (axis != KIVI_AXIS_PER_CHANNEL && axis != KIVI_AXIS_PER_TOKEN) return KIVI_ERR_ARG;
    if (bits < (symmetric ? 2 : 1) || bits > 8) return KIVI_ERR_ARG;
    if (outlier != 0 && outlier != 1) return KIVI_ERR_ARG;
    if (axis == KIVI_AXIS_PER_CHANNEL ? T % G != 0 : D % G != 0) return KIVI_ERR_ARG;
    if (axis == KIVI_AXIS_PER_TOKEN && (G < 8 || G > 256 || (G & (G - 1)) != 0))
        return KIVI_ERR_UNSUPPORTED;
    if (T > (1LL << 33) / D || N > (1LL << 62) / (T * D)) return KIVI_ERR_UNSUPPORTED;

    FqParams p;
    p.x = (const uint16_t *)x;
    p.xhat = xhat;
    p.sq_err = sq_err;
    p.N = N;
    p.T = T;
    p.D = D;
    p.G = G;
    const int unit_lanes = axis == KIVI_AXIS_PER_TOKEN ? 32 * kTokenUnitsPerLane
                                                       : 32 * kChannelUnitsPerLane;
    if (axis == KIVI_AXIS_PER_TOKEN) {
        p.lpg = G / 8;  // G is a power of two in [8, 256] here
        p.units = T * (D / 8);
    } else {
        p.lpg = 1;
        p.units = (T / G) * (D / 4);
    }
    p.chunks = (p.units + unit_lanes - 1) / unit_lanes;
    p.items = N * p.chunks;
    p.div_chunks = make_magic((unsigned long long)p.chunks);
    p.div_pieces = make_magic((unsigned long long)(D / 4));
    p.L = symmetric ? (float)((1 << (bits - 1)) - 1) : (float)((1 << bits) - 1);

    cudaStream_t st = (cudaStream_t)stream;
    if (sq_err && cudaMemsetAsync(sq_err, 0, (size_t)N * sizeof(double), st) != cudaSuccess)
        return KIVI_ERR_CUDA;
    cudaError_t e;
    if (dtype == KIVI_BF16)
        e = symmetric ? launch_fq<KIVI_BF16, true>(axis, outlier, p, st)
                      : launch_fq<KIVI_BF16, false>(axis, outlier, p, st);
    else
        e = symmetric ? launch_fq<KIVI_F16, true>(axis, outlier, p, st)
                      : launch_fq<KIVI_F16, false>(axis, outlier, p, st);
    return e == cudaSuccess ? KIVI_OK : KIVI_ERR_CUDA;
}
