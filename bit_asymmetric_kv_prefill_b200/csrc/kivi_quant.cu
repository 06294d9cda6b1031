// kivi_quant.cu -- prefill quantizer and residual append/flush kernels.
//
// Keys are grouped per channel over 32 consecutive tokens and values per token
// over 32 consecutive channels ("KIVI Quantization Secures Llama-2 Accuracy at
// Two Bits", paragraphs 2-3; record kv-efficiency/kivi-2bit-llama2-13b-mha-4k,
// "Quant method": kivi-2bit-per-channel-k-per-token-v).  Each CTA takes one
// group tile (32 tokens x D channels of K and of V) at a time:
//   1. the tile is staged into padded shared memory with cp.async, double
//      buffered across the CTA's groups;
//   2. statistics: per-channel key min/max with paired (bf16x2 / f16x2)
//      min/max over 16 rows per thread, the two row halves merged by a warp
//      shuffle; per-token value min/max over each 32-channel group;
//   3. each group's fp16 scale/zero and its three code thresholds.  The code
//      clamp(rint(fl(x - z) / s), 0, 3) equals the number of thresholds x has
//      reached, x_k being the smallest input value whose fp32 difference to z
//      passes the k-th exact fp32 bound (see code_params); x_k is found by a
//      bounded search around z + E_k that evaluates the definition itself;
//   4. codes: two channels at a time, three paired `x >= x_k` compares give
//      lane masks, two logic ops turn them into the pair's two 2-bit codes and
//      one multiply-add shifts them into the word;
//   5. the finished 24*D-byte group block leaves with coalesced 16-byte stores.
// The residual rows of a prefill and the appended token of a flush are copied
// by the same launch.
#include <cstring>

#include <cuda_runtime.h>

#include "kivi_common.cuh"
#include "kivi_internal.h"

namespace kivi {

// ---- input dtype helpers (bits are carried as uint16 / packed uint32) ----------
template <int DT>
struct In;

template <>
struct In<1> {  // bfloat16
    static constexpr uint16_t kInf = 0x7F80u, kNegInf = 0xFF80u;
    __device__ static float f(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }
    __device__ static uint16_t from_float_rd(float y) { return __bfloat16_as_ushort(__float2bfloat16_rd(y)); }
    __device__ static __nv_bfloat162 v(uint32_t u)
    {
        __nv_bfloat162 r;
        memcpy(&r, &u, 4);
        return r;
    }
    __device__ static uint32_t u(__nv_bfloat162 x)
    {
        uint32_t r;
        memcpy(&r, &x, 4);
        return r;
    }
    __device__ static uint32_t vmin(uint32_t a, uint32_t b) { return u(__hmin2(v(a), v(b))); }
    __device__ static uint32_t vmax(uint32_t a, uint32_t b) { return u(__hmax2(v(a), v(b))); }
    __device__ static uint32_t ge_mask(uint32_t a, uint32_t b) { return __hge2_mask(v(a), v(b)); }
};

template <>
struct In<0> {  // IEEE fp16
    static constexpr uint16_t kInf = 0x7C00u, kNegInf = 0xFC00u;
    __device__ static float f(uint16_t b) { return __half2float(__ushort_as_half(b)); }
    __device__ static uint16_t from_float_rd(float y) { return __half_as_ushort(__float2half_rd(y)); }
    __device__ static __half2 v(uint32_t u)
    {
        __half2 r;
        memcpy(&r, &u, 4);
        return r;
    }
    __device__ static uint32_t u(__half2 x)
    {
        uint32_t r;
        memcpy(&r, &x, 4);
        return r;
    }
    __device__ static uint32_t vmin(uint32_t a, uint32_t b) { return u(__hmin2(v(a), v(b))); }
    __device__ static uint32_t vmax(uint32_t a, uint32_t b) { return u(__hmax2(v(a), v(b))); }
    __device__ static uint32_t ge_mask(uint32_t a, uint32_t b) { return __hge2_mask(v(a), v(b)); }
};

// Neighbours in value order of a 16-bit sign-magnitude float (both zeros are
// the value 0; the infinities are fixed points).
template <int DT>
__device__ __forceinline__ uint16_t next_up(uint16_t b)
{
    // Value order: +-0 -> smallest positive subnormal, negatives step towards
    // zero, positives away from it, +inf stays (selects, no branches).
    const uint16_t up = (b & 0x8000u) ? (uint16_t)(b - 1) : (uint16_t)(b + 1);
    const uint16_t r = (b & 0x7fffu) == 0 ? (uint16_t)0x0001u : up;
    return b == In<DT>::kInf ? b : r;
}
template <int DT>
__device__ __forceinline__ uint16_t next_down(uint16_t b)
{
    if ((b & 0x7fffu) == 0) return 0x8001u;
    if (b & 0x8000u) return b == In<DT>::kNegInf ? b : (uint16_t)(b + 1);
    return (uint16_t)(b - 1);
}

// Does input value x reach threshold e: fl32(x - z) > e (the definition's
// fp32 subtraction, compared against the exact fp32 bound)?
template <int DT>
__device__ __forceinline__ bool passes(uint16_t x, float e, float z)
{
    return __fsub_rn(In<DT>::f(x), z) > e;
}

// Smallest input value x (as bits) with fl32(x - z) > e; +inf when none.
// fl32(x - z) is non-decreasing in x, so {x : passes} is an upper set.  The
// start c = RD_dtype(RD_fp32(z + e)) satisfies c - z <= e, so it never
// passes; stepping up reaches the least passing value, normally in one or two
// steps.  Should that not happen within 4 steps, a binary search over the
// value-ordered 16-bit patterns settles it.
template <int DT>
__device__ __noinline__ uint16_t min_passing_slow(uint16_t x, float e, float z);

template <int DT>
__device__ __forceinline__ uint16_t min_passing(float e, float z)
{
    if (!(e < __int_as_float(0x7f800000))) return In<DT>::kInf;
    // The first two steps, evaluated side by side; rarely more are needed.
    const uint16_t x0 = In<DT>::from_float_rd(__fadd_rd(z, e));
    const uint16_t x1 = next_up<DT>(x0), x2 = next_up<DT>(x1);
    const bool p1 = passes<DT>(x1, e, z), p2 = passes<DT>(x2, e, z);
    if (p1 | p2) return p1 ? x1 : x2;
    return min_passing_slow<DT>(x2, e, z);
}

// Continuation from x (not passing): two more steps, then a bisection.
template <int DT>
__device__ __noinline__ uint16_t min_passing_slow(uint16_t x, float e, float z)
{
#pragma unroll 1
    for (int i = 0; i < 2; ++i) {
        x = next_up<DT>(x);
        if (passes<DT>(x, e, z)) return x;
    }
    // Value-order key of a pattern: negatives reversed below the positives.
    auto key_bits = [](int k) -> uint16_t {
        return k < 0x8000 ? (uint16_t)(0xffff - k) : (uint16_t)(k - 0x8000);
    };
    int lo = 0x8000 - (In<DT>::kInf & 0x7fff), hi = 0x8000 + In<DT>::kInf;  // -inf .. +inf
#pragma unroll 1
    while (lo < hi) {
        const int mid = (lo + hi) >> 1;
        if (passes<DT>(key_bits(mid), e, z)) hi = mid;
        else lo = mid + 1;
    }
    return key_bits(lo);
}

// Two codes of a channel pair x (packed) against packed thresholds t1..t3:
// bit pattern (c_lo at bits 0-1, c_hi at bits 16-17).  Masks m_k are 0xffff
// per half where x >= t_k; since m1 >= m2 >= m3, bit1 of a code is m2 and
// bit0 is m1 ^ m2 ^ m3.
template <int DT>
__device__ __forceinline__ uint32_t code_pair_bits(uint32_t x, uint32_t t1, uint32_t t2, uint32_t t3)
{
    const uint32_t m1 = In<DT>::ge_mask(x, t1), m2 = In<DT>::ge_mask(x, t2), m3 = In<DT>::ge_mask(x, t3);
    uint32_t a, r;
    asm("lop3.b32 %0, %1, %2, %3, 0x28;" : "=r"(a) : "r"(m1), "r"(m3), "r"(0x00010001u));  // (m1^m3)&K
    asm("lop3.b32 %0, %1, %2, %3, 0x78;" : "=r"(r) : "r"(a), "r"(m2), "r"(0x00030003u));  // a^(m2&M)
    return r;
}

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem)
{
    uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

constexpr int kQuantThreads = 256;
#ifndef KIVI_QUANT_CTAS
#define KIVI_QUANT_CTAS 4   // resident CTAs per SM (persistent grid; measured best)
#endif

// The CTA works as two independent halves: threads [0, D) take the key tile,
// the rest the value tile, each with its own named barrier (ids 1 and 2), so
// that neither waits for the other; the halves share only the SM.
template <int D>
__device__ __forceinline__ void half_sync(int tid)
{
    if (tid < D)
        asm volatile("bar.sync 1, %0;" ::"n"(D) : "memory");
    else
        asm volatile("bar.sync 2, %0;" ::"n"(kQuantThreads - D) : "memory");
}

template <int D>
struct QuantSmem {
    static constexpr int RS = D + 8;                      // padded row, elements
    static constexpr int TILE = 32 * RS;                  // one K or V tile
    static constexpr int TILES_BYTES = 2 * 2 * TILE * 2;  // 2 buffers x (K, V)
    static constexpr int THRK = TILES_BYTES;              // uint16 [3][D]
    static constexpr int TS = 4 * (D / 32) + 4;           // padded token row of thrV
    static constexpr int THRV = THRK + 3 * D * 2;         // uint16 [32][TS]: [D/32][4] + pad
    static constexpr int OUTB = (THRV + 32 * TS * 2 + 15) / 16 * 16;
    static constexpr int BYTES = OUTB + 24 * D;
};

// Work item of a quantizer launch: group g of sequence s (destination group
// g_dst0 + g), or (copy) the residual copy of sequence s's source rows
// [copy_row0, copy_row0 + r_copy).
struct QItem {
    long long s;
    int g, g_dst0, r_copy, copy_row0;
    bool copy;
};

template <bool SEG>
__device__ __forceinline__ QItem locate(const QuantParams &p, const QuantSegs *sg, long long item)
{
    QItem q;
    if constexpr (SEG) {
        int lo = 0, hi = sg->nseg - 1;   // the last segment with item0 <= item
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (sg->item0[mid] <= item) lo = mid;
            else hi = mid - 1;
        }
        const long long local = item - sg->item0[lo];
        const long long ngi = (long long)sg->nseq[lo] * sg->n_g[lo];
        q.g_dst0 = sg->g_dst0[lo];
        q.r_copy = sg->r_copy[lo];
        q.copy_row0 = sg->copy_row0[lo];
        q.copy = local >= ngi;
        if (q.copy) {
            q.s = sg->seq0[lo] + (local - ngi);
            q.g = 0;
        } else {
            const long long si = local / sg->n_g[lo];
            q.s = sg->seq0[lo] + si;
            q.g = (int)(local - si * sg->n_g[lo]);
        }
    } else {
        const long long n_group_items = p.seqs * (long long)p.n_g;
        q.g_dst0 = (int)p.g_dst0;
        q.r_copy = p.r_copy;
        q.copy_row0 = (int)p.copy_row0;
        q.copy = item >= n_group_items;
        if (q.copy) {
            q.s = item - n_group_items;
            q.g = 0;
        } else {
            q.s = div_floor(item, p.div_ng);
            q.g = (int)(item - q.s * p.n_g);
        }
    }
    return q;
}

template <int D, int DT>
__device__ void quantize_tile(const QuantParams &p, long long s, int g, long long g_dst0,
                              const uint16_t *tk, const uint16_t *tv, uint16_t *thrK, uint16_t *thrV,
                              uint8_t *outb)
{
    using L = Layout<D>;
    using H = In<DT>;
    constexpr int RS = QuantSmem<D>::RS;
    constexpr int NJ = L::NJ, CPL = L::CPL, TPW = L::TPW, KW = L::KW;
    const int tid = threadIdx.x;

    if (tid < D) {
        // Keys, per channel: thread (pair cp, row set hh) takes 16 rows of a
        // channel pair, rows 8b + 4hh + {0..3} (the two sets 4 rows apart sit
        // in disjoint banks); they meet through a shuffle with lane ^ 1.
        const int cp = tid >> 1, hh = tid & 1;
        const uint16_t *col = tk + hh * 4 * RS + 2 * cp;
        auto row = [&](int i) { return (const uint32_t *)(col + (((i >> 2) << 3) + (i & 3)) * RS); };
        uint32_t mn = *row(0), mx = mn;
        uint32_t mn1 = *row(1), mx1 = mn1;
#pragma unroll
        for (int r = 2; r < 16; r += 2) {
            const uint32_t v0 = *row(r);
            const uint32_t v1 = *row(r + 1);
            mn = H::vmin(mn, v0);
            mx = H::vmax(mx, v0);
            mn1 = H::vmin(mn1, v1);
            mx1 = H::vmax(mx1, v1);
        }
        mn = H::vmin(mn, mn1);
        mx = H::vmax(mx, mx1);
        mn = H::vmin(mn, __shfl_xor_sync(0xffffffffu, mn, 1));
        mx = H::vmax(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        const int ch = 2 * cp + hh;
        const uint16_t mnb = (uint16_t)(hh ? mn >> 16 : mn), mxb = (uint16_t)(hh ? mx >> 16 : mx);
        const CodeParams c = code_params(H::f(mnb), H::f(mxb));
        thrK[ch] = min_passing<DT>(c.e1, c.z);
        thrK[D + ch] = min_passing<DT>(c.e2, c.z);
        thrK[2 * D + ch] = min_passing<DT>(c.e3, c.z);
        const int off = L::KM + km_offset<D>(k_perm_index<D>(ch));
        *(uint16_t *)(outb + off) = c.s_bits;
        *(uint16_t *)(outb + off + D / 16) = c.z_bits;
    } else {
        // Values, per token: one (token, 32-channel group) per thread.
        for (int qd = tid - D; qd < 32 * NJ; qd += kQuantThreads - D) {
            const int t = qd / NJ, j = qd % NJ;
            const uint4 *row = (const uint4 *)(tv + t * RS + j * 32);
            uint4 a = row[0];
            uint32_t mn = H::vmin(a.x, a.y), mx = H::vmax(a.x, a.y);
            mn = H::vmin(mn, H::vmin(a.z, a.w));
            mx = H::vmax(mx, H::vmax(a.z, a.w));
#pragma unroll
            for (int q = 1; q < 4; ++q) {
                a = row[q];
                mn = H::vmin(mn, H::vmin(H::vmin(a.x, a.y), H::vmin(a.z, a.w)));
                mx = H::vmax(mx, H::vmax(H::vmax(a.x, a.y), H::vmax(a.z, a.w)));
            }
            mn = H::vmin(mn, (mn >> 16) | (mn << 16));
            mx = H::vmax(mx, (mx >> 16) | (mx << 16));
            const CodeParams c = code_params(H::f((uint16_t)mn), H::f((uint16_t)mx));
            uint16_t *tr = thrV + t * QuantSmem<D>::TS + j * 4;
            tr[0] = min_passing<DT>(c.e1, c.z);
            tr[1] = min_passing<DT>(c.e2, c.z);
            tr[2] = min_passing<DT>(c.e3, c.z);
            const int off = L::VM + t * (D / 8) + j * 2;
            *(uint16_t *)(outb + off) = c.s_bits;
            *(uint16_t *)(outb + off + D / 16) = c.z_bits;
        }
    }
    half_sync<D>(tid);

    if (tid < D) {
        // Key code words: thread -> (lane, token pair, word slot k); tokens tok
        // and tok+2 of the lane share the word's 16 channels and thresholds.
        const int lane = tid / (2 * KW), rem = tid % (2 * KW);
        const int tokp = rem / KW, k = rem % KW;
        const int cs = lane & 3, tq = lane >> 2;
        // The word's 16 channels come in runs of RUN contiguous channels
        // (one run when D >= 128, one per RoPE half when D == 64).
        constexpr int RUN = L::HALF < 16 ? L::HALF : 16;
        uint32_t t1[8], t2[8], t3[8];
        int base[16 / RUN];
#pragma unroll
        for (int r = 0; r < 16 / RUN; ++r) {
            base[r] = k_channel<D>(cs, 16 * k + r * RUN);
#pragma unroll
            for (int v = 0; v < RUN / 8; ++v) {
                const uint4 a = *(const uint4 *)(thrK + base[r] + 8 * v);
                const uint4 b = *(const uint4 *)(thrK + D + base[r] + 8 * v);
                const uint4 c = *(const uint4 *)(thrK + 2 * D + base[r] + 8 * v);
                const int i0 = r * (RUN / 2) + 4 * v;
                t1[i0] = a.x; t1[i0 + 1] = a.y; t1[i0 + 2] = a.z; t1[i0 + 3] = a.w;
                t2[i0] = b.x; t2[i0 + 1] = b.y; t2[i0 + 2] = b.z; t2[i0 + 3] = b.w;
                t3[i0] = c.x; t3[i0 + 1] = c.y; t3[i0 + 2] = c.z; t3[i0 + 3] = c.w;
            }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int tok = tokp + 2 * h;
            const uint16_t *row = tk + (4 * tq + tok) * RS;
            uint32_t x[8];
#pragma unroll
            for (int r = 0; r < 16 / RUN; ++r)
#pragma unroll
                for (int v = 0; v < RUN / 8; ++v) {
                    const uint4 a = *(const uint4 *)(row + base[r] + 8 * v);
                    const int i0 = r * (RUN / 2) + 4 * v;
                    x[i0] = a.x; x[i0 + 1] = a.y; x[i0 + 2] = a.z; x[i0 + 3] = a.w;
                }
            uint32_t word = 0;
#pragma unroll
            for (int i = 7; i >= 0; --i) word = word * 4u + code_pair_bits<DT>(x[i], t1[i], t2[i], t3[i]);
            *(uint32_t *)(outb + L::KC + code_word_offset(lane, tok * KW + k)) = word;
        }
    } else {
        // Value code words: thread -> (lane = 16*th + co, word u).
        for (int vp = tid - D; vp < 2 * D; vp += kQuantThreads - D) {
            const int lane = vp / L::WPL, u = vp % L::WPL;
            const int co = lane & 15, th = lane >> 4;
            const int j = co * CPL / 32;
            // TPW tokens x CPL channels: per token one threshold triple (one
            // 8-byte load) and CPL/2 channel pairs (CPL/8 16-byte loads).
            uint32_t x[8], b1[TPW], b2[TPW], b3[TPW];
#pragma unroll
            for (int tt = 0; tt < TPW; ++tt) {
                const int t = 16 * th + u * TPW + tt;
                const uint2 tr = *(const uint2 *)(thrV + t * QuantSmem<D>::TS + j * 4);
                b1[tt] = __byte_perm(tr.x, 0, 0x1010);
                b2[tt] = __byte_perm(tr.x, 0, 0x3232);
                b3[tt] = __byte_perm(tr.y, 0, 0x1010);
                const uint16_t *row = tv + t * RS + co * CPL;
                if constexpr (CPL >= 8) {
#pragma unroll
                    for (int v = 0; v < CPL / 8; ++v) {
                        const uint4 a = *(const uint4 *)(row + 8 * v);
                        const int i0 = tt * (CPL / 2) + 4 * v;
                        x[i0] = a.x; x[i0 + 1] = a.y; x[i0 + 2] = a.z; x[i0 + 3] = a.w;
                    }
                } else {
                    const uint2 a = *(const uint2 *)row;
                    x[tt * 2] = a.x;
                    x[tt * 2 + 1] = a.y;
                }
            }
            uint32_t word = 0;
#pragma unroll
            for (int i = 7; i >= 0; --i) {
                const int tt = i / (CPL / 2);
                word = word * 4u + code_pair_bits<DT>(x[i], b1[tt], b2[tt], b3[tt]);
            }
            *(uint32_t *)(outb + L::VC + code_word_offset(lane, u)) = word;
        }
    }
    half_sync<D>(tid);

    // Each half stores its own 12*D bytes: [Kc, Km) and [Vc, Vm).
    uint4 *dst = (uint4 *)(p.packed + ((s * p.ngcap) + g_dst0 + g) * (long long)L::GB);
    {
        const int h = tid < D ? 0 : 1, ht = tid < D ? tid : tid - D;
        const int nthr = tid < D ? D : kQuantThreads - D;
        const uint4 *src = (const uint4 *)(outb + h * 12 * D);
        uint4 *d = dst + h * (12 * D / 16);
        for (int c = ht; c < 12 * D / 16; c += nthr) d[c] = src[c];
    }

    if (p.newK != nullptr && g == 0) {
        // The flush has read residual slot 0 into shared memory (each half's
        // tile was complete before that half's first barrier): the new token
        // may land, each half writing its own row.
        const int which = tid < D ? 0 : 1, ht = tid < D ? tid : tid - D;
        for (int q = ht; q < D / 8; q += (tid < D ? D : kQuantThreads - D)) {
            const uint16_t *src = (which ? p.newV : p.newK) + s * D + q * 8;
            uint16_t *d = (which ? p.resV : p.resK) + s * (long long)p.R * D + q * 8;
            *(uint4 *)d = *(const uint4 *)src;
        }
    }
}

template <int D, int DT, bool SEG>
__device__ __forceinline__ void quant_body(const QuantParams &p, const QuantSegs *sg)
{
    using S = QuantSmem<D>;
    extern __shared__ __align__(16) unsigned char smem[];
    uint16_t *tiles = (uint16_t *)smem;
    uint16_t *thrK = (uint16_t *)(smem + S::THRK);
    uint16_t *thrV = (uint16_t *)(smem + S::THRV);
    uint8_t *outb = smem + S::OUTB;

    long long n_items;
    if constexpr (SEG) n_items = sg->item0[sg->nseg];
    else n_items = p.seqs * (long long)p.n_g + (p.r_copy > 0 ? p.seqs : 0);
    const int tid = threadIdx.x;

    auto issue = [&](long long item, int buf) {
        if (item >= n_items) return;
        const QItem q = locate<SEG>(p, sg, item);
        if (q.copy) return;
        const long long s = q.s;
        const int g = q.g;
        const long long row0 = s * p.src_seq_rows + (long long)g * 32;
        const uint16_t *k = p.srcK + row0 * D;
        const uint16_t *v = p.srcV + row0 * D;
        // The key half copies the key tile, the value half the value tile.
        const bool kh = tid < D;
        uint16_t *t = tiles + (buf * 2 + (kh ? 0 : 1)) * S::TILE;
        const uint16_t *src = kh ? k : v;
        const int ht = kh ? tid : tid - D, nthr = kh ? D : kQuantThreads - D;
        for (int c = ht; c < 32 * (D / 8); c += nthr) {
            const int row = c / (D / 8), col = (c % (D / 8)) * 8;
            cp_async16(t + row * S::RS + col, src + row * D + col);
        }
    };

    long long item = blockIdx.x;
    int buf = 0;
    issue(item, 0);
    cp_async_commit();
    for (; item < n_items; item += gridDim.x, buf ^= 1) {
        issue(item + gridDim.x, buf ^ 1);
        cp_async_commit();
        cp_async_wait<1>();
        half_sync<D>(tid);
        const QItem q = locate<SEG>(p, sg, item);
        if (!q.copy) {
            quantize_tile<D, DT>(p, q.s, q.g, q.g_dst0, tiles + (buf * 2 + 0) * S::TILE,
                                 tiles + (buf * 2 + 1) * S::TILE, thrK, thrV, outb);
        } else {
            // Prefill residual: rows [copy_row0, copy_row0 + r_copy) -> slots.
            const long long s = q.s;
            const long long n16 = (long long)q.r_copy * (D / 8);
            const uint4 *sk = (const uint4 *)(p.srcK + (s * p.src_seq_rows + q.copy_row0) * D);
            const uint4 *sv = (const uint4 *)(p.srcV + (s * p.src_seq_rows + q.copy_row0) * D);
            uint4 *dk = (uint4 *)(p.resK + s * (long long)p.R * D);
            uint4 *dv = (uint4 *)(p.resV + s * (long long)p.R * D);
            const bool kh = tid < D;
            const uint4 *sr = kh ? sk : sv;
            uint4 *dr = kh ? dk : dv;
            for (long long c = kh ? tid : tid - D; c < n16; c += kh ? D : kQuantThreads - D) dr[c] = sr[c];
        }
        half_sync<D>(tid);
    }
    cp_async_wait<0>();
}

template <int D, int DT>
__global__ void __launch_bounds__(kQuantThreads, KIVI_QUANT_CTAS) quant_kernel(QuantParams p)
{
    quant_body<D, DT, false>(p, nullptr);
}

template <int D, int DT>
__global__ void __launch_bounds__(kQuantThreads, KIVI_QUANT_CTAS)
    quant_kernel_seg(QuantParams p, const __grid_constant__ QuantSegs sg)
{
    quant_body<D, DT, true>(p, &sg);
}

// Plain append: token rows [seqs][D] -> residual slot `slot` of each sequence.
// One 16-byte chunk of k_t and of v_t per thread; N16 = D/8 chunks per row.
template <int N16>
__global__ void append_kernel(const uint4 *k, const uint4 *v, uint4 *resK, uint4 *resV,
                              long long seqs, int R, int slot)
{
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= seqs * N16) return;
    const long long s = i / N16;
    const long long d = (s * R + slot) * N16 + (i % N16);
    const uint4 a = __ldcs(k + i), b = __ldcs(v + i);
    resK[d] = a;
    resV[d] = b;
}

// Append into per-batch-element slots: sequence s = b*H_kv + h takes slot
// st.slot[b], or nothing when it is negative.
template <int N16>
__global__ void append_slots_kernel(const uint4 *k, const uint4 *v, uint4 *resK, uint4 *resV,
                                    long long seqs, int H_kv, int R, const __grid_constant__ SlotTab st)
{
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= seqs * N16) return;
    const long long s = i / N16;
    const int slot = st.slot[s / H_kv];
    if (slot < 0) return;
    const long long d = (s * R + slot) * N16 + (i % N16);
    const uint4 a = __ldcs(k + i), b = __ldcs(v + i);
    resK[d] = a;
    resV[d] = b;
}

int num_sms()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
    return n;
}

template <int D, int DT>
static cudaError_t launch_quant_t(const QuantParams &p, const QuantSegs *segs, cudaStream_t st)
{
    using S = QuantSmem<D>;
    const long long items = segs ? segs->item0[segs->nseg]
                                 : p.seqs * (long long)p.n_g + (p.r_copy > 0 ? p.seqs : 0);
    if (items == 0) return cudaSuccess;
    long long grid = (long long)num_sms() * KIVI_QUANT_CTAS;
    if (grid > items) grid = items;
    QuantParams q = p;
    q.div_ng = make_magic((unsigned long long)(p.n_g > 0 ? p.n_g : 1));
    if (segs) {
        static PerDeviceOnce once;
        const cudaError_t e = set_smem_once(once, quant_kernel_seg<D, DT>, S::BYTES);
        if (e != cudaSuccess) return e;
        quant_kernel_seg<D, DT><<<(unsigned)grid, kQuantThreads, S::BYTES, st>>>(q, *segs);
    } else {
        static PerDeviceOnce once;
        const cudaError_t e = set_smem_once(once, quant_kernel<D, DT>, S::BYTES);
        if (e != cudaSuccess) return e;
        quant_kernel<D, DT><<<(unsigned)grid, kQuantThreads, S::BYTES, st>>>(q);
    }
    return cudaGetLastError();
}

cudaError_t launch_quant(int D, int dtype, const QuantParams &p, const QuantSegs *segs, cudaStream_t st)
{
    if (D == 64) return dtype ? launch_quant_t<64, 1>(p, segs, st) : launch_quant_t<64, 0>(p, segs, st);
    if (D == 128) return dtype ? launch_quant_t<128, 1>(p, segs, st) : launch_quant_t<128, 0>(p, segs, st);
    return cudaErrorInvalidValue;
}

cudaError_t launch_append(int D, const uint16_t *k, const uint16_t *v, uint16_t *resK,
                          uint16_t *resV, long long seqs, int R, int slot, cudaStream_t st)
{
    const long long total = seqs * (D / 8);
    const int block = 128;
    const long long grid = (total + block - 1) / block;
    if (D == 64)
        append_kernel<8><<<(unsigned)grid, block, 0, st>>>((const uint4 *)k, (const uint4 *)v,
                                                          (uint4 *)resK, (uint4 *)resV, seqs, R, slot);
    else
        append_kernel<16><<<(unsigned)grid, block, 0, st>>>((const uint4 *)k, (const uint4 *)v,
                                                           (uint4 *)resK, (uint4 *)resV, seqs, R, slot);
    return cudaGetLastError();
}

cudaError_t launch_append_slots(int D, const uint16_t *k, const uint16_t *v, uint16_t *resK,
                                uint16_t *resV, long long seqs, int H_kv, int R, const SlotTab &slots,
                                cudaStream_t st)
{
    const long long total = seqs * (D / 8);
    const int block = 128;
    const long long grid = (total + block - 1) / block;
    if (D == 64)
        append_slots_kernel<8><<<(unsigned)grid, block, 0, st>>>((const uint4 *)k, (const uint4 *)v,
                                                                 (uint4 *)resK, (uint4 *)resV, seqs, H_kv, R,
                                                                 slots);
    else
        append_slots_kernel<16><<<(unsigned)grid, block, 0, st>>>((const uint4 *)k, (const uint4 *)v,
                                                                  (uint4 *)resK, (uint4 *)resV, seqs, H_kv, R,
                                                                  slots);
    return cudaGetLastError();
}

}  // namespace kivi
