// kivi_quant.cu -- prefill quantizer and residual append/flush kernels.
//
// Keys are grouped per channel over 32 consecutive tokens and values per token
// over 32 consecutive channels ("KIVI Quantization Secures Llama-2 Accuracy at
// Two Bits", paragraphs 2-3; record kv-efficiency/kivi-2bit-llama2-13b-mha-4k,
// "Quant method": kivi-2bit-per-channel-k-per-token-v).  One warp quantizes
// one key tile or one value tile (32 tokens x D channels) at a time, holding
// it in registers, and writes its half of the 24*D-byte group block; warps
// never wait for each other:
//   1. the tile is staged into the warp's shared buffer with cp.async (the
//      next tile's copy overlaps the current tile's parameters and codes) and
//      read row-wide into registers (keys: each lane takes D/32 channels of
//      every token; values: each lane takes the CPL channels of 16 tokens
//      that it owns in the block's code layout);
//   2. statistics with paired (bf16x2 / f16x2) min/max: per key channel
//      within the lane, per value token within the lane and then across the
//      lanes of its 32-channel group by shuffles;
//   3. each group's fp16 scale/zero and its three code thresholds.  The code
//      clamp(rint(fl(x - z) / s), 0, 3) equals the number of thresholds x has
//      reached, x_k being the smallest input value whose fp32 difference to z
//      passes the k-th exact fp32 bound (see code_params); x_k is found by a
//      search from z + E_k that evaluates the definition itself;
//   4. codes: two channels at a time, three paired `x >= x_k` compares give
//      lane masks, two logic ops turn them into the pair's two 2-bit codes at
//      their word position; key words are assembled across the lanes that
//      share them by shuffles;
//   5. value code words leave as coalesced 16-byte stores, key words as
//      4-byte stores that fill whole 16-byte chunks per warp store.
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
// start c = RD_dtype(RD_fp32(z + e)) satisfies c - z <= e (rounding to
// nearest is monotone and e is an fp32 value), so it never passes.  Its
// successor x1 lies above z + e, so it passes whenever x1 - z is exact in
// fp32, i.e. unless x1 and z are many binades apart; otherwise stepping on,
// and after three more steps a binary search over the value-ordered 16-bit
// patterns, settles it.
template <int DT>
__device__ __noinline__ uint16_t min_passing_slow(uint16_t x, float e, float z);

template <int DT>
__device__ __forceinline__ uint16_t min_passing(float e, float z)
{
    if (!(e < __int_as_float(0x7f800000))) return In<DT>::kInf;
    const uint16_t c = In<DT>::from_float_rd(__fadd_rd(z, e));
    // The successor of c in value order (c is finite: a rounding down of a
    // finite sum never gives +inf).
    const uint16_t x1 = (c & 0x7fffu) == 0 ? (uint16_t)0x0001u
                        : (c & 0x8000u)    ? (uint16_t)(c - 1)
                                           : (uint16_t)(c + 1);
    if (passes<DT>(x1, e, z)) return x1;
    return min_passing_slow<DT>(x1, e, z);
}

// Continuation from x (not passing): three more steps, then a bisection.
template <int DT>
__device__ __noinline__ uint16_t min_passing_slow(uint16_t x, float e, float z)
{
#pragma unroll 1
    for (int i = 0; i < 3; ++i) {
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

// ---- one warp per key tile or value tile ------------------------------------
// Work unit 2*item is the key tile of group item, 2*item + 1 its value tile
// (or, for a copy item, its key and value rows); a warp takes the units at
// positions gw, gw + W, ... (W warps in the grid, even) counted from the last
// unit down, so it always works on one kind of tile.  A warp holds its tile
// in registers and writes its own part of the group block; warps never wait
// for each other.

// Two codes of a channel pair x against packed thresholds t1..t3, placed at
// the word bits K1 (0x00010001 << 2i) and K3 (0x00030003 << 2i) of pair i.
// Masks m_k are 0xffff per half where x >= t_k; as m1 >= m2 >= m3, bit 1 of
// a code is m2 and bit 0 is m1 ^ m2 ^ m3.
template <int DT>
__device__ __forceinline__ uint32_t code_pair_at(uint32_t x, uint32_t t1, uint32_t t2, uint32_t t3, uint32_t K1,
                                                 uint32_t K3)
{
    const uint32_t m1 = In<DT>::ge_mask(x, t1), m2 = In<DT>::ge_mask(x, t2), m3 = In<DT>::ge_mask(x, t3);
    uint32_t a, r;
    asm("lop3.b32 %0, %1, %2, %3, 0x28;" : "=r"(a) : "r"(m1), "r"(m3), "r"(K1));  // (m1^m3)&K1
    asm("lop3.b32 %0, %1, %2, %3, 0x78;" : "=r"(r) : "r"(a), "r"(m2), "r"(K3));   // a^(m2&K3)
    return r;
}

// Packed (a.lo, b.lo) and (a.hi, b.hi) of two 16-bit pairs.
__device__ __forceinline__ uint32_t lo_halves(uint32_t a, uint32_t b) { return __byte_perm(a, b, 0x5410); }
__device__ __forceinline__ uint32_t hi_halves(uint32_t a, uint32_t b) { return __byte_perm(a, b, 0x7632); }

// Key tile: 32 tokens x D channels, one group per channel, staged in shared
// memory.  Lane l holds the CK = D/32 channels [CK*l, CK*l + CK) of all 32
// tokens (a whole row per warp load), so each channel's min/max,
// scale, zero and thresholds are the lane's own.  The lane's channel pairs
// are pairs i0, i0 + 1 of one 16-channel code word (a word of slice cs, local
// channels 16k..16k+15); the 4 (D = 128) or 8 (D = 64) lanes of a word OR
// their codes together in a transposing shuffle, which leaves each lane one
// complete word per chunk of 4 or 8 tokens.
template <int D, int DT, typename F>
__device__ __forceinline__ void key_tile(const uint16_t *tile, uint8_t *blk, int lane, F &&after_stats)
{
    using L = Layout<D>;
    using H = In<DT>;
    constexpr int CK = D / 32, NP = CK / 2;
    constexpr int NL = D == 128 ? 2 : 3;         // lanes per word = 2^NL
    constexpr int CH = 1 << NL;                  // tokens per chunk
    const int c0 = CK * lane;

    uint32_t x[32][NP];
#pragma unroll
    for (int t = 0; t < 32; ++t) {
        if constexpr (NP == 2) {
            const uint2 v = *(const uint2 *)(tile + t * D + c0);
            x[t][0] = v.x;
            x[t][1] = v.y;
        } else {
            x[t][0] = *(const uint32_t *)(tile + t * D + c0);
        }
    }

    // Per channel pair: min/max over the 32 tokens, then each channel's
    // parameters and thresholds (packed per pair: low half channel c, high
    // half channel c + 1).
    uint32_t T1[NP], T2[NP], T3[NP], mnp[NP], mxp[NP];
#pragma unroll
    for (int pp = 0; pp < NP; ++pp) {
        uint32_t mn[4], mx[4];
#pragma unroll
        for (int a = 0; a < 4; ++a) mn[a] = mx[a] = x[a][pp];
#pragma unroll
        for (int t = 4; t < 32; ++t) {
            mn[t & 3] = H::vmin(mn[t & 3], x[t][pp]);
            mx[t & 3] = H::vmax(mx[t & 3], x[t][pp]);
        }
        mnp[pp] = H::vmin(H::vmin(mn[0], mn[1]), H::vmin(mn[2], mn[3]));
        mxp[pp] = H::vmax(H::vmax(mx[0], mx[1]), H::vmax(mx[2], mx[3]));
    }
    after_stats();
    // One channel per iteration (a loop, to keep the code small): its 16-bit
    // min/max shift out of mn64/mx64 and its results shift into t*s, ss, zs.
    uint64_t mn64 = mnp[0], mx64 = mxp[0];
    if constexpr (NP == 2) {
        mn64 |= (uint64_t)mnp[1] << 32;
        mx64 |= (uint64_t)mxp[1] << 32;
    }
    uint64_t t1s = 0, t2s = 0, t3s = 0, ss = 0, zs = 0;
#pragma unroll 1
    for (int ch = 0; ch < CK; ++ch) {
        const CodeParams c = code_params(H::f((uint16_t)mn64), H::f((uint16_t)mx64));
        mn64 >>= 16;
        mx64 >>= 16;
        const int sh = 16 * ch;
        t1s |= (uint64_t)min_passing<DT>(c.e1, c.z) << sh;
        t2s |= (uint64_t)min_passing<DT>(c.e2, c.z) << sh;
        t3s |= (uint64_t)min_passing<DT>(c.e3, c.z) << sh;
        ss |= (uint64_t)c.s_bits << sh;
        zs |= (uint64_t)c.z_bits << sh;
    }
#pragma unroll
    for (int pp = 0; pp < NP; ++pp) {
        T1[pp] = (uint32_t)(t1s >> (32 * pp));
        T2[pp] = (uint32_t)(t2s >> (32 * pp));
        T3[pp] = (uint32_t)(t3s >> (32 * pp));
        // Channels c, c + 1 have consecutive permuted indices (even first).
        const int off = L::KM + km_offset<D>(k_perm_index<D>(c0 + 2 * pp));
        *(uint32_t *)(blk + off) = (uint32_t)(ss >> (32 * pp));
        *(uint32_t *)(blk + off + D / 16) = (uint32_t)(zs >> (32 * pp));
    }

    // Word position of the lane's pairs and of its words after the exchange.
    const int P0 = k_perm_index<D>(c0);
    const int cs = P0 / (D / 4), L0 = P0 % (D / 4);
    const int k = L0 / 16, i0 = (L0 % 16) / 2;
    uint32_t K1[NP], K3[NP];
#pragma unroll
    for (int pp = 0; pp < NP; ++pp) {
        K1[pp] = 0x00010001u << (2 * (i0 + pp));
        K3[pp] = 0x00030003u << (2 * (i0 + pp));
    }
    // Lane bit of exchange level r: 0, 1 and (D = 64) 4; token offset kept.
    constexpr int LB[3] = {0, 1, 4};
    int jt = 0;
#pragma unroll
    for (int r = 0; r < NL; ++r) jt |= ((lane >> LB[r]) & 1) << r;
    const int off0 = L::KC + code_word_offset(4 * (jt / 4) + cs, (jt % 4) * L::KW + k);

#pragma unroll
    for (int m = 0; m < 32 / CH; ++m) {
        uint32_t w[CH];
#pragma unroll
        for (int q = 0; q < CH; ++q) {
            const int t = m * CH + q;
            uint32_t acc = 0;
#pragma unroll
            for (int pp = 0; pp < NP; ++pp) acc |= code_pair_at<DT>(x[t][pp], T1[pp], T2[pp], T3[pp], K1[pp], K3[pp]);
            w[q] = acc;
        }
#pragma unroll
        for (int r = 0; r < NL; ++r) {
            const bool b = (lane >> LB[r]) & 1;
#pragma unroll
            for (int e = 0; e < (CH >> (r + 1)); ++e) {
                const uint32_t lo = w[2 * e], hi = w[2 * e + 1];
                const uint32_t send = b ? lo : hi, keep = b ? hi : lo;
                w[e] = keep | __shfl_xor_sync(0xffffffffu, send, 1 << LB[r]);
            }
        }
        // w[0]: the word of token m*CH + jt (layout lane 4*(t/4) + cs, word
        // (t%4)*KW + k); consecutive chunks are CH*16 bytes apart.
        *(uint32_t *)(blk + off0 + m * CH * 16) = w[0];
    }
}

// Value tile: 32 tokens x D channels, one group per (token, 32 channels).
// Lane l = 16*th + co holds exactly what it owns in the block's value codes:
// channels [co*CPL, (co+1)*CPL) of tokens 16th..16th+15.  A token's group
// spans LG = 32/CPL lanes; they reduce its (min, -max) in a transposing
// shuffle that leaves each lane 16/LG of the tokens, whose parameters it
// computes and publishes (thresholds replicated in both halves) in the warp's
// shared array `thr` [32 tokens][NJ].
template <int D, int DT, typename F>
__device__ __forceinline__ void value_tile(const uint16_t *tile, uint8_t *blk, int lane, uint4 *thr,
                                           F &&after_stats)
{
    using L = Layout<D>;
    using H = In<DT>;
    constexpr int CPL = L::CPL, NPV = CPL / 2, TPW = L::TPW, NJ = L::NJ, WPL = L::WPL;
    constexpr int LG = kG / CPL;              // lanes per value group
    constexpr int NLV = LG == 4 ? 2 : 3;      // log2(LG)
    constexpr int TL = 16 / LG;               // tokens per lane after the exchange
    const int co = lane & 15, th = lane >> 4;
    const int j = co * CPL / kG, jl = lane & (LG - 1);

    uint32_t x[16][NPV];
    const uint16_t *base = tile + (16 * th) * D + co * CPL;
#pragma unroll
    for (int tt = 0; tt < 16; ++tt) {
        if constexpr (NPV == 4) {
            const uint4 v = *(const uint4 *)(base + tt * D);
            x[tt][0] = v.x;
            x[tt][1] = v.y;
            x[tt][2] = v.z;
            x[tt][3] = v.w;
        } else {
            const uint2 v = *(const uint2 *)(base + tt * D);
            x[tt][0] = v.x;
            x[tt][1] = v.y;
        }
    }

    // (min, -max) of each token over the lane's channels, packed.
    uint32_t M[16];
#pragma unroll
    for (int tt = 0; tt < 16; ++tt) {
        uint32_t mn = x[tt][0], mx = x[tt][0];
#pragma unroll
        for (int pp = 1; pp < NPV; ++pp) {
            mn = H::vmin(mn, x[tt][pp]);
            mx = H::vmax(mx, x[tt][pp]);
        }
        const uint32_t nmx = mx ^ 0x80008000u;
        M[tt] = H::vmin(lo_halves(mn, nmx), hi_halves(mn, nmx));
    }
    after_stats();
    // Over the LG lanes of the group: level r keeps the tokens whose bit r is
    // the lane's bit r.  M[m] then holds token m*LG + jl.
#pragma unroll
    for (int r = 0; r < NLV; ++r) {
        const bool b = (lane >> r) & 1;
#pragma unroll
        for (int e = 0; e < (16 >> (r + 1)); ++e) {
            const uint32_t lo = M[2 * e], hi = M[2 * e + 1];
            const uint32_t send = b ? lo : hi, keep = b ? hi : lo;
            M[e] = H::vmin(keep, __shfl_xor_sync(0xffffffffu, send, 1 << r));
        }
    }
    __syncwarp();   // the previous tile's thresholds have been read
    // One token per iteration (a loop, to keep the code small): M rotates.
#pragma unroll 1
    for (int m = 0; m < TL; ++m) {
        const uint32_t cur = M[0];
#pragma unroll
        for (int k = 0; k + 1 < TL; ++k) M[k] = M[k + 1];
        const int t = 16 * th + m * LG + jl;
        const float mnf = H::f((uint16_t)cur);
        const float mxf = -H::f((uint16_t)(cur >> 16));
        const CodeParams c = code_params(mnf, mxf);
        const uint32_t t1 = min_passing<DT>(c.e1, c.z), t2 = min_passing<DT>(c.e2, c.z),
                       t3 = min_passing<DT>(c.e3, c.z);
        thr[t * NJ + j] = make_uint4(t1 * 0x10001u, t2 * 0x10001u, t3 * 0x10001u, 0u);
        const int off = L::VM + t * (D / 8) + j * 2;
        *(uint16_t *)(blk + off) = c.s_bits;
        *(uint16_t *)(blk + off + D / 16) = c.z_bits;
    }
    __syncwarp();

    // Word u: tokens 16th + u*TPW + q, pair i = q*NPV + pp at bits 2i, 16+2i.
    uint32_t wv[WPL];
#pragma unroll
    for (int u = 0; u < WPL; ++u) {
        uint4 b[TPW];
#pragma unroll
        for (int q = 0; q < TPW; ++q) b[q] = thr[(16 * th + u * TPW + q) * NJ + j];
        uint32_t word = 0;
#pragma unroll
        for (int i = 7; i >= 0; --i) {
            const int q = i / NPV, pp = i % NPV;
            word = word * 4u + code_pair_bits<DT>(x[u * TPW + q][pp], b[q].x, b[q].y, b[q].z);
        }
        wv[u] = word;
    }
#pragma unroll
    for (int c = 0; c < WPL / 4; ++c)
        *(uint4 *)(blk + L::VC + (c * 32 + lane) * 16) = make_uint4(wv[4 * c], wv[4 * c + 1], wv[4 * c + 2], wv[4 * c + 3]);
}

constexpr int kQuantWarps = 8;   // warps per CTA

// Shared memory per warp: the staged tile (32 rows of D), then the value
// tile's thresholds [32 tokens][NJ].
template <int D>
struct QuantWarpSmem {
    static constexpr int TILE = 32 * D * 2;
    static constexpr int THR = 32 * Layout<D>::NJ * 16;
    static constexpr int PER_WARP = TILE + THR;
    static constexpr int BYTES = kQuantWarps * PER_WARP;
};

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem)
{
    const uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// A warp's units, one after another; the tile of the next unit is staged into
// the warp's buffer (cp.async) as soon as the current tile's statistics have
// consumed the buffer, so its load overlaps the parameters and codes.
template <int D, int DT, bool SEG>
__device__ __forceinline__ void quant_warps(const QuantParams &p, const QuantSegs *sg)
{
    using S = QuantWarpSmem<D>;
    extern __shared__ __align__(16) unsigned char qsm[];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    uint16_t *tile = (uint16_t *)(qsm + wid * S::PER_WARP);
    uint4 *thr = (uint4 *)(qsm + wid * S::PER_WARP + S::TILE);
    long long n_items;
    if constexpr (SEG) n_items = sg->item0[sg->nseg];
    else n_items = p.seqs * (long long)p.n_g + (p.r_copy > 0 ? p.seqs : 0);
    const long long n_units = 2 * n_items;
    const long long nw = (long long)gridDim.x * kQuantWarps;

    // Units run from the last down, so that the residual copies (the last
    // items) start first and overlap the tiles.
    auto item_of = [&](long long unit) { return (n_units - 1 - unit) >> 1; };
    // Stage unit u's tile (nothing for a copy item).
    auto stage = [&](const QItem &q, bool vhalf) {
        if (q.copy) return;
        const uint4 *src =
            (const uint4 *)((vhalf ? p.srcV : p.srcK) + (q.s * p.src_seq_rows + (long long)q.g * 32) * D);
#pragma unroll
        for (int c = 0; c < S::TILE / 16 / 32; ++c) cp_async16((uint4 *)tile + c * 32 + lane, src + c * 32 + lane);
    };

    long long unit = (long long)blockIdx.x * kQuantWarps + wid;
    // Position unit runs work unit n_units - 1 - unit (value tile when odd);
    // nw is even, so a warp keeps its kind of tile.
    const bool vhalf = (n_units - 1 - unit) & 1;
    if (unit >= n_units) return;
    QItem q = locate<SEG>(p, sg, item_of(unit));
    stage(q, vhalf);
    cp_async_commit();
    for (;;) {
        const long long next = unit + nw;
        const bool has_next = next < n_units;
        QItem qn = q;
        if (has_next) qn = locate<SEG>(p, sg, item_of(next));
        // After the current tile's statistics: stage the next tile.
        auto after_stats = [&]() {
            __syncwarp();
            if (has_next) stage(qn, vhalf);
            cp_async_commit();
        };
        if (q.copy) {
            // Prefill residual: source rows [copy_row0, copy_row0 + r_copy)
            // -> slots, 32 rows at a time through the warp's buffer (one
            // round trip to memory per 32 rows), then the next tile is staged.
            const uint4 *sr = (const uint4 *)((vhalf ? p.srcV : p.srcK) + (q.s * p.src_seq_rows + q.copy_row0) * D);
            uint4 *dr = (uint4 *)((vhalf ? p.resV : p.resK) + q.s * (long long)p.R * D);
            uint4 *buf = (uint4 *)tile;
            for (int r0 = 0; r0 < q.r_copy; r0 += 32) {
                const int n16 = (q.r_copy - r0 < 32 ? q.r_copy - r0 : 32) * (D / 8);
                const int c0 = r0 * (D / 8);
                for (int c = lane; c < n16; c += 32) cp_async16(buf + c, sr + c0 + c);
                cp_async_commit();
                cp_async_wait_all();
                __syncwarp();
                for (int c = lane; c < n16; c += 32) dr[c0 + c] = buf[c];
                __syncwarp();
            }
            after_stats();
        } else {
            cp_async_wait_all();
            __syncwarp();
            uint8_t *blk = p.packed + (q.s * p.ngcap + q.g_dst0 + q.g) * (long long)Layout<D>::GB;
            if (!vhalf) key_tile<D, DT>(tile, blk, lane, after_stats);
            else value_tile<D, DT>(tile, blk, lane, thr, after_stats);
            if (p.newK != nullptr && q.g == 0) {
                // A flush: the tile (residual slots 0..31) was read before
                // its statistics, so the new token may replace slot 0 (the
                // key warp its key row, the value warp its value row).
                const uint4 *ns = (const uint4 *)((vhalf ? p.newV : p.newK) + q.s * D);
                uint4 *nd = (uint4 *)((vhalf ? p.resV : p.resK) + q.s * (long long)p.R * D);
                for (int c = lane; c < D / 8; c += 32) nd[c] = ns[c];
            }
        }
        if (!has_next) break;
        unit = next;
        q = qn;
    }
    cp_async_wait_all();
}

#ifndef KIVI_QUANT_CTAS
#define KIVI_QUANT_CTAS 2   // resident CTAs of 8 warps per SM (persistent grid)
#endif

template <int D, int DT>
__global__ void __launch_bounds__(kQuantWarps * 32, KIVI_QUANT_CTAS) quant_kernel(QuantParams p)
{
    quant_warps<D, DT, false>(p, nullptr);
}

template <int D, int DT>
__global__ void __launch_bounds__(kQuantWarps * 32, KIVI_QUANT_CTAS)
    quant_kernel_seg(QuantParams p, const __grid_constant__ QuantSegs sg)
{
    quant_warps<D, DT, true>(p, &sg);
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
    const long long items = segs ? segs->item0[segs->nseg]
                                 : p.seqs * (long long)p.n_g + (p.r_copy > 0 ? p.seqs : 0);
    if (items == 0) return cudaSuccess;
    // Two work units (key tile, value tile) per item, one warp each.
    long long grid = (long long)num_sms() * KIVI_QUANT_CTAS;
    const long long need = (2 * items + kQuantWarps - 1) / kQuantWarps;
    if (grid > need) grid = need;
    QuantParams q = p;
    q.div_ng = make_magic((unsigned long long)(p.n_g > 0 ? p.n_g : 1));
    using S = QuantWarpSmem<D>;
    if (segs) {
        static PerDeviceOnce once;
        const cudaError_t e = set_smem_once(once, quant_kernel_seg<D, DT>, S::BYTES);
        if (e != cudaSuccess) return e;
        quant_kernel_seg<D, DT><<<(unsigned)grid, kQuantWarps * 32, S::BYTES, st>>>(q, *segs);
    } else {
        static PerDeviceOnce once;
        const cudaError_t e = set_smem_once(once, quant_kernel<D, DT>, S::BYTES);
        if (e != cudaSuccess) return e;
        quant_kernel<D, DT><<<(unsigned)grid, kQuantWarps * 32, S::BYTES, st>>>(q);
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
