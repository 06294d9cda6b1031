// kivi_common.cuh -- layout of the packed KIVI cache, the exact 2-bit code
// parameters, and the decode work split.  Internal to the CUDA library.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

namespace kivi {

constexpr int kG = 32;          // tokens per key group, channels per value group
constexpr int kResTok = 6;      // residual tokens per decode item (one stage)
constexpr int kErrWaitTimeout = 1;
// Longest pre-RoPE cache: decode reduces RoPE angles (position * inv_freq,
// inv_freq <= 1) modulo 2pi exactly below 2^17 * 2pi = 823,549.
constexpr long long kRopeMaxTokens = 823000;

// ---------------------------------------------------------------------------
// Packed group block.  One block per (sequence, group of 32 quantized tokens),
// 24*D bytes, laid out so that one bulk copy brings a whole group into shared
// memory and every lane's reads there are conflict-free 16-byte loads:
//
//   [0,    8D)  Kc  K codes.  Lane l = 4*tq + cs holds tokens 4tq..4tq+3 and
//                   the D/4 channels of slice cs (D/8 from each RoPE half, so
//                   that rotate-half partners stay in one lane): D/16 words,
//                   word u = tok*(D/64) + k covers local channels
//                   L = 16k..16k+15.  Words are stored [u/4][lane][u%4].
//   [8D,  12D)  Km  K scale/zero per channel, permuted order P = cs*(D/4) + L,
//                   lane l owns P in [l*D/32, (l+1)*D/32): D/32 fp16 scales
//                   then D/32 fp16 zeros.
//   [12D, 20D)  Vc  V codes.  Lane l = 16*th + co holds the D/16 channels of
//                   octet co, [co*D/16, (co+1)*D/16), for tokens 16th..16th+15:
//                   D/16 words, word u covers tokens 16th + u*TPW + [0, TPW).
//   [20D, 24D)  Vm  V scale/zero per token: D/32 fp16 scales then D/32 zeros.
//
// A 32-bit word holds 16 two-bit codes as 8 pairs: pair i has its first code
// at bits [2i, 2i+1] and its second at bits [16+2i, 17+2i].  In a K word pair
// i is local channels (16k+2i, 16k+2i+1); in a V word pair i is token
// 16th + u*TPW + i/(CPL/2), channels co*CPL + 2*(i%(CPL/2)) and the next one.
// Both halves of a pair sit at the same shift, so one mask reads both: from
// the word and from the word shifted right by 16 (keys, one logic op per
// code), or as the two 16-bit halves of one register (values, one logic op
// per pair).
// ---------------------------------------------------------------------------
template <int D>
struct Layout {
    static_assert(D % 64 == 0, "head_dim must be a multiple of 64");
    static constexpr int GB = 24 * D;    // group block bytes
    static constexpr int KC = 0;
    static constexpr int KM = 8 * D;
    static constexpr int VC = 12 * D;
    static constexpr int VM = 20 * D;
    static constexpr int WPL = D / 16;   // code words per lane (K or V)
    static constexpr int KW = D / 64;    // K words per token per lane
    static constexpr int HALF = D / 8;   // channels per lane per RoPE half
    static constexpr int SLICE = D / 4;  // K channels per lane
    static constexpr int QPL = D / 32;   // K scale/zero entries per lane
    static constexpr int CPL = D / 16;   // V channels per lane
    static constexpr int TPW = 16 / CPL; // tokens per V word
    static constexpr int NJ = D / kG;    // value groups per token
};

// Byte offset, inside the Kc or Vc region, of lane-local word u of lane l.
__host__ __device__ inline int code_word_offset(int lane, int u)
{
    return ((u >> 2) * 32 + lane) * 16 + (u & 3) * 4;
}

// K channel held at local index L (0..D/4-1) of channel slice cs.
template <int D>
__host__ __device__ inline int k_channel(int cs, int L)
{
    constexpr int n = D / 8;
    return L < n ? cs * n + L : D / 2 + cs * n + (L - n);
}

// Inverse: (cs, L) of channel d, as the permuted index P = cs*(D/4) + L.
template <int D>
__host__ __device__ inline int k_perm_index(int d)
{
    constexpr int n = D / 8;
    int cs, L;
    if (d < D / 2) {
        cs = d / n;
        L = d % n;
    } else {
        cs = (d - D / 2) / n;
        L = n + (d - D / 2) % n;
    }
    return cs * (D / 4) + L;
}

// Byte offset inside Km of the scale (zero: + D/16) of permuted index P.
template <int D>
__host__ __device__ inline int km_offset(int P)
{
    int lane = P / (D / 32), e = P % (D / 32);
    return lane * (D / 8) + e * 2;
}

// ---------------------------------------------------------------------------
// Exact code parameters.  With s = fp16((max-min)/3) > 0 and z = fp16(min),
// the definition code = clamp(rint(fl(fl(x - z) / s)), 0, 3) (fp32, rint half
// to even) equals [d > E1] + [d > E2] + [d > E3] with d = fl(x - z), because
// division and rounding are monotone:
//   rint(y) >= 1  <=> y > 0.5   <=> d/s > 0.5 + 2^-25  (a tie rounds to 0.5)
//   rint(y) >= 2  <=> y >= 1.5  <=> d/s >= 1.5 - 2^-24 (a tie rounds to 1.5)
//   rint(y) >= 3  <=> y > 2.5   <=> d/s > 2.5 + 2^-23  (a tie rounds to 2.5)
// s has at most 11 significant bits, so s/2, 1.5s and 2.5s are exact in fp32,
// and each bound times s lies strictly inside one fp32 ulp next to them
// ((0.5 + 2^-25)s in (s/2, succ(s/2)), (1.5 - 2^-24)s in (pred(1.5s), 1.5s),
// (2.5 + 2^-23)s in (2.5s, succ(2.5s))).  For an fp32 d the three tests are
// therefore d > s/2, d > pred(1.5s) and d > 2.5s.  A zero scale gives
// thresholds +inf (all codes 0).
// ---------------------------------------------------------------------------
struct CodeParams {
    uint16_t s_bits, z_bits;
    float e1, e2, e3, z;
};

__device__ __forceinline__ CodeParams code_params(float mn, float mx)
{
    CodeParams p;
    float range = __fsub_rn(mx, mn);
    float s32 = __fdiv_rn(range, 3.0f);
    uint16_t sb = __half_as_ushort(__float2half_rn(s32));
    uint16_t zb = __half_as_ushort(__float2half_rn(mn));
    if ((sb & 0x7fffu) == 0) sb = 0;
    if ((zb & 0x7fffu) == 0) zb = 0;
    p.s_bits = sb;
    p.z_bits = zb;
    float sf = __half2float(__ushort_as_half(sb));
    p.z = __half2float(__ushort_as_half(zb));
    if (sf == 0.0f) {
        p.e1 = p.e2 = p.e3 = __int_as_float(0x7f800000);
    } else {
        p.e1 = __fmul_rn(sf, 0.5f);
        p.e2 = __int_as_float(__float_as_int(__fmul_rn(sf, 1.5f)) - 1);
        p.e3 = __fmul_rn(sf, 2.5f);
    }
    return p;
}

__device__ __forceinline__ uint32_t code_of(float x, float z, float e1, float e2, float e3)
{
    float d = __fsub_rn(x, z);
    return (uint32_t)(d > e1) + (uint32_t)(d > e2) + (uint32_t)(d > e3);
}

// ---------------------------------------------------------------------------
// Decode work split.  Per sequence the work is n_groups quantized groups
// (weight wg each) followed by ceil(r/kResTok) residual items (weight wr
// each); sequences are concatenated and the total cut into `warps` equal
// contiguous ranges [lo_w, hi_w), lo_w = floor(w*Tot/warps), with
// warps <= Tot so that no range is empty.  An item belongs to the warp whose
// range holds the item's start.  A warp contributes one partial result to
// every sequence its range intersects, so sequence s gets
// last(s) - first(s) + 1 partials, first(s) = owner(s*C),
// last(s) = owner((s+1)*C - 1).
// ---------------------------------------------------------------------------
// Division by a run-time constant d >= 1 as a multiply and shifts, exact
// for numerators 0 <= a < 2^53 (Granlund and Montgomery, "Division by
// invariant integers using multiplication", 1994, round-up method): with
// l = ceil(log2 d) and M = floor(2^(53+l)/d) + 1, 2^(53+l) < M d <= 2^(53+l) + 2^l,
// so floor(a/d) = floor(a M / 2^(53+l)).  The product's high word is taken
// after shifting a left by sa = max(0, 11-l); sb = max(0, l-11) finishes it.
struct Magic {
    unsigned long long M;
    int sa, sb;
};

__host__ inline Magic make_magic(unsigned long long d)
{
    int l = 0;
    while ((1ULL << l) < d) ++l;
    Magic m;
    m.M = (unsigned long long)((((unsigned __int128)1) << (53 + l)) / d) + 1;
    m.sa = l < 11 ? 11 - l : 0;
    m.sb = l > 11 ? l - 11 : 0;
    return m;
}

__host__ __device__ __forceinline__ unsigned long long mulhi64(unsigned long long a,
                                                                 unsigned long long b)
{
#ifdef __CUDA_ARCH__
    return __umul64hi(a, b);
#else
    return (unsigned long long)(((unsigned __int128)a * b) >> 64);
#endif
}

// floor(a / d) for 0 <= a < 2^53, m = make_magic(d).
__host__ __device__ __forceinline__ long long div_floor(long long a, Magic m)
{
    return (long long)(mulhi64((unsigned long long)a << m.sa, m.M) >> m.sb);
}

struct ItemRange {
    long long first, second;
};

struct Split {
    long long seqs, n_groups, n_res_items, C, Tot, warps;
    int wg, wr;
    Magic mC, mT, mW, mG, mR;   // division by C, Tot, warps, wg, wr (div_floor)

    // The division constants, from the host (the kernel takes them from its
    // parameters).
    __host__ void set_magics()
    {
        mC = make_magic((unsigned long long)C);
        mT = make_magic((unsigned long long)Tot);
        mW = make_magic((unsigned long long)warps);
        mG = make_magic((unsigned long long)wg);
        mR = make_magic((unsigned long long)wr);
    }

    __host__ __device__ __forceinline__ void init(long long seqs_, long long n_groups_, int r, int wg_,
                                  int wr_, long long warps_)
    {
        seqs = seqs_;
        n_groups = n_groups_;
        n_res_items = (r + kResTok - 1) / kResTok;
        wg = wg_;
        wr = wr_;
        C = n_groups * wg + n_res_items * wr;
        Tot = C * seqs;
        warps = warps_;
    }
    __host__ __device__ __forceinline__ long long n_items() const { return n_groups + n_res_items; }
    __host__ __device__ __forceinline__ long long lo(long long w) const { return div_floor(w * Tot, mW); }
    __host__ __device__ __forceinline__ long long owner(long long pos) const
    {
        return div_floor((pos + 1) * warps - 1, mT);
    }
    __host__ __device__ __forceinline__ long long seq_of(long long pos) const { return div_floor(pos, mC); }
    __host__ __device__ __forceinline__ long long item_start(long long idx) const
    {
        return idx < n_groups ? idx * wg : n_groups * wg + (idx - n_groups) * wr;
    }
    // Smallest item index whose start is >= rel (rel in [0, C]); n_items() if
    // there is none.
    __host__ __device__ __forceinline__ long long first_item_at(long long rel) const
    {
        long long gend = n_groups * wg;
        if (n_groups > 0 && rel <= gend - wg) return div_floor(rel + wg - 1, mG);
        if (rel <= gend) return n_groups;
        long long idx = n_groups + div_floor(rel - gend + wr - 1, mR);
        return idx < n_items() ? idx : n_items();
    }
    // Items of sequence s owned by warp w: [first, second).
    __host__ __device__ __forceinline__ ItemRange items(long long s, long long w) const
    {
        const long long base = s * C;
        const long long a = lo(w), b = lo(w + 1);
        const long long ra = a > base ? a - base : 0;
        const long long rb = b < base + C ? b - base : C;
        if (ra >= rb) return ItemRange{0, 0};
        const long long i0 = first_item_at(ra), i1 = first_item_at(rb);
        return ItemRange{i0, i1 < i0 ? i0 : i1};
    }
};

// ---------------------------------------------------------------------------
// Per-batch-element lengths of a ragged cache (batch element b's sequences,
// b*H_kv .. b*H_kv + H_kv - 1, hold n_q = ng[b]*kG quantized and r[b]
// residual tokens).  The decode split concatenates the sequences' weights
// (ng*wg + ceil(r/kResTok)*wr each); off[b] is where element b's first
// sequence starts and off[nb] the total.  Passed to kernels by value.
// ---------------------------------------------------------------------------
constexpr int kMaxRaggedB = 512;
struct RaggedTab {
    int nb;
    int ng[kMaxRaggedB];
    int r[kMaxRaggedB];
    long long off[kMaxRaggedB + 1];
};

}  // namespace kivi
