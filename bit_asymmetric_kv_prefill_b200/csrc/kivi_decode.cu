// kivi_decode.cu -- split-K flash-decoding attention over the packed 2-bit
// KIVI cache plus its full-precision residual.
//
// One decode query per head attends to every cached token: the grouped 2-bit
// history and the newest r <= R residual tokens (KIVI: A Tuning-Free Asymmetric
// 2bit Quantization for KV Cache, Key points; record
// kv-efficiency/kivi-2bit-llama2-13b-mha-4k, "KV bytes basis").  The pass is a
// memory-bound GEMV, so it runs on the CUDA cores:
//
//  * Work split: the flattened (sequence, item) list, items being 32-token
//    groups and 6-token residual slices, is cut into equal contiguous weight
//    ranges, one per warp of a one-CTA-per-SM grid (Split in kivi_common.cuh).
//  * Each warp streams its items through a private ring of shared-memory
//    stages filled by cp.async.bulk (the bulk-copy engine) and completed on
//    mbarriers; every wait is bounded and reports through the status word.
//  * Keys: per group the lane folds the per-channel scale into the query,
//    q'_d = q_d * s_d, and the zero into one bias b = sum_d q_d z_d, so that
//    q.k = sum_d q'_d c_d + b.  A code AND-ed out of its word is the fp32
//    denormal c * 2^(2i-149); the query carries the matching power of two,
//    so one logic op per code and one fp32x2 FMA per two codes accumulate
//    the exact products (no conversion step).
//  * Values: the token weight b_t = p_t s_t (times a per-head power of two)
//    goes through shared memory as f16; a code pair AND-ed out of its word is
//    two f16 subnormals, each multiplied by the weight in one mixed
//    f16 x f16 -> fp32 FMA; sum_t p_t z_t stays in fp32.  Lanes own channels.
//  * Softmax is online in fp32 in the log2 domain (the query carries
//    log2(e)/sqrt(D)); the running max is only raised when a score exceeds it
//    by more than 8, which keeps all rescaling rare.
//  * Each warp writes one unnormalised partial (o, m, l) per sequence it
//    touches; the warp that arrives last on the sequence's ticket (atomic
//    counter, no waiting) merges them with a log-sum-exp combine and writes
//    the fp32 output.
//  * Pre-RoPE caches dequantize keys explicitly and rotate them at their
//    absolute positions (KIVI article, paragraph 4; KVQuant summary,
//    "Pre-RoPE Key Quantization"), sin/cos from an exact Cody-Waite angle
//    reduction and the hardware sine/cosine.
//  * With kivi_append_decode the residual slice that holds the appended
//    token takes it from the caller's k_t/v_t and stores it to the residual.
#include <utility>

#include <cuda_runtime.h>

#include "kivi_common.cuh"
#include "kivi_decode_ops.cuh"
#include "kivi_internal.h"

namespace kivi {

// Build-time tuning knobs (defaults are the measured best on B200).
#ifndef KIVI_DECODE_STAGES
#define KIVI_DECODE_STAGES 3
#endif
#ifndef KIVI_DECODE_MAXW
#define KIVI_DECODE_MAXW 16
#endif
#ifndef KIVI_DECODE_MAXW_GQA
#define KIVI_DECODE_MAXW_GQA 12   // four or more query heads per kv head
#endif
#ifndef KIVI_DECODE_MAXW_GQA_ROPE
#define KIVI_DECODE_MAXW_GQA_ROPE 8   // the same with pre-RoPE keys
#endif
#ifndef KIVI_PDL
#define KIVI_PDL 1   // programmatic dependent launch of the decode
#endif
#ifndef KIVI_DECODE_CTA_WARPS_GQA
#define KIVI_DECODE_CTA_WARPS_GQA 4   // warps per CTA, 4+ query heads per kv head (0: one CTA per SM)
#endif
#ifndef KIVI_KEYS_SCALAR
#define KIVI_KEYS_SCALAR 1   // four query heads: key dot products as scalar FMAs
#endif
#ifndef KIVI_MERGE_FANIN
#define KIVI_MERGE_FANIN 8   // partials merged per first-level block (0: one level)
#endif
#ifndef KIVI_ROPE_UNROLL
#define KIVI_ROPE_UNROLL 1   // pre-RoPE key loop: pair-steps unrolled (measured best)
#endif

constexpr int kRopeUnroll = KIVI_ROPE_UNROLL;
#ifndef KIVI_DECODE_STAGES_GQA
#define KIVI_DECODE_STAGES_GQA 3   // four or more query heads per kv head
#endif
#ifndef KIVI_DECODE_STAGES_GQA_ROPE
#define KIVI_DECODE_STAGES_GQA_ROPE 4   // the same with pre-RoPE keys
#endif
// Ring depth (shared-memory stages per warp) of an instantiation.
template <int HG, bool ROPE>
constexpr int ring_stages()
{
    return HG >= 4 ? (ROPE ? KIVI_DECODE_STAGES_GQA_ROPE : KIVI_DECODE_STAGES_GQA) : KIVI_DECODE_STAGES;
}

// ---- shared-memory plan per warp ------------------------------------------------
template <int D, int HG, bool ROPE>
struct WarpSmem {
    using L = Layout<D>;
    static constexpr int QPS = D / 4 + 4;           // padded q' slice (floats)
    static constexpr int PPS = 40;                  // padded weight row (f16), one head
    static constexpr int PPS2 = 36;                 // padded weight row (u32), head pairs
    static constexpr int NST = ring_stages<HG, ROPE>();
    static constexpr int RING = 0;                  // NST x GB
    static constexpr int QP = NST * L::GB;          // float [HG][4][QPS]
    static constexpr int PPF = 32 * HG + 4;                   // padded weight row (fp32), [token][head]
    static constexpr int PP = QP + HG * 4 * QPS * 4;          // f16 [HG][NJ][PPS]
    static constexpr int PP_BYTES = values_f32<D, HG>() ? L::NJ * PPF * 4
                                    : HG == 1 ? L::NJ * PPS * 2 : (HG / 2) * L::NJ * PPS2 * 4;
    static constexpr int QS = PP + PP_BYTES;                  // float [HG][D]
    static constexpr int SZS = D / 4 + 4;                     // padded slice row (float2)
    static constexpr int SZ = QS + HG * D * 4;                // float2 [4][SZS] (RoPE)
    static constexpr int QRS = D / 8 + 2;                     // padded pair row (float2)
    static constexpr int QR = SZ + (ROPE ? 4 * SZS * 8 : 0);  // float2 [HG][4][QRS] (RoPE)
    static constexpr int FRS = D / 8 + 4;                     // padded frequency row (float)
    static constexpr int FR = QR + (ROPE ? HG * 4 * QRS * 8 : 0);    // float [4][FRS] (RoPE)
    static constexpr int BAR = FR + (ROPE ? 4 * FRS * 4 : 0);        // uint64 [NST]
    static constexpr int BYTES = (BAR + NST * 8 + 15) / 16 * 16;
};

template <int D, int HG, bool ROPE>
struct DecodeShape {
    static constexpr int PER_WARP = WarpSmem<D, HG, ROPE>::BYTES;
    static constexpr int MAXW = 232448 / PER_WARP;
    // Registers are shared per SM sub-partition (4 per SM), so warp counts
    // that are multiples of 4 use them best: 12 warps leave 168 registers a
    // thread, 8 leave 255.  Pre-RoPE keys with four or more query heads per
    // kv head need more than 168 (measured 12.6% faster at 8 warps, 4 stages);
    // so do eight query heads per kv head (1.5 KB of spills at 12 warps;
    // 364 -> 225 us at 8 warps on a 16 x 8-kv-head, 8K-token cache); four
    // heads without RoPE fit 168 and run faster at 12 warps.
    static constexpr int CAP = HG >= 8   ? KIVI_DECODE_MAXW_GQA_ROPE
                               : HG >= 4 ? (ROPE ? KIVI_DECODE_MAXW_GQA_ROPE : KIVI_DECODE_MAXW_GQA)
                                         : KIVI_DECODE_MAXW;
    static constexpr int NW = MAXW > CAP ? CAP : MAXW;   // warps per SM
    // Warps per CTA: a CTA of CW warps, NW / CW of them per SM.  A smaller CTA
    // leaves the SM as soon as its own warps are done, so the next launch (a
    // programmatic dependent) can start there while other warps finish.  That
    // pays for the long grouped-query launches (1.3% at Mistral-7B shape, 0.6%
    // on the pre-RoPE long context); for one query head per kv head whole-SM
    // CTAs were 5-10% faster (4-warp CTAs 35.3 against 32.2 us on a
    // Llama-2-7B layer), so those keep one CTA per SM.
    static constexpr int CW_REQ = HG >= 4 ? KIVI_DECODE_CTA_WARPS_GQA : 0;
    static constexpr int CW = CW_REQ > 0 && NW % (CW_REQ > 0 ? CW_REQ : 1) == 0 ? CW_REQ : NW;
    static constexpr int CTAS = NW / CW;
    static constexpr int SMEM = CW * PER_WARP;   // per CTA
};

// ---- the kernel ---------------------------------------------------------------
template <int D, int HG, int DT, bool ROPE, bool RAGGED>
__device__ __forceinline__ void decode_body(const DecodeParams &p, const RaggedTab *rt)
{
    using L = Layout<D>;
    using W = WarpSmem<D, HG, ROPE>;
    constexpr int CW = DecodeShape<D, HG, ROPE>::CW;   // warps per CTA
    constexpr int CPL = L::CPL, QPL = L::QPL, NJ = L::NJ, KW = L::KW, HALF = L::HALF, TPW = L::TPW;
    constexpr int PSTRIDE = D + 4;
    constexpr int kSt = W::NST;
    constexpr bool VF32 = values_f32<D, HG>();

    extern __shared__ __align__(128) unsigned char smem_all[];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long gw = (long long)blockIdx.x * CW + warp;
#if KIVI_PDL
    // The next launch on the stream may be scheduled as soon as every CTA of
    // this one has started (it waits for this launch's memory itself).
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
#endif
    if (gw >= p.warps) return;  // warp-uniform

    unsigned char *ws = smem_all + warp * W::BYTES;
    unsigned char *ring = ws + W::RING;
    float *qp = (float *)(ws + W::QP);
    uint16_t *pp = (uint16_t *)(ws + W::PP);
    float *qs = (float *)(ws + W::QS);
    float2 *sz = (float2 *)(ws + W::SZ);
    float2 *qr = (float2 *)(ws + W::QR);
    float *frq = (float *)(ws + W::FR);
    const uint32_t bar0 = smem_addr(ws + W::BAR);
    const uint32_t magic = p.magic;
    const float2 neg = make_float2(p.neg_magic, p.neg_magic);

    // The ring's barriers first: they need nothing from the split.
    if (lane == 0) {
        for (int i = 0; i < kSt; ++i) mbar_init(bar0 + 8 * i, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }

    // This warp's share of the flattened (sequence, item) list: sequences
    // s_first..s_last, items [i_first, ...) of the first and [..., i_end) of
    // the last; the sequences between are whole.  Item indices fit 32 bits.
    Split sp;
    sp.init(p.seqs, p.n_groups, p.r, p.wg, p.wr, p.warps);
    sp.mC = p.div_C;
    sp.mT = p.div_Tot;
    sp.mW = p.div_warps;
    sp.mG = p.div_wg;
    sp.mR = p.div_wr;
    if constexpr (RAGGED) sp.Tot = rt->off[rt->nb];
    // Per-sequence lengths and work layout: one length for every sequence,
    // or (ragged caches) the lengths of the sequence's batch element.
    auto elem = [&](int s) { return (int)div_floor(s, p.div_Hkv); };
    auto ng_of = [&](int s) -> int {
        if constexpr (RAGGED) return rt->ng[elem(s)];
        else return (int)p.n_groups;
    };
    auto r_of = [&](int s) -> int {
        if constexpr (RAGGED) return rt->r[elem(s)];
        else return p.r;
    };
    auto nq_of = [&](int s) -> long long {
        if constexpr (RAGGED) return (long long)rt->ng[elem(s)] * kG;
        else return p.n_q;
    };
    // The appended token's residual slot (fused append), -1 if none.
    auto new_slot_of = [&](int s) -> int {
        if constexpr (RAGGED) return p.newK != nullptr ? r_of(s) - 1 : -1;
        else return p.new_slot;
    };
    auto C_of = [&](int s) -> long long {
        if constexpr (RAGGED) return (long long)ng_of(s) * p.wg + (long long)((r_of(s) + kResTok - 1) / kResTok) * p.wr;
        else return sp.C;
    };
    auto start_of = [&](int s) -> long long {
        if constexpr (RAGGED) {
            const int b = elem(s);
            return rt->off[b] + (long long)(s - b * p.H_kv) * C_of(s);
        } else {
            return (long long)s * sp.C;
        }
    };
    auto seq_of = [&](long long pos) -> int {
        if constexpr (RAGGED) {
            int lo_b = 0, hi_b = rt->nb - 1;   // the last element with off[b] <= pos
            while (lo_b < hi_b) {
                const int mid = (lo_b + hi_b + 1) >> 1;
                if (rt->off[mid] <= pos) lo_b = mid;
                else hi_b = mid - 1;
            }
            const int s0 = lo_b * p.H_kv;
            return s0 + (int)((pos - rt->off[lo_b]) / C_of(s0));
        } else {
            return (int)sp.seq_of(pos);
        }
    };
    // Items of sequence s owned by warp w: [first, second).
    auto items_of = [&](int s, long long w) -> ItemRange {
        if constexpr (RAGGED) {
            const long long base = start_of(s), C = C_of(s);
            const long long ng = ng_of(s), nit = ng + (r_of(s) + kResTok - 1) / kResTok;
            const long long a = sp.lo(w), b2 = sp.lo(w + 1);
            const long long ra = a > base ? a - base : 0;
            const long long rb = b2 < base + C ? b2 - base : C;
            if (ra >= rb) return ItemRange{0, 0};
            auto first_at = [&](long long rel) -> long long {
                const long long gend = ng * p.wg;
                if (ng > 0 && rel <= gend - p.wg) return div_floor(rel + p.wg - 1, p.div_wg);
                if (rel <= gend) return ng;
                const long long idx = ng + div_floor(rel - gend + p.wr - 1, p.div_wr);
                return idx < nit ? idx : nit;
            };
            const long long i0 = first_at(ra), i1 = first_at(rb);
            return ItemRange{i0, i1 < i0 ? i0 : i1};
        } else {
            return sp.items(s, w);
        }
    };
    auto n_items_of = [&](int s) -> int {
        if constexpr (RAGGED) return ng_of(s) + (r_of(s) + kResTok - 1) / kResTok;
        else return (int)sp.n_items();
    };
    // (The warp index enters as an opaque register: measured, this keeps the
    // split's 64-bit arithmetic on the vector pipes and the prologue short.)
    long long gwo = gw;
    asm volatile("" : "+l"(gwo));
    const long long lo = sp.lo(gwo), hi = sp.lo(gwo + 1);
    const int s_first = seq_of(lo), s_last = seq_of(hi - 1);
    int i_first, i_end;
    i_first = (int)items_of(s_first, gwo).first;
    i_end = (int)items_of(s_last, gwo).second;
    auto seq_items = [&](int s, int *i0, int *i1) {
        *i0 = s == s_first ? i_first : 0;
        *i1 = s == s_last ? i_end : n_items_of(s);
        if (*i1 < *i0) *i1 = *i0;
    };

    // The query rows of the warp's next sequence travel in registers ahead of
    // use (packed pairs of the cache dtype), starting with the first one.
    constexpr int QW = HG * D / 64;
    uint32_t qnext[QW];
    auto load_q = [&](int s) {
        const int b = (int)div_floor(s, p.div_Hkv), hk = s - b * p.H_kv;
        const uint32_t *qg = (const uint32_t *)(p.q + ((long long)b * p.H_q + (long long)hk * HG) * D);
#pragma unroll
        for (int i = 0; i < QW; ++i) qnext[i] = __ldg(qg + lane + 32 * i);
    };
#if KIVI_PDL
    // Launched as a programmatic dependent of the previous launch on the
    // stream: everything above ran while that launch was finishing; from
    // here on the kernel reads global memory it may have written (the query,
    // the cache), so it waits for its completion and memory first.
    asm volatile("griddepcontrol.wait;" ::: "memory");
#endif
    load_q(s_first);   // ahead of the ring's copies, which it would queue behind
    __syncwarp();

    // Prefetch iterator over the warp's items, possibly across sequences.
    int pf_s = s_first, pf_i, pf_e;
    seq_items(pf_s, &pf_i, &pf_e);
    auto pf_advance = [&]() {
        while (pf_i >= pf_e && pf_s < s_last) {
            ++pf_s;
            seq_items(pf_s, &pf_i, &pf_e);
        }
    };
    pf_advance();
    // Ring bookkeeping: items issued/consumed, the stage of the next issue,
    // and the stage and phase parity of the next item to consume.
    int issued = 0, consumed = 0, ist = 0, cst = 0;
    uint32_t cph = 0;
    const uint32_t ring_s = smem_addr(ring);
    auto issue_next = [&]() {
        pf_advance();
        if (pf_i >= pf_e) return;
        const uint32_t bar = bar0 + 8 * ist;
        const uint32_t dst = ring_s + ist * L::GB;
        ist = ist + 1 == kSt ? 0 : ist + 1;
        const int pf_ng = ng_of(pf_s);
        if (pf_i < pf_ng) {
            const uint8_t *src = p.packed + ((long long)pf_s * p.ngcap + pf_i) * (long long)L::GB;
            lane0_expect_copy(lane, bar, dst, src, L::GB, L::GB);
        } else {
            const int t0 = (pf_i - pf_ng) * kResTok;
            const int nt = min(kResTok, r_of(pf_s) - t0);
            const uint32_t bytes = (uint32_t)nt * D * 2;
            const long long row = (long long)pf_s * p.R + t0;
            const int nn = new_slot_of(pf_s) - t0;   // the appended token's row in this slice
            if (p.newK != nullptr && nn >= 0 && nn < nt) {
                // Fused append: the slice's last row comes from the caller's
                // k_t/v_t (slot new_slot, the residual's newest); the rows
                // before it from the residual.
                const uint32_t head = (uint32_t)nn * D * 2;
                lane0_expect_copy(lane, bar, dst + head, p.newK + (long long)pf_s * D, D * 2, 2 * bytes);
                lane0_copy(lane, bar, dst + kResTok * D * 2 + head, p.newV + (long long)pf_s * D, D * 2);
                if (nn > 0) {
                    lane0_copy(lane, bar, dst, p.resK + row * D, head);
                    lane0_copy(lane, bar, dst + kResTok * D * 2, p.resV + row * D, head);
                }
                if (nn + 1 < nt) {   // (the appended token is the newest: never taken)
                    const uint32_t tail = (uint32_t)(nt - nn - 1) * D * 2;
                    lane0_copy(lane, bar, dst + head + D * 2, p.resK + (row + nn + 1) * D, tail);
                    lane0_copy(lane, bar, dst + kResTok * D * 2 + head + D * 2, p.resV + (row + nn + 1) * D, tail);
                }
            } else {
                lane0_expect_copy(lane, bar, dst, p.resK + row * D, bytes, 2 * bytes);
                lane0_copy(lane, bar, dst + kResTok * D * 2, p.resV + row * D, bytes);
            }
        }
        ++issued;
        ++pf_i;
    };
    for (int i = 0; i < kSt; ++i) issue_next();

    bool failed = false;
    // Bounded wait for the next stage.  With p.expire_first_wait (testing the
    // failure path) the warp's first consuming wait gives up at once; every
    // later wait, the drain's included, keeps the full bound.
    auto wait_stage = [&]() -> bool {
        const uint32_t bar = bar0 + 8 * cst;
        const int limit = (p.expire_first_wait && consumed == 0 && !failed) ? 0 : kWaitLimit;
        for (int it = 0; it < limit; ++it)
            if (__all_sync(FULL, mbar_try_wait(bar, cph))) return true;
        return false;
    };
    auto next_stage = [&]() {
        ++consumed;
        if (++cst == kSt) {
            cst = 0;
            cph ^= 1u;
        }
    };

    const int tq = lane >> 2, cs = lane & 3;   // K mapping: 4 tokens x slice cs
    const int pcs = lane >> 3;                  // q' writer: permuted slice
    const int pL0 = (lane & 7) * QPL;           //   and first local index
    const int vco = lane & 15, vth = lane >> 4; // V mapping: channel octet, token half
    const int jl = vco * CPL / 32;              //   value group of the lane's channels
    // V: token t = lane's weight factor undoing the shift its pairs are read
    // at, 2^-(2*((t mod TPW)*CPL/2 mod 4)).
    const float vtok = pow2i(-2 * (((lane % TPW) * (CPL / 2)) & 3));

    // RoPE: inverse frequencies of the pairs of slice c4, frq[c4][i] for pair
    // c4*D/8 + i (rows padded against bank conflicts).
    if constexpr (ROPE) {
        for (int e = lane; e < D / 2; e += 32) frq[(e / HALF) * W::FRS + e % HALF] = __ldg(p.inv_freq + e);
        __syncwarp();
    }

    // Log-sum-exp merge of n partial rows of head h: slots k_first,
    // k_first + k_step, ... of the rows at pbase.  Each round trip loads the
    // (m, l) and the lane's QPL channels of 8 rows together and folds them
    // into a running (max, sum, row).  With `dst` the normalised result goes
    // there; without, the unnormalised merge (a partial of the same form)
    // replaces row k_first.
    auto merge_rows = [&](float *pbase, int k_first, int k_step, int n, int h, float *dst) {
        float M = -INFINITY, lacc = 0.f;
        float oo[QPL];
#pragma unroll
        for (int c = 0; c < QPL; ++c) oo[c] = 0.f;
        for (int k0 = 0; k0 < n; k0 += 8) {
            float2 ml[8];
            float v[8][QPL];
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                if (k0 + j < n) {
                    const float *row = pbase + ((long long)(k_first + (k0 + j) * k_step) * HG + h) * PSTRIDE;
                    ml[j] = __ldcg((const float2 *)(row + D));
#pragma unroll
                    for (int c = 0; c < QPL; c += 2) {
                        const float2 x = __ldcg((const float2 *)(row + lane * QPL + c));
                        v[j][c] = x.x;
                        v[j][c + 1] = x.y;
                    }
                } else {
                    ml[j] = make_float2(-INFINITY, 0.f);
#pragma unroll
                    for (int c = 0; c < QPL; ++c) v[j][c] = 0.f;
                }
            }
            float mx = M;
#pragma unroll
            for (int j = 0; j < 8; ++j) mx = fmaxf(mx, ml[j].x);
            if (mx == -INFINITY) continue;   // only empty partials so far
            const float a = ex2(M - mx);
            lacc *= a;
#pragma unroll
            for (int c = 0; c < QPL; ++c) oo[c] *= a;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                const float wj = ex2(ml[j].x - mx);
                lacc = fmaf(wj, ml[j].y, lacc);
#pragma unroll
                for (int c = 0; c < QPL; ++c) oo[c] = fmaf(wj, v[j][c], oo[c]);
            }
            M = mx;
        }
        if (dst) {
            const float inv = 1.0f / lacc;
#pragma unroll
            for (int c = 0; c < QPL; c += 2)
                *(float2 *)(dst + lane * QPL + c) = make_float2(oo[c] * inv, oo[c + 1] * inv);
        } else {
            float *row = pbase + ((long long)k_first * HG + h) * PSTRIDE;
            __syncwarp();   // every lane has read the row's (m, l)
#pragma unroll
            for (int c = 0; c < QPL; c += 2) __stcg((float2 *)(row + lane * QPL + c), make_float2(oo[c], oo[c + 1]));
            if (lane == 0) __stcg((float2 *)(row + D), make_float2(M, lacc));
        }
    };

    for (int s = s_first; s <= s_last && !failed; ++s) {
        int i0, i1;
        seq_items(s, &i0, &i1);
        const int b = (int)div_floor(s, p.div_Hkv), hk = s - b * p.H_kv;
        const int n_groups = ng_of(s), r_s = r_of(s), new_slot = new_slot_of(s);
        const long long n_q_s = nq_of(s);

        // Scaled query in shared memory (fp32) and the lane's q' inputs; then
        // the next sequence's query is requested (with four or more query
        // heads per group the registers are short: those load in place).
        if (HG > 2 && s != s_first) load_q(s);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < QW; ++i) {
            const int e = 2 * (lane + 32 * i);
            qs[e] = to_f<DT>((uint16_t)qnext[i]) * p.qscale;
            qs[e + 1] = to_f<DT>((uint16_t)(qnext[i] >> 16)) * p.qscale;
        }
        __syncwarp();
        if constexpr (ROPE) {
            // Rotate-half partners side by side: qr[h][cs][i] = (q_i, q_{i+D/2})
            // of slice cs, channel i = cs*D/8 + i'.
            for (int e = lane; e < HG * 4 * HALF; e += 32) {
                const int h = e / (4 * HALF), r = e % (4 * HALF), c4 = r / HALF, i = r % HALF;
                qr[(h * 4 + c4) * W::QRS + i] =
                    make_float2(qs[h * D + c4 * HALF + i], qs[h * D + D / 2 + c4 * HALF + i]);
            }
            __syncwarp();
        }
        if (HG <= 2 && s < s_last) load_q(s + 1);
        // The q'-writer lane's query channels: held in registers with one or
        // two query heads per kv head (measured faster than re-reading shared
        // memory every group); with four heads, where registers are short,
        // re-read each group as one 16-byte load per head (QREG false).
        constexpr bool QREG = HG <= 2;
        float qreg[QREG ? HG : 1][QPL];
        if constexpr (QREG) {
#pragma unroll
            for (int h = 0; h < HG; ++h)
#pragma unroll
                for (int e = 0; e < QPL; ++e) qreg[h][e] = qs[h * D + k_channel<D>(pcs, pL0 + e)];
        }

        float m[HG], lsum[HG], zacc[HG][NJ];
        float2 accV[HG][CPL / 2];
        // accV[h][mm] holds sum_t p_t s_t c_t 2^(2mm-24) * 2^ev[h].
        int ev[HG];
        float evs[HG];   // 2^ev * vtok
        bool ev_fresh[HG];
#pragma unroll
        for (int h = 0; h < HG; ++h) {
            ev[h] = 0;
            evs[h] = vtok;
            ev_fresh[h] = true;
            m[h] = -INFINITY;
            lsum[h] = 0.f;
#pragma unroll
            for (int j = 0; j < NJ; ++j) zacc[h][j] = 0.f;
#pragma unroll
            for (int c = 0; c < CPL / 2; ++c) accV[h][c] = make_float2(0.f, 0.f);
        }

        // Online softmax update with the lane's score s_h for one token (or
        // -inf), counted in l when `own` holds.
        auto softmax_step = [&](float (&sc)[HG], float (&pr)[HG], bool own) {
#pragma unroll
            for (int h = 0; h < HG; ++h) {
                const bool need = sc[h] > m[h] + kRescaleSlack;
                if (__any_sync(FULL, need)) {
                    const float mn = fmaxf(m[h], warp_max(sc[h]));
                    const float alpha = ex2(m[h] - mn);
                    lsum[h] *= alpha;
#pragma unroll
                    for (int j = 0; j < NJ; ++j) zacc[h][j] *= alpha;
#pragma unroll
                    for (int c = 0; c < CPL / 2; ++c) {
                        accV[h][c].x *= alpha;
                        accV[h][c].y *= alpha;
                    }
                    m[h] = mn;
                }
                pr[h] = ex2(sc[h] - m[h]);
                if (own) lsum[h] += pr[h];
            }
        };

        for (int it = i0; it < i1; ++it) {
            if (!wait_stage()) {
                failed = true;
                break;
            }
            const unsigned char *st = ring + cst * L::GB;
            if (it < n_groups) {
                // ---------------- quantized group of 32 tokens ----------------
                const uint16_t *km = (const uint16_t *)(st + L::KM + lane * (D / 8));
                float bias[HG];
                if constexpr (!ROPE) {
                    // Scales with their channel's code-pair factor folded in.
                    float sk[QPL], zk[QPL];
#pragma unroll
                    for (int e = 0; e < QPL; ++e) {
                        sk[e] = f16f(km[e]) * kq_scale(((pL0 + e) & 15) >> 1);
                        zk[e] = f16f(km[QPL + e]);
                    }
                    float bp[HG];
#pragma unroll
                    for (int h = 0; h < HG; ++h) {
                        bp[h] = 0.f;
                        float qv[QPL], qh[QPL];
#pragma unroll
                        for (int e = 0; e < QPL; ++e) {
                            // (the lane's QPL channels are consecutive and 16-byte aligned)
                            qh[e] = QREG ? qreg[QREG ? h : 0][e] : qs[h * D + k_channel<D>(pcs, pL0) + e];
                            qv[e] = qh[e] * sk[e];
                            bp[h] = fmaf(qh[e], zk[e], bp[h]);
                        }
                        float *dstq = qp + (h * 4 + pcs) * W::QPS + pL0;
#pragma unroll
                        for (int e = 0; e < QPL; e += 2) *(float2 *)(dstq + e) = make_float2(qv[e], qv[e + 1]);
                    }
                    warp_sum_n<HG>(bp, bias, lane);
                } else {
                    // Scales carry the inverse of each code pair's shift.
#pragma unroll
                    for (int e = 0; e < QPL; ++e)
                        sz[pcs * W::SZS + pL0 + e] =
                            make_float2(f16f(km[e]) * pair_scale(((pL0 + e) & 15) >> 1), f16f(km[QPL + e]));
                }
                __syncwarp();

                // Keys: lane (tq, cs) scores tokens 4tq..4tq+3 over slice cs.
                uint32_t kw[L::WPL];
#pragma unroll
                for (int c = 0; c < L::WPL / 4; ++c) {
                    uint4 v4 = *(const uint4 *)(st + L::KC + (c * 32 + lane) * 16);
                    kw[4 * c] = v4.x;
                    kw[4 * c + 1] = v4.y;
                    kw[4 * c + 2] = v4.z;
                    kw[4 * c + 3] = v4.w;
                }
                float part[4][HG];
                if constexpr (!ROPE && HG == 4 && KIVI_KEYS_SCALAR) {
                    // Scalar FMAs: each query value stays the multiplicand of
                    // four consecutive FMAs (one per token), which sustains
                    // more multiply-adds per clock than fp32x2 FMAs whose
                    // three operands all change (measured on B200).
                    float accs[4][HG];
#pragma unroll
                    for (int t = 0; t < 4; ++t)
#pragma unroll
                        for (int h = 0; h < HG; ++h) accs[t][h] = 0.f;
#pragma unroll
                    for (int k = 0; k < KW; ++k) {
#pragma unroll
                        for (int i = 0; i < 16; i += 4) {
                            // codes of local channels 16k + i + e, e = 0..3
                            float c[4][4];
#pragma unroll
                            for (int t = 0; t < 4; ++t) {
                                const uint32_t w = kw[t * KW + k], w16 = w >> 16;
                                c[t][0] = __uint_as_float(w & (3u << i));
                                c[t][1] = __uint_as_float(w16 & (3u << i));
                                c[t][2] = __uint_as_float(w & (12u << i));
                                c[t][3] = __uint_as_float(w16 & (12u << i));
                            }
#pragma unroll
                            for (int h = 0; h < HG; ++h) {
                                const float4 q4 = *(const float4 *)(qp + (h * 4 + cs) * W::QPS + 16 * k + i);
                                const float qe[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
                                for (int e = 0; e < 4; ++e)
#pragma unroll
                                    for (int t = 0; t < 4; ++t) accs[t][h] = fmaf(qe[e], c[t][e], accs[t][h]);
                            }
                        }
                    }
#pragma unroll
                    for (int t = 0; t < 4; ++t)
#pragma unroll
                        for (int h = 0; h < HG; ++h) part[t][h] = accs[t][h];
                } else if constexpr (!ROPE) {
                    float2 acc[4][HG];
#pragma unroll
                    for (int t = 0; t < 4; ++t)
#pragma unroll
                        for (int h = 0; h < HG; ++h) acc[t][h] = make_float2(0.f, 0.f);
#pragma unroll
                    for (int k = 0; k < KW; ++k) {
                        uint32_t kw16[4];
#pragma unroll
                        for (int t = 0; t < 4; ++t) kw16[t] = kw[t * KW + k] >> 16;
#pragma unroll
                        for (int i = 0; i < 16; i += 4) {
                            float4 q4[HG];
#pragma unroll
                            for (int h = 0; h < HG; ++h)
                                q4[h] = *(const float4 *)(qp + (h * 4 + cs) * W::QPS + 16 * k + i);
#pragma unroll
                            for (int t = 0; t < 4; ++t) {
                                const uint32_t w = kw[t * KW + k];
                                const float2 c01 = make_float2(__uint_as_float(w & (3u << i)),
                                                               __uint_as_float(kw16[t] & (3u << i)));
                                const float2 c23 = make_float2(__uint_as_float(w & (12u << i)),
                                                               __uint_as_float(kw16[t] & (12u << i)));
#pragma unroll
                                for (int h = 0; h < HG; ++h) {
                                    acc[t][h] = ffma2(make_float2(q4[h].x, q4[h].y), c01, acc[t][h]);
                                    acc[t][h] = ffma2(make_float2(q4[h].z, q4[h].w), c23, acc[t][h]);
                                }
                            }
                        }
                    }
#pragma unroll
                    for (int t = 0; t < 4; ++t)
#pragma unroll
                        for (int h = 0; h < HG; ++h) part[t][h] = acc[t][h].x + acc[t][h].y;
                } else {
                    // Dequantize, rotate at absolute positions, dot with q, two
                    // rotate-half pairs (i, i+1) of the slice at a time, each
                    // pair's scale/zero, frequencies and query pairs loaded once
                    // for the lane's 4 tokens.
                    const long long tbase = (long long)it * kG + 4 * tq;
                    float d0[4][HG], d1[4][HG];
#pragma unroll
                    for (int t = 0; t < 4; ++t)
#pragma unroll
                        for (int h = 0; h < HG; ++h) d0[t][h] = d1[t][h] = 0.f;
#pragma unroll kRopeUnroll
                    for (int i = 0; i < HALF; i += 2) {
                        // Local channels i, i+1 (first RoPE half) and HALF+i,
                        // HALF+i+1 (their partners); word k = L/16, pair (L%16)/2.
                        const int Lx = i, Ly = HALF + i;
                        const float4 sx = *(const float4 *)(sz + cs * W::SZS + Lx);
                        const float4 sy = *(const float4 *)(sz + cs * W::SZS + Ly);
                        const float2 f2 = *(const float2 *)(frq + cs * W::FRS + i);
                        float4 qq[HG];
#pragma unroll
                        for (int h = 0; h < HG; ++h) qq[h] = *(const float4 *)(qr + (h * 4 + cs) * W::QRS + i);
#pragma unroll
                        for (int t = 0; t < 4; ++t) {
                            const float pos = (float)(tbase + t);
                            const uint32_t wx = kw[t * KW + Lx / 16], wy = kw[t * KW + Ly / 16];
                            const float2 cx = code_pair(wx, wx >> 16, (Lx % 16) / 2, magic, neg);
                            const float2 cy = code_pair(wy, wy >> 16, (Ly % 16) / 2, magic, neg);
                            const float x0 = fmaf(cx.x, sx.x, sx.y), x1 = fmaf(cx.y, sx.z, sx.w);
                            const float y0 = fmaf(cy.x, sy.x, sy.y), y1 = fmaf(cy.y, sy.z, sy.w);
                            float sn0, cn0, sn1, cn1;
                            rope_sincos(__fmul_rn(pos, f2.x), &sn0, &cn0);
                            rope_sincos(__fmul_rn(pos, f2.y), &sn1, &cn1);
                            const float rx0 = x0 * cn0 - y0 * sn0, ry0 = y0 * cn0 + x0 * sn0;
                            const float rx1 = x1 * cn1 - y1 * sn1, ry1 = y1 * cn1 + x1 * sn1;
#pragma unroll
                            for (int h = 0; h < HG; ++h) {
                                d0[t][h] = fmaf(qq[h].x, rx0, d0[t][h]);
                                d1[t][h] = fmaf(qq[h].y, ry0, d1[t][h]);
                                d0[t][h] = fmaf(qq[h].z, rx1, d0[t][h]);
                                d1[t][h] = fmaf(qq[h].w, ry1, d1[t][h]);
                            }
                        }
                    }
#pragma unroll
                    for (int t = 0; t < 4; ++t)
#pragma unroll
                        for (int h = 0; h < HG; ++h) part[t][h] = d0[t][h] + d1[t][h];
                }
                // Transpose-reduce the 4 token partials over the 4 slices: lane
                // (tq, cs) ends with token 4tq + cs = lane.
                float sc[HG];
#pragma unroll
                for (int h = 0; h < HG; ++h) {
                    const bool hiB = cs & 2, loB = cs & 1;
                    float send0 = hiB ? part[0][h] : part[2][h];
                    float send1 = hiB ? part[1][h] : part[3][h];
                    float k0 = (hiB ? part[2][h] : part[0][h]) + __shfl_xor_sync(FULL, send0, 2);
                    float k1 = (hiB ? part[3][h] : part[1][h]) + __shfl_xor_sync(FULL, send1, 2);
                    float send = loB ? k0 : k1;
                    float keep = (loB ? k1 : k0) + __shfl_xor_sync(FULL, send, 1);
                    if constexpr (ROPE) sc[h] = keep;
                    else sc[h] = fmaf(keep, kKunscale, bias[h]);
                }
                float pr[HG];
                softmax_step(sc, pr, true);

                // Token weights b = p s 2^ev (times the lane's shift factor)
                // for token `lane`, as f16 rows [h][j][token]; with two or
                // more query heads, head pairs share a word: u32 rows
                // [j][h/2][token] holding (b_h, b_h+1).
                const uint16_t *vm = (const uint16_t *)(st + L::VM + lane * (D / 8));
                float svj[NJ];
#pragma unroll
                for (int j = 0; j < NJ; ++j) {
                    svj[j] = f16f(vm[j]);
                    const float zvj = f16f(vm[NJ + j]);
#pragma unroll
                    for (int h = 0; h < HG; ++h) zacc[h][j] = fmaf(pr[h], zvj, zacc[h][j]);
                }
                if constexpr (VF32) {
                    // fp32 weights b[j][token][h] = p_h s_j 2^kVexp, one
                    // 16-byte row entry per (group j, token) holding the heads.
                    float ps[HG];
#pragma unroll
                    for (int h = 0; h < HG; ++h) ps[h] = pr[h] * pow2i(kVexp);
                    float *ppf = (float *)pp;
#pragma unroll
                    for (int j = 0; j < NJ; ++j)
                        *(float4 *)(ppf + j * W::PPF + lane * HG) =
                            make_float4(ps[0] * svj[j], ps[1] * svj[j], ps[2] * svj[j], ps[3] * svj[j]);
                }
                float fh[HG];
#pragma unroll
                for (int h = 0; h < HG && !VF32; ++h) {
                    float f = pr[h] * evs[h];   // evs carries the lane's vtok
                    float bm = 0.f;
#pragma unroll
                    for (int j = 0; j < NJ; ++j) bm = fmaxf(bm, f * svj[j]);
                    if (__any_sync(FULL, !(bm < kVLimit)) || ev_fresh[h]) {
                        // Rare: choose 2^d putting the largest weight near
                        // kVTarget (first group with a nonzero weight), or
                        // bring it below the f16 range; accV follows.
                        const float mx = warp_max(bm);
                        if (mx > 0.f && mx <= 3.0e38f) {
                            const int e = (int)((__float_as_uint(mx) >> 23) & 0xff) - 127;
                            int d = kVTargetExp - e;
                            if (!ev_fresh[h] && d > 0) d = 0;
                            const int en = max(-100, min(100, ev[h] + d));
                            d = en - ev[h];
                            const int d1 = d / 2, d2 = d - d1;
#pragma unroll
                            for (int c = 0; c < CPL / 2; ++c) {
                                accV[h][c].x = accV[h][c].x * pow2i(d1) * pow2i(d2);
                                accV[h][c].y = accV[h][c].y * pow2i(d1) * pow2i(d2);
                            }
                            evs[h] = pow2i(en) * vtok;
                            f = pr[h] * evs[h];
                            ev[h] = en;
                            ev_fresh[h] = false;
                        }
                    }
                    fh[h] = f;
                }
                if constexpr (VF32) {
                } else if constexpr (HG == 1) {
#pragma unroll
                    for (int j = 0; j < NJ; ++j)
                        pp[j * W::PPS + lane] = __half_as_ushort(__float2half_rn(fh[0] * svj[j]));
                } else {
                    uint32_t *pp32 = (uint32_t *)pp;
#pragma unroll
                    for (int j = 0; j < NJ; ++j)
#pragma unroll
                        for (int hp = 0; hp < HG / 2; ++hp) {
                            const __half2 b2 = __floats2half2_rn(fh[2 * hp] * svj[j], fh[2 * hp + 1] * svj[j]);
                            pp32[(j * (HG / 2) + hp) * W::PPS2 + lane] = *(const uint32_t *)&b2;
                        }
                }
                __syncwarp();

                // Values: lane (vco, vth) owns channels [vco*CPL, (vco+1)*CPL)
                // of tokens 16*vth .. 16*vth + 15.
                uint32_t vw[L::WPL];
#pragma unroll
                for (int c = 0; c < L::WPL / 4; ++c) {
                    uint4 v4 = *(const uint4 *)(st + L::VC + (c * 32 + lane) * 16);
                    vw[4 * c] = v4.x;
                    vw[4 * c + 1] = v4.y;
                    vw[4 * c + 2] = v4.z;
                    vw[4 * c + 3] = v4.w;
                }
                if constexpr (VF32) {
                    // Word u holds tokens A = 16vth + 2u (pairs 0..3, bits 2m
                    // and 16 + 2m: channels 2m, 2m + 1 of the lane's octet)
                    // and B = A + 1 (pairs 4..7, bits 8 + 2m and 24 + 2m).
                    const float *ppf = (const float *)pp + jl * W::PPF + (16 * vth) * HG;
#pragma unroll
                    for (int u = 0; u < L::WPL; ++u) {
                        const uint32_t w = vw[u], w8 = w >> 8, w16 = w >> 16, w24 = w >> 24;
                        const float4 bA = *(const float4 *)(ppf + (2 * u) * HG);
                        const float4 bB = *(const float4 *)(ppf + (2 * u + 1) * HG);
                        const float wa[4] = {bA.x, bA.y, bA.z, bA.w}, wb[4] = {bB.x, bB.y, bB.z, bB.w};
#pragma unroll
                        for (int mm = 0; mm < CPL / 2; ++mm) {
                            const uint32_t msk = 3u << (2 * mm);
                            const float2 cA = make_float2(__uint_as_float(w & msk), __uint_as_float(w16 & msk));
                            const float2 cB = make_float2(__uint_as_float(w8 & msk), __uint_as_float(w24 & msk));
#pragma unroll
                            for (int h = 0; h < HG; ++h) {
                                accV[h][mm] = ffma2(make_float2(wa[h], wa[h]), cA, accV[h][mm]);
                                accV[h][mm] = ffma2(make_float2(wb[h], wb[h]), cB, accV[h][mm]);
                            }
                        }
                    }
                } else {
                // The weights of the lane's 16 tokens: one head, two tokens
                // per word (HG == 1), or one token, two heads per word.
                constexpr int PBW = HG == 1 ? 8 : 16;
                uint32_t pb[HG == 1 ? 1 : HG / 2][PBW];
#pragma unroll
                for (int hp = 0; hp < (HG == 1 ? 1 : HG / 2); ++hp) {
                    const uint4 *src = HG == 1
                        ? (const uint4 *)(pp + jl * W::PPS + 16 * vth)
                        : (const uint4 *)((const uint32_t *)pp + (jl * (HG / 2) + hp) * W::PPS2 + 16 * vth);
#pragma unroll
                    for (int c = 0; c < PBW / 4; ++c) {
                        const uint4 a = src[c];
                        pb[hp][4 * c] = a.x;
                        pb[hp][4 * c + 1] = a.y;
                        pb[hp][4 * c + 2] = a.z;
                        pb[hp][4 * c + 3] = a.w;
                    }
                }
#pragma unroll
                for (int u = 0; u < L::WPL; ++u) {
                    const uint32_t w = vw[u], w8 = w >> 8;
#pragma unroll
                    for (int tt = 0; tt < TPW; ++tt) {
#pragma unroll
                        for (int mm = 0; mm < CPL / 2; ++mm) {
                            const int i = tt * (CPL / 2) + mm;
                            const uint32_t x = (i < 4 ? w : w8) & (0x00030003u << (2 * (i & 3)));
#pragma unroll
                            for (int h = 0; h < HG; ++h) {
                                // The weight's half: the token's parity (one
                                // head) or the head's parity (head pairs).
                                const uint32_t bw = HG == 1 ? pb[0][(u * TPW + tt) >> 1] : pb[h / 2][u * TPW + tt];
                                const bool odd = HG == 1 ? (tt & 1) : (h & 1);
                                if (!odd) {
                                    accV[h][mm].x = hfma_f32<0, 0>(x, bw, accV[h][mm].x);
                                    accV[h][mm].y = hfma_f32<1, 0>(x, bw, accV[h][mm].y);
                                } else {
                                    accV[h][mm].x = hfma_f32<0, 1>(x, bw, accV[h][mm].x);
                                    accV[h][mm].y = hfma_f32<1, 1>(x, bw, accV[h][mm].y);
                                }
                            }
                        }
                    }
                }
                }
            } else {
                // ---------------- residual slice of up to 6 tokens ----------------
                const int t0 = (it - n_groups) * kResTok;
                const int nt = min(kResTok, r_s - t0);
                const uint16_t *rk = (const uint16_t *)st;
                const uint16_t *rv = (const uint16_t *)(st + kResTok * D * 2);
                if (p.newK != nullptr && new_slot >= t0 && new_slot < t0 + nt) {
                    // Fused append: this warp persists the new token into its
                    // residual slot (read by later launches' bulk copies).
                    constexpr int C16 = D / 8;   // 16-byte chunks per row
                    const int nn = new_slot - t0;
                    const long long drow = ((long long)s * p.R + new_slot) * D;
                    for (int c = lane; c < 2 * C16; c += 32) {
                        const int which = c / C16, q16 = c % C16;
                        const uint4 v = *(const uint4 *)((which ? rv : rk) + nn * D + q16 * 8);
                        *(uint4 *)((which ? p.resV : p.resK) + drow + q16 * 8) = v;
                    }
                }
                const bool valid = tq < nt;
                float sc[HG];
                {
                    float kx[2][HALF];
                    if (valid) {
#pragma unroll
                        for (int half = 0; half < 2; ++half) {
                            const uint16_t *src = rk + tq * D + half * (D / 2) + cs * HALF;
#pragma unroll
                            for (int i = 0; i < HALF; i += 8) {
                                uint4 v4 = *(const uint4 *)(src + i);
                                const uint16_t *e = (const uint16_t *)&v4;
#pragma unroll
                                for (int z = 0; z < 8; ++z) kx[half][i + z] = to_f<DT>(e[z]);
                            }
                        }
                        if constexpr (ROPE) {
                            const float pos = (float)(n_q_s + t0 + tq);
#pragma unroll
                            for (int i = 0; i < HALF; ++i) {
                                float sn, cn;
                                rope_sincos(__fmul_rn(pos, frq[cs * W::FRS + i]), &sn, &cn);
                                const float x = kx[0][i], y = kx[1][i];
                                kx[0][i] = x * cn - y * sn;
                                kx[1][i] = y * cn + x * sn;
                            }
                        }
                    } else {
#pragma unroll
                        for (int half = 0; half < 2; ++half)
#pragma unroll
                            for (int i = 0; i < HALF; ++i) kx[half][i] = 0.f;
                    }
#pragma unroll
                    for (int h = 0; h < HG; ++h) {
                        float d0 = 0.f, d1 = 0.f;
#pragma unroll
                        for (int i = 0; i < HALF; ++i) {
                            d0 = fmaf(qs[h * D + cs * HALF + i], kx[0][i], d0);
                            d1 = fmaf(qs[h * D + D / 2 + cs * HALF + i], kx[1][i], d1);
                        }
                        float d = d0 + d1;
                        d += __shfl_xor_sync(FULL, d, 1);
                        d += __shfl_xor_sync(FULL, d, 2);
                        sc[h] = valid ? d : -INFINITY;
                    }
                }
                float pr[HG];
                softmax_step(sc, pr, valid && cs == 0);
                // Residual values: lane (vco, vth) takes tokens of parity vth,
                // with the same per-pair factor 2^(2m) as the quantized codes.
                for (int t0 = 0; t0 < nt; t0 += 2) {
                    const int t = t0 + vth;
                    const bool ok = t < nt;
                    float vx[CPL];
                    if (ok) {
                        const uint16_t *vrow = rv + t * D + vco * CPL;
#pragma unroll
                        for (int c = 0; c < CPL; ++c) vx[c] = to_f<DT>(vrow[c]);
                    } else {
#pragma unroll
                        for (int c = 0; c < CPL; ++c) vx[c] = 0.f;
                    }
#pragma unroll
                    for (int h = 0; h < HG; ++h) {
                        const float pt = __shfl_sync(FULL, pr[h], 4 * (ok ? t : t0)) *
                                         pow2i(VF32 ? kVexp - 149 : ev[h] - 24);
#pragma unroll
                        for (int c = 0; c < CPL; c += 2) {
                            const float pa = pt * pow2i(c);   // 2^(2mm), mm = c/2
                            accV[h][c / 2] = ffma2(make_float2(pa, pa), make_float2(vx[c], vx[c + 1]),
                                                   accV[h][c / 2]);
                        }
                    }
                }
            }
            // Stage consumed: refill it with the item kSt ahead.
            __syncwarp();
            next_stage();
            issue_next();
        }
        if (failed) break;

        // ---------------- this warp's partial for sequence s ----------------
        const long long first = sp.owner(start_of(s));
        const long long last = sp.owner(start_of(s) + C_of(s) - 1);
        const int count = (int)(last - first + 1);
        const int slot = (int)(gw - first);
        // lt: the softmax sum; zt: the zero term of the lane's value group jl
        // (picked by selects: a lane-dependent index would put the array on
        // the stack).
        float lt[HG], zt[HG];
#pragma unroll
        for (int h = 0; h < HG; ++h) {
            lt[h] = warp_sum(lsum[h]);
            zt[h] = 0.f;
#pragma unroll
            for (int j = 0; j < NJ; ++j) {
                const float zj = warp_sum(zacc[h][j]);
                zt[h] = jl == j ? zj : zt[h];
            }
        }
        // Undo the per-pair factor 2^(2m), join the two token halves and add
        // the zero term: lane (vco, vth) then holds channels vco*CPL + c.
        float o[HG][CPL];
#pragma unroll
        for (int h = 0; h < HG; ++h)
#pragma unroll
            for (int c = 0; c < CPL; c += 2) {
                const float2 a = accV[h][c / 2];
                // 2^(24 - 2mm - ev), or 2^(149 - kVexp - 2mm) for fp32 weights
                const float f = pow2i(VF32 ? 149 - kVexp - c : 24 - c - ev[h]);
                const float x = a.x + __shfl_xor_sync(FULL, a.x, 16);
                const float y = a.y + __shfl_xor_sync(FULL, a.y, 16);
                o[h][c] = fmaf(x, f, zt[h]);
                o[h][c + 1] = fmaf(y, f, zt[h]);
            }
        float *outrow = p.out + ((long long)b * p.H_q + (long long)hk * HG) * D;
        if (count == 1) {
            if (vth == 0) {
#pragma unroll
                for (int h = 0; h < HG; ++h) {
                    const float inv = 1.0f / lt[h];
#pragma unroll
                    for (int c = 0; c < CPL; c += 2)
                        *(float2 *)(outrow + h * D + vco * CPL + c) =
                            make_float2(o[h][c] * inv, o[h][c + 1] * inv);
                }
            }
            continue;
        }
        // Compact partial rows: sequence s uses rows first(s) + s + slot, so
        // the rows of consecutive sequences never meet (first(s + 1) >=
        // last(s)) and warps + sequences rows serve any split.
        float *pbase = p.partials + ((first + s) * HG) * (long long)PSTRIDE;
#pragma unroll
        for (int h = 0; h < HG; ++h) {
            float *prow = pbase + ((long long)slot * HG + h) * PSTRIDE;
            if (vth == 0) {
#pragma unroll
                for (int c = 0; c < CPL; c += 2)
                    *(float2 *)(prow + vco * CPL + c) = make_float2(o[h][c], o[h][c + 1]);
            }
            if (lane == 0) *(float2 *)(prow + D) = make_float2(m[h], lt[h]);
        }
        // Merge.  A sequence split over at most 2F warps is merged by the
        // last of them in one pass.  Longer ones merge in two levels, so
        // that no single warp walks every partial at the end: slots are cut
        // into blocks of F, the last warp of each block folds its block into
        // the block's first row, and the last block to finish folds those
        // rows into the output.  Each merge reads its rows in slot order, so
        // the result does not depend on which warp finishes last.
        constexpr int F = KIVI_MERGE_FANIN > 0 ? KIVI_MERGE_FANIN : 1;
        const bool two_level = KIVI_MERGE_FANIN > 0 && count > 2 * F;
        const int n_blocks = two_level ? (count + F - 1) / F : count;
        const int kstep = two_level ? F : 1;
        // Level 0 is this warp's block (only when it holds more than one
        // partial), level 1 the whole sequence; a warp that is not the last
        // to arrive at a level leaves the sequence.  (One loop, so that the
        // merge is generated once.)
        int kb = 0, k0 = 0, cnt = 0, lvl = 1;
        if (two_level) {
            kb = slot / F;
            k0 = kb * F;
            cnt = count - k0 < F ? count - k0 : F;
            if (cnt > 1) lvl = 0;
        }
        __syncwarp();
#pragma unroll 1
        for (; lvl < 2; ++lvl) {
            int *tk = lvl == 0 ? p.tickets + p.seqs + (first + s + kb) : p.tickets + s;
            const int need = lvl == 0 ? cnt : n_blocks;
            // Every lane fences its own row stores (one warp instruction
            // either way) before lane 0 takes the ticket.
            __threadfence();
            int last = 0;
            if (lane == 0) last = atomicAdd(tk, 1) == need - 1;
            if (!__shfl_sync(FULL, last, 0)) break;
            __threadfence();
#pragma unroll 1
            for (int h = 0; h < HG; ++h)
                merge_rows(pbase, lvl == 0 ? k0 : 0, lvl == 0 ? 1 : kstep, need, h,
                           lvl == 0 ? nullptr : outrow + h * D);
            __syncwarp();
            if (lane == 0) *tk = 0;
        }
    }

    if (failed) {
        if (lane == 0) atomicCAS(p.err, 0, kErrWaitTimeout);
        // Let the copies already in flight land before the warp leaves.
        while (consumed < issued) {
            wait_stage();
            next_stage();
        }
    }
}

template <int D, int HG, int DT, bool ROPE>
__global__ void __launch_bounds__(DecodeShape<D, HG, ROPE>::CW * 32, DecodeShape<D, HG, ROPE>::CTAS)
    decode_kernel(const DecodeParams p)
{
    decode_body<D, HG, DT, ROPE, false>(p, nullptr);
}

// Caches whose batch elements hold different lengths: the same body, lengths
// per batch element from the table.
template <int D, int HG, int DT, bool ROPE>
__global__ void __launch_bounds__(DecodeShape<D, HG, ROPE>::CW * 32, DecodeShape<D, HG, ROPE>::CTAS)
    decode_kernel_ragged(const DecodeParams p, const __grid_constant__ RaggedTab rt)
{
    decode_body<D, HG, DT, ROPE, true>(p, &rt);
}

template <int D, int HG, bool ROPE>
static int warps_per_sm()
{
    return DecodeShape<D, HG, ROPE>::NW;
}

int decode_warps_per_sm(int D, int HG, int pre_rope)
{
#define KIVI_NW(DD, HH)                                                            \
    if (D == DD && HG == HH) return pre_rope ? warps_per_sm<DD, HH, true>()        \
                                             : warps_per_sm<DD, HH, false>();
    KIVI_NW(64, 1) KIVI_NW(64, 2) KIVI_NW(64, 4) KIVI_NW(64, 8)
    KIVI_NW(128, 1) KIVI_NW(128, 2) KIVI_NW(128, 4) KIVI_NW(128, 8)
#undef KIVI_NW
    return 0;
}

// Launch a decode kernel; with KIVI_PDL as a programmatic dependent of the
// previous launch on the stream (its CTAs may start while that launch
// finishes and wait in the kernel before their first global read).
template <typename... Params, typename... Args>
static cudaError_t launch_kernel(void (*kernel)(Params...), unsigned grid, unsigned block, size_t smem,
                                 cudaStream_t st, Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = KIVI_PDL ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

template <int D, int HG, int DT, bool ROPE>
static cudaError_t launch_decode_t(const DecodeParams &p, const RaggedTab *rt, cudaStream_t st)
{
    using S = DecodeShape<D, HG, ROPE>;
    const unsigned grid = (unsigned)((p.warps + S::CW - 1) / S::CW);
    cudaError_t e;
    if (rt) {
        static PerDeviceOnce once;
        e = set_smem_once(once, decode_kernel_ragged<D, HG, DT, ROPE>, S::SMEM);
        if (e == cudaSuccess)
            e = launch_kernel(decode_kernel_ragged<D, HG, DT, ROPE>, grid, S::CW * 32, S::SMEM, st, p, *rt);
    } else {
        static PerDeviceOnce once;
        e = set_smem_once(once, decode_kernel<D, HG, DT, ROPE>, S::SMEM);
        if (e == cudaSuccess) e = launch_kernel(decode_kernel<D, HG, DT, ROPE>, grid, S::CW * 32, S::SMEM, st, p);
    }
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

template <int D, int HG>
static cudaError_t launch_decode_hg(int dtype, int pre_rope, const DecodeParams &p, const RaggedTab *rt,
                                    cudaStream_t st)
{
    if (dtype) {
        return pre_rope ? launch_decode_t<D, HG, 1, true>(p, rt, st) : launch_decode_t<D, HG, 1, false>(p, rt, st);
    }
    return pre_rope ? launch_decode_t<D, HG, 0, true>(p, rt, st) : launch_decode_t<D, HG, 0, false>(p, rt, st);
}

cudaError_t launch_decode(int D, int HG, int dtype, int pre_rope, const DecodeParams &p,
                          const RaggedTab *rt, cudaStream_t st)
{
#define KIVI_CASE(DD, HH) \
    if (D == DD && HG == HH) return launch_decode_hg<DD, HH>(dtype, pre_rope, p, rt, st);
    KIVI_CASE(64, 1) KIVI_CASE(64, 2) KIVI_CASE(64, 4) KIVI_CASE(64, 8)
    KIVI_CASE(128, 1) KIVI_CASE(128, 2) KIVI_CASE(128, 4) KIVI_CASE(128, 8)
#undef KIVI_CASE
    return cudaErrorInvalidValue;
}

}  // namespace kivi
