// kivi_api.cu -- the C ABI (include/kivi.h): argument checks, device memory
// plan, host-side sequence bookkeeping, kernel launches and the test-only
// export to the canonical unpacked layout.
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include <cuda_runtime.h>

#include "../../include/kivi.h"
#include "kivi_common.cuh"
#include "kivi_internal.h"

using namespace kivi;

namespace {

constexpr int kAbiVersion = 1;
constexpr int kMaxWarpsPerCta = 32;  // upper bound over decode shapes
constexpr int kMaxGroupHeads = 8;    // largest H_q/H_kv served
constexpr size_t kAlign = 256;

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

struct Plan {
    long long seqs, ngcap;
    long long part_rows;   // decode partial rows: every split has at most warps + seqs
    long long tick_count;  // decode tickets: one per sequence, one per partial row
    size_t off_packed, off_resK, off_resV, off_part, off_tick, off_err, off_freq, total;
    size_t codes, meta, residual, scratch;
};

kivi_status check_config(const kivi_config *c)
{
    if (!c) return KIVI_ERR_ARG;
    if (c->B < 1 || c->H_kv < 1 || c->D < 1 || c->G < 1 || c->R < 1 || c->T_max < 1)
        return KIVI_ERR_ARG;
    if (c->dtype != KIVI_F16 && c->dtype != KIVI_BF16) return KIVI_ERR_ARG;
    if (c->R % c->G != 0 || c->D % c->G != 0) return KIVI_ERR_ARG;
    if (c->G != kG) return KIVI_ERR_UNSUPPORTED;
    if (c->D != 64 && c->D != 128) return KIVI_ERR_UNSUPPORTED;
    if (c->pre_rope && !(c->rope_theta > 1.0f)) return KIVI_ERR_ARG;
    if (c->pre_rope && c->T_max > kRopeMaxTokens) return KIVI_ERR_UNSUPPORTED;
    return KIVI_OK;
}

kivi_status make_plan(const kivi_config *c, int sms, Plan *p)
{
    p->seqs = (long long)c->B * c->H_kv;
    p->ngcap = (c->T_max + c->G - 1) / c->G;
    const long long max_warps = (long long)sms * kMaxWarpsPerCta;
    p->part_rows = max_warps + p->seqs;
    const size_t gb = (size_t)24 * c->D;
    const size_t packed = (size_t)p->seqs * p->ngcap * gb;
    const size_t res = (size_t)p->seqs * c->R * c->D * 2;
    const size_t part = (size_t)p->part_rows * kMaxGroupHeads * (c->D + 4) * sizeof(float);
    p->tick_count = p->seqs + p->part_rows;
    const size_t tick = (size_t)p->tick_count * sizeof(int);
    const size_t freq = (size_t)(c->D / 2) * sizeof(float);
    size_t off = 0;
    p->off_packed = off;
    off = align_up(off + packed);
    p->off_resK = off;
    off = align_up(off + res);
    p->off_resV = off;
    off = align_up(off + res);
    p->off_part = off;
    off = align_up(off + part);
    p->off_tick = off;
    off = align_up(off + tick);
    p->off_err = off;
    off = align_up(off + sizeof(int));
    p->off_freq = off;
    off = align_up(off + freq);
    p->total = off;
    p->codes = packed / 24 * 16;  // 8D + 8D of every 24D-byte block
    p->meta = packed / 24 * 8;    // 4D + 4D
    p->residual = 2 * res;
    p->scratch = part + tick + sizeof(int) + freq;
    return KIVI_OK;
}

bool aligned16(const void *p) { return ((uintptr_t)p & 15u) == 0; }


// Split weights: a quantized group and a residual slice of kResTok tokens move
// the same number of bytes (24*D); the residual slice needs far fewer
// instructions, so it counts a little less.
int env_int(const char *name, int dflt)
{
    const char *s = std::getenv(name);
    if (!s || !*s) return dflt;
    int v = std::atoi(s);
    return v > 0 ? v : dflt;
}

}  // namespace

struct kivi_cache {
    kivi_config cfg;
    Plan plan;
    int dev, sms;
    unsigned char *base;
    bool owns;
    uint8_t *packed;
    uint16_t *resK, *resV;
    float *partials;
    int *tickets, *err;
    float *inv_freq;
    long long n_q;   // the split of every sequence, while the lengths agree
    int r;
    bool prefilled;
    // Batch elements of different lengths: element b's sequences hold nq_b[b]
    // quantized and r_b[b] residual tokens (the vectors are valid while
    // `ragged`; n_q and r otherwise).
    bool ragged;
    std::vector<long long> nq_b;
    std::vector<int> r_b;
    int wg, wr;
    int expire_first_wait;   // testing only (kivi_debug_expire_first_wait)
};

namespace {

long long nq_at(const kivi_cache *c, int b) { return c->ragged ? c->nq_b[b] : c->n_q; }
int r_at(const kivi_cache *c, int b) { return c->ragged ? c->r_b[b] : c->r; }

// After per-element updates: if every element holds the same split again,
// the cache is uniform.
void settle(kivi_cache *c)
{
    bool same = true;
    for (int b = 1; b < c->cfg.B && same; ++b)
        same = c->nq_b[b] == c->nq_b[0] && c->r_b[b] == c->r_b[0];
    c->ragged = !same;
    if (same) {
        c->n_q = c->nq_b[0];
        c->r = c->r_b[0];
    }
}

// The decode split of a ragged cache: per batch element its groups, its
// residual tokens and where its work starts.
void ragged_table(const kivi_cache *c, RaggedTab *rt)
{
    const int B = c->cfg.B, H = c->cfg.H_kv;
    rt->nb = B;
    rt->off[0] = 0;
    for (int b = 0; b < B; ++b) {
        rt->ng[b] = (int)(c->nq_b[b] / kG);
        rt->r[b] = c->r_b[b];
        const long long C = (long long)rt->ng[b] * c->wg + (long long)((rt->r[b] + kResTok - 1) / kResTok) * c->wr;
        rt->off[b + 1] = rt->off[b] + (long long)H * C;
    }
}

// Every call that touches a cache's device memory must run with the cache's
// device current: its launches, scratch and SM count belong to that device.
bool on_cache_device(const kivi_cache *c)
{
    int d = -1;
    return cudaGetDevice(&d) == cudaSuccess && d == c->dev;
}

}  // namespace

extern "C" {

int kivi_abi_version(void) { return kAbiVersion; }

const char *kivi_status_string(kivi_status s)
{
    switch (s) {
    case KIVI_OK: return "ok";
    case KIVI_ERR_ARG: return "invalid argument";
    case KIVI_ERR_UNSUPPORTED: return "unsupported shape";
    case KIVI_ERR_CAPACITY: return "capacity exceeded";
    case KIVI_ERR_STATE: return "invalid cache state";
    case KIVI_ERR_OOM: return "out of device memory";
    case KIVI_ERR_CUDA: return "CUDA error";
    case KIVI_ERR_DEVICE: return "device-side bounded wait failed";
    }
    return "unknown status";
}

kivi_status kivi_cache_required_bytes(const kivi_config *cfg, size_t *bytes)
{
    kivi_status st = check_config(cfg);
    if (st != KIVI_OK) return st;
    if (!bytes) return KIVI_ERR_ARG;
    Plan p;
    make_plan(cfg, num_sms(), &p);
    *bytes = p.total;
    return KIVI_OK;
}

kivi_status kivi_cache_create_ex(const kivi_config *cfg, kivi_cache **out)
{
    kivi_status st = check_config(cfg);
    if (st != KIVI_OK) return st;
    if (!out) return KIVI_ERR_ARG;
    *out = nullptr;
    kivi_cache *c = new (std::nothrow) kivi_cache();
    if (!c) return KIVI_ERR_OOM;
    c->cfg = *cfg;
    if (cudaGetDevice(&c->dev) != cudaSuccess) {
        delete c;
        return KIVI_ERR_CUDA;
    }
    c->sms = num_sms();
    make_plan(cfg, c->sms, &c->plan);
    if (cfg->workspace) {
        if (cfg->workspace_bytes < c->plan.total || ((uintptr_t)cfg->workspace % kAlign) != 0) {
            delete c;
            return cfg->workspace_bytes < c->plan.total ? KIVI_ERR_OOM : KIVI_ERR_ARG;
        }
        c->base = (unsigned char *)cfg->workspace;
        c->owns = false;
    } else {
        if (cudaMalloc(&c->base, c->plan.total) != cudaSuccess) {
            cudaGetLastError();
            delete c;
            return KIVI_ERR_OOM;
        }
        c->owns = true;
    }
    c->packed = c->base + c->plan.off_packed;
    c->resK = (uint16_t *)(c->base + c->plan.off_resK);
    c->resV = (uint16_t *)(c->base + c->plan.off_resV);
    c->partials = (float *)(c->base + c->plan.off_part);
    c->tickets = (int *)(c->base + c->plan.off_tick);
    c->err = (int *)(c->base + c->plan.off_err);
    c->inv_freq = (float *)(c->base + c->plan.off_freq);
    cudaError_t e = cudaMemset(c->tickets, 0, c->plan.tick_count * sizeof(int));
    if (e == cudaSuccess) e = cudaMemset(c->err, 0, sizeof(int));
    if (e == cudaSuccess && cfg->pre_rope) {
        // inv_freq_i = fp32(theta^(-2i/D)), rounded once from double.
        std::vector<float> f(cfg->D / 2);
        for (int i = 0; i < cfg->D / 2; ++i)
            f[i] = (float)std::pow((double)cfg->rope_theta, -2.0 * (double)i / (double)cfg->D);
        e = cudaMemcpy(c->inv_freq, f.data(), f.size() * sizeof(float), cudaMemcpyHostToDevice);
    }
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    if (e != cudaSuccess) {
        if (c->owns) cudaFree(c->base);
        delete c;
        return KIVI_ERR_CUDA;
    }
    c->n_q = 0;
    c->r = 0;
    c->prefilled = false;
    c->ragged = false;
    try {
        c->nq_b.assign(cfg->B, 0);
        c->r_b.assign(cfg->B, 0);
    } catch (...) {
        if (c->owns) cudaFree(c->base);
        delete c;
        return KIVI_ERR_OOM;
    }
    c->expire_first_wait = 0;
    c->wg = env_int("KIVI_SPLIT_WG", 4);
    c->wr = env_int("KIVI_SPLIT_WR", 3);
    *out = c;
    return KIVI_OK;
}

kivi_status kivi_cache_create(int B, int H_kv, int D, int G, int R, kivi_dtype dtype,
                              long long T_max, kivi_cache **out)
{
    kivi_config cfg;
    std::memset(&cfg, 0, sizeof cfg);
    cfg.B = B;
    cfg.H_kv = H_kv;
    cfg.D = D;
    cfg.G = G;
    cfg.R = R;
    cfg.dtype = dtype;
    cfg.T_max = T_max;
    cfg.rope_theta = 10000.0f;
    return kivi_cache_create_ex(&cfg, out);
}

kivi_status kivi_cache_destroy(kivi_cache *c)
{
    if (!c) return KIVI_ERR_ARG;
    cudaError_t e = cudaSuccess;
    if (c->owns) e = cudaFree(c->base);
    delete c;
    return cuda_status(e);
}

kivi_status kivi_cache_reset(kivi_cache *c)
{
    if (!c) return KIVI_ERR_ARG;
    c->n_q = 0;
    c->r = 0;
    c->prefilled = false;
    c->ragged = false;
    return KIVI_OK;
}

kivi_status kivi_cache_length(const kivi_cache *c, long long *n_q, int *r)
{
    if (!c || !n_q || !r) return KIVI_ERR_ARG;
    if (c->ragged) return KIVI_ERR_STATE;
    *n_q = c->n_q;
    *r = c->r;
    return KIVI_OK;
}

kivi_status kivi_cache_length_at(const kivi_cache *c, int b, long long *n_q, int *r)
{
    if (!c || !n_q || !r || b < 0 || b >= c->cfg.B) return KIVI_ERR_ARG;
    *n_q = nq_at(c, b);
    *r = r_at(c, b);
    return KIVI_OK;
}

kivi_status kivi_cache_bytes(const kivi_cache *c, kivi_bytes *out)
{
    if (!c || !out) return KIVI_ERR_ARG;
    out->codes = c->plan.codes;
    out->meta = c->plan.meta;
    out->residual = c->plan.residual;
    out->scratch = c->plan.scratch;
    out->total = c->plan.total;
    return KIVI_OK;
}

kivi_status kivi_prefill(kivi_cache *c, const void *K, const void *V, long long T, void *stream)
{
    if (!c || !K || !V || !aligned16(K) || !aligned16(V)) return KIVI_ERR_ARG;
    if (!on_cache_device(c)) return KIVI_ERR_ARG;
    if (c->prefilled) return KIVI_ERR_STATE;
    if (T < 1) return KIVI_ERR_ARG;
    if (T > c->cfg.T_max) return KIVI_ERR_CAPACITY;
    const int R = c->cfg.R, D = c->cfg.D;
    const long long n_q = (long long)R * ((T - 1) / R);
    const int r = (int)(T - n_q);
    QuantParams q;
    q.srcK = (const uint16_t *)K;
    q.srcV = (const uint16_t *)V;
    q.src_seq_rows = T;
    q.packed = c->packed;
    q.ngcap = c->plan.ngcap;
    q.g_dst0 = 0;
    q.n_g = (int)(n_q / kG);
    q.seqs = c->plan.seqs;
    q.resK = c->resK;
    q.resV = c->resV;
    q.R = R;
    q.r_copy = r;
    q.copy_row0 = n_q;
    q.newK = q.newV = nullptr;
    cudaError_t e = launch_quant(D, c->cfg.dtype, q, nullptr, (cudaStream_t)stream);
    if (e != cudaSuccess) return KIVI_ERR_CUDA;
    c->n_q = n_q;
    c->r = r;
    c->ragged = false;
    c->prefilled = true;
    return KIVI_OK;
}

kivi_status kivi_prefill_ragged(kivi_cache *c, const void *K, const void *V, long long T_pad,
                                const long long *T_b, void *stream)
{
    if (!c || !K || !V || !T_b || !aligned16(K) || !aligned16(V)) return KIVI_ERR_ARG;
    if (!on_cache_device(c)) return KIVI_ERR_ARG;
    if (c->prefilled) return KIVI_ERR_STATE;
    const int B = c->cfg.B, H = c->cfg.H_kv, R = c->cfg.R, D = c->cfg.D;
    if (B > kMaxRaggedB) return KIVI_ERR_UNSUPPORTED;
    if (T_pad < 1) return KIVI_ERR_ARG;
    if (T_pad > c->cfg.T_max) return KIVI_ERR_CAPACITY;
    for (int b = 0; b < B; ++b)
        if (T_b[b] < 1 || T_b[b] > T_pad) return KIVI_ERR_ARG;
    // One segment per run of consecutive batch elements of one length.
    QuantSegs sg;
    sg.nseg = 0;
    sg.item0[0] = 0;
    for (int b = 0; b < B; ++b) {
        const long long n_q = (long long)R * ((T_b[b] - 1) / R);
        const int r = (int)(T_b[b] - n_q), n_g = (int)(n_q / kG);
        const int k = sg.nseg - 1;
        if (k >= 0 && sg.n_g[k] == n_g && sg.r_copy[k] == r) {
            sg.nseq[k] += H;
        } else {
            sg.seq0[sg.nseg] = b * H;
            sg.nseq[sg.nseg] = H;
            sg.n_g[sg.nseg] = n_g;
            sg.g_dst0[sg.nseg] = 0;
            sg.r_copy[sg.nseg] = r;
            sg.copy_row0[sg.nseg] = (int)n_q;
            ++sg.nseg;
        }
    }
    for (int k = 0; k < sg.nseg; ++k)
        sg.item0[k + 1] = sg.item0[k] + (long long)sg.nseq[k] * (sg.n_g[k] + 1);
    QuantParams q;
    q.srcK = (const uint16_t *)K;
    q.srcV = (const uint16_t *)V;
    q.src_seq_rows = T_pad;
    q.packed = c->packed;
    q.ngcap = c->plan.ngcap;
    q.g_dst0 = 0;
    q.n_g = 1;
    q.seqs = c->plan.seqs;
    q.resK = c->resK;
    q.resV = c->resV;
    q.R = R;
    q.r_copy = 0;
    q.copy_row0 = 0;
    q.newK = q.newV = nullptr;
    cudaError_t e = launch_quant(D, c->cfg.dtype, q, &sg, (cudaStream_t)stream);
    if (e != cudaSuccess) return KIVI_ERR_CUDA;
    for (int b = 0; b < B; ++b) {
        c->nq_b[b] = (long long)R * ((T_b[b] - 1) / R);
        c->r_b[b] = (int)(T_b[b] - c->nq_b[b]);
    }
    settle(c);
    c->prefilled = true;
    return KIVI_OK;
}

namespace {

// Append to a ragged cache: batch elements whose residual is full flush it
// (one quantizer launch over segments of them), the others take the token
// in their own slot.
kivi_status append_ragged(kivi_cache *c, const void *k_t, const void *v_t, cudaStream_t st)
{
    const int B = c->cfg.B, H = c->cfg.H_kv, R = c->cfg.R, D = c->cfg.D;
    for (int b = 0; b < B; ++b)
        if (c->nq_b[b] + c->r_b[b] + 1 > c->cfg.T_max) return KIVI_ERR_CAPACITY;
    QuantSegs sg;
    sg.nseg = 0;
    sg.item0[0] = 0;
    SlotTab sl;
    bool plain = false;
    for (int b = 0; b < B; ++b) {
        if (c->r_b[b] == R) {
            sl.slot[b] = -1;
            const int k = sg.nseg - 1;
            const int g_dst0 = (int)(c->nq_b[b] / kG);
            if (k >= 0 && sg.seq0[k] + sg.nseq[k] == b * H && sg.g_dst0[k] == g_dst0) {
                sg.nseq[k] += H;
            } else {
                sg.seq0[sg.nseg] = b * H;
                sg.nseq[sg.nseg] = H;
                sg.n_g[sg.nseg] = R / kG;
                sg.g_dst0[sg.nseg] = g_dst0;
                sg.r_copy[sg.nseg] = 0;
                sg.copy_row0[sg.nseg] = 0;
                ++sg.nseg;
            }
        } else {
            sl.slot[b] = c->r_b[b];
            plain = true;
        }
    }
    for (int k = 0; k < sg.nseg; ++k) sg.item0[k + 1] = sg.item0[k] + (long long)sg.nseq[k] * sg.n_g[k];
    cudaError_t e = cudaSuccess;
    if (sg.nseg > 0) {
        QuantParams q;
        q.srcK = c->resK;
        q.srcV = c->resV;
        q.src_seq_rows = R;
        q.packed = c->packed;
        q.ngcap = c->plan.ngcap;
        q.g_dst0 = 0;
        q.n_g = R / kG;
        q.seqs = c->plan.seqs;
        q.resK = c->resK;
        q.resV = c->resV;
        q.R = R;
        q.r_copy = 0;
        q.copy_row0 = 0;
        q.newK = (const uint16_t *)k_t;
        q.newV = (const uint16_t *)v_t;
        e = launch_quant(D, c->cfg.dtype, q, &sg, st);
    }
    if (e == cudaSuccess && plain)
        e = launch_append_slots(D, (const uint16_t *)k_t, (const uint16_t *)v_t, c->resK, c->resV,
                                c->plan.seqs, H, R, sl, st);
    if (e != cudaSuccess) return KIVI_ERR_CUDA;
    for (int b = 0; b < B; ++b) {
        if (c->r_b[b] == R) {
            c->nq_b[b] += R;
            c->r_b[b] = 1;
        } else {
            c->r_b[b] += 1;
        }
    }
    settle(c);
    return KIVI_OK;
}

}  // namespace

kivi_status kivi_append(kivi_cache *c, const void *k_t, const void *v_t, void *stream)
{
    if (!c || !k_t || !v_t || !aligned16(k_t) || !aligned16(v_t)) return KIVI_ERR_ARG;
    if (!on_cache_device(c)) return KIVI_ERR_ARG;
    if (!c->prefilled) return KIVI_ERR_STATE;
    if (c->ragged) return append_ragged(c, k_t, v_t, (cudaStream_t)stream);
    if (c->n_q + c->r + 1 > c->cfg.T_max) return KIVI_ERR_CAPACITY;
    const int R = c->cfg.R, D = c->cfg.D;
    cudaError_t e;
    if (c->r == R) {
        QuantParams q;
        q.srcK = c->resK;
        q.srcV = c->resV;
        q.src_seq_rows = R;
        q.packed = c->packed;
        q.ngcap = c->plan.ngcap;
        q.g_dst0 = c->n_q / kG;
        q.n_g = R / kG;
        q.seqs = c->plan.seqs;
        q.resK = c->resK;
        q.resV = c->resV;
        q.R = R;
        q.r_copy = 0;
        q.copy_row0 = 0;
        q.newK = (const uint16_t *)k_t;
        q.newV = (const uint16_t *)v_t;
        e = launch_quant(D, c->cfg.dtype, q, nullptr, (cudaStream_t)stream);
        if (e != cudaSuccess) return KIVI_ERR_CUDA;
        c->n_q += R;
        c->r = 1;
        return KIVI_OK;
    }
    e = launch_append(D, (const uint16_t *)k_t, (const uint16_t *)v_t, c->resK, c->resV,
                      c->plan.seqs, R, c->r, (cudaStream_t)stream);
    if (e != cudaSuccess) return KIVI_ERR_CUDA;
    c->r += 1;
    return KIVI_OK;
}

kivi_status kivi_append_decode(kivi_cache *c, const void *k_t, const void *v_t, const void *q,
                               int H_q, float *out, void *stream)
{
    if (!c || !k_t || !v_t || !aligned16(k_t) || !aligned16(v_t)) return KIVI_ERR_ARG;
    if (!on_cache_device(c)) return KIVI_ERR_ARG;
    if (!c->prefilled) return KIVI_ERR_STATE;
    bool flush = false;
    for (int b = 0; b < c->cfg.B; ++b) {
        if (nq_at(c, b) + r_at(c, b) + 1 > c->cfg.T_max) return KIVI_ERR_CAPACITY;
        flush = flush || r_at(c, b) == c->cfg.R;
        if (!c->ragged) break;
    }
    if (flush) {   // a flush is due: the quantizer runs first
        const kivi_status st = kivi_append(c, k_t, v_t, stream);
        return st != KIVI_OK ? st : kivi_decode_attn(c, q, H_q, out, stream);
    }
    // The split sees the token already appended; undone if anything fails
    // before the launch.
    auto bump = [&](int d) {
        if (c->ragged)
            for (int b = 0; b < c->cfg.B; ++b) c->r_b[b] += d;
        else
            c->r += d;
    };
    bump(1);
    DecodeParams p;
    RaggedTab rt;
    bool ragged = false;
    long long rows = 0;
    int D = 0, HG = 0, dtype = 0, pre_rope = 0;
    kivi_status st = decode_params_external_scratch(c, q, H_q, out, &p, &D, &HG, &dtype, &pre_rope, &rt,
                                                    &ragged, &rows);
    if (st == KIVI_OK && rows > c->plan.part_rows) st = KIVI_ERR_UNSUPPORTED;
    if (st != KIVI_OK) {
        bump(-1);
        return st;
    }
    p.partials = c->partials;
    p.tickets = c->tickets;
    p.newK = (const uint16_t *)k_t;
    p.newV = (const uint16_t *)v_t;
    p.new_slot = c->ragged ? -1 : c->r - 1;   // ragged: each sequence's r - 1, in the kernel
    const cudaError_t e = launch_decode(D, HG, dtype, pre_rope, p, ragged ? &rt : nullptr, (cudaStream_t)stream);
    if (e != cudaSuccess) bump(-1);
    return cuda_status(e);
}

kivi_status kivi_decode_attn(kivi_cache *c, const void *q, int H_q, float *out, void *stream)
{
    DecodeParams p;
    RaggedTab rt;
    bool ragged = false;
    long long rows = 0;
    int D = 0, HG = 0, dtype = 0, pre_rope = 0;
    kivi_status st = decode_params_external_scratch(c, q, H_q, out, &p, &D, &HG, &dtype, &pre_rope, &rt,
                                                    &ragged, &rows);
    if (st != KIVI_OK) return st;
    if (rows > c->plan.part_rows) return KIVI_ERR_UNSUPPORTED;
    p.partials = c->partials;
    p.tickets = c->tickets;
    cudaError_t e = launch_decode(D, HG, dtype, pre_rope, p, ragged ? &rt : nullptr, (cudaStream_t)stream);
    return cuda_status(e);
}

kivi_status kivi_debug_expire_first_wait(kivi_cache *c, int on)
{
    if (!c) return KIVI_ERR_ARG;
    c->expire_first_wait = on ? 1 : 0;
    return KIVI_OK;
}

kivi_status kivi_device_status(kivi_cache *c, int *code)
{
    if (!c || !code) return KIVI_ERR_ARG;
    if (!on_cache_device(c)) return KIVI_ERR_ARG;
    cudaError_t e = cudaDeviceSynchronize();
    if (e == cudaSuccess) e = cudaMemcpy(code, c->err, sizeof(int), cudaMemcpyDeviceToHost);
    if (e == cudaSuccess && *code != 0) {
        e = cudaMemset(c->err, 0, sizeof(int));
        if (e == cudaSuccess) e = cudaMemset(c->tickets, 0, c->plan.tick_count * sizeof(int));
        if (e == cudaSuccess) e = cudaDeviceSynchronize();
    }
    return cuda_status(e);
}

}  // extern "C"

namespace {

template <int D>
void unpack_groups(long long nseq, const std::vector<uint8_t> &blk, long long n_g,
                   uint8_t *codesK, uint8_t *codesV, uint16_t *sK, uint16_t *zK, uint16_t *sV,
                   uint16_t *zV)
{
    using L = Layout<D>;
    const long long nq = n_g * kG;
    for (long long s = 0; s < nseq; ++s) {
        for (long long g = 0; g < n_g; ++g) {
            const uint8_t *b = blk.data() + (s * n_g + g) * L::GB;
            for (int lane = 0; lane < 32; ++lane) {
                for (int u = 0; u < L::WPL; ++u) {
                    uint32_t kw, vw;
                    std::memcpy(&kw, b + L::KC + code_word_offset(lane, u), 4);
                    std::memcpy(&vw, b + L::VC + code_word_offset(lane, u), 4);
                    // K word u = tok*KW + k of lane (tq, cs): pair i is local
                    // channels 16k+2i (bits 2i) and 16k+2i+1 (bits 16+2i).
                    const int tok = u / L::KW, k = u % L::KW;
                    const long long tK = g * kG + 4 * (lane >> 2) + tok;
                    // V word u of lane (co, th): pair i is token
                    // 16th + u*TPW + i/(CPL/2), channels co*CPL + 2*(i%(CPL/2)) + {0,1}.
                    const int co = lane & 15, th = lane >> 4;
                    for (int i = 0; i < 8; ++i) {
                        const int d0 = k_channel<D>(lane & 3, 16 * k + 2 * i);
                        const int d1 = k_channel<D>(lane & 3, 16 * k + 2 * i + 1);
                        if (codesK) {
                            codesK[(s * nq + tK) * D + d0] = (kw >> (2 * i)) & 3u;
                            codesK[(s * nq + tK) * D + d1] = (kw >> (16 + 2 * i)) & 3u;
                        }
                        const long long tV = g * kG + 16 * th + u * L::TPW + i / (L::CPL / 2);
                        const int dv = co * L::CPL + 2 * (i % (L::CPL / 2));
                        if (codesV) {
                            codesV[(s * nq + tV) * D + dv] = (vw >> (2 * i)) & 3u;
                            codesV[(s * nq + tV) * D + dv + 1] = (vw >> (16 + 2 * i)) & 3u;
                        }
                    }
                }
            }
            for (int d = 0; d < D; ++d) {
                const int off = L::KM + km_offset<D>(k_perm_index<D>(d));
                uint16_t sb, zb;
                std::memcpy(&sb, b + off, 2);
                std::memcpy(&zb, b + off + D / 16, 2);
                if (sK) sK[(s * n_g + g) * D + d] = sb;
                if (zK) zK[(s * n_g + g) * D + d] = zb;
            }
            for (int t = 0; t < kG; ++t) {
                for (int j = 0; j < L::NJ; ++j) {
                    const int off = L::VM + t * (D / 8) + j * 2;
                    uint16_t sb, zb;
                    std::memcpy(&sb, b + off, 2);
                    std::memcpy(&zb, b + off + D / 16, 2);
                    const long long tt = g * kG + t;
                    if (sV) sV[(s * nq + tt) * L::NJ + j] = sb;
                    if (zV) zV[(s * nq + tt) * L::NJ + j] = zb;
                }
            }
        }
    }
}

}  // namespace

extern "C" kivi_status kivi_export(const kivi_cache *c, long long seq0, long long nseq,
                                   uint8_t *codesK, uint8_t *codesV, uint16_t *sK, uint16_t *zK,
                                   uint16_t *sV, uint16_t *zV, void *resK, void *resV)
{
    if (!c || seq0 < 0 || nseq < 0 || seq0 + nseq > c->plan.seqs) return KIVI_ERR_ARG;
    if (!c->prefilled) return KIVI_ERR_STATE;
    if (nseq == 0) return KIVI_OK;
    const int D = c->cfg.D, R = c->cfg.R, H = c->cfg.H_kv;
    // The sequences exported share one split (all of them, unless ragged).
    const int b0 = (int)(seq0 / H), b1 = (int)((seq0 + nseq - 1) / H);
    const long long n_q = nq_at(c, b0);
    const int r = r_at(c, b0);
    for (int b = b0 + 1; b <= b1; ++b)
        if (nq_at(c, b) != n_q || r_at(c, b) != r) return KIVI_ERR_ARG;
    const long long n_g = n_q / kG;
    const size_t gb = (size_t)24 * D;
    cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return KIVI_ERR_CUDA;
    if (n_g > 0 && (codesK || codesV || sK || zK || sV || zV)) {
        std::vector<uint8_t> blk((size_t)nseq * n_g * gb);
        e = cudaMemcpy2D(blk.data(), n_g * gb, c->packed + (size_t)seq0 * c->plan.ngcap * gb,
                         c->plan.ngcap * gb, n_g * gb, nseq, cudaMemcpyDeviceToHost);
        if (e != cudaSuccess) return KIVI_ERR_CUDA;
        if (D == 64) unpack_groups<64>(nseq, blk, n_g, codesK, codesV, sK, zK, sV, zV);
        else unpack_groups<128>(nseq, blk, n_g, codesK, codesV, sK, zK, sV, zV);
    }
    const size_t row = (size_t)D * 2;
    const size_t off = (size_t)seq0 * R * D;
    if (resK) {
        e = cudaMemcpy2D(resK, r * row, c->resK + off, (size_t)R * row, r * row, nseq,
                         cudaMemcpyDeviceToHost);
        if (e != cudaSuccess) return KIVI_ERR_CUDA;
    }
    if (resV) {
        e = cudaMemcpy2D(resV, r * row, c->resV + off, (size_t)R * row, r * row, nseq,
                         cudaMemcpyDeviceToHost);
        if (e != cudaSuccess) return KIVI_ERR_CUDA;
    }
    return KIVI_OK;
}

extern "C" kivi_status kivi_decode_split(long long seqs, long long n_groups, int r, int wg, int wr,
                                         long long warps, long long seq, long long warp,
                                         long long out[4])
{
    if (!out || seqs < 1 || n_groups < 0 || r < 0 || wg < 1 || wr < 1 || warps < 1) return KIVI_ERR_ARG;
    Split sp;
    sp.init(seqs, n_groups, r, wg, wr, warps);
    if (sp.Tot < 1 || warps > sp.Tot || seq < 0 || seq >= seqs || warp < 0 || warp >= warps)
        return KIVI_ERR_ARG;
    if ((double)sp.Tot * (double)(warps + 1) >= 9007199254740992.0) return KIVI_ERR_UNSUPPORTED;
    sp.set_magics();
    out[0] = sp.owner(seq * sp.C);
    out[1] = sp.owner((seq + 1) * sp.C - 1);
    const ItemRange it = sp.items(seq, warp);
    out[2] = it.first;
    out[3] = it.second;
    return KIVI_OK;
}

namespace kivi {

// Launch parameters of a decode call on cache c, validated exactly as
// kivi_decode_attn validates them, with the scratch pointers (partials,
// tickets) and the partial slot count left for the caller to fill.
kivi_status decode_params_external_scratch(kivi_cache *c, const void *q, int H_q, float *out,
                                           DecodeParams *p, int *D, int *HG, int *dtype,
                                           int *pre_rope, RaggedTab *rt, bool *ragged, long long *rows)
{
    if (!c || !q || !out || !p || !rt || !ragged || !rows || !aligned16(q) || !aligned16(out))
        return KIVI_ERR_ARG;
    if (!on_cache_device(c)) return KIVI_ERR_ARG;
    if (!c->prefilled) return KIVI_ERR_STATE;
    if (H_q < 1 || H_q % c->cfg.H_kv != 0) return KIVI_ERR_ARG;
    const int hg = H_q / c->cfg.H_kv;
    const int nw = decode_warps_per_sm(c->cfg.D, hg, c->cfg.pre_rope);
    if (nw == 0 || hg > kMaxGroupHeads) return KIVI_ERR_UNSUPPORTED;
    *ragged = c->ragged;
    Split sp;
    long long Tot, warps = (long long)c->sms * nw;
    if (c->ragged) {
        ragged_table(c, rt);
        Tot = rt->off[rt->nb];
        if (warps > Tot) warps = Tot;
        sp.init(c->plan.seqs, rt->ng[0], rt->r[0], c->wg, c->wr, warps);
        sp.Tot = Tot;
    } else {
        sp.init(c->plan.seqs, c->n_q / kG, c->r, c->wg, c->wr, 1);
        if (warps > sp.Tot) warps = sp.Tot;
        sp.init(c->plan.seqs, c->n_q / kG, c->r, c->wg, c->wr, warps);
        Tot = sp.Tot;
    }
    // The split's divisions are exact for numerators below 2^53 (div_floor).
    if ((double)Tot * (double)(warps + 1) >= 9007199254740992.0) return KIVI_ERR_UNSUPPORTED;
    sp.set_magics();
    p->div_C = sp.mC;
    p->div_Tot = sp.mT;
    p->div_warps = sp.mW;
    p->div_wg = sp.mG;
    p->div_wr = sp.mR;
    p->div_Hkv = make_magic((unsigned long long)c->cfg.H_kv);
    p->packed = c->packed;
    p->ngcap = c->plan.ngcap;
    p->resK = c->resK;
    p->resV = c->resV;
    p->R = c->cfg.R;
    p->q = (const uint16_t *)q;
    p->out = out;
    p->partials = nullptr;
    p->tickets = nullptr;
    p->err = c->err;
    p->H_kv = c->cfg.H_kv;
    p->H_q = H_q;
    p->seqs = c->plan.seqs;
    p->n_groups = c->ragged ? 0 : c->n_q / kG;
    p->r = c->ragged ? 1 : c->r;
    p->n_q = c->ragged ? 0 : c->n_q;
    p->wg = c->wg;
    p->wr = c->wr;
    p->warps = warps;
    *rows = warps + p->seqs;
    p->qscale = (float)(1.4426950408889634 / std::sqrt((double)c->cfg.D));
    p->inv_freq = c->inv_freq;
    p->newK = p->newV = nullptr;
    p->new_slot = -1;
    p->expire_first_wait = c->expire_first_wait;
    p->magic = 0x4B000000u;
    p->neg_magic = -8388608.0f;
    *D = c->cfg.D;
    *HG = hg;
    *dtype = c->cfg.dtype;
    *pre_rope = c->cfg.pre_rope;
    return KIVI_OK;
}

}  // namespace kivi
