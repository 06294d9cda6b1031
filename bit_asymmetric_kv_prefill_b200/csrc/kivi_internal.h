// kivi_internal.h -- kernel launch interface between the C ABI and the CUDA
// kernels.  Internal to the library.
#pragma once

#include <atomic>
#include <cstdint>
#include <cuda_runtime.h>

#include "kivi.h"
#include "kivi_common.cuh"

namespace kivi {

// Quantize whole groups of 32 tokens into the packed store (prefill and the
// flush of a full residual), optionally copying the prefill's residual rows and
// writing an appended token into residual slot 0 after the flush has read it.
struct QuantParams {
    const uint16_t *srcK, *srcV;  // rows of source group 0 of sequence 0
    long long src_seq_rows;       // rows between consecutive sequences in src
    uint8_t *packed;              // [seqs][ngcap][24*D]
    long long ngcap;              // group capacity per sequence
    long long g_dst0;             // destination index of source group 0
    int n_g;                      // groups per sequence to quantize
    long long seqs;
    uint16_t *resK, *resV;        // [seqs][R][D]
    int R;
    int r_copy;                   // prefill: residual rows to copy (0: none)
    long long copy_row0;          // prefill: first source row of the residual
    const uint16_t *newK, *newV;  // flush: token to store in slot 0 (or null)
    Magic div_ng;                 // division by n_g (set by launch_quant)
};

// Segments of a quantizer launch whose sequences do not share one length
// (ragged prefill, or a flush of some batch elements): segment k covers
// sequences [seq0, seq0 + nseq), each quantizing n_g groups from its source
// rows 0.. into destination groups g_dst0.., then (r_copy > 0) copying source
// rows [copy_row0, copy_row0 + r_copy) into residual slots 0..  Work items of
// segment k: [item0[k], item0[k + 1]), the group items first.
constexpr int kMaxQuantSegs = kMaxRaggedB;
struct QuantSegs {
    int nseg;
    int seq0[kMaxQuantSegs], nseq[kMaxQuantSegs], n_g[kMaxQuantSegs], g_dst0[kMaxQuantSegs];
    int r_copy[kMaxQuantSegs], copy_row0[kMaxQuantSegs];
    long long item0[kMaxQuantSegs + 1];
};

// Residual slot per batch element for an append (-1: the element is skipped).
struct SlotTab {
    int slot[kMaxRaggedB];
};

struct DecodeParams {
    const uint8_t *packed;
    long long ngcap;
    const uint16_t *resK, *resV;
    int R;
    const uint16_t *q;
    float *out;
    float *partials;     // rows of [HG][D+4]: sequence s, partial slot k at row first(s) + s + k
    int *tickets;        // [seqs + partial rows]: sequence s at s, merge block of row r at seqs + r
    int *err;            // status word
    int H_kv, H_q;
    long long seqs;
    long long n_groups;  // quantized groups per sequence
    int r;               // residual tokens
    long long n_q;       // absolute position of residual slot 0
    int wg, wr;          // split weights of a group / a residual item
    long long warps;     // total warps of the split (<= total weight)
    Magic div_C, div_Tot, div_warps, div_wg, div_wr, div_Hkv;   // divisions of the split
    float qscale;        // log2(e) / sqrt(D)
    uint32_t magic;      // bits of 2^23 (the code-to-float exponent)
    float neg_magic;     // -2^23
    const float *inv_freq;  // RoPE inverse frequencies [D/2] (pre-RoPE caches)
    // Fused append: the token at residual slot new_slot is read from newK /
    // newV ([seqs][D]) and stored to the residual by the decode (else null, -1).
    const uint16_t *newK, *newV;
    int new_slot;
    // Testing the failure path: each warp's first consuming wait gives up at
    // once (the kernel then reports a failed wait and drains its copies).
    int expire_first_wait;
};

int num_sms();

// Status of a CUDA runtime result, as every entry point reports it.
inline kivi_status cuda_status(cudaError_t e) { return e == cudaSuccess ? KIVI_OK : KIVI_ERR_CUDA; }

// A kernel's dynamic shared-memory limit belongs to each device's context, so
// it is raised once per device.  The flags are per device and atomic: host
// threads driving caches on different devices each configure their own; two
// threads racing on one device both make the same (idempotent) call.
constexpr int kMaxDevices = 64;
struct PerDeviceOnce {
    std::atomic<bool> done[kMaxDevices];
};

template <typename Kernel>
cudaError_t set_smem_once(PerDeviceOnce &once, Kernel kernel, int bytes)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (once.done[dev].load(std::memory_order_acquire)) return cudaSuccess;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) once.done[dev].store(true, std::memory_order_release);
    return e;
}

// segs: null for one length across the sequences (the QuantParams fields),
// else the segments (QuantParams' n_g, g_dst0, r_copy, copy_row0 unused).
cudaError_t launch_quant(int D, int dtype, const QuantParams &p, const QuantSegs *segs,
                         cudaStream_t st);
cudaError_t launch_append(int D, const uint16_t *k, const uint16_t *v, uint16_t *resK,
                          uint16_t *resV, long long seqs, int R, int slot, cudaStream_t st);
// Append into per-batch-element slots (slots->slot[b] < 0: element b skipped).
cudaError_t launch_append_slots(int D, const uint16_t *k, const uint16_t *v, uint16_t *resK,
                                uint16_t *resV, long long seqs, int H_kv, int R, const SlotTab &slots,
                                cudaStream_t st);
// Resident decode warps per SM for this shape (0 if unsupported).
int decode_warps_per_sm(int D, int HG, int pre_rope);
// rt: null for one length across the sequences, else the ragged table.
cudaError_t launch_decode(int D, int HG, int dtype, int pre_rope, const DecodeParams &p,
                          const RaggedTab *rt, cudaStream_t st);
// Launch parameters of a decode call on cache c, validated as every decode
// entry point validates them; the scratch pointers (partials, tickets) are
// left null.  A ragged cache fills *rt and sets *ragged.  *rows is the
// number of partial rows (each HG x (D + 4) floats) the split needs.
kivi_status decode_params_external_scratch(kivi_cache *c, const void *q, int H_q, float *out,
                                           DecodeParams *p, int *D, int *HG, int *dtype,
                                           int *pre_rope, RaggedTab *rt, bool *ragged,
                                           long long *rows);

}  // namespace kivi
