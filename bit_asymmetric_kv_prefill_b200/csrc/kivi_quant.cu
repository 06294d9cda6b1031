// kivi_quant.cu -- prefill quantizer and residual append/flush kernels.
//
// Keys are grouped per channel over 32 consecutive tokens and values per token
// over 32 consecutive channels ("KIVI Quantization Secures Llama-2 Accuracy at
// Two Bits", paragraphs 2-3; record kv-efficiency/kivi-2bit-llama2-13b-mha-4k,
// "Quant method": kivi-2bit-per-channel-k-per-token-v).  Each CTA takes one
// group tile (32 tokens x D channels of K and of V) at a time:
//   1. the tile is staged into padded shared memory with cp.async, double
//      buffered across the CTA's groups;
//   2. per-channel key min/max (one thread per channel) and per-token value
//      min/max (warp-shuffle reductions over the 32 channels of a group) give
//      the fp16 scale/zero and three exact fp32 code thresholds per group;
//   3. every 32-bit word of 16 codes is built by one thread and the finished
//      24*D-byte group block is written out with coalesced 16-byte stores.
// The residual rows of a prefill and the appended token of a flush are copied
// by the same launch.
#include <cuda_runtime.h>

#include "kivi_common.cuh"
#include "kivi_internal.h"

namespace kivi {

template <int DT>
__device__ __forceinline__ float to_f(uint16_t b)
{
    if constexpr (DT == 1) return __uint_as_float((uint32_t)b << 16);  // bf16
    else return __half2float(__ushort_as_half(b));                     // fp16
}

__device__ __forceinline__ void cp_async16(void *smem, const void *gmem)
{
    uint32_t s = (uint32_t)__cvta_generic_to_shared(smem);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ float warp_min(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fminf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}
__device__ __forceinline__ float warp_max(float x)
{
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
    return x;
}

constexpr int kQuantThreads = 256;

template <int D>
struct QuantSmem {
    static constexpr int RS = D + 8;                      // padded row, elements
    static constexpr int TILE = 32 * RS;                  // one K or V tile
    static constexpr int TILES_BYTES = 2 * 2 * TILE * 2;  // 2 buffers x (K, V)
    static constexpr int STATK = TILES_BYTES;             // float4 [D]
    static constexpr int STATV = STATK + D * 16;          // float4 [32][D/32]
    static constexpr int OUTB = STATV + 32 * (D / 32) * 16;
    static constexpr int BYTES = OUTB + 24 * D;
};

template <int D, int DT>
__device__ void quantize_tile(const QuantParams &p, long long item, const uint16_t *tk,
                              const uint16_t *tv, float4 *statK, float4 *statV, uint8_t *outb)
{
    using L = Layout<D>;
    constexpr int RS = QuantSmem<D>::RS;
    const int tid = threadIdx.x;
    const long long s = item / p.n_g;
    const int g = (int)(item % p.n_g);

    if (tid < D) {
        // Keys, per channel: min/max over the 32 tokens of channel tid.
        float mn = to_f<DT>(tk[tid]), mx = mn;
#pragma unroll 8
        for (int t = 1; t < 32; ++t) {
            float x = to_f<DT>(tk[t * RS + tid]);
            mn = fminf(mn, x);
            mx = fmaxf(mx, x);
        }
        CodeParams cp = code_params(mn, mx);
        statK[tid] = make_float4(cp.e1, cp.e2, cp.e3, cp.z);
        int off = L::KM + km_offset<D>(k_perm_index<D>(tid));
        *(uint16_t *)(outb + off) = cp.s_bits;
        *(uint16_t *)(outb + off + D / 16) = cp.z_bits;
    } else {
        // Values, per token: warp-shuffle min/max over 32 channels.
        const int nvw = (kQuantThreads - D) / 32;
        const int w = (tid - D) >> 5, lane = tid & 31;
        for (int t = w; t < 32; t += nvw) {
#pragma unroll
            for (int j = 0; j < L::NJ; ++j) {
                float x = to_f<DT>(tv[t * RS + j * 32 + lane]);
                float mn = warp_min(x), mx = warp_max(x);
                if (lane == 0) {
                    CodeParams cp = code_params(mn, mx);
                    statV[t * L::NJ + j] = make_float4(cp.e1, cp.e2, cp.e3, cp.z);
                    int off = L::VM + t * (D / 8) + j * 2;
                    *(uint16_t *)(outb + off) = cp.s_bits;
                    *(uint16_t *)(outb + off + D / 16) = cp.z_bits;
                }
            }
        }
    }
    __syncthreads();

    // Key code words: thread -> (lane, token pair, word slot k); tokens tok and
    // tok+2 of the lane share the 16 channels, so their thresholds load once.
    if (tid < D) {
        const int lane = tid / (2 * L::KW), rem = tid % (2 * L::KW);
        const int tokp = rem / L::KW, k = rem % L::KW;
        const int cs = lane & 3, tq = lane >> 2;
        constexpr int RUN = (D / 8) < 16 ? (D / 8) : 16;  // contiguous channels
        float4 th[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) th[i] = statK[k_channel<D>(cs, 16 * k + i)];
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int tok = tokp + 2 * h;
            const int t = 4 * tq + tok;
            uint32_t word = 0;
#pragma unroll
            for (int r0 = 0; r0 < 16; r0 += RUN) {
                const int c0 = k_channel<D>(cs, 16 * k + r0);
                uint16_t xs[RUN];
#pragma unroll
                for (int v = 0; v < RUN; v += 8)
                    *(uint4 *)&xs[v] = *(const uint4 *)&tk[t * RS + c0 + v];
#pragma unroll
                for (int i = 0; i < RUN; ++i) {
                    const float4 e = th[r0 + i];
                    word |= code_of(to_f<DT>(xs[i]), e.w, e.x, e.y, e.z) << (2 * (r0 + i));
                }
            }
            *(uint32_t *)(outb + L::KC + code_word_offset(lane, tok * L::KW + k)) = word;
        }
    }
    // Value code words: thread -> (lane, word u); TPW tokens x CPL channels.
    for (int vp = tid; vp < 2 * D; vp += kQuantThreads) {
        const int lane = vp / L::WPL, u = vp % L::WPL;
        const int j = lane * L::CPL / 32;
        uint32_t word = 0;
#pragma unroll
        for (int tt = 0; tt < L::TPW; ++tt) {
            const int t = u * L::TPW + tt;
            const float4 e = statV[t * L::NJ + j];
            uint16_t xs[L::CPL];
            if constexpr (L::CPL == 4) {
                *(uint2 *)xs = *(const uint2 *)&tv[t * RS + lane * 4];
            } else {
#pragma unroll
                for (int c = 0; c < L::CPL; ++c) xs[c] = tv[t * RS + lane * L::CPL + c];
            }
#pragma unroll
            for (int c = 0; c < L::CPL; ++c)
                word |= code_of(to_f<DT>(xs[c]), e.w, e.x, e.y, e.z) << (2 * (tt * L::CPL + c));
        }
        *(uint32_t *)(outb + L::VC + code_word_offset(lane, u)) = word;
    }
    __syncthreads();

    uint4 *dst = (uint4 *)(p.packed + ((s * p.ngcap) + p.g_dst0 + g) * (long long)L::GB);
    for (int c = tid; c < L::GB / 16; c += kQuantThreads) dst[c] = ((const uint4 *)outb)[c];

    if (p.newK != nullptr && g == 0) {
        // The flush has read residual slot 0 into shared memory (the tile was
        // complete before the first __syncthreads): the new token may land.
        for (int c = tid; c < 2 * (D / 8); c += kQuantThreads) {
            const int which = c / (D / 8), q = c % (D / 8);
            const uint16_t *src = (which ? p.newV : p.newK) + s * D + q * 8;
            uint16_t *d = (which ? p.resV : p.resK) + s * (long long)p.R * D + q * 8;
            *(uint4 *)d = *(const uint4 *)src;
        }
    }
}

template <int D, int DT>
__global__ void __launch_bounds__(kQuantThreads) quant_kernel(QuantParams p)
{
    using S = QuantSmem<D>;
    extern __shared__ __align__(16) unsigned char smem[];
    uint16_t *tiles = (uint16_t *)smem;
    float4 *statK = (float4 *)(smem + S::STATK);
    float4 *statV = (float4 *)(smem + S::STATV);
    uint8_t *outb = smem + S::OUTB;

    const long long n_group_items = p.seqs * (long long)p.n_g;
    const long long n_items = n_group_items + (p.r_copy > 0 ? p.seqs : 0);
    const int tid = threadIdx.x;

    auto issue = [&](long long item, int buf) {
        if (item >= n_group_items) return;
        const long long s = item / p.n_g;
        const int g = (int)(item % p.n_g);
        const long long row0 = s * p.src_seq_rows + (long long)g * 32;
        const uint16_t *k = p.srcK + row0 * D;
        const uint16_t *v = p.srcV + row0 * D;
        uint16_t *tk = tiles + (buf * 2 + 0) * S::TILE;
        uint16_t *tv = tiles + (buf * 2 + 1) * S::TILE;
        for (int c = tid; c < 32 * (D / 8); c += kQuantThreads) {
            const int row = c / (D / 8), col = (c % (D / 8)) * 8;
            cp_async16(tk + row * S::RS + col, k + row * D + col);
            cp_async16(tv + row * S::RS + col, v + row * D + col);
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
        __syncthreads();
        if (item < n_group_items) {
            quantize_tile<D, DT>(p, item, tiles + (buf * 2 + 0) * S::TILE,
                                 tiles + (buf * 2 + 1) * S::TILE, statK, statV, outb);
        } else {
            // Prefill residual: rows [copy_row0, copy_row0 + r_copy) -> slots.
            const long long s = item - n_group_items;
            const long long n16 = (long long)p.r_copy * (D / 8);
            const uint4 *sk = (const uint4 *)(p.srcK + (s * p.src_seq_rows + p.copy_row0) * D);
            const uint4 *sv = (const uint4 *)(p.srcV + (s * p.src_seq_rows + p.copy_row0) * D);
            uint4 *dk = (uint4 *)(p.resK + s * (long long)p.R * D);
            uint4 *dv = (uint4 *)(p.resV + s * (long long)p.R * D);
            for (long long c = tid; c < n16; c += kQuantThreads) {
                dk[c] = sk[c];
                dv[c] = sv[c];
            }
        }
        __syncthreads();
    }
    cp_async_wait<0>();
}

// Plain append: token rows [seqs][D] -> residual slot `slot` of each sequence.
__global__ void append_kernel(const uint4 *k, const uint4 *v, uint4 *resK, uint4 *resV,
                              long long seqs, int R, int slot, int n16)
{
    long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    long long total = seqs * n16;
    if (i >= total) return;
    long long s = i / n16;
    int c = (int)(i % n16);
    long long d = (s * R + slot) * n16 + c;
    resK[d] = k[i];
    resV[d] = v[i];
}

int num_sms()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 148;
    return n;
}

template <int D, int DT>
static cudaError_t launch_quant_t(const QuantParams &p, cudaStream_t st)
{
    using S = QuantSmem<D>;
    static bool configured = false;
    if (!configured) {
        cudaError_t e = cudaFuncSetAttribute(quant_kernel<D, DT>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, S::BYTES);
        if (e != cudaSuccess) return e;
        configured = true;
    }
    const long long items = p.seqs * (long long)p.n_g + (p.r_copy > 0 ? p.seqs : 0);
    if (items == 0) return cudaSuccess;
    long long grid = (long long)num_sms() * 4;
    if (grid > items) grid = items;
    quant_kernel<D, DT><<<(unsigned)grid, kQuantThreads, S::BYTES, st>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_quant(int D, int dtype, const QuantParams &p, cudaStream_t st)
{
    if (D == 64) return dtype ? launch_quant_t<64, 1>(p, st) : launch_quant_t<64, 0>(p, st);
    if (D == 128) return dtype ? launch_quant_t<128, 1>(p, st) : launch_quant_t<128, 0>(p, st);
    return cudaErrorInvalidValue;
}

cudaError_t launch_append(int D, const uint16_t *k, const uint16_t *v, uint16_t *resK,
                          uint16_t *resV, long long seqs, int R, int slot, cudaStream_t st)
{
    const int n16 = D / 8;
    const long long total = seqs * n16;
    const int block = 256;
    const long long grid = (total + block - 1) / block;
    append_kernel<<<(unsigned)grid, block, 0, st>>>((const uint4 *)k, (const uint4 *)v,
                                                     (uint4 *)resK, (uint4 *)resV, seqs, R, slot,
                                                     n16);
    return cudaGetLastError();
}

}  // namespace kivi
