// kivi_levels.cu -- quantize-dequantize with non-uniform levels per group
// (kivi_fake_quant_levels), the KVQuant variant the pages name: "Non-Uniform
// KV Cache Quantization" (KVQuant summary).  The pages give only the name;
// here every group keeps its minimum and maximum and codes each element by
// the nearest of `nlev` normalized levels on [min, max]:
//   u = (x - min) / (max - min)              (IEEE fp64: subtract, divide)
//   code = argmin_k |u - l_k|                (the first level on ties)
//   x_hat = fp32(min + (max - min) * l_code) (fp64 multiply, then add)
// and a constant group decodes to its value with code 0.  The levels come
// from the caller (fitted offline on calibration data in KVQuant; fitted on
// the data itself by Lloyd's algorithm in this project's diagnostics).
//
// The decision is taken in fp64 exactly as written, so the codes and x_hat
// are those of a plain evaluation of the formulas above.  One thread owns one
// group: per channel, consecutive threads own consecutive channels of the
// same rows (coalesced); per token, a thread reads its G contiguous channels.
// The group is read twice, min/max first and codes second (the second pass
// hits L1/L2).  The work is a diagnostic, not on the decode path; its cost is
// the fp64 division and the nlev distance tests per element.
#include <cstdint>

#include <cuda_runtime.h>

#include "../../include/kivi.h"
#include "kivi_common.cuh"
#include "kivi_internal.h"

namespace kivi {
namespace {

constexpr int kLvThreads = 256;
constexpr int kMaxLevels = 256;

struct LvParams {
    const uint16_t *x;   // [N][T][D]
    float *xhat;         // [N][T][D] or null
    uint8_t *codes;      // [N][T][D] or null
    double *sq_err;      // [N] or null
    long long N, T;
    int D, G, nlev, axis;
    long long groups_per_matrix, groups;
    double lev[kMaxLevels];
};

template <int DT>
__device__ __forceinline__ float load_x(const uint16_t *p)
{
    const uint16_t b = __ldg(p);
    if constexpr (DT == KIVI_BF16) return __uint_as_float((uint32_t)b << 16);
    else return __half2float(__ushort_as_half(b));
}

template <int DT>
__global__ void __launch_bounds__(kLvThreads) levels_kernel(const __grid_constant__ LvParams p)
{
    const long long stride = (long long)gridDim.x * kLvThreads;
    for (long long gi = (long long)blockIdx.x * kLvThreads + threadIdx.x; gi - threadIdx.x < p.groups;
         gi += stride) {
        const bool active = gi < p.groups;
        long long n = 0, base = 0, step = 1;
        if (active) {
            n = gi / p.groups_per_matrix;
            const long long r = gi - n * p.groups_per_matrix;
            if (p.axis == KIVI_AXIS_PER_CHANNEL) {
                // group (g, d): tokens [gG, gG + G) of channel d
                const long long g = r / p.D, d = r - g * p.D;
                base = n * p.T * p.D + g * p.G * p.D + d;
                step = p.D;
            } else {
                // group (t, j): channels [jG, jG + G) of token t
                const long long nj = p.D / p.G;
                const long long t = r / nj, j = r - t * nj;
                base = n * p.T * p.D + t * p.D + j * p.G;
                step = 1;
            }
        }
        double err = 0.0;
        if (active) {
            float mn = load_x<DT>(p.x + base), mx = mn;
            for (int i = 1; i < p.G; ++i) {
                const float v = load_x<DT>(p.x + base + i * step);
                mn = fminf(mn, v);
                mx = fmaxf(mx, v);
            }
            const double dmn = (double)mn;
            const double range = __dsub_rn((double)mx, dmn);
            for (int i = 0; i < p.G; ++i) {
                const long long at = base + i * step;
                const float v = load_x<DT>(p.x + at);
                int c = 0;
                float xh = mn;
                if (range > 0.0) {
                    const double u = __ddiv_rn(__dsub_rn((double)v, dmn), range);
                    double best = fabs(__dsub_rn(u, p.lev[0]));
                    for (int k = 1; k < p.nlev; ++k) {
                        const double e = fabs(__dsub_rn(u, p.lev[k]));
                        if (e < best) {
                            best = e;
                            c = k;
                        }
                    }
                    xh = __double2float_rn(__dadd_rn(dmn, __dmul_rn(range, p.lev[c])));
                }
                if (p.xhat) p.xhat[at] = xh;
                if (p.codes) p.codes[at] = (uint8_t)c;
                const double df = __dsub_rn((double)v, (double)xh);
                err = __fma_rn(df, df, err);
            }
        }
        if (p.sq_err) {
            // One atomic per warp when its lanes share the matrix, else per lane.
            const unsigned act = __ballot_sync(0xffffffffu, active);
            const long long n0 = __shfl_sync(0xffffffffu, n, 0);
            if (__all_sync(0xffffffffu, !active || n == n0) && act == 0xffffffffu) {
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) err += __shfl_xor_sync(0xffffffffu, err, o);
                if ((threadIdx.x & 31) == 0) atomicAdd(p.sq_err + n0, err);
            } else if (active) {
                atomicAdd(p.sq_err + n, err);
            }
        }
    }
}

}  // namespace
}  // namespace kivi

using namespace kivi;

extern "C" kivi_status kivi_fake_quant_levels(const void *x, kivi_dtype dtype, long long N, long long T,
                                              int D, int axis, int G, int nlev, const double *levels,
                                              float *xhat, uint8_t *codes, double *sq_err, void *stream)
{
    if (!x || !levels || (!xhat && !codes && !sq_err)) return KIVI_ERR_ARG;
    if (((uintptr_t)x & 15u) || ((uintptr_t)xhat & 15u) || ((uintptr_t)sq_err & 7u)) return KIVI_ERR_ARG;
    if (dtype != KIVI_F16 && dtype != KIVI_BF16) return KIVI_ERR_ARG;
    if (N < 1 || T < 1 || D < 1 || G < 1) return KIVI_ERR_ARG;
    if (axis != KIVI_AXIS_PER_CHANNEL && axis != KIVI_AXIS_PER_TOKEN) return KIVI_ERR_ARG;
    if (axis == KIVI_AXIS_PER_CHANNEL ? T % G != 0 : D % G != 0) return KIVI_ERR_ARG;
    if (nlev < 2 || nlev > kMaxLevels) return KIVI_ERR_ARG;
    for (int k = 0; k < nlev; ++k)
        if (!(levels[k] >= 0.0 && levels[k] <= 1.0)) return KIVI_ERR_ARG;
    if (T > (1LL << 40) / D || N > (1LL << 62) / (T * D)) return KIVI_ERR_UNSUPPORTED;

    LvParams p;
    p.x = (const uint16_t *)x;
    p.xhat = xhat;
    p.codes = codes;
    p.sq_err = sq_err;
    p.N = N;
    p.T = T;
    p.D = D;
    p.G = G;
    p.nlev = nlev;
    p.axis = axis;
    p.groups_per_matrix = T * (long long)D / G;
    p.groups = N * p.groups_per_matrix;
    for (int k = 0; k < kMaxLevels; ++k) p.lev[k] = k < nlev ? levels[k] : 0.0;

    cudaStream_t st = (cudaStream_t)stream;
    if (sq_err && cudaMemsetAsync(sq_err, 0, (size_t)N * sizeof(double), st) != cudaSuccess)
        return KIVI_ERR_CUDA;
    long long grid = (p.groups + kLvThreads - 1) / kLvThreads;
    const long long cap = (long long)num_sms() * (2048 / kLvThreads);
    if (grid > cap) grid = cap;
    if (dtype == KIVI_BF16) levels_kernel<KIVI_BF16><<<(unsigned)grid, kLvThreads, 0, st>>>(p);
    else levels_kernel<KIVI_F16><<<(unsigned)grid, kLvThreads, 0, st>>>(p);
    return cuda_status(cudaGetLastError());
}
