// kivi_noalloc.cu -- decode attention whose scratch lives in a fixed device
// array, for callers that may not allocate device memory.
//
// kivi_decode_attn keeps its split-K partials and per-sequence tickets in the
// cache's own buffers.  Some hosts cannot give the library any memory beyond
// the cache itself and the call's inputs and outputs: an engine that plans
// every device byte up front and forbids allocation once it is serving, a
// plugin that only receives pointers from its host application, or code on a
// path where cudaMalloc's implicit device-wide synchronisation is not
// acceptable.  kivi_decode_attn_noalloc runs the same decode kernel with its
// scratch in a file-scope device array of kNoAllocScratchBytes, which every
// GPU that loads this library holds until the process exits.
#include <cstdint>
#include <mutex>

#include <cuda_runtime.h>

#include "../../include/kivi.h"
#include "kivi_common.cuh"
#include "kivi_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB per device
using kivi::kMaxDevices;

// Tickets first, then the partials.  Shared by every call on the device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_mu;
void *g_scratch_addr[kMaxDevices];

// Device address of g_noalloc_scratch on the current device, looked up once
// per device (the host-side symbol is only a stand-in, not a device address).
// The address is kept for the life of the process: a cudaDeviceReset (or any
// reset of the device's primary context) while this library is loaded
// invalidates it, so the library must not outlive such a reset.
cudaError_t scratch_on_current_device(void **addr)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_addr[dev]) {
        void *ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev] = ptr;
    }
    *addr = g_scratch_addr[dev];
    return cudaSuccess;
}

}  // namespace

extern "C" kivi_status kivi_decode_attn_noalloc(kivi_cache *c, const void *q, int H_q, float *out,
                                                void *stream)
{
    kivi::DecodeParams p;
    kivi::RaggedTab rt;
    bool ragged = false;
    long long rows = 0;
    int D = 0, HG = 0, dtype = 0, pre_rope = 0;
    kivi_status st = kivi::decode_params_external_scratch(c, q, H_q, out, &p, &D, &HG, &dtype,
                                                          &pre_rope, &rt, &ragged, &rows);
    if (st != KIVI_OK) return st;
    // One ticket per sequence and one per partial row (merge blocks).
    const size_t tick_count = (size_t)p.seqs + (size_t)rows;
    const size_t tick_bytes = (tick_count * sizeof(int) + 255) / 256 * 256;
    const size_t part_bytes = (size_t)rows * HG * (D + 4) * sizeof(float);
    if (tick_bytes + part_bytes > kNoAllocScratchBytes) return KIVI_ERR_CAPACITY;
    void *base = nullptr;
    cudaError_t e = scratch_on_current_device(&base);
    if (e != cudaSuccess) {
        cudaGetLastError();   // the lookup's error is not a launch failure: clear it
        return KIVI_ERR_CUDA;
    }
    p.tickets = (int *)base;
    p.partials = (float *)((unsigned char *)base + tick_bytes);
    // The array keeps the previous call's contents: the tickets must start at 0.
    e = cudaMemsetAsync(p.tickets, 0, tick_count * sizeof(int), (cudaStream_t)stream);
    if (e == cudaSuccess)
        e = kivi::launch_decode(D, HG, dtype, pre_rope, p, ragged ? &rt : nullptr, (cudaStream_t)stream);
    return kivi::cuda_status(e);
}
