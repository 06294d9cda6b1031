/*
 * kivi.h -- C ABI of the B200 (sm_100a) KIVI asymmetric 2-bit KV cache.
 *
 * The method (KIVI: A Tuning-Free Asymmetric 2bit Quantization for KV Cache;
 * "KIVI Quantization Secures Llama-2 Accuracy at Two Bits", paragraphs 1-4;
 * record kv-efficiency/kivi-2bit-llama2-13b-mha-4k, fields "KV bytes basis"
 * and "Quant method"):
 *   - keys are quantized per channel: one (scale, zero) per channel per G
 *     consecutive tokens; values per token: one (scale, zero) per G
 *     consecutive channels of a token; 2-bit codes, zero = group minimum,
 *     scale = (max - min)/3, code = clamp(rint((x - zero)/scale), 0, 3), with
 *     scale and zero stored as IEEE fp16 and codes taken against the stored
 *     values;
 *   - the newest tokens stay in a full-precision residual of R slots; prefill
 *     of T tokens quantizes n_q = R*floor((T-1)/R) and keeps r = T - n_q in
 *     [1, R]; an append into a full residual first quantizes all R residual
 *     tokens into the grouped store;
 *   - decode attention softmax(q.k/sqrt(D)) v runs directly over the packed
 *     cache plus the residual; query head h reads kv head h / (H_q/H_kv);
 *   - optionally keys are quantized before RoPE (KIVI article, paragraph 4;
 *     KVQuant summary, "Pre-RoPE Key Quantization") and rotated at dequant:
 *     rotate-half pairs (i, i+D/2), absolute positions from 0, angle =
 *     fp32(t * inv_freq_i), inv_freq_i = fp32(theta^(-2i/D)).
 *
 * Conventions shared by every call
 *   - Pointers named K, V, k_t, v_t, q, out are DEVICE pointers owned by the
 *     caller, 16-byte aligned, contiguous:
 *       K, V      [B, H_kv, T, D]  cache dtype
 *       k_t, v_t  [B, H_kv, D]     cache dtype
 *       q         [B, H_q, D]      cache dtype, already rotated by RoPE
 *       out       [B, H_q, D]      fp32
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *     stream).  Every call that launches work is asynchronous on it; calls on
 *     one cache must be ordered by the caller (one stream per cache).
 *   - Arguments are checked before any launch; on an error status nothing
 *     was launched and the cache is unchanged.  KIVI_ERR_CUDA reports a
 *     launch or runtime failure (cudaGetLastError), after which the cache
 *     contents are undefined.
 *   - A cache belongs to the CUDA device that was current when it was
 *     created.  prefill, append, decode and the device-status read must be
 *     called with that device current; otherwise they return KIVI_ERR_ARG
 *     and launch nothing.
 *   - Sequence lengths live on the host (no device->host synchronisation in
 *     prefill, append or decode).
 *   - A cache is not thread-safe.  No call allocates device memory except
 *     kivi_cache_create / kivi_cache_create_ex without a workspace.
 */
#ifndef KIVI_H
#define KIVI_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KIVI_API __attribute__((visibility("default")))
#else
#define KIVI_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct kivi_cache kivi_cache; /* opaque; one per layer */

typedef enum { KIVI_F16 = 0, KIVI_BF16 = 1 } kivi_dtype;

typedef enum {
    KIVI_OK = 0,
    KIVI_ERR_ARG = 1,         /* bad pointer, size or alignment */
    KIVI_ERR_UNSUPPORTED = 2, /* valid but not built (e.g. D not in {64,128}) */
    KIVI_ERR_CAPACITY = 3,    /* would exceed T_max tokens */
    KIVI_ERR_STATE = 4,       /* prefill twice, decode/append before prefill */
    KIVI_ERR_OOM = 5,         /* device allocation failed / workspace too small */
    KIVI_ERR_CUDA = 6,        /* CUDA runtime or launch error */
    KIVI_ERR_DEVICE = 7       /* a kernel reported a failed bounded wait */
} kivi_status;

/*
 * Cache geometry.  Supported: D in {64, 128}, G == 32, R a positive multiple
 * of G, dtype KIVI_F16 or KIVI_BF16, 1 <= T_max.  T_max bounds the total
 * number of tokens (prefill plus appends).  pre_rope != 0 stores keys before
 * RoPE and rotates them in decode with base rope_theta (e.g. 10000); such a
 * cache supports T_max <= 823000 (the decode's angle reduction is exact for
 * angles below 2^17 * 2pi), larger T_max gives KIVI_ERR_UNSUPPORTED.
 * workspace: optional caller-owned device memory of at least
 * kivi_cache_required_bytes(cfg) bytes, 256-byte aligned, which then holds
 * every device buffer of the cache (the library allocates nothing); it must
 * outlive the cache.
 */
typedef struct {
    int B, H_kv, D, G, R;
    kivi_dtype dtype;
    long long T_max;
    int pre_rope;
    float rope_theta;
    void *workspace;
    size_t workspace_bytes;
} kivi_config;

/* Device bytes of a cache, by purpose (allocated capacity). */
typedef struct {
    size_t codes;    /* 2-bit K and V codes for ceil(T_max/G)*G tokens */
    size_t meta;     /* fp16 scale and zero of every K and V group */
    size_t residual; /* R slots of K and V in the cache dtype */
    size_t scratch;  /* decode partials, tickets, status word, RoPE table */
    size_t total;    /* all of the above, with alignment padding */
} kivi_bytes;

/* Library version of this ABI (bumped on incompatible changes). */
KIVI_API int kivi_abi_version(void);

/* Human-readable name of a status code (static string). */
KIVI_API const char *kivi_status_string(kivi_status s);

/* Create a cache on the current CUDA device; allocates its device memory with
 * cudaMalloc.  pre_rope = 0.  *out receives the handle. */
KIVI_API kivi_status kivi_cache_create(int B, int H_kv, int D, int G, int R, kivi_dtype dtype,
                                       long long T_max, kivi_cache **out);

/* Create from a full configuration (pre-RoPE keys, caller workspace). */
KIVI_API kivi_status kivi_cache_create_ex(const kivi_config *cfg, kivi_cache **out);

/* Device bytes needed for cfg (ignores cfg->workspace). */
KIVI_API kivi_status kivi_cache_required_bytes(const kivi_config *cfg, size_t *bytes);

/* Quantize the first n_q = R*floor((T-1)/R) tokens of K, V into the grouped
 * store and copy the last r = T - n_q tokens into the residual.
 * 1 <= T <= T_max; KIVI_ERR_STATE if already prefilled (see kivi_cache_reset). */
KIVI_API kivi_status kivi_prefill(kivi_cache *c, const void *K, const void *V, long long T,
                         void *stream);

/*
 * Prefill a batch whose elements hold different numbers of tokens (the
 * method's batches are uniform; this serves batches raised to the memory wall
 * with prompts of mixed lengths, KIVI article paragraph 4).  K, V are
 * [B, H_kv, T_pad, D] with batch element b's tokens in rows [0, T_b[b]) of
 * each of its heads; T_b is a HOST array of B lengths, 1 <= T_b[b] <= T_pad
 * <= T_max.  Each element splits as kivi_prefill would for its own length
 * (n_q = R*floor((T_b-1)/R) quantized, r = T_b - n_q residual).  Afterwards
 * kivi_append, kivi_decode_attn, kivi_append_decode and
 * kivi_decode_attn_noalloc keep their signatures and work per element: an
 * element whose residual is full flushes on its next append, the others
 * append in place; decode attends over each element's own tokens.  While the
 * elements' lengths differ, kivi_cache_length returns KIVI_ERR_STATE (use
 * kivi_cache_length_at) and kivi_export needs a range of sequences of one
 * length (e.g. one element's H_kv heads).  B <= 512, else
 * KIVI_ERR_UNSUPPORTED.  KIVI_ERR_STATE if already prefilled. */
KIVI_API kivi_status kivi_prefill_ragged(kivi_cache *c, const void *K, const void *V, long long T_pad,
                                         const long long *T_b, void *stream);

/* Append one token per (batch, kv head).  If the residual holds R tokens they
 * are first quantized as tokens [n_q, n_q+R) (n_q += R, r = 0); the token then
 * goes to residual slot r (r += 1).  KIVI_ERR_CAPACITY past T_max tokens. */
KIVI_API kivi_status kivi_append(kivi_cache *c, const void *k_t, const void *v_t, void *stream);

/* Decode attention of one query per head over all n_q + r tokens.
 * H_q a multiple of H_kv with H_q/H_kv in {1, 2, 4, 8}.  out is fp32. */
KIVI_API kivi_status kivi_decode_attn(kivi_cache *c, const void *q, int H_q, float *out,
                             void *stream);

/* kivi_append then kivi_decode_attn in one launch (the pages have no
 * counterpart; this is the decode step of a model, fused): the decode reads
 * the appended token from k_t/v_t and stores it to the residual itself.  When
 * the residual is full (a flush is due) it runs the two calls.  Arguments,
 * layouts and errors are those of the two calls; on an error before the
 * launch the cache is unchanged. */
KIVI_API kivi_status kivi_append_decode(kivi_cache *c, const void *k_t, const void *v_t,
                               const void *q, int H_q, float *out, void *stream);

/*
 * Decode attention exactly as kivi_decode_attn, for callers that must not
 * allocate device memory (no part of the method corresponds to this call: it
 * only changes where the decode's scratch lives).  Engines that plan all
 * device memory ahead and forbid allocation while serving, plugins that only
 * receive pointers from their host, and paths that cannot afford cudaMalloc's
 * device-wide synchronisation can use it: the split-K partials and
 * per-sequence tickets go into one fixed 8 MiB (8,388,608-byte) array inside
 * the library, which every GPU that loads the library holds until the process
 * exits.  The call itself
 * allocates nothing and calls no allocating routine.
 *   - The first call on a device looks up that array's device address (once
 *     per device, with the device current); make that first call before any
 *     stream capture.  The address is kept until the process exits, so the
 *     library must not outlive a reset of the device (cudaDeviceReset).
 *   - Every call shares the array and it keeps the last call's contents; the
 *     call clears the tickets it needs on `stream` before its kernel.  Calls
 *     whose kernels overlap on the GPU (any caches, any streams) race on the
 *     array: order them, e.g. on one stream.
 *   - Returns KIVI_ERR_CAPACITY, launching nothing, when the call's scratch
 *     (rows = warps + B*H_kv partial rows of (H_q/H_kv)*(D+4) fp32, warps
 *     being the decode's work streams, at most the SM count times 16, plus
 *     B*H_kv + rows int tickets) exceeds the array.
 * Arguments, layouts and other errors as kivi_decode_attn.
 */
KIVI_API kivi_status kivi_decode_attn_noalloc(kivi_cache *c, const void *q, int H_q, float *out,
                                              void *stream);

/* Forget the cached tokens (host counters only; device buffers are kept). */
KIVI_API kivi_status kivi_cache_reset(kivi_cache *c);

/* Current split: n_q quantized tokens, r residual tokens (KIVI_ERR_STATE
 * while the batch elements' lengths differ). */
KIVI_API kivi_status kivi_cache_length(const kivi_cache *c, long long *n_q, int *r);

/* Current split of batch element b (0 <= b < B). */
KIVI_API kivi_status kivi_cache_length_at(const kivi_cache *c, int b, long long *n_q, int *r);

/* Allocated device bytes of the cache, by purpose. */
KIVI_API kivi_status kivi_cache_bytes(const kivi_cache *c, kivi_bytes *out);

/*
 * Copy sequences [seq0, seq0 + nseq) of the cache (sequence = b*H_kv + h) to
 * HOST arrays in the canonical unpacked layout (testing and inspection;
 * synchronises the device).  Arrays are caller-owned host memory:
 *   codesK, codesV [nseq, n_q, D]   uint8 in {0..3}
 *   sK, zK         [nseq, n_q/G, D] fp16 bits
 *   sV, zV         [nseq, n_q, D/G] fp16 bits
 *   resK, resV     [nseq, r, D]     cache dtype
 * Any array pointer may be NULL to skip it.
 */
KIVI_API kivi_status kivi_export(const kivi_cache *c, long long seq0, long long nseq,
                                 uint8_t *codesK, uint8_t *codesV, uint16_t *sK, uint16_t *zK,
                                 uint16_t *sV, uint16_t *zV, void *resK, void *resV);

/* Read (synchronously) and clear the cache's device status word: 0 if every
 * bounded wait in its kernels completed, else the code of the first failure. */
KIVI_API kivi_status kivi_device_status(kivi_cache *c, int *code);

/* Testing the failure path (no part of the method corresponds to this call):
 * with on != 0, every later decode launch on c (kivi_decode_attn,
 * kivi_append_decode, kivi_decode_attn_noalloc) has each warp's first wait
 * for its staged data give up at once.  The warps then record
 * KIVI_DEVICE_WAIT_TIMEOUT in the status word, let the copies they issued
 * land (those waits keep their full bound) and return without writing their
 * results, so `out` is undefined, and a fused append may not have stored its
 * token: as after any device-side failure, reset and prefill the cache again
 * before relying on its contents.  kivi_device_status reports and clears the
 * failure; with on = 0 the next launch runs normally.  Nothing faults or
 * hangs. */
KIVI_API kivi_status kivi_debug_expire_first_wait(kivi_cache *c, int on);

/* Status word value recorded when a bounded wait in a kernel gave up. */
#define KIVI_DEVICE_WAIT_TIMEOUT 1

/* Release the cache (frees its memory unless it lives in a caller workspace). */
KIVI_API kivi_status kivi_cache_destroy(kivi_cache *c);

/*
 * Host-side view of the decode work split, for inspection and tests; needs no
 * GPU.  The flattened work of all B*H_kv sequences (n_groups quantized groups
 * and ceil(r/6) residual items of up to 6 tokens each, weighted wg and wr) is
 * cut into `warps` equal contiguous ranges.  For sequence `seq` it reports
 * out[0] = first warp, out[1] = last warp (inclusive), and for warp `warp`
 * out[2], out[3] = the half-open item range it owns in that sequence
 * (empty if out[2] == out[3]).
 */
KIVI_API kivi_status kivi_decode_split(long long seqs, long long n_groups, int r, int wg, int wr,
                              long long warps, long long seq, long long warp,
                              long long out[4]);

/*
 * Diagnostic quantization under the groupings the KIVI article compares
 * ("KIVI Quantization Secures Llama-2 Accuracy at Two Bits", paragraphs 2-3:
 * keys and values grouped per token or per channel; record
 * kv-efficiency/kivi-2bit-llama2-13b-mha-4k, "Quality": the naive symmetric
 * per-token 2-bit baseline), optionally dense-and-sparse.  It quantizes and dequantizes N independent
 * [T, D] matrices and reports the result and its squared error; it does not
 * touch any cache.
 *
 *   x       DEVICE [N, T, D] in `dtype`, 16-byte aligned, caller-owned.
 *   axis    KIVI_AXIS_PER_CHANNEL: group g of channel d is tokens [gG, gG+G)
 *           of column d (the KIVI key grouping; T % G == 0, any G >= 1);
 *           KIVI_AXIS_PER_TOKEN: group j of token t is channels [jG, jG+G) of
 *           row t (the KIVI value grouping; D % G == 0, G a power of two in
 *           [8, 256], else KIVI_ERR_UNSUPPORTED).
 *   bits    1..8 (asymmetric) or 2..8 (symmetric).
 *   symmetric = 0: zero = fp16(group min), scale = fp16((max - min)/(2^bits - 1))
 *           (subtraction and division rounded in fp32), code = clamp(rint((x -
 *           zero)/scale), 0, 2^bits - 1) with IEEE fp32 division and rint half
 *           to even, x_hat = code*scale + zero rounded once to fp32; at bits = 2
 *           this is the cache's own code.  symmetric != 0 (absmax, no zero):
 *           scale = fp16(max|x| / (2^(bits-1) - 1)), code = clamp(rint(x/scale),
 *           -2^(bits-1), 2^(bits-1) - 1), x_hat = code*scale.  A zero scale
 *           gives code 0.  A stored zero of either sign is +0.
 *   outlier 0, or 1 for dense-and-sparse groups (KVQuant summary, "Per-Vector
 *           Dense-and-Sparse Quantization"): each group's element of largest
 *           |x| (the first on ties) is kept exactly, x_hat = x, and the group's
 *           statistics and codes cover the other G - 1 elements only.
 *   xhat    DEVICE [N, T, D] fp32, 16-byte aligned, or NULL.
 *   sq_err  DEVICE [N] fp64, 8-byte aligned, or NULL: set to the sum over each
 *           matrix of (x - x_hat)^2.  Each difference is rounded to fp32 and
 *           squared and summed in fp32 over runs of at most 8 elements (one
 *           rounding per element, fused); the run sums are added in fp64 in an
 *           unspecified order.  Relative error below 10 * 2^-24.
 * At least one of xhat, sq_err is non-NULL; D is a multiple of 8; T*D <= 2^33
 * (else KIVI_ERR_UNSUPPORTED).  Values whose fp16 scale or zero overflows
 * (|x| near 65504) give non-finite results.  Asynchronous on `stream`; errors
 * as the other calls (KIVI_ERR_ARG for bad pointers, sizes or alignment).
 */
typedef enum { KIVI_AXIS_PER_CHANNEL = 0, KIVI_AXIS_PER_TOKEN = 1 } kivi_axis;

KIVI_API kivi_status kivi_fake_quant(const void *x, kivi_dtype dtype, long long N, long long T,
                                     int D, int axis, int G, int bits, int symmetric,
                                     int outlier, float *xhat, double *sq_err, void *stream);

/*
 * Diagnostic quantization with non-uniform levels per group (KVQuant summary,
 * "Non-Uniform KV Cache Quantization"; the pages give only the name).  Every
 * group (axis and G as in kivi_fake_quant, any G >= 1 dividing T per channel
 * or D per token) keeps its minimum and maximum (fp32) and codes each element
 * by the nearest of nlev normalized levels on [min, max]:
 *   u = (x - min) / (max - min)               IEEE fp64 subtract and divide
 *   code = argmin_k |u - levels[k]|           the first level on ties
 *   x_hat = fp32(min + (max - min) * levels[code])   fp64 multiply, then add
 * A group with max == min decodes to its value with code 0.  It touches no
 * cache.
 *   x       DEVICE [N, T, D] in `dtype`, 16-byte aligned.
 *   levels  HOST array of nlev doubles in [0, 1] (any order), 2 <= nlev <= 256;
 *           copied into the launch.
 *   xhat    DEVICE [N, T, D] fp32, 16-byte aligned, or NULL.
 *   codes   DEVICE [N, T, D] uint8, or NULL.
 *   sq_err  DEVICE [N] fp64, 8-byte aligned, or NULL: sum over each matrix of
 *           (x - x_hat)^2 in fp64 (summation order unspecified).
 * At least one output is non-NULL.  Asynchronous on `stream`; KIVI_ERR_ARG for
 * bad pointers, sizes, levels or alignment.
 */
KIVI_API kivi_status kivi_fake_quant_levels(const void *x, kivi_dtype dtype, long long N, long long T,
                                            int D, int axis, int G, int nlev, const double *levels,
                                            float *xhat, uint8_t *codes, double *sq_err, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* KIVI_H */
