/*
 * arkv.h -- C ABI of libarkv, the B200 (sm_100a) decode path of the ARKV
 * tri-state KV cache.
 *
 * Method: "ARKV: Adaptive and Resource-Efficient KV Cache Management under
 * Limited Memory Budget for Long-Context Inference in LLMs" (gist.science),
 * 기술요약 §2 (methodology):
 *   §2.가  per-layer Original:Quantization (OQ) ratio from the prefill attention's
 *          entropy, variance and kurtosis;
 *   §2.나  heavy-hitter score S_k = mu_k + gamma * sigma_k^2 of each token, from
 *          the attention it receives, updated every decode step;
 *   §2.다  every token is Original (bf16), Quantized (FP8 E4M3, per-token-per-head
 *          absmax scale) or Evicted under a byte budget; the W newest tokens are
 *          always Original; quantized tokens are dequantized right before
 *          attention and attended together with the originals.
 *
 * Layout.  A *row* is one (sequence b, kv-head g) pair of one layer,
 * row = b * hkv + g, R = batch * hkv rows per layer.  Each row owns two segments
 * of slots, in no particular order:
 *   bf16 segment  k16, v16 [R][cap_bf16][D] bf16 bits, pos16 [R][cap_bf16] int32,
 *                 mu16, m2_16 [R][cap_bf16] double (Welford mean and M2);
 *   fp8 segment   k8, v8 [R][cap_fp8][D] E4M3 codes, sk, sv [R][cap_fp8] float
 *                 scales, pos8 int32, mu8, m2_8 double [R][cap_fp8];
 *   n_bf16 [R], n_fp8 [R]  live slots of each segment (slots 0 .. n-1).
 * The Welford count of a token is not stored: it is the number of observations
 * so far, a function of its position, its sequence's prefill length ctx_len[b],
 * n_obs and the decode step (see arkv_score_update).
 *
 * Conventions.
 *   - Every pointer is a device pointer the caller owns and allocated, except
 *     where a comment says "host".  The library allocates nothing and keeps no
 *     global state; calls on different streams with different buffers are
 *     independent.
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and returns ARKV_OK or a negative status at once; host-side
 *     argument errors return ARKV_EINVAL before anything is launched.
 *     arkv_last_error_string() describes the last failure of the calling thread.
 *   - Device-side conditions (a segment would exceed its capacity) cannot be
 *     returned synchronously; kernels skip the write that would overflow and OR a
 *     bit into *cache->status (ARKV_STATUS_*), which the caller reads when it
 *     synchronises.
 *   - Workspaces (`ws`, `ws_bytes`) are caller-owned scratch of at least
 *     arkv_workspace_bytes() bytes, 256-byte aligned.  The decode workspace must be
 *     zero-filled once before its first use; the library leaves it reusable.
 *     Calls that share a workspace must be ordered on one stream.
 */
#ifndef ARKV_H
#define ARKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *arkv_stream_t;   /* same type as cudaStream_t */

#define ARKV_OK          0
#define ARKV_EINVAL     (-1)   /* null pointer, bad shape or size, workspace too small */
#define ARKV_ECAPACITY  (-2)   /* a capacity that the host can check is too small */
#define ARKV_ECUDA      (-3)   /* a CUDA launch or memset failed */

#define ARKV_STATUS_BF16_FULL  1   /* an append found the bf16 segment full; token dropped */
#define ARKV_STATUS_FP8_FULL   2   /* a reassignment found the fp8 segment full; demotion became eviction */
#define ARKV_STATUS_TIMEOUT    4   /* a kernel gave up waiting for its own bulk copy (a bug, never expected) */

#define ARKV_TIER_ORIGINAL   0
#define ARKV_TIER_QUANTIZED  1
#define ARKV_TIER_EVICTED    2

/* FP8 formats of the Quantized tier (§2.다 "low precision, e.g. FP8"; OCP FP8):
 * codes = RNE(x / s) with saturation, s = amax / FMAX per token and head. */
#define ARKV_FMT_E4M3  0   /* 4 exponent bits, 3 mantissa bits, FMAX = 448 (default) */
#define ARKV_FMT_E5M2  1   /* 5 exponent bits, 2 mantissa bits, FMAX = 57344 */

/* Shapes and policy of one layer.  hq % hkv == 0, hq / hkv (the query group
 * G) in 1..4, head_dim 64 or 128, window >= 1, 1 <= n_obs, budget_frac in
 * (0, 1], gamma >= 0, quant_format ARKV_FMT_E4M3 or ARKV_FMT_E5M2. */
typedef struct arkv_cfg {
    int32_t batch;
    int32_t hq;             /* query heads */
    int32_t hkv;            /* key/value heads */
    int32_t head_dim;       /* D */
    int32_t window;         /* W: newest tokens always kept bf16 (§2.다 protected window) */
    int32_t n_obs;          /* prefill observation queries per sequence (last n_obs positions) */
    float   gamma;          /* weight of sigma^2 in S (§2.나) */
    float   budget_frac;    /* beta: bytes kept per row <= beta * N_t * 4D (§2.다 memory budget) */
    int32_t cap_bf16;       /* slots per row, bf16 segment */
    int32_t cap_fp8;        /* slots per row, fp8 segment */
    int32_t quant_format;   /* ARKV_FMT_*: FP8 format of the Quantized tier */
    int32_t early_start;    /* 0 or 1, arkv_decode_attn only: see there */
} arkv_cfg;

/* Device buffers of one layer's packed cache (see Layout above). */
typedef struct arkv_layer_cache {
    uint16_t *k16, *v16;
    int32_t  *pos16;
    double   *mu16, *m2_16;
    uint8_t  *k8, *v8;
    float    *sk, *sv;
    int32_t  *pos8;
    double   *mu8, *m2_8;
    int32_t  *n_bf16, *n_fp8;
    int32_t  *status;       /* one int32, sticky ARKV_STATUS_* bits */
} arkv_layer_cache;

/* Workspace kinds for arkv_workspace_bytes. */
#define ARKV_WS_DECODE    0   /* arkv_decode_attn + arkv_score_update (shared, persists between them) */
#define ARKV_WS_REASSIGN  1   /* arkv_reassign */
#define ARKV_WS_PREFILL   2   /* arkv_prefill_stats and arkv_quantize_pack */

/* Bytes of workspace a call needs.  n_ctx_max: the padded prefill length (the
 * stride of the prefill K/V arrays), used by ARKV_WS_PREFILL only. */
size_t arkv_workspace_bytes(const arkv_cfg *cfg, int which, int32_t n_ctx_max);

/* Row capacities that hold every state a row can reach while its context grows
 * to n_ctx_max tokens with an Original share r and reassignments at least every
 * reassign_interval steps: cap_fp8 = the largest kept count, cap_bf16 = the
 * largest Original count + W + reassign_interval.  Host only.  Returns ARKV_EINVAL
 * on bad arguments. */
int arkv_row_capacity(const arkv_cfg *cfg, int32_t n_ctx_max, float r,
                      int32_t reassign_interval, int32_t *cap_bf16, int32_t *cap_fp8);

/* §2.가: prefill attention statistics of one layer and the initial scores.
 * For every sequence b, query head h and observation i (position
 * P = ctx_len[b] - n_obs + i), p = softmax over keys 0..P of q.k/sqrt(D), and
 *   H = -sum p ln p / ln(P+1),  v = (P+1) sum p^2 - 1,
 *   kappa = m4 / m2^2 - 3, m_j = mean over the P+1 keys of (p - 1/(P+1))^j.
 * stats_out (device, 3 doubles) receives the means of (H, v, kappa) over all
 * (b, h, i); query_stats (device, nullable) receives them per query,
 * [batch][hq][n_obs][3] doubles.  Every key k < ctx_len[b] of row (b, g) gets the
 * Welford state of its observations x_k(i) = sum over the group's G heads of
 * p, i = 0..n_obs-1 with P_i >= k: mu0, m2_0 [R][n_ctx_max] doubles.
 *   q_obs  [batch][hq][n_obs][D] bf16 bits (queries at the last n_obs positions)
 *   k      [batch][hkv][n_ctx_max][D] bf16 bits (keys 0 .. ctx_len[b]-1 used)
 *   ctx_len [batch] int32, n_obs <= ctx_len[b] <= n_ctx_max
 * Computed with float64 dot products and sums. */
int arkv_prefill_stats(const arkv_cfg *cfg, const uint16_t *q_obs, const uint16_t *k,
                       int32_t n_ctx_max, const int32_t *ctx_len, double *stats_out,
                       double *query_stats, double *mu0, double *m2_0, void *ws, size_t ws_bytes,
                       arkv_stream_t stream);

/* §2.가 / reading R-9: per-layer Original share from the layer statistics.
 * Host only, pure.  stats [layers][3] host doubles (H, v, kappa means);
 *   s_l = ((1 - H_l) + v_l/(1+v_l) + k_l/(1+k_l)) / 3,  k_l = max(kappa_l, 0),
 *   r_l = clip(r_bar * s_l / mean_l s_l, 0.05, 0.95)  (r_bar if the mean is 0).
 * r_out [layers] host floats. */
int arkv_oq_ratio(const double *stats, int32_t layers, double r_bar, float *r_out);

/* §2.다: the reassignment right after prefill, and the initial pack.
 * Ranks the tokens of every row that are older than the window by
 * S = mu0 + gamma * m2_0 / n (n = min(n_obs, ctx_len[b] - pos), float64, ties by
 * position), keeps the budget's
 * n_sel, makes the first n_o of them Original and quantizes the rest, evicts the
 * others, and writes the cache: bf16 segment = Originals + the W newest tokens,
 * fp8 segment = the Quantized tokens (codes = RNE_FP8(x / s), s = amax / FMAX in
 * float32, s = 1 if amax = 0, in cfg's quant_format), both in position order.  Counts follow
 *   Rb = beta*N*4D - W*4D, n_sel = min(floor(Rb / (r*4D + (1-r)*(2D+8))), candidates),
 *   n_o = floor(r * n_sel)            (float64, operations in this order).
 *   k, v [batch][hkv][n_ctx_max][D] bf16 bits; mu0, m2_0 from arkv_prefill_stats;
 *   tier_out [R][n_ctx_max] uint8 ARKV_TIER_* per position (device, nullable).
 * Returns ARKV_ECAPACITY when cfg's capacities cannot hold the kept counts. */
int arkv_quantize_pack(const arkv_cfg *cfg, float r, const uint16_t *k, const uint16_t *v,
                       int32_t n_ctx_max, const int32_t *ctx_len, const double *mu0,
                       const double *m2_0, arkv_layer_cache *cache, uint8_t *tier_out,
                       void *ws, size_t ws_bytes, arkv_stream_t stream);

/* §2.다 reconstruction: decode step `step` (0-based) of one layer.
 * Appends (k_new, v_new) of every row as an Original token at position
 * ctx_len[b] + step, then for every query head h of group g
 *   o_h = sum_k p_hk v^_k,  p_hk = softmax_k(q_h . k^_k / sqrt(D))
 * over the row's live tokens, with k^ = k for bf16 slots and k^ = code * scale for
 * fp8 slots (v^ likewise).  o is written in float32.  Each token's raw logits and
 * each head's softmax max and sum are left in `ws` for arkv_score_update.
 *   q [batch][hq][D], k_new, v_new [batch][hkv][D] bf16 bits; o [batch][hq][D] float;
 *   all four 16-byte aligned.
 * The row's bf16 count (n_bf16) is advanced past the new token when the call
 * completes.  A full bf16 segment sets ARKV_STATUS_BF16_FULL and drops the new
 * token.
 * The kernel is launched as a programmatic dependent of the kernel before it on
 * the stream, and lets the kernel after it launch the same way: its blocks may be
 * resident before the previous kernel has finished.  With cfg->early_start = 0
 * they read nothing before it has finished and its writes are visible.  With
 * cfg->early_start = 1 they first read this layer's cache (codes, scales, counts
 * n_bf16 and n_fp8) and ctx_len, and wait only before q, k_new, v_new, o, ws and
 * every write: set it only when neither of the two kernels that precede the call
 * on the stream writes those buffers (for example, consecutive calls on other
 * layers' caches). */
int arkv_decode_attn(const arkv_cfg *cfg, int32_t step, const uint16_t *q, const uint16_t *k_new,
                     const uint16_t *v_new, const int32_t *ctx_len, arkv_layer_cache *cache,
                     float *o, void *ws, size_t ws_bytes, arkv_stream_t stream);

/* §2.나: the score observation and running mean/variance of decode step `step`.
 * For every live token k of every row, x_k = sum over the group's heads of p_hk
 * (from the logits arkv_decode_attn of the same step left in ws), then one
 * Welford step n += 1; d = x - mu; mu += d / n; M2 += d (x - mu), where n counts
 * the token's observations: min(n_obs, ctx_len[b] - pos) + step for prefill
 * tokens, step - (pos - ctx_len[b]) for decode tokens, before this step.
 * S_k = mu_k + gamma * M2_k / n (population variance) is what arkv_reassign ranks.
 * Arithmetic and state in float64. */
int arkv_score_update(const arkv_cfg *cfg, int32_t step, const int32_t *ctx_len,
                      arkv_layer_cache *cache, const void *ws, size_t ws_bytes,
                      arkv_stream_t stream);

/* §2.다: tier reassignment after decode step `step` (context N_t = ctx_len[b] +
 * step + 1).  The W newest positions stay Original.  The other live tokens are
 * ranked by (S descending, position ascending), S = mu + gamma * M2 / n evaluated in
 * float64 and ranked on its 64-bit pattern; the first n_sel (budget counts as
 * in arkv_quantize_pack, with N_t) are kept; walking them in rank order, the first
 * n_o still in bf16 stay Original, the other kept bf16 tokens are quantized into
 * the fp8 segment, kept fp8 tokens keep their codes; all others are evicted.
 * Segments are compacted in place by moving tokens into vacated slots.
 *   tier_dbg [R][cap_bf16 + cap_fp8] uint8 (device, nullable): the new tier of
 *   every slot as it was before the call (bf16 slots first, then fp8 slots).  When
 *   the fp8 segment cannot take every demotion (ARKV_STATUS_FP8_FULL), the
 *   demotions that did not fit are evicted and reported as ARKV_TIER_EVICTED. */
int arkv_reassign(const arkv_cfg *cfg, int32_t step, float r, const int32_t *ctx_len,
                  arkv_layer_cache *cache, uint8_t *tier_dbg, void *ws, size_t ws_bytes,
                  arkv_stream_t stream);

/* The device float32 -> FP8 conversion the quantizer uses (round to nearest
 * even, saturate to +-FMAX) in `format` (ARKV_FMT_*), for testing:
 * out[i] = code(x[i]), n elements. */
int arkv_fp8_encode(int32_t format, const float *x, uint8_t *out, size_t n, arkv_stream_t stream);

/* Host <-> device transfer for the decode loop's inputs and outputs, done by a
 * device kernel instead of the copy engine: copies `bytes` from src to dst, either of
 * which may be device memory or page-locked host memory (cudaHostAlloc /
 * cudaHostRegister; the device reads and writes it over the bus under unified
 * addressing).  Captured into a CUDA graph it is a kernel node, which keeps
 * programmatic dependent launches and the graph's concurrent branches intact around
 * it, where a copy-engine node between kernels costs a synchronisation.
 * bytes a multiple of 16 and both addresses 16-byte aligned, else ARKV_EINVAL.
 * Pointers the device cannot address (pageable host memory) are rejected with
 * ARKV_EINVAL before any launch (cudaPointerGetAttributes); make the first call on
 * a buffer outside any stream capture.  The buffers must not overlap. */
int arkv_copy_async(void *dst, const void *src, size_t bytes, arkv_stream_t stream);

/* Allocation-free tier reassignment.  The paper has no counterpart: this is an
 * interface for callers that cannot allocate device memory when they reassign --
 * code running while a CUDA graph is captured (cudaMalloc is not a stream
 * operation a capture can record), serving engines that reserve all device
 * memory at start-up and forbid later allocations, plugins whose host framework
 * owns the allocator.  It computes exactly what arkv_reassign computes, with the
 * same arguments except the workspace: its scratch is a static device array of
 * ARKV_NOALLOC_SCRATCH_BYTES that every GPU loading this library holds until the
 * process exits.  The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call before
 * any stream capture.  The address is remembered together with the CUDA context
 * it belongs to: after the context is destroyed and recreated (cudaDeviceReset),
 * the next call looks it up again, so make that call outside a capture too.  All
 * calls share the array and it keeps the last call's
 * contents (nothing in it needs to start at zero); calls whose executions overlap
 * on the GPU race on it, so the caller must order them.  A layer whose scratch
 * (arkv_workspace_bytes(cfg, ARKV_WS_REASSIGN, 0)) exceeds the array is rejected
 * with ARKV_EINVAL and a message; it calls no allocating routine. */
#define ARKV_NOALLOC_SCRATCH_BYTES (24u << 20)
int arkv_reassign_noalloc(const arkv_cfg *cfg, int32_t step, float r, const int32_t *ctx_len,
                          arkv_layer_cache *cache, uint8_t *tier_dbg, arkv_stream_t stream);

/* Message of the calling thread's last failure ("" if none). */
const char *arkv_last_error_string(void);

#ifdef __cplusplus
}
#endif

#endif /* ARKV_H */
