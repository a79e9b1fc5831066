// Internal declarations shared by the libarkv translation units.
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "arkv.h"

namespace arkv {

constexpr int kGP = 4;                 // query-group width the kernels are laid out for
constexpr int kRowThreads = 1024;      // one CTA per row for selection / compaction

// ------------------------------------------------------------------ numerics
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }
__device__ __forceinline__ float bf16_to_f32(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }

// exp((raw - m) / sqrt(D)) for raw, m in units of the unscaled dot product.  The
// argument is formed in float64 and carried as a float pair, so that its rounding
// does not enter the result: exp(a_hi + a_lo) ~ expf(a_hi) * (1 + a_lo).
__device__ __forceinline__ float exp_scaled(float raw, float m, double inv_sqrt_d) {
    const double a = ((double)raw - (double)m) * inv_sqrt_d;
    const float a_hi = (float)a;
    const float a_lo = (float)(a - (double)a_hi);
    const float e = expf(a_hi);
    return fmaf(e, a_lo, e);
}

// Observations a token has after the score update of decode step t (t = -1: after
// prefill): every prefill token at position pos < n0 was seen by the observation
// queries at positions >= pos (at most n_obs of them), and every live token is
// observed once per decode step from the step that appended it.
__device__ __forceinline__ int obs_count_after(int pos, int n0, int t, int n_obs) {
    return pos < n0 ? min(n_obs, n0 - pos) + t + 1 : t - (pos - n0) + 1;
}

// Order-preserving map of a double to uint64 (larger value -> larger key).  A
// score is never NaN, so every key of a real score is nonzero: 0 is free to mark
// a non-candidate.
__device__ __forceinline__ uint64_t double_key(double f) {
    const uint64_t u = (uint64_t)__double_as_longlong(f);
    return (u & 0x8000000000000000ull) ? ~u : (u | 0x8000000000000000ull);
}

// S = mu + gamma * (M2 / n) (ARKV 기술요약 §2.나, population variance), float64,
// each operation rounded on its own (no contraction), as the oracle evaluates it.
__device__ __forceinline__ double score_f64(double mu, double m2, int n, float gamma) {
    return __dadd_rn(mu, __dmul_rn((double)gamma, __ddiv_rn(m2, (double)n)));
}

// Budget counts of one row, float64 with the operations in a fixed order so that
// every implementation doing the same operations obtains the same integers.
__host__ __device__ inline void budget_counts(float beta, int n_t, float r, int D, int W,
                                              int n_cand, int* n_sel, int* n_o) {
    const double b_o = 4.0 * D, b_q = 2.0 * D + 8.0;
#ifdef __CUDA_ARCH__
    const double rb = __dsub_rn(__dmul_rn(__dmul_rn((double)beta, (double)n_t), b_o),
                                __dmul_rn((double)W, b_o));
    const double denom = __dadd_rn(__dmul_rn((double)r, b_o),
                                   __dmul_rn(__dsub_rn(1.0, (double)r), b_q));
    long long ns = rb > 0 ? (long long)floor(__ddiv_rn(rb, denom)) : 0;
#else
    volatile double t1 = (double)beta * (double)n_t;
    volatile double t2 = t1 * b_o;
    volatile double t3 = (double)W * b_o;
    const double rb = t2 - t3;
    volatile double d1 = (double)r * b_o;
    volatile double d2 = (1.0 - (double)r) * b_q;
    const double denom = d1 + d2;
    long long ns = rb > 0 ? (long long)floor(rb / denom) : 0;
#endif
    if (ns > n_cand) ns = n_cand;
    if (ns < 0) ns = 0;
    *n_sel = (int)ns;
#ifdef __CUDA_ARCH__
    *n_o = (int)floor(__dmul_rn((double)r, (double)ns));
#else
    volatile double ro = (double)r * (double)ns;
    *n_o = (int)floor(ro);
#endif
}

// Quantize one token-head vector held by a warp (EPL elements per lane, lane l
// holds elements [l*EPL, (l+1)*EPL)) to FP8 in format FMT (ARKV_FMT_*):
// s = amax / FMAX (1 if amax == 0), codes = RNE_FP8(x / s) with saturation.
// Writes EPL codes per lane and returns s.
template <int EPL, int FMT>
__device__ __forceinline__ float quantize_warp(const float (&x)[EPL], uint8_t* codes_out) {
    constexpr float kFmax = FMT == ARKV_FMT_E5M2 ? 57344.0f : 448.0f;
    constexpr __nv_fp8_interpretation_t kInterp = FMT == ARKV_FMT_E5M2 ? __NV_E5M2 : __NV_E4M3;
    float amax = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) amax = fmaxf(amax, fabsf(x[e]));
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, m));
    const float s = amax == 0.f ? 1.0f : __fdiv_rn(amax, kFmax);
    uint8_t c[EPL];
#pragma unroll
    for (int e = 0; e < EPL; e += 2) {
        float2 y = make_float2(__fdiv_rn(x[e], s), __fdiv_rn(x[e + 1], s));
        __nv_fp8x2_storage_t p = __nv_cvt_float2_to_fp8x2(y, __NV_SATFINITE, kInterp);
        c[e] = (uint8_t)(p & 0xff);
        c[e + 1] = (uint8_t)(p >> 8);
    }
#pragma unroll
    for (int e = 0; e < EPL; ++e) codes_out[e] = c[e];
    return s;
}

// ------------------------------------------------------------------ launch parameters
struct LayerDims {
    int batch, hq, hkv, G, D, W, n_obs;
    float gamma, beta;
    int cap_o, cap_q;
    int R;
    int fmt;   // ARKV_FMT_* of the Quantized tier
};

struct AttnParams {
    CUtensorMap tm_k16, tm_v16;   // [R*cap_bf16][D] bf16, boxes of 16 rows x 128 bytes, 128B swizzle
    CUtensorMap tm_k8, tm_v8;     // [R*cap_fp8][D] FP8 codes, boxes of 16 rows x D bytes
    LayerDims d;
    int step;
    const uint16_t* q;
    const uint16_t* k_new;
    const uint16_t* v_new;
    const int32_t* ctx_len;
    arkv_layer_cache c;
    float* o;
    float* logit16;     // [R][4][lstride_o] raw logits of every head, by slot
    float* logit8;      // [R][4][lstride_q]
    float* part_o;      // [parts][4][D]  one partial per CTA
    float2* part_ml;    // [parts][4]
    float2* ml;         // [R][4]  final (max, sum) per head
    unsigned* counter;  // [R]  the rows' tickets (zero between calls)
    int lstride_o, lstride_q;
    double inv_sqrt_d;
    int early_start;    // read the cache before waiting for the previous kernel
};

struct ScoreParams {
    LayerDims d;
    int step;
    const int32_t* ctx_len;
    arkv_layer_cache c;
    const float* logit16;
    const float* logit8;
    const float2* ml;
    int lstride_o, lstride_q;
    double inv_sqrt_d;
};

// Decode workspace layout (byte offsets), shared by arkv_decode_attn and
// arkv_score_update.
struct DecodeWs {
    size_t logit16, logit8, part_o, part_ml, ml, counter, total;
    int parts;                       // partial slots: the largest grid of one call
    int lstride_o, lstride_q;
};
DecodeWs decode_ws_layout(const LayerDims& d);

cudaError_t launch_decode_attn(AttnParams& p, cudaStream_t s);   // fills the tensor maps
cudaError_t launch_score_update(const ScoreParams& p, cudaStream_t s);
cudaError_t launch_copy16(void* dst, const void* src, size_t bytes, cudaStream_t s);   // bytes % 16 == 0

struct ReassignParams {
    LayerDims d;
    int step;
    float r;
    const int32_t* ctx_len;
    arkv_layer_cache c;
    uint8_t* tier_dbg;
    uint64_t* key_ws;   // [R][cap_o + cap_q] keys (used when they do not fit in shared memory)
    int32_t* idx_ws;    // [R][2][cap_o + cap_q] scratch slot lists
};
size_t reassign_ws_bytes(const LayerDims& d);
cudaError_t launch_reassign(const ReassignParams& p, cudaStream_t s);

struct PackParams {
    LayerDims d;
    float r;
    const uint16_t* k;
    const uint16_t* v;
    int n_stride;
    const int32_t* ctx_len;
    const double* mu0;
    const double* m2_0;
    arkv_layer_cache c;
    uint8_t* tier_out;
    uint64_t* key_ws;   // [R][n_stride]
    int32_t* idx_ws;    // [R][n_stride]
};
cudaError_t launch_quantize_pack(const PackParams& p, cudaStream_t s);

struct PrefillParams {
    LayerDims d;
    const uint16_t* q_obs;
    const uint16_t* k;
    int n_stride;
    const int32_t* ctx_len;
    double* stats_out;
    double* query_stats;    // [B][Hq][n_obs][3]
    double* mu0;
    double* m2_0;
    double* part;           // ws [R][n_obs][4][key ranges][6] partial sums of the sweep
    double* qml;            // ws [R][n_obs][4][2] final (max, sum) per query
};
// Prefill workspace layout (byte offsets), shared by arkv_prefill_stats and
// arkv_quantize_pack (keys, idx).
struct PrefillWs {
    size_t part, qml, qstat, keys, idx, total;
};
PrefillWs prefill_ws_layout(const LayerDims& d, int n_stride);
cudaError_t launch_prefill_stats(const PrefillParams& p, cudaStream_t s);

cudaError_t launch_fp8_encode(int fmt, const float* x, uint8_t* out, size_t n, cudaStream_t s);

// Replace the calling thread's last-error message (see arkv_last_error_string).
void set_last_error(const char* msg);

// Raise a kernel's dynamic shared-memory limit to the device's opt-in maximum,
// once per (kernel, device); later launches (including ones being captured into a
// CUDA graph) then only launch.
template <class K>
cudaError_t allow_max_dyn_smem(K kernel, unsigned char (&done)[64]) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 64 && __atomic_load_n(&done[dev], __ATOMIC_ACQUIRE)) return cudaSuccess;
    int optin = 0;
    e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (e != cudaSuccess) return e;
    cudaFuncAttributes fa;
    e = cudaFuncGetAttributes(&fa, kernel);
    if (e != cudaSuccess) return e;
    // static and dynamic shared memory share the per-block limit
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             optin - (int)fa.sharedSizeBytes);
    if (e == cudaSuccess)   // ask for the largest shared-memory carveout, so that occupancy is not cut by L1
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                                 (int)cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess && dev < 64) __atomic_store_n(&done[dev], 1, __ATOMIC_RELEASE);
    return e;
}

}  // namespace arkv
