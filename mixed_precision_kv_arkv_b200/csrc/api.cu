// extern "C" entry points of libarkv: argument checks, workspace carving and
// kernel launches.  See include/arkv.h for the contract of every call.
#include <math.h>
#include <stdio.h>
#include <string.h>

#include <climits>

#include "arkv_internal.cuh"

namespace {

thread_local char g_err[512] = "";

int fail(int code, const char* fmt, const char* what) {
    snprintf(g_err, sizeof g_err, fmt, what);
    return code;
}

int cuda_fail(cudaError_t e, const char* where) {
    snprintf(g_err, sizeof g_err, "%s: %s", where, cudaGetErrorString(e));
    return ARKV_ECUDA;
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

int check_cfg(const arkv_cfg* c) {
    if (!c) return fail(ARKV_EINVAL, "%s is null", "cfg");
    if (c->batch < 1 || c->hq < 1 || c->hkv < 1 || c->hq % c->hkv != 0)
        return fail(ARKV_EINVAL, "%s: need batch, hq, hkv >= 1 and hq %% hkv == 0", "cfg");
    const int G = c->hq / c->hkv;
    if (G > arkv::kGP) return fail(ARKV_EINVAL, "%s: query group hq/hkv must be 1..4", "cfg");
    if (c->head_dim != 64 && c->head_dim != 128)
        return fail(ARKV_EINVAL, "%s: head_dim must be 64 or 128", "cfg");
    if (c->window < 1 || c->n_obs < 1) return fail(ARKV_EINVAL, "%s: window and n_obs must be >= 1", "cfg");
    if (!(c->gamma >= 0.f) || !isfinite(c->gamma)) return fail(ARKV_EINVAL, "%s: gamma must be finite and >= 0", "cfg");
    if (!(c->budget_frac > 0.f && c->budget_frac <= 1.f))
        return fail(ARKV_EINVAL, "%s: budget_frac must be in (0, 1]", "cfg");
    if (c->cap_bf16 < 1 || c->cap_fp8 < 1) return fail(ARKV_EINVAL, "%s: capacities must be >= 1", "cfg");
    if (c->quant_format != ARKV_FMT_E4M3 && c->quant_format != ARKV_FMT_E5M2)
        return fail(ARKV_EINVAL, "%s: quant_format must be ARKV_FMT_E4M3 or ARKV_FMT_E5M2", "cfg");
    if (c->early_start != 0 && c->early_start != 1) return fail(ARKV_EINVAL, "%s: early_start must be 0 or 1", "cfg");
    return ARKV_OK;
}

arkv::LayerDims dims(const arkv_cfg* c) {
    arkv::LayerDims d{};
    d.batch = c->batch; d.hq = c->hq; d.hkv = c->hkv; d.G = c->hq / c->hkv; d.D = c->head_dim;
    d.W = c->window; d.n_obs = c->n_obs; d.gamma = c->gamma; d.beta = c->budget_frac;
    d.cap_o = c->cap_bf16; d.cap_q = c->cap_fp8; d.R = c->batch * c->hkv;
    d.fmt = c->quant_format;
    return d;
}

int check_cache(const arkv_layer_cache* c) {
    if (!c) return fail(ARKV_EINVAL, "%s is null", "cache");
    const void* ptrs[] = {c->k16, c->v16, c->pos16, c->mu16, c->m2_16, c->k8, c->v8, c->sk, c->sv,
                          c->pos8, c->mu8, c->m2_8, c->n_bf16, c->n_fp8, c->status};
    for (const void* q : ptrs)
        if (!q) return fail(ARKV_EINVAL, "%s has a null buffer", "cache");
    if (!aligned(c->k16, 16) || !aligned(c->v16, 16) || !aligned(c->k8, 16) || !aligned(c->v8, 16))
        return fail(ARKV_EINVAL, "%s: k16, v16, k8, v8 must be 16-byte aligned", "cache");
    const void* words[] = {c->pos16, c->sk, c->sv, c->pos8, c->n_bf16, c->n_fp8, c->status};
    for (const void* q : words)
        if (!aligned(q, 4)) return fail(ARKV_EINVAL, "%s: 4-byte buffers must be 4-byte aligned", "cache");
    const void* dwords[] = {c->mu16, c->m2_16, c->mu8, c->m2_8};
    for (const void* q : dwords)
        if (!aligned(q, 8)) return fail(ARKV_EINVAL, "%s: mu and M2 buffers must be 8-byte aligned", "cache");
    return ARKV_OK;
}

int check_ws(const void* ws, size_t have, size_t need) {
    if (need > 0 && !ws) return fail(ARKV_EINVAL, "%s is null", "workspace");
    if (!aligned(ws, 256)) return fail(ARKV_EINVAL, "%s must be 256-byte aligned", "workspace");
    if (have < need) return fail(ARKV_EINVAL, "%s is smaller than arkv_workspace_bytes()", "workspace");
    return ARKV_OK;
}

#define ARKV_TRY(x)                   \
    do {                              \
        const int _rc = (x);          \
        if (_rc != ARKV_OK) return _rc; \
    } while (0)

}  // namespace

void arkv::set_last_error(const char* msg) { snprintf(g_err, sizeof g_err, "%s", msg); }

extern "C" {

const char* arkv_last_error_string(void) { return g_err; }

size_t arkv_workspace_bytes(const arkv_cfg* cfg, int which, int32_t n_ctx_max) {
    if (check_cfg(cfg) != ARKV_OK) return 0;
    const arkv::LayerDims d = dims(cfg);
    switch (which) {
        case ARKV_WS_DECODE: return arkv::decode_ws_layout(d).total;
        case ARKV_WS_REASSIGN: return arkv::reassign_ws_bytes(d);
        case ARKV_WS_PREFILL: return n_ctx_max > 0 ? arkv::prefill_ws_layout(d, n_ctx_max).total : 0;
        default: return 0;
    }
}

int arkv_row_capacity(const arkv_cfg* cfg, int32_t n_ctx_max, float r, int32_t reassign_interval,
                      int32_t* cap_bf16, int32_t* cap_fp8) {
    if (!cfg || !cap_bf16 || !cap_fp8) return fail(ARKV_EINVAL, "%s: null argument", "arkv_row_capacity");
    if (n_ctx_max < cfg->window || !(r >= 0.f && r <= 1.f) || reassign_interval < 1 || cfg->head_dim <= 0 ||
        !(cfg->budget_frac > 0.f && cfg->budget_frac <= 1.f) || cfg->window < 1)
        return fail(ARKV_EINVAL, "%s: bad argument", "arkv_row_capacity");
    int n_sel, n_o;
    arkv::budget_counts(cfg->budget_frac, n_ctx_max, r, cfg->head_dim, cfg->window, INT_MAX, &n_sel, &n_o);
    *cap_bf16 = n_o + cfg->window + reassign_interval;
    *cap_fp8 = n_sel > 0 ? n_sel : 1;
    return ARKV_OK;
}

int arkv_oq_ratio(const double* stats, int32_t layers, double r_bar, float* r_out) {
    if (!stats || !r_out || layers < 1) return fail(ARKV_EINVAL, "%s: bad argument", "arkv_oq_ratio");
    double mean = 0.0;
    for (int l = 0; l < layers; ++l) {
        const double H = stats[3 * l], v = stats[3 * l + 1], k = fmax(stats[3 * l + 2], 0.0);
        mean += ((1.0 - H) + v / (1.0 + v) + k / (1.0 + k)) / 3.0;
    }
    mean /= layers;
    for (int l = 0; l < layers; ++l) {
        const double H = stats[3 * l], v = stats[3 * l + 1], k = fmax(stats[3 * l + 2], 0.0);
        const double s = ((1.0 - H) + v / (1.0 + v) + k / (1.0 + k)) / 3.0;
        double r = mean > 0 ? r_bar * s / mean : r_bar;
        if (mean > 0) r = fmin(fmax(r, 0.05), 0.95);
        r_out[l] = (float)r;
    }
    return ARKV_OK;
}

int arkv_prefill_stats(const arkv_cfg* cfg, const uint16_t* q_obs, const uint16_t* k, int32_t n_ctx_max,
                       const int32_t* ctx_len, double* stats_out, double* query_stats, double* mu0,
                       double* m2_0, void* ws, size_t ws_bytes, arkv_stream_t stream) {
    ARKV_TRY(check_cfg(cfg));
    if (!q_obs || !k || !ctx_len || !stats_out || !mu0 || !m2_0)
        return fail(ARKV_EINVAL, "%s: null argument", "arkv_prefill_stats");
    if (!aligned(q_obs, 16) || !aligned(k, 16))
        return fail(ARKV_EINVAL, "%s: q_obs and k must be 16-byte aligned", "arkv_prefill_stats");
    if (n_ctx_max < cfg->n_obs) return fail(ARKV_EINVAL, "%s: n_ctx_max < n_obs", "arkv_prefill_stats");
    const arkv::LayerDims d = dims(cfg);
    const arkv::PrefillWs w = arkv::prefill_ws_layout(d, n_ctx_max);
    ARKV_TRY(check_ws(ws, ws_bytes, w.total));
    arkv::PrefillParams p{};
    p.d = d; p.q_obs = q_obs; p.k = k; p.n_stride = n_ctx_max; p.ctx_len = ctx_len;
    p.stats_out = stats_out;
    p.query_stats = query_stats ? query_stats : (double*)((char*)ws + w.qstat);
    p.mu0 = mu0; p.m2_0 = m2_0;
    p.part = (double*)((char*)ws + w.part);
    p.qml = (double*)((char*)ws + w.qml);
    const cudaError_t e = arkv::launch_prefill_stats(p, (cudaStream_t)stream);
    return e == cudaSuccess ? ARKV_OK : cuda_fail(e, "arkv_prefill_stats");
}

int arkv_quantize_pack(const arkv_cfg* cfg, float r, const uint16_t* k, const uint16_t* v, int32_t n_ctx_max,
                       const int32_t* ctx_len, const double* mu0, const double* m2_0, arkv_layer_cache* cache,
                       uint8_t* tier_out, void* ws, size_t ws_bytes, arkv_stream_t stream) {
    ARKV_TRY(check_cfg(cfg));
    ARKV_TRY(check_cache(cache));
    if (!k || !v || !ctx_len || !mu0 || !m2_0) return fail(ARKV_EINVAL, "%s: null argument", "arkv_quantize_pack");
    if (!aligned(k, 16) || !aligned(v, 16)) return fail(ARKV_EINVAL, "%s: k, v must be 16-byte aligned", "arkv_quantize_pack");
    if (!(r >= 0.f && r <= 1.f)) return fail(ARKV_EINVAL, "%s: r must be in [0, 1]", "arkv_quantize_pack");
    if (n_ctx_max < cfg->window) return fail(ARKV_EINVAL, "%s: n_ctx_max < window", "arkv_quantize_pack");
    int n_sel, n_o;
    arkv::budget_counts(cfg->budget_frac, n_ctx_max, r, cfg->head_dim, cfg->window, INT_MAX, &n_sel, &n_o);
    if (cfg->cap_bf16 < n_o + cfg->window || cfg->cap_fp8 < n_sel - n_o)
        return fail(ARKV_ECAPACITY, "%s: capacities below the kept counts at n_ctx_max", "arkv_quantize_pack");
    const arkv::LayerDims d = dims(cfg);
    const arkv::PrefillWs w = arkv::prefill_ws_layout(d, n_ctx_max);
    ARKV_TRY(check_ws(ws, ws_bytes, w.total));
    arkv::PackParams p{};
    p.d = d; p.r = r; p.k = k; p.v = v; p.n_stride = n_ctx_max; p.ctx_len = ctx_len; p.mu0 = mu0; p.m2_0 = m2_0;
    p.c = *cache; p.tier_out = tier_out;
    p.key_ws = (uint64_t*)((char*)ws + w.keys);
    p.idx_ws = (int32_t*)((char*)ws + w.idx);
    const cudaError_t e = arkv::launch_quantize_pack(p, (cudaStream_t)stream);
    return e == cudaSuccess ? ARKV_OK : cuda_fail(e, "arkv_quantize_pack");
}

int arkv_decode_attn(const arkv_cfg* cfg, int32_t step, const uint16_t* q, const uint16_t* k_new,
                     const uint16_t* v_new, const int32_t* ctx_len, arkv_layer_cache* cache, float* o,
                     void* ws, size_t ws_bytes, arkv_stream_t stream) {
    ARKV_TRY(check_cfg(cfg));
    ARKV_TRY(check_cache(cache));
    if (!q || !k_new || !v_new || !ctx_len || !o) return fail(ARKV_EINVAL, "%s: null argument", "arkv_decode_attn");
    if (!aligned(q, 16) || !aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(o, 16))
        return fail(ARKV_EINVAL, "%s: q, k_new, v_new and o must be 16-byte aligned", "arkv_decode_attn");
    if (step < 0) return fail(ARKV_EINVAL, "%s: step < 0", "arkv_decode_attn");
    const arkv::LayerDims d = dims(cfg);
    const arkv::DecodeWs w = arkv::decode_ws_layout(d);
    ARKV_TRY(check_ws(ws, ws_bytes, w.total));
    arkv::AttnParams p{};
    p.d = d; p.step = step; p.q = q; p.k_new = k_new; p.v_new = v_new; p.ctx_len = ctx_len; p.c = *cache; p.o = o;
    char* base = (char*)ws;
    p.logit16 = (float*)(base + w.logit16);
    p.logit8 = (float*)(base + w.logit8);
    p.part_o = (float*)(base + w.part_o);
    p.part_ml = (float2*)(base + w.part_ml);
    p.ml = (float2*)(base + w.ml);
    p.counter = (unsigned*)(base + w.counter);
    p.lstride_o = w.lstride_o;
    p.lstride_q = w.lstride_q;
    p.inv_sqrt_d = 1.0 / sqrt((double)d.D);
    p.early_start = cfg->early_start;
    const cudaError_t e = arkv::launch_decode_attn(p, (cudaStream_t)stream);   // also encodes the tensor maps
    return e == cudaSuccess ? ARKV_OK : cuda_fail(e, "arkv_decode_attn");
}

int arkv_score_update(const arkv_cfg* cfg, int32_t step, const int32_t* ctx_len, arkv_layer_cache* cache,
                      const void* ws, size_t ws_bytes, arkv_stream_t stream) {
    ARKV_TRY(check_cfg(cfg));
    ARKV_TRY(check_cache(cache));
    if (!ctx_len) return fail(ARKV_EINVAL, "%s: null argument", "arkv_score_update");
    if (step < 0) return fail(ARKV_EINVAL, "%s: step < 0", "arkv_score_update");
    const arkv::LayerDims d = dims(cfg);
    const arkv::DecodeWs w = arkv::decode_ws_layout(d);
    ARKV_TRY(check_ws(ws, ws_bytes, w.total));
    arkv::ScoreParams p{};
    p.d = d; p.step = step; p.ctx_len = ctx_len; p.c = *cache;
    const char* base = (const char*)ws;
    p.logit16 = (const float*)(base + w.logit16);
    p.logit8 = (const float*)(base + w.logit8);
    p.ml = (const float2*)(base + w.ml);
    p.lstride_o = w.lstride_o;
    p.lstride_q = w.lstride_q;
    p.inv_sqrt_d = 1.0 / sqrt((double)d.D);
    const cudaError_t e = arkv::launch_score_update(p, (cudaStream_t)stream);
    return e == cudaSuccess ? ARKV_OK : cuda_fail(e, "arkv_score_update");
}

int arkv_reassign(const arkv_cfg* cfg, int32_t step, float r, const int32_t* ctx_len, arkv_layer_cache* cache,
                  uint8_t* tier_dbg, void* ws, size_t ws_bytes, arkv_stream_t stream) {
    ARKV_TRY(check_cfg(cfg));
    ARKV_TRY(check_cache(cache));
    if (!ctx_len) return fail(ARKV_EINVAL, "%s: null argument", "arkv_reassign");
    if (!(r >= 0.f && r <= 1.f)) return fail(ARKV_EINVAL, "%s: r must be in [0, 1]", "arkv_reassign");
    if (step < 0) return fail(ARKV_EINVAL, "%s: step < 0", "arkv_reassign");
    const arkv::LayerDims d = dims(cfg);
    const size_t need = arkv::reassign_ws_bytes(d);
    ARKV_TRY(check_ws(ws, ws_bytes, need));
    arkv::ReassignParams p{};
    p.d = d; p.step = step; p.r = r; p.ctx_len = ctx_len; p.c = *cache; p.tier_dbg = tier_dbg;
    const size_t slots = (size_t)(d.cap_o + d.cap_q);
    const size_t idx_bytes = (slots * 2 * 4 * d.R + 255) & ~(size_t)255;
    p.idx_ws = (int32_t*)ws;
    p.key_ws = (uint64_t*)((char*)ws + idx_bytes);
    const cudaError_t e = arkv::launch_reassign(p, (cudaStream_t)stream);
    return e == cudaSuccess ? ARKV_OK : cuda_fail(e, "arkv_reassign");
}

// True if the device can address ptr: device memory, or page-locked host memory mapped
// into the unified address space (its device pointer is the host pointer).
static bool device_addressable(const void* ptr) {
    cudaPointerAttributes at{};
    if (cudaPointerGetAttributes(&at, ptr) != cudaSuccess) {
        (void)cudaGetLastError();
        return false;
    }
    if (at.type == cudaMemoryTypeDevice || at.type == cudaMemoryTypeManaged) return true;
    return at.type == cudaMemoryTypeHost && at.devicePointer == ptr;
}

int arkv_copy_async(void* dst, const void* src, size_t bytes, arkv_stream_t stream) {
    if (bytes == 0) return ARKV_OK;
    if (!dst || !src) return fail(ARKV_EINVAL, "%s: null argument", "arkv_copy_async");
    if ((bytes & 15) || !aligned(dst, 16) || !aligned(src, 16))
        return fail(ARKV_EINVAL, "%s: bytes and both addresses must be multiples of 16", "arkv_copy_async");
    const uintptr_t d0 = (uintptr_t)dst, s0 = (uintptr_t)src;
    if (d0 < s0 + bytes && s0 < d0 + bytes) return fail(ARKV_EINVAL, "%s: the buffers overlap", "arkv_copy_async");
    if (!device_addressable(dst) || !device_addressable(src))
        return fail(ARKV_EINVAL, "%s: a buffer is not device-addressable (pageable host memory?)", "arkv_copy_async");
    const cudaError_t e = arkv::launch_copy16(dst, src, bytes, (cudaStream_t)stream);
    return e == cudaSuccess ? ARKV_OK : cuda_fail(e, "arkv_copy_async");
}

int arkv_fp8_encode(int32_t format, const float* x, uint8_t* out, size_t n, arkv_stream_t stream) {
    if (format != ARKV_FMT_E4M3 && format != ARKV_FMT_E5M2)
        return fail(ARKV_EINVAL, "%s: unknown format", "arkv_fp8_encode");
    if (n > 0 && (!x || !out)) return fail(ARKV_EINVAL, "%s: null argument", "arkv_fp8_encode");
    const cudaError_t e = arkv::launch_fp8_encode(format, x, out, n, (cudaStream_t)stream);
    return e == cudaSuccess ? ARKV_OK : cuda_fail(e, "arkv_fp8_encode");
}

}  // extern "C"
