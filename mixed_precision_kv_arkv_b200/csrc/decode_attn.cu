// Decode attention over the tri-state cache (ARKV, 기술요약 §2.다: quantized tokens
// are dequantized right before attention and attended together with the
// originals) and the score observation that feeds §2.나.
//
// One CTA handles one split of one row: kSplitBf16 consecutive bf16 slots or
// kSplitFp8 consecutive fp8 slots.  Its 4 warps take 16-token tiles in turn.
// Inside a warp, a token's D elements are spread over LP = D/8 lanes (8 elements,
// one 16-byte bf16 load or one 8-byte fp8 load each), so a tile is 16 tokens
// with every K/V byte loaded exactly once, in full 32-byte sectors, and the query
// group's G <= 4 heads share it.  The per-lane partial dot products (8 tokens x 4
// heads) are reduced across the LP lanes by a transposing butterfly: each lane
// visits its tokens in an order permuted by its lane bits, so every shuffle step
// keeps half of the values and adds the partner's other half with no selects.
// After log2(LP) steps each lane owns two finished logits (one token, two heads).
// Those feed the online softmax; probabilities go through shared memory to the
// lanes that hold the token's V slices.  FP8 codes are converted in registers and
// their per-token scales are applied to the finished dot product (K) and folded
// into the probability (V).  The last CTA of a row to finish merges the split
// partials and writes o.
#include <math.h>

#include "arkv_internal.cuh"

namespace arkv {

namespace {

constexpr float kNegInf = -INFINITY;
constexpr unsigned kFull = 0xffffffffu;

template <int D>
struct Geo {
    static constexpr int LP = D / 8;   // lanes per token
    static constexpr int NS = LP / 2;  // tokens per lane per tile
    static constexpr int TG = 32 / LP; // token groups per warp
    static_assert(TG * NS == 16, "tile must be 16 tokens");
};

__device__ __forceinline__ uint4 ld_stream16(const void* ptr) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(ptr));
    return r;
}

__device__ __forceinline__ uint2 ld_stream8(const void* ptr) {
    uint2 r;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0,%1}, [%2];"
                 : "=r"(r.x), "=r"(r.y)
                 : "l"(ptr));
    return r;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 u, float (&f)[8]) {
    f[0] = bf16_lo(u.x); f[1] = bf16_hi(u.x);
    f[2] = bf16_lo(u.y); f[3] = bf16_hi(u.y);
    f[4] = bf16_lo(u.z); f[5] = bf16_hi(u.z);
    f[6] = bf16_lo(u.w); f[7] = bf16_hi(u.w);
}

__device__ __forceinline__ float2 e4m3x2_to_f32(uint32_t pair) {
    __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(pair & 0xffffu), __NV_E4M3);
    return __half22float2(*reinterpret_cast<__half2*>(&h));
}

__device__ __forceinline__ void e4m3x8_to_f32(const uint2 u, float (&f)[8]) {
    float2 a = e4m3x2_to_f32(u.x), b = e4m3x2_to_f32(u.x >> 16);
    float2 c = e4m3x2_to_f32(u.y), d = e4m3x2_to_f32(u.y >> 16);
    f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
    f[4] = c.x; f[5] = c.y; f[6] = d.x; f[7] = d.y;
}

template <bool FP8>
struct Raw { using T = uint4; };
template <>
struct Raw<true> { using T = uint2; };

// Streams the tiles of one segment range [seg_begin, seg_end) of a row.
template <int D, bool FP8>
__device__ __forceinline__ void attend_segment(
    const AttnParams& p, int row, int seg_begin, int seg_end, int new_slot,
    const void* kbase, const void* vbase, const uint16_t* knew, const uint16_t* vnew,
    const float* skbase, const float* svbase, float* logit_row, int cap,
    const float (&qf)[4][8], float (&m_run)[4], float (&l_run)[2], float (&oacc)[4][8],
    float (*sm_p)[4]) {
    using Gm = Geo<D>;
    constexpr int LP = Gm::LP, NS = Gm::NS;
    using RawT = typename Raw<FP8>::T;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int tg = lane / LP, ds = lane % LP, perm = ds >> 1, hp = ds & 1;
    const int G = p.d.G;
    const double inv = p.inv_sqrt_d;
    constexpr int EB = FP8 ? 1 : 2;   // element bytes

    for (int t0 = seg_begin + warp * 16; t0 < seg_end; t0 += 64) {
        RawT kr[NS], vr[NS];
        bool valid[NS];
#pragma unroll
        for (int s = 0; s < NS; ++s) {
            const int tok = t0 + tg * NS + (s ^ perm);
            valid[s] = tok < seg_end;
            const size_t slot = (size_t)min(tok, cap - 1);
            const char* ks = (const char*)kbase + slot * D * EB;
            const char* vs = (const char*)vbase + slot * D * EB;
            if (!FP8 && tok == new_slot) {
                ks = (const char*)knew;
                vs = (const char*)vnew;
            }
            if constexpr (FP8) {
                kr[s] = ld_stream8(ks + ds * 8 * EB);
                vr[s] = ld_stream8(vs + ds * 8 * EB);
            } else {
                kr[s] = ld_stream16(ks + ds * 8 * EB);
                vr[s] = ld_stream16(vs + ds * 8 * EB);
            }
        }
        // owner token of this lane after the butterfly, and its fp8 scales
        const int otok = t0 + tg * NS + perm;
        const bool ovalid = otok < seg_end;
        float sk_o = 1.f, sv_o = 1.f;
        if constexpr (FP8) {
            const int os = min(otok, cap - 1);
            sk_o = __ldg(skbase + os);
            sv_o = __ldg(svbase + os);
        }

        // partial dot products: 8 elements x 4 head positions per token slot
        float acc[NS][4];
#pragma unroll
        for (int s = 0; s < NS; ++s) {
            float kf[8];
            if constexpr (FP8) e4m3x8_to_f32(kr[s], kf);
            else bf16x8_to_f32(kr[s], kf);
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                float a = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) a = fmaf(qf[h][e], kf[e], a);
                acc[s][h] = a;
            }
        }
        // transposing butterfly over the LP lanes of a token group
#pragma unroll
        for (int half = NS / 2, m = LP / 2; half >= 1; half >>= 1, m >>= 1) {
#pragma unroll
            for (int s = 0; s < half; ++s)
#pragma unroll
                for (int h = 0; h < 4; ++h)
                    acc[s][h] += __shfl_xor_sync(kFull, acc[s + half][h], m);
        }
        float r0 = acc[0][0] + __shfl_xor_sync(kFull, acc[0][2], 1);
        float r1 = acc[0][1] + __shfl_xor_sync(kFull, acc[0][3], 1);
        if constexpr (FP8) {
            r0 *= sk_o;
            r1 *= sk_o;
        }
        const int h0 = 2 * hp, h1 = 2 * hp + 1;
        if (ovalid) {
            *reinterpret_cast<float2*>(logit_row + (size_t)otok * 4 + h0) = make_float2(r0, r1);
        }
        const bool v0ok = ovalid && h0 < G, v1ok = ovalid && h1 < G;
        const float x0 = v0ok ? r0 : kNegInf, x1 = v1ok ? r1 : kNegInf;

        // tile max of every head (warp-uniform)
        float t0m = x0, t1m = x1;
#pragma unroll
        for (int m = 2; m < 32; m <<= 1) {
            t0m = fmaxf(t0m, __shfl_xor_sync(kFull, t0m, m));
            t1m = fmaxf(t1m, __shfl_xor_sync(kFull, t1m, m));
        }
        const float u0m = __shfl_xor_sync(kFull, t0m, 1), u1m = __shfl_xor_sync(kFull, t1m, 1);
        float tmax[4];
        tmax[0] = hp ? u0m : t0m;
        tmax[1] = hp ? u1m : t1m;
        tmax[2] = hp ? t0m : u0m;
        tmax[3] = hp ? t1m : u1m;
        bool changed = false;
        float alpha[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const float mn = fmaxf(m_run[h], tmax[h]);
            alpha[h] = 1.f;
            if (mn != m_run[h]) {
                changed = true;
                alpha[h] = (m_run[h] == kNegInf) ? 0.f : exp_scaled(m_run[h], mn, inv);
                m_run[h] = mn;
            }
        }
        if (changed) {
#pragma unroll
            for (int h = 0; h < 4; ++h)
#pragma unroll
                for (int e = 0; e < 8; ++e) oacc[h][e] *= alpha[h];
            l_run[0] *= hp ? alpha[2] : alpha[0];
            l_run[1] *= hp ? alpha[3] : alpha[1];
        }
        const float mh0 = hp ? m_run[2] : m_run[0];
        const float mh1 = hp ? m_run[3] : m_run[1];
        float p0 = v0ok ? exp_scaled(r0, mh0, inv) : 0.f;
        float p1 = v1ok ? exp_scaled(r1, mh1, inv) : 0.f;
        l_run[0] += p0;
        l_run[1] += p1;
        if constexpr (FP8) {
            p0 = v0ok ? p0 * sv_o : 0.f;
            p1 = v1ok ? p1 * sv_o : 0.f;
        }
        *reinterpret_cast<float2*>(&sm_p[tg * NS + perm][h0]) = make_float2(p0, p1);
        __syncwarp();
#pragma unroll
        for (int s = 0; s < NS; ++s) {
            const float4 pp = *reinterpret_cast<const float4*>(&sm_p[tg * NS + (s ^ perm)][0]);
            float vf[8];
            if constexpr (FP8) e4m3x8_to_f32(vr[s], vf);
            else bf16x8_to_f32(vr[s], vf);
            if (!valid[s]) {
#pragma unroll
                for (int e = 0; e < 8; ++e) vf[e] = 0.f;
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                oacc[0][e] = fmaf(pp.x, vf[e], oacc[0][e]);
                oacc[1][e] = fmaf(pp.y, vf[e], oacc[1][e]);
                oacc[2][e] = fmaf(pp.z, vf[e], oacc[2][e]);
                oacc[3][e] = fmaf(pp.w, vf[e], oacc[3][e]);
            }
        }
        __syncwarp();
    }
}

template <int D>
__global__ void __launch_bounds__(kAttnThreads) decode_attn_kernel(const AttnParams p) {
    using Gm = Geo<D>;
    constexpr int LP = Gm::LP;
    const LayerDims& d = p.d;
    const int row = blockIdx.y, b = row / d.hkv, g = row - b * d.hkv;
    const int split = blockIdx.x;
    const int nsplit = p.nsplit_o + p.nsplit_q;
    const bool fp8 = split >= p.nsplit_o;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int tg = lane / LP, ds = lane % LP, hp = ds & 1;
    const int G = d.G;

    __shared__ __align__(16) float sm_p[4][16][4];
    __shared__ __align__(16) float sm_o[4][4][D];
    __shared__ float sm_m[4][4], sm_l[4][4];
    __shared__ float2 sm_ml[4];
    __shared__ int sm_last;
    extern __shared__ float sm_w[];   // [nsplit][4] merge weights (last CTA)

    const int n0 = p.ctx_len[b];
    const int n16_old = min(max(p.c.n_bf16[row], 0), d.cap_o);   // counts are clamped to the
    const bool append = n16_old < d.cap_o;                          // capacities before any use
    const int n_live16 = n16_old + (append ? 1 : 0);
    const int n8 = min(max(p.c.n_fp8[row], 0), d.cap_q);
    const uint16_t* knew = p.k_new + ((size_t)b * d.hkv + g) * D;
    const uint16_t* vnew = p.v_new + ((size_t)b * d.hkv + g) * D;

    // append: the CTA whose split covers the new slot stores the token
    if (!fp8 && append && split == n16_old / kSplitBf16) {
        const size_t sl = (size_t)row * d.cap_o + n16_old;
        for (int e = tid; e < D; e += blockDim.x) {
            p.c.k16[sl * D + e] = knew[e];
            p.c.v16[sl * D + e] = vnew[e];
        }
        if (tid == 0) {
            p.c.pos16[sl] = n0 + p.step;
            p.c.mu16[sl] = 0.f;
            p.c.m2_16[sl] = 0.f;
        }
    }
    if (!append && split == 0 && tid == 0) atomicOr(p.c.status, ARKV_STATUS_BF16_FULL);

    // query registers: head position hpos holds head hpos ^ (2 * hp)
    float qf[4][8];
#pragma unroll
    for (int hpos = 0; hpos < 4; ++hpos) {
        const int h = hpos ^ (2 * hp);
        if (h < G) {
            const uint4 u = *reinterpret_cast<const uint4*>(
                p.q + (((size_t)b * d.hq + g * G + h) * D + ds * 8));
            bf16x8_to_f32(u, qf[hpos]);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) qf[hpos][e] = 0.f;
        }
    }

    float m_run[4] = {kNegInf, kNegInf, kNegInf, kNegInf};
    float l_run[2] = {0.f, 0.f};
    float oacc[4][8];
#pragma unroll
    for (int h = 0; h < 4; ++h)
#pragma unroll
        for (int e = 0; e < 8; ++e) oacc[h][e] = 0.f;

    if (!fp8) {
        const int s0 = split * kSplitBf16, s1 = min(s0 + kSplitBf16, n_live16);
        attend_segment<D, false>(p, row, s0, s1, append ? n16_old : -1,
                                 p.c.k16 + (size_t)row * d.cap_o * D,
                                 p.c.v16 + (size_t)row * d.cap_o * D, knew, vnew, nullptr, nullptr,
                                 p.logit16 + (size_t)row * d.cap_o * 4, d.cap_o, qf, m_run, l_run,
                                 oacc, sm_p[warp]);
    } else {
        const int s0 = (split - p.nsplit_o) * kSplitFp8, s1 = min(s0 + kSplitFp8, n8);
        attend_segment<D, true>(p, row, s0, s1, -1, p.c.k8 + (size_t)row * d.cap_q * D,
                                p.c.v8 + (size_t)row * d.cap_q * D, nullptr, nullptr,
                                p.c.sk + (size_t)row * d.cap_q, p.c.sv + (size_t)row * d.cap_q,
                                p.logit8 + (size_t)row * d.cap_q * 4, d.cap_q, qf, m_run, l_run,
                                oacc, sm_p[warp]);
    }

    // warp totals: o over token groups, l over the lanes owning a head pair
#pragma unroll
    for (int m = LP; m < 32; m <<= 1)
#pragma unroll
        for (int h = 0; h < 4; ++h)
#pragma unroll
            for (int e = 0; e < 8; ++e) oacc[h][e] += __shfl_xor_sync(kFull, oacc[h][e], m);
#pragma unroll
    for (int m = 2; m < 32; m <<= 1) {
        l_run[0] += __shfl_xor_sync(kFull, l_run[0], m);
        l_run[1] += __shfl_xor_sync(kFull, l_run[1], m);
    }
    if (tg == 0) {
#pragma unroll
        for (int h = 0; h < 4; ++h)
#pragma unroll
            for (int e = 0; e < 8; ++e) sm_o[warp][h][ds * 8 + e] = oacc[h][e];
    }
    if (lane < 2) {
        sm_l[warp][2 * lane] = l_run[0];
        sm_l[warp][2 * lane + 1] = l_run[1];
    }
    if (lane == 0) {
#pragma unroll
        for (int h = 0; h < 4; ++h) sm_m[warp][h] = m_run[h];
    }
    (void)hp;
    __syncthreads();

    // CTA partial (unnormalised o, running max, sum) of this split
    const double inv = p.inv_sqrt_d;
    const size_t pbase = (size_t)row * nsplit + split;
    for (int idx = tid; idx < 4 * D; idx += blockDim.x) {
        const int h = idx / D, dd = idx - h * D;
        float M = kNegInf;
#pragma unroll
        for (int w = 0; w < 4; ++w) M = fmaxf(M, sm_m[w][h]);
        float O = 0.f, L = 0.f;
        if (M != kNegInf) {
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                if (sm_m[w][h] == kNegInf) continue;
                const float wt = exp_scaled(sm_m[w][h], M, inv);
                O = fmaf(sm_o[w][h][dd], wt, O);
                L = fmaf(sm_l[w][h], wt, L);
            }
        }
        p.part_o[(pbase * 4 + h) * D + dd] = O;
        if (dd == 0) p.part_ml[pbase * 4 + h] = make_float2(M, L);
    }

    // the last CTA of the row merges the splits
    __threadfence();
    __syncthreads();
    if (tid == 0) sm_last = (atomicAdd(&p.counter[row], 1u) == (unsigned)(nsplit - 1));
    __syncthreads();
    if (!sm_last) return;
    __threadfence();

    if (tid < 4) {
        const int h = tid;
        float M = kNegInf;
        for (int s = 0; s < nsplit; ++s)
            M = fmaxf(M, __ldcg(&p.part_ml[((size_t)row * nsplit + s) * 4 + h]).x);
        float L = 0.f;
        for (int s = 0; s < nsplit; ++s) {
            const float2 ml = __ldcg(&p.part_ml[((size_t)row * nsplit + s) * 4 + h]);
            const float wt = (ml.y > 0.f && M != kNegInf) ? exp_scaled(ml.x, M, inv) : 0.f;
            sm_w[s * 4 + h] = wt;
            L = fmaf(ml.y, wt, L);
        }
        sm_ml[h] = make_float2(M, L);
        p.ml[(size_t)row * 4 + h] = make_float2(M, L);
    }
    __syncthreads();
    for (int idx = tid; idx < G * D; idx += blockDim.x) {
        const int h = idx / D, dd = idx - h * D;
        float acc = 0.f;
        for (int s = 0; s < nsplit; ++s) {
            const float wt = sm_w[s * 4 + h];
            if (wt != 0.f)
                acc = fmaf(__ldcg(&p.part_o[(((size_t)row * nsplit + s) * 4 + h) * D + dd]), wt, acc);
        }
        p.o[((size_t)b * d.hq + g * G + h) * D + dd] = acc / sm_ml[h].y;
    }
    if (tid == 0) {
        p.counter[row] = 0u;
        if (append) p.c.n_bf16[row] = n16_old + 1;
    }
}

__global__ void score_update_kernel(const ScoreParams p) {
    const LayerDims& d = p.d;
    const int row = blockIdx.y, b = row / d.hkv;
    __shared__ float2 sml[4];
    __shared__ float sinvl[4];
    if (threadIdx.x < 4) {
        const float2 ml = p.ml[(size_t)row * 4 + threadIdx.x];
        sml[threadIdx.x] = ml;
        sinvl[threadIdx.x] = ml.y;
    }
    __syncthreads();
    const int n16 = min(max(p.c.n_bf16[row], 0), d.cap_o);
    const int n8 = min(max(p.c.n_fp8[row], 0), d.cap_q);
    const int n0 = p.ctx_len[b];
    const int i0 = blockIdx.x * kScoreSlotsPerCta;
    const int i1 = min(i0 + kScoreSlotsPerCta, n16 + n8);
    for (int i = i0 + threadIdx.x; i < i1; i += blockDim.x) {
        const bool bf = i < n16;
        const size_t sl = bf ? (size_t)row * d.cap_o + i : (size_t)row * d.cap_q + (i - n16);
        const float4 lg = bf ? reinterpret_cast<const float4*>(p.logit16)[sl]
                             : reinterpret_cast<const float4*>(p.logit8)[sl];
        const float lv[4] = {lg.x, lg.y, lg.z, lg.w};
        double x = 0.0;
        for (int h = 0; h < d.G; ++h)
            x += (double)exp_scaled(lv[h], sml[h].x, p.inv_sqrt_d) / (double)sinvl[h];
        const int pos = bf ? p.c.pos16[sl] : p.c.pos8[sl];
        const int n = obs_count_after(pos, n0, p.step, d.n_obs);
        float* mu = bf ? p.c.mu16 + sl : p.c.mu8 + sl;
        float* m2 = bf ? p.c.m2_16 + sl : p.c.m2_8 + sl;
        double mv = *mu, qv = *m2;
        const double dl = x - mv;
        mv += dl / (double)n;
        qv += dl * (x - mv);
        *mu = (float)mv;
        *m2 = (float)qv;
    }
}

}  // namespace

DecodeWs decode_ws_layout(const LayerDims& d) {
    DecodeWs w{};
    w.nsplit_o = (d.cap_o + kSplitBf16 - 1) / kSplitBf16;
    w.nsplit_q = (d.cap_q + kSplitFp8 - 1) / kSplitFp8;
    const size_t ns = (size_t)(w.nsplit_o + w.nsplit_q);
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    size_t off = 0;
    w.counter = off; off = al(off + sizeof(unsigned) * d.R);
    w.ml = off;      off = al(off + sizeof(float2) * d.R * 4);
    w.part_ml = off; off = al(off + sizeof(float2) * d.R * ns * 4);
    w.part_o = off;  off = al(off + sizeof(float) * d.R * ns * 4 * d.D);
    w.logit16 = off; off = al(off + sizeof(float) * 4 * (size_t)d.R * d.cap_o);
    w.logit8 = off;  off = al(off + sizeof(float) * 4 * (size_t)d.R * d.cap_q);
    w.total = off;
    return w;
}

cudaError_t launch_decode_attn(const AttnParams& p, cudaStream_t s) {
    const dim3 grid(p.nsplit_o + p.nsplit_q, p.d.R);
    const size_t dyn = sizeof(float) * 4 * (size_t)(p.nsplit_o + p.nsplit_q);
    static unsigned char done128[64], done64[64];
    if (p.d.D == 128) {
        if (dyn > 48 * 1024) {
            const cudaError_t e = allow_max_dyn_smem(decode_attn_kernel<128>, done128);
            if (e != cudaSuccess) return e;
        }
        decode_attn_kernel<128><<<grid, kAttnThreads, dyn, s>>>(p);
    } else {
        if (dyn > 48 * 1024) {
            const cudaError_t e = allow_max_dyn_smem(decode_attn_kernel<64>, done64);
            if (e != cudaSuccess) return e;
        }
        decode_attn_kernel<64><<<grid, kAttnThreads, dyn, s>>>(p);
    }
    return cudaGetLastError();
}

cudaError_t launch_score_update(const ScoreParams& p, cudaStream_t s) {
    const dim3 grid((p.d.cap_o + p.d.cap_q + kScoreSlotsPerCta - 1) / kScoreSlotsPerCta, p.d.R);
    score_update_kernel<<<grid, 256, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace arkv
