// Decode attention over the tri-state cache (ARKV, 기술요약 §2.다: quantized tokens
// are dequantized right before attention and attended together with the
// originals) and the score observation that feeds §2.나.
//
// One CTA per split of one row: kSplitBf16 consecutive bf16 slots or kSplitFp8
// consecutive fp8 slots, 4 warps.  Each warp streams every fourth 16-token tile
// of the split through its own ring of kStages shared-memory stages, filled by
// TMA tensor loads (16 rows x 128 bytes per box, 128-byte swizzle) completing on
// per-stage mbarriers (waits are bounded).
//
// Per tile the query group's heads (G <= 4) meet the tile on the tensor cores,
// warp-level m16n8k16:
//   S^T[16 tok][8] = K[16 tok][D] * Q^T[D][8]        (heads 0..3, columns 4..7 zero)
// with one accumulator per 16-wide k block (summed afterwards in float32), and
//   O^T[D][8] += V^T[D][16 tok] * [P_hi | P_lo][16 tok][8]
// where the high and low halves of P fill the mma's 8 columns (heads 0..3 high,
// 4..7 low), so that one mma keeps ~16 significant bits of every probability.
// bf16 tiles feed the mma directly (ldmatrix, ldmatrix.trans).  FP8 tiles are
// converted to f16 (exact for E4M3): K fragments from 4-byte loads, V^T fragments
// from the 8-bit transposing ldmatrix (m16n16.trans.b8: lane (g, t) receives
// tokens 4t..4t+3 at dims g and g+8, so the k positions 2t, 2t+1 | 2t+8, 2t+9
// carry tokens 4t, 4t+1 | 4t+2, 4t+3 and P's rows are permuted to match).  The
// per-token K scale multiplies the finished logit; the V scale is folded into P
// relative to the largest V scale the warp will meet, and the constant comes
// back out of the warp's partial.  The softmax runs in float32 registers with a
// reference maximum that moves only when a logit exceeds it by 2^8 (so most
// tiles need no cross-lane reduction); raw logits go to the workspace for the
// score update.  The CTA combines its warps
// into one (max, sum, unnormalised o) partial per split; merge_kernel combines a
// row's splits and writes o.
#include <math.h>
#include <mutex>

#include <cudaTypedefs.h>

#include "arkv_internal.cuh"

namespace arkv {

namespace {

constexpr float kNegInf = -INFINITY;
constexpr unsigned kFull = 0xffffffffu;

#ifndef ARKV_STAGES
#define ARKV_STAGES 2
#endif
constexpr int kStages = ARKV_STAGES;     // tiles in flight per warp
constexpr int kWarps = 4;
constexpr int kSpinLimit = 1 << 20;      // bounded mbarrier waits (~1 s worst case)

// ------------------------------------------------------------------ shared-memory layout
template <int D>
struct Smem {
    static constexpr int kTileBytes = 16 * D * 2;                       // 16 rows of bf16
    static constexpr int kStage = 2 * kTileBytes;                       // K tile then V tile
    static constexpr int kRing = kWarps * kStages * kStage;
    static constexpr int kBars = kRing;                                 // uint64 [4][kStages]
    static constexpr int kP = kBars + kWarps * kStages * 8;             // float [4][16][8]
    static constexpr int kM = kP + kWarps * 16 * 8 * 4;                 // float [4][4]
    static constexpr int kL = kM + 16 * 4;                              // float [4][4]
    static constexpr int kRed = kL + 16 * 4;                            // float [4][4]
    static constexpr int kMax = kRed + 16 * 4;                          // float [4]
    static constexpr int kAbort = kMax + 16;                            // int: a wait gave up
    static constexpr int kBytes = kAbort + 16 + 1024;                   // + alignment slack
    static constexpr int kO = 0;                                        // float [4][4][D], in the idle ring
    static_assert(4 * 4 * D * 4 <= kRing, "the epilogue buffer must fit in the ring");
};

// Byte offset of (row, byte) in a 16-row tile of `rowb`-byte rows written by a TMA
// load with the matching swizzle (128-byte rows: 16-byte chunks XOR row % 8;
// 64-byte rows: XOR (row / 2) % 4).  Tiles sit at 1024-byte aligned addresses.
template <int ROWB>
__device__ __forceinline__ int swz(int row, int byte) {
    if constexpr (ROWB == 128) return row * 128 + (byte ^ ((row & 7) << 4));
    else return row * 64 + (byte ^ (((row >> 1) & 3) << 4));
}

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* ptr) {
    return (uint32_t)__cvta_generic_to_shared(ptr);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

// 2-D tiled TMA load (no multicast) of the box at (x, y) completing on `bar`.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits for a phase of `bar` at most kSpinLimit polls; false if it gave up.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
    for (int i = 0; i < kSpinLimit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

template <bool F16>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    if constexpr (F16)
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    else
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], const void* ptr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(ptr)));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* ptr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(smem_u32(ptr)));
}

// 16 x 16 bytes, transposed: lane (g, t) receives rows 4t..4t+3 (of the row
// addresses lanes 0..15 supply, in that order) at columns g (r0) and g + 8 (r1).
__device__ __forceinline__ void ldsm_b8_trans(uint32_t& r0, uint32_t& r1, const void* ptr) {
    asm volatile("ldmatrix.sync.aligned.m16n16.x1.trans.shared.b8 {%0,%1}, [%2];"
                 : "=r"(r0), "=r"(r1)
                 : "r"(smem_u32(ptr)));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Two E4M3 codes (low byte first) -> f16x2, exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t pair) {
    __half2_raw h = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)(pair & 0xffffu), __NV_E4M3);
    return (uint32_t)h.x | ((uint32_t)h.y << 16);
}

// ------------------------------------------------------------------ one tile
// Fragment conventions of m16n8k16: g = lane / 4, t = lane % 4.  ks: the stage
// (K tile, V tile at +VOFF); tokens t0 .. t0+15 of a segment ending at seg_end.
// sk*/sv*: the FP8 scales of this lane's tokens t0+g, t0+g+8 (1 for bf16);
// vnorm: the warp's V-scale normaliser (FP8): 64 / the largest V scale of the warp's tiles.
template <int D, bool FP8>
__device__ __forceinline__ void attend_tile(const char* ks, int t0, int seg_end, int G, float c2, float skA,
                                            float skB, float svA, float svB, float vnorm, float* logit_row,
                                            const uint32_t (&qb)[D / 16][2], float (&m_run)[2],
                                            float (&l_run)[2], float (&oacc)[D / 16][4], float (*sm_p)[8]) {
    constexpr int KB = D / 16;                       // k blocks (QK^T) and m tiles (PV)
    constexpr int ROWB = FP8 ? D : 128;              // bytes per row of one TMA box
    constexpr int VOFF = Smem<D>::kTileBytes;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const char* vs = ks + VOFF;
    const int tokA = t0 + g, tokB = t0 + g + 8;          // this lane's two tokens (QK^T rows)
    const bool okA = tokA < seg_end, okB = tokB < seg_end;
    const bool h0ok = 2 * t < G, h1ok = 2 * t + 1 < G;   // heads of this lane's logits

    // ---- S^T = K Q^T, one accumulator per k block, summed in float32
    float sacc[KB][4];
#pragma unroll
    for (int kk = 0; kk < KB; ++kk) {
        uint32_t a[4];
        if constexpr (FP8) {
            // k positions (2t, 2t+1 | 2t+8, 2t+9) <- dims 16 kk + 4t + (0, 1 | 2, 3)
            const uint32_t wA = *reinterpret_cast<const uint32_t*>(ks + swz<ROWB>(g, 16 * kk + 4 * t));
            const uint32_t wB = *reinterpret_cast<const uint32_t*>(ks + swz<ROWB>(g + 8, 16 * kk + 4 * t));
            a[0] = e4m3x2_to_f16x2(wA);
            a[2] = e4m3x2_to_f16x2(wA >> 16);
            a[1] = e4m3x2_to_f16x2(wB);
            a[3] = e4m3x2_to_f16x2(wB >> 16);
        } else {
            // ldmatrix x4: lane l supplies row (l & 7) + 8 ((l >> 3) & 1), dims 16 kk + 8 (l >> 4)
            const int r = (lane & 7) + 8 * ((lane >> 3) & 1);
            const int byte = 32 * kk + 16 * (lane >> 4);
            ldsm_x4(a, ks + (byte >> 7) * 2048 + swz<128>(r, byte & 127));
        }
        sacc[kk][0] = sacc[kk][1] = sacc[kk][2] = sacc[kk][3] = 0.f;
        mma16816<FP8>(sacc[kk], a, qb[kk][0], qb[kk][1]);
    }
#pragma unroll
    for (int w = KB / 2; w >= 1; w >>= 1)
#pragma unroll
        for (int kk = 0; kk < w; ++kk)
#pragma unroll
            for (int e = 0; e < 4; ++e) sacc[kk][e] += sacc[kk + w][e];
    // this lane: tokens A = g, B = g + 8; heads 2t, 2t+1 (t >= 2: zero columns)
    float s[4] = {sacc[0][0], sacc[0][1], sacc[0][2], sacc[0][3]};
    if constexpr (FP8) {
        s[0] *= skA; s[1] *= skA; s[2] *= skB; s[3] *= skB;
    }
    if (t < 2) {
        if (okA) *reinterpret_cast<float2*>(logit_row + (size_t)tokA * 4 + 2 * t) = make_float2(s[0], s[1]);
        if (okB) *reinterpret_cast<float2*>(logit_row + (size_t)tokB * 4 + 2 * t) = make_float2(s[2], s[3]);
    }
    const bool v0 = okA && h0ok, v1 = okA && h1ok, v2 = okB && h0ok, v3 = okB && h1ok;
    // online softmax for heads 2t, 2t+1 (uniform over the lanes sharing t), with a
    // lazy reference: it moves only when a logit exceeds it by more than 8 in log2
    // units, so probabilities stay below 2^8 and most tiles skip the reductions
    const bool need = (v0 && (s[0] - m_run[0]) * c2 > 8.f) || (v1 && (s[1] - m_run[1]) * c2 > 8.f) ||
                      (v2 && (s[2] - m_run[0]) * c2 > 8.f) || (v3 && (s[3] - m_run[1]) * c2 > 8.f);
    float al0 = 1.f, al1 = 1.f;
    if (__any_sync(kFull, need)) {
        float mx0 = fmaxf(v0 ? s[0] : kNegInf, v2 ? s[2] : kNegInf);
        float mx1 = fmaxf(v1 ? s[1] : kNegInf, v3 ? s[3] : kNegInf);
#pragma unroll
        for (int m = 4; m < 32; m <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(kFull, mx0, m));
            mx1 = fmaxf(mx1, __shfl_xor_sync(kFull, mx1, m));
        }
        const float n0 = fmaxf(m_run[0], mx0), n1 = fmaxf(m_run[1], mx1);
        al0 = (n0 == kNegInf || m_run[0] == n0) ? 1.f : exp2f((m_run[0] - n0) * c2);
        al1 = (n1 == kNegInf || m_run[1] == n1) ? 1.f : exp2f((m_run[1] - n1) * c2);
        m_run[0] = n0;
        m_run[1] = n1;
        // o columns of this lane: heads 2 (t & 1), +1, high (t < 2) or low (t >= 2) half
        const float b0 = __shfl_xor_sync(kFull, al0, 2), b1 = __shfl_xor_sync(kFull, al1, 2);
        const float oa0 = t < 2 ? al0 : b0, oa1 = t < 2 ? al1 : b1;
        if (__any_sync(kFull, oa0 != 1.f || oa1 != 1.f)) {   // a reference moved: rescale o
#pragma unroll
            for (int mt = 0; mt < KB; ++mt) {
                oacc[mt][0] *= oa0; oacc[mt][1] *= oa1;
                oacc[mt][2] *= oa0; oacc[mt][3] *= oa1;
            }
        }
    }
    const float p0 = v0 ? exp2f((s[0] - m_run[0]) * c2) : 0.f;
    const float p1 = v1 ? exp2f((s[1] - m_run[1]) * c2) : 0.f;
    const float p2 = v2 ? exp2f((s[2] - m_run[0]) * c2) : 0.f;
    const float p3 = v3 ? exp2f((s[3] - m_run[1]) * c2) : 0.f;
    l_run[0] = fmaf(l_run[0], al0, p0 + p2);
    l_run[1] = fmaf(l_run[1], al1, p1 + p3);
    // P (times V scale / normaliser for FP8) to shared memory, [token][head]
    float w0 = p0, w1 = p1, w2 = p2, w3 = p3;
    if constexpr (FP8) {
        const float fa = svA * vnorm, fb = svB * vnorm;
        w0 *= fa; w1 *= fa; w2 *= fb; w3 *= fb;
    }
    if (t < 2) {
        *reinterpret_cast<float2*>(&sm_p[g][2 * t]) = make_float2(w0, w1);
        *reinterpret_cast<float2*>(&sm_p[g + 8][2 * t]) = make_float2(w2, w3);
    }
    __syncwarp();
    // B fragment [P_hi | P_lo]: lane (g, t) holds column g (head g & 3, high half if
    // g < 4) at the k positions 2t, 2t+1 | 2t+8, 2t+9, i.e. tokens
    // bf16: 2t, 2t+1 | 2t+8, 2t+9;  FP8 (permuted to the b8 ldmatrix): 4t, 4t+1 | 4t+2, 4t+3
    const int hc = g & 3;
    const int ta = FP8 ? 4 * t : 2 * t, tb = FP8 ? 4 * t + 2 : 2 * t + 8;
    const float e0 = sm_p[ta][hc], e1 = sm_p[ta + 1][hc], e2 = sm_p[tb][hc], e3 = sm_p[tb + 1][hc];
    uint32_t bb0, bb1;
    if constexpr (FP8) {
        const uint32_t h0 = pack_f16(e0, e1), h1 = pack_f16(e2, e3);
        if (g < 4) {
            bb0 = h0; bb1 = h1;
        } else {
            const __half2 x0 = *reinterpret_cast<const __half2*>(&h0), x1 = *reinterpret_cast<const __half2*>(&h1);
            bb0 = pack_f16(e0 - __low2float(x0), e1 - __high2float(x0));
            bb1 = pack_f16(e2 - __low2float(x1), e3 - __high2float(x1));
        }
    } else {
        const uint32_t h0 = pack_bf16(e0, e1), h1 = pack_bf16(e2, e3);
        if (g < 4) {
            bb0 = h0; bb1 = h1;
        } else {
            const __nv_bfloat162 x0 = *reinterpret_cast<const __nv_bfloat162*>(&h0);
            const __nv_bfloat162 x1 = *reinterpret_cast<const __nv_bfloat162*>(&h1);
            bb0 = pack_bf16(e0 - __low2float(x0), e1 - __high2float(x0));
            bb1 = pack_bf16(e2 - __low2float(x1), e3 - __high2float(x1));
        }
    }
    // past the segment end the tile holds stale slots or zero fill: P is 0 there,
    // and a partial tile also zeroes those V elements so that no stale bit pattern
    // can reach the accumulator (same token order as the B fragment)
    const bool partial = t0 + 16 > seg_end;   // warp-uniform
    uint32_t m01 = 0xffffffffu, m23 = 0xffffffffu;
    if (partial) {
        m01 = (t0 + ta < seg_end ? 0xffffu : 0u) | (t0 + ta + 1 < seg_end ? 0xffff0000u : 0u);
        m23 = (t0 + tb < seg_end ? 0xffffu : 0u) | (t0 + tb + 1 < seg_end ? 0xffff0000u : 0u);
    }
#pragma unroll
    for (int mt = 0; mt < KB; ++mt) {
        uint32_t a[4];
        if constexpr (FP8) {
            // lanes 0..15 supply token rows 0..15 at dims 16 mt .. 16 mt + 15
            uint32_t r0, r1;
            ldsm_b8_trans(r0, r1, vs + swz<ROWB>(lane & 15, 16 * mt));
            a[0] = e4m3x2_to_f16x2(r0);          // dim g,     tokens 4t, 4t+1
            a[2] = e4m3x2_to_f16x2(r0 >> 16);    // dim g,     tokens 4t+2, 4t+3
            a[1] = e4m3x2_to_f16x2(r1);          // dim g + 8, tokens 4t, 4t+1
            a[3] = e4m3x2_to_f16x2(r1 >> 16);    // dim g + 8, tokens 4t+2, 4t+3
        } else {
            // ldmatrix.trans matrix q = lane / 8: tokens 8 (q / 2) + lane % 8, dims 16 mt + 8 (q % 2)
            const int tok = (lane & 7) + 8 * (lane >> 4);
            const int byte = 2 * (16 * mt + 8 * ((lane >> 3) & 1));
            ldsm_x4_trans(a, vs + (byte >> 7) * 2048 + swz<128>(tok, byte & 127));
        }
        if (partial) {
            a[0] &= m01; a[1] &= m01; a[2] &= m23; a[3] &= m23;
        }
        mma16816<FP8>(oacc[mt], a, bb0, bb1);
    }
}

// Q^T B fragments of head g (zero past G) of a row: for block kk, b0 holds the
// k positions 2t, 2t+1 and b1 2t+8, 2t+9 -- dims 16 kk + (2t, 2t+1 | 2t+8, 2t+9)
// for bf16 (ldmatrix layout), dims 16 kk + 4t + (0, 1 | 2, 3) in f16 for FP8.
template <int D>
__device__ __forceinline__ void load_q(const AttnParams& p, int row, bool fp8, uint32_t (&qb)[D / 16][2]) {
    const int lane = threadIdx.x & 31, fg = lane >> 2, ft = lane & 3;
    const int b = row / p.d.hkv, gk = row - b * p.d.hkv, G = p.d.G;
    const bool hv = fg < G;
    const uint16_t* qrow = p.q + ((size_t)b * p.d.hq + gk * G + (hv ? fg : 0)) * D;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t x = 0u, y = 0u;
        if (hv) {
            if (fp8) {
                const uint2 u = *reinterpret_cast<const uint2*>(qrow + 16 * kk + 4 * ft);
                x = pack_f16(bf16_lo(u.x), bf16_hi(u.x));
                y = pack_f16(bf16_lo(u.y), bf16_hi(u.y));
            } else {
                x = *reinterpret_cast<const uint32_t*>(qrow + 16 * kk + 2 * ft);
                y = *reinterpret_cast<const uint32_t*>(qrow + 16 * kk + 2 * ft + 8);
            }
        }
        qb[kk][0] = x;
        qb[kk][1] = y;
    }
}

template <int D>
__global__ void __launch_bounds__(32 * kWarps) decode_attn_kernel(const __grid_constant__ AttnParams p) {
    using SL = Smem<D>;
    constexpr int KB = D / 16;
    constexpr int STAGE = SL::kStage;
    constexpr int VOFF = SL::kTileBytes;
    constexpr int NB16 = D * 2 / 128;                // bf16 boxes per tile
    const LayerDims& d = p.d;
    // CTA order, longest work first: the FP8 splits of every row (rows fastest), then
    // the bf16 splits.  An FP8 split holds twice the tokens of a bf16 split and costs
    // more per tile, so dispatching it last would leave the longest CTAs in the tail.
    const int nq = p.nsplit_q * d.R, bid = blockIdx.x;
    const int row = bid < nq ? bid % d.R : (bid - nq) % d.R;
    const int split = bid < nq ? p.nsplit_o + bid / d.R : (bid - nq) / d.R;
    const int b = row / d.hkv, gk = row - b * d.hkv;
    const int nsplit = p.nsplit_o + p.nsplit_q;
    const bool fp8 = split >= p.nsplit_o;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int fg = lane >> 2, ft = lane & 3;

    // the split's slot range; the bf16 segment includes the slot of the new token
    const int n16_old = min(max(p.c.n_bf16[row], 0), d.cap_o);   // counts are clamped to the
    const bool append = n16_old < d.cap_o;                          // capacities before any use;
    int s0, s1;                                                     // merge_kernel advances n_bf16
    if (!fp8) {
        s0 = split * kSplitBf16;
        s1 = min(s0 + kSplitBf16, n16_old + (append ? 1 : 0));
    } else {
        s0 = (split - p.nsplit_o) * kSplitFp8;
        s1 = min(s0 + kSplitFp8, min(max(p.c.n_fp8[row], 0), d.cap_q));
    }
    if (s0 >= s1) return;                            // nothing live in this split

    extern __shared__ char smem_raw[];
    char* smem = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + SL::kBars) + warp * kStages;
    float (*sm_p)[8] = reinterpret_cast<float (*)[16][8]>(smem + SL::kP)[warp];
    char* ring = smem + warp * kStages * STAGE;
    if (lane == 0) {
#pragma unroll
        for (int st = 0; st < kStages; ++st) mbar_init(&bars[st], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // append: the CTA whose split covers the new slot stores the token before any
    // tensor load reads that slot (the proxy fence orders the two)
    if (!fp8 && append && n16_old >= s0 && n16_old < s1) {
        const uint16_t* kn = p.k_new + ((size_t)b * d.hkv + gk) * D;
        const uint16_t* vn = p.v_new + ((size_t)b * d.hkv + gk) * D;
        const size_t sl = (size_t)row * d.cap_o + n16_old;
        for (int c = tid; c < D / 8; c += blockDim.x) {
            *reinterpret_cast<uint4*>(p.c.k16 + sl * D + 8 * c) = *reinterpret_cast<const uint4*>(kn + 8 * c);
            *reinterpret_cast<uint4*>(p.c.v16 + sl * D + 8 * c) = *reinterpret_cast<const uint4*>(vn + 8 * c);
        }
        if (tid == 0) {
            p.c.pos16[sl] = p.ctx_len[b] + p.step;
            p.c.mu16[sl] = 0.0;
            p.c.m2_16[sl] = 0.0;
        }
        asm volatile("fence.proxy.async.global;" ::: "memory");
    }
    int* sm_abort = reinterpret_cast<int*>(smem + SL::kAbort);
    if (tid == 0) *sm_abort = 0;
    __syncthreads();

    // this warp's tiles: s0 + 16 (warp + 4 i)
    const int first = s0 + 16 * warp;
    const int ntiles = first < s1 ? (s1 - first + 16 * kWarps - 1) / (16 * kWarps) : 0;
    const int ybase = fp8 ? row * d.cap_q : row * d.cap_o;
    auto issue = [&](int i) {
        const int st = i % kStages;
        const int y = ybase + first + 16 * kWarps * i;
        char* kd = ring + st * STAGE;
        if (!fp8) {
            mbar_expect_tx(&bars[st], 2 * 16 * D * 2);
#pragma unroll
            for (int bx = 0; bx < NB16; ++bx) {
                tma_load_2d(kd + bx * 2048, &p.tm_k16, bx * 64, y, &bars[st]);
                tma_load_2d(kd + VOFF + bx * 2048, &p.tm_v16, bx * 64, y, &bars[st]);
            }
        } else {
            mbar_expect_tx(&bars[st], 2 * 16 * D);
            tma_load_2d(kd, &p.tm_k8, 0, y, &bars[st]);
            tma_load_2d(kd + VOFF, &p.tm_v8, 0, y, &bars[st]);
        }
    };
    if (lane == 0)
        for (int i = 0; i < min(kStages, ntiles); ++i) issue(i);

    float m_run[2] = {kNegInf, kNegInf}, l_run[2] = {0.f, 0.f}, oacc[KB][4];
#pragma unroll
    for (int mt = 0; mt < KB; ++mt) oacc[mt][0] = oacc[mt][1] = oacc[mt][2] = oacc[mt][3] = 0.f;
    uint32_t qb[KB][2];
    load_q<D>(p, row, fp8, qb);
    const float c2 = (float)(p.inv_sqrt_d * 1.4426950408889634);   // log2(e) / sqrt(D)
    const float* skb = p.c.sk + (size_t)row * d.cap_q;
    const float* svb = p.c.sv + (size_t)row * d.cap_q;
    float vmax = 1.f, vnorm = 1.f;                   // FP8: the warp's largest V scale
    float nskA = 1.f, nskB = 1.f, nsvA = 1.f, nsvB = 1.f;
    if (fp8) {
        vmax = 0.f;
        for (int i = 0; i < ntiles; ++i) {
            const int tk = first + 16 * kWarps * i + (lane & 15);
            if (tk < s1) vmax = fmaxf(vmax, __ldg(svb + tk));
        }
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(kFull, vmax, m));
        vnorm = vmax > 0.f ? 64.f / vmax : 0.f;   // p < 2^8: p sv vnorm < 2^14, inside f16
        const int a = min(first + fg, d.cap_q - 1), c = min(first + fg + 8, d.cap_q - 1);
        nskA = __ldg(skb + a); nskB = __ldg(skb + c);
        nsvA = __ldg(svb + a); nsvB = __ldg(svb + c);
    }
    float* logit_row = fp8 ? p.logit8 + (size_t)row * d.cap_q * 4 : p.logit16 + (size_t)row * d.cap_o * 4;
    for (int i = 0; i < ntiles; ++i) {
        const int st = i % kStages;
        const int t0 = first + 16 * kWarps * i;
        if (!mbar_wait(&bars[st], (uint32_t)((i / kStages) & 1))) {
            // a copy did not land in time: flag it, give every copy this warp issued
            // (this one included) a last bounded chance to land, and leave the ring
            // alone from here on (the epilogue below does not reuse it)
            if (lane == 0) {
                atomicOr(p.c.status, ARKV_STATUS_TIMEOUT);
                atomicExch(sm_abort, 1);
            }
            for (int j = i; j < min(i + kStages, ntiles); ++j)
                mbar_wait(&bars[j % kStages], (uint32_t)((j / kStages) & 1));
            break;
        }
        const char* ks = ring + st * STAGE;
        if (!fp8) {
            attend_tile<D, false>(ks, t0, s1, d.G, c2, 1.f, 1.f, 1.f, 1.f, 1.f, logit_row, qb, m_run, l_run,
                                  oacc, sm_p);
        } else {
            const float skA = nskA, skB = nskB, svA = nsvA, svB = nsvB;
            if (i + 1 < ntiles) {      // the next tile's scales, one tile ahead
                const int a = min(t0 + 16 * kWarps + fg, d.cap_q - 1), c = min(t0 + 16 * kWarps + fg + 8, d.cap_q - 1);
                nskA = __ldg(skb + a); nskB = __ldg(skb + c);
                nsvA = __ldg(svb + a); nsvB = __ldg(svb + c);
            }
            attend_tile<D, true>(ks, t0, s1, d.G, c2, skA, skB, svA, svB, vnorm, logit_row, qb, m_run, l_run,
                                 oacc, sm_p);
        }
        __syncwarp();
        if (lane == 0 && i + kStages < ntiles) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            issue(i + kStages);
        }
    }

    __syncthreads();   // every warp has drained its ring: the epilogue may reuse it
    const size_t pb = (size_t)row * nsplit + split;
    if (*sm_abort) {
        // a wait gave up: copies may still be landing in the ring, so write an empty
        // partial (weight 0 in the merge) without touching shared memory; the status
        // bit already tells the caller that this call's output is not to be used
        for (int idx = tid; idx < 4 * D; idx += blockDim.x) {
            p.part_o[(pb * 4 + idx / D) * D + idx % D] = 0.f;
            if (idx % D == 0) p.part_ml[pb * 4 + idx / D] = make_float2(kNegInf, 0.f);
        }
        return;
    }
    float (*sm_o)[4][D] = reinterpret_cast<float (*)[4][D]>(smem + SL::kO);
    float (*sm_m)[4] = reinterpret_cast<float (*)[4]>(smem + SL::kM);
    float (*sm_l)[4] = reinterpret_cast<float (*)[4]>(smem + SL::kL);
    float (*sm_w)[4] = reinterpret_cast<float (*)[4]>(smem + SL::kRed);
    float* sm_max = reinterpret_cast<float*>(smem + SL::kMax);
    // warp totals.  l: over the lanes sharing a head pair (all fg).  o: oacc[mt] =
    // (dim 16 mt + fg, columns 2 ft, 2 ft + 1) and (dim 16 mt + fg + 8, same
    // columns); columns 0..3 hold the high half, 4..7 the low half of heads 0..3.
    // FP8 partials carry the V-scale normaliser, taken out here.
#pragma unroll
    for (int m = 4; m < 32; m <<= 1) {
        l_run[0] += __shfl_xor_sync(kFull, l_run[0], m);
        l_run[1] += __shfl_xor_sync(kFull, l_run[1], m);
    }
    const float un = fp8 ? vmax * (1.f / 64.f) : 1.f;
#pragma unroll
    for (int mt = 0; mt < KB; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) oacc[mt][e] += __shfl_xor_sync(kFull, oacc[mt][e], 2);
    if (ft < 2) {
#pragma unroll
        for (int mt = 0; mt < KB; ++mt) {
            sm_o[warp][2 * ft][16 * mt + fg] = oacc[mt][0] * un;
            sm_o[warp][2 * ft + 1][16 * mt + fg] = oacc[mt][1] * un;
            sm_o[warp][2 * ft][16 * mt + fg + 8] = oacc[mt][2] * un;
            sm_o[warp][2 * ft + 1][16 * mt + fg + 8] = oacc[mt][3] * un;
        }
        if (fg == 0) {
            sm_l[warp][2 * ft] = l_run[0];
            sm_l[warp][2 * ft + 1] = l_run[1];
            sm_m[warp][2 * ft] = m_run[0];
            sm_m[warp][2 * ft + 1] = m_run[1];
        }
    }
    __syncthreads();
    if (tid < 16) {
        const int w = tid >> 2, h = tid & 3;
        float M = kNegInf;
#pragma unroll
        for (int v = 0; v < kWarps; ++v) M = fmaxf(M, sm_m[v][h]);
        sm_w[w][h] = (M == kNegInf || sm_m[w][h] == kNegInf) ? 0.f : exp_scaled(sm_m[w][h], M, p.inv_sqrt_d);
        if (w == 0) sm_max[h] = M;
    }
    __syncthreads();
    for (int idx = tid; idx < 4 * D; idx += blockDim.x) {
        const int h = idx / D, dd = idx - h * D;
        float O = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) O = fmaf(sm_o[w][h][dd], sm_w[w][h], O);
        p.part_o[(pb * 4 + h) * D + dd] = O;
        if (dd == 0) {
            float L = 0.f;
#pragma unroll
            for (int w = 0; w < kWarps; ++w) L = fmaf(sm_l[w][h], sm_w[w][h], L);
            p.part_ml[pb * 4 + h] = make_float2(sm_max[h], L);
        }
    }
}

// Merges the split partials of one (row, head): M = max of the split maxima,
// L = sum of l_s exp((m_s - M)/sqrt(D)), o = sum of o_s exp(..) / L.  4 x D
// threads: thread (q, d) sums the splits s = q mod 4 of output dim d, so every
// thread has only a few independent loads in flight.  Also publishes (M, L) for
// the score update.  The row's bf16 count is advanced past the appended token by
// the last of the row's G merge CTAs to finish (a ticket in the workspace): every
// merge CTA of the row reads the count it was launched with, so it may only move
// once all of them have read it.
template <int D>
__global__ void __launch_bounds__(4 * D) merge_kernel(const AttnParams p) {
    const LayerDims& d = p.d;
    const int row = blockIdx.x, h = blockIdx.y;
    const int b = row / d.hkv, g = row - b * d.hkv;
    const int nsplit = p.nsplit_o + p.nsplit_q;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    extern __shared__ float sm_w[];                  // [nlive] weights, then [4][D] partial sums
    __shared__ float sm_red[4 * D / 32];
    __shared__ float sm_ML[2];
    const double inv = p.inv_sqrt_d;
    // the live splits of the row: j < nlo -> bf16 split j, else fp8 split j - nlo
    const int n16_old = min(max(p.c.n_bf16[row], 0), d.cap_o);
    const int nl16 = n16_old + (n16_old < d.cap_o ? 1 : 0);
    const int n8 = min(max(p.c.n_fp8[row], 0), d.cap_q);
    const int nlo = (nl16 + kSplitBf16 - 1) / kSplitBf16, nlive = nlo + (n8 + kSplitFp8 - 1) / kSplitFp8;
    auto split_of = [&](int j) { return j < nlo ? j : p.nsplit_o + (j - nlo); };
    const float2* pml = p.part_ml + (size_t)row * nsplit * 4;
    // the partial outputs this thread sums (splits q, q + 4, ...) do not depend on
    // the weights: their loads are issued first, so their latency overlaps the
    // reductions below
    const int q = tid / D, dd = tid - q * D;
    const float* po = p.part_o + (size_t)row * nsplit * 4 * D + (size_t)h * D + dd;
    constexpr int kPre = 12;
    float pre[kPre];
#pragma unroll
    for (int k = 0; k < kPre; ++k) {
        const int sidx = q + 4 * k;
        pre[k] = sidx < nlive ? po[(size_t)split_of(sidx) * 4 * D] : 0.f;
    }

    float mloc = kNegInf;
    for (int s = tid; s < nlive; s += blockDim.x) mloc = fmaxf(mloc, pml[split_of(s) * 4 + h].x);
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) mloc = fmaxf(mloc, __shfl_xor_sync(kFull, mloc, m));
    if (lane == 0) sm_red[warp] = mloc;
    __syncthreads();
    if (tid == 0) {
        float M = kNegInf;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) M = fmaxf(M, sm_red[w]);
        sm_ML[0] = M;
    }
    __syncthreads();
    const float M = sm_ML[0];
    float lloc = 0.f;
    for (int s = tid; s < nlive; s += blockDim.x) {
        const float2 ml = pml[split_of(s) * 4 + h];
        const float wt = (ml.y > 0.f && M != kNegInf) ? exp_scaled(ml.x, M, inv) : 0.f;
        sm_w[s] = wt;
        lloc = fmaf(ml.y, wt, lloc);
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) lloc += __shfl_xor_sync(kFull, lloc, m);
    __syncthreads();
    if (lane == 0) sm_red[warp] = lloc;
    __syncthreads();
    if (tid == 0) {
        float L = 0.f;
        for (int w = 0; w < (int)(blockDim.x >> 5); ++w) L += sm_red[w];
        sm_ML[1] = L;
        p.ml[(size_t)row * 4 + h] = make_float2(M, L);
    }
    __syncthreads();   // the weights
    float acc = 0.f;
#pragma unroll
    for (int k = 0; k < kPre; ++k) {
        const int sidx = q + 4 * k;
        if (sidx < nlive && sm_w[sidx] != 0.f) acc = fmaf(pre[k], sm_w[sidx], acc);
    }
#pragma unroll 4
    for (int s = q + 4 * kPre; s < nlive; s += 4) {
        const float wt = sm_w[s];
        if (wt != 0.f) acc = fmaf(po[(size_t)split_of(s) * 4 * D], wt, acc);
    }
    float* sm_acc = sm_w + nsplit;
    sm_acc[q * D + dd] = acc;
    __syncthreads();
    if (q == 0 && h < d.G) {
        const float o = (sm_acc[dd] + sm_acc[D + dd]) + (sm_acc[2 * D + dd] + sm_acc[3 * D + dd]);
        p.o[((size_t)b * d.hq + g * d.G + h) * D + dd] = o / sm_ML[1];
    }
    if (tid == 0) {
        __threadfence();                                 // this CTA's reads of the count come first
        if (atomicAdd(&p.counter[row], 1u) == (unsigned)(d.G - 1)) {
            p.counter[row] = 0u;                         // ready for the next call
            if (n16_old < d.cap_o) p.c.n_bf16[row] = n16_old + 1;
            else atomicOr(p.c.status, ARKV_STATUS_BF16_FULL);   // the new token was dropped
        }
    }
}

// One thread per live slot: x = sum over the group's heads of exp((raw - M)/sqrt(D)) / L,
// then one Welford step with the token's observation count.
__global__ void __launch_bounds__(256) score_update_kernel(const ScoreParams p) {
    const LayerDims& d = p.d;
    const int row = blockIdx.y, b = row / d.hkv;
    __shared__ float2 sml[4];   // final (max, sum) of every head
    if (threadIdx.x < 4) sml[threadIdx.x] = __ldg(&p.ml[(size_t)row * 4 + threadIdx.x]);
    __syncthreads();
    const int n16 = min(max(__ldg(&p.c.n_bf16[row]), 0), d.cap_o);
    const int n8 = min(max(__ldg(&p.c.n_fp8[row]), 0), d.cap_q);
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n16 + n8) return;
    const bool bf = i < n16;
    const size_t sl = bf ? (size_t)row * d.cap_o + i : (size_t)row * d.cap_q + (i - n16);
    const float4 lg = __ldg(bf ? reinterpret_cast<const float4*>(p.logit16) + sl
                               : reinterpret_cast<const float4*>(p.logit8) + sl);
    const int pos = __ldg(bf ? p.c.pos16 + sl : p.c.pos8 + sl);
    double* __restrict__ mu = bf ? p.c.mu16 + sl : p.c.mu8 + sl;
    double* __restrict__ m2 = bf ? p.c.m2_16 + sl : p.c.m2_8 + sl;
    const double mu_old = *mu, m2_old = *m2;
    const float lv[4] = {lg.x, lg.y, lg.z, lg.w};
    double x = 0.0;
#pragma unroll
    for (int h = 0; h < 4; ++h)
        if (h < d.G) x += (double)exp_scaled(lv[h], sml[h].x, p.inv_sqrt_d) / (double)sml[h].y;
    const int n = obs_count_after(pos, __ldg(&p.ctx_len[b]), p.step, d.n_obs);
    double mv = mu_old, qv = m2_old;
    const double dl = x - mv;
    mv += dl / (double)n;
    qv += dl * (x - mv);
    *mu = mv;
    *m2 = qv;
}

// ------------------------------------------------------------------ tensor maps
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// 2-D map over rows x D elements of one cache array, 16-row boxes of `box_inner`
// elements.
bool make_map(CUtensorMap* m, const void* base, CUtensorMapDataType dt, int elem_bytes, int D, long long rows,
              int box_inner, CUtensorMapSwizzle sw) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)D * elem_bytes};
    cuuint32_t box[2] = {(cuuint32_t)box_inner, 16};
    cuuint32_t es[2] = {1, 1};
    return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
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

cudaError_t launch_decode_attn(AttnParams& p, cudaStream_t s) {
    const LayerDims& d = p.d;
    const int D = d.D;
    const bool ok = make_map(&p.tm_k16, p.c.k16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, (long long)d.R * d.cap_o, 64,
                             CU_TENSOR_MAP_SWIZZLE_128B) &&
                    make_map(&p.tm_v16, p.c.v16, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, (long long)d.R * d.cap_o, 64,
                             CU_TENSOR_MAP_SWIZZLE_128B) &&
                    make_map(&p.tm_k8, p.c.k8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, D, (long long)d.R * d.cap_q, D,
                             D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B) &&
                    make_map(&p.tm_v8, p.c.v8, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, D, (long long)d.R * d.cap_q, D,
                             D == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B);
    if (!ok) return cudaErrorInvalidValue;
    const int nsplit = p.nsplit_o + p.nsplit_q;
    const dim3 mgrid(d.R, d.G);
    const size_t mdyn = sizeof(float) * ((size_t)nsplit + 4 * (size_t)D);
    if (mdyn > 48 * 1024) return cudaErrorInvalidValue;
    static unsigned char done128[64], done64[64];
    if ((long long)nsplit * d.R > 0x7fffffffLL) return cudaErrorInvalidValue;
    const dim3 grid(nsplit * d.R);   // one CTA per (split, row); order set in the kernel
    if (D == 128) {
        const cudaError_t e = allow_max_dyn_smem(decode_attn_kernel<128>, done128);
        if (e != cudaSuccess) return e;
        decode_attn_kernel<128><<<grid, 32 * kWarps, Smem<128>::kBytes, s>>>(p);
        merge_kernel<128><<<mgrid, 4 * 128, mdyn, s>>>(p);
    } else {
        const cudaError_t e = allow_max_dyn_smem(decode_attn_kernel<64>, done64);
        if (e != cudaSuccess) return e;
        decode_attn_kernel<64><<<grid, 32 * kWarps, Smem<64>::kBytes, s>>>(p);
        merge_kernel<64><<<mgrid, 4 * 64, mdyn, s>>>(p);
    }
    return cudaGetLastError();
}

cudaError_t launch_score_update(const ScoreParams& p, cudaStream_t s) {
    const dim3 grid((p.d.cap_o + p.d.cap_q + 255) / 256, p.d.R);
    score_update_kernel<<<grid, 256, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace arkv
