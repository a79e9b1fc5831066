// Prefill attention statistics and initial scores (ARKV, 기술요약 §2.가: per-layer
// Original:Quantization ratio from attention entropy, variance and kurtosis;
// §2.나: the scores start from the attention each token received in prefill).
//
// Three launches per layer, all float64:
//  1. prefill_sweep_kernel: one sweep over each row's keys, cut into key ranges
//     (one CTA per range and 8 observation positions x the group's heads).  For
//     every query it keeps an online softmax reference m and the sums
//       S0 = sum e^(a-m), T1 = sum (a-m) e^(a-m), S2, S3, S4 = sum e^(j(a-m)),
//     a = q.k / sqrt(D), rescaled whenever m moves, and writes one partial per
//     (query, range).  The statistics need no second sweep: with L = S0,
//       sum p ln p = T1/L - ln L,  sum p^j = S_j / L^j.
//  2. prefill_query_kernel: merges each query's partials in range order into
//     (M, L) and its entropy, variance and kurtosis; the central moments about
//     1/n follow from sum p^j by the binomial expansion (sum p = 1).
//  3. prefill_observe_kernel: each CTA owns a block of keys, walks the
//     observation queries in order and applies one Welford step per query that
//     sees the key, x_k(i) = sum over the group's heads of exp(a - M) / L: the
//     initial (mu, M2) of every key, in the oracle's order and without atomics.
// A fixed-order reduction gives the layer means.
#include <math.h>

#include "arkv_internal.cuh"

namespace arkv {

namespace {

constexpr int kPfThreads = 256;
constexpr int kPfPositions = 8;   // observation positions per CTA (one per warp)
constexpr int kPfTile = 64;       // keys per shared-memory tile (lane owns keys l, l + 32)
constexpr int kPfRange = 1024;    // keys per sweep CTA
constexpr int kPart = 6;          // doubles per partial: m, S0, T1, S2, S3, S4

template <int D>
__device__ __forceinline__ void load_key_tile(double* sk, const uint16_t* krow, int kt, int kend) {
    constexpr int SD = D + 1;
    constexpr int WPR = D / 8;   // uint4 words per key
    for (int w = threadIdx.x; w < kPfTile * WPR; w += blockDim.x) {
        const int kk = w / WPR, c = (w - kk * WPR) * 8;
        const int key = kt + kk;
        double* dst = sk + kk * SD + c;
        if (key < kend) {
            const uint4 u = *reinterpret_cast<const uint4*>(krow + (size_t)key * D + c);
            dst[0] = bf16_lo(u.x); dst[1] = bf16_hi(u.x);
            dst[2] = bf16_lo(u.y); dst[3] = bf16_hi(u.y);
            dst[4] = bf16_lo(u.z); dst[5] = bf16_hi(u.z);
            dst[6] = bf16_lo(u.w); dst[7] = bf16_hi(u.w);
        } else {
#pragma unroll
            for (int e = 0; e < 8; ++e) dst[e] = 0.0;
        }
    }
}

// The 32 query vectors (8 positions x 4 head slots) of positions i0 .. i0+7 of
// row (b, g), float64 in shared memory; zero for head slots >= G and positions >= n_obs.
template <int D>
__device__ __forceinline__ void load_query_tile(double* sq, const PrefillParams& p, int b, int g, int i0) {
    constexpr int SD = D + 1;
    const LayerDims& d = p.d;
    for (int w = threadIdx.x; w < 32 * D; w += blockDim.x) {
        const int qi = w / D, e = w - qi * D;
        const int ww = qi / 4, h = qi - ww * 4;
        const int ii = i0 + ww;
        double v = 0.0;
        if (h < d.G && ii < d.n_obs)
            v = bf16_to_f32(p.q_obs[(((size_t)b * d.hq + g * d.G + h) * d.n_obs + ii) * D + e]);
        sq[qi * SD + e] = v;
    }
}

// dot[h][j] = q(warp's position, head h) . k(tile key lane + 32 j), float64.
template <int D>
__device__ __forceinline__ void tile_dots(const double* sq, const double* sk, int warp, int lane,
                                          double (&dot)[4][2]) {
    constexpr int SD = D + 1;
#pragma unroll
    for (int h = 0; h < 4; ++h) dot[h][0] = dot[h][1] = 0.0;
    const double* q0 = sq + (warp * 4) * SD;
    const double* k0 = sk + lane * SD;
#pragma unroll 4
    for (int e = 0; e < D; ++e) {
        double qv[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) qv[h] = q0[h * SD + e];
        const double ka = k0[e], kb = k0[32 * SD + e];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            dot[h][0] = fma(qv[h], ka, dot[h][0]);
            dot[h][1] = fma(qv[h], kb, dot[h][1]);
        }
    }
}

// Online sums of one query over some keys (see the file comment).
struct Moments {
    double m, s0, t1, s2, s3, s4;
};

__device__ __forceinline__ void moments_add(Moments& a, double x) {
    if (x > a.m) {                                   // the reference moves up to x
        if (a.s0 > 0.0) {
            const double dl = a.m - x, r = exp(dl), r2 = r * r;
            a.t1 = (a.t1 + dl * a.s0) * r;
            a.s0 = a.s0 * r + 1.0;
            a.s2 = a.s2 * r2 + 1.0;
            a.s3 = a.s3 * (r2 * r) + 1.0;
            a.s4 = a.s4 * (r2 * r2) + 1.0;
        } else {
            a.s0 = a.s2 = a.s3 = a.s4 = 1.0;
            a.t1 = 0.0;
        }
        a.m = x;
    } else {
        const double dl = x - a.m, e = exp(dl), e2 = e * e;
        a.s0 += e;
        a.t1 = fma(dl, e, a.t1);
        a.s2 += e2;
        a.s3 = fma(e2, e, a.s3);
        a.s4 = fma(e2, e2, a.s4);
    }
}

__device__ __forceinline__ Moments moments_merge(const Moments& a, const Moments& b) {
    if (b.s0 == 0.0) return a;
    if (a.s0 == 0.0) return b;
    Moments r;
    r.m = fmax(a.m, b.m);
    const double da = a.m - r.m, db = b.m - r.m;
    const double ra = exp(da), rb = exp(db);
    r.s0 = a.s0 * ra + b.s0 * rb;
    r.t1 = (a.t1 + da * a.s0) * ra + (b.t1 + db * b.s0) * rb;
    r.s2 = a.s2 * (ra * ra) + b.s2 * (rb * rb);
    r.s3 = a.s3 * (ra * ra * ra) + b.s3 * (rb * rb * rb);
    r.s4 = a.s4 * ((ra * ra) * (ra * ra)) + b.s4 * ((rb * rb) * (rb * rb));
    return r;
}

__device__ __forceinline__ Moments moments_shfl_xor(const Moments& a, int mask) {
    Moments b;
    b.m = __shfl_xor_sync(0xffffffffu, a.m, mask);
    b.s0 = __shfl_xor_sync(0xffffffffu, a.s0, mask);
    b.t1 = __shfl_xor_sync(0xffffffffu, a.t1, mask);
    b.s2 = __shfl_xor_sync(0xffffffffu, a.s2, mask);
    b.s3 = __shfl_xor_sync(0xffffffffu, a.s3, mask);
    b.s4 = __shfl_xor_sync(0xffffffffu, a.s4, mask);
    return b;
}

// ------------------------------------------------------------------ 1. the sweep
template <int D>
__global__ void __launch_bounds__(kPfThreads) prefill_sweep_kernel(const PrefillParams p) {
    constexpr int SD = D + 1;
    const LayerDims& d = p.d;
    const int row = blockIdx.z, b = row / d.hkv, g = row - b * d.hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    extern __shared__ double smem[];
    double* sq = smem;                          // [32][SD]
    double* sk = sq + 32 * SD;                  // [kPfTile][SD]

    const int n0 = min(p.ctx_len[b], p.n_stride);
    const int i0 = blockIdx.x * kPfPositions;
    const int i = i0 + warp;                                    // this warp's observation
    const int P = n0 - d.n_obs + i;                             // its position
    const int i_last = min(d.n_obs, i0 + kPfPositions) - 1;
    const int kend = min(n0, n0 - d.n_obs + i_last + 1);        // keys any warp of the CTA sees
    const int k_lo = blockIdx.y * kPfRange, k_hi = min(kend, k_lo + kPfRange);
    const uint16_t* krow = p.k + ((size_t)b * d.hkv + g) * p.n_stride * D;
    const double inv_sqrt_d = 1.0 / sqrt((double)D);

    load_query_tile<D>(sq, p, b, g, i0);
    Moments mo[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) mo[h] = Moments{-INFINITY, 0.0, 0.0, 0.0, 0.0, 0.0};
    for (int kt = k_lo; kt < k_hi; kt += kPfTile) {
        __syncthreads();
        load_key_tile<D>(sk, krow, kt, k_hi);
        __syncthreads();
        double dot[4][2];
        tile_dots<D>(sq, sk, warp, lane, dot);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int key = kt + lane + 32 * j;
            if (i >= d.n_obs || key >= k_hi || key > P) continue;
#pragma unroll
            for (int h = 0; h < 4; ++h)
                if (h < d.G) moments_add(mo[h], dot[h][j] * inv_sqrt_d);
        }
    }
#pragma unroll
    for (int h = 0; h < 4; ++h)
#pragma unroll
        for (int msk = 16; msk >= 1; msk >>= 1) mo[h] = moments_merge(mo[h], moments_shfl_xor(mo[h], msk));
    if (lane == 0 && i < d.n_obs) {
        const int nks = gridDim.y;
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            if (h >= d.G) continue;
            double* out = p.part + ((((size_t)row * d.n_obs + i) * 4 + h) * nks + blockIdx.y) * kPart;
            out[0] = mo[h].m; out[1] = mo[h].s0; out[2] = mo[h].t1;
            out[3] = mo[h].s2; out[4] = mo[h].s3; out[5] = mo[h].s4;
        }
    }
}

// ------------------------------------------------------------------ 2. per query
// One thread per (row, observation, head < G): merge the ranges in order, then
//   H = -(sum p ln p) / ln n,  v = n sum p^2 - 1,
//   m2 = (sum p^2 - c) / n,  m4 = (sum p^4 - 4c sum p^3 + 6c^2 sum p^2 - 3c^3) / n,
//   kappa = m4 / m2^2 - 3 (0 when m2 = 0),  c = 1/n, n = P + 1 keys.
// A central moment below the rounding noise of its expansion is taken as zero (the
// attention is uniform to working precision).
__global__ void prefill_query_kernel(const PrefillParams p, int nks) {
    const LayerDims& d = p.d;
    const size_t q = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t nq = (size_t)d.R * d.n_obs * 4;
    if (q >= nq) return;
    const int h = (int)(q % 4);
    const int i = (int)((q / 4) % d.n_obs);
    const int row = (int)(q / 4 / d.n_obs);
    if (h >= d.G) return;
    const int b = row / d.hkv, g = row - b * d.hkv;
    const double* part = p.part + q * nks * kPart;
    Moments a{-INFINITY, 0.0, 0.0, 0.0, 0.0, 0.0};
    for (int ks = 0; ks < nks; ++ks) {
        const double* x = part + (size_t)ks * kPart;
        a = moments_merge(a, Moments{x[0], x[1], x[2], x[3], x[4], x[5]});
    }
    const int n0 = min(p.ctx_len[b], p.n_stride);
    const double n = (double)(n0 - d.n_obs + i + 1);
    const double L = a.s0, il = 1.0 / L;
    const double lnL = log(L);
    const double sp2 = a.s2 * il * il, sp3 = a.s3 * (il * il * il), sp4 = a.s4 * ((il * il) * (il * il));
    const double c = 1.0 / n;
    const double H = n > 1.0 ? -(a.t1 * il - lnL) / log(n) : 0.0;
    const double v = n * sp2 - 1.0;
    constexpr double kNoise = 64.0 * 1.1102230246251565e-16;   // 64 units of rounding
    double m2 = (sp2 - c) / n;
    if (fabs(sp2 - c) <= kNoise * sp2) m2 = 0.0;
    double m4 = (sp4 - 4.0 * c * sp3 + 6.0 * c * c * sp2 - 3.0 * c * c * c) / n;
    if (fabs(m4) * n <= kNoise * (sp4 + 4.0 * c * sp3 + 6.0 * c * c * sp2 + 3.0 * c * c * c)) m4 = 0.0;
    const double kappa = m2 > 0.0 ? m4 / (m2 * m2) - 3.0 : 0.0;
    double* st = p.query_stats + (((size_t)b * d.hq + g * d.G + h) * d.n_obs + i) * 3;
    st[0] = H;
    st[1] = v;
    st[2] = kappa;
    p.qml[q * 2] = a.m;
    p.qml[q * 2 + 1] = L;
}

// ------------------------------------------------------------------ 3. initial scores
// A CTA owns keys [k0, k0 + kPfTile) of one row and walks the observation queries in
// order, 8 positions per step (one per warp); per step every key gets the
// observations of the positions that see it, applied in position order.
template <int D>
__global__ void __launch_bounds__(kPfThreads) prefill_observe_kernel(const PrefillParams p) {
    constexpr int SD = D + 1;
    const LayerDims& d = p.d;
    const int row = blockIdx.y, b = row / d.hkv, g = row - b * d.hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    extern __shared__ double smem[];
    double* sq = smem;                          // [32][SD]
    double* sk = sq + 32 * SD;                  // [kPfTile][SD]
    double* sx = sk + kPfTile * SD;             // [kPfPositions][kPfTile] observations

    const int n0 = min(p.ctx_len[b], p.n_stride);
    const int k0 = blockIdx.x * kPfTile;
    if (k0 >= n0) return;
    const uint16_t* krow = p.k + ((size_t)b * d.hkv + g) * p.n_stride * D;
    const double inv_sqrt_d = 1.0 / sqrt((double)D);
    load_key_tile<D>(sk, krow, k0, n0);
    double mu = 0.0, m2 = 0.0;                  // Welford state of key k0 + tid (tid < kPfTile)
    int cnt = 0;
    // the first position that sees key k0 + kPfTile - 1 is n0 - n_obs + i >= key; every
    // position before the first query tile that sees any key of the block is skipped
    const int i_first = max(0, k0 - (n0 - d.n_obs));
    for (int i0 = (i_first / kPfPositions) * kPfPositions; i0 < d.n_obs; i0 += kPfPositions) {
        __syncthreads();
        load_query_tile<D>(sq, p, b, g, i0);
        __syncthreads();
        double dot[4][2];
        tile_dots<D>(sq, sk, warp, lane, dot);
        const int i = i0 + warp, P = n0 - d.n_obs + i;
#pragma unroll
        for (int j = 0; j < 2; ++j) {
            const int key = k0 + lane + 32 * j;
            double x = -1.0;                    // marks "no observation"
            if (i < d.n_obs && key < n0 && key <= P) {
                x = 0.0;
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    if (h >= d.G) continue;
                    const double* ml = p.qml + (((size_t)row * d.n_obs + i) * 4 + h) * 2;
                    x += exp(dot[h][j] * inv_sqrt_d - ml[0]) / ml[1];
                }
            }
            sx[warp * kPfTile + lane + 32 * j] = x;
        }
        __syncthreads();
        if (tid < kPfTile) {
#pragma unroll
            for (int w = 0; w < kPfPositions; ++w) {
                const double x = sx[w * kPfTile + tid];
                if (x < 0.0) continue;
                ++cnt;
                const double dl = x - mu;
                mu += dl / cnt;
                m2 += dl * (x - mu);
            }
        }
    }
    const int key = k0 + tid;
    if (tid < kPfTile && key < n0) {
        p.mu0[(size_t)row * p.n_stride + key] = mu;
        p.m2_0[(size_t)row * p.n_stride + key] = m2;
    }
}

// Layer means of (H, v, kappa) over every (sequence, query head, observation), in a
// fixed order.
__global__ void prefill_layer_mean_kernel(const PrefillParams p) {
    const LayerDims& d = p.d;
    const size_t nq = (size_t)d.batch * d.hq * d.n_obs;
    __shared__ double part[3][256];
    double s[3] = {0.0, 0.0, 0.0};
    for (size_t q = threadIdx.x; q < nq; q += blockDim.x)
        for (int c = 0; c < 3; ++c) s[c] += p.query_stats[q * 3 + c];
    for (int c = 0; c < 3; ++c) part[c][threadIdx.x] = s[c];
    __syncthreads();
    for (int w = blockDim.x / 2; w >= 1; w >>= 1) {
        if ((int)threadIdx.x < w)
            for (int c = 0; c < 3; ++c) part[c][threadIdx.x] += part[c][threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x < 3) p.stats_out[threadIdx.x] = part[threadIdx.x][0] / (double)nq;
}

int key_ranges(int n_stride) { return (n_stride + kPfRange - 1) / kPfRange; }

}  // namespace

PrefillWs prefill_ws_layout(const LayerDims& d, int n_stride) {
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    const size_t nq = (size_t)d.R * d.n_obs * 4;
    PrefillWs w{};
    size_t off = 0;
    w.part = off;  off = al(off + sizeof(double) * nq * key_ranges(n_stride) * kPart);
    w.qml = off;   off = al(off + sizeof(double) * nq * 2);
    w.qstat = off; off = al(off + sizeof(double) * (size_t)d.batch * d.hq * d.n_obs * 3);
    w.keys = off;  off = al(off + sizeof(uint64_t) * (size_t)d.R * n_stride);
    w.idx = off;   off = al(off + sizeof(int32_t) * (size_t)d.R * n_stride);
    w.total = off;
    return w;
}

cudaError_t launch_prefill_stats(const PrefillParams& p, cudaStream_t s) {
    const LayerDims& d = p.d;
    const int nks = key_ranges(p.n_stride);
    const int SD = d.D + 1;
    const size_t dyn_sweep = sizeof(double) * ((size_t)32 * SD + (size_t)kPfTile * SD);
    const size_t dyn_obs = dyn_sweep + sizeof(double) * kPfPositions * kPfTile;
    static unsigned char done[4][64];
    const dim3 gsweep((d.n_obs + kPfPositions - 1) / kPfPositions, nks, d.R);
    const dim3 gobs((p.n_stride + kPfTile - 1) / kPfTile, d.R);
    cudaError_t e;
    if (d.D == 128) {
        if ((e = allow_max_dyn_smem(prefill_sweep_kernel<128>, done[0])) != cudaSuccess) return e;
        prefill_sweep_kernel<128><<<gsweep, kPfThreads, dyn_sweep, s>>>(p);
    } else {
        if ((e = allow_max_dyn_smem(prefill_sweep_kernel<64>, done[1])) != cudaSuccess) return e;
        prefill_sweep_kernel<64><<<gsweep, kPfThreads, dyn_sweep, s>>>(p);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const size_t nq = (size_t)d.R * d.n_obs * 4;
    prefill_query_kernel<<<(unsigned)((nq + 255) / 256), 256, 0, s>>>(p, nks);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if (d.D == 128) {
        if ((e = allow_max_dyn_smem(prefill_observe_kernel<128>, done[2])) != cudaSuccess) return e;
        prefill_observe_kernel<128><<<gobs, kPfThreads, dyn_obs, s>>>(p);
    } else {
        if ((e = allow_max_dyn_smem(prefill_observe_kernel<64>, done[3])) != cudaSuccess) return e;
        prefill_observe_kernel<64><<<gobs, kPfThreads, dyn_obs, s>>>(p);
    }
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    prefill_layer_mean_kernel<<<1, 256, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace arkv
