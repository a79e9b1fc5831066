// Prefill attention statistics and initial scores (ARKV, 기술요약 §2.가: per-layer
// Original:Quantization ratio from attention entropy, variance and kurtosis;
// §2.나: the scores start from the attention each token received in prefill).
//
// One CTA takes 8 observation positions x 4 head slots (32 queries) of one row
// and streams the row's keys twice in 128-key tiles staged in shared memory as
// float64: the first sweep forms each query's softmax max and sum, the second its
// probabilities, from which it accumulates sum p ln p, sum p^2 and the central
// moments, and each key's group-summed probability x_k(i).  Each lane owns 4 keys
// of a tile and the warp's 4 queries (a 4x4 register tile of float64 dot
// products).  Keys gather sum x and sum x^2 over all positions i through
// float64 atomics; a finishing kernel turns them into (mu, M2) and reduces the
// per-query statistics to the layer means in a fixed order.
#include <math.h>

#include "arkv_internal.cuh"

namespace arkv {

namespace {

constexpr int kPfThreads = 256;
constexpr int kPfPositions = 8;   // observation positions per CTA (one per warp)
constexpr int kPfTile = 128;      // keys per tile

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

template <int D>
__device__ __forceinline__ void tile_dots(const double* sq, const double* sk, int warp, int lane,
                                          double (&dot)[4][4]) {
    constexpr int SD = D + 1;
#pragma unroll
    for (int h = 0; h < 4; ++h)
#pragma unroll
        for (int j = 0; j < 4; ++j) dot[h][j] = 0.0;
    const double* q0 = sq + (warp * 4) * SD;
    const double* k0 = sk + lane * SD;
#pragma unroll 4
    for (int e = 0; e < D; ++e) {
        double qv[4], kv[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) qv[h] = q0[h * SD + e];
#pragma unroll
        for (int j = 0; j < 4; ++j) kv[j] = k0[j * 32 * SD + e];
#pragma unroll
        for (int h = 0; h < 4; ++h)
#pragma unroll
            for (int j = 0; j < 4; ++j) dot[h][j] = fma(qv[h], kv[j], dot[h][j]);
    }
}

template <int D>
__global__ void __launch_bounds__(kPfThreads) prefill_stats_kernel(const PrefillParams p) {
    constexpr int SD = D + 1;
    const LayerDims& d = p.d;
    const int row = blockIdx.y, b = row / d.hkv, g = row - b * d.hkv;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = d.G;
    extern __shared__ double smem[];
    double* sq = smem;                          // [32][SD]
    double* sk = sq + 32 * SD;                  // [kPfTile][SD]
    double* sx = sk + kPfTile * SD;             // [kPfTile][2] sum x, sum x^2 of this tile

    const int n0 = min(p.ctx_len[b], p.n_stride);
    const int i = blockIdx.x * kPfPositions + warp;          // observation index of this warp
    const bool wvalid = i < d.n_obs;
    const int P = n0 - d.n_obs + i;                          // its position
    const int i_last = min(d.n_obs, (int)(blockIdx.x + 1) * kPfPositions) - 1;
    const int kend = min(n0, n0 - d.n_obs + i_last + 1);     // keys any warp of the CTA sees
    const uint16_t* krow = p.k + ((size_t)b * d.hkv + g) * p.n_stride * D;
    const double inv_sqrt_d = 1.0 / sqrt((double)D);

    for (int w = tid; w < 32 * D; w += blockDim.x) {
        const int qi = w / D, e = w - qi * D;
        const int ww = qi / 4, h = qi - ww * 4;
        const int ii = blockIdx.x * kPfPositions + ww;
        double v = 0.0;
        if (h < G && ii < d.n_obs)
            v = bf16_to_f32(p.q_obs[(((size_t)b * d.hq + g * G + h) * d.n_obs + ii) * D + e]);
        sq[qi * SD + e] = v;
    }

    // sweep 1: softmax max and sum of each query
    double m[4], l[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) { m[h] = -INFINITY; l[h] = 0.0; }
    for (int kt = 0; kt < kend; kt += kPfTile) {
        __syncthreads();
        load_key_tile<D>(sk, krow, kt, kend);
        __syncthreads();
        double dot[4][4];
        tile_dots<D>(sq, sk, warp, lane, dot);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int key = kt + lane + 32 * j;
            if (!wvalid || key > P) continue;
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                if (h >= G) continue;
                const double s = dot[h][j] * inv_sqrt_d;
                if (s > m[h]) { l[h] = l[h] * exp(m[h] - s) + 1.0; m[h] = s; }
                else l[h] += exp(s - m[h]);
            }
        }
    }
#pragma unroll
    for (int h = 0; h < 4; ++h) {
#pragma unroll
        for (int msk = 16; msk >= 1; msk >>= 1) {
            const double mo = __shfl_xor_sync(0xffffffffu, m[h], msk);
            const double lo = __shfl_xor_sync(0xffffffffu, l[h], msk);
            const double mn = fmax(m[h], mo);
            if (mn == -INFINITY) continue;
            l[h] = (m[h] == -INFINITY ? 0.0 : l[h] * exp(m[h] - mn)) +
                   (mo == -INFINITY ? 0.0 : lo * exp(mo - mn));
            m[h] = mn;
        }
    }
    double lnl[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) lnl[h] = l[h] > 0 ? log(l[h]) : 0.0;
    const double n_keys = (double)(P + 1), inv_n = 1.0 / n_keys;

    // sweep 2: probabilities, per-query sums and per-key observations
    double splnp[4], sp2[4], sd2[4], sd4[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) { splnp[h] = sp2[h] = sd2[h] = sd4[h] = 0.0; }
    double* sumx = p.sumx + (size_t)row * p.n_stride * 2;
    for (int kt = 0; kt < kend; kt += kPfTile) {
        __syncthreads();
        load_key_tile<D>(sk, krow, kt, kend);
        for (int w = tid; w < kPfTile * 2; w += blockDim.x) sx[w] = 0.0;
        __syncthreads();
        double dot[4][4];
        tile_dots<D>(sq, sk, warp, lane, dot);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int key = kt + lane + 32 * j;
            if (!wvalid || key > P) continue;
            double x = 0.0;
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                if (h >= G) continue;
                const double a = dot[h][j] * inv_sqrt_d - m[h];
                const double pr = exp(a) / l[h];
                splnp[h] += pr * (a - lnl[h]);
                sp2[h] += pr * pr;
                const double dl = pr - inv_n;
                const double dl2 = dl * dl;
                sd2[h] += dl2;
                sd4[h] += dl2 * dl2;
                x += pr;
            }
            atomicAdd(&sx[(lane + 32 * j) * 2], x);
            atomicAdd(&sx[(lane + 32 * j) * 2 + 1], x * x);
        }
        __syncthreads();
        for (int kk = tid; kk < kPfTile; kk += blockDim.x) {
            const int key = kt + kk;
            if (key < kend) {
                atomicAdd(&sumx[(size_t)key * 2], sx[kk * 2]);
                atomicAdd(&sumx[(size_t)key * 2 + 1], sx[kk * 2 + 1]);
            }
        }
    }
#pragma unroll
    for (int h = 0; h < 4; ++h) {
#pragma unroll
        for (int msk = 16; msk >= 1; msk >>= 1) {
            splnp[h] += __shfl_xor_sync(0xffffffffu, splnp[h], msk);
            sp2[h] += __shfl_xor_sync(0xffffffffu, sp2[h], msk);
            sd2[h] += __shfl_xor_sync(0xffffffffu, sd2[h], msk);
            sd4[h] += __shfl_xor_sync(0xffffffffu, sd4[h], msk);
        }
    }
    if (lane == 0 && wvalid) {
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            if (h >= G) continue;
            const double H = n_keys > 1 ? -splnp[h] / log(n_keys) : 0.0;
            const double v = n_keys * sp2[h] - 1.0;
            const double m2 = sd2[h] * inv_n, m4 = sd4[h] * inv_n;
            const double kappa = m2 > 0 ? m4 / (m2 * m2) - 3.0 : 0.0;
            double* out = p.query_stats + (((size_t)b * d.hq + g * G + h) * d.n_obs + i) * 3;
            out[0] = H;
            out[1] = v;
            out[2] = kappa;
        }
    }
}

// mu0, M2_0 of every prefill key from sum x and sum x^2 of its observations.
__global__ void prefill_welford_kernel(const PrefillParams p) {
    const LayerDims& d = p.d;
    const int row = blockIdx.y, b = row / d.hkv;
    const int n0 = min(p.ctx_len[b], p.n_stride);
    const double* sumx = p.sumx + (size_t)row * p.n_stride * 2;
    for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < n0; k += gridDim.x * blockDim.x) {
        const int cnt = min(d.n_obs, n0 - k);
        const double sx = sumx[(size_t)k * 2], sx2 = sumx[(size_t)k * 2 + 1];
        const double mu = sx / cnt;
        const double m2 = fmax(sx2 - sx * mu, 0.0);
        p.mu0[(size_t)row * p.n_stride + k] = mu;
        p.m2_0[(size_t)row * p.n_stride + k] = m2;
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

}  // namespace

size_t prefill_ws_bytes(const LayerDims& d, int n_stride) {
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    return al(sizeof(double) * (size_t)d.R * n_stride * 2) +
           al(sizeof(double) * (size_t)d.batch * d.hq * d.n_obs * 3) +
           al(sizeof(uint32_t) * (size_t)d.R * n_stride) + al(sizeof(int32_t) * (size_t)d.R * n_stride);
}

cudaError_t launch_prefill_stats(const PrefillParams& p, cudaStream_t s) {
    const LayerDims& d = p.d;
    cudaError_t e = cudaMemsetAsync(p.sumx, 0, sizeof(double) * (size_t)d.R * p.n_stride * 2, s);
    if (e != cudaSuccess) return e;
    const dim3 grid((d.n_obs + kPfPositions - 1) / kPfPositions, d.R);
    const int SD = d.D + 1;
    const size_t dyn = sizeof(double) * ((size_t)32 * SD + (size_t)kPfTile * SD + kPfTile * 2);
    static unsigned char done128[64], done64[64];
    if (d.D == 128) {
        e = allow_max_dyn_smem(prefill_stats_kernel<128>, done128);
        if (e != cudaSuccess) return e;
        prefill_stats_kernel<128><<<grid, kPfThreads, dyn, s>>>(p);
    } else {
        e = allow_max_dyn_smem(prefill_stats_kernel<64>, done64);
        if (e != cudaSuccess) return e;
        prefill_stats_kernel<64><<<grid, kPfThreads, dyn, s>>>(p);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    prefill_welford_kernel<<<dim3(64, d.R), 256, 0, s>>>(p);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    prefill_layer_mean_kernel<<<1, 256, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace arkv
