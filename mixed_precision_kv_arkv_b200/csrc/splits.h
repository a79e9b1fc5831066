// How one arkv_decode_attn call shares a row's 16-token tiles: among the CTAs of the
// row, then among the 4 warps of a CTA.  Plain integer arithmetic, compiled for the
// device (the decode kernel) and for the host (the CPU tests check that every split
// partitions the tiles and balances the ring entries).  A bf16 tile is two ring
// entries (its K, then its V), an FP8 tile one.
#pragma once

#if defined(__CUDACC__)
#define ARKV_HD __host__ __device__ __forceinline__
#else
#define ARKV_HD inline
#endif

namespace arkv {

constexpr int kSplitWarps = 4;   // warps of a decode CTA

// The FP8 tiles before CTA c of a row split over n CTAs (T16 bf16 and T8 FP8 tiles;
// CTA c takes bf16 tiles [floor(T16 c / n), floor(T16 (c + 1) / n)) and FP8 tiles
// [F(c), F(c + 1))).  F(c) = round(T8 c / n + 2 frac(T16 c / n)): the FP8 share is
// shifted by up to two tiles so that the CTAs' ring entries differ by at most one.
// F grows with c when T8 >= 2n; below that the plain split floor(T8 c / n) is used.
// F(0) = 0 and F(n) = T8 either way.
ARKV_HD int fp8_tiles_before(long long T16, long long T8, long long n, long long c) {
    if (T8 < 2 * n) return (int)(T8 * c / n);
    return (int)((2 * T8 * c + 4 * ((T16 * c) % n) + n) / (2 * n));
}

// This warp's FP8 tiles among its CTA's L8: a contiguous run [*start, *start + *count).
// The bf16 tiles are dealt round robin (warp v gets ceil((L16 - v) / 4) of them); the
// FP8 tiles then level the warps' entry counts: first the warps one bf16 tile short,
// then all four evenly, so that no two warps differ by more than one entry whenever L8
// allows it.  Every warp computes the same split, so the runs partition the L8 tiles.
ARKV_HD void warp_fp8_share(int L16, int L8, int warp, int* start, int* count) {
    constexpr int W = kSplitWarps;
    int b[W], f[W];
#pragma unroll
    for (int v = 0; v < W; ++v) b[v] = L16 > v ? 2 * ((L16 - v + W - 1) / W) : 0;
    const int hi = b[0], lo = b[W - 1];   // b is non-increasing, hi - lo is 0 or 2
    int nlo = 0;
#pragma unroll
    for (int v = 0; v < W; ++v) nlo += b[v] == lo ? 1 : 0;   // the last nlo warps
    const int gap = (hi - lo) * nlo;
    if (L8 <= gap) {   // only the low warps take FP8 tiles
#pragma unroll
        for (int v = 0; v < W; ++v) {
            const int j = v - (W - nlo);
            f[v] = j < 0 ? 0 : L8 / nlo + (j < L8 % nlo ? 1 : 0);
        }
    } else {
        const int rest = L8 - gap;
#pragma unroll
        for (int v = 0; v < W; ++v) f[v] = (b[v] == lo ? hi - lo : 0) + rest / W + (v < rest % W ? 1 : 0);
    }
    int s0 = 0, cnt = 0;   // (selects, not an indexed load: the arrays stay in registers)
#pragma unroll
    for (int v = 0; v < W; ++v) {
        s0 += v < warp ? f[v] : 0;
        cnt = v == warp ? f[v] : cnt;
    }
    *start = s0;
    *count = cnt;
}

}  // namespace arkv
