// Tier selection and cache compaction (ARKV, 기술요약 §2.다: tri-state assignment
// under a memory budget with a protected window of the W newest tokens).
//
// One 1024-thread CTA per row.  Candidate tokens (live tokens older than the
// window) get a 64-bit order-preserving key of their float64 score
// S = mu + gamma*M2/n (0 marks a non-candidate).  Two MSB-first radix selections
// (8-bit digits, shared-memory histograms) find the n_sel-th best candidate and
// the n_o-th best kept bf16 token; equal scores are ordered by position through a
// second radix pass on the position.  The keys live in shared memory when they
// fit, otherwise in a global workspace (L2-resident).
//
// Compaction is in place: in each segment the survivors that sit above the new
// live count move into the vacated slots below it (k-th source -> k-th hole, both
// in slot order), and demoted bf16 tokens are quantized straight into vacated or
// new fp8 slots, so a reassignment moves O(changes) bytes, not the cache.
#include <math.h>

#include "arkv_internal.cuh"

namespace arkv {

namespace {

constexpr int kSmemKeyLimit = 24 * 1024;   // 8-byte keys kept in shared memory up to this many slots

constexpr int kCand = 2048;                 // candidate list of a radix selection, once it is this small

struct RowShared {
    unsigned hist[256];
    int warp_sum[33];
    int sel[4];
    int misc[16];
    int ncand;
    int cand[kCand];
};

// ------------------------------------------------------------------ block helpers
__device__ __forceinline__ int block_sum(int v, RowShared& sh) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
    __syncthreads();
    if (lane == 0) sh.warp_sum[warp] = v;
    __syncthreads();
    int t = 0;
    const int nw = blockDim.x >> 5;
    for (int w = 0; w < nw; ++w) t += sh.warp_sum[w];
    __syncthreads();
    return t;
}

// Calls f(i, rank) for every i in [begin, end) with pred(i), rank = number of
// earlier such i.  Returns the count.  All threads must call it.  Each warp owns a
// contiguous chunk of the range: it counts its chunk (ballots), one block scan of
// the warps' counts gives every warp its first rank, and a second walk over the
// chunk emits in order.
template <class Pred, class F>
__device__ int block_enumerate(int begin, int end, Pred pred, F f, RowShared& sh) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    const int n = max(end - begin, 0);
    const int chunk = (((n + nw - 1) / nw) + 31) & ~31;
    const int c0 = begin + warp * chunk, c1 = min(c0 + chunk, end);
    int cnt = 0;
    for (int i0 = c0; i0 < c1; i0 += 32) {
        const int i = i0 + lane;
        cnt += __popc(__ballot_sync(0xffffffffu, i < c1 && pred(i)));
    }
    __syncthreads();                       // earlier users of warp_sum are done
    if (lane == 0) sh.warp_sum[warp] = cnt;
    __syncthreads();
    if (warp == 0) {
        const int v = lane < nw ? sh.warp_sum[lane] : 0;
        int x = v;
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, m);
            if (lane >= m) x += y;
        }
        sh.warp_sum[lane] = x - v;         // exclusive
        if (lane == 31) sh.warp_sum[32] = x;
    }
    __syncthreads();
    int off = sh.warp_sum[warp];
    const int total = sh.warp_sum[32];
    for (int i0 = c0; i0 < c1; i0 += 32) {
        const int i = i0 + lane;
        const bool fl = i < c1 && pred(i);
        const unsigned bal = __ballot_sync(0xffffffffu, fl);
        if (fl) f(i, off + __popc(bal & ((1u << lane) - 1u)));
        off += __popc(bal);
    }
    __syncthreads();
    return total;
}

template <class Pred>
__device__ int block_count(int begin, int end, Pred pred, RowShared& sh) {
    int c = 0;
    for (int i = begin + threadIdx.x; i < end; i += blockDim.x) c += pred(i) ? 1 : 0;
    return block_sum(c, sh);
}

// Selection of the k best eligible elements by (key descending, position
// ascending).  Element i is selected iff key(i) > cut, or key(i) == cut and
// (all_ties or pos(i) <= pos_max).
struct Sel {
    uint64_t cut;
    int all_ties;
    int pos_max;
};

__device__ __forceinline__ bool sel_in(const Sel& s, uint64_t key, int pos) {
    return key > s.cut || (key == s.cut && (s.all_ties || pos <= s.pos_max));
}

// One histogram update per group of lanes holding the same digit.
__device__ __forceinline__ void hist_add(unsigned* hist, bool valid, unsigned digit) {
    const unsigned peers = __match_any_sync(0xffffffffu, valid ? digit : 0x100u);
    if (valid && (threadIdx.x & 31) == (unsigned)(__ffs(peers) - 1)) atomicAdd(&hist[digit], (unsigned)__popc(peers));
}

// k-th largest key (of unsigned type KT) among eligible elements (1 <= k <= count):
// returns cut and, through need/eq, how many of the elements equal to cut are
// taken / exist.  8-bit digits from the top; once the elements that share the
// prefix found so far number at most kCand, they are gathered into a list and the
// remaining digits are taken over the list only.
template <class KT, class KeyF, class Elig>
__device__ KT radix_kth(KeyF key, Elig elig, int n, int k, int* need, int* eq, RowShared& sh) {
    KT prefix = 0, pmask = 0;
    int kk = k, last_eq = 0, nl = -1;       // nl >= 0: the candidates are listed
    for (int shift = 8 * (int)sizeof(KT) - 8; shift >= 0; shift -= 8) {
        for (int i = threadIdx.x; i < 256; i += blockDim.x) sh.hist[i] = 0;
        __syncthreads();
        if (nl < 0) {
            for (int base = 0; base < n; base += blockDim.x) {
                const int i = base + threadIdx.x;
                bool v = i < n && elig(i);
                KT kv = 0;
                if (v) { kv = key(i); v = (kv & pmask) == prefix; }
                hist_add(sh.hist, v, (unsigned)(kv >> shift) & 255u);
            }
        } else {
            for (int base = 0; base < nl; base += blockDim.x) {
                const int j = base + threadIdx.x;
                bool v = j < nl;
                KT kv = 0;
                if (v) { kv = key(sh.cand[j]); v = (kv & pmask) == prefix; }
                hist_add(sh.hist, v, (unsigned)(kv >> shift) & 255u);
            }
        }
        __syncthreads();
        if (threadIdx.x < 32) {
            const int lane = threadIdx.x;
            // lane covers bins 255-8*lane down to 248-8*lane (descending)
            int cnt[8], s = 0;
#pragma unroll
            for (int j = 0; j < 8; ++j) {
                cnt[j] = (int)sh.hist[255 - 8 * lane - j];
                s += cnt[j];
            }
            int incl = s;
#pragma unroll
            for (int m = 1; m < 32; m <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, incl, m);
                if (lane >= m) incl += y;
            }
            const int excl = incl - s;
            if (excl < kk && kk <= incl) {
                int above = excl;
#pragma unroll
                for (int j = 0; j < 8; ++j) {
                    if (above < kk && kk <= above + cnt[j]) {
                        sh.sel[0] = 255 - 8 * lane - j;
                        sh.sel[1] = above;
                        sh.sel[2] = cnt[j];
                    }
                    above += cnt[j];
                }
            }
            if (lane == 0) sh.ncand = 0;
        }
        __syncthreads();
        const KT bin = (KT)sh.sel[0];
        kk -= sh.sel[1];
        last_eq = sh.sel[2];
        prefix |= bin << shift;
        pmask |= (KT)0xff << shift;
        if (nl < 0 && shift > 0 && last_eq <= kCand) {
            // gather the elements that share the prefix (any order: only counts follow)
            for (int base = 0; base < n; base += blockDim.x) {
                const int i = base + threadIdx.x;
                const bool v = i < n && elig(i) && (key(i) & pmask) == prefix;
                const unsigned bal = __ballot_sync(0xffffffffu, v);
                int slot0 = 0;
                if ((threadIdx.x & 31) == 0 && bal) slot0 = atomicAdd(&sh.ncand, __popc(bal));
                slot0 = __shfl_sync(0xffffffffu, slot0, 0);
                if (v) sh.cand[slot0 + __popc(bal & ((1u << (threadIdx.x & 31)) - 1u))] = i;
            }
            __syncthreads();
            nl = sh.ncand;
        }
        __syncthreads();
    }
    *need = kk;
    *eq = last_eq;
    return prefix;
}

// The k best eligible elements by (key desc, pos asc).  n_elig = number eligible.
template <class KeyF, class PosF, class Elig>
__device__ Sel select_best(KeyF key, PosF pos, Elig elig, int n, int k, int n_elig, RowShared& sh) {
    Sel s;
    if (k <= 0) {
        s.cut = ~0ull; s.all_ties = 0; s.pos_max = -1;
        return s;
    }
    if (k >= n_elig) {
        s.cut = 0ull; s.all_ties = 1; s.pos_max = 0;
        return s;
    }
    int need, eq;
    s.cut = radix_kth<uint64_t>(key, elig, n, k, &need, &eq, sh);
    s.all_ties = need >= eq;
    s.pos_max = 0;
    if (!s.all_ties) {
        const uint64_t cut = s.cut;
        int need2, eq2;
        const uint32_t c2 = radix_kth<uint32_t>([&](int i) { return ~(uint32_t)pos(i); },
                                                [&](int i) { return elig(i) && key(i) == cut; }, n, need,
                                                &need2, &eq2, sh);
        s.pos_max = (int)~c2;
    }
    return s;
}

// ------------------------------------------------------------------ data movement
template <int D>
__device__ __forceinline__ void warp_copy_bf16_row(uint16_t* dst, const uint16_t* src) {
    const int lane = threadIdx.x & 31;
    constexpr int W = D * 2 / 16;   // 16-byte words per row
    for (int w = lane; w < W; w += 32)
        reinterpret_cast<uint4*>(dst)[w] = reinterpret_cast<const uint4*>(src)[w];
}

template <int D>
__device__ __forceinline__ void warp_copy_fp8_row(uint8_t* dst, const uint8_t* src) {
    const int lane = threadIdx.x & 31;
    constexpr int W = D / 8;   // 8-byte words per row
    for (int w = lane; w < W; w += 32)
        reinterpret_cast<uint2*>(dst)[w] = reinterpret_cast<const uint2*>(src)[w];
}

// Quantize one bf16 row (D elements) held in global memory into codes + scale, in
// the layer's FP8 format.
template <int D>
__device__ __forceinline__ float warp_quantize_row(const uint16_t* src, uint8_t* dst, int fmt) {
    constexpr int EPL = D / 32;
    const int lane = threadIdx.x & 31;
    float x[EPL];
#pragma unroll
    for (int e = 0; e < EPL; ++e) x[e] = bf16_to_f32(src[lane * EPL + e]);
    uint8_t c[EPL];
    const float s = fmt == ARKV_FMT_E5M2 ? quantize_warp<EPL, ARKV_FMT_E5M2>(x, c)
                                         : quantize_warp<EPL, ARKV_FMT_E4M3>(x, c);
#pragma unroll
    for (int e = 0; e < EPL; ++e) dst[lane * EPL + e] = c[e];
    return s;
}

// ------------------------------------------------------------------ reassignment
constexpr int kKeyBatch = 8;   // slots per thread whose loads are in flight together (key build)

// Slot outcomes, frozen before any data moves.
constexpr uint64_t kStayBf16 = 0, kDemote = 1, kEvict = 2, kStayFp8 = 3;

template <int D>
__global__ void __launch_bounds__(kRowThreads) reassign_kernel(const ReassignParams p) {
    const LayerDims& d = p.d;
    const int row = blockIdx.x, b = row / d.hkv;
    const int tid = threadIdx.x, warp = tid >> 5, nwarps = blockDim.x >> 5;
    __shared__ RowShared sh;
    extern __shared__ uint64_t sm_keys[];

    const int n16 = min(max(p.c.n_bf16[row], 0), d.cap_o);
    const int n8 = min(max(p.c.n_fp8[row], 0), d.cap_q);
    const int n = n16 + n8;
    const int n0 = p.ctx_len[b];
    const int nt = n0 + p.step + 1;
    const int winlo = nt - d.W;
    const size_t slots = (size_t)(d.cap_o + d.cap_q);
    const size_t b16 = (size_t)row * d.cap_o, b8 = (size_t)row * d.cap_q;
    uint64_t* keys = (slots <= (size_t)kSmemKeyLimit) ? sm_keys : p.key_ws + (size_t)row * slots;
    int32_t* src_list = p.idx_ws + (size_t)row * 2 * slots;   // [slots]
    int32_t* hole_list = src_list + slots;                    // [slots]

    auto pos_of = [&](int i) -> int { return i < n16 ? p.c.pos16[b16 + i] : p.c.pos8[b8 + (i - n16)]; };

    // keys: 0 for window tokens (never candidates), order-preserving map of S otherwise.
    // kKeyBatch slots per thread at a time, all their loads issued before any of them is
    // used, so that the row's ~n / 1024 memory latencies per thread overlap
    int ncand = 0;
    for (int base = 0; base < n; base += kKeyBatch * (int)blockDim.x) {
        int pos[kKeyBatch];
        double mu[kKeyBatch], m2[kKeyBatch];
#pragma unroll
        for (int u = 0; u < kKeyBatch; ++u) {
            const int i = base + u * (int)blockDim.x + tid;
            const bool bf = i < n16;
            const size_t sl = bf ? b16 + i : b8 + (i - n16);
            const bool in = i < n;
            pos[u] = in ? (bf ? p.c.pos16[sl] : p.c.pos8[sl]) : 0;
            mu[u] = in ? (bf ? p.c.mu16[sl] : p.c.mu8[sl]) : 0.0;
            m2[u] = in ? (bf ? p.c.m2_16[sl] : p.c.m2_8[sl]) : 0.0;
        }
#pragma unroll
        for (int u = 0; u < kKeyBatch; ++u) {
            const int i = base + u * (int)blockDim.x + tid;
            if (i >= n) break;
            uint64_t key = 0;
            if (i >= n16 || pos[u] < winlo) {
                key = double_key(score_f64(mu[u], m2[u], obs_count_after(pos[u], n0, p.step, d.n_obs), d.gamma));
                ++ncand;
            }
            keys[i] = key;
        }
    }
    ncand = block_sum(ncand, sh);
    if (tid == 0) {
        int n_sel, n_o;
        budget_counts(d.beta, nt, p.r, d.D, d.W, ncand, &n_sel, &n_o);
        sh.misc[0] = n_sel;
        sh.misc[1] = n_o;
    }
    __syncthreads();
    const int n_sel = sh.misc[0], n_o = sh.misc[1];

    auto keyf = [&](int i) -> uint64_t { return keys[i]; };
    const Sel keep = select_best(keyf, pos_of, [&](int i) { return keys[i] != 0u; }, n, n_sel,
                                 ncand, sh);
    auto kept = [&](int i) -> bool {
        const uint64_t k = keys[i];
        return k != 0u && sel_in(keep, k, k == keep.cut ? pos_of(i) : 0);
    };
    auto kept16 = [&](int i) -> bool { return i < n16 && kept(i); };
    const int n_kept16 = block_count(0, n16, kept16, sh);
    const Sel orig = select_best(keyf, pos_of, kept16, n, min(n_o, n_kept16), n_kept16, sh);

    // freeze the outcome of every slot
    for (int i = tid; i < n; i += blockDim.x) {
        const uint64_t k = keys[i];
        uint64_t st;
        if (i < n16) {
            if (k == 0u) {
                st = kStayBf16;   // window
            } else {
                const int pos = (k == keep.cut || k == orig.cut) ? pos_of(i) : 0;
                const bool kp = sel_in(keep, k, pos);
                st = !kp ? kEvict : (sel_in(orig, k, pos) ? kStayBf16 : kDemote);
            }
        } else {
            st = sel_in(keep, k, k == keep.cut ? pos_of(i) : 0) ? kStayFp8 : kEvict;
        }
        keys[i] = st;
    }
    __syncthreads();
    auto is_stay16 = [&](int i) { return keys[i] == kStayBf16; };
    auto is_demote = [&](int i) { return keys[i] == kDemote; };
    auto is_stay8 = [&](int j) { return keys[n16 + j] == kStayFp8; };

    const int n16_new = block_count(0, n16, is_stay16, sh);
    const int n8_stay = block_count(0, n8, is_stay8, sh);
    int n_dem = block_count(0, n16, is_demote, sh);
    if (n8_stay + n_dem > d.cap_q) {          // demotions past the fp8 capacity are evicted
        n_dem = d.cap_q - n8_stay;
        if (tid == 0) atomicOr(p.c.status, ARKV_STATUS_FP8_FULL);
    }
    const int n8_new = n8_stay + n_dem;

    // debug tiers: demotions are reported where they are enumerated below (the ones
    // past the fp8 capacity become evictions)
    uint8_t* td = p.tier_dbg ? p.tier_dbg + (size_t)row * slots : nullptr;
    if (td) {
        for (int i = tid; i < n16; i += blockDim.x) {
            const uint64_t st = keys[i];
            if (st != kDemote) td[i] = st == kStayBf16 ? ARKV_TIER_ORIGINAL : ARKV_TIER_EVICTED;
        }
        for (int j = tid; j < n8; j += blockDim.x)
            td[d.cap_o + j] = keys[n16 + j] == kStayFp8 ? ARKV_TIER_QUANTIZED : ARKV_TIER_EVICTED;
    }

    // ---------------- fp8 segment: vacated slots below n8_new (then new slots up to
    // n8_new) receive, in order, the survivors above n8_new and the demoted tokens
    const int lo8 = min(n8, n8_new);
    const int nh8 = block_enumerate(0, lo8, [&](int j) { return !is_stay8(j); },
                                    [&](int j, int r) { hole_list[r] = j; }, sh);
    for (int j = n8 + tid; j < n8_new; j += blockDim.x) hole_list[nh8 + (j - n8)] = j;
    const int n_mov8 = block_enumerate(n8_new, n8, is_stay8, [&](int j, int r) { src_list[r] = j; }, sh);
    __syncthreads();
    for (int r = warp; r < n_mov8; r += nwarps) {
        const int src = src_list[r], dst = hole_list[r];
        warp_copy_fp8_row<D>(p.c.k8 + (b8 + dst) * D, p.c.k8 + (b8 + src) * D);
        warp_copy_fp8_row<D>(p.c.v8 + (b8 + dst) * D, p.c.v8 + (b8 + src) * D);
        if ((tid & 31) == 0) {
            p.c.sk[b8 + dst] = p.c.sk[b8 + src];
            p.c.sv[b8 + dst] = p.c.sv[b8 + src];
            p.c.pos8[b8 + dst] = p.c.pos8[b8 + src];
            p.c.mu8[b8 + dst] = p.c.mu8[b8 + src];
            p.c.m2_8[b8 + dst] = p.c.m2_8[b8 + src];
        }
    }
    __syncthreads();
    block_enumerate(0, n16, is_demote, [&](int i, int r) {
        src_list[r] = i;
        if (td) td[i] = r < n_dem ? ARKV_TIER_QUANTIZED : ARKV_TIER_EVICTED;
    }, sh);
    __syncthreads();
    for (int r = warp; r < n_dem; r += nwarps) {
        const int src = src_list[r], dst = hole_list[n_mov8 + r];
        const float skv = warp_quantize_row<D>(p.c.k16 + (b16 + src) * D, p.c.k8 + (b8 + dst) * D, d.fmt);
        const float svv = warp_quantize_row<D>(p.c.v16 + (b16 + src) * D, p.c.v8 + (b8 + dst) * D, d.fmt);
        if ((tid & 31) == 0) {
            p.c.sk[b8 + dst] = skv;
            p.c.sv[b8 + dst] = svv;
            p.c.pos8[b8 + dst] = p.c.pos16[b16 + src];
            p.c.mu8[b8 + dst] = p.c.mu16[b16 + src];
            p.c.m2_8[b8 + dst] = p.c.m2_16[b16 + src];
        }
    }
    __syncthreads();

    // ---------------- bf16 segment: survivors above n16_new move into the vacated
    // slots below it (demoted tokens have been read above)
    block_enumerate(0, n16_new, [&](int i) { return !is_stay16(i); },
                    [&](int i, int r) { hole_list[r] = i; }, sh);
    const int n_mov16 = block_enumerate(n16_new, n16, is_stay16, [&](int i, int r) { src_list[r] = i; }, sh);
    __syncthreads();
    for (int r = warp; r < n_mov16; r += nwarps) {
        const int src = src_list[r], dst = hole_list[r];
        warp_copy_bf16_row<D>(p.c.k16 + (b16 + dst) * D, p.c.k16 + (b16 + src) * D);
        warp_copy_bf16_row<D>(p.c.v16 + (b16 + dst) * D, p.c.v16 + (b16 + src) * D);
        if ((tid & 31) == 0) {
            p.c.pos16[b16 + dst] = p.c.pos16[b16 + src];
            p.c.mu16[b16 + dst] = p.c.mu16[b16 + src];
            p.c.m2_16[b16 + dst] = p.c.m2_16[b16 + src];
        }
    }
    __syncthreads();
    if (tid == 0) {
        p.c.n_bf16[row] = n16_new;
        p.c.n_fp8[row] = n8_new;
    }
}

// ------------------------------------------------------------------ initial pack
template <int D>
__global__ void __launch_bounds__(kRowThreads) pack_kernel(const PackParams p) {
    const LayerDims& d = p.d;
    const int row = blockIdx.x, b = row / d.hkv, g = row - b * d.hkv;
    const int tid = threadIdx.x, warp = tid >> 5, nwarps = blockDim.x >> 5;
    __shared__ RowShared sh;
    extern __shared__ uint64_t sm_keys[];

    const int n0 = min(p.ctx_len[b], p.n_stride);
    const int winlo = n0 - d.W;
    const size_t src_row = ((size_t)b * d.hkv + g) * p.n_stride;
    const size_t b16 = (size_t)row * d.cap_o, b8 = (size_t)row * d.cap_q;
    uint64_t* keys = (p.n_stride <= kSmemKeyLimit) ? sm_keys : p.key_ws + (size_t)row * p.n_stride;
    int32_t* rank = p.idx_ws + (size_t)row * p.n_stride;

    int ncand = 0;
    for (int i = tid; i < n0; i += blockDim.x) {
        uint64_t key = 0;
        if (i < winlo) {
            key = double_key(score_f64(p.mu0[src_row + i], p.m2_0[src_row + i],
                                       obs_count_after(i, n0, -1, d.n_obs), d.gamma));
            ++ncand;
        }
        keys[i] = key;
    }
    ncand = block_sum(ncand, sh);
    if (tid == 0) {
        int n_sel, n_o;
        budget_counts(d.beta, n0, p.r, d.D, d.W, ncand, &n_sel, &n_o);
        sh.misc[0] = n_sel;
        sh.misc[1] = n_o;
    }
    __syncthreads();
    const int n_sel = sh.misc[0], n_o = sh.misc[1];
    auto keyf = [&](int i) -> uint64_t { return keys[i]; };
    auto posf = [&](int i) -> int { return i; };
    const Sel keep = select_best(keyf, posf, [&](int i) { return keys[i] != 0u; }, n0, n_sel, ncand, sh);
    auto kept = [&](int i) -> bool { return keys[i] != 0u && sel_in(keep, keys[i], i); };
    const Sel orig = select_best(keyf, posf, kept, n0, n_o, n_sel, sh);
    auto is_o = [&](int i) -> bool { return keys[i] == 0u || (kept(i) && sel_in(orig, keys[i], i)); };
    auto is_q = [&](int i) -> bool { return kept(i) && !sel_in(orig, keys[i], i); };

    // slot of every token: rank among its tier, in position order
    const int c16 = block_enumerate(0, n0, is_o, [&](int i, int r) { rank[i] = r; }, sh);
    const int c8 = block_enumerate(0, n0, is_q, [&](int i, int r) { rank[i] = r; }, sh);
    const bool over16 = c16 > d.cap_o, over8 = c8 > d.cap_q;
    if (tid == 0 && (over16 || over8))
        atomicOr(p.c.status, over16 ? ARKV_STATUS_BF16_FULL : ARKV_STATUS_FP8_FULL);
    __syncthreads();
    if (p.tier_out) {
        uint8_t* to = p.tier_out + (size_t)row * p.n_stride;
        for (int i = tid; i < n0; i += blockDim.x)
            to[i] = is_o(i) ? ARKV_TIER_ORIGINAL : (is_q(i) ? ARKV_TIER_QUANTIZED : ARKV_TIER_EVICTED);
    }
    for (int i = warp; i < n0; i += nwarps) {
        const uint64_t k = keys[i];
        const bool o = k == 0u || (k != 0u && sel_in(keep, k, i) && sel_in(orig, k, i));
        const bool q = !o && k != 0u && sel_in(keep, k, i);
        if (!o && !q) continue;
        const int r = rank[i];
        const uint16_t* ks = p.k + (src_row + i) * D;
        const uint16_t* vs = p.v + (src_row + i) * D;
        if (o) {
            if (r >= d.cap_o) continue;
            warp_copy_bf16_row<D>(p.c.k16 + (b16 + r) * D, ks);
            warp_copy_bf16_row<D>(p.c.v16 + (b16 + r) * D, vs);
            if ((tid & 31) == 0) {
                p.c.pos16[b16 + r] = i;
                p.c.mu16[b16 + r] = p.mu0[src_row + i];
                p.c.m2_16[b16 + r] = p.m2_0[src_row + i];
            }
        } else {
            if (r >= d.cap_q) continue;
            const float skv = warp_quantize_row<D>(ks, p.c.k8 + (b8 + r) * D, d.fmt);
            const float svv = warp_quantize_row<D>(vs, p.c.v8 + (b8 + r) * D, d.fmt);
            if ((tid & 31) == 0) {
                p.c.sk[b8 + r] = skv;
                p.c.sv[b8 + r] = svv;
                p.c.pos8[b8 + r] = i;
                p.c.mu8[b8 + r] = p.mu0[src_row + i];
                p.c.m2_8[b8 + r] = p.m2_0[src_row + i];
            }
        }
    }
    if (tid == 0) {
        p.c.n_bf16[row] = min(c16, d.cap_o);
        p.c.n_fp8[row] = min(c8, d.cap_q);
    }
}

template <int FMT>
__global__ void fp8_encode_kernel(const float* x, uint8_t* out, size_t n) {
    constexpr __nv_fp8_interpretation_t kInterp = FMT == ARKV_FMT_E5M2 ? __NV_E5M2 : __NV_E4M3;
    const size_t i = ((size_t)blockIdx.x * blockDim.x + threadIdx.x) * 2;
    if (i + 1 < n) {
        const __nv_fp8x2_storage_t c = __nv_cvt_float2_to_fp8x2(make_float2(x[i], x[i + 1]), __NV_SATFINITE, kInterp);
        out[i] = (uint8_t)(c & 0xff);
        out[i + 1] = (uint8_t)(c >> 8);
    } else if (i < n) {
        const __nv_fp8x2_storage_t c = __nv_cvt_float2_to_fp8x2(make_float2(x[i], 0.f), __NV_SATFINITE, kInterp);
        out[i] = (uint8_t)(c & 0xff);
    }
}

unsigned char g_smem_reassign128[64], g_smem_reassign64[64], g_smem_pack128[64], g_smem_pack64[64];

}  // namespace

size_t reassign_ws_bytes(const LayerDims& d) {
    const size_t per_row = (size_t)(d.cap_o + d.cap_q);
    const size_t keys = (d.cap_o + d.cap_q <= kSmemKeyLimit) ? 0 : per_row * 8 * d.R;
    return ((per_row * 2 * 4 * d.R + 255) & ~(size_t)255) + keys + 256;
}

cudaError_t launch_reassign(const ReassignParams& p, cudaStream_t s) {
    const size_t slots = (size_t)(p.d.cap_o + p.d.cap_q);
    const size_t dyn = slots <= (size_t)kSmemKeyLimit ? slots * 8 : 0;
    cudaError_t e;
    if (p.d.D == 128) {
        e = allow_max_dyn_smem(reassign_kernel<128>, g_smem_reassign128);
        if (e != cudaSuccess) return e;
        reassign_kernel<128><<<p.d.R, kRowThreads, dyn, s>>>(p);
    } else {
        e = allow_max_dyn_smem(reassign_kernel<64>, g_smem_reassign64);
        if (e != cudaSuccess) return e;
        reassign_kernel<64><<<p.d.R, kRowThreads, dyn, s>>>(p);
    }
    return cudaGetLastError();
}

cudaError_t launch_quantize_pack(const PackParams& p, cudaStream_t s) {
    const size_t dyn = p.n_stride <= kSmemKeyLimit ? (size_t)p.n_stride * 8 : 0;
    cudaError_t e;
    if (p.d.D == 128) {
        e = allow_max_dyn_smem(pack_kernel<128>, g_smem_pack128);
        if (e != cudaSuccess) return e;
        pack_kernel<128><<<p.d.R, kRowThreads, dyn, s>>>(p);
    } else {
        e = allow_max_dyn_smem(pack_kernel<64>, g_smem_pack64);
        if (e != cudaSuccess) return e;
        pack_kernel<64><<<p.d.R, kRowThreads, dyn, s>>>(p);
    }
    return cudaGetLastError();
}

cudaError_t launch_fp8_encode(int fmt, const float* x, uint8_t* out, size_t n, cudaStream_t s) {
    if (n == 0) return cudaSuccess;
    const size_t pairs = (n + 1) / 2;
    const unsigned blocks = (unsigned)((pairs + 255) / 256);
    if (fmt == ARKV_FMT_E5M2) fp8_encode_kernel<ARKV_FMT_E5M2><<<blocks, 256, 0, s>>>(x, out, n);
    else fp8_encode_kernel<ARKV_FMT_E4M3><<<blocks, 256, 0, s>>>(x, out, n);
    return cudaGetLastError();
}

}  // namespace arkv
