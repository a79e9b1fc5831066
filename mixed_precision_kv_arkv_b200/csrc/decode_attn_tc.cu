// Decode attention over the tri-state cache for head_dim 128 on the fifth-generation
// tensor cores (ARKV, 기술요약 §2.다: quantized tokens are dequantized right before
// attention and attended together with the originals; the raw logits feed the score
// observation of §2.나).
//
// One persistent CTA per SM.  The live tiles of a layer (128 tokens each, row by
// row: a row's bf16 tiles, then its fp8 tiles) are dealt out stream-K style: CTA c
// takes one contiguous range of equal cost (a bf16 tile costs 2, an fp8 tile 1, in
// proportion to the bytes they stream).  Within a range, the tiles of one split
// (kSplitBf16 bf16 or kSplitFp8 fp8 slots) form a piece with its own partial; a
// split cut by a range boundary has two partials (slots 0 and 1), merged by
// merge_kernel with all the others.  Warp roles:
//   warps 0, 10 producers: walk the range and stream K (warp 0, with the row's query
//               group and the tile metadata) and V (warp 10) of every tile with TMA
//               (128-byte swizzle) into two rings of kSlots 32 KB slots; each
//               appends its half of the new token.
//   warp 1      MMA issuer (one thread): per tile
//                 S[128 tok][16]   = K[128 tok][128] . Q^T                 (tcgen05, K-major A and B)
//                 O^T[128 d][16]  += V^T[128 d][128 tok] . P[128 tok][16]  (MN-major A and B)
//               with S and O in tensor memory (two S buffers, one O per piece, two
//               pieces in flight); QK^T and PV are issued as soon as their inputs
//               are ready, and a K slot is freed as soon as its QK^T completes.
//   warps 2-5   softmax warpgroup: thread = token (tensor-memory lane).  Reads its
//               four logits, stores them for the score update, keeps an online
//               softmax whose reference maximum moves only when a logit exceeds it
//               by 8 in log2 units (then O is rescaled in tensor memory), and writes
//               its probabilities as [P_hi | P_lo] (16 significant bits) for the PV.
//   warps 6-9   converter warpgroup: FP8 tiles arrive as E4M3 codes in the upper
//               half of their slots and are rewritten in place as f16 (exact) in the
//               layout of a bf16 tile, so the MMA sees one tile format; the tile's
//               scales are staged in shared memory, and the FP8 query group is
//               converted to f16 once per piece.
// FP8 tiles: the per-token K scale multiplies the logit; the V scale is folded into
// P relative to a power-of-two piece scale (moved lazily like the maximum), which
// the epilogue divides back out.
//
// Every wait is bounded: a wait that runs out raises ARKV_STATUS_TIMEOUT, sets a
// CTA-wide abort flag that every role checks at a uniform point, and the CTA drains
// its copies and tensor-core work before it frees tensor memory and returns.
#include <math.h>

#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cudaTypedefs.h>

#include "arkv_internal.cuh"

namespace arkv {

namespace {

constexpr int kD = 128;
constexpr int kTok = 128;                  // tokens per tile
constexpr int kSlots = 3;                  // slots per ring (K ring, V ring)
constexpr int kThreads = 352;   // 11 warps
constexpr int kSpin = 1 << 20;             // polls per bounded drain wait
constexpr int kNaps = 1 << 16;             // suspending polls per bounded wait
constexpr uint32_t kSlotBytes = 32768;     // one K or V tile: 2 regions of 128 rows x 128 B

// shared-memory map (offsets from a 1024-byte aligned base).  The query group
// (4 rows) and P (8 columns) are the first halves of UMMA operands of 16 rows /
// columns; their second halves are all zero and shared by every buffer through the
// descriptors' stride offsets.
constexpr int kNQ = 4;                                   // query-group / O buffers (pieces in flight)
constexpr uint32_t kOffK = 0;
constexpr uint32_t kOffV = kSlots * kSlotBytes;
constexpr uint32_t kOffQb = 2 * kSlots * kSlotBytes;    // bf16 query group [kNQ][2 regions][8 rows][128 B]
constexpr uint32_t kOffQh = kOffQb + kNQ * 2048;         // f16 query group, same layout
constexpr uint32_t kOffQz = kOffQh + kNQ * 2048;         // 8 zero rows of 128 B
constexpr uint32_t kOffP = kOffQz + 1024;                // P [2][128 tok][16 B]
constexpr uint32_t kOffPz = kOffP + 2 * 2048;            // 128 x 16 B of zeros (P columns 8..15)
constexpr uint32_t kOffBar = kOffPz + 2048;
constexpr int kBarKFull = 0, kBarVFull = 3, kBarConvK = 6, kBarConvV = 9, kBarKEmpty = 12, kBarVEmpty = 15,
              kBarSFull = 18, kBarSEmpty = 20, kBarPFull = 22, kBarPEmpty = 24, kBarOFull = 26, kBarOEmpty = 30,
              kBarQFull = 34, kBarQEmpty = 38, kBarFin = 42, kNumBars = 43;
constexpr uint32_t kOffMeta = kOffBar + 384;             // TileMeta [kSlots]
constexpr uint32_t kOffRed = kOffMeta + 128;             // float [4 warps][8]
constexpr uint32_t kOffMisc = kOffRed + 128;             // tensor-memory base, abort flag
constexpr uint32_t kOffScale = kOffMisc + 16;            // float [kSlots][2][128]: FP8 K and V scales
constexpr uint32_t kOffCnt = kOffScale + kSlots * 2 * kTok * 4;   // int2 [kRowsInSmem]
constexpr int kRowsInSmem = 512;
constexpr uint32_t kSmemBytes = kOffCnt + 8 * kRowsInSmem + 1024;   // + alignment slack
constexpr uint32_t kZeroBytes = kOffBar - kOffQb;                    // query groups, P and the zero blocks
static_assert(kNumBars * 8 <= 384, "barrier block");
static_assert(kSmemBytes <= 232448, "shared memory per CTA");
static_assert(kOffQz % 1024 == 0 && kOffQb % 1024 == 0 && kOffQh % 1024 == 0, "swizzle atoms");

// tensor-memory columns (fp32): S[2] at 0 and 16, O[kNQ] at 32, 48, 64, 80
constexpr uint32_t kTmemCols = 128;

enum : int { kFirst = 1, kLast = 2, kWhole = 4, kDone = 8 };
struct TileMeta {
    int row, fp8, t0, ntok, flags, split, slot, pad;
};

// instruction descriptors (kind::f16, fp32 accumulate, M = 128, N = 16)
constexpr uint32_t kIdescBase = (1u << 4) | ((16u >> 3) << 17) | ((128u >> 4) << 24);
constexpr uint32_t kIdescBf16 = (1u << 7) | (1u << 10);   // A and B bf16 (else f16)
constexpr uint32_t kIdescMN = (1u << 15) | (1u << 16);    // A and B MN-major (else K-major)

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ bool mbar_try_wait_hint(uint32_t bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\tselp.u32 %0, 1, 0, p;\n}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0;
}
// Suspends for at most about `ns` nanoseconds or until the phase completes.
__device__ __forceinline__ void mbar_nap(uint32_t bar, uint32_t parity, uint32_t ns) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%0], %1, %2;\n}" ::"r"(bar),
        "r"(parity), "r"(ns)
        : "memory");
}
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// named barrier over one warpgroup (ids 1, 2); OR-reduction of a predicate
__device__ __forceinline__ void wg_sync(int id) { asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory"); }
__device__ __forceinline__ bool wg_or(bool v, int id) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\tbar.red.or.pred p, %2, 128, q;\n\tselp.u32 %0, 1, 0, p;\n}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id)
        : "memory");
    return r != 0;
}

// Shared-memory matrix descriptor: start, leading / stride byte offsets, version 1,
// layout (2 = 128-byte swizzle, 0 = no swizzle).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
    return (uint64_t)((addr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | ((uint64_t)layout << 61);
}
__device__ __forceinline__ void umma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, bool acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"((uint32_t)acc)
        : "memory");
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
__device__ __forceinline__ void tmem_ld4(uint32_t addr, float (&v)[4]) {
    uint32_t r[4];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int k = 0; k < 4; ++k) v[k] = __uint_as_float(r[k]);
}
__device__ __forceinline__ void tmem_ld8(uint32_t addr, float (&v)[8]) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(addr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = __uint_as_float(r[k]);
}
__device__ __forceinline__ void tmem_st8(uint32_t addr, const float (&v)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"r"(addr),
                 "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
                 "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
                 "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7]))
                 : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
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

// Byte offset of 16-byte chunk `c` of row `r` in a region of 128-byte rows written
// with the 128-byte swizzle (the region starts 1024-byte aligned).
__device__ __forceinline__ uint32_t sw128(int r, int c) { return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4)); }

struct Ctx {
    uint32_t base;     // shared address of the aligned base
    char* gbase;       // generic pointer of the same
    volatile int* abort_flag;
    int* status;
    __device__ uint32_t bar(int i) const { return base + kOffBar + 8u * i; }
    // Bounded wait: false if it ran out (or the CTA is aborting).  Each poll
    // suspends the thread until the phase completes or about 20 us pass, so a
    // waiting thread costs the SM almost nothing (at most ~1.3 s in all).
    __device__ bool wait(int i, uint32_t parity) const {
        const uint32_t b = bar(i);
        for (int k = 0; k < kNaps; ++k) {
            if (mbar_try_wait_hint(b, parity, 20000)) return true;
            if (*abort_flag) return false;
        }
        return false;
    }
    __device__ void fail() const {
        *abort_flag = 1;
        atomicOr(status, ARKV_STATUS_TIMEOUT);
    }
    // Lane 0 waits; the outcome is made warp-uniform by the shuffle, which also
    // orders the other lanes after lane 0's acquire.  A failure raises the abort
    // flag; work after a failed wait runs on stale data and is discarded: the roles
    // stop at their next abort check.
    __device__ bool warp_wait(int i, uint32_t parity) const {
        bool ok = true;
        if ((threadIdx.x & 31) == 0) ok = wait(i, parity);
        ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;   // (orders the other lanes after lane 0's acquire)
        if (!ok && (threadIdx.x & 31) == 0) fail();
        return ok;
    }
};


// Counts of row r before this call: (bf16, fp8), clamped to the capacities.
__device__ __forceinline__ int2 row_counts(const AttnParams& p, const int2* cnt, int r) {
    if (r < kRowsInSmem) return cnt[r];
    return make_int2(min(max(p.c.n_bf16[r], 0), p.d.cap_o), min(max(p.c.n_fp8[r], 0), p.d.cap_q));
}
// Live slots of row r: (bf16 including the slot of the new token, fp8).
__device__ __forceinline__ int2 row_live(const AttnParams& p, const int2* cnt, int r) {
    const int2 c = row_counts(p, cnt, r);
    return make_int2(c.x + (c.x < p.d.cap_o ? 1 : 0), c.y);
}
__device__ __forceinline__ int tiles_of(int n) { return (n + kTok - 1) / kTok; }
__device__ __forceinline__ long long row_cost(int2 c) { return 2LL * tiles_of(c.x) + tiles_of(c.y); }

// The tiles of this CTA's cost range [lo, hi), in order.
struct Walk {
    long long lo, hi;
    int R, r;            // current row
    long long x;         // cost position of the row's first tile
    int2 c;              // live counts of the row
    int seg, j;          // segment (0 bf16, 1 fp8) and tile index in it
    bool valid;
};

__device__ __forceinline__ long long tile_pos(const Walk& w) {
    return w.seg == 0 ? w.x + 2LL * w.j : w.x + 2LL * tiles_of(w.c.x) + w.j;
}

// Moves past exhausted segments and rows (the result is not checked against hi).
__device__ void walk_norm(const AttnParams& p, const int2* cnt, Walk& w) {
    for (;;) {
        if (w.seg == 0 && w.j >= tiles_of(w.c.x)) { w.seg = 1; w.j = 0; }
        if (w.seg == 1 && w.j >= tiles_of(w.c.y)) {
            w.x += row_cost(w.c);
            if (++w.r >= w.R) { w.valid = false; return; }
            w.c = row_live(p, cnt, w.r);
            w.seg = 0; w.j = 0;
            continue;
        }
        return;
    }
}
__device__ __forceinline__ void walk_next(const AttnParams& p, const int2* cnt, Walk& w) {
    ++w.j;
    walk_norm(p, cnt, w);
}

struct Tile {
    int row, fp8, j, t0, ntok, split, first_of_split, last_of_split;
};

__device__ __forceinline__ Tile tile_of(const AttnParams& p, const Walk& w) {
    Tile t;
    t.row = w.r;
    t.fp8 = w.seg;
    t.j = w.j;
    t.t0 = w.j * kTok;
    const int n = w.seg == 0 ? w.c.x : w.c.y;
    t.ntok = min(kTok, n - t.t0);
    const int per = w.seg == 0 ? kSplitBf16 / kTok : kSplitFp8 / kTok;   // tiles per split
    t.split = w.seg == 0 ? w.j / per : p.nsplit_o + w.j / per;
    t.first_of_split = (w.j / per) * per;
    t.last_of_split = min(t.first_of_split + per, tiles_of(n)) - 1;
    return t;
}

// ------------------------------------------------------------------ roles
// This CTA's range of the cost sequence and the walk positioned at its first tile.
// At least 8 cost units per range, so that a split (cost 4) is cut by at most one
// range boundary.  Warp-uniform.
__device__ Walk walk_begin(const AttnParams& p, const int2* cnt) {
    const int lane = threadIdx.x & 31, R = p.d.R;
    long long total = 0;
    for (int base = 0; base < R; base += 32) {
        const int r = base + lane;
        long long c = r < R ? row_cost(row_live(p, cnt, r)) : 0;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) c += __shfl_xor_sync(0xffffffffu, c, o);
        total += c;
    }
    const long long G = max(1LL, min((long long)gridDim.x, total / 8));
    Walk w{};
    w.R = R;
    w.valid = blockIdx.x < G && total > 0;
    w.lo = total * blockIdx.x / G;
    w.hi = total * (blockIdx.x + 1) / G;
    if (!w.valid) return w;
    // the row holding cost position lo
    long long base_cost = 0, x0 = 0;
    int r0 = -1;
    for (int base = 0; base < R && r0 < 0; base += 32) {
        const int r = base + lane;
        const long long c = r < R ? row_cost(row_live(p, cnt, r)) : 0;
        long long incl = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const long long v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        const unsigned hit = __ballot_sync(0xffffffffu, r < R && base_cost + incl > w.lo);
        if (hit) {
            const int f = __ffs(hit) - 1;
            r0 = base + f;
            x0 = base_cost + __shfl_sync(0xffffffffu, incl - c, f);
        }
        base_cost += __shfl_sync(0xffffffffu, incl, 31);
    }
    w.valid = r0 >= 0;
    if (!w.valid) return w;
    w.r = r0;
    w.x = x0;
    w.c = row_live(p, cnt, r0);
    const long long t16 = tiles_of(w.c.x);
    if (w.lo < w.x + 2 * t16) {
        w.seg = 0;
        w.j = (int)((w.lo - w.x + 1) / 2);   // first bf16 tile starting at or after lo
    } else {
        w.seg = 1;
        w.j = (int)(w.lo - w.x - 2 * t16);
    }
    walk_norm(p, cnt, w);
    w.valid = w.valid && tile_pos(w) < w.hi;
    return w;
}

// Producers: warp 0 streams K (and the query group, and the tile metadata), warp 10
// streams V; both walk the same tile sequence.  The new token goes to slot n_bf16
// before the tensor load that reads that slot (each warp writes its half; the proxy
// fence orders the write and the load).
__device__ void producer(const AttnParams& p, const Ctx& cx, bool is_v) {
    const LayerDims& d = p.d;
    const int lane = threadIdx.x & 31;
    TileMeta* meta = reinterpret_cast<TileMeta*>(cx.gbase + kOffMeta);
    const int2* cnt = reinterpret_cast<const int2*>(cx.gbase + kOffCnt);
    Walk w = walk_begin(p, cnt);
    int i = 0, n = 0;            // tile index, piece ordinal
    int last = -1;               // last tile whose load was issued
    bool ok = true, in_piece = false;
    int cur_slot = 0;
    const int ring_full = is_v ? kBarVFull : kBarKFull, ring_empty = is_v ? kBarVEmpty : kBarKEmpty;
    const uint32_t ring_off = is_v ? kOffV : kOffK;
    const CUtensorMap* tm16 = is_v ? &p.tm_v16 : &p.tm_k16;
    const CUtensorMap* tm8 = is_v ? &p.tm_v8 : &p.tm_k8;
    for (; w.valid && tile_pos(w) < w.hi && ok; ++i) {
        const Tile t = tile_of(p, w);
        const int b = t.row / d.hkv, gk = t.row - b * d.hkv;
        // piece flags (K warp)
        int f = 0;
        if (!in_piece) {
            f |= kFirst;
            cur_slot = t.j == t.first_of_split ? 0 : 1;
        }
        const bool end_of_split = t.j == t.last_of_split;
        if (end_of_split || tile_pos(w) + (t.fp8 ? 1 : 2) >= w.hi) {
            f |= kLast;
            if (end_of_split && cur_slot == 0) f |= kWhole;   // the piece holds the whole split
        }
        in_piece = !(f & kLast);
        if (!is_v && (f & kFirst)) {   // the row's query group for this piece
            const int qb = n % kNQ;
            if (lane == 0) {
                if (!cx.wait(kBarQEmpty + qb, ((n / kNQ) & 1) ^ 1)) { cx.fail(); ok = false; }
                if (ok) {
                    const uint32_t qdst = cx.base + kOffQb + qb * 2048;
                    mbar_expect_tx(cx.bar(kBarQFull + qb), 2 * 4 * 128);
                    const int y = b * d.hq + gk * d.G;
                    tma_load_2d(qdst, &p.tm_q, 0, y, cx.bar(kBarQFull + qb));
                    tma_load_2d(qdst + 1024, &p.tm_q, 64, y, cx.bar(kBarQFull + qb));
                }
            }
            ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
            ++n;
        }
        if (!t.fp8) {
            const int n16 = row_counts(p, cnt, t.row).x;
            if (n16 < d.cap_o && n16 >= t.t0 && n16 < t.t0 + t.ntok) {
                const size_t sl = (size_t)t.row * d.cap_o + n16;
                if (lane < 16) {
                    const uint16_t* src = (is_v ? p.v_new : p.k_new) + ((size_t)b * d.hkv + gk) * kD;
                    uint16_t* dst = (is_v ? p.c.v16 : p.c.k16) + sl * kD;
                    reinterpret_cast<uint4*>(dst)[lane] = reinterpret_cast<const uint4*>(src)[lane];
                }
                if (!is_v && lane == 0) {
                    p.c.pos16[sl] = p.ctx_len[b] + p.step;
                    p.c.mu16[sl] = 0.f;
                    p.c.m2_16[sl] = 0.f;
                }
                asm volatile("fence.proxy.async.global;" ::: "memory");
                __syncwarp();
            }
        }
        const int s = i % kSlots;
        if (lane == 0 && ok) {
            if (!cx.wait(ring_empty + s, ((i / kSlots) & 1) ^ 1)) { cx.fail(); ok = false; }
            if (ok) {
                if (!is_v) {
                    TileMeta m;
                    m.row = t.row; m.fp8 = t.fp8; m.t0 = t.t0; m.ntok = t.ntok; m.flags = f;
                    m.split = t.split; m.slot = cur_slot; m.pad = 0;
                    meta[s] = m;
                }
                const uint32_t dst = cx.base + ring_off + s * kSlotBytes, bar = cx.bar(ring_full + s);
                if (!t.fp8) {
                    const int y = t.row * d.cap_o + t.t0;
                    mbar_expect_tx(bar, kSlotBytes);
                    tma_load_2d(dst, tm16, 0, y, bar);
                    tma_load_2d(dst + 16384, tm16, 64, y, bar);
                } else {
                    mbar_expect_tx(bar, kSlotBytes / 2);
                    tma_load_2d(dst + 16384, tm8, 0, t.row * d.cap_q + t.t0, bar);
                }
                last = i;
            }
        }
        ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
        walk_next(p, cnt, w);
    }
    // end of the stream: a K slot that carries only the done flag
    if (!is_v && lane == 0 && ok) {
        const int s = i % kSlots;
        if (cx.wait(kBarKEmpty + s, ((i / kSlots) & 1) ^ 1)) {
            meta[s].flags = kDone;
            mbar_arrive(cx.bar(kBarKFull + s));
        } else {
            cx.fail();
        }
    }
    // after an abort, let every issued copy land before the CTA can leave (on the
    // normal path the consumers have waited for every tile before the done flag)
    if (lane == 0 && !ok && last >= 0)
        for (int s = 0; s < kSlots; ++s) {
            const int ls = last - ((last - s) % kSlots + kSlots) % kSlots;   // last use of slot s
            if (ls >= 0) {
                const uint32_t bb = cx.bar(ring_full + s), par = (ls / kSlots) & 1;
                for (int k = 0; k < kSpin && !mbar_try_wait(bb, par); ++k) {
                }
            }
        }
    __syncwarp();
}

// Issues QK^T of the next tile as soon as its K (and, for FP8, its conversion),
// its S buffer and, at a piece's first tile, the query group and an O buffer are
// ready; and the PV of the oldest tile as soon as its probabilities and its V are.
// At most two tiles sit between their QK^T and their PV (two S and P buffers).
__device__ void mma_issuer(const AttnParams& p, const Ctx& cx, uint32_t tmem) {
    const int lane = threadIdx.x & 31;
    const TileMeta* meta = reinterpret_cast<const TileMeta*>(cx.gbase + kOffMeta);
    if (lane == 0) {
        int iq = 0, ip = 0, n = -1;
        int fp8cnt[kSlots] = {0, 0, 0};
        int t_ob[2], t_fp8[2], t_last[2], t_first[2], t_cv[2];   // tiles between QK^T and PV
        // conditions already seen for the next QK^T (a bit each: K landed, S free,
        // query group and O buffer, FP8 conversion) and for the oldest PV (P, V, conversion);
        // a barrier is tested only until it is seen, since every test is a round trip
        uint32_t qk_seen = 0, pv_seen = 0;
        TileMeta m{};
        bool done = false;
        int idle = 0;
        for (;;) {
            bool prog = false;
            if (!done && iq - ip < 2) {
                const int s = iq % kSlots;
                if (!(qk_seen & 1) && mbar_test(cx.bar(kBarKFull + s), (iq / kSlots) & 1)) {
                    qk_seen |= 1;
                    m = meta[s];
                    if (m.flags & kDone) { done = true; prog = true; }
                }
                if ((qk_seen & 1) && !done) {
                    const bool first = (m.flags & kFirst) != 0;
                    const int nn = first ? n + 1 : n;
                    if (!(qk_seen & 2) && mbar_test(cx.bar(kBarSEmpty + (iq & 1)), ((iq >> 1) & 1) ^ 1)) qk_seen |= 2;
                    if (!first) qk_seen |= 4;
                    else if (!(qk_seen & 4) && mbar_test(cx.bar(kBarQFull + nn % kNQ), (nn / kNQ) & 1) &&
                             mbar_test(cx.bar(kBarOEmpty + nn % kNQ), ((nn / kNQ) & 1) ^ 1))
                        qk_seen |= 4;
                    if (!m.fp8) qk_seen |= 8;
                    else if (!(qk_seen & 8) && mbar_test(cx.bar(kBarConvK + s), fp8cnt[s] & 1)) qk_seen |= 8;
                    if (qk_seen == 15) {
                        n = nn;
                        const int cvpar = fp8cnt[s] & 1;   // this tile's conversion phase
                        if (m.fp8) ++fp8cnt[s];
                        tc_fence_after();
                        // S = K Q^T: A = the K tile (two 64-dim regions), B = the query group
                        const uint32_t kbase = cx.base + kOffK + s * kSlotBytes;
                        const uint32_t qbase = cx.base + (m.fp8 ? kOffQh : kOffQb) + (n % kNQ) * 2048;
                        const uint32_t idesc = kIdescBase | (m.fp8 ? 0u : kIdescBf16);
                        // descriptors of the first k step of each 64-dim region; a k step
                        // of 16 dims advances the start address by 32 bytes
                        const uint64_t a0 = smem_desc(kbase, 16, 1024, 2);
                        const uint64_t b0 = smem_desc(qbase, 16, cx.base + kOffQz - qbase, 2);   // rows 8..15:
                        const uint64_t b1 = smem_desc(qbase + 1024, 16, cx.base + kOffQz - qbase - 1024, 2);   // zeros
#pragma unroll
                        for (int k = 0; k < kD / 16; ++k)
                            umma(tmem + 16 * (iq & 1), a0 + (uint64_t)((k >> 2) * 1024 + (k & 3) * 2),
                                 (k < 4 ? b0 : b1) + (uint64_t)((k & 3) * 2), idesc, k > 0);
                        umma_commit(cx.bar(kBarSFull + (iq & 1)));
                        umma_commit(cx.bar(kBarKEmpty + s));
                        if (m.flags & kLast) umma_commit(cx.bar(kBarQEmpty + n % kNQ));   // the piece's last read of Q
                        const int t = iq & 1;
                        t_ob[t] = n % kNQ; t_fp8[t] = m.fp8; t_cv[t] = cvpar;
                        t_last[t] = (m.flags & kLast) != 0; t_first[t] = first;
                        ++iq;
                        qk_seen = 0;
                        prog = true;
                    }
                }
            }
            if (ip < iq) {
                const int t = ip & 1, s = ip % kSlots;
                if (!(pv_seen & 1) && mbar_test(cx.bar(kBarPFull + t), (ip >> 1) & 1)) pv_seen |= 1;
                if (!(pv_seen & 2) && mbar_test(cx.bar(kBarVFull + s), (ip / kSlots) & 1)) pv_seen |= 2;
                if (!t_fp8[t]) pv_seen |= 4;
                else if (!(pv_seen & 4) && mbar_test(cx.bar(kBarConvV + s), t_cv[t])) pv_seen |= 4;
                if (pv_seen == 7) {
                    tc_fence_after();
                    // O^T += V^T P: A = the V tile read MN-major, B = P (MN-major, no swizzle)
                    const uint32_t vbase = cx.base + kOffV + s * kSlotBytes;
                    const uint32_t pbase = cx.base + kOffP + t * 2048;
                    const uint32_t idesc = kIdescBase | kIdescMN | (t_fp8[t] ? 0u : kIdescBf16);
                    const uint32_t dO = tmem + 32 + 16 * t_ob[t];
                    // a k step of 16 tokens advances V by 2048 bytes and P by 256 bytes
                    const uint64_t a0 = smem_desc(vbase, 16384, 1024, 2);
                    const uint64_t b0 = smem_desc(pbase, 128, cx.base + kOffPz - pbase, 0);
#pragma unroll
                    for (int k = 0; k < kTok / 16; ++k)
                        umma(dO, a0 + (uint64_t)(k * 128), b0 + (uint64_t)(k * 16), idesc, !(t_first[t] && k == 0));
                    umma_commit(cx.bar(kBarPEmpty + t));
                    umma_commit(cx.bar(kBarVEmpty + s));
                    if (t_last[t]) umma_commit(cx.bar(kBarOFull + t_ob[t]));
                    ++ip;
                    pv_seen = 0;
                    prog = true;
                }
            }
            if (done && ip == iq) break;
            if (prog) {
                idle = 0;
            } else {
                ++idle;
                if ((idle & 63) == 0 && *cx.abort_flag) break;
                if (idle > (1 << 18)) { cx.fail(); break; }
                // block on the one event most likely next: the oldest tile's P, else the next K
                if (ip < iq && !(pv_seen & 1)) mbar_nap(cx.bar(kBarPFull + (ip & 1)), (ip >> 1) & 1, 500);
                else if (!(qk_seen & 1)) mbar_nap(cx.bar(kBarKFull + iq % kSlots), (iq / kSlots) & 1, 500);
                else if (ip < iq && !(pv_seen & 2)) mbar_nap(cx.bar(kBarVFull + ip % kSlots), (ip / kSlots) & 1, 500);
                else __nanosleep(32);
            }
        }
        // drain: every issued tensor-core operation completes before tensor memory is freed
        umma_commit(cx.bar(kBarFin));
        const uint32_t fb = cx.bar(kBarFin);
        for (int k = 0; k < kSpin && !mbar_try_wait(fb, 0); ++k) {
        }
    }
    __syncwarp();
}

// E4M3 codes of one 128-byte swizzled row (8 chunks) -> f16 into the two 64-dim
// regions of a slot, same row, 128-byte swizzle.
__device__ __forceinline__ void write_f16_row(char* slot, int r, const uint4 (&raw)[8]) {
#pragma unroll
    for (int c = 0; c < 8; ++c) {
        const uint4 k = raw[c];
        uint4 lo, hi;   // dims 16c .. 16c+7, 16c+8 .. 16c+15
        lo.x = e4m3x2_to_f16x2(k.x); lo.y = e4m3x2_to_f16x2(k.x >> 16);
        lo.z = e4m3x2_to_f16x2(k.y); lo.w = e4m3x2_to_f16x2(k.y >> 16);
        hi.x = e4m3x2_to_f16x2(k.z); hi.y = e4m3x2_to_f16x2(k.z >> 16);
        hi.z = e4m3x2_to_f16x2(k.w); hi.w = e4m3x2_to_f16x2(k.w >> 16);
        char* reg = slot + (c >> 2) * 16384;
        *reinterpret_cast<uint4*>(reg + sw128(r, 2 * (c & 3))) = lo;
        *reinterpret_cast<uint4*>(reg + sw128(r, 2 * (c & 3) + 1)) = hi;
    }
}

// FP8 tiles: K (with the tile's scales) is converted as soon as it lands and
// gates the tile's QK^T; V, which lands about one tile later, is converted in the
// next iteration and gates the tile's PV.
__device__ void converter(const AttnParams& p, const Ctx& cx) {
    const LayerDims& d = p.d;
    const int ct = threadIdx.x - 192, lane = threadIdx.x & 31;
    const TileMeta* meta = reinterpret_cast<const TileMeta*>(cx.gbase + kOffMeta);
    float* scales = reinterpret_cast<float*>(cx.gbase + kOffScale);
    int n = -1;
    int prev_s = -1, prev_i = 0;   // an FP8 tile whose V is still to be converted
    auto convert_v = [&](int s, int i) {
        cx.warp_wait(kBarVFull + s, (i / kSlots) & 1);
        char* vs = cx.gbase + kOffV + s * kSlotBytes;
        uint4 raw[8];
#pragma unroll
        for (int c = 0; c < 8; ++c) raw[c] = *reinterpret_cast<const uint4*>(vs + 16384 + sw128(ct, c));
        wg_sync(2);   // every code has been read: the slot may be overwritten
        write_f16_row(vs, ct, raw);
        fence_proxy_async_smem();
        wg_sync(2);
        if (ct == 0) mbar_arrive(cx.bar(kBarConvV + s));
    };
    for (int i = 0;; ++i) {
        const int s = i % kSlots;
        cx.warp_wait(kBarKFull + s, (i / kSlots) & 1);
        if (wg_or(*cx.abort_flag != 0, 2)) { prev_s = -1; break; }
        const TileMeta m = meta[s];
        if (m.flags & kDone) break;
        if (m.flags & kFirst) ++n;
        if (m.fp8) {
            // this token's scales (the loads overlap the conversion)
            float sk = 0.f, sv = 0.f;
            if (ct < m.ntok) {
                sk = __ldg(p.c.sk + (size_t)m.row * d.cap_q + m.t0 + ct);
                sv = __ldg(p.c.sv + (size_t)m.row * d.cap_q + m.t0 + ct);
            }
            if (m.flags & kFirst) {   // the piece's query group in f16
                cx.warp_wait(kBarQFull + n % kNQ, (n / kNQ) & 1);
                const int h = ct >> 5, j = ct & 31;   // head h, dims 4j .. 4j+3
                const uint32_t off = (uint32_t)((j >> 4) * 1024) + sw128(h, (j & 15) >> 1) + (j & 1) * 8;
                const uint2 w = *reinterpret_cast<const uint2*>(cx.gbase + kOffQb + (n % kNQ) * 2048 + off);
                const float a0 = __uint_as_float(w.x << 16), a1 = __uint_as_float(w.x & 0xffff0000u);
                const float a2 = __uint_as_float(w.y << 16), a3 = __uint_as_float(w.y & 0xffff0000u);
                *reinterpret_cast<uint2*>(cx.gbase + kOffQh + (n % kNQ) * 2048 + off) =
                    make_uint2(pack_f16(a0, a1), pack_f16(a2, a3));
            }
            // token row ct: codes in the upper half of the slot, 128-byte rows
            char* ks = cx.gbase + kOffK + s * kSlotBytes;
            uint4 raw[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) raw[c] = *reinterpret_cast<const uint4*>(ks + 16384 + sw128(ct, c));
            wg_sync(2);   // every code has been read: the slot may be overwritten
            write_f16_row(ks, ct, raw);
            scales[(s * 2 + 0) * kTok + ct] = sk;
            scales[(s * 2 + 1) * kTok + ct] = sv;
            fence_proxy_async_smem();
            wg_sync(2);
            if (ct == 0) mbar_arrive(cx.bar(kBarConvK + s));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(cx.bar(kBarKEmpty + s));
        if (prev_s >= 0) convert_v(prev_s, prev_i);
        prev_s = m.fp8 ? s : -1;
        prev_i = i;
    }
    if (prev_s >= 0) convert_v(prev_s, prev_i);
}

// A finished piece whose partial is written one tile later (its O then is complete
// without waiting; the piece's O buffer is not reused before the piece after next).
struct PendingPiece {
    bool live;
    int row, split, slot, whole, fp8, n;
    float vsc, mref[4], l[4];
};

__device__ __forceinline__ void write_partial(const AttnParams& p, const Ctx& cx, uint32_t tmem, uint32_t lane_off,
                                              float* red, const PendingPiece& pp) {
    const int lane = threadIdx.x & 31, q = (threadIdx.x >> 5) & 3, r = 32 * q + lane;
    const int nsplit = p.nsplit_o + p.nsplit_q;
    float lt[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
        float x = pp.l[h];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
        lt[h] = x;
    }
    if (lane == 0)
#pragma unroll
        for (int h = 0; h < 4; ++h) red[q * 8 + h] = lt[h];
    const int ob = pp.n % kNQ;
    cx.warp_wait(kBarOFull + ob, (pp.n / kNQ) & 1);
    tc_fence_after();
    float o8[8];
    tmem_ld8(tmem + 32 + 16 * ob + lane_off, o8);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(cx.bar(kBarOEmpty + ob));
    wg_sync(1);
    const size_t ps = (size_t)pp.row * nsplit + pp.split;   // the split; partial slot pp.slot
    const size_t pb = ps * 2 + pp.slot;
    const float un = pp.fp8 ? (pp.vsc > 0.f ? 1.f / pp.vsc : 0.f) : 1.f;
#pragma unroll
    for (int h = 0; h < 4; ++h) p.part_o[(pb * 4 + h) * kD + r] = (o8[h] + o8[4 + h]) * un;
    if (threadIdx.x - 64 < 4) {
        const int h = threadIdx.x - 64;
        const float L = (red[h] + red[8 + h]) + (red[16 + h] + red[24 + h]);
        p.part_ml[pb * 4 + h] = make_float2(pp.mref[h], L);
        if (pp.whole) p.part_ml[(ps * 2 + 1) * 4 + h] = make_float2(-INFINITY, 0.f);
    }
    wg_sync(1);   // the scratch is read by everyone before its next use
}

__device__ void softmax_wg(const AttnParams& p, const Ctx& cx, uint32_t tmem) {
    const LayerDims& d = p.d;
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31, q = w & 3;
    const int r = 32 * q + lane;                       // token (and output dim) of this thread
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    const TileMeta* meta = reinterpret_cast<const TileMeta*>(cx.gbase + kOffMeta);
    const float* scales = reinterpret_cast<const float*>(cx.gbase + kOffScale);
    float* red = reinterpret_cast<float*>(cx.gbase + kOffRed);   // [4][8]
    const float c2 = (float)(p.inv_sqrt_d * 1.4426950408889634);   // log2(e) / sqrt(D)
    int n = -1, tile_in_piece = 0, cur_row = -1, cur_fp8 = -1;
    int fp8cnt[kSlots] = {0, 0, 0};
    // The reference maximum (and the FP8 V scale) carry over between the pieces of
    // one row -- a piece's partial is exact relative to any reference -- so they
    // move only when a logit exceeds them; l and O restart with every piece.
    float mref[4], mc[4], l[4], vsc = 0.f;
    for (int h = 0; h < 4; ++h) { mref[h] = -INFINITY; mc[h] = -INFINITY; l[h] = 0.f; }
    PendingPiece pend;
    pend.live = false;
    for (int i = 0;; ++i) {
        const int s = i % kSlots, b = i & 1;
        cx.warp_wait(kBarKFull + s, (i / kSlots) & 1);
        const TileMeta m = meta[s];
        if (m.flags & kDone) break;
        if (m.flags & kFirst) {
            ++n;
            tile_in_piece = 0;
            if (m.row != cur_row || m.fp8 != cur_fp8) {
                for (int h = 0; h < 4; ++h) { mref[h] = -INFINITY; mc[h] = -INFINITY; }
                vsc = 0.f;
                cur_row = m.row;
                cur_fp8 = m.fp8;
            }
            for (int h = 0; h < 4; ++h) l[h] = 0.f;
        }
        const int ob = n % kNQ;
        const bool valid = r < m.ntok;
        const int slot = m.t0 + r;
        // FP8 scales from the converter; the K slot (and the scales) are released
        // only after they are read, so the conversion barrier cannot run a phase ahead
        float sk = 1.f, sv = 0.f;
        if (m.fp8) {
            cx.warp_wait(kBarConvK + s, fp8cnt[s] & 1);
            ++fp8cnt[s];
            sk = scales[(s * 2 + 0) * kTok + r];
            sv = scales[(s * 2 + 1) * kTok + r];
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(cx.bar(kBarKEmpty + s));
        // logits of this token
        cx.warp_wait(kBarSFull + b, (i >> 1) & 1);
        tc_fence_after();
        float sl[4];
        tmem_ld4(tmem + 16 * b + lane_off, sl);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(cx.bar(kBarSEmpty + b));
        if (m.fp8) {
#pragma unroll
            for (int h = 0; h < 4; ++h) sl[h] *= sk;
        }
        if (valid) {
            float* lr = (m.fp8 ? p.logit8 + (size_t)m.row * d.cap_q * 4 : p.logit16 + (size_t)m.row * d.cap_o * 4);
            *reinterpret_cast<float4*>(lr + (size_t)slot * 4) = make_float4(sl[0], sl[1], sl[2], sl[3]);
        }
        // does the reference maximum (or the V scale) have to move?  One reduction
        // per tile; it also carries the abort flag, checked uniformly when raised.
        bool need = false;
#pragma unroll
        for (int h = 0; h < 4; ++h) need |= valid && h < d.G && sl[h] * c2 > mc[h] + 8.f;
        if (m.fp8) need |= valid && (vsc == 0.f || sv * vsc > 16.f);
        const bool ab = *cx.abort_flag != 0;
        if (wg_or(need || ab, 1)) {
            if (wg_or(ab, 1)) break;
            float tm[4], vm = 0.f;
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                float x = (valid && h < d.G) ? sl[h] : -INFINITY;
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
                tm[h] = x;
            }
            if (m.fp8) {
                vm = valid ? sv : 0.f;
#pragma unroll
                for (int o = 16; o >= 1; o >>= 1) vm = fmaxf(vm, __shfl_xor_sync(0xffffffffu, vm, o));
            }
            if (lane == 0) {
#pragma unroll
                for (int h = 0; h < 4; ++h) red[q * 8 + h] = tm[h];
                red[q * 8 + 4] = vm;
            }
            wg_sync(1);
            float ao[4];
            float vsc_new = vsc;
            if (m.fp8) {
                const float vmax = fmaxf(fmaxf(red[4], red[12]), fmaxf(red[20], red[28]));
                if (vmax > 0.f && (vsc == 0.f || vmax * vsc > 16.f)) {
                    int e;
                    frexpf(vmax, &e);                 // vmax < 2^e
                    vsc_new = ldexpf(1.f, -e);        // vmax * vsc_new < 1
                }
            }
            const float vratio = (vsc == 0.f) ? 1.f : vsc_new / vsc;   // a power of two
#pragma unroll
            for (int h = 0; h < 4; ++h) {
                const float t = fmaxf(fmaxf(red[h], red[8 + h]), fmaxf(red[16 + h], red[24 + h]));
                const float nm = fmaxf(mref[h], t);
                const float nmc = nm * c2;
                float al = (mc[h] == -INFINITY) ? 0.f : exp2f(mc[h] - nmc);
                if (nm == -INFINITY) al = 1.f;
                ao[h] = al * vratio;
                l[h] *= al;
                mref[h] = nm;
                mc[h] = (nm == -INFINITY) ? -INFINITY : nmc;
            }
            vsc = vsc_new;
            if (tile_in_piece > 0) {   // O holds earlier tiles of this piece: rescale it
                const int pi = i - 1;
                cx.warp_wait(kBarPEmpty + (pi & 1), (pi >> 1) & 1);
                tc_fence_after();
                float o8[8];
                const uint32_t oaddr = tmem + 32 + 16 * ob + lane_off;
                tmem_ld8(oaddr, o8);
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    o8[h] *= ao[h];
                    o8[4 + h] *= ao[h];
                }
                tmem_st8(oaddr, o8);
            }
            wg_sync(1);   // the scratch is read by everyone before its next use
        }
        // probabilities (times V scale for FP8), split into high and low halves
        float w4[4];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
            const float pr = (valid && h < d.G) ? exp2f(fmaf(sl[h], c2, -mc[h])) : 0.f;
            l[h] += pr;
            w4[h] = m.fp8 ? pr * (sv * vsc) : pr;
        }
        uint4 pk;
        if (m.fp8) {
            const uint32_t h01 = pack_f16(w4[0], w4[1]), h23 = pack_f16(w4[2], w4[3]);
            const __half2 x01 = *reinterpret_cast<const __half2*>(&h01), x23 = *reinterpret_cast<const __half2*>(&h23);
            pk = make_uint4(h01, h23, pack_f16(w4[0] - __low2float(x01), w4[1] - __high2float(x01)),
                            pack_f16(w4[2] - __low2float(x23), w4[3] - __high2float(x23)));
        } else {
            const uint32_t h01 = pack_bf16(w4[0], w4[1]), h23 = pack_bf16(w4[2], w4[3]);
            const __nv_bfloat162 x01 = *reinterpret_cast<const __nv_bfloat162*>(&h01);
            const __nv_bfloat162 x23 = *reinterpret_cast<const __nv_bfloat162*>(&h23);
            pk = make_uint4(h01, h23, pack_bf16(w4[0] - __low2float(x01), w4[1] - __high2float(x01)),
                            pack_bf16(w4[2] - __low2float(x23), w4[3] - __high2float(x23)));
        }
        cx.warp_wait(kBarPEmpty + b, ((i >> 1) & 1) ^ 1);
        *reinterpret_cast<uint4*>(cx.gbase + kOffP + b * 2048 + r * 16) = pk;
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(cx.bar(kBarPFull + b));
        ++tile_in_piece;
        // the previous piece's partial, now that its O is complete
        if (pend.live) {
            write_partial(p, cx, tmem, lane_off, red, pend);
            pend.live = false;
        }
        if (m.flags & kLast) {
            pend.live = true;
            pend.row = m.row; pend.split = m.split; pend.slot = m.slot; pend.whole = (m.flags & kWhole) != 0;
            pend.fp8 = m.fp8; pend.n = n; pend.vsc = vsc;
#pragma unroll
            for (int h = 0; h < 4; ++h) { pend.mref[h] = mref[h]; pend.l[h] = l[h]; }
        }
    }
    if (pend.live && !wg_or(*cx.abort_flag != 0, 1)) write_partial(p, cx, tmem, lane_off, red, pend);
}

__global__ void __launch_bounds__(kThreads, 1) decode_attn_tc_kernel(const __grid_constant__ AttnParams p) {
    extern __shared__ char smem_raw[];
    char* g = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    Ctx cx;
    cx.gbase = g;
    cx.base = smem_u32(g);
    cx.abort_flag = reinterpret_cast<volatile int*>(g + kOffMisc + 4);
    cx.status = p.c.status;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(g + kOffMisc);
    const int warp = threadIdx.x >> 5;

    // live counts of the rows (read once; the producer walks its range with them)
    {
        int2* cnt = reinterpret_cast<int2*>(g + kOffCnt);
        const int rows = p.d.R < kRowsInSmem ? p.d.R : kRowsInSmem;
        for (int r = threadIdx.x; r < rows; r += kThreads)
            cnt[r] = make_int2(min(max(p.c.n_bf16[r], 0), p.d.cap_o), min(max(p.c.n_fp8[r], 0), p.d.cap_q));
    }
    // query / probability buffers start at zero (rows and columns past the group stay zero)
    for (uint32_t o = threadIdx.x * 16; o < kZeroBytes; o += kThreads * 16)
        *reinterpret_cast<uint4*>(g + kOffQb + o) = make_uint4(0, 0, 0, 0);
    if (threadIdx.x == 0) {
        for (int k = 0; k < kNumBars; ++k) {
            uint32_t c = 1;
            if (k >= kBarKEmpty && k < kBarKEmpty + kSlots) c = 1 + 4 + 4;   // QK^T, converter and softmax warps
            if ((k >= kBarSEmpty && k < kBarSEmpty + 2) || (k >= kBarPFull && k < kBarPFull + 2) ||
                (k >= kBarOEmpty && k < kBarOEmpty + kNQ))
                c = 4;
            mbar_init(cx.bar(k), c);
        }
        *cx.abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    fence_proxy_async_smem();
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(tmem_slot);

    if (warp == 0) producer(p, cx, false);
    else if (warp == 10) producer(p, cx, true);
    else if (warp == 1) mma_issuer(p, cx, tmem);
    else if (warp < 6) softmax_wg(p, cx, tmem);
    else converter(p, cx);

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
}

}  // namespace

cudaError_t launch_decode_attn_tc_kernel(const AttnParams& p, int ctas, cudaStream_t s) {
    static bool done[64];
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev >= 0 && dev < 64 && !done[dev]) {
        e = cudaFuncSetAttribute(decode_attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
        if (e != cudaSuccess) return e;
        done[dev] = true;
    }
    decode_attn_tc_kernel<<<ctas, kThreads, kSmemBytes, s>>>(p);
    return cudaGetLastError();
}

}  // namespace arkv
