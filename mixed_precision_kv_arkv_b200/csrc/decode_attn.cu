// Decode attention over the tri-state cache (ARKV, 기술요약 §2.다: quantized tokens
// are dequantized right before attention and attended together with the
// originals) and the score observation that feeds §2.나.
//
// One wave of CTAs (as many as the GPU holds at once) shares the rows in
// proportion to their lengths; each CTA takes about the same fraction of its row's
// bf16 tiles and of its FP8 tiles (16 tokens each; the FP8 split is shifted so that
// the CTAs' ring entries match).  Its 4 warps each take bf16 tiles round robin and
// one run of FP8 tiles (sized so that the warps' entries match), interleaved evenly,
// each warp through its own ring of 4 shared-memory slots (a bf16 tile takes two, K
// and V, each freed as soon as it is read; an FP8 tile one) filled by TMA tensor
// loads (16 rows per box, 128-byte swizzle; 64-byte for FP8 rows of 64 bytes)
// completing on per-slot mbarriers (waits are bounded).
//
// Tile math on the warp-level tensor cores (m16n8k16).  S^T = K Q^T: K is the A
// operand (16 tokens of a k block per mma), the queries the B operand (column n =
// head n & 3, zero past G), so lane (g, t) finds the logits of tokens g and g + 8
// for heads 2t, 2t + 1 (lanes t >= 2 repeat t - 2).  Two register transposes
// (movmatrix) turn its probabilities into the B fragment of
//   O^T[D x 8] += V^T[D x 16 tok] * [P_hi | P_lo][16 tok x 8]
// (columns 0..3: the 16-bit high part of each head's probabilities, 4..7 the low
// part p - hi, so one mma carries ~16 significant bits of every probability); a
// lane's accumulator columns are its own heads, and hi and lo meet once at the end
// (lanes t, t ^ 2).
//   bf16 tiles: K fragments by ldmatrix, V^T fragments by ldmatrix.trans.
//   FP8 tiles: codes are converted to f16 in registers (exact; E5M2 is the high
//   byte of an f16, E4M3 goes through the hardware conversion).  K: each 4-byte
//   word a lane reads (dims 4t..4t+3 of a 16-dim chunk of one token) is its A
//   fragment pair for that k block, and the query is loaded with the same
//   dimension order; V: the 8-bit transposing ldmatrix gives lane (g, t) the four
//   rows its address lanes 4t..4t+3 supplied, and the rows are supplied in the
//   token order 0,1,8,9, 2,3,10,11, ... so that they are tokens 2t, 2t+1, 8+2t,
//   9+2t -- the k positions of the bf16 path.  The per-token K scale multiplies the
//   finished logit; the V scale is folded into P, and every P is multiplied by 64 /
//   (the largest V scale of the warp's FP8 tiles so far; the accumulator is
//   rescaled when it grows), which keeps p * sv inside f16 and comes back out of
//   the partial.
// Softmax in float32 with a reference maximum per head that moves only when a logit
// exceeds it by 2^8 (so most tiles need no reduction, which is three shuffles over
// the 8 token lanes when it happens).  Raw logits go to the workspace for the score
// update.  The CTA combines its warps into one (max, sum, unnormalised o) partial;
// the last CTA of a row to finish (a ticket in the workspace) merges the row's
// partials and the new token into o and each head's final (max, sum), stores the
// new token in the cache and advances the row's bf16 count past it.
#include <math.h>
#include <mutex>

#include <cudaTypedefs.h>

#include "arkv_internal.cuh"
#include "splits.h"

namespace arkv {

namespace {

constexpr float kNegInf = -INFINITY;
constexpr unsigned kFull = 0xffffffffu;

#ifndef ARKV_MIN_CTAS
#define ARKV_MIN_CTAS 3
#endif
#ifndef ARKV_QK_CHAINS
#define ARKV_QK_CHAINS 2
#endif
constexpr int kQkChains = ARKV_QK_CHAINS;   // independent QK^T accumulator chains per tile
constexpr int kWarps = 4;
static_assert(kWarps == kSplitWarps, "the tile splits assume the decode CTA's warp count");
#ifndef ARKV_ROW_MULTIPLE
#define ARKV_ROW_MULTIPLE 1
#endif
constexpr bool kRowMultiple = ARKV_ROW_MULTIPLE != 0;


constexpr int kSlots = 4;                  // ring slots per warp: a bf16 tile takes 2, an FP8 tile 1
constexpr int kSpinLimit = 1 << 20;        // bounded mbarrier waits (~1 s worst case)
constexpr int kMaxGrid = 2048;             // CTAs of one call at most (partial slots in the workspace)

// ------------------------------------------------------------------ shared-memory layout
template <int D>
struct Smem {
    static constexpr int kSlot = 16 * D * 2;                            // 16 rows of bf16: one K or V tile
    static constexpr int kRing = kWarps * kSlots * kSlot;
    static constexpr int kBars = kRing;                                 // uint64 [4][kSlots]
    static constexpr int kM = kBars + kWarps * kSlots * 8;              // float [4][4]
    static constexpr int kL = kM + 16 * 4;                              // float [4][4]
    static constexpr int kRed = kL + 16 * 4;                            // float [4][4]
    static constexpr int kMax = kRed + 16 * 4;                          // float [4]
    static constexpr int kAbort = kMax + 16;                            // int: a wait gave up
    static constexpr int kShare = kAbort + 16;                          // int [8] + int64 [4]: grid share
    static constexpr int kTileq = kShare + 64;                          // int [4][kSlots]: tile of each slot
    static constexpr int kSc = kTileq + kWarps * kSlots * 4;            // float [4][kSlots][32]: FP8 scales
    static constexpr int kBytes = kSc + kWarps * kSlots * 32 * 4 + 1024;   // + alignment slack
    static constexpr int kO = 0;                                        // float [4][4][D], in the idle ring
    static_assert(4 * 4 * D * 4 <= kRing, "the epilogue buffer must fit in the ring");
};

// Byte offset of 16-byte chunk `chunk` of row `row` in a tile of `ROWB`-byte rows
// written by a TMA load with the matching swizzle (128-byte rows: chunk XOR
// row % 8; 64-byte rows: chunk XOR (row / 2) % 4).  Tiles sit at 1024-byte
// aligned addresses.
template <int ROWB>
__device__ __forceinline__ uint32_t swz_chunk(int row, int chunk) {
    if constexpr (ROWB == 128) return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4));
    else return (uint32_t)(row * 64 + ((chunk ^ ((row >> 1) & 3)) << 4));
}

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* ptr) {
    return (uint32_t)__cvta_generic_to_shared(ptr);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

#ifndef ARKV_EVICT_FIRST
#define ARKV_EVICT_FIRST 1
#endif

// L2 policy for the cache stream: every K/V byte is read once per call, so it is
// marked evict-first and the small buffers written beside it (logits, partials,
// score state) keep their place in L2 for the score update that follows.
__device__ __forceinline__ uint64_t stream_policy() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

// 2-D tiled TMA load (no multicast) of the box at (x, y) completing on `bar`.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
#if ARKV_EVICT_FIRST
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(stream_policy())
        : "memory");
#else
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
        "[%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
        : "memory");
#endif
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

// Waits for a phase of `bar` at most kSpinLimit polls; false if it gave up.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) {
    for (int i = 0; i < kSpinLimit; ++i)
        if (mbar_try_wait(bar, parity)) return true;
    return false;
}

// Programmatic dependent launch: let the next kernel on the stream launch (its
// blocks take SM slots as this grid's blocks exit), and wait until the kernel
// before this one has finished with its writes visible.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// 4-byte asynchronous copy global -> shared (one cp.async group per commit).
__device__ __forceinline__ void cp_async4(uint32_t dst, const void* src) {
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// L2 prefetch of the 128-byte line holding `ptr`.
__device__ __forceinline__ void prefetch_l2(const void* ptr) {
    asm volatile("prefetch.global.L2 [%0];" ::"l"(ptr) : "memory");
}

// atomicAdd(p, 1) with acquire-release semantics at device scope.
__device__ __forceinline__ unsigned ticket_acq_rel(unsigned* p) {
    unsigned old;
    asm volatile("atom.add.acq_rel.gpu.u32 %0, [%1], 1;" : "=r"(old) : "l"(p) : "memory");
    return old;
}

__device__ __forceinline__ void prefetch_map(const CUtensorMap* m) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// d += a * b on m16n8k16 (f16 or bf16 operands, float32 accumulate).
template <bool F16>
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    if constexpr (F16)
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
    else
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// Two 16 x 16-byte matrices, transposed (rows from lanes 0..15, then 16..31): lane
// (g, t) receives, of each matrix, the rows its lanes 4t..4t+3 supplied at byte
// column g (r[0], r[2]) and g + 8 (r[1], r[3]).
__device__ __forceinline__ void ldsm_b8_x2_trans(uint32_t (&r)[4], uint32_t addr) {
    asm volatile("ldmatrix.sync.aligned.m16n16.x2.trans.shared.b8 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}

// Transpose of an 8 x 8 matrix of 16-bit elements held one row pair per lane (lane
// 4 r + c holds row r, columns 2c, 2c + 1): afterwards lane 4 r + c holds row r of
// the transpose, i.e. column r of the input at rows 2c, 2c + 1.
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t a) {
    uint32_t d;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
    return d;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
    __half2 v = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Four FP8 codes (low byte first) -> two f16x2 words (codes 0,1 and 2,3), exact.
// E4M3: the hardware conversion.  E5M2 is the upper byte of an f16 with the same
// value, so the codes only move into place.
template <int FMT>
__device__ __forceinline__ void fp8x4_to_f16(uint32_t w, uint32_t& lo, uint32_t& hi) {
    if constexpr (FMT == ARKV_FMT_E5M2) {
        lo = __byte_perm(w, 0u, 0x1404);   // bytes: 0, code 0, 0, code 1
        hi = __byte_perm(w, 0u, 0x3424);   // bytes: 0, code 2, 0, code 3
    } else {
        asm("{\n\t.reg .b16 a, b;\n\tmov.b32 {a, b}, %2;\n\t"
            "cvt.rn.f16x2.e4m3x2 %0, a;\n\tcvt.rn.f16x2.e4m3x2 %1, b;\n}"
            : "=r"(lo), "=r"(hi)
            : "r"(w));
    }
}

// 2^x, the special-function unit's approximation (relative error a few 2^-23).
__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ------------------------------------------------------------------ per-lane addresses
// Shared-memory byte offsets of the fragment loads of one lane, K from the tile's K
// slot and V from its V slot; index j = 0..3 selects a 32-byte column pair (two
// 16-byte chunks) of the row.  A bf16 tile has a K slot and a V slot; an FP8 tile
// holds K and V (16 x D bytes each) in one slot.  Fragment conventions of
// m16n8k16: lane = 4 g + t.
template <int D, bool FP8>
struct LaneOffsets {
    uint32_t k[4], v[4];
    __device__ __forceinline__ LaneOffsets() {
        const int lane = threadIdx.x & 31, m = lane >> 3;
        constexpr int VOFF = FP8 ? 16 * D : 0;   // a bf16 tile's V has a slot of its own
        if constexpr (!FP8) {
            // K, ldmatrix.x4: matrix m = (tokens 8 (m >> 1) .., chunk 2j + (m & 1)) -> the
            // B fragments (b0, b1) of n-tiles 0 and 1 for k block j (16 dims = 2 chunks).
            // V, ldmatrix.x4.trans, the same matrices -> the A fragment (a0, a1, a2, a3)
            // of V^T for the 16 dims of block j
            const int tk = (lane & 7) + 8 * (m >> 1);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                k[j] = swz_chunk<128>(tk, (2 * j + (m & 1)) & 7);
                v[j] = VOFF + k[j];
            }
        } else {
            constexpr int ROWB = D;   // one byte per dimension
            // K, ldmatrix.x4 of 8 rows x 16 bytes: lane (g, t) receives bytes 4t..4t+3
            // of token g (+8 for matrices 2, 3) in chunk 2j + (m & 1)
            const int tk = (lane & 7) + 8 * (m >> 1);
            // V, ldmatrix.m16n16.x2.trans.b8: lanes 0..15 supply the rows of matrix 0
            // (chunk 2j), lanes 16..31 those of matrix 1 (chunk 2j + 1), in the token
            // order 0,1,8,9,2,3,10,11,4,5,12,13,6,7,14,15
            const int i = lane & 15;
            const int tv = (i >> 2) * 2 + (i & 1) + 8 * ((i >> 1) & 1);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                k[j] = (2 * j < D / 16) ? swz_chunk<ROWB>(tk, 2 * j + (m & 1)) : 0u;
                v[j] = (2 * j < D / 16) ? VOFF + swz_chunk<ROWB>(tv, 2 * j + (lane >> 4)) : 0u;
            }
        }
    }
};

// ------------------------------------------------------------------ one tile
struct RowState {
    float m[2];   // reference maxima of this lane's two heads (raw logit units)
    float l[2];   // this lane's share of their sums of probabilities
};

// One 16-token tile (tokens t0 .. t0+15 of a segment ending at seg_end) held at
// shared address `st` (its first ring slot).
//
// S^T = K Q^T on m16n8k16: K is the A operand (16 tokens x 16 dims per k block, the
// same ldmatrix loads that would give it as a B operand, in another register order),
// and the queries are the B operand (qa: column n = head n & 3, so columns 4..7 repeat
// the group).  Lane (g, t) then holds the logits of tokens g and g + 8 for columns 2t
// and 2t + 1: heads 2t, 2t + 1 for t < 2, and the same heads again for t >= 2, whose
// lanes supply the low parts of P.  P (16 tokens x 8 columns [hi | lo], 16-bit) is
// taken to the B fragment of O^T += V^T P by two register transposes (movmatrix).
// The accumulator columns of a lane are its own two heads, so a change of the
// softmax reference rescales them without any exchange between lanes.
//
// skv/svv: FP8 scales of tokens g and g + 8 (unused for bf16); vnorm: the warp's
// V-scale normaliser.  hv0/hv1: the lane's heads are real; lo: the lane supplies low
// parts (t >= 2).  logit_row: the row's raw logits [head][lstride].  `sv` is the
// shared address of the V tile (the K slot's address for FP8 tiles); `mid` runs
// between QK^T and PV (it frees the K slot and waits for the V slot of a bf16 tile)
// and returns false if V did not arrive, in which case PV is skipped.
template <int D, bool FP8, int FMT, typename Mid>
__device__ __forceinline__ void attend_tile(uint32_t st, uint32_t sv, const LaneOffsets<D, FP8>& off, int t0,
                                            int seg_end, bool hv0, bool hv1, bool lo, float c2,
                                            const float (&skv)[2], const float (&svv)[2], float vnorm,
                                            float* logit_row, int lstride, const uint32_t (&qa)[D / 16][2],
                                            RowState& rs, float (&oacc)[D / 16][4], Mid&& mid) {
    constexpr int KB = D / 16;   // k blocks of QK^T, m-tiles of PV
    constexpr int C = kQkChains;
    const int lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;

    // ---- S^T = K Q^T, C independent accumulator chains (k blocks dealt round robin);
    // element e: (token g, column 2t), (g, 2t + 1), (g + 8, 2t), (g + 8, 2t + 1)
    float sa[C][4];
#pragma unroll
    for (int c = 0; c < C; ++c) sa[c][0] = sa[c][1] = sa[c][2] = sa[c][3] = 0.f;
    if constexpr (!FP8) {
        // ldmatrix.x4 of block kk: (tokens 0-7, dims 2t..), (tokens 0-7, dims 8+2t..),
        // (tokens 8-15, dims 2t..), (tokens 8-15, dims 8+2t..) = A fragment a0, a2, a1, a3
#pragma unroll
        for (int kk = 0; kk < KB; ++kk) {
            uint32_t a[4];
            ldsm_x4(a, st + off.k[kk & 3] + (kk >> 2) * 2048);
            mma16816<false>(sa[kk % C], a[0], a[2], a[1], a[3], qa[kk][0], qa[kk][1]);
        }
    } else {
        // words: (token g, block 2j), (g, 2j + 1), (g + 8, 2j), (g + 8, 2j + 1), each four
        // codes = dims 4t..4t+3 of the block: codes 0,1 at k = 2t, 2t+1, codes 2,3 at
        // k = 2t+8, 2t+9 (the queries' dims are ordered to match)
#pragma unroll
        for (int j = 0; j < KB / 2; ++j) {
            uint32_t w[4];
            ldsm_x4(w, st + off.k[j]);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t a0, a1, a2, a3;
                fp8x4_to_f16<FMT>(w[h], a0, a2);
                fp8x4_to_f16<FMT>(w[2 + h], a1, a3);
                const int kk = 2 * j + h;
                mma16816<true>(sa[kk % C], a0, a1, a2, a3, qa[kk][0], qa[kk][1]);
            }
        }
    }
#pragma unroll
    for (int c = 1; c < C; ++c) {
        sa[0][0] += sa[c][0]; sa[0][1] += sa[c][1]; sa[0][2] += sa[c][2]; sa[0][3] += sa[c][3];
    }
    float s[4] = {sa[0][0], sa[0][1], sa[0][2], sa[0][3]};
    if constexpr (FP8) {
        s[0] *= skv[0]; s[1] *= skv[0]; s[2] *= skv[1]; s[3] *= skv[1];
    }
    const int tA = t0 + g, tB = t0 + 8 + g;
    const bool inA = tA < seg_end, inB = tB < seg_end;
    const bool v[4] = {hv0 && inA, hv1 && inA, hv0 && inB, hv1 && inB};
    if (!lo) {   // raw logits for the score update, [head][slot]
        float* l0 = logit_row + (size_t)(2 * t) * lstride;
        float* l1 = l0 + lstride;
        if (v[0]) l0[tA] = s[0];
        if (v[1]) l1[tA] = s[1];
        if (v[2]) l0[tB] = s[2];
        if (v[3]) l1[tB] = s[3];
    }

    // ---- online softmax with a lazy reference per head (moves only past 2^8)
    float a[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) a[e] = (s[e] - rs.m[e & 1]) * c2;
    const bool need = (v[0] && a[0] > 8.f) || (v[1] && a[1] > 8.f) || (v[2] && a[2] > 8.f) || (v[3] && a[3] > 8.f);
    if (__any_sync(kFull, need)) {
        float mx[2] = {fmaxf(v[0] ? s[0] : kNegInf, v[2] ? s[2] : kNegInf),
                       fmaxf(v[1] ? s[1] : kNegInf, v[3] ? s[3] : kNegInf)};
        float al[2];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
#pragma unroll
            for (int m = 4; m <= 16; m <<= 1) mx[c] = fmaxf(mx[c], __shfl_xor_sync(kFull, mx[c], m));   // over tokens
            const float mn = fmaxf(rs.m[c], mx[c]);
            al[c] = (mn == rs.m[c] || rs.m[c] == kNegInf) ? (rs.m[c] == kNegInf ? 0.f : 1.f)
                                                           : ex2((rs.m[c] - mn) * c2);
            rs.m[c] = mn;
            rs.l[c] *= al[c];
        }
        if (al[0] != 1.f || al[1] != 1.f) {   // this lane's accumulator columns are its two heads
#pragma unroll
            for (int mt = 0; mt < KB; ++mt) {
                oacc[mt][0] *= al[0]; oacc[mt][1] *= al[1]; oacc[mt][2] *= al[0]; oacc[mt][3] *= al[1];
            }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) a[e] = (s[e] - rs.m[e & 1]) * c2;
    }
    float p[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) p[e] = v[e] ? ex2(a[e]) : 0.f;
    rs.l[0] += p[0] + p[2];
    rs.l[1] += p[1] + p[3];
    // the accumulator holds O * vnorm: FP8 tiles fold their V scale in as well
    const float fA = FP8 ? svv[0] * vnorm : vnorm, fB = FP8 ? svv[1] * vnorm : vnorm;
    p[0] *= fA; p[1] *= fA; p[2] *= fB; p[3] *= fB;
    // P rows g (tokens 0-7) and g + 8 (tokens 8-15), columns 2t, 2t + 1: high parts for
    // t < 2, low parts p - hi for t >= 2; transposed into the B fragment (k = tokens
    // 2t, 2t+1 in b0 and 8+2t, 9+2t in b1, n = column g)
    uint32_t r0, r1;
    if constexpr (FP8) {
        const uint32_t h0 = pack_f16(p[0], p[1]), h1 = pack_f16(p[2], p[3]);
        const __half2 x0 = *reinterpret_cast<const __half2*>(&h0), x1 = *reinterpret_cast<const __half2*>(&h1);
        r0 = lo ? pack_f16(p[0] - __low2float(x0), p[1] - __high2float(x0)) : h0;
        r1 = lo ? pack_f16(p[2] - __low2float(x1), p[3] - __high2float(x1)) : h1;
    } else {
        const uint32_t h0 = pack_bf16(p[0], p[1]), h1 = pack_bf16(p[2], p[3]);
        r0 = lo ? pack_bf16(p[0] - bf16_lo(h0), p[1] - bf16_hi(h0)) : h0;
        r1 = lo ? pack_bf16(p[2] - bf16_lo(h1), p[3] - bf16_hi(h1)) : h1;
    }
    const uint32_t b0 = movmatrix_trans(r0), b1 = movmatrix_trans(r1);

    // ---- O^T += V^T [P_hi | P_lo].  Past the segment end the tile holds stale slots or
    // zero fill: P is 0 there, and a partial tile also zeroes those V elements so that
    // no stale bit pattern can reach the accumulator (k = 2t, 2t+1: tokens 2t, 2t+1;
    // k = 2t+8, 2t+9: tokens 8+2t, 9+2t)
    const int kA = t0 + 2 * t, kB = t0 + 8 + 2 * t;
    const bool partial = t0 + 16 > seg_end;          // warp-uniform
    uint32_t m0 = 0xffffffffu, m1 = 0xffffffffu;
    if (partial) {
        m0 = (kA < seg_end ? 0xffffu : 0u) | (kA + 1 < seg_end ? 0xffff0000u : 0u);
        m1 = (kB < seg_end ? 0xffffu : 0u) | (kB + 1 < seg_end ? 0xffff0000u : 0u);
    }
    if (!mid()) return;
    if constexpr (!FP8) {
#pragma unroll
        for (int mt = 0; mt < KB; ++mt) {
            uint32_t af[4];   // A fragment of V^T for dims 16 mt .. 16 mt + 15
            ldsm_x4_trans(af, sv + off.v[mt & 3] + (mt >> 2) * 2048);
            if (partial) { af[0] &= m0; af[1] &= m0; af[2] &= m1; af[3] &= m1; }
            mma16816<false>(oacc[mt], af[0], af[1], af[2], af[3], b0, b1);
        }
    } else {
#pragma unroll
        for (int j = 0; j < KB / 2; ++j) {
            uint32_t r[4];   // chunk 2j: dims +g (r0), +8+g (r1); chunk 2j+1: r2, r3
            ldsm_b8_x2_trans(r, sv + off.v[j]);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                uint32_t a0, a2, a1, a3;
                fp8x4_to_f16<FMT>(r[2 * h], a0, a2);
                fp8x4_to_f16<FMT>(r[2 * h + 1], a1, a3);
                if (partial) { a0 &= m0; a1 &= m0; a2 &= m1; a3 &= m1; }
                mma16816<true>(oacc[2 * j + h], a0, a1, a2, a3, b0, b1);
            }
        }
    }
}

// Query fragments of column g of Q^T (the B operand of S^T = K Q^T: b0, b1 of every k
// block): head g & 3 (columns 0..3 and 4..7 repeat the group; heads >= G give zero):
// bf16 in natural dimension order; f16 for FP8 tiles, in the order of the 4-byte K
// words (dims 16 kk + 4t .. + 3).  qs: the group's queries in global memory, [G][D]
// bf16, read directly by every lane (an L2 hit after the prefetch).
template <int D>
__device__ __forceinline__ void load_q(const uint16_t* qs, bool fp8, int G, uint32_t (&qa)[D / 16][2]) {
    const int lane = threadIdx.x & 31, h = (lane >> 2) & 3, t = lane & 3;
    const bool ok = h < G;   // rows of heads >= G are zero
    const uint16_t* qrow = qs + (ok ? h : 0) * D;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t x = 0u, y = 0u;
        if (fp8) {
            const uint2 u = ok ? *reinterpret_cast<const uint2*>(qrow + 16 * kk + 4 * t) : make_uint2(0u, 0u);
            x = pack_f16(bf16_lo(u.x), bf16_hi(u.x));
            y = pack_f16(bf16_lo(u.y), bf16_hi(u.y));
        } else if (ok) {
            x = *reinterpret_cast<const uint32_t*>(qrow + 16 * kk + 2 * t);
            y = *reinterpret_cast<const uint32_t*>(qrow + 16 * kk + 2 * t + 8);
        }
        qa[kk][0] = x;
        qa[kk][1] = y;
    }
}

// This CTA's place in the grid: the call runs one wave of P CTAs, shared among the
// rows in proportion to their lengths.  Row r gets n_r = base(r+1) - base(r) >= 1
// CTAs, base(r) = r + F(Wb(r)), F(w) = floor((2 (P - R) w + Wtot) / (2 Wtot)) (the
// nearest integer to w (P - R) / Wtot, exact), with Wb(r) the summed lengths
// (ctx_len of the row's sequence + step + 1) of the rows before it.  F is monotone
// with F(0) = 0 and F(Wtot) = P - R; it is exact integer arithmetic on ctx_len
// (which no CTA modifies), so every CTA, and every thread that meets a boundary
// from either side, derives the same shares -- a floating-point F would not: equal
// lengths put w (P - R) / Wtot + 1/2 exactly on integers, where two evaluations of
// the same formula may round apart.  The CTA's 128 threads own
// contiguous runs of rows: one block scan gives Wb, and the thread whose run holds
// this CTA's row also hands over that row's counts, loaded with the lengths.
struct Share {
    int row, c, n, base, n16, n8;
};

__device__ __forceinline__ Share grid_share(const AttnParams& p, char* sm) {
    constexpr int kRowsReg = 4;   // rows per thread whose counts are loaded up front
    const LayerDims& d = p.d;
    int* out = reinterpret_cast<int*>(sm);
    long long* wsum = reinterpret_cast<long long*>(sm + 32);
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, bid = blockIdx.x;
    const int per = (d.R + kWarps * 32 - 1) / (kWarps * 32);
    const int r0 = min(d.R, tid * per), r1 = min(d.R, r0 + per);
    long long mine = 0;
    int c16[kRowsReg], c8[kRowsReg];
#pragma unroll
    for (int j = 0; j < kRowsReg; ++j) {
        const int r = r0 + j;
        c16[j] = r < r1 ? p.c.n_bf16[r] : 0;
        c8[j] = r < r1 ? p.c.n_fp8[r] : 0;
    }
    for (int r = r0; r < r1; ++r) mine += (long long)__ldg(&p.ctx_len[r / d.hkv]) + p.step + 1;
    long long incl = mine;
#pragma unroll
    for (int m = 1; m < 32; m <<= 1) {
        const long long y = __shfl_up_sync(kFull, incl, m);
        if (lane >= m) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    long long wb = incl - mine, tot = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
        const long long x = wsum[w];
        tot += x;
        if (w < warp) wb += x;
    }
    tot = tot > 0 ? tot : 1;
    const long long two_extra = 2ll * (gridDim.x - d.R), den = 2 * tot;
    // the quotient from a float64 estimate (within one of it: it is at most P) and an
    // exact integer correction, with no 64-bit division
    auto F = [&](long long w) {
        const long long num = two_extra * w + tot;
        long long q = (long long)((double)num / (double)den);
        while (q > 0 && q * den > num) --q;
        while ((q + 1) * den <= num) ++q;
        return (int)q;
    };
    for (int r = r0, j = 0; r < r1; ++r, ++j) {
        const long long L = (long long)__ldg(&p.ctx_len[r / d.hkv]) + p.step + 1;
        const int lo = r + F(wb), hi = r + 1 + F(wb + L);
        if (bid >= lo && bid < hi) {
            int n16 = 0, n8 = 0;
#pragma unroll
            for (int k = 0; k < kRowsReg; ++k)
                if (k == j) { n16 = c16[k]; n8 = c8[k]; }
            if (j >= kRowsReg) { n16 = p.c.n_bf16[r]; n8 = p.c.n_fp8[r]; }
            out[0] = r; out[1] = bid - lo; out[2] = hi - lo; out[3] = lo; out[4] = n16; out[5] = n8;
        }
        wb += L;
    }
    __syncthreads();
    return Share{out[0], out[1], out[2], out[3], out[4], out[5]};
}

// The CTA's tiles: bf16 tiles [a16, e16) and FP8 tiles [a8, e8) of its row (16
// tokens each), shared among the warps as described at the tile list below.  Each
// warp streams its tiles, the two kinds interleaved, through
// its own ring of kSlots slots (a bf16 tile takes two, an FP8 tile one) filled by
// TMA; an FP8 tile's 16 K and 16 V scales come with it, one 4-byte cp.async per lane
// into the slot's scale area (one cp.async group per issued tile).  The CTA then
// combines its warps into one (max, sum, unnormalised o) partial in slot blockIdx.x.
//
// With early_start the warps fill their rings before the wait for the previous
// kernel, so that this call's cache starts streaming while that kernel finishes.
// The tiles cover the row's tokens before this call's append; the new token is
// attended by the row's merge.
//
// The V scale is folded into P in f16, so P is also multiplied by vnorm = 64 / (the
// largest V scale among the warp's FP8 tiles so far): p sv vnorm <= 2^8 * 64 stays
// inside f16 and well above its subnormals.  vnorm starts at 1 and the accumulator
// is rescaled when an FP8 tile raises the maximum; since the accumulator holds
// O * vnorm, bf16 tiles multiply their P by the current vnorm too.  It comes back
// out of the partial.
template <int D, int FMT>
__device__ __forceinline__ void cta_body(const AttnParams& p, char* smem, int row, int n16, int n8, int a16,
                                         int e16, int a8, int e8) {
    using SL = Smem<D>;
    constexpr int KB = D / 16;
    constexpr int SLOT = SL::kSlot;
    const LayerDims& d = p.d;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = lane >> 2, t = lane & 3;
    const uint32_t sbase = smem_u32(smem);
    const uint32_t ring = sbase + warp * kSlots * SLOT;
    const uint32_t bars = sbase + SL::kBars + warp * kSlots * 8;
    int* sm_abort = reinterpret_cast<int*>(smem + SL::kAbort);
    int* sm_tq = reinterpret_cast<int*>(smem + SL::kTileq) + warp * kSlots;      // (tile << 1) | fp8, by slot
    float* sm_sc = reinterpret_cast<float*>(smem + SL::kSc) + warp * kSlots * 32;  // scales, by slot
    const uint32_t sc_base = smem_u32(sm_sc);
    const int b = row / d.hkv, gk = row - b * d.hkv;

    // this warp's tiles: bf16 tiles warp, warp + 4, ... of [a16, e16) and its run of
    // FP8 tiles (warp_fp8_share: the four warps stream about the same bytes),
    // interleaved evenly (after i tiles, floor(i nt8 / nt) of them are FP8), so that
    // the FP8 tiles' heavier arithmetic per byte is spread over the whole stream
    const int L16 = e16 - a16, L8 = e8 - a8;
    const int nt16 = L16 > warp ? (L16 - warp + kWarps - 1) / kWarps : 0;
    int f8_start, nt8;
    warp_fp8_share(L16, L8, warp, &f8_start, &nt8);
    const int nt = nt16 + nt8;
    // producer state (every lane keeps it; lane 0 issues the tensor loads).  The ring
    // holds entries, one slot each: a bf16 tile is two (its K, then its V), so its K slot
    // is refilled as soon as QK^T has read it; an FP8 tile is one (K and V)
    int iss = 0, half = 0, ipos = 0, free_slots = kSlots, ient = 0;
    int berr = 0, i16 = 0, i8 = 0, enc = 0;   // the interleave (Bresenham) and the tile being issued
    auto try_issue = [&]() {
        while (iss < nt && free_slots > 0) {
            if (half == 0) {   // the next tile: (tile << 1) | fp8
                berr += nt8;
                if (berr >= nt) {
                    berr -= nt;
                    enc = ((a8 + f8_start + i8++) << 1) | 1;
                } else {
                    enc = (a16 + warp + kWarps * i16++) << 1;
                }
            }
            const bool f8 = enc & 1;
            const int jt = enc >> 1;
            const uint32_t dst = ring + ipos * SLOT, bar = bars + 8 * ipos;
            if (lane == 0) {
                if (!f8) {
                    const int y = row * d.cap_o + 16 * jt;
                    const CUtensorMap* m = half == 0 ? &p.tm_k16 : &p.tm_v16;
                    mbar_expect_tx(bar, SLOT);
#pragma unroll
                    for (int bx = 0; bx < D * 2 / 128; ++bx) tma_load_2d(dst + bx * 2048, m, bx * 64, y, bar);
                } else {
                    const int y = row * d.cap_q + 16 * jt;
                    mbar_expect_tx(bar, 2 * 16 * D);
                    tma_load_2d(dst, &p.tm_k8, 0, y, bar);
                    tma_load_2d(dst + 16 * D, &p.tm_v8, 0, y, bar);
                }
            }
            if (f8) {   // lanes 0..15: K scales of the tile's tokens, 16..31: V scales
                const int tok = min(16 * jt + (lane & 15), d.cap_q - 1);
                cp_async4(sc_base + (ipos * 32 + lane) * 4,
                          (lane < 16 ? p.c.sk : p.c.sv) + (size_t)row * d.cap_q + tok);
            }
            cp_async_commit();   // one group per entry
            sm_tq[ipos] = enc;
            ipos = (ipos + 1) & (kSlots - 1);
            --free_slots;
            ++ient;
            if (f8 || half == 1) {
                ++iss;
                half = 0;
            } else {
                half = 1;
            }
        }
    };
    try_issue();

    // this lane's heads: columns 2t, 2t + 1 of S^T, heads (2t) & 3 and (2t + 1) & 3;
    // lanes t >= 2 repeat those of t - 2 and supply the low parts of P
    const bool hv0 = ((2 * t) & 3) < d.G, hv1 = ((2 * t + 1) & 3) < d.G, lo = t >= 2;
    const float c2 = (float)(p.inv_sqrt_d * 1.4426950408889634);   // log2(e) / sqrt(D)
    RowState rs{{kNegInf, kNegInf}, {0.f, 0.f}};
    float oacc[KB][4];
#pragma unroll
    for (int mt = 0; mt < KB; ++mt) oacc[mt][0] = oacc[mt][1] = oacc[mt][2] = oacc[mt][3] = 0.f;

    // everything above read only this layer's cache and ctx_len; q, k_new, v_new and
    // the workspace may come from the previous kernel.  Before the wait (with
    // early_start) the group's queries are only prefetched to L2 (a prefetch reads
    // nothing the kernel uses: L2 stays coherent with the previous kernel's writes),
    // and so are the row's new key and value, which the row's merge reads at the very
    // end of the call, when the next call's ring fills keep HBM busy (0.35 us per call
    // at the LLaMA3-8B shape)
    constexpr int kLines = D * 2 / 128;   // 128-byte lines of one bf16 row
    if (tid < 4 * kLines && tid / kLines < d.G) {
        const int h = tid / kLines, c = tid % kLines;
        prefetch_l2(p.q + ((size_t)b * d.hq + gk * d.G + h) * D + 64 * c);
    }
    if (tid >= 32 && tid < 32 + 2 * kLines) {
        const int w = (tid - 32) / kLines, c = (tid - 32) % kLines;
        prefetch_l2((w == 0 ? p.k_new : p.v_new) + ((size_t)b * d.hkv + gk) * D + 64 * c);
    }
    if (p.early_start) pdl_wait();

    int pos = 0;          // ring slot of the next entry to consume
    uint32_t ph = 0;      // parity of every slot's next phase
    int cent = 0;         // entries consumed
    bool aborted = false;
    auto wait_entry = [&]() -> bool {
        if (mbar_wait(bars + 8 * pos, (ph >> pos) & 1u)) return true;
        // a copy did not land in time: flag it, give every copy this warp has in flight
        // (this one included) a last bounded chance to land, and leave the ring alone
        if (lane == 0) {
            atomicOr(p.c.status, ARKV_STATUS_TIMEOUT);
            atomicExch(sm_abort, 1);
        }
        uint32_t q = ph;
        for (int j = cent, sp = pos; j < ient; ++j) {
            mbar_wait(bars + 8 * sp, (q >> sp) & 1u);
            q ^= 1u << sp;
            sp = (sp + 1) & (kSlots - 1);
        }
        return false;
    };
    auto release = [&]() {   // frees the entry at pos
        ph ^= 1u << pos;
        pos = (pos + 1) & (kSlots - 1);
        ++free_slots;
        ++cent;
        __syncwarp();
        try_issue();
    };

    // query fragments for both kinds of tile (bf16 in natural dimension order, f16 in
    // the FP8 words' order), held for the whole interleaved stream
    uint32_t qa16[KB][2], qa8[KB][2];
    // (each warp loads its own fragments from global memory, an L2 hit after the
    // prefetch: no staging through shared memory and no block barrier before the stream)
    const uint16_t* qg = p.q + ((size_t)b * d.hq + gk * d.G) * D;   // the group's queries
    if (nt16 > 0) load_q<D>(qg, false, d.G, qa16);
    if (nt8 > 0) load_q<D>(qg, true, d.G, qa8);
    const LaneOffsets<D, false> off16;
    const LaneOffsets<D, true> off8;
    float* const logit16 = p.logit16 + (size_t)row * 4 * p.lstride_o;
    float* const logit8 = p.logit8 + (size_t)row * 4 * p.lstride_q;
    const float one[2] = {1.f, 1.f};
    // vcur: the largest V scale seen (0 before any FP8 tile); the accumulator holds
    // O * vnorm, so every tile's P, bf16 tiles' included, carries the current vnorm
    float vnorm = 1.f, vcur = 0.f;
    for (int i = 0; i < nt; ++i) {
        const int te = sm_tq[pos];
        const int t0 = 16 * (te >> 1);
        if (!wait_entry()) { aborted = true; break; }
        if (!(te & 1)) {   // ---- a bf16 tile: its K entry, then its V entry
            const uint32_t sk = ring + pos * SLOT, sv = ring + ((pos + 1) & (kSlots - 1)) * SLOT;
            bool v_ok = true;
            attend_tile<D, false, FMT>(sk, sv, off16, t0, n16, hv0, hv1, lo, c2, one, one, vnorm, logit16,
                                       p.lstride_o, qa16, rs, oacc,
                                       [&]() {   // K is read: free its slot, then wait for V
                                           release();
                                           v_ok = wait_entry();
                                           return v_ok;
                                       });
            if (!v_ok) { aborted = true; break; }
            release();
        } else {           // ---- an FP8 tile: K and V in one entry, scales beside it
            // this tile's scale group (the groups of later entries may still be in flight)
            switch (ient - cent - 1) {
                case 0: cp_async_wait<0>(); break;
                case 1: cp_async_wait<1>(); break;
                case 2: cp_async_wait<2>(); break;
                default: cp_async_wait<3>(); break;
            }
            __syncwarp();
            // scales of this lane's tokens g and g + 8; zero past the segment end, where P
            // is zero and a stale scale (NaN or Inf bits included) must not reach p * sv
            const float* sc = sm_sc + pos * 32;
            const bool okA = t0 + g < n8, okB = t0 + 8 + g < n8;
            const float skv[2] = {okA ? sc[g] : 0.f, okB ? sc[8 + g] : 0.f};
            const float svv[2] = {okA ? sc[16 + g] : 0.f, okB ? sc[24 + g] : 0.f};
            float m = fmaxf(svv[0], svv[1]);
#pragma unroll
            for (int x = 4; x <= 16; x <<= 1) m = fmaxf(m, __shfl_xor_sync(kFull, m, x));   // the tile's largest V scale
            if (m > vcur) {
                const float vn = 64.f / m, f = vn / vnorm;
#pragma unroll
                for (int mt = 0; mt < KB; ++mt) {
                    oacc[mt][0] *= f; oacc[mt][1] *= f; oacc[mt][2] *= f; oacc[mt][3] *= f;
                }
                vnorm = vn;
                vcur = m;
            }
            const uint32_t st = ring + pos * SLOT;
            attend_tile<D, true, FMT>(st, st, off8, t0, n8, hv0, hv1, lo, c2, skv, svv, vnorm, logit8, p.lstride_q,
                                      qa8, rs, oacc, []() { return true; });
            release();
        }
    }
    cp_async_wait<0>();

    __syncthreads();   // every warp has drained its ring: the epilogue may reuse it
    const size_t pb = blockIdx.x;
    if (*sm_abort) {
        // a wait gave up: copies may still be landing in the ring, so write an empty
        // partial (weight 0 in the merge) without touching shared memory; the status
        // bit already tells the caller that this call's output is not to be used
        for (int idx = tid; idx < 4 * D; idx += blockDim.x) {
            p.part_o[(pb * 4 + idx / D) * D + idx % D] = 0.f;
            if (idx % D == 0) p.part_ml[pb * 4 + idx / D] = make_float2(kNegInf, 0.f);
        }
        return;   // the caller still takes the row's ticket
    }
    float (*sm_o)[4][D] = reinterpret_cast<float (*)[4][D]>(smem + SL::kO);
    float (*sm_m)[4] = reinterpret_cast<float (*)[4]>(smem + SL::kM);
    float (*sm_l)[4] = reinterpret_cast<float (*)[4]>(smem + SL::kL);
    float (*sm_w)[4] = reinterpret_cast<float (*)[4]>(smem + SL::kRed);
    float* sm_max = reinterpret_cast<float*>(smem + SL::kMax);
    // warp totals: l of heads 2t, 2t + 1 over the 8 lanes of column pair t (lanes t >= 2
    // repeat t - 2).  o: oacc[mt] = O^T at dims 16 mt + g (c0, c1) and 16 mt + g + 8
    // (c2, c3), columns 2t, 2t+1; columns 0..3 hold the high part, 4..7 the low part of
    // heads 0..3, so lanes t and t ^ 2 add up.  The accumulator carries vnorm, taken out
    // here.
    float l0 = rs.l[0], l1 = rs.l[1];
#pragma unroll
    for (int x = 4; x <= 16; x <<= 1) {
        l0 += __shfl_xor_sync(kFull, l0, x);
        l1 += __shfl_xor_sync(kFull, l1, x);
    }
    const float un = vcur > 0.f ? vcur * (1.f / 64.f) : 1.f;   // 1 / vnorm
#pragma unroll
    for (int mt = 0; mt < KB; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) oacc[mt][e] += __shfl_xor_sync(kFull, oacc[mt][e], 2);
    if (t < 2) {
#pragma unroll
        for (int mt = 0; mt < KB; ++mt) {
            sm_o[warp][2 * t][16 * mt + g] = oacc[mt][0] * un;
            sm_o[warp][2 * t + 1][16 * mt + g] = oacc[mt][1] * un;
            sm_o[warp][2 * t][16 * mt + g + 8] = oacc[mt][2] * un;
            sm_o[warp][2 * t + 1][16 * mt + g + 8] = oacc[mt][3] * un;
        }
    }
    if (lane < 2) {   // g = 0, t = lane: heads 2t, 2t + 1
        sm_l[warp][2 * lane] = l0;
        sm_l[warp][2 * lane + 1] = l1;
        sm_m[warp][2 * lane] = rs.m[0];
        sm_m[warp][2 * lane + 1] = rs.m[1];
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

// The row's merge, run by the last of its CTAs to finish: M = max of the partial
// maxima, L = sum of l_s exp((m_s - M)/sqrt(D)), o = sum of o_s exp(..) / L over
// the row's partials (slots base .. base + n - 1), for every head of the group,
// one warp per head (lane l owns dims 4l .. 4l+3 for D = 128, 2l, 2l+1 for D = 64).
// The partials are taken kBatch at a time with every load of a batch in flight at
// once (lane q < kBatch also loads (m, l) of partial q); a batch whose maximum
// exceeds the running M rescales what came before.  Partials with l = 0 carry no
// weight and do not enter M.
// The new token (slot s_new >= 0; -1: the bf16 segment is full and the token is
// dropped) enters here as one more term: its logit q . k_new (float32 products of
// the bf16 values, summed over the warp), its weight exp((q.k - M')/sqrt(D)) and
// its value v_new; its raw logit goes to the workspace with the others, and the
// token is stored in slot s_new at position pos_new for later calls (no tensor load
// of this call reads that slot).  Publishes (M, L) for the score update.  Every
// global load of the merge is issued before its arithmetic, so that the merge ends in
// stores only.
template <int D>
__device__ __forceinline__ void row_merge(const AttnParams& p, int row, int base, int n, int s_new, int pos_new) {
    constexpr int VEC = D / 32;
    constexpr int kBatch = 16;
    const LayerDims& d = p.d;
    const int lane = threadIdx.x & 31, h = threadIdx.x >> 5;
    if (h >= d.G) return;
    const int b = row / d.hkv, gk = row - b * d.hkv;
    const float2* pml = p.part_ml + (size_t)base * 4 + h;
    const float* po = p.part_o + ((size_t)base * 4 + h) * D + VEC * lane;
    // the new token's query, key and value dims of this lane, loaded with the first batch
    const uint16_t* qh = p.q + ((size_t)b * d.hq + gk * d.G + h) * D + VEC * lane;
    const uint16_t* kn = p.k_new + ((size_t)b * d.hkv + gk) * D + VEC * lane;
    const uint16_t* vn = p.v_new + ((size_t)b * d.hkv + gk) * D + VEC * lane;
    uint2 q2 = make_uint2(0u, 0u), k2 = q2, v2 = q2;
    if (s_new >= 0) {
        if constexpr (VEC == 4) {
            q2 = *reinterpret_cast<const uint2*>(qh); k2 = *reinterpret_cast<const uint2*>(kn);
            v2 = *reinterpret_cast<const uint2*>(vn);
        } else {
            q2.x = *reinterpret_cast<const uint32_t*>(qh); k2.x = *reinterpret_cast<const uint32_t*>(kn);
            v2.x = *reinterpret_cast<const uint32_t*>(vn);
        }
    }
    float M = kNegInf, L = 0.f, acc[VEC];
#pragma unroll
    for (int e = 0; e < VEC; ++e) acc[e] = 0.f;
    for (int j0 = 0; j0 < n; j0 += kBatch) {
        const int cnt = min(kBatch, n - j0);
        const float2 ml = lane < cnt ? __ldcg(pml + (size_t)(j0 + lane) * 4) : make_float2(kNegInf, 0.f);
        float v[kBatch][VEC];
#pragma unroll
        for (int q = 0; q < kBatch; ++q) {
            const float* src = po + (size_t)(j0 + q) * 4 * D;
            if constexpr (VEC == 4) {
                const float4 x = q < cnt ? __ldcg(reinterpret_cast<const float4*>(src)) : make_float4(0.f, 0.f, 0.f, 0.f);
                v[q][0] = x.x; v[q][1] = x.y; v[q][2] = x.z; v[q][3] = x.w;
            } else {
                const float2 x = q < cnt ? __ldcg(reinterpret_cast<const float2*>(src)) : make_float2(0.f, 0.f);
                v[q][0] = x.x; v[q][1] = x.y;
            }
        }
        float mb = ml.y > 0.f ? ml.x : kNegInf;
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) mb = fmaxf(mb, __shfl_xor_sync(kFull, mb, m));
        if (mb == kNegInf) continue;                            // warp-uniform: no weight in this batch
        if (mb > M) {
            const float sc = M == kNegInf ? 0.f : exp_scaled(M, mb, p.inv_sqrt_d);
            L *= sc;
#pragma unroll
            for (int e = 0; e < VEC; ++e) acc[e] *= sc;
            M = mb;
        }
        const float wl = ml.y > 0.f ? exp_scaled(ml.x, M, p.inv_sqrt_d) : 0.f;
        L = fmaf(ml.y, wl, L);
#pragma unroll
        for (int q = 0; q < kBatch; ++q) {
            const float w = __shfl_sync(kFull, wl, q);
#pragma unroll
            for (int e = 0; e < VEC; ++e) acc[e] = fmaf(v[q][e], w, acc[e]);
        }
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) L += __shfl_xor_sync(kFull, L, m);
    if (s_new >= 0) {
        float kv[VEC], vv[VEC], qv[VEC];
        qv[0] = bf16_lo(q2.x); qv[1] = bf16_hi(q2.x);
        kv[0] = bf16_lo(k2.x); kv[1] = bf16_hi(k2.x);
        vv[0] = bf16_lo(v2.x); vv[1] = bf16_hi(v2.x);
        if constexpr (VEC == 4) {
            qv[2] = bf16_lo(q2.y); qv[3] = bf16_hi(q2.y);
            kv[2] = bf16_lo(k2.y); kv[3] = bf16_hi(k2.y);
            vv[2] = bf16_lo(v2.y); vv[3] = bf16_hi(v2.y);
        }
        float sdot = 0.f;
#pragma unroll
        for (int e = 0; e < VEC; ++e) sdot = fmaf(qv[e], kv[e], sdot);
#pragma unroll
        for (int m = 16; m >= 1; m >>= 1) sdot += __shfl_xor_sync(kFull, sdot, m);
        const float Mn = fmaxf(M, sdot);
        const float sc = M == kNegInf ? 0.f : exp_scaled(M, Mn, p.inv_sqrt_d);
        const float wn = exp_scaled(sdot, Mn, p.inv_sqrt_d);
        L = fmaf(L, sc, wn);
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc[e] = fmaf(acc[e], sc, wn * vv[e]);
        M = Mn;
        if (lane == 0) p.logit16[((size_t)row * 4 + h) * p.lstride_o + s_new] = sdot;
        if (h == 0) {   // the token into slot s_new for the calls that follow
            const size_t s16 = (size_t)row * d.cap_o + s_new;
            if constexpr (VEC == 4) {
                *reinterpret_cast<uint2*>(p.c.k16 + s16 * D + VEC * lane) = k2;
                *reinterpret_cast<uint2*>(p.c.v16 + s16 * D + VEC * lane) = v2;
            } else {
                *reinterpret_cast<uint32_t*>(p.c.k16 + s16 * D + VEC * lane) = k2.x;
                *reinterpret_cast<uint32_t*>(p.c.v16 + s16 * D + VEC * lane) = v2.x;
            }
            if (lane == 0) {
                p.c.pos16[s16] = pos_new;
                p.c.mu16[s16] = 0.0;
                p.c.m2_16[s16] = 0.0;
            }
        }
    }
    float* out = p.o + ((size_t)b * d.hq + gk * d.G + h) * D + VEC * lane;
    const float inv = 1.f / L;
    if constexpr (VEC == 4)
        *reinterpret_cast<float4*>(out) = make_float4(acc[0] * inv, acc[1] * inv, acc[2] * inv, acc[3] * inv);
    else
        *reinterpret_cast<float2*>(out) = make_float2(acc[0] * inv, acc[1] * inv);
    if (lane == 0) p.ml[(size_t)row * 4 + h] = make_float2(M, L);
}

template <int D, int FMT>
__global__ void __launch_bounds__(32 * kWarps, ARKV_MIN_CTAS) decode_attn_kernel(const __grid_constant__ AttnParams p) {
    using SL = Smem<D>;
    const LayerDims& d = p.d;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    __shared__ unsigned sm_ticket;
    extern __shared__ char smem_raw[];
    char* smem = reinterpret_cast<char*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    pdl_launch_dependents();
    if (tid == 0) {
        prefetch_map(&p.tm_k16); prefetch_map(&p.tm_v16); prefetch_map(&p.tm_k8); prefetch_map(&p.tm_v8);
    }
    if (!p.early_start) pdl_wait();
    const Share sh = grid_share(p, smem + SL::kShare);
    const int row = sh.row;

    // the row's counts, read once by every CTA of the row; the last one to finish
    // advances n_bf16, so no CTA of the row can see the advanced count
    const int n16 = min(max(sh.n16, 0), d.cap_o);   // counts are clamped to the
    const int n8 = min(max(sh.n8, 0), d.cap_q);      // capacities before any use
    const bool append = n16 < d.cap_o;               // the new token goes to slot n16
    const int pos_new = p.ctx_len[row / d.hkv] + p.step;   // at this position (read at entry)
    // this CTA's share of the row: about the same fraction of each segment's 16-token
    // tiles, so that every CTA of the row has about the same mix of bf16 and FP8 work
    // (the FP8 split evens out the ring entries: fp8_tiles_before)
    const int T16 = (n16 + 15) / 16, T8 = (n8 + 15) / 16;
    const int a16 = (int)((long long)T16 * sh.c / sh.n), e16 = (int)((long long)T16 * (sh.c + 1) / sh.n);
    const int a8 = fp8_tiles_before(T16, T8, sh.n, sh.c), e8 = fp8_tiles_before(T16, T8, sh.n, sh.c + 1);

    if (e16 > a16 || e8 > a8) {
        if (lane == 0) {
            const uint32_t bars = smem_u32(smem + SL::kBars) + warp * kSlots * 8;
#pragma unroll
            for (int st = 0; st < kSlots; ++st) mbar_init(bars + 8 * st, 1);
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
        if (tid == 0) *reinterpret_cast<int*>(smem + SL::kAbort) = 0;
        __syncthreads();
        cta_body<D, FMT>(p, smem, row, n16, n8, a16, e16, a8, e8);
    } else {
        if (p.early_start) pdl_wait();
        for (int idx = tid; idx < 4 * D; idx += blockDim.x) {   // nothing to attend: an empty partial
            p.part_o[(size_t)blockIdx.x * 4 * D + idx] = 0.f;
            if (idx < 4) p.part_ml[(size_t)blockIdx.x * 4 + idx] = make_float2(kNegInf, 0.f);
        }
    }

    // the row's ticket: every CTA of the row takes one after its partial is written.
    // Thread 0's acquire-release atomic is cumulative over the CTA's writes ordered
    // before it by the barrier (release), and the barrier after it orders the last
    // CTA's reads of the other partials after it (acquire); the last one merges and
    // moves the bf16 count
    __syncthreads();
    if (tid == 0) sm_ticket = ticket_acq_rel(&p.counter[row]);
    __syncthreads();
    if (sm_ticket != (unsigned)(sh.n - 1)) return;
    row_merge<D>(p, row, sh.base, sh.n, append ? n16 : -1, pos_new);
    if (tid == 0) {
        p.counter[row] = 0u;                                   // ready for the next call
        if (append) p.c.n_bf16[row] = n16 + 1;
        else atomicOr(p.c.status, ARKV_STATUS_BF16_FULL);      // the new token was dropped
    }
}

// One thread per live slot: x = sum over the group's heads of exp((raw - M)/sqrt(D)) / L,
// then one Welford step with the token's observation count (float64 state).
__global__ void __launch_bounds__(256) score_update_kernel(const ScoreParams p) {
    const LayerDims& d = p.d;
    const int row = blockIdx.y, b = row / d.hkv;
    __shared__ float sm_m[4];
    __shared__ double sm_il[4];   // 1 / L of every head
    if (threadIdx.x < 4) {
        const float2 ml = __ldg(&p.ml[(size_t)row * 4 + threadIdx.x]);
        sm_m[threadIdx.x] = ml.x;
        sm_il[threadIdx.x] = 1.0 / (double)ml.y;
    }
    __syncthreads();
    const int n16 = min(max(__ldg(&p.c.n_bf16[row]), 0), d.cap_o);
    const int n8 = min(max(__ldg(&p.c.n_fp8[row]), 0), d.cap_q);
    const int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n16 + n8) return;
    const bool bf = i < n16;
    const int slot = bf ? i : i - n16;
    const size_t sl = bf ? (size_t)row * d.cap_o + slot : (size_t)row * d.cap_q + slot;
    const float* lg = bf ? p.logit16 + (size_t)row * 4 * p.lstride_o + slot
                         : p.logit8 + (size_t)row * 4 * p.lstride_q + slot;
    const size_t hs = bf ? p.lstride_o : p.lstride_q;
    const int pos = __ldg(bf ? p.c.pos16 + sl : p.c.pos8 + sl);
    double* __restrict__ mu = bf ? p.c.mu16 + sl : p.c.mu8 + sl;
    double* __restrict__ m2 = bf ? p.c.m2_16 + sl : p.c.m2_8 + sl;
    float raw[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) raw[h] = h < d.G ? __ldg(lg + h * hs) : 0.f;
    const double mu_old = *mu, m2_old = *m2;
    double x = 0.0;
#pragma unroll
    for (int h = 0; h < 4; ++h)
        if (h < d.G) x += (double)exp_scaled(raw[h], sm_m[h], p.inv_sqrt_d) * sm_il[h];
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
    w.parts = d.R > kMaxGrid ? d.R : kMaxGrid;
    w.lstride_o = (d.cap_o + 3) & ~3;   // logit rows padded to 16 bytes
    w.lstride_q = (d.cap_q + 3) & ~3;
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    size_t off = 0;
    w.counter = off; off = al(off + sizeof(unsigned) * d.R);
    w.ml = off;      off = al(off + sizeof(float2) * d.R * 4);
    w.part_ml = off; off = al(off + sizeof(float2) * (size_t)w.parts * 4);
    w.part_o = off;  off = al(off + sizeof(float) * (size_t)w.parts * 4 * d.D);
    w.logit16 = off; off = al(off + sizeof(float) * 4 * (size_t)d.R * w.lstride_o);
    w.logit8 = off;  off = al(off + sizeof(float) * 4 * (size_t)d.R * w.lstride_q);
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
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    static unsigned char done[4][64];
    static int resident[4][64];   // CTAs of the kernel one SM holds, per device
    static int sms[64];
    auto go = [&](auto kernel, int which, int bytes) {
        cudaError_t err = allow_max_dyn_smem(kernel, done[which]);
        if (err != cudaSuccess) return err;
        if (dev < 64 && resident[which][dev] == 0) {
            int n = 0, m = 0;
            if ((err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, kernel, 32 * kWarps, bytes)) != cudaSuccess)
                return err;
            if ((err = cudaDeviceGetAttribute(&m, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return err;
            sms[dev] = m;
            resident[which][dev] = n > 0 ? n : 1;
        }
        // one wave of CTAs, at most one per 16 units (eight bf16 tiles) of the largest
        // cache, at least one per row.  When a multiple of R keeps at least 7/8 of the
        // wave it is taken: rows of equal length then get equal numbers of CTAs (with 412
        // CTAs for 32 rows, 4 rows get 12 and carry 8% more per CTA, and set the tail)
        const long long units = (long long)d.R * (2 * ((d.cap_o + 16) / 16) + (d.cap_q + 15) / 16);
        long long P = dev < 64 ? (long long)sms[dev] * resident[which][dev] : 444;
        if (kRowMultiple && d.R <= P && (P / d.R) * d.R * 8 >= P * 7) P = (P / d.R) * d.R;
        P = P < units / 16 ? P : units / 16;
        if (P > kMaxGrid) P = kMaxGrid;
        if (P < d.R) P = d.R;
        // a programmatic dependent of the previous kernel on the stream (the kernel
        // waits for it with griddepcontrol.wait before it reads what that kernel may write)
        cudaLaunchConfig_t lc{};
        lc.gridDim = dim3((unsigned)P);
        lc.blockDim = dim3(32 * kWarps);
        lc.dynamicSmemBytes = (size_t)bytes;
        lc.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        lc.attrs = attr;
        lc.numAttrs = 1;
        return cudaLaunchKernelEx(&lc, kernel, p);
    };
    if (D == 128)
        e = d.fmt == ARKV_FMT_E5M2 ? go(decode_attn_kernel<128, ARKV_FMT_E5M2>, 0, Smem<128>::kBytes)
                                   : go(decode_attn_kernel<128, ARKV_FMT_E4M3>, 1, Smem<128>::kBytes);
    else
        e = d.fmt == ARKV_FMT_E5M2 ? go(decode_attn_kernel<64, ARKV_FMT_E5M2>, 2, Smem<64>::kBytes)
                                   : go(decode_attn_kernel<64, ARKV_FMT_E4M3>, 3, Smem<64>::kBytes);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_score_update(const ScoreParams& p, cudaStream_t s) {
    const dim3 grid((p.d.cap_o + p.d.cap_q + 255) / 256, p.d.R);
    score_update_kernel<<<grid, 256, 0, s>>>(p);
    return cudaGetLastError();
}

}  // namespace arkv
