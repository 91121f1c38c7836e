// ssa_fused.cuh -- the fused, persistent decode kernel for bf16, d in {64,128}.
//
// One cooperative launch runs the whole decode step ("Simplified Sparse
// Attention via Gist Tokens": sec. 3.2 gist scoring, sec. 3.3 top-k and hybrid
// attention over the unfolded context, sec. 3.5 coarse-to-fine selection,
// sec. 3.6 split partial attention plus combination).
//
// Static, byte-balanced schedule.  The work of a call is laid out as global
// lists; each is the concatenation over (sequence, KV head) pairs of that
// pair's elements:
//   SCORE  summary slots to score: chunks (single level) or superchunks
//   META   64-row tiles of meta-gist K/V                       (two level)
//   CAND   candidate chunks to score                           (two level)
//   GIST   64-row tiles of gist K/V: every complete chunk (single level) or
//          the candidate chunks (two level)
//   RAW    64-row tiles of raw K/V: the selected chunks, then the tail
// Every block takes an equal contiguous share of every list.  A share may
// cross pair boundaries; a (block, pair) intersection is a segment and yields
// one partial (m, l, o) per query head.  Each block runs, in this order: its
// SCORE share; the top-k of the pairs it owns; [its META share; its CAND
// share; the second top-k of its pairs;] its GIST share; its RAW share; the
// combination of the pairs whose last attention element it holds.  A wait (a
// pair's scores complete, a selection published, a pair's partials complete)
// is always on work of an earlier phase, which never waits on a later one,
// and all blocks are co-resident (cooperative launch), so every wait ends;
// each is also bounded.
//
// Logits mode (single level, whole step): the scoring phase keeps every
// head's logit of its gist rows in shared memory, and the gist phase streams
// only the values of the same rows (the block's gist share is its score
// share), so half the bytes go through the ring and most of them arrive
// while the top-k runs.
//
// Gist and meta tiles need the selection only to mask excluded rows, so the
// producer issues them before the selection exists and the consumers apply
// the mask once it is published: the selection latency hides behind loads.
//
// Block layout: 4 consumer warps + 1 producer warp.  The producer streams
// 64-row tiles with 2-D TMA (128-byte swizzle) into a ring of stages (slot A:
// keys, slot B: values; score and value-only stages use both slots for one
// kind of row).  Each consumer warp takes 16 rows of every 64-row box:
// Q.K^T and P.V run on tensor cores (mma.sync m16n8k16, bf16 in, fp32
// accumulate; the GQA group's query heads are the M rows; scoring uses the
// keys as M rows, 16 keys x 8 heads per MMA), the softmax is an fp32 online
// softmax in the log2 domain, and P enters the P.V product as bf16 hi + lo
// parts (~16 significant bits).
#pragma once

#include "ssa_device.cuh"
#include "ssa_internal.h"

namespace ssa {
namespace fused {

constexpr int kConsumerWarps = 4;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;
constexpr int kBoxRows = 64;          // rows per TMA box and per attention tile
constexpr int kRowmaxCap = 1024;      // summary rows per score sub-item
constexpr int kBarConsumers = 1;      // named barrier id of the consumer warps
constexpr int kMaxGrid = kFusedMaxGrid;
constexpr int kMaxTopkEntries = 1024;  // largest topk / topk_super the library accepts
constexpr int kLogitBytes = 16 * 1024; // shared memory for the kept logits (logits mode)
// P.V formulation: heads as the M rows of the MMA (false: heads as N, dims as M)
#ifndef SSA_PV_HEADS_M
#define SSA_PV_HEADS_M 1
#endif
constexpr bool kPvHeadsM = SSA_PV_HEADS_M != 0;
// P in the P.V products: bf16 hi + lo parts (about 16 mantissa bits), or
// the bf16 part alone (SSA_PV_LO=0: half the P.V tensor-core work)
#ifndef SSA_PV_LO
#define SSA_PV_LO 1
#endif
constexpr bool kPvLo = SSA_PV_LO != 0;

// Rows of kept logits a block can hold for G query heads, and the row stride
// of one head's logits (a multiple of 32 plus 8: conflict-free reads).
__host__ __device__ inline int logit_rows_cap(int G) {
    const int r = (kLogitBytes / (4 * G) - 8) / 32 * 32;
    return r > 0 ? r : 0;
}

enum : int { K_END = 0, K_SCORE = 1, K_ATTN = 2, K_SELECT = 3, K_COMBINE = 4, K_GISTV = 5 };
// F_SEGBEG / F_SEGEND: a scoring sub-item is the first / last of its segment
enum : int { F_FIRST = 1, F_LAST = 2, F_QLOAD = 4, F_SEGBEG = 8, F_SEGEND = 16 };
enum : int { L_SCORE = 0, L_CAND = 1, L_META = 2, L_GIST = 3, L_RAW = 4, kNumLists = 5 };
// what a K_SELECT stage does
enum : int { SEL_CHUNKS = 0, SEL_SUPER = 1, SEL_CAND = 2, SEL_VALIDATE = 3 };
// which published selection masks the rows of an attention segment
enum : int { MASK_NONE = 0, MASK_CHUNK = 1, MASK_SUPER = 2 };

// Control words: after a 64-word header (unused), one record of
// Plan::pair_ints words per pair:
//   line 0   completion counter: attention segments written;
//   line 1   published counts: count + 1 (0: not published yet; kBadBit:
//            the caller's selection was rejected);
//   then     the published selection, entry + 1 (0: not written yet): topk
//            chunk entries, then topk_super superchunk entries.
// Every word is written at most once per call and cleared by the pair's
// combination, so a reader needs no separate ready flag.
constexpr int kLineInts = 32;
constexpr int C_ARR = 2 * kLineInts;
enum : int {
    A_ATTN = 2,               // attention segments written
    A_COUNT = kLineInts,      // published chunk selection count
    A_SCOUNT = kLineInts + 1, // published superchunk selection count
    A_ENTRIES = 2 * kLineInts // chunk entries, then superchunk entries
};
constexpr int kBadBit = 1 << 30;

struct StageMeta {
    int kind, pair, nvalid, flags;
    // K_SCORE: a0 row offset in the sub-item, a1 slots, a2 -inf pad slots,
    //          a3 destination index, a4 rows per slot, a5 level (1: candidates)
    // K_ATTN:  a0 first summary row of the tile, a1 mask kind, a2 rows per
    //          masked slot, a3 attention list (0 META, 1 GIST, 2 RAW)
    // K_SELECT: a0 what to do (SEL_*)
    // K_GISTV: a0 first gist row of the stage (in the pair), a2 rows per chunk;
    //          slot A / slot B hold the values of rows 0..63 / 64..127
    int a0, a1, a2, a3, a4, a5;
    int pad0;
    int lrow;   // logits mode: row of the stage's first row in the block's kept logits
};

template <int D>
struct Cfg {
    static constexpr int kSlotBytes = kBoxRows * D * 2;
    static constexpr int kStageBytes = 2 * kSlotBytes;
    static constexpr int kStages = (D == 64) ? 6 : 3;
    static constexpr int kBoxBytes = kBoxRows * D * 2;  // one 64-row box, all D columns
};

struct SmemLayout {
    int ring, qbuf, qbytes, meta, bars, psel, psup, plan, bits, uni, logit, misc, total;
};

__host__ __device__ inline int mask_words_for(const Plan& p) { return (p.M_max + 31) / 32; }

template <int D>
__host__ __device__ inline SmemLayout smem_layout(const Plan& p) {
    SmemLayout L;
    const int NS = p.stages > 0 ? p.stages : Cfg<D>::kStages;
    const int G = p.G;
    int o = 0;
    L.ring = o;
    o += NS * Cfg<D>::kStageBytes;
    L.qbytes = ((G * D * 2) + 127) / 128 * 128;
    L.qbuf = o;
    o += NS * L.qbytes;
    L.meta = o;
    o += NS * (int)sizeof(StageMeta);
    o = (o + 15) / 16 * 16;
    L.bars = o;
    o += 2 * NS * 8;
    L.psel = o;
    o += ((p.topk + 3) / 4 * 4) * 4;
    L.psup = o;
    o += (((p.h2 ? p.topk_super : 0) + 3) / 4 * 4) * 4;
    L.plan = o;  // lengths [B], then per list prefixes [B + 1]
    o += (p.B + kNumLists * (p.B + 1)) * 4;
    o = (o + 15) / 16 * 16;
    L.bits = o;  // selection bitmap of the current segment's pair
    o += ((mask_words_for(p) + 3) / 4 * 4) * 4;
    L.uni = o;
    // the consumers use this area for one thing at a time
    int u = kRowmaxCap * 4 + kConsumerWarps * 32 * 8;           // score rows + lists
    const int tk = (int)sizeof(TopkScratch);                     // top-k
    u = u > tk ? u : tk;
    const int mg = kConsumerWarps * G * (D + 2) * 4;             // warp merge
    u = u > mg ? u : mg;
    o += (u + 15) / 16 * 16;
    L.logit = o;
    // + 128 rows of padding: a 128-row tile's reads may run past the last
    // head's kept rows (those rows are masked, but stay inside the area)
    if (p.logits) o += (G * p.logit_stride + 128) * 4;
    L.misc = o;
    o += 64;
    L.total = o + 1024;  // slack to align the ring to 1024 bytes
    return L;
}

// Timeline trace: builds compiled with SSA_TRACE record (cycles, event, a, b)
// per block into Plan::trace; the product build compiles these to nothing.
enum : int { TR_KSTART = 1, TR_SEG, TR_P_SEL, TR_C_SEG0, TR_C_SEG1, TR_C_SEL0, TR_C_SEL1,
             TR_C_COMB0, TR_C_COMB1, TR_KEND, TR_C_SELW, TR_C_SCD };
#ifdef SSA_TRACE
__device__ __forceinline__ void trace_event(const Plan& p, int* counter, int ev, int a, int b) {
    if (!p.trace) return;
    const int i = atomicAdd(counter, 1);
    if (i >= p.trace_cap) return;
    const uint64_t t = (ev & 0x80) ? now_ns() : (uint64_t)clock64();
    p.trace[(size_t)blockIdx.x * p.trace_cap + i] =
        make_uint4((uint32_t)t, (uint32_t)(t >> 32), (uint32_t)ev | ((uint32_t)a << 8), (uint32_t)b);
}
#define SSA_TR(ev, a, b) trace_event(p, &misc[15], (ev), (a), (b))
// probe points inside the block top-k (thread 0 only): event 13, a = point
struct TraceProbe {
    const Plan& p;
    int* counter;
    int pair;
    __device__ void operator()(int point) const {
        if (threadIdx.x == 0) trace_event(p, counter, 13, point, pair);
    }
};
#define SSA_PROBE(pair) TraceProbe{p, &misc[15], (pair)}
#else
#define SSA_PROBE(pair) NoProbe()
#define SSA_TR(ev, a, b) ((void)0)
#endif

struct ConsumerSync {
    __device__ void operator()() const { named_sync(kBarConsumers, kConsumers); }
    __device__ bool or_(bool pred) const { return named_sync_or(kBarConsumers, kConsumers, pred); }
};

// swizzled (128B) address of 16-byte unit `chunk` of row `row` in a slot
template <int D>
__device__ __forceinline__ uint32_t tile_addr(uint32_t slot, int row, int chunk) {
    const int sub = chunk >> 3, cc = chunk & 7;
    return slot + sub * (kBoxRows * 128) + row * 128 + ((cc ^ (row & 7)) << 4);
}

// S[head][token] for 16 rows starting at r0 of a key slot (2 n-tiles of 8).
template <int D>
__device__ __forceinline__ void qk16(uint32_t slot, int r0, const uint32_t (&qa)[D / 16][4],
                                     float (&s)[2][4], int lane) {
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) s[i][c] = 0.f;
    const int row = r0 + ((lane >> 4) << 3) + (lane & 7);
    const int csel = (lane >> 3) & 1;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(tile_addr<D>(slot, row, 2 * kk + csel), b0, b1, b2, b3);
        mma_bf16_16816(s[0], qa[kk], b0, b1);
        mma_bf16_16816(s[1], qa[kk], b2, b3);
    }
}

// S^T[token][head] for 16 rows starting at r0 of a key slot, with the keys as
// the M operand: the A fragments are the key rows (the same ldmatrix loads as
// qk16, reordered) and the B fragments are the query registers.  st[nt] holds
// heads 8 nt .. 8 nt + 7: st[nt][0..1] token g8, heads 2 tig, 2 tig + 1;
// st[nt][2..3] token g8 + 8.
template <int D, int NT>
__device__ __forceinline__ void qkT16(uint32_t slot, int r0, const uint32_t (&qa)[D / 16][4],
                                      float (&st)[NT][4], int lane) {
#pragma unroll
    for (int i = 0; i < NT; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) st[i][c] = 0.f;
    const int row = r0 + ((lane >> 4) << 3) + (lane & 7);
    const int csel = (lane >> 3) & 1;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(tile_addr<D>(slot, row, 2 * kk + csel), b0, b1, b2, b3);
        const uint32_t a[4] = {b0, b2, b1, b3};
        mma_bf16_16816(st[0], a, qa[kk][0], qa[kk][2]);
        if (NT == 2) mma_bf16_16816(st[NT - 1], a, qa[kk][1], qa[kk][3]);
    }
}

// Scores of the 16-row blocks `w` of the two 64-row boxes of a score stage
// (rows 16 w.. of slot A, and 64 + 16 w.. of slot B) by warp w: per row, the
// maximum over the group's query heads of q.k / sqrt(d), into rowmax.  With
// lg != nullptr, also keeps every head's logit in the log2 domain
// (q.k / sqrt(d) * log2 e) at lg[head * lstride + row].
template <int D, int NT>
__device__ __forceinline__ void score_rows2(uint32_t slotA, uint32_t slotB, int w, int nvalid,
                                            int G, const uint32_t (&qa)[D / 16][4], float scale,
                                            float* rowmax, float* lg, int lstride,
                                            float scale_log2, int lane) {
    const int g8 = lane >> 2, tig = lane & 3;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int r0 = 64 * j + 16 * w;
        if (r0 >= nvalid) break;
        float st[NT][4];
        qkT16<D, NT>(j ? slotB : slotA, 16 * w, qa, st, lane);
        if (lg) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int h = nt * 8 + 2 * tig + (c & 1);
                    const int row = r0 + 8 * (c >> 1) + g8;
                    if (h < G && row < nvalid) lg[h * lstride + row] = st[nt][c] * scale_log2;
                }
        }
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            float v = -INFINITY;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                const int h = nt * 8 + 2 * tig;
                if (h < G) v = fmaxf(v, st[nt][2 * half]);
                if (h + 1 < G) v = fmaxf(v, st[nt][2 * half + 1]);
            }
            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 1));
            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 2));
            const int lr = r0 + 8 * half + g8;
            if (tig == 0 && lr < nvalid) rowmax[lr] = v * scale;
        }
    }
}

// O^T += V^T . P^T for 16 rows starting at r0 of a value slot, with the
// head dimension as the M operand (so a GQA group of <= 8 heads fills one
// 8-wide N tile): the A fragments are the value rows (ldmatrix.trans, the
// same loads as a P.V product, reordered); the B fragments are P in the
// layout a Q.K^T accumulator already has (p[nt] tokens 0..7, p[2 + nt]
// tokens 8..15 of head 8 nt + g8), as bf16 hi and lo parts.
// acc[nt][mm][c]: heads 8 nt + 2 tig + (c & 1), dims 16 mm + g8 + 8 (c >> 1).
template <int D>
__device__ __forceinline__ void pvT16(uint32_t slot, int r0, const uint32_t (&phi)[4],
                                      const uint32_t (&plo)[4], float (&acc)[2][D / 16][4],
                                      bool two, int lane) {
    const int row = r0 + (lane & 15);
    const int csel = lane >> 4;
#pragma unroll
    for (int mm = 0; mm < D / 16; ++mm) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_trans(tile_addr<D>(slot, row, 2 * mm + csel), b0, b1, b2, b3);
        const uint32_t a[4] = {b0, b2, b1, b3};
        mma_bf16_16816(acc[0][mm], a, phi[0], phi[2]);
        if (kPvLo) mma_bf16_16816(acc[0][mm], a, plo[0], plo[2]);
        if (two) {
            mma_bf16_16816(acc[1][mm], a, phi[1], phi[3]);
            if (kPvLo) mma_bf16_16816(acc[1][mm], a, plo[1], plo[3]);
        }
    }
}

// acc += P(hi + lo) . V for 16 rows at r0 of a value slot with the heads as
// the M rows (P straight from a Q.K^T accumulator; rows 8..15 are heads
// 8..15).  The same accumulator storage read as acc8(x) = x-th 8-dim tile:
// lane holds heads g8 (c < 2) / g8 + 8, dims 8 x + 2 tig + (c & 1).
template <int D>
__device__ __forceinline__ float (&acc8(float (&acc)[2][D / 16][4], int x))[4] {
    return acc[x / (D / 16)][x % (D / 16)];
}
template <int D>
__device__ __forceinline__ void pvM16(uint32_t slot, int r0, const uint32_t (&phi)[4],
                                      const uint32_t (&plo)[4], float (&acc)[2][D / 16][4],
                                      int lane) {
    const int row = r0 + (lane & 15);
    const int csel = lane >> 4;
#pragma unroll
    for (int nn = 0; nn < D / 16; ++nn) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_trans(tile_addr<D>(slot, row, 2 * nn + csel), b0, b1, b2, b3);
        mma_bf16_16816(acc8<D>(acc, 2 * nn), phi, b0, b1);
        if (kPvLo) mma_bf16_16816(acc8<D>(acc, 2 * nn), plo, b0, b1);
        mma_bf16_16816(acc8<D>(acc, 2 * nn + 1), phi, b2, b3);
        if (kPvLo) mma_bf16_16816(acc8<D>(acc, 2 * nn + 1), plo, b2, b3);
    }
}

// Multiplies the accumulator columns of the heads of n tile r by alpha (held,
// S-layout, by the lanes of group g8 = head): each lane fetches the factors of
// its two heads 8 r + 2 tig and 8 r + 2 tig + 1.
template <int D>
__device__ __forceinline__ void rescale_acc(float (&acc)[2][D / 16][4], int r, float alpha,
                                            int tig) {
    if (kPvHeadsM) {
#pragma unroll
        for (int x = 0; x < D / 8; ++x) {
            acc8<D>(acc, x)[2 * r] *= alpha;
            acc8<D>(acc, x)[2 * r + 1] *= alpha;
        }
        return;
    }
    const float a0 = __shfl_sync(0xffffffffu, alpha, (2 * tig) << 2);
    const float a1 = __shfl_sync(0xffffffffu, alpha, (2 * tig + 1) << 2);
#pragma unroll
    for (int mm = 0; mm < D / 16; ++mm) {
        acc[r][mm][0] *= a0;
        acc[r][mm][1] *= a1;
        acc[r][mm][2] *= a0;
        acc[r][mm][3] *= a1;
    }
}

// Online-softmax update and P.V for NSB 16-row blocks of one warp.  sc holds
// the blocks' logits in the log2 domain in the layout of a Q.K^T accumulator
// with the heads as M rows (sc[i][nt][c]: head g8 (c < 2) or g8 + 8, token
// nt * 8 + 2 tig + (c & 1)); excluded tokens are -inf.  One max / rescale per
// call; block i's values are the 16 rows at vrow[i] of slot vslot[i] (blocks
// with valid[i] false are skipped).
template <int D, int NSB>
__device__ __forceinline__ void softmax_pv(float (&sc)[NSB][2][4], const uint32_t (&vslot)[NSB],
                                           const int (&vrow)[NSB], const bool (&valid)[NSB],
                                           float (&mrow)[2], float (&lrow)[2],
                                           float (&acc)[2][D / 16][4], bool two_rows, int lane) {
    const int tig = lane & 3;
    uint32_t phi[NSB][4], plo[NSB][4];
#pragma unroll
    for (int i = 0; i < NSB; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) phi[i][c] = plo[i][c] = 0u;
#pragma unroll
    for (int r = 0; r < 2; ++r) {
        if (r == 1 && !two_rows) break;
        float mx = -INFINITY;
#pragma unroll
        for (int i = 0; i < NSB; ++i)
            mx = fmaxf(mx, fmaxf(fmaxf(sc[i][0][2 * r], sc[i][0][2 * r + 1]),
                                 fmaxf(sc[i][1][2 * r], sc[i][1][2 * r + 1])));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
        const float mnew = fmaxf(mrow[r], mx);
        const float ref = (mnew == -INFINITY) ? 0.f : mnew;
        const float alpha = exp2f(mrow[r] - ref);
        float lsum = 0.f;
#pragma unroll
        for (int i = 0; i < NSB; ++i) {
            const float p00 = exp2f(sc[i][0][2 * r] - ref), p01 = exp2f(sc[i][0][2 * r + 1] - ref);
            const float p10 = exp2f(sc[i][1][2 * r] - ref), p11 = exp2f(sc[i][1][2 * r + 1] - ref);
            lsum += (p00 + p01) + (p10 + p11);
            if (kPvLo) {
                split_bf16(p00, p01, phi[i][r], plo[i][r]);          // tokens 0..7
                split_bf16(p10, p11, phi[i][2 + r], plo[i][2 + r]);  // tokens 8..15
            } else {
                phi[i][r] = pack_bf16(p00, p01);
                phi[i][2 + r] = pack_bf16(p10, p11);
            }
        }
        lrow[r] = lrow[r] * alpha + lsum;
        mrow[r] = mnew;
        if (__any_sync(0xffffffffu, alpha != 1.f)) rescale_acc<D>(acc, r, alpha, tig);
    }
#pragma unroll
    for (int i = 0; i < NSB; ++i)
        if (valid[i]) {
            if (kPvHeadsM) pvM16<D>(vslot[i], vrow[i], phi[i], plo[i], acc, lane);
            else pvT16<D>(vslot[i], vrow[i], phi[i], plo[i], acc, two_rows, lane);
        }
}

// ---------------------------------------------------------------- plan ---

// Derived sizes of one pair from its raw length n (0 for an invalid length).
struct PairSizes {
    int n, M, T;            // raw length, complete chunks, tail tokens
    int S, R, ks, Mc, kc;   // superchunks, remainder chunks, kept superchunks,
                            // candidates (single level: M), kept chunks
};

__device__ __forceinline__ PairSizes pair_sizes(const Plan& p, int n) {
    PairSizes z;
    z.n = n;
    z.M = n / p.C;
    z.T = n - z.M * p.C;
    if (p.h2) {
        z.S = z.M / p.J;
        z.R = z.M - z.S * p.J;
        z.ks = min(p.topk_super, z.S);
        z.Mc = z.ks * p.J + z.R;
    } else {
        z.S = z.R = z.ks = 0;
        z.Mc = z.M;
    }
    z.kc = min(p.topk, z.Mc);
    return z;
}

// Elements of list `L` for one pair of raw length n.
__device__ __forceinline__ int list_count(const Plan& p, int L, int n) {
    const PairSizes z = pair_sizes(p, n);
    const int tpc = (p.C + kBoxRows - 1) / kBoxRows;
    switch (L) {
        case L_SCORE:
            if (p.mode == kModeAttnOnly) return 0;
            if (p.mode == kModeScoreOnly) return p.M_max;
            return p.h2 ? z.S : z.M;
        case L_CAND:
            return p.h2 ? z.Mc : 0;
        case L_META:
            return p.h2 ? (z.S * p.gm + kBoxRows - 1) / kBoxRows : 0;
        case L_GIST:
            if (p.mode == kModeScoreOnly) return 0;
            if (!p.h2) return (z.M * p.g + kBoxRows - 1) / kBoxRows;
            return z.ks * ((p.J * p.g + kBoxRows - 1) / kBoxRows) +
                   (z.R * p.g + kBoxRows - 1) / kBoxRows;
        case L_RAW:
            if (p.mode == kModeScoreOnly) return 0;
            return z.kc * tpc + (z.T + kBoxRows - 1) / kBoxRows;
    }
    return 0;
}

// The block-local plan: lengths per sequence and prefix sums per list.
struct PlanView {
    const Plan& p;
    const int* nb;   // [B] raw lengths (0: invalid)
    const int* ps;   // [kNumLists][B + 1] prefix over sequences of Hkv * count
    int nblocks;

    __device__ int total(int L) const { return ps[L * (p.B + 1) + p.B]; }
    __device__ int parts(int L) const { return min(nblocks, total(L)); }
    // share of block c in list L: [lo, hi)
    __device__ void share(int L, int c, int& lo, int& hi) const {
        const long long t = total(L), n = parts(L);
        if (c >= n) {
            lo = hi = 0;
            return;
        }
        lo = (int)((t * c) / n);
        hi = (int)((t * (c + 1)) / n);
    }
    // block holding element x of list L
    __device__ int block_of(int L, int x) const {
        const long long t = total(L), n = parts(L);
        return (int)(((long long)(x + 1) * n - 1) / t);
    }
    // pair holding element x of list L, its first element and element count
    __device__ void locate(int L, int x, int& pair, int& first, int& count) const {
        const int* q = ps + L * (p.B + 1);
        int lo = 0, hi = p.B;  // q[lo] <= x < q[hi]
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (q[mid] <= x) lo = mid; else hi = mid;
        }
        count = list_count(p, L, nb[lo]);
        const int j = (x - q[lo]) / count;
        pair = lo * p.Hkv + j;
        first = q[lo] + j * count;
    }
    // blocks holding the segments of pair `pair` in list L: [c0, c0 + n)
    __device__ void pair_blocks(int L, int pair, int& c0, int& n) const {
        const int b = pair / p.Hkv, j = pair % p.Hkv;
        const int count = list_count(p, L, nb[b]);
        if (count == 0) {
            c0 = n = 0;
            return;
        }
        const int first = ps[L * (p.B + 1) + b] + j * count;
        c0 = block_of(L, first);
        n = block_of(L, first + count - 1) - c0 + 1;
    }
};

// Pairs whose top-k block c runs: those with floor(pair * N / P) == c.  Their
// combination runs on the mirrored block N - 1 - c.
__device__ __forceinline__ void owned_pairs(int c, int N, int P, int& lo, int& hi) {
    lo = (int)(((long long)c * P + N - 1) / N);
    hi = (int)(((long long)(c + 1) * P + N - 1) / N);
}

// Partial of segment (attention list a, block c, pair), query head h.  Along
// a list, the segments' (block + pair) strictly increase, so the slots differ.
__device__ __forceinline__ size_t partial_offset(const Plan& p, int a, int c, int pair, int h,
                                                 int D) {
    const size_t slot = (size_t)a * (kMaxGrid + p.n_pairs) + c + pair;
    return (slot * p.G + h) * (size_t)(D + 2);
}

// ------------------------------------------------------------ producer ---

template <int D>
struct Producer {
    const Plan& p;
    const CUtensorMap* tm[6];  // k_raw, v_raw, k_gist, v_gist, k_meta, v_meta
    uint8_t* ring;
    uint8_t* qbuf;
    int qbytes;
    StageMeta* meta;
    uint64_t* full;
    uint64_t* empty;
    int* ctrl;
    int lane;
    long long long_limit;  // bound of ring waits (several device-side waits)
    int stage = 0, round = 0;
    bool dead = false;     // a ring wait ran out: issue nothing more
    int* trace_ctr = nullptr;
    uint64_t pol_keep = 0, pol_once = 0;

    __device__ int* rec(int a, int pair) const { return ctrl + C_ARR + pair * p.pair_ints + a; }

    // Next free stage; false once the ring is given up.
    __device__ bool acquire(int& s) {
        s = stage;
        if (dead) return false;
        if (round > 0) {
            bool ok = true;
            if (lane == 0) ok = mbar_wait(&empty[s], (uint32_t)((round - 1) & 1), long_limit);
            ok = __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
            if (!ok) {
                dead = true;
                return false;
            }
        }
        return true;
    }
    __device__ void advance() {
        if (++stage == p.stages) {
            stage = 0;
            ++round;
        }
    }
    __device__ uint8_t* slot(int s, int which) {
        return ring + (size_t)s * Cfg<D>::kStageBytes + which * Cfg<D>::kSlotBytes;
    }
    // one 64-row box (all D columns) of map `m` at global row y into slot,
    // with an L2 policy: summary keys are read twice (scoring, attention) and
    // kept in L2 in between; everything else is read once
    __device__ void box(int s, int which, const CUtensorMap* m, int y, uint64_t pol) {
#pragma unroll
        for (int sub = 0; sub < D / 64; ++sub)
            tma_load_2d_hint(slot(s, which) + sub * (kBoxRows * 128), m, sub * 64, y, &full[s],
                             pol);
    }
    __device__ void load_q(int s, int pair) {
        const int b = pair / p.Hkv, j = pair % p.Hkv;
        const __nv_bfloat16* src =
            static_cast<const __nv_bfloat16*>(p.q) + ((size_t)b * p.Hq + (size_t)j * p.G) * D;
        bulk_load(qbuf + (size_t)s * qbytes, src, (uint32_t)(p.G * D * 2), &full[s]);
    }
    // a stage without data (select, combine, end, empty segment)
    __device__ void push_plain(const StageMeta& m) {
        int s;
        if (!acquire(s)) return;
        if (lane == 0) {
            meta[s] = m;
            mbar_arrive(&full[s]);
        }
        __syncwarp();
        advance();
    }
    // Waits until every stage this warp issued has landed (bounded), so no
    // copy is in flight when the block exits, whatever the consumers did.
    __device__ void drain() {
        const int NS = p.stages;
        const int issued = round * NS + stage;
        if (lane == 0)
            for (int i = 0; i < NS && i < issued; ++i) {
                const int idx = issued - 1 - i;
                mbar_wait(&full[idx % NS], (uint32_t)((idx / NS) & 1), long_limit);
            }
        __syncwarp();
    }

    // Scores `nslot` consecutive summary slots of `ntok` rows each, starting
    // at global row y0 of map m, into dst[0..nslot), then writes `npad` slots
    // of -inf.  Split into sub-items of at most `per_rows` rows.
    // (seg_first / seg_last: this run starts / ends its block's segment of
    // the pair; a candidate segment is several runs)
    __device__ void score_run(int pair, int level, const CUtensorMap* m, int y0, int nslot,
                              int npad, int dst, int ntok, int per_rows, int lrow0,
                              bool seg_first = true, bool seg_last = true) {
        const int per = max(1, per_rows / ntok);  // slots per sub-item
        int s0 = 0;
        do {
            const int ns = min(per, nslot - s0);
            const int np = (s0 + ns >= nslot) ? npad : 0;
            const int rows = ns * ntok;
            const int segf = (seg_first && s0 == 0 ? F_SEGBEG : 0) |
                             (seg_last && s0 + ns >= nslot ? F_SEGEND : 0);
            if (rows <= 0) {
                StageMeta mt = {};
                mt.kind = K_SCORE;
                mt.pair = pair;
                mt.flags = F_FIRST | F_LAST | segf;
                mt.a2 = np;
                mt.a3 = dst + s0;
                mt.a4 = ntok;
                mt.a5 = level;
                push_plain(mt);
            }
            for (int off = 0; off < rows; off += 2 * kBoxRows) {
                int s;
                if (!acquire(s)) return;
                const int nv = min(2 * kBoxRows, rows - off);
                const int nbox = (nv + kBoxRows - 1) / kBoxRows;
                const bool first = off == 0;
                if (lane == 0) {
                    StageMeta mt = {};
                    mt.kind = K_SCORE;
                    mt.pair = pair;
                    mt.nvalid = nv;
                    mt.flags = (first ? (F_FIRST | F_QLOAD) : 0) |
                               (off + 2 * kBoxRows >= rows ? (F_LAST | segf) : 0);
                    mt.a0 = off;
                    mt.a1 = ns;
                    mt.a2 = np;
                    mt.a3 = dst + s0;
                    mt.a4 = ntok;
                    mt.a5 = level;
                    mt.lrow = lrow0 + s0 * ntok + off;
                    meta[s] = mt;
                    const uint32_t bytes = nbox * Cfg<D>::kBoxBytes + (first ? p.G * D * 2 : 0);
                    mbar_arrive_expect_tx(&full[s], bytes);
#ifdef SSA_TRACE
                    trace_event(p, trace_ctr, 14, 1, round * p.stages + s);
#endif
                    if (first) load_q(s, pair);
                    for (int bx = 0; bx < nbox; ++bx)
                        box(s, bx, m, y0 + s0 * ntok + off + bx * kBoxRows, pol_keep);
                }
                __syncwarp();
                advance();
            }
            s0 += ns;
        } while (s0 < nslot);
    }

    // Reads a published selection (count word, `cap` entries at `ent`) into
    // shared `dst` as plain indices.  One round of relaxed loads per attempt;
    // polls with back-off until the count and its entries are all written.
    // Returns the count and sets `bad` for a rejected caller selection; a
    // wait that runs out records a timeout and returns 0.
    __device__ int fetch_selection(const int* cnt_word, const int* ent, int cap, int* dst,
                                   bool& bad) {
        bad = false;
        if (dead) return 0;
        const long long c0 = clock64(), lim = wait_cycles(p.wait_limit);
        unsigned sleep_ns = 32;
        for (;;) {
            int cw = lane == 0 ? ld_relaxed(cnt_word) : 0;
            int e[4];
            for (int base = 0; base < max(cap, 1); base += 128) {
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int c = base + 32 * r + lane;
                    e[r] = c < cap ? ld_relaxed(ent + c) : 1;
                }
                cw = __shfl_sync(0xffffffffu, cw, 0);
                // not published yet: write nothing, retry (dst holds `cap` words)
                const int k = cw == 0 ? 0 : min((cw & (kBadBit - 1)) - 1, cap);
                bool ok = cw != 0;
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int c = base + 32 * r + lane;
                    if (c < k) {
                        ok = ok && e[r] != 0;
                        dst[c] = e[r] - 1;
                    }
                }
                if (!__all_sync(0xffffffffu, ok)) break;
                if (base + 128 >= min(k, cap)) {
                    __syncwarp();
                    bad = (cw & kBadBit) != 0;
                    return k;
                }
            }
            if (clock64() - c0 > lim) {
                if (lane == 0) report_status(kStatusTimeout);
                return 0;
            }
            __nanosleep(sleep_ns);
            if (sleep_ns < 512) sleep_ns *= 2;
        }
    }
};

// ------------------------------------------------------------ the kernel ---

template <int D>
__global__ void __launch_bounds__(kThreads, 2)
    fused_kernel(const __grid_constant__ Plan p, const __grid_constant__ CUtensorMap tm_kraw,
                 const __grid_constant__ CUtensorMap tm_vraw,
                 const __grid_constant__ CUtensorMap tm_kgist,
                 const __grid_constant__ CUtensorMap tm_vgist,
                 const __grid_constant__ CUtensorMap tm_kmeta,
                 const __grid_constant__ CUtensorMap tm_vmeta) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const SmemLayout L = smem_layout<D>(p);
    const int NS = p.stages;
    uint8_t* ring = smem + L.ring;
    uint8_t* qbuf = smem + L.qbuf;
    StageMeta* meta = reinterpret_cast<StageMeta*>(smem + L.meta);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint64_t* empty = full + NS;
    int* psel = reinterpret_cast<int*>(smem + L.psel);
    int* psup = reinterpret_cast<int*>(smem + L.psup);
    int* nbv = reinterpret_cast<int*>(smem + L.plan);
    int* psv = nbv + p.B;
    uint32_t* bits = reinterpret_cast<uint32_t*>(smem + L.bits);
    uint8_t* uni = smem + L.uni;
    float* logits = reinterpret_cast<float*>(smem + L.logit);
    int* misc = reinterpret_cast<int*>(smem + L.misc);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int P = p.n_pairs, N = gridDim.x, cta = blockIdx.x;
    int* ctrl = p.ctrl;
    auto rec = [&](int a, int pair) -> int* { return ctrl + C_ARR + pair * p.pair_ints + a; };
    // ring waits span at most a few bounded device-side waits of the other side
    const long long long_limit = 8 * p.wait_limit;

    // ---- prologue: barriers and the block-local plan (the same in every block)
    if (warp == kConsumerWarps && lane == 0) {
        // the tensor maps' descriptors are fetched while the lengths load
        prefetch_tensormap(&tm_kraw);
        prefetch_tensormap(&tm_vraw);
        prefetch_tensormap(&tm_kgist);
        prefetch_tensormap(&tm_vgist);
        prefetch_tensormap(&tm_kmeta);
        prefetch_tensormap(&tm_vmeta);
    }
    if (threadIdx.x == 0) {
        misc[15] = 0;
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        fence_barrier_init();
    }
    for (int b = threadIdx.x; b < p.B; b += blockDim.x) {
        const int n = __ldg(p.seq_lens + b);
        const bool ok = n >= 1 && n <= p.n_max;
        if (!ok && cta == 0) report_status(kStatusBadInput);
        nbv[b] = ok ? n : 0;
    }
    __syncthreads();
    if (warp < kNumLists) {  // warp w: exclusive prefix over sequences of list w
        int carry = 0;
        for (int b0 = 0; b0 < p.B; b0 += 32) {
            const int b = b0 + lane;
            const int v = b < p.B ? p.Hkv * list_count(p, warp, nbv[b]) : 0;
            int x = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            if (b < p.B) psv[warp * (p.B + 1) + b] = carry + x - v;
            carry += __shfl_sync(0xffffffffu, x, 31);
        }
        if (lane == 0) psv[warp * (p.B + 1) + p.B] = carry;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        SSA_TR(TR_KSTART | 0x80, 0, 0);
        SSA_TR(TR_KSTART, 0, 0);
    }
    const PlanView pv{p, nbv, psv, N};
    const bool so = p.mode == kModeScoreOnly;
    const int score_rows = min(kRowmaxCap, max(p.score_rows, 1));

    // ================================================================ producer
    if (warp == kConsumerWarps) {
        Producer<D> pr{p,    {&tm_kraw, &tm_vraw, &tm_kgist, &tm_vgist, &tm_kmeta, &tm_vmeta},
                       ring, qbuf, L.qbytes, meta, full, empty, ctrl, lane, long_limit};
        pr.pol_once = l2_policy_evict_first();
        pr.trace_ctr = &misc[15];
        pr.pol_keep = so ? pr.pol_once : l2_policy_evict_last();
        int sel_lo, sel_hi;
        owned_pairs(cta, N, P, sel_lo, sel_hi);

        // -------- this block's share of a scoring list (first level or candidates)
        auto score_list = [&](int Ls) {
            int lo, hi;
            pv.share(Ls, cta, lo, hi);
            int seg_base = 0;  // rows of this share scored so far (kept-logit rows)
            for (int x = lo; x < hi;) {
                int pair, first, count;
                pv.locate(Ls, x, pair, first, count);
                const int i0 = x - first, i1 = min(hi, first + count) - first;
                const PairSizes z = pair_sizes(p, nbv[pair / p.Hkv]);
                if (lane == 0) SSA_TR(TR_SEG, Ls, pair);
                if (Ls == L_SCORE && !p.h2) {
                    // score-only calls also cover the slots past M (as -inf)
                    const int nv = max(0, min(i1, z.M) - i0);
                    const int npad = (i1 - i0) - nv;
                    pr.score_run(pair, 0, &tm_kgist, (pair * p.M_max + i0) * p.g, nv, npad,
                                 pair * p.M_max + i0, p.g, score_rows, seg_base);
                    seg_base += nv * p.g;
                } else if (Ls == L_SCORE) {
                    pr.score_run(pair, 0, &tm_kmeta, (pair * p.S_max + i0) * p.gm, i1 - i0, 0,
                                 pair * p.S_max + i0, p.gm, score_rows, 0);
                } else {
                    // candidates: runs of consecutive chunks (J per kept
                    // superchunk, in superchunk order, then the remainder),
                    // addressed through the published superchunk selection
                    bool bad;
                    const int ks = pr.fetch_selection(rec(A_SCOUNT, pair),
                                                      rec(A_ENTRIES + p.topk, pair),
                                                      p.topk_super, psup, bad);
                    for (int c = i0; c < i1;) {
                        int chunk0, run;
                        if (c < ks * p.J) {
                            chunk0 = psup[c / p.J] * p.J + c % p.J;
                            run = min(i1, (c / p.J + 1) * p.J) - c;
                        } else {
                            chunk0 = z.S * p.J + (c - ks * p.J);
                            run = i1 - c;
                        }
                        pr.score_run(pair, 1, &tm_kgist, (pair * p.M_max + chunk0) * p.g, run, 0,
                                     pair * p.Mc_max + c, p.g, score_rows, 0, c == i0, c + run >= i1);
                        c += run;
                    }
                }
                x = first + i1;
            }
        };

        // -------- this block's share of an attention list (META, GIST or RAW)
        auto attn_list = [&](int La) {
            const int alist = La == L_META ? 0 : La == L_GIST ? 1 : 2;
            const int tpc = (p.C + kBoxRows - 1) / kBoxRows;
            const int tsc = (p.J * p.g + kBoxRows - 1) / kBoxRows;
            int lo, hi;
            pv.share(La, cta, lo, hi);
            for (int x = lo; x < hi;) {
                int pair, first, count;
                pv.locate(La, x, pair, first, count);
                const int u0 = x - first, u1 = min(hi, first + count) - first;
                const PairSizes z = pair_sizes(p, nbv[pair / p.Hkv]);
                if (lane == 0) SSA_TR(TR_SEG, La, pair);
                int ks = 0, ksel = 0;
                bool bad = false;
                if (La == L_GIST && p.h2) {
                    bool b2;
                    ks = pr.fetch_selection(rec(A_SCOUNT, pair), rec(A_ENTRIES + p.topk, pair),
                                            p.topk_super, psup, b2);
                }
                if (La == L_RAW) {
                    ksel = pr.fetch_selection(rec(A_COUNT, pair), rec(A_ENTRIES, pair), p.topk,
                                              psel, bad);
                    if (lane == 0) SSA_TR(TR_P_SEL, pair, ksel);
                }
                bool emitted = false;
                // each tile is issued once the next is known, so the last
                // tile of the segment carries F_LAST
                int pend_src = -1, pend_y = 0, pend_nv = 0, pend_r0 = 0;
                auto emit = [&](bool last) {
                    int s;
                    if (!pr.acquire(s)) return;
                    if (lane == 0) {
                        StageMeta mt = {};
                        mt.kind = K_ATTN;
                            mt.pair = pair;
                        mt.nvalid = pend_nv;
                        mt.flags = (emitted ? 0 : (F_FIRST | F_QLOAD)) | (last ? F_LAST : 0);
                        mt.a0 = pend_r0;
                        mt.a1 = La == L_META ? MASK_SUPER : La == L_GIST ? MASK_CHUNK : MASK_NONE;
                        mt.a2 = La == L_META ? p.gm : p.g;
                        mt.a3 = alist;
                        meta[s] = mt;
                        const uint32_t bytes = 2 * Cfg<D>::kBoxBytes + (emitted ? 0 : p.G * D * 2);
                        mbar_arrive_expect_tx(&full[s], bytes);
#ifdef SSA_TRACE
                        trace_event(p, &misc[15], 14, 2, pr.round * NS + s);
#endif
                        if (!emitted) pr.load_q(s, pair);
                        const CUtensorMap* km =
                            pend_src == 0 ? &tm_kraw : pend_src == 1 ? &tm_kgist : &tm_kmeta;
                        const CUtensorMap* vm =
                            pend_src == 0 ? &tm_vraw : pend_src == 1 ? &tm_vgist : &tm_vmeta;
                        pr.box(s, 0, km, pend_y, pr.pol_once);
                        pr.box(s, 1, vm, pend_y, pr.pol_once);
                    }
                    __syncwarp();
                    pr.advance();
                    emitted = true;
                };
                for (int u = u0; u < u1; ++u) {
                    int src, y, nv, r0;
                    if (La == L_META) {
                        r0 = u * kBoxRows;
                        nv = min(kBoxRows, z.S * p.gm - r0);
                        src = 2;
                        y = pair * p.S_max * p.gm + r0;
                    } else if (La == L_GIST && !p.h2) {
                        r0 = u * kBoxRows;
                        nv = min(kBoxRows, z.M * p.g - r0);
                        src = 1;
                        y = pair * p.M_max * p.g + r0;
                    } else if (La == L_GIST) {
                        if (u < z.ks * tsc) {
                            const int sl = u / tsc, part = u % tsc;
                            if (sl >= ks) continue;
                            r0 = psup[sl] * p.J * p.g + part * kBoxRows;
                            nv = min(kBoxRows, p.J * p.g - part * kBoxRows);
                        } else {
                            r0 = z.S * p.J * p.g + (u - z.ks * tsc) * kBoxRows;
                            nv = min(kBoxRows, z.M * p.g - r0);
                        }
                        src = 1;
                        y = pair * p.M_max * p.g + r0;
                    } else {
                        // a rejected caller selection: the pair attends to nothing
                        if (bad) continue;
                        if (u < z.kc * tpc) {
                            const int c = u / tpc, part = u % tpc;
                            if (c >= ksel) continue;
                            r0 = psel[c] * p.C + part * kBoxRows;
                            nv = min(kBoxRows, p.C - part * kBoxRows);
                        } else {
                            r0 = z.M * p.C + (u - z.kc * tpc) * kBoxRows;
                            nv = min(kBoxRows, z.n - r0);
                        }
                        src = 0;
                        y = pair * p.n_max + r0;
                    }
                    if (pend_src >= 0) emit(false);
                    pend_src = src;
                    pend_y = y;
                    pend_nv = nv;
                    pend_r0 = r0;
                }
                if (pend_src >= 0) {
                    emit(true);
                } else {
                    // nothing of the context falls in this segment: neutral partial
                    StageMeta mt = {};
                    mt.kind = K_ATTN;
                    mt.pair = pair;
                    mt.flags = F_FIRST | F_LAST;
                    mt.a1 = MASK_NONE;
                    mt.a3 = alist;
                    pr.push_plain(mt);
                }
                x = first + u1;
            }
        };

        // -------- logits mode: the values of this block's scored gist rows, in
        // the same order as its score share (issued before the selection)
        auto gistv_list = [&]() {
            int lo, hi;
            pv.share(L_SCORE, cta, lo, hi);
            int seg_base = 0;
            for (int x = lo; x < hi;) {
                int pair, first, count;
                pv.locate(L_SCORE, x, pair, first, count);
                const int i0 = x - first, i1 = min(hi, first + count) - first;
                const int rows = (i1 - i0) * p.g, row0 = i0 * p.g;
                if (lane == 0) SSA_TR(TR_SEG, L_GIST, pair);
                for (int off = 0; off < rows; off += 2 * kBoxRows) {
                    int s;
                    if (!pr.acquire(s)) return;
                    const int nv = min(2 * kBoxRows, rows - off);
                    if (lane == 0) {
                        StageMeta mt = {};
                        mt.kind = K_GISTV;
                        mt.pair = pair;
                        mt.nvalid = nv;
                        mt.flags = (off == 0 ? F_FIRST : 0) | (off + 2 * kBoxRows >= rows ? F_LAST : 0);
                        mt.a0 = row0 + off;
                        mt.a2 = p.g;
                        mt.a3 = 1;
                            mt.lrow = seg_base + off;
                        meta[s] = mt;
                        const int nbox = (nv + kBoxRows - 1) / kBoxRows;
                        mbar_arrive_expect_tx(&full[s], nbox * Cfg<D>::kBoxBytes);
                        for (int bx = 0; bx < nbox; ++bx)
                            pr.box(s, bx, &tm_vgist, pair * p.M_max * p.g + row0 + off + bx * kBoxRows,
                                   pr.pol_once);
                    }
                    __syncwarp();
                    pr.advance();
                }
                seg_base += rows;
                x = first + i1;
            }
        };

        auto selects = [&](int what) {
            for (int pair = sel_lo; pair < sel_hi; ++pair) {
                StageMeta mt = {};
                mt.kind = K_SELECT;
                mt.pair = pair;
                mt.flags = F_FIRST | F_LAST;
                mt.a0 = what;
                pr.push_plain(mt);
            }
        };

        // The phases of this mode, run by one loop so that each phase's code
        // exists once in the kernel (instruction cache).
        enum : int { OP_SCORE = 1, OP_SELECT, OP_GISTV, OP_ATTN };
        int prog[8], np = 0;
        if (so) {
            prog[np++] = OP_SCORE << 8 | L_SCORE;
        } else if (!p.h2) {
            if (p.mode == kModeAttnOnly) {
                prog[np++] = OP_SELECT << 8 | SEL_VALIDATE;
            } else {
                prog[np++] = OP_SCORE << 8 | L_SCORE;
                prog[np++] = OP_SELECT << 8 | SEL_CHUNKS;
            }
            prog[np++] = p.logits ? OP_GISTV << 8 : (OP_ATTN << 8 | L_GIST);
            prog[np++] = OP_ATTN << 8 | L_RAW;
        } else {
            prog[np++] = OP_SCORE << 8 | L_SCORE;
            prog[np++] = OP_SELECT << 8 | SEL_SUPER;
            prog[np++] = OP_ATTN << 8 | L_META;
            prog[np++] = OP_SCORE << 8 | L_CAND;
            prog[np++] = OP_SELECT << 8 | SEL_CAND;
            prog[np++] = OP_ATTN << 8 | L_GIST;
            prog[np++] = OP_ATTN << 8 | L_RAW;
        }
#pragma unroll 1
        for (int i = 0; i < np; ++i) {
            const int op = prog[i] >> 8, arg = prog[i] & 255;
            if (op == OP_SCORE) score_list(arg);
            else if (op == OP_SELECT) selects(arg);
            else if (op == OP_GISTV) gistv_list();
            else attn_list(arg);
        }
        if (!so) {
            // The combination of pair p runs on the block that holds p's last
            // attention element (its last raw tile; else its last gist / meta
            // tile), right after that block's own share, so it waits only for
            // the other segments of p, which finish at about the same time.
            // Pairs without any attention element go to block p mod N.
            const int Lg = p.logits ? L_SCORE : L_GIST;
            const int order[3] = {L_RAW, Lg, L_META};
            auto cnt = [&](int L, int pair) { return list_count(p, L, nbv[pair / p.Hkv]); };
            for (int oi = 0; oi < 3; ++oi) {
                const int La = order[oi];
                if (La == L_META && !p.h2) continue;
                int lo, hi;
                pv.share(La, cta, lo, hi);
                for (int x = lo; x < hi;) {
                    int pair, first, count;
                    pv.locate(La, x, pair, first, count);
                    const int i1 = min(hi, first + count) - first;
                    bool mine = i1 == count;  // this block holds the pair's last element
                    for (int oj = 0; oj < oi && mine; ++oj)
                        if (!(order[oj] == L_META && !p.h2)) mine = cnt(order[oj], pair) == 0;
                    if (mine) {
                        StageMeta mt = {};
                        mt.kind = K_COMBINE;
                        mt.pair = pair;
                        mt.flags = F_FIRST | F_LAST;
                        pr.push_plain(mt);
                    }
                    x = first + i1;
                }
            }
            for (int pair = cta; pair < P; pair += N) {
                bool none = cnt(L_RAW, pair) == 0 && cnt(Lg, pair) == 0;
                if (p.h2) none = none && cnt(L_META, pair) == 0;
                if (none) {
                    StageMeta mt = {};
                    mt.kind = K_COMBINE;
                    mt.pair = pair;
                    mt.flags = F_FIRST | F_LAST;
                    pr.push_plain(mt);
                }
            }
        }
        StageMeta end = {};
        end.kind = K_END;
        pr.push_plain(end);
        pr.drain();
        return;
    }

    // ================================================================ consumers
    const int tid = threadIdx.x;  // 0..127
    const int g8 = lane >> 2, tig = lane & 3;
    const float scale = rsqrtf((float)D);
    const float scale_log2 = scale * 1.4426950408889634f;
    float* rowmax = reinterpret_cast<float*>(uni);
    float* merge = reinterpret_cast<float*>(uni);
    TopkScratch& tsc = *reinterpret_cast<TopkScratch*>(uni);
    ConsumerSync csync;
    const bool two_rows = p.G > 8;  // query heads 8..15 of the group present
    const int mask_words = mask_words_for(p);

    uint32_t qa[D / 16][4];
    // fast selection: this warp's 32 best chunks of the current scoring segment
    unsigned long long segrun = 1ull;
    unsigned long long* wlists = reinterpret_cast<unsigned long long*>(uni + kRowmaxCap * 4);
    float acc[2][D / 16][4];  // O^T: [head n tile][dim m tile][fragment]
    float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk)
#pragma unroll
        for (int c = 0; c < 4; ++c) qa[kk][c] = 0u;
    auto zero_acc = [&]() {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int mm = 0; mm < D / 16; ++mm)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[nt][mm][c] = 0.f;
    };
    zero_acc();

    // Loads the published selection (chunks or superchunks) of `pair` into
    // the shared bitmap.  One round of loads reads the count and every entry
    // (self-validating: 0 = not written yet); rounds repeat until complete.
    // A rejected caller selection excludes every row.  (Loading the
    // selections of several pairs at once would make a segment wait for the
    // latest of them.)
    auto load_bitmap = [&](int pair, int level) {
        for (int w = tid; w < mask_words; w += kConsumers) bits[w] = 0u;
        const int* cnt_word = rec(level == MASK_SUPER ? A_SCOUNT : A_COUNT, pair);
        const int* ent = rec(level == MASK_SUPER ? A_ENTRIES + p.topk : A_ENTRIES, pair);
        const int cap = level == MASK_SUPER ? p.topk_super : p.topk;
        constexpr int kPer = (kMaxTopkEntries + kConsumers - 1) / kConsumers;
        int e[kPer];
        int cw = 0;
        const long long c0 = clock64(), lim = wait_cycles(p.wait_limit);
        bool missing;
        for (;;) {
            cw = ld_relaxed(cnt_word);
#pragma unroll
            for (int j = 0; j < kPer; ++j) {
                const int c = tid + kConsumers * j;
                e[j] = c < cap ? ld_relaxed(ent + c) : 1;
            }
            const int k = (cw == 0 || (cw & kBadBit)) ? 0 : min((cw & (kBadBit - 1)) - 1, cap);
            missing = cw == 0;
#pragma unroll
            for (int j = 0; j < kPer; ++j) missing |= (tid + kConsumers * j < k) && e[j] == 0;
            // every thread takes the same branch: the vote decides (the first
            // vote also orders the clearing of the bitmap before the updates)
            const bool expired = clock64() - c0 > lim;
            if (!csync.or_(missing && !expired)) break;
            __nanosleep(64);
        }
        if (missing) report_status(kStatusTimeout);
        const int k = (cw == 0 || (cw & kBadBit)) ? 0 : min((cw & (kBadBit - 1)) - 1, cap);
#pragma unroll
        for (int j = 0; j < kPer; ++j) {
            const int c = tid + kConsumers * j;
            if (c < k && e[j] != 0) atomicOr(&bits[(e[j] - 1) >> 5], 1u << ((e[j] - 1) & 31));
        }
        if (cw & kBadBit)
            for (int w = tid; w < mask_words; w += kConsumers) bits[w] = ~0u;
        csync();
    };

    int stage = 0, round = 0;
    int seg_mask = MASK_NONE;
    StageMeta mt;
    const uint32_t ring_s = smem_u32(ring);
    // Waits for the next stage and reads its description.  The producer's
    // own waits are bounded and it always closes the ring with an END stage;
    // this bound only fails if it is gone, and then no warp gets a stage.
    auto wait_stage = [&]() -> bool {
        if (!mbar_wait(&full[stage], (uint32_t)(round & 1), long_limit)) return false;
        mt = meta[stage];
#ifdef SSA_TRACE
        if (lane == 0 && warp == 0) trace_event(p, &misc[15], 15, mt.kind, round * NS + stage);
#endif
        return true;
    };
    auto advance = [&]() {
        if (++stage == NS) {
            stage = 0;
            ++round;
        }
    };
    auto release = [&]() {
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);
#ifdef SSA_TRACE
        if (lane == 0 && warp == 0) trace_event(p, &misc[15], 16, mt.kind, round * NS + stage);
#endif
    };
    auto load_q = [&]() {
            const uint8_t* qs = qbuf + (size_t)stage * L.qbytes;
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk)
#pragma unroll
                for (int half = 0; half < 2; ++half) {
                    const int col = 16 * kk + 8 * half + 2 * tig;
                    qa[kk][half * 2 + 0] =
                        g8 < p.G ? *reinterpret_cast<const uint32_t*>(qs + (g8 * D + col) * 2) : 0u;
                    qa[kk][half * 2 + 1] =
                        g8 + 8 < p.G ? *reinterpret_cast<const uint32_t*>(qs + ((g8 + 8) * D + col) * 2)
                                     : 0u;
                }
    };
    auto seg_start = [&](int pair) {
                if (tid == 0) SSA_TR(TR_C_SEG0, mt.a3, pair);
                mrow[0] = mrow[1] = -INFINITY;
                lrow[0] = lrow[1] = 0.f;
                zero_acc();
                seg_mask = mt.kind == K_GISTV ? MASK_CHUNK : mt.a1;
                if (seg_mask != MASK_NONE) load_bitmap(pair, seg_mask);
    };
    auto seg_end = [&](int pair) {
                // ---- merge the 4 warps' states: one partial per head and segment
                const int G = p.G;
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    float l = lrow[r];
                    l += __shfl_xor_sync(0xffffffffu, l, 1);
                    l += __shfl_xor_sync(0xffffffffu, l, 2);
                    const int h = g8 + 8 * r;
                    if (h < G && tig == 0) {
                        float* mg = merge + ((size_t)warp * G + h) * (D + 2);
                        mg[0] = mrow[r];
                        mg[1] = l;
                    }
                }
                if (kPvHeadsM) {
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        const int h = g8 + 8 * r;
                        if (h < G) {
                            float* mg = merge + ((size_t)warp * G + h) * (D + 2);
#pragma unroll
                            for (int x = 0; x < D / 8; ++x)
                                *reinterpret_cast<float2*>(mg + 2 + x * 8 + 2 * tig) =
                                    make_float2(acc8<D>(acc, x)[2 * r], acc8<D>(acc, x)[2 * r + 1]);
                        }
                    }
                } else {
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int mm = 0; mm < D / 16; ++mm)
#pragma unroll
                            for (int c = 0; c < 4; ++c) {
                                const int h = 8 * nt + 2 * tig + (c & 1);
                                const int dim = 16 * mm + g8 + 8 * (c >> 1);
                                if (h < G)
                                    merge[((size_t)warp * G + h) * (D + 2) + 2 + dim] = acc[nt][mm][c];
                            }
                }
                csync();
                for (int h = warp; h < G; h += kConsumerWarps) {
                    float mw[kConsumerWarps], f[kConsumerWarps];
                    float mx = -INFINITY;
#pragma unroll
                    for (int w = 0; w < kConsumerWarps; ++w) {
                        mw[w] = merge[((size_t)w * G + h) * (D + 2)];
                        mx = fmaxf(mx, mw[w]);
                    }
                    float lsum = 0.f;
#pragma unroll
                    for (int w = 0; w < kConsumerWarps; ++w) {
                        f[w] = (mw[w] == -INFINITY) ? 0.f : exp2f(mw[w] - mx);
                        lsum += f[w] * merge[((size_t)w * G + h) * (D + 2) + 1];
                    }
                    float* dstp = p.partials + partial_offset(p, mt.a3, cta, pair, h, D);
                    if (lane == 0) *reinterpret_cast<float2*>(dstp) = make_float2(mx, lsum);
                    for (int d0 = 2 * lane; d0 < D; d0 += 64) {
                        float ox = 0.f, oy = 0.f;
#pragma unroll
                        for (int w = 0; w < kConsumerWarps; ++w) {
                            const float2 a = *reinterpret_cast<const float2*>(
                                merge + ((size_t)w * G + h) * (D + 2) + 2 + d0);
                            ox += f[w] * a.x;
                            oy += f[w] * a.y;
                        }
                        *reinterpret_cast<float2*>(dstp + 2 + d0) = make_float2(ox, oy);
                    }
                }
                csync();
                if (tid == 0) red_release_add(rec(A_ATTN, pair), 1);
                if (tid == 0) SSA_TR(TR_C_SEG1, mt.a3, pair);
    };

    // Each kind of stage has its own loop over consecutive stages of that
    // kind, so the code a data stage runs is one compact region.
    bool alive = wait_stage();
    while (alive && mt.kind != K_END) {
        if (mt.kind == K_ATTN) {
            // Two consecutive stages of one segment at a time: each warp then
            // has two independent 16-row blocks (Q.K^T, one softmax update,
            // P.V), which hides more of the tensor-core latency.
            do {
                const int pair = mt.pair;
                if (mt.flags & F_QLOAD) load_q();
                if (mt.flags & F_FIRST) seg_start(pair);
                const int s0 = stage;
                const StageMeta m0 = mt;
                int s1 = -1;
                StageMeta m1 = m0;
                if (!(m0.flags & F_LAST)) {
                    // the next stage belongs to the same segment
                    advance();
                    alive = wait_stage();
                    if (alive) {
                        s1 = stage;
                        m1 = mt;
                    }
                }
                const int rbase = 16 * warp;
                const int nv1 = s1 >= 0 ? m1.nvalid : 0;
                // excluded rows: lanes 0..15 test the first stage's rows,
                // lanes 16..31 the second's
                bool e;
                {
                    const StageMeta& mm = lane < 16 ? m0 : m1;
                    const int nvx = lane < 16 ? m0.nvalid : nv1;
                    const int lr = rbase + (lane & 15);
                    e = lr >= nvx;
                    if (!e && seg_mask != MASK_NONE) {
                        const int sid = (mm.a0 + lr) / mm.a2;
                        e = (bits[sid >> 5] >> (sid & 31)) & 1u;
                    }
                }
                const uint32_t ex = __ballot_sync(0xffffffffu, e);
                const uint32_t slotA0 = ring_s + s0 * Cfg<D>::kStageBytes;
                const uint32_t slotA1 = s1 >= 0 ? ring_s + s1 * Cfg<D>::kStageBytes : slotA0;
                const bool ok[2] = {rbase < m0.nvalid, rbase < nv1};
                float sc[2][2][4];
#pragma unroll
                for (int i = 0; i < 2; ++i) {
                    if (ok[i]) {
                        qk16<D>(i ? slotA1 : slotA0, rbase, qa, sc[i], lane);
                    } else {
#pragma unroll
                        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                            for (int c = 0; c < 4; ++c) sc[i][nt][c] = 0.f;
                    }
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            const int t = 16 * i + nt * 8 + 2 * tig + (c & 1);
                            sc[i][nt][c] = ((ex >> t) & 1u) ? -INFINITY : sc[i][nt][c] * scale_log2;
                        }
                }
                if (ok[0] || ok[1]) {
                    const uint32_t vs[2] = {slotA0 + Cfg<D>::kSlotBytes, slotA1 + Cfg<D>::kSlotBytes};
                    const int vr[2] = {rbase, rbase};
                    softmax_pv<D, 2>(sc, vs, vr, ok, mrow, lrow, acc, two_rows, lane);
                }
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&empty[s0]);
                    if (s1 >= 0) mbar_arrive(&empty[s1]);
                }
#ifdef SSA_TRACE
                if (lane == 0 && warp == 0) trace_event(p, &misc[15], 16, K_ATTN, round * NS + stage);
#endif
                if ((s1 >= 0 ? m1.flags : m0.flags) & F_LAST) seg_end(pair);
                if (!alive) break;
                advance();
                alive = wait_stage();
            } while (alive && mt.kind == K_ATTN);
            continue;
        }
        if (mt.kind == K_GISTV) {
            do {
                const uint32_t slotA = ring_s + stage * Cfg<D>::kStageBytes;
                const uint32_t slotB = slotA + Cfg<D>::kSlotBytes;
                const int pair = mt.pair;
                if (mt.flags & F_FIRST) seg_start(pair);
                {
                // ---- values of up to 128 scored gist rows, logits kept in shared
                // memory; warp w takes rows 16w.. (slot A) and 64 + 16w.. (slot B);
                // lane l tests row 16w + l (l < 16) or 64 + 16w + l - 16
                const int rb[2] = {16 * warp, 64 + 16 * warp};
                bool e;
                {
                    // (branch-free: the row's slot word is read for every lane)
                    const int lr = (lane < 16 ? rb[0] : rb[1]) + (lane & 15);
                    const int row = mt.a0 + min(lr, max(mt.nvalid - 1, 0));
                    const int sid = p.g_shift >= 0 ? row >> p.g_shift : row / mt.a2;
                    e = (lr >= mt.nvalid) | ((bits[sid >> 5] >> (sid & 31)) & 1u);
                }
                const uint32_t ex = __ballot_sync(0xffffffffu, e);
                float sc[2][2][4];
                const float* lg = logits + mt.lrow;
                const int ls = p.logit_stride;
                // lanes of heads past G read head 0's logits (their P rows are
                // never used): no divergent loads
                const int ha = g8 < p.G ? g8 : 0, hb = g8 + 8 < p.G ? g8 + 8 : 0;
#pragma unroll
                for (int i = 0; i < 2; ++i)
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt) {
                        // a segment's kept rows start at any row: the pair of rows is
                        // read as one 8-byte word only where it is aligned
                        const int t = rb[i] + nt * 8 + 2 * tig;
                        const float* la = lg + ha * ls + t;
                        const float* lb = lg + hb * ls + t;
                        float2 a, b2 = make_float2(0.f, 0.f);
                        if (!(mt.lrow & 1)) {
                            a = *reinterpret_cast<const float2*>(la);
                            if (two_rows) b2 = *reinterpret_cast<const float2*>(lb);
                        } else {
                            a = make_float2(la[0], la[1]);
                            if (two_rows) b2 = make_float2(lb[0], lb[1]);
                        }
                        const int tb = 16 * i + nt * 8 + 2 * tig;
                        const bool x0 = (ex >> tb) & 1u, x1 = (ex >> (tb + 1)) & 1u;
                        sc[i][nt][0] = x0 ? -INFINITY : a.x;
                        sc[i][nt][1] = x1 ? -INFINITY : a.y;
                        sc[i][nt][2] = x0 ? -INFINITY : b2.x;
                        sc[i][nt][3] = x1 ? -INFINITY : b2.y;
                    }
                const uint32_t vs[2] = {slotA, slotB};
                const int vr[2] = {16 * warp, 16 * warp};
                const bool ok[2] = {rb[0] < mt.nvalid, rb[1] < mt.nvalid};
                if (ok[0]) softmax_pv<D, 2>(sc, vs, vr, ok, mrow, lrow, acc, two_rows, lane);
                }
                release();
                if (mt.flags & F_LAST) seg_end(pair);
                advance();
                alive = wait_stage();
            } while (alive && mt.kind == K_GISTV);
            continue;
        }
        if (mt.kind == K_SCORE) {
            do {
                const uint32_t slotA = ring_s + stage * Cfg<D>::kStageBytes;
                const uint32_t slotB = slotA + Cfg<D>::kSlotBytes;
                const int pair = mt.pair;
                (void)pair;
                if (mt.flags & F_QLOAD) load_q();
            {
                // ---- warp w scores rows 16w.. of box 0 (slot A) and of box 1 (slot B)
                float* lg = p.logits && mt.a5 == 0 ? logits + mt.lrow : nullptr;
                if (two_rows)
                    score_rows2<D, 2>(slotA, slotB, warp, mt.nvalid, p.G, qa, scale, rowmax + mt.a0,
                                      lg, p.logit_stride, scale_log2, lane);
                else
                    score_rows2<D, 1>(slotA, slotB, warp, mt.nvalid, p.G, qa, scale, rowmax + mt.a0,
                                      lg, p.logit_stride, scale_log2, lane);
            }
            release();
            if (mt.flags & F_LAST) {
                csync();
                if (p.fastsel) {
                    // slot score = max over its summary rows (sec. 3.2); the
                    // segment keeps only its 32 best chunks (key, ~chunk):
                    // no chunk outside them can be among the pair's top-k
                    if (mt.flags & F_SEGBEG) segrun = 1ull;
                    // slot index in the pair's list of this level (chunk, superchunk
                    // or candidate position)
                    const int lstride = mt.a5 == 1 ? p.Mc_max : p.h2 ? p.S_max : p.M_max;
                    const uint32_t cbase = (uint32_t)(mt.a3 - pair * lstride);
                    for (int i0 = 32 * warp; i0 < mt.a1; i0 += kConsumers) {
                        const int i = i0 + lane;
                        unsigned long long x = 1ull;
                        if (i < mt.a1) {
                            float v = -INFINITY;
                            if (mt.a4 == 8) {
                                // 8 summary rows per slot: two 16-byte loads
                                const float4* r4 = reinterpret_cast<const float4*>(rowmax + i * 8);
                                const float4 u = r4[0], w = r4[1];
                                v = fmaxf(fmaxf(fmaxf(u.x, u.y), fmaxf(u.z, u.w)),
                                          fmaxf(fmaxf(w.x, w.y), fmaxf(w.z, w.w)));
                            } else {
                                for (int t = 0; t < mt.a4; ++t) v = fmaxf(v, rowmax[i * mt.a4 + t]);
                            }
                            x = ((unsigned long long)score_key(v) << 32) | (uint32_t)~(cbase + i);
                        }
                        segrun = warp_merge_desc(segrun, warp_sort_desc(x, lane), lane);
                    }
                    if (mt.flags & F_SEGEND) {
                        wlists[warp * 32 + lane] = segrun;
                        csync();
                        if (warp == 0) {
                            unsigned long long x = segrun;
#pragma unroll 1
                            for (int w = 1; w < kConsumerWarps; ++w)
                                x = warp_merge_desc(x, wlists[w * 32 + lane], lane);
                            // never 0 (a written entry); the selection polls for it
                            p.cands[((size_t)mt.a5 * (kMaxGrid + P) + cta + pair) * kSegList + lane] = x;
                        }
                    }
                } else {
                    // slot score = max over its summary rows (sec. 3.2)
                    float* dst = mt.a5 == 1 ? p.cand_scores : p.h2 ? p.super_scores : p.scores;
                    for (int i = tid; i < mt.a1 + mt.a2; i += kConsumers) {
                        float v = -INFINITY;
                        if (i < mt.a1 && mt.a4 == 8) {
                            // 8 summary rows per slot: two 16-byte loads
                            const float4* r4 = reinterpret_cast<const float4*>(rowmax + i * 8);
                            const float4 u = r4[0], w = r4[1];
                            v = fmaxf(fmaxf(fmaxf(u.x, u.y), fmaxf(u.z, u.w)),
                                      fmaxf(fmaxf(w.x, w.y), fmaxf(w.z, w.w)));
                        } else if (i < mt.a1) {
                            for (int t = 0; t < mt.a4; ++t) v = fmaxf(v, rowmax[i * mt.a4 + t]);
                        }
                        // for the selection, +0 is stored as -0 (same rank): an
                        // all-zero word means "not written yet"
                        dst[mt.a3 + i] = (so || v != 0.f) ? v : -0.f;
                    }
                }
                csync();
                if (tid == 0) SSA_TR(TR_C_SCD, mt.a5, pair);
            }
                advance();
                alive = wait_stage();
            } while (alive && mt.kind == K_SCORE);
            continue;
        }
        {
            const int pair = mt.pair;
            if (mt.kind == K_SELECT) {
            release();
            if (tid == 0) SSA_TR(TR_C_SEL0, mt.a0, pair);
            const PairSizes z = pair_sizes(p, nbv[pair / p.Hkv]);
            const int what = mt.a0;
            if (what != SEL_VALIDATE) {
                // ---- selection for this pair (sec. 3.3 top-k; sec. 3.5 levels).
                // The scores are self-validating (a written score is never all
                // zero bits): the top-k polls until every one is present, and
                // afterwards this block clears them for the next call.
                float* vals;
                int nv;
                if (p.fastsel) {
                    // merge the 32-best lists of the pair's scoring segments of
                    // this level; the first k of the merged list are the top-k
                    vals = nullptr;
                    nv = 0;
                    const int lvl = what == SEL_CAND ? 1 : 0;
                    int c0, nseg;
                    pv.pair_blocks(lvl ? L_CAND : L_SCORE, pair, c0, nseg);
                    unsigned long long run = 1ull;
                    const long long t0 = clock64(), lim = wait_cycles(p.wait_limit);
                    bool late = false;
                    for (int sg = warp; sg < nseg; sg += kConsumerWarps) {
                        unsigned long long* src =
                            p.cands + ((size_t)lvl * (kMaxGrid + P) + c0 + sg + pair) * kSegList;
                        unsigned long long x = ld_relaxed_u64(src + lane);
                        while (__any_sync(0xffffffffu, x == 0ull)) {
                            if (__shfl_sync(0xffffffffu, (int)(clock64() - t0 > lim), 0)) {
                                late = true;
                                break;
                            }
                            __nanosleep(32);
                            if (x == 0ull) x = ld_relaxed_u64(src + lane);
                        }
                        if (x == 0ull) x = 1ull;
                        src[lane] = 0ull;  // cleared for the next call
                        run = warp_merge_desc(run, x, lane);
                    }
                    if (late && lane == 0) report_status(kStatusTimeout);
                    wlists[warp * 32 + lane] = run;
                    csync();
                    if (warp == 0) {
#pragma unroll 1
                        for (int w = 1; w < kConsumerWarps; ++w)
                            run = warp_merge_desc(run, wlists[w * 32 + lane], lane);
                        const bool sup_level = what == SEL_SUPER;
                        const int k = sup_level ? z.ks : z.kc;
                        int idx = lane < k ? (int)~(uint32_t)run : INT_MAX;
                        idx = warp_sort_asc(idx, lane);
                        if (what == SEL_CAND && lane < k) {
                            // candidate position -> chunk id (an increasing map); the
                            // superchunks come from their published copy (entry + 1)
                            const int pos = idx;
                            if (pos < z.ks * p.J) {
                                const int* sup = rec(A_ENTRIES + p.topk, pair);
                                int e = ld_relaxed(sup + pos / p.J);
                                const long long c1 = clock64();
                                while (e == 0 && clock64() - c1 < lim) {
                                    __nanosleep(64);
                                    e = ld_relaxed(sup + pos / p.J);
                                }
                                if (e == 0) report_status(kStatusTimeout);
                                idx = (e - 1) * p.J + pos % p.J;
                            } else {
                                idx = z.S * p.J + (pos - z.ks * p.J);
                            }
                        }
                        const int cap = sup_level ? p.topk_super : p.topk;
                        int* out = sup_level ? p.sel_super + (size_t)pair * p.topk_super
                                             : p.sel_idx + (size_t)pair * p.topk;
                        int* pub = rec(sup_level ? A_ENTRIES + p.topk : A_ENTRIES, pair);
                        if (lane < cap) out[lane] = lane < k ? idx : -1;
                        if (lane < k) pub[lane] = idx + 1;
                        if (lane == 0) *rec(sup_level ? A_SCOUNT : A_COUNT, pair) = k + 1;
                    }
                } else if (what == SEL_SUPER) {
                    vals = p.super_scores + (size_t)pair * p.S_max;
                    nv = z.S;
                    block_topk<kConsumers>(vals, nv, p.topk_super,
                                           p.sel_super + (size_t)pair * p.topk_super, tsc, csync,
                                           NoProbe(), rec(A_ENTRIES + p.topk, pair), p.wait_limit);
                    if (tid == 0) *rec(A_SCOUNT, pair) = z.ks + 1;
                } else if (what == SEL_CHUNKS) {
                    vals = p.scores + (size_t)pair * p.M_max;
                    nv = z.M;
                    block_topk<kConsumers>(vals, nv, p.topk, p.sel_idx + (size_t)pair * p.topk, tsc,
                                           csync, SSA_PROBE(pair), rec(A_ENTRIES, pair),
                                           p.wait_limit);
                    if (tid == 0) *rec(A_COUNT, pair) = z.kc + 1;
                } else {
                    vals = p.cand_scores + (size_t)pair * p.Mc_max;
                    nv = z.Mc;
                    int* out = p.sel_idx + (size_t)pair * p.topk;
                    block_topk<kConsumers>(vals, nv, p.topk, out, tsc, csync, NoProbe(), nullptr,
                                           p.wait_limit);
                    csync();
                    // candidate position -> chunk id (an increasing map); the
                    // superchunks come from their published copy (entry + 1)
                    const int* sup = rec(A_ENTRIES + p.topk, pair);
                    int* pub = rec(A_ENTRIES, pair);
                    for (int c = tid; c < p.topk; c += kConsumers) {
                        const int pos = out[c];
                        if (pos >= 0) {
                            int m;
                            if (pos < z.ks * p.J) {
                                int e = ld_relaxed(sup + pos / p.J);
                                const long long c0 = clock64(), lim = wait_cycles(p.wait_limit);
                                while (e == 0 && clock64() - c0 < lim) {
                                    __nanosleep(64);
                                    e = ld_relaxed(sup + pos / p.J);
                                }
                                if (e == 0) report_status(kStatusTimeout);
                                m = (e - 1) * p.J + pos % p.J;
                            } else {
                                m = z.S * p.J + (pos - z.ks * p.J);
                            }
                            out[c] = m;
                            pub[c] = m + 1;
                        }
                    }
                    if (tid == 0) *rec(A_COUNT, pair) = z.kc + 1;
                }
                csync();
                for (int i = tid; i < nv; i += kConsumers) vals[i] = 0.f;
                csync();  // the shared union area is free again
            } else {
                // ---- check a caller-given selection and publish it
                const int* sl = p.sel_idx + (size_t)pair * p.topk;
                if (tid == 0) {
                    misc[2] = 1;
                    misc[3] = 0;
                }
                csync();
                for (int c = tid; c < p.topk; c += kConsumers) {
                    const int v = sl[c];
                    const int prev = c > 0 ? sl[c - 1] : -1;
                    bool ok;
                    if (v < 0) {
                        ok = (v == -1);
                    } else {
                        // ascending chunk ids, entries before any -1
                        ok = (v < z.M) && (c == 0 || (prev >= 0 && prev < v));
                        atomicAdd(&misc[3], 1);
                    }
                    if (!ok) misc[2] = 0;
                }
                csync();
                const bool good = misc[2] != 0;
                if (good) {
                    int* pub = rec(A_ENTRIES, pair);
                    for (int c = tid; c < misc[3]; c += kConsumers) pub[c] = sl[c] + 1;
                }
                if (tid == 0) {
                    if (!good) report_status(kStatusBadInput);
                    if (!(p.debug_flags & 1))
                        st_release(rec(A_COUNT, pair), good ? misc[3] + 1 : (kBadBit | 1));
                }
                csync();
            }
            if (tid == 0) SSA_TR(TR_C_SEL1, what, pair);
        } else {  // K_COMBINE
            release();
            if (tid == 0) SSA_TR(TR_C_COMB0, 0, pair);
            // ---- combination of the pair's partial passes (sec. 3.6)
            const int G = p.G;
            const int b = pair / p.Hkv, j = pair % p.Hkv;
            int c0[3], nseg[3];
            pv.pair_blocks(L_META, pair, c0[0], nseg[0]);
            pv.pair_blocks(p.logits ? L_SCORE : L_GIST, pair, c0[1], nseg[1]);
            pv.pair_blocks(L_RAW, pair, c0[2], nseg[2]);
            const int NP = nseg[0] + nseg[1] + nseg[2];
            if (tid == 0) {
                wait_geq(rec(A_ATTN, pair), NP, p.wait_limit);
                bool bad = false;
                if (p.mode == kModeAttnOnly) {
                    wait_geq(rec(A_COUNT, pair), 1, p.wait_limit);
                    bad = (ld_acquire(rec(A_COUNT, pair)) & kBadBit) != 0;
                }
                misc[5] = bad;
            }
            csync();
            const bool bad = misc[5] != 0;
            // lane i of a warp handles segments i, i + 32, ...: its partial's
            // address (for head 0) and, per head, its weight
            auto seg_base = [&](int s) -> const float* {
                int a = 0;
                while (a < 2 && s >= nseg[a]) s -= nseg[a++];
                return p.partials + partial_offset(p, a, c0[a] + s, pair, 0, D);
            };
            // combinations of up to this many partials load in one round
            constexpr int kCombineOne = D == 64 ? 16 : 8;
            if (NP <= kCombineOne) {
                // One round of loads: every lane reads the (m, l) of segment
                // `lane` and its columns of every segment's output together.
                for (int h = warp; h < G; h += kConsumerWarps) {
                    float* op = p.out + ((size_t)b * p.Hq + (size_t)j * G + h) * D;
                    float2 ml = make_float2(-INFINITY, 0.f);
                    if (lane < NP)
                        ml = __ldcg(reinterpret_cast<const float2*>(seg_base(lane) + (size_t)h * (D + 2)));
                    float2 a[kCombineOne][D / 64];
#pragma unroll
                    for (int u = 0; u < kCombineOne; ++u) {
                        if (u < NP) {
                            const float* q = seg_base(u) + (size_t)h * (D + 2) + 2;
#pragma unroll
                            for (int t = 0; t < D / 64; ++t)
                                a[u][t] = __ldcg(reinterpret_cast<const float2*>(q + 64 * t + 2 * lane));
                        } else {
#pragma unroll
                            for (int t = 0; t < D / 64; ++t) a[u][t] = make_float2(0.f, 0.f);
                        }
                    }
                    float mx = ml.x;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                    const float ref = (mx == -INFINITY) ? 0.f : mx;
                    const float fl = (ml.x == -INFINITY) ? 0.f : exp2f(ml.x - ref);
                    float lsum = fl * ml.y;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
                    float ox[D / 64][2];
#pragma unroll
                    for (int t = 0; t < D / 64; ++t) ox[t][0] = ox[t][1] = 0.f;
#pragma unroll
                    for (int u = 0; u < kCombineOne; ++u) {
                        const float f = __shfl_sync(0xffffffffu, fl, u);
#pragma unroll
                        for (int t = 0; t < D / 64; ++t) {
                            ox[t][0] += f * a[u][t].x;
                            ox[t][1] += f * a[u][t].y;
                        }
                    }
                    const float inv = (!bad && lsum > 0.f) ? 1.f / lsum : 0.f;
#pragma unroll
                    for (int t = 0; t < D / 64; ++t)
                        *reinterpret_cast<float2*>(op + 64 * t + 2 * lane) =
                            make_float2(ox[t][0] * inv, ox[t][1] * inv);
                }
            } else
            for (int h = warp; h < G; h += kConsumerWarps) {
                float* op = p.out + ((size_t)b * p.Hq + (size_t)j * G + h) * D;
                float ox[D / 64][2];
#pragma unroll
                for (int t = 0; t < D / 64; ++t) ox[t][0] = ox[t][1] = 0.f;
                float mx = -INFINITY, lsum = 0.f;
                // pass 1: maxima and normaliser (one load per lane and 32 segments)
                for (int sb = 0; sb < NP; sb += 32) {
                    float2 ml = make_float2(-INFINITY, 0.f);
                    if (sb + lane < NP)
                        ml = __ldcg(reinterpret_cast<const float2*>(seg_base(sb + lane) +
                                                                    (size_t)h * (D + 2)));
                    float m32 = ml.x;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1)
                        m32 = fmaxf(m32, __shfl_xor_sync(0xffffffffu, m32, o));
                    const float mnew = fmaxf(mx, m32);
                    const float ref = (mnew == -INFINITY) ? 0.f : mnew;
                    const float alpha = exp2f(mx - ref);
                    const float fl = (ml.x == -INFINITY) ? 0.f : exp2f(ml.x - ref);
                    float l32 = fl * ml.y;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) l32 += __shfl_xor_sync(0xffffffffu, l32, o);
                    lsum = lsum * alpha + l32;
#pragma unroll
                    for (int t = 0; t < D / 64; ++t) {
                        ox[t][0] *= alpha;
                        ox[t][1] *= alpha;
                    }
                    mx = mnew;
                    // pass 2 for these 32 segments: weighted sum of their outputs,
                    // kCB independent loads in flight per lane
                    const float* mine = (sb + lane < NP)
                                            ? seg_base(sb + lane) + (size_t)h * (D + 2) + 2
                                            : p.partials;
                    const int cnt = min(32, NP - sb);
                    constexpr int kCB = D == 64 ? 16 : 4;
                    for (int i0 = 0; i0 < cnt; i0 += kCB) {
                        float2 a[kCB][D / 64];
                        float f[kCB];
#pragma unroll
                        for (int u = 0; u < kCB; ++u) {
                            const int i = (i0 + u) & 31;
                            const float* q = reinterpret_cast<const float*>(__shfl_sync(
                                0xffffffffu, reinterpret_cast<uintptr_t>(mine), i));
                            f[u] = __shfl_sync(0xffffffffu, fl, i);
                            if (i0 + u < cnt) {
#pragma unroll
                                for (int t = 0; t < D / 64; ++t)
                                    a[u][t] = __ldcg(reinterpret_cast<const float2*>(
                                        q + 64 * t + 2 * lane));
                            } else {
                                f[u] = 0.f;
#pragma unroll
                                for (int t = 0; t < D / 64; ++t) a[u][t] = make_float2(0.f, 0.f);
                            }
                        }
#pragma unroll
                        for (int u = 0; u < kCB; ++u)
#pragma unroll
                            for (int t = 0; t < D / 64; ++t) {
                                ox[t][0] += f[u] * a[u][t].x;
                                ox[t][1] += f[u] * a[u][t].y;
                            }
                    }
                }
                const float inv = (!bad && lsum > 0.f) ? 1.f / lsum : 0.f;
#pragma unroll
                for (int t = 0; t < D / 64; ++t)
                    *reinterpret_cast<float2*>(op + 64 * t + 2 * lane) =
                        make_float2(ox[t][0] * inv, ox[t][1] * inv);
            }
            csync();
            {
                // clear this pair's record for the next call
                int* r = rec(0, pair);
                const int used = A_ENTRIES + p.topk + (p.h2 ? p.topk_super : 0);
                for (int a = tid; a < used; a += kConsumers) r[a] = 0;
            }
            if (tid == 0) SSA_TR(TR_C_COMB1, 0, pair);
        }
        }
        advance();
        alive = wait_stage();
    }
    if (tid == 0) {
        SSA_TR(TR_KEND, 0, 0);
        SSA_TR(TR_KEND | 0x80, 0, 0);
    }
}

}  // namespace fused
}  // namespace ssa
