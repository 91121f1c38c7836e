// ssa_fused.cuh -- the fused, persistent decode kernel for bf16, d in {64,128}.
//
// One launch runs the whole decode step ("Simplified Sparse Attention via
// Gist Tokens", sec. 3.2 scoring, sec. 3.3 top-k + hybrid attention, sec. 3.5
// coarse-to-fine selection, sec. 3.6 split partial attention + combination):
//
//   score items    -- gist keys (two level: meta-gist keys) of a slot range
//   select items   -- one per (sequence, KV head) pair: top-k over its
//                     scores (or: check a caller-given selection)
//   cand items     -- two level only: gist keys of the candidate chunks
//   select items   -- two level only: top-k over the candidates
//   attention      -- a range of 64-row tiles of the unfolded context
//   combine items  -- one per pair: merge its split partials into `out`
//
// Work is handed out by a global ticket counter in that order.  An item only
// ever waits for items with smaller tickets (a count of finished items, or a
// published selection), and a ticket is only taken by a running block, so
// the waits always end; each is bounded anyway.  Items signal completion with
// a release increment and never wait on it themselves, so no item's tail
// holds a block.  A combine item resets its pair's control words for the
// next call.
//
// Block layout: 4 consumer warps + 1 producer warp.  The producer streams
// 64-row tiles with 2-D TMA (128-byte swizzle) into a ring of stages (slot A:
// keys, slot B: values; score stages use both slots for keys) and never
// stalls the consumers on control flow.  Each consumer warp takes 16 rows of
// every stage: Q.K^T and P.V run on tensor cores (mma.sync m16n8k16, bf16 in,
// fp32 accumulate; the GQA group's query heads are the M rows), the softmax
// is an fp32 online softmax in the log2 domain, and P is fed to the P.V
// product as bf16 hi + lo parts so it keeps ~16 significant bits.
#pragma once

#include "ssa_device.cuh"
#include "ssa_internal.h"

namespace ssa {
namespace fused {

constexpr int kConsumerWarps = 4;
constexpr int kConsumers = kConsumerWarps * 32;
constexpr int kThreads = kConsumers + 32;
constexpr int kBoxRows = 64;          // rows per TMA box and per attention tile
constexpr int kRowmaxCap = 1024;      // summary rows per score item
constexpr int kBarConsumers = 1;      // named barrier id of the consumer warps

enum : int { K_END = 0, K_SCORE = 1, K_ATTN = 2, K_SELECT = 3, K_COMBINE = 4 };
enum : int { F_FIRST = 1, F_LAST = 2, F_QLOAD = 4 };
enum : int { L_GIST = 0, L_META = 1, L_CAND = 2, L_VALIDATE = 3 };

// Control words.  The ticket and exit counters sit in their own 128-byte
// lines, then one record of Plan::pair_ints words per (sequence, KV head):
//   line 0   completion counters (score, candidate and attention items);
//   line 1   published counts: count + 1 (0: not published yet; kBadBit:
//            the caller's selection was rejected);
//   then     the published selection itself, entry + 1 (0: not written yet):
//            topk chunk entries, then topk_super superchunk entries.
// Every word is written once per call and cleared by the pair's combine item,
// so a reader needs no separate ready flag: one round of relaxed loads tells
// whether the count and every entry it needs are there.
constexpr int kLineInts = 32;
constexpr int C_TICKET = 0, C_EXIT = kLineInts, C_ARR = 2 * kLineInts;
enum : int {
    A_DONE_A = 0,             // score items (first level) finished
    A_DONE_B = 1,             // candidate score items finished
    A_ATTN = 2,               // attention partials written (4 per item)
    A_COUNT = kLineInts,      // published chunk selection count
    A_SCOUNT = kLineInts + 1, // published superchunk selection count
    A_ENTRIES = 2 * kLineInts // chunk entries, then superchunk entries
};
constexpr int kBadBit = 1 << 30;

struct StageMeta {
    int kind, pair, nvalid, flags;
    int row_off, item, nslot, npad;
    int dst, ntok;
    uint32_t rmask_lo, rmask_hi;  // attention: excluded rows of the tile
};

template <int D>
struct Cfg {
    static constexpr int kSlotBytes = kBoxRows * D * 2;
    static constexpr int kStageBytes = 2 * kSlotBytes;
    static constexpr int kStages = (D == 64) ? 6 : 3;
    static constexpr int kBoxBytes = kBoxRows * D * 2;  // one 64-row box, all D columns
};

struct SmemLayout {
    int ring, qbuf, qbytes, meta, bars, psel, psup, uni, misc, total;
};

template <int D>
__host__ __device__ inline SmemLayout smem_layout(const Plan& p) {
    SmemLayout L;
    const int NS = Cfg<D>::kStages;
    const int G = p.G;
    const int topk_super = p.h2 ? p.topk_super : 0;
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
    o += ((topk_super + 3) / 4 * 4) * 4;
    o = (o + 15) / 16 * 16;
    L.uni = o;
    // the consumers use this area for one thing at a time
    int u = kRowmaxCap * 4;                                      // score rows
    const int tk = (int)sizeof(TopkScratch);                     // top-k
    u = u > tk ? u : tk;
    const int cmb = 3 * G * p.attn_items * kConsumerWarps * 4;   // combination
    u = u > cmb ? u : cmb;
    o += (u + 15) / 16 * 16;
    L.misc = o;
    o += 64;
    L.total = o + 1024;  // slack to align the ring to 1024 bytes
    return L;
}

// Timeline trace: builds compiled with SSA_TRACE record (time, event, a, b)
// per block into Plan::trace; the product build compiles these to nothing.
enum : int { TR_KSTART = 1, TR_TICKET, TR_P_READY, TR_P_ISSUED, TR_C_FIRST, TR_C_LAST,
             TR_C_DONE, TR_C_TOPK0, TR_C_TOPK1, TR_C_COMB0, TR_C_COMB1, TR_KEND };
#ifdef SSA_TRACE
// Events carry the per-SM cycle counter (cheap); KSTART and KEND also record
// the global timer in a second event (ev | 0x80) so blocks can be aligned.
__device__ __forceinline__ void trace_event(const Plan& p, int* counter, int ev, int a, int b) {
    if (!p.trace) return;
    const int i = atomicAdd(counter, 1);
    if (i >= p.trace_cap) return;
    const uint64_t t = (ev & 0x80) ? now_ns() : (uint64_t)clock64();
    p.trace[(size_t)blockIdx.x * p.trace_cap + i] =
        make_uint4((uint32_t)t, (uint32_t)(t >> 32), (uint32_t)ev | ((uint32_t)a << 8), (uint32_t)b);
}
#define SSA_TR(ev, a, b) trace_event(p, &misc[15], (ev), (a), (b))
struct TraceProbe {
    const Plan& p;
    int* counter;
    int pair;
    __device__ void operator()(int stage) const {
        if ((threadIdx.x & 31) == 0 && threadIdx.x < 128)
            trace_event(p, counter, 13, stage + 16 * (threadIdx.x >> 5), pair);
    }
};
#define SSA_PROBE(pair) TraceProbe{p, &misc[15], (pair)}
#else
#define SSA_PROBE(pair) NoProbe()
#define SSA_TR(ev, a, b) ((void)0)
#endif

__device__ __forceinline__ int pair_of(const StageMeta& m) { return m.pair; }

struct ConsumerSync {
    __device__ void operator()() const { named_sync(kBarConsumers, kConsumers); }
};

__device__ __forceinline__ int seq_len_checked(const Plan& p, int b) {
    int n = __ldg(p.seq_lens + b);
    if (n < 1 || n > p.n_max) return -1;
    return n;
}

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

// acc[dim n-tile] += P(hi+lo) * V for 16 rows starting at r0 of a value slot.
template <int D>
__device__ __forceinline__ void pv16(uint32_t slot, int r0, const uint32_t (&phi)[4],
                                     const uint32_t (&plo)[4], float (&acc)[D / 8][4], int lane) {
    const int row = r0 + (lane & 15);
    const int csel = lane >> 4;
#pragma unroll
    for (int nn = 0; nn < D / 16; ++nn) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_trans(tile_addr<D>(slot, row, 2 * nn + csel), b0, b1, b2, b3);
        mma_bf16_16816(acc[2 * nn], phi, b0, b1);
        mma_bf16_16816(acc[2 * nn], plo, b0, b1);
        mma_bf16_16816(acc[2 * nn + 1], phi, b2, b3);
        mma_bf16_16816(acc[2 * nn + 1], plo, b2, b3);
    }
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
    int* psel;
    int* psup;
    int lane;
    int stage = 0, round = 0;

    __device__ int acquire() {
        const int s = stage;
        if (round > 0) {
            if (lane == 0) mbar_wait(&empty[s], (uint32_t)((round - 1) & 1), p.wait_limit);
            __syncwarp();
        }
        return s;
    }
    __device__ void advance() {
        if (++stage == Cfg<D>::kStages) {
            stage = 0;
            ++round;
        }
    }
    __device__ uint8_t* slot(int s, int which) {
        return ring + (size_t)s * Cfg<D>::kStageBytes + which * Cfg<D>::kSlotBytes;
    }
    // one 64-row box (all D columns) of map `m` at global row y into slot
    __device__ void box(int s, int which, const CUtensorMap* m, int y) {
#pragma unroll
        for (int sub = 0; sub < D / 64; ++sub)
            tma_load_2d(slot(s, which) + sub * (kBoxRows * 128), m, sub * 64, y, &full[s]);
    }
    __device__ void load_q(int s, int b, int j) {
        const __nv_bfloat16* src =
            static_cast<const __nv_bfloat16*>(p.q) + ((size_t)b * p.Hq + (size_t)j * p.G) * D;
        bulk_load(qbuf + (size_t)s * qbytes, src, (uint32_t)(p.G * D * 2), &full[s]);
    }
    __device__ void push_plain(int kind, int pair, int flags, int item) {
        const int s = acquire();
        if (lane == 0) {
            StageMeta m = {};
            m.kind = kind;
            m.pair = pair;
            m.flags = flags;
            m.item = item;
            meta[s] = m;
            mbar_arrive(&full[s]);
        }
        __syncwarp();
        advance();
    }

    // Score item: rows [0, rows) of a summary tensor starting at global row y0.
    __device__ void score_item(int pair, int level, const CUtensorMap* m, int y0, int rows,
                               int nslot, int npad, int dst, int ntok) {
        const int b = pair / p.Hkv, j = pair % p.Hkv;
        if (rows <= 0) {
            const int s = acquire();
            if (lane == 0) {
                StageMeta mt = {};
                mt.kind = K_SCORE;
                mt.pair = pair;
                mt.flags = F_FIRST | F_LAST;
                mt.item = level;
                mt.nslot = 0;
                mt.npad = npad;
                mt.dst = dst;
                mt.ntok = ntok;
                meta[s] = mt;
                mbar_arrive(&full[s]);
            }
            __syncwarp();
            advance();
            return;
        }
        for (int off = 0; off < rows; off += 2 * kBoxRows) {
            const int s = acquire();
            const int nv = min(2 * kBoxRows, rows - off);
            const int nbox = (nv + kBoxRows - 1) / kBoxRows;
            const bool first = off == 0;
            if (lane == 0) {
                StageMeta mt = {};
                mt.kind = K_SCORE;
                mt.pair = pair;
                mt.nvalid = nv;
                mt.flags = (first ? (F_FIRST | F_QLOAD) : 0) |
                           (off + 2 * kBoxRows >= rows ? F_LAST : 0);
                mt.row_off = off;
                mt.item = level;
                mt.nslot = nslot;
                mt.npad = npad;
                mt.dst = dst;
                mt.ntok = ntok;
                meta[s] = mt;
                uint32_t bytes = nbox * Cfg<D>::kBoxBytes + (first ? p.G * D * 2 : 0);
                mbar_arrive_expect_tx(&full[s], bytes);
                if (first) load_q(s, b, j);
                for (int bx = 0; bx < nbox; ++bx) box(s, bx, m, y0 + off + bx * kBoxRows);
            }
            __syncwarp();
            advance();
        }
    }

    // Reads a published selection (count word, `cap` entries at `ent`) into
    // shared `dst` as plain indices.  One round of relaxed loads per attempt;
    // polls with back-off until the count and its entries are all written.
    // Returns the count and sets `bad` for a rejected caller selection; a
    // wait that runs out records a timeout and returns 0.
    __device__ int fetch_selection(const int* cnt_word, const int* ent, int cap, int* dst,
                                   bool& bad) {
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
                bad = false;
                return 0;
            }
            __nanosleep(sleep_ns);
            if (sleep_ns < 512) sleep_ns *= 2;
        }
    }

    // Rows of [r0, r0+cnt) (in units where slot x covers rows [x*ntok, x*ntok+ntok))
    // that belong to one of the n sorted slots in list[]: bit r set.
    __device__ uint64_t excluded_rows(const int* list, int n, int r0, int cnt, int ntok) {
        uint64_t bits = 0;
        for (int c = lane; c < n; c += 32) {
            const int x = list[c];
            const int lo = max(x * ntok, r0), hi = min(x * ntok + ntok, r0 + cnt);
            for (int r = lo; r < hi; ++r) bits |= 1ull << (r - r0);
        }
        uint32_t lo32 = __reduce_or_sync(0xffffffffu, (uint32_t)bits);
        uint32_t hi32 = __reduce_or_sync(0xffffffffu, (uint32_t)(bits >> 32));
        return ((uint64_t)hi32 << 32) | lo32;
    }
};

// Tile descriptor of one attention unit.
struct Tile {
    int src;      // 0 raw, 1 gist, 2 meta
    int y;        // global row of the TMA box
    int nvalid;   // rows of the tile in the context (before exclusions)
    uint64_t excl;
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
    constexpr int NS = Cfg<D>::kStages;
    uint8_t* ring = smem + L.ring;
    uint8_t* qbuf = smem + L.qbuf;
    StageMeta* meta = reinterpret_cast<StageMeta*>(smem + L.meta);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
    uint64_t* empty = full + NS;
    int* psel = reinterpret_cast<int*>(smem + L.psel);
    int* psup = reinterpret_cast<int*>(smem + L.psup);
    uint8_t* uni = smem + L.uni;
    int* misc = reinterpret_cast<int*>(smem + L.misc);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        misc[15] = 0;
        for (int s = 0; s < NS; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kConsumerWarps);
        }
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        SSA_TR(TR_KSTART | 0x80, 0, 0);
        SSA_TR(TR_KSTART, 0, 0);
    }

    // ticket phases, in hand-out order
    const int P = p.n_pairs;
    const bool so = p.mode == kModeScoreOnly;
    const int nA = (p.mode == kModeAttnOnly) ? 0 : P * p.score_items;  // score items
    const int nS1 = so ? 0 : P;                                         // first selection
    const int nB = p.h2 ? P * p.cand_items : 0;                         // candidate scoring
    const int nS2 = p.h2 ? P : 0;                                       // second selection
    const int nC = so ? 0 : P * p.attn_items;                           // attention
    const int nD = so ? 0 : P;                                          // combination
    const int oS1 = nA, oB = oS1 + nS1, oS2 = oB + nB, oC = oS2 + nS2, oD = oC + nC;
    const int total = oD + nD;
    int* ctrl = p.ctrl;
    auto arr = [&](int a, int pair) -> int* { return ctrl + C_ARR + pair * p.pair_ints + a; };

    // ================================================================ producer
    if (warp == kConsumerWarps) {
        Producer<D> pr{p, {&tm_kraw, &tm_vraw, &tm_kgist, &tm_vgist, &tm_kmeta, &tm_vmeta},
                       ring, qbuf, L.qbytes, meta, full, empty, psel, psup, lane};
        if (lane == 0) {
            for (int i = 0; i < 6; ++i) prefetch_tensormap(pr.tm[i]);
        }
        // lane 0 keeps one ticket in hand: the atomic for the next item is
        // issued as soon as the current one is known, so its latency overlaps
        // the current item's issue work.
        // Scoring alone never waits, so it strides over items statically and
        // needs no control words.
        const bool dyn = p.mode != kModeScoreOnly;
        int next_t = 0;
        if (lane == 0) next_t = dyn ? atomicAdd(ctrl + C_TICKET, 1) : (int)blockIdx.x;
        for (;;) {
            const int t = __shfl_sync(0xffffffffu, next_t, 0);
            if (t >= total) {
                pr.push_plain(K_END, 0, 0, 0);
                break;
            }
            if (lane == 0) next_t = dyn ? atomicAdd(ctrl + C_TICKET, 1) : t + (int)gridDim.x;
            if (lane == 0) SSA_TR(TR_TICKET, t < oS1 ? 0 : t < oC ? 1 : t < oD ? 2 : 3, t);

            if (t < oS1) {
                const int pair = t / p.score_items, i = t % p.score_items;
                const int b = pair / p.Hkv;
                int n = seq_len_checked(p, b);
                if (n < 0) {
                    if (lane == 0 && i == 0 && pair % p.Hkv == 0) report_status(kStatusBadInput);
                    n = 0;
                }
                const int M = n / p.C;
                if (!p.h2) {
                    const int s0 = i * p.score_spi;
                    const int s1 = min(s0 + p.score_spi, p.M_max);
                    const int vs = max(0, min(M, s1) - s0);
                    const int npad = (p.mode == kModeScoreOnly) ? (s1 - s0 - vs) : 0;
                    pr.score_item(pair, L_GIST, &tm_kgist, (pair * p.M_max + s0) * p.g, vs * p.g,
                                  vs, npad, pair * p.M_max + s0, p.g);
                } else {
                    const int S = M / p.J;
                    const int s0 = i * p.score_spi;
                    const int s1 = min(s0 + p.score_spi, p.S_max);
                    const int vs = max(0, min(S, s1) - s0);
                    pr.score_item(pair, L_META, &tm_kmeta, (pair * p.S_max + s0) * p.gm,
                                  vs * p.gm, vs, 0, pair * p.S_max + s0, p.gm);
                }
                if (lane == 0) SSA_TR(TR_P_ISSUED, 0, t);
                continue;
            }
            if (t < oB || (t >= oS2 && t < oC)) {
                // selection item: after every score item of the pair is done
                const bool first = t < oB;
                const int pair = first ? t - oS1 : t - oS2;
                int level;
                if (!first) {
                    level = L_CAND;
                    if (lane == 0) wait_geq(arr(A_DONE_B, pair), p.cand_items, p.wait_limit);
                } else if (p.mode == kModeAttnOnly) {
                    level = L_VALIDATE;
                } else {
                    level = p.h2 ? L_META : L_GIST;
                    if (lane == 0) wait_geq(arr(A_DONE_A, pair), p.score_items, p.wait_limit);
                }
                __syncwarp();
                pr.push_plain(K_SELECT, pair, F_FIRST | F_LAST, level);
                continue;
            }
            if (t >= oD) {
                // combination item: after every attention item of the pair
                const int pair = t - oD;
                if (lane == 0)
                    wait_geq(arr(A_ATTN, pair), p.attn_items * kConsumerWarps, p.wait_limit);
                __syncwarp();
                pr.push_plain(K_COMBINE, pair, F_FIRST | F_LAST, 0);
                continue;
            }
            if (t < oS2) {
                const int u = t - oB;
                const int pair = u / p.cand_items, i = u % p.cand_items;
                const int b = pair / p.Hkv;
                int n = seq_len_checked(p, b);
                if (n < 0) n = 0;
                const int M = n / p.C, S = M / p.J, R = M - S * p.J;
                bool bad_s;
                const int ks = pr.fetch_selection(arr(A_SCOUNT, pair),
                                                  arr(A_ENTRIES + p.topk, pair), p.topk_super,
                                                  psup, bad_s);
                int chunk0 = 0, nch = 0, c0 = 0;
                if (i < p.topk_super) {
                    if (i < ks) {
                        chunk0 = psup[i] * p.J;
                        nch = p.J;
                        c0 = i * p.J;
                    }
                } else {
                    chunk0 = S * p.J;
                    nch = R;
                    c0 = ks * p.J;
                }
                pr.score_item(pair, L_CAND, &tm_kgist, (pair * p.M_max + chunk0) * p.g, nch * p.g,
                              nch, 0, pair * p.Mc_max + c0, p.g);
                if (lane == 0) SSA_TR(TR_P_ISSUED, 1, t);
                continue;
            }
            // ------------------------------------------------ attention item
            const int u = t - oC;
            const int pair = u / p.attn_items, item = u % p.attn_items;
            const int b = pair / p.Hkv, j = pair % p.Hkv;
            int n = seq_len_checked(p, b);
            if (n < 0) n = 0;
            const int M = n / p.C, T = n - M * p.C;
            const int tpc = (p.C + kBoxRows - 1) / kBoxRows;
            int Ug = 0, Um = 0, Ucs = 0, Urem = 0, tsc = 0, S = 0, R = 0, kmax_s = 0, kmax_c;
            if (!p.h2) {
                Ug = (M * p.g + kBoxRows - 1) / kBoxRows;
                kmax_c = min(p.topk, M);
            } else {
                S = M / p.J;
                R = M - S * p.J;
                kmax_s = min(p.topk_super, S);
                Um = (S * p.gm + kBoxRows - 1) / kBoxRows;
                tsc = (p.J * p.g + kBoxRows - 1) / kBoxRows;
                Ucs = kmax_s * tsc;
                Urem = (R * p.g + kBoxRows - 1) / kBoxRows;
                kmax_c = min(p.topk, kmax_s * p.J + R);
            }
            const int Usum = Ug + Um + Ucs + Urem;  // summary tiles
            const int Ur = kmax_c * tpc;
            const int Ut = (T + kBoxRows - 1) / kBoxRows;
            const long long U = (long long)Usum + Ur + Ut;
            const int u0 = (int)((U * item) / p.attn_items);
            const int u1 = (int)((U * (item + 1)) / p.attn_items);

            bool have_sel = false, bad_sel = false;
            int ksel = 0, ksup = 0;
            auto need_selection = [&]() {
                if (have_sel) return;
                have_sel = true;
                ksel = pr.fetch_selection(arr(A_COUNT, pair), arr(A_ENTRIES, pair), p.topk, psel,
                                          bad_sel);
                if (p.h2) {
                    bool b2;
                    ksup = pr.fetch_selection(arr(A_SCOUNT, pair), arr(A_ENTRIES + p.topk, pair),
                                              p.topk_super, psup, b2);
                }
                if (lane == 0) SSA_TR(TR_P_READY, pair, item);
                if (bad_sel) {  // rejected caller selection: this pair attends to nothing
                    ksel = 0;
                    ksup = 0;
                }
            };

            Tile pending{};
            bool has_pending = false, emitted = false;
            auto emit = [&](const Tile& tl, bool last) {
                const int s = pr.acquire();
                if (lane == 0) {
                    StageMeta mt = {};
                    mt.kind = K_ATTN;
                    mt.pair = pair;
                    mt.nvalid = tl.nvalid;
                    mt.flags = (emitted ? 0 : (F_FIRST | F_QLOAD)) | (last ? F_LAST : 0);
                    mt.item = item;
                    mt.rmask_lo = (uint32_t)tl.excl;
                    mt.rmask_hi = (uint32_t)(tl.excl >> 32);
                    meta[s] = mt;
                    uint32_t bytes = 2 * Cfg<D>::kBoxBytes + (emitted ? 0 : p.G * D * 2);
                    mbar_arrive_expect_tx(&full[s], bytes);
                    if (!emitted) pr.load_q(s, b, j);
                    const CUtensorMap* km = tl.src == 0 ? &tm_kraw : tl.src == 1 ? &tm_kgist : &tm_kmeta;
                    const CUtensorMap* vm = tl.src == 0 ? &tm_vraw : tl.src == 1 ? &tm_vgist : &tm_vmeta;
                    pr.box(s, 0, km, tl.y);
                    pr.box(s, 1, vm, tl.y);
                }
                __syncwarp();
                pr.advance();
                emitted = true;
            };

            for (int v = u0; v < u1; ++v) {
                Tile tl{};
                bool ok = true;
                if (v < Usum) {
                    need_selection();
                    if (!p.h2) {
                        const int r0 = v * kBoxRows;
                        tl.src = 1;
                        tl.nvalid = min(kBoxRows, M * p.g - r0);
                        tl.y = pair * p.M_max * p.g + r0;
                        tl.excl = pr.excluded_rows(psel, ksel, r0, tl.nvalid, p.g);
                    } else if (v < Um) {
                        const int r0 = v * kBoxRows;
                        tl.src = 2;
                        tl.nvalid = min(kBoxRows, S * p.gm - r0);
                        tl.y = pair * p.S_max * p.gm + r0;
                        tl.excl = pr.excluded_rows(psup, ksup, r0, tl.nvalid, p.gm);
                    } else {
                        const int w = v - Um;
                        int r0, cnt;
                        if (w < Ucs) {
                            const int slot = w / tsc, part = w % tsc;
                            if (slot >= ksup) {
                                ok = false;
                            } else {
                                r0 = psup[slot] * p.J * p.g + part * kBoxRows;
                                cnt = min(kBoxRows, p.J * p.g - part * kBoxRows);
                            }
                        } else {
                            r0 = S * p.J * p.g + (w - Ucs) * kBoxRows;
                            cnt = min(kBoxRows, M * p.g - r0);
                        }
                        if (ok) {
                            tl.src = 1;
                            tl.nvalid = cnt;
                            tl.y = pair * p.M_max * p.g + r0;
                            tl.excl = pr.excluded_rows(psel, ksel, r0, cnt, p.g);
                        }
                    }
                    if (ok) {
                        const uint64_t valid =
                            tl.nvalid >= 64 ? ~0ull : ((1ull << tl.nvalid) - 1ull);
                        if ((tl.excl & valid) == valid) ok = false;  // every row excluded
                    }
                } else if (v < Usum + Ur) {
                    need_selection();
                    const int c = (v - Usum) / tpc, part = (v - Usum) % tpc;
                    if (c >= ksel) {
                        ok = false;
                    } else {
                        const int m = psel[c];
                        tl.src = 0;
                        tl.nvalid = min(kBoxRows, p.C - part * kBoxRows);
                        tl.y = pair * p.n_max + m * p.C + part * kBoxRows;
                        tl.excl = 0;
                    }
                } else {
                    const int r0 = M * p.C + (v - Usum - Ur) * kBoxRows;
                    tl.src = 0;
                    tl.nvalid = min(kBoxRows, n - r0);
                    tl.y = pair * p.n_max + r0;
                    tl.excl = 0;
                }
                if (bad_sel) ok = false;
                if (!ok) continue;
                if (has_pending) emit(pending, false);
                pending = tl;
                has_pending = true;
            }
            if (lane == 0) SSA_TR(TR_P_ISSUED, 2, t);
            if (has_pending) {
                emit(pending, true);
            } else {
                // nothing of the context falls in this item: neutral partial
                const int s = pr.acquire();
                if (lane == 0) {
                    StageMeta mt = {};
                    mt.kind = K_ATTN;
                    mt.pair = pair;
                    mt.nvalid = 0;
                    mt.flags = F_FIRST | F_LAST;
                    mt.item = item;
                    meta[s] = mt;
                    mbar_arrive(&full[s]);
                }
                __syncwarp();
                pr.advance();
            }
        }
        return;
    }

    // ================================================================ consumers
    const int tid = threadIdx.x;  // 0..127
    const int g8 = lane >> 2, tig = lane & 3;
    const float scale = rsqrtf((float)D);
    const float scale_log2 = scale * 1.4426950408889634f;
    float* rowmax = reinterpret_cast<float*>(uni);
    TopkScratch& tsc = *reinterpret_cast<TopkScratch*>(uni);
    float* cmb = reinterpret_cast<float*>(uni);
    ConsumerSync csync;

    uint32_t qa[D / 16][4];
    float acc[D / 8][4];
    float mrow[2], lrow[2];
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk)
#pragma unroll
        for (int c = 0; c < 4; ++c) qa[kk][c] = 0u;

    int stage = 0, round = 0;
    for (;;) {
        if (!mbar_wait(&full[stage], (uint32_t)(round & 1), p.wait_limit)) break;
        const StageMeta mt = meta[stage];
        if (mt.kind == K_END) break;
        if (tid == 0 && (mt.flags & F_FIRST)) SSA_TR(TR_C_FIRST, mt.kind, pair_of(mt));
        const uint32_t slotA = smem_u32(ring + (size_t)stage * Cfg<D>::kStageBytes);
        const uint32_t slotB = slotA + Cfg<D>::kSlotBytes;
        if (mt.flags & F_QLOAD) {
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
        }
        const int pair = mt.pair;

        if (mt.kind == K_SCORE) {
#pragma unroll
            for (int sl = 0; sl < 2; ++sl) {
                const int rbase = sl * kBoxRows + 16 * warp;
                if (rbase < mt.nvalid) {
                    float s[2][4];
                    qk16<D>(sl ? slotB : slotA, 16 * warp, qa, s, lane);
#pragma unroll
                    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                        for (int c = 0; c < 2; ++c) {
                            float v = g8 < p.G ? s[nt][c] : -INFINITY;
                            if (g8 + 8 < p.G) v = fmaxf(v, s[nt][2 + c]);
                            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
                            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
                            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
                            const int lr = rbase + nt * 8 + 2 * tig + c;
                            if (g8 == 0 && lr < mt.nvalid) rowmax[mt.row_off + lr] = v * scale;
                        }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            if (mt.flags & F_LAST) {
                if (tid == 0) SSA_TR(TR_C_LAST, K_SCORE, pair);
                csync();
                float* dst = mt.item == L_GIST ? p.scores
                             : mt.item == L_META ? p.super_scores
                                                 : p.cand_scores;
                for (int i = tid; i < mt.nslot + mt.npad; i += kConsumers) {
                    float v = -INFINITY;
                    if (i < mt.nslot)
                        for (int t = 0; t < mt.ntok; ++t) v = fmaxf(v, rowmax[i * mt.ntok + t]);
                    dst[mt.dst + i] = v;
                }
                csync();
                if (p.mode != kModeScoreOnly && tid == 0)
                    red_release_add(arr(mt.item == L_CAND ? A_DONE_B : A_DONE_A, pair), 1);
                if (tid == 0) SSA_TR(TR_C_DONE, K_SCORE, pair);
            }
        } else if (mt.kind == K_SELECT) {
#ifdef SSA_TRACE
            if (lane == 0) trace_event(p, &misc[15], 13, 15 + 16 * warp, pair);
#endif
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            if (tid == 0) SSA_TR(TR_C_TOPK0, mt.item, pair);
            if (mt.item != L_VALIDATE) {
                // ---- selection for this pair (sec. 3.3 top-k; sec. 3.5 levels)
                const int b = pair / p.Hkv;
                int n = seq_len_checked(p, b);
                if (n < 0) n = 0;
                const int M = n / p.C;
                if (mt.item == L_META) {
                    const int S = M / p.J;
                    block_topk<kConsumers>(p.super_scores + (size_t)pair * p.S_max, S,
                                           p.topk_super,
                                           p.sel_super + (size_t)pair * p.topk_super,
                                           tsc, csync, NoProbe(), arr(A_ENTRIES + p.topk, pair));
                    if (tid == 0) *arr(A_SCOUNT, pair) = min(p.topk_super, S) + 1;
                } else {
                    int k;
                    if (mt.item == L_GIST) {
                        block_topk<kConsumers>(p.scores + (size_t)pair * p.M_max, M, p.topk,
                                               p.sel_idx + (size_t)pair * p.topk, tsc, csync,
                                               SSA_PROBE(pair), arr(A_ENTRIES, pair));
                        k = min(p.topk, M);
                    } else {
                        const int S = M / p.J, R = M - S * p.J;
                        const int ks = min(p.topk_super, S);
                        const int nc = ks * p.J + R;
                        int* out = p.sel_idx + (size_t)pair * p.topk;
                        block_topk<kConsumers>(p.cand_scores + (size_t)pair * p.Mc_max, nc,
                                               p.topk, out, tsc, csync);
                        csync();
                        // candidate position -> chunk id (increasing map); the
                        // superchunks come from their published copy (entry + 1)
                        const int* sup = arr(A_ENTRIES + p.topk, pair);
                        int* pub = arr(A_ENTRIES, pair);
                        for (int c = tid; c < p.topk; c += kConsumers) {
                            const int pos = out[c];
                            if (pos >= 0) {
                                int m;
                                if (pos < ks * p.J) {
                                    int e = ld_relaxed(sup + pos / p.J);
                                    for (int tries = 0; e == 0 && tries < (1 << 20); ++tries) {
                                        __nanosleep(64);
                                        e = ld_relaxed(sup + pos / p.J);
                                    }
                                    if (e == 0) report_status(kStatusTimeout);
                                    m = (e - 1) * p.J + pos % p.J;
                                } else {
                                    m = S * p.J + (pos - ks * p.J);
                                }
                                out[c] = m;
                                pub[c] = m + 1;
                            }
                        }
                        k = min(p.topk, nc);
                    }
                    if (tid == 0) *arr(A_COUNT, pair) = k + 1;
                }
                csync();  // the shared union area is free again for the next item
            } else {
                // ---- validate a caller-given selection and publish it
                const int b = pair / p.Hkv;
                int n = seq_len_checked(p, b);
                if (n < 0) n = 0;
                const int M = n / p.C;
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
                        ok = (v < M) && (c == 0 || (prev >= 0 && prev < v));
                        atomicAdd(&misc[3], 1);
                    }
                    if (!ok) misc[2] = 0;
                }
                csync();
                const bool good = misc[2] != 0;
                if (good) {
                    int* pub = arr(A_ENTRIES, pair);
                    for (int c = tid; c < misc[3]; c += kConsumers) pub[c] = sl[c] + 1;
                }
                if (tid == 0) {
                    if (!good) report_status(kStatusBadInput);
                    if (!(p.debug_flags & 1))
                        st_release(arr(A_COUNT, pair), good ? misc[3] + 1 : (kBadBit | 1));
                }
                csync();
            }
            if (tid == 0) SSA_TR(TR_C_TOPK1, mt.item, pair);
        } else if (mt.kind == K_COMBINE) {
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);
            if (tid == 0) SSA_TR(TR_C_COMB0, 0, pair);
            const int G = p.G;
            // ---- combination of the pair's partial passes (sec. 3.6)
            const int b = pair / p.Hkv, j = pair % p.Hkv;
            bool bad = false;
            if (p.mode == kModeAttnOnly) {
                if (tid == 0) {
                    wait_geq(arr(A_COUNT, pair), 1, p.wait_limit);
                    misc[4] = (ld_acquire(arr(A_COUNT, pair)) & kBadBit) != 0;
                }
                csync();
                bad = misc[4] != 0;
            }
            const int NP = p.attn_items * kConsumerWarps;  // one partial per item and warp
            const size_t stride = (size_t)G * (D + 2);
            const float* pbase = p.partials + (size_t)pair * NP * stride;
            float* mS = cmb;               // [G][NP] maxima
            float* lS = cmb + G * NP;      // [G][NP] sums
            float* fS = cmb + 2 * G * NP;  // [G][NP] weights
            for (int base = 0; base < G * NP; base += kConsumers * 4) {
                float mv[4], lv[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int idx = base + u * kConsumers + tid;
                    const int h = idx / NP, sp = idx - (idx / NP) * NP;
                    const float* pp = pbase + sp * stride + (size_t)h * (D + 2);
                    mv[u] = idx < G * NP ? __ldcg(pp) : -INFINITY;
                    lv[u] = idx < G * NP ? __ldcg(pp + 1) : 0.f;
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int idx = base + u * kConsumers + tid;
                    if (idx < G * NP) {
                        mS[idx] = mv[u];
                        lS[idx] = lv[u];
                    }
                }
            }
            csync();
            for (int h = warp; h < G; h += kConsumerWarps) {
                float mx = -INFINITY;
                for (int sp = lane; sp < NP; sp += 32) mx = fmaxf(mx, mS[h * NP + sp]);
#pragma unroll
                for (int o = 16; o > 0; o >>= 1)
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
                float Lsum = 0.f;
                for (int sp = lane; sp < NP; sp += 32) {
                    const float ms = mS[h * NP + sp];
                    const float f = (ms == -INFINITY) ? 0.f : exp2f(ms - mx);
                    fS[h * NP + sp] = f;
                    Lsum += f * lS[h * NP + sp];
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) Lsum += __shfl_xor_sync(0xffffffffu, Lsum, o);
                __syncwarp();
                float* op = p.out + ((size_t)b * p.Hq + (size_t)j * G + h) * D;
                const float inv = (!bad && Lsum > 0.f) ? 1.f / Lsum : 0.f;
#pragma unroll
                for (int d0 = 2 * lane; d0 < D; d0 += 64) {
                    float ox = 0.f, oy = 0.f;
                    const float* col = pbase + (size_t)h * (D + 2) + 2 + d0;
#pragma unroll 8
                    for (int sp = 0; sp < NP; ++sp) {
                        const float2 a = __ldcg(reinterpret_cast<const float2*>(col + sp * stride));
                        const float f = fS[h * NP + sp];
                        ox += f * a.x;
                        oy += f * a.y;
                    }
                    *reinterpret_cast<float2*>(op + d0) = make_float2(ox * inv, oy * inv);
                }
            }
            csync();
            {
                // clear this pair's record for the next call
                int* rec = arr(0, pair);
                const int used = A_ENTRIES + p.topk + (p.h2 ? p.topk_super : 0);
                for (int a = tid; a < used; a += kConsumers) rec[a] = 0;
            }
            if (tid == 0) SSA_TR(TR_C_COMB1, 0, pair);
        } else {  // K_ATTN
            if (mt.flags & F_FIRST) {
                mrow[0] = mrow[1] = -INFINITY;
                lrow[0] = lrow[1] = 0.f;
#pragma unroll
                for (int nt = 0; nt < D / 8; ++nt)
#pragma unroll
                    for (int c = 0; c < 4; ++c) acc[nt][c] = 0.f;
            }
            const int rbase = 16 * warp;
            if (rbase < mt.nvalid) {
                float s[2][4];
                qk16<D>(slotA, rbase, qa, s, lane);
                const uint64_t excl = ((uint64_t)mt.rmask_hi << 32) | mt.rmask_lo;
#pragma unroll
                for (int nt = 0; nt < 2; ++nt)
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int lr = rbase + nt * 8 + 2 * tig + (c & 1);
                        const bool out = lr >= mt.nvalid || ((excl >> lr) & 1ull);
                        s[nt][c] = out ? -INFINITY : s[nt][c] * scale_log2;
                    }
                uint32_t phi[4], plo[4];
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    float mx = fmaxf(fmaxf(s[0][2 * r], s[0][2 * r + 1]),
                                     fmaxf(s[1][2 * r], s[1][2 * r + 1]));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                    const float mnew = fmaxf(mrow[r], mx);
                    const float ref = (mnew == -INFINITY) ? 0.f : mnew;
                    const float alpha = exp2f(mrow[r] - ref);
                    const float p00 = exp2f(s[0][2 * r] - ref), p01 = exp2f(s[0][2 * r + 1] - ref);
                    const float p10 = exp2f(s[1][2 * r] - ref), p11 = exp2f(s[1][2 * r + 1] - ref);
                    lrow[r] = lrow[r] * alpha + (p00 + p01 + p10 + p11);
                    mrow[r] = mnew;
#pragma unroll
                    for (int nt = 0; nt < D / 8; ++nt) {
                        acc[nt][2 * r] *= alpha;
                        acc[nt][2 * r + 1] *= alpha;
                    }
                    split_bf16(p00, p01, phi[r], plo[r]);          // tokens 0..7
                    split_bf16(p10, p11, phi[2 + r], plo[2 + r]);  // tokens 8..15
                }
                pv16<D>(slotB, rbase, phi, plo, acc, lane);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[stage]);

            if (mt.flags & F_LAST) {
                if (tid == 0) SSA_TR(TR_C_LAST, K_ATTN, pair);
                // ---- write this warp's partial (m, l, acc) for its heads; the
                // combination merges the warps' partials, so items end without
                // a block-wide barrier
                const int G = p.G;
#pragma unroll
                for (int r = 0; r < 2; ++r) {
                    float l = lrow[r];
                    l += __shfl_xor_sync(0xffffffffu, l, 1);
                    l += __shfl_xor_sync(0xffffffffu, l, 2);
                    const int h = g8 + 8 * r;
                    if (h < G) {
                        float* dstp = p.partials +
                                      ((((size_t)pair * p.attn_items + mt.item) * kConsumerWarps +
                                        warp) * G + h) * (D + 2);
                        if (tig == 0) *reinterpret_cast<float2*>(dstp) = make_float2(mrow[r], l);
#pragma unroll
                        for (int nt = 0; nt < D / 8; ++nt)
                            *reinterpret_cast<float2*>(dstp + 2 + nt * 8 + 2 * tig) =
                                make_float2(acc[nt][2 * r], acc[nt][2 * r + 1]);
                    }
                }
                __syncwarp();
                if (lane == 0) red_release_add(arr(A_ATTN, pair), 1);
                if (tid == 0) SSA_TR(TR_C_DONE, K_ATTN, pair);
            }
        }
        if (++stage == NS) {
            stage = 0;
            ++round;
        }
    }
    // ---- last block out resets the ticket for the next launch
    csync();
    if (tid == 0) {
        SSA_TR(TR_KEND, 0, 0);
        SSA_TR(TR_KEND | 0x80, 0, 0);
    }
    if (p.mode != kModeScoreOnly && tid == 0) {
        __threadfence();
        const int old = atomicAdd(ctrl + C_EXIT, 1);
        if (old == (int)gridDim.x - 1) {
            ctrl[C_TICKET] = 0;
            ctrl[C_EXIT] = 0;
            __threadfence();
        }
    }
}

}  // namespace fused
}  // namespace ssa
