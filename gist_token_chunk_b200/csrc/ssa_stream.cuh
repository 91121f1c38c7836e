// ssa_stream.cuh -- the streaming decode kernel: single level, bf16, d = 64,
// GQA groups of at most 8 query heads, topk <= 128, at most 2048 chunks per
// sequence.
//
// "Simplified Sparse Attention via Gist Tokens": sec. 3.2 (each chunk is
// scored from its gist tokens only), sec. 3.3 (top-k chunks, then one
// attention pass over the unfolded context: gist K/V of the unselected
// chunks, raw K/V of the selected chunks, the raw tail), sec. 3.6 (split
// partial attention and a combination of the partials).
//
// Work.  A call is laid out as two lists, each the concatenation over the
// (sequence, KV head) pairs of that pair's elements:
//   CHUNKS  the pair's complete chunks
//   TILES   32-token tiles of raw K/V: the selected chunks' tiles (in chunk
//           order), then the tail's
// Every warp of a block but the last is a worker with its own ring of
// shared-memory stages, which it fills itself (lane 0 issues 2-D TMA copies,
// no multicast) and consumes in order.  Each worker takes an equal
// contiguous share of both lists and runs, in this order:
//   1. scoring: the gist keys of its chunks, 64 rows per stage (Q.K^T on the
//      tensor cores with the keys as the M operand); every head's logit of
//      its gist rows stays in shared memory, and at the end of a (worker,
//      pair) segment the chunk scores go to the workspace;
//   2. gist values: the values of the same gist rows, 64 per stage, attended
//      with the kept logits once the pair's selection is published (rows of
//      selected chunks masked); the copies are issued before it exists;
//   3. raw tiles: 32 K rows + 32 V rows per stage, addressed through the
//      published selection, attended (Q.K^T and P.V on the tensor cores).
// Each (list, pair) segment of a worker ends with one partial (m, l, o) per
// query head in the workspace.  The last warp of each block is the control
// warp: it computes the top-k of the pairs the block owns as soon as their
// chunk scores are complete, publishes it and writes sel_idx, then combines
// the partials of its (pair, query head) tasks into the output.
//
// Everything one warp hands to another (chunk scores, published selections,
// partials) carries the launch's epoch in its own 32-bit word, so a reader
// knows what this launch wrote without counters or clearing; the epoch moves
// on when the last block of a launch finishes.  A worker waits for a
// selection only after every one of its own chunks is scored, and a control
// warp publishes all selections it owns before it waits for partials, so
// every wait ends (the launch is cooperative: all blocks are resident); each
// wait is also bounded.
#pragma once

#include <type_traits>

#include "ssa_device.cuh"
#include "ssa_internal.h"

namespace ssa {
namespace stream {

constexpr int kD = 64;
constexpr int kWorkers = 6;                    // worker warps per block
constexpr int kThreads = (kWorkers + 1) * 32;  // + the control warp
constexpr int kStages = 3;                     // ring stages per worker
constexpr int kSlotBytes = 8192;               // 64 gist rows, or 32 raw K + 32 raw V rows
constexpr int kGistRows = 64;
constexpr int kRawRows = 32;
constexpr int kMaxG = 8;
constexpr int kMaxChunks = 2048;               // chunks per sequence (M_max): 64 key columns
constexpr int kMaxTopk = 64;                   // the running top list holds 64
constexpr int kMaxBlocks = 160;                // sizes the partial slots
constexpr int kSelCand = 256;                  // top-k candidates ranked exactly
constexpr int kRecBytes = 272;                 // one partial: epoch, pad, m, l, o[64] (fp32)

// A pair's chunk keys are stored transposed: with n = ceil(M / 32), chunk c
// (lane c / n, column c % n) sits at word (c % n) * 32 + c / n, so the warp
// that ranks them reads each lane's chunks as one contiguous run without
// bank conflicts.  Row stride: 32 * ceil(M_max / 32) words.
__host__ __device__ inline int score_stride(int M_max) { return (M_max + 31) / 32 * 32; }
__host__ __device__ inline int score_pos(int c, int n) { return (c % n) * 32 + c / n; }
__host__ __device__ inline int sel_stride(int topk) { return (topk + 31) / 32 * 32 + 32; }
__host__ __device__ inline int kcap_for(int topk) { return topk < 32 ? 32 : (topk + 31) / 32 * 32; }

enum : int { K_SCORE = 0, K_GISTV = 1, K_RAW = 2, K_DONE = 3 };
enum : int { F_FIRST = 1, F_LAST = 2, F_Q = 4 };

// One ring stage, written by the worker when it issues the copies.
struct Desc {
    int kind, pair, nvalid, flags;
    int lrow;  // gist stages: logits row (worker-local) of the stage's first row
    int c0;    // gist stages: first chunk of the segment (index in the pair)
    int nch;   // gist stages: chunks of the segment
    int off;   // gist stages: row offset of the stage in the segment
};

struct Layout {
    int ring, qs, bars, desc, lg, rmax, bits, selc, cand, sbuf, cbar, plan, misc, total;
    int qbytes, lstride, bwords, kcap;
};

// Shared memory of one block (the same on host and device).  Per worker: its
// ring, the query slots of its stages, barriers and descriptors, the kept
// logits [G][lstride] and row maxima of its gist rows, the selection bitmap
// of its current gist segment and a two-entry cache of published selections.
__host__ __device__ inline Layout layout(const Plan& p) {
    Layout L;
    int o = 0;
    // every area starts on a 16-byte boundary (bulk copies, vector access)
    auto take = [&](int bytes) {
        const int at = o;
        o += (bytes + 15) / 16 * 16;
        return at;
    };
    L.ring = take(kWorkers * kStages * kSlotBytes);
    L.qbytes = (p.G * kD * 2 + 127) / 128 * 128;
    L.qs = take(kWorkers * kStages * L.qbytes);
    L.bars = take(kWorkers * kStages * 8);
    L.desc = take(kWorkers * kStages * (int)sizeof(Desc));
    // + 72 rows: a 16-row block may read up to 63 rows past the last kept
    // row (masked), and a stride of 8 mod 32 words spreads the banks
    L.lstride = p.st_rcap + 72;
    L.lg = take(kWorkers * p.G * L.lstride * 4);
    L.rmax = take(kWorkers * p.st_rcap * 4);
    L.bwords = p.st_rcap / 32 + 2;
    L.bits = take(kWorkers * L.bwords * 4);
    L.kcap = kcap_for(p.topk);
    L.selc = take(kWorkers * 2 * L.kcap * 4);
    L.cand = take(kSelCand * 8);                    // the control warp's top-k candidates
    L.sbuf = take(score_stride(p.M_max) * 8);       // its copy of one pair's chunk scores
    L.cbar = take(16);
    L.plan = take((p.B + 2 * (p.B + 1)) * 4);
    L.misc = take(64);
    L.total = o + 1024;  // slack to align the ring to 1024 bytes
    return L;
}

// ------------------------------------------------------------- small ops ---

__device__ __forceinline__ unsigned ld_relaxed_u32(const unsigned* p) {
    unsigned v;
    asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_relaxed_u32(unsigned* p, unsigned v) {
    asm volatile("st.relaxed.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void st_relaxed_u64(unsigned long long* p, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}
// Orders this thread's earlier shared-memory reads (generic proxy) before its
// later bulk copies into the same memory (async proxy).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ unsigned long long tagged(unsigned tag, unsigned v) {
    return ((unsigned long long)tag << 32) | v;
}

// Byte offset of 16-byte unit `c` of row `r` in a TMA box with 128-byte
// rows and the 128-byte swizzle (the box starts on a 1024-byte boundary).
__device__ __forceinline__ uint32_t swz(int r, int c) {
    return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
}

// ------------------------------------------------------------------ plan ---

// Elements of list L (0: chunks, 1: raw tiles) of one pair of raw length n.
__device__ __forceinline__ int list_count(const Plan& p, int L, int n) {
    const int M = n / p.C;
    if (L == 0) return M;
    const int T = n - M * p.C;
    const int tpc = (p.C + kRawRows - 1) / kRawRows;
    return min(p.topk, M) * tpc + (T + kRawRows - 1) / kRawRows;
}

// The plan every block computes from seq_lens: lengths and per-list prefix
// sums over sequences (Hkv pairs of equal counts per sequence).
struct View {
    const Plan& p;
    const int* nb;   // [B] raw lengths (0: invalid)
    const int* ps0;  // [B + 1] chunk-list prefix
    const int* ps1;  // [B + 1] tile-list prefix
    int W;           // workers of the launch

    __device__ const int* ps(int L) const { return L ? ps1 : ps0; }
    __device__ int total(int L) const { return ps(L)[p.B]; }
    __device__ int parts(int L) const { return min(W, total(L)); }
    // share of worker w in list L: [lo, hi)
    __device__ void share(int L, int w, int& lo, int& hi) const {
        const long long t = total(L), n = parts(L);
        if (w >= n) {
            lo = hi = 0;
            return;
        }
        lo = (int)((t * w) / n);
        hi = (int)((t * (w + 1)) / n);
    }
    // worker holding element x of list L
    __device__ int worker_of(int L, int x) const {
        const long long t = total(L), n = parts(L);
        return (int)(((long long)(x + 1) * n - 1) / t);
    }
    // pair holding element x of list L, the list index of its element 0, and
    // its element count
    __device__ void locate(int L, int x, int& pair, int& first, int& count) const {
        const int* q = ps(L);
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
    // workers holding the segments of `pair` in list L: [w0, w1]; false if
    // the pair has no element there
    __device__ bool pair_workers(int L, int pair, int& w0, int& w1) const {
        const int b = pair / p.Hkv, j = pair - b * p.Hkv;
        const int count = list_count(p, L, nb[b]);
        if (count == 0) return false;
        const int first = ps(L)[b] + j * count;
        w0 = worker_of(L, first);
        w1 = worker_of(L, first + count - 1);
        return true;
    }
};

// Partial of query head h for worker w's segment of `pair` in list L: 272
// bytes (epoch word, pad, m, l, o[64]).  Along a list the segments' (worker
// + pair) strictly increase, so slots differ, and the segments of one pair
// are consecutive slots: [list][head][slot].
__device__ __forceinline__ char* part_rec(const Plan& p, int L, int h, int w, int pair) {
    const size_t s = ((size_t)L * p.G + h) * p.st_part_slots + w + pair;
    return p.st_part + s * (size_t)kRecBytes;
}

// ------------------------------------------------- stage generator (issue) ---

// The worker's stage sequence: scoring stages of its chunk share, gist-value
// stages of the same share, raw-tile stages of its tile share.  Every lane
// runs it identically.
struct Gen {
    int phase = K_SCORE;
    int x = 0, hi = 0;                  // position in the phase's list, end of the share
    int pair = 0, first = 0, i0 = 0, i1 = 0;
    int off = 0;                        // gist: row offset in the segment; raw: tile offset
    int lbase = 0;                      // gist: logits row of the segment start
    bool in_seg = false;

    // Moves to the next segment when needed; false once the worker is done.
    __device__ bool ready(const View& v, int w) {
        while (!in_seg) {
            if (phase == K_DONE) return false;
            if (x >= hi) {
                ++phase;
                if (phase == K_DONE) return false;
                v.share(phase == K_RAW ? 1 : 0, w, x, hi);
                lbase = 0;
                continue;
            }
            const int Ls = phase == K_RAW ? 1 : 0;
            int cnt;
            v.locate(Ls, x, pair, first, cnt);
            i0 = x - first;
            i1 = min(hi, first + cnt) - first;
            off = 0;
            in_seg = true;
        }
        return true;
    }
};

// Timeline trace: builds compiled with SSA_TRACE record per warp (clock64,
// global timer, event | a << 8, b) into Plan::trace; the product build
// compiles these to nothing.
#ifdef SSA_TRACE
// events 1 (warp start) and 29 (warp end) also carry the global timer (ns)
#define ST_TR(ev, a, b)                                                                       \
    do {                                                                                      \
        if (p.trace && lane == 0 && tr_n < p.trace_cap) {                                      \
            const unsigned long long c_ = clock64();                                           \
            const uint32_t g_ = ((ev) == 1 || (ev) == 29) ? (uint32_t)now_ns() : 0u;           \
            p.trace[((size_t)blockIdx.x * 8 + warp) * p.trace_cap + tr_n] =                    \
                make_uint4((uint32_t)c_, g_, (uint32_t)(ev) | ((uint32_t)(a) << 8), (uint32_t)(b)); \
        }                                                                                     \
        ++tr_n;                                                                               \
    } while (0)
#else
#define ST_TR(ev, a, b) ((void)0)
#endif

// --------------------------------------------------------------- kernel ---


// Running top list of E = 32 KW composites (KW = 1 or 2; entry i of the list
// in register i / 32 of lane i % 32), descending; 0 marks an empty entry.
// Merges a descending 32-entry batch bt into it (the top E of the union:
// the element-wise maximum of the list and the reversed batch is bitonic,
// and one bitonic merge sorts it).
template <int KW>
__device__ __forceinline__ void run_merge(unsigned long long (&run)[2], unsigned long long bt,
                                          int lane) {
    const unsigned long long br = __shfl_sync(0xffffffffu, bt, 31 - lane);
    if (KW == 1) {
        run[0] = warp_merge_desc(run[0], bt, lane);
        return;
    }
    run[1] = cmax_u64(run[1], br);
    const unsigned long long hi = cmax_u64(run[0], run[1]), lo = cmin_u64(run[0], run[1]);
    run[0] = hi;
    run[1] = lo;
#pragma unroll
    for (int j = 16; j > 0; j >>= 1)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
            const unsigned long long o = __shfl_xor_sync(0xffffffffu, run[r], j);
            run[r] = (lane & j) == 0 ? cmax_u64(run[r], o) : cmin_u64(run[r], o);
        }
}

// Ascending bitonic sort of 32 KW ints (entry i in register i / 32 of lane
// i % 32).
template <int KW>
__device__ __forceinline__ void sort_asc(int (&v)[2], int lane) {
#pragma unroll
    for (int kk = 2; kk <= 32 * KW; kk <<= 1)
#pragma unroll
        for (int jj = kk >> 1; jj > 0; jj >>= 1) {
            if (jj == 32) {
                const int a = min(v[0], v[1]), b = max(v[0], v[1]);
                v[0] = a;
                v[1] = b;
                continue;
            }
#pragma unroll
            for (int r = 0; r < KW; ++r) {
                const int i = 32 * r + lane;
                const int o = __shfl_xor_sync(0xffffffffu, v[r], jj);
                const bool keep_min = ((i & jj) == 0) == ((i & kk) == 0);
                v[r] = keep_min ? min(v[r], o) : max(v[r], o);
            }
        }
}

// Top-k of one pair's chunks by one warp (sec. 3.3: the k chunks with the
// largest scores, ties to the lower chunk), 0 < k < M.  sc holds the pair's
// tagged order-preserving keys (score_key) in the transposed layout of
// score_pos with n = ceil(M / 32) columns: lane l ranks chunks l n .. l n +
// n - 1 (word j * 32 + l holds chunk l n + j; 0 past M).  Calls emit(pos,
// chunk) for the k selected chunks, pos 0..k-1 in ascending chunk order.
// `cand` is shared scratch of kSelCand entries.
//
// tau0 > 0 is a lower bound on the k-th largest key given by the caller;
// otherwise one comes from the per-lane r-th largest keys v_l (r = 2, or 4
// for k > 64): the q = ceil(k / r) lanes with the largest v_l hold at least
// q r >= k keys >= their v_l, so the k-th largest key is >= the q-th largest
// v_l.  The keys >= tau (few for any spread of scores) go to `cand` as
// composites key << 32 | ~chunk in chunk order and are ranked exactly by
// counting larger composites.  If tau leaves too many (many equal scores), an
// MSB-first bisection on the key bits over all keys finds the k-th largest
// key instead.
// (branch-free: the load is always in bounds; j is clamped to the columns)
__device__ __forceinline__ uint32_t lane_key(const unsigned long long* sc, int n, int M, int lane,
                                             int j) {
    const uint32_t v = (uint32_t)sc[min(j, n - 1) * 32 + lane];
    return (j < n && lane * n + j < M) ? v : 0u;
}

__device__ __forceinline__ int warp_excl_scan(int v, int lane, int& total) {
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    total = __shfl_sync(0xffffffffu, x, 31);
    return x - v;
}

#ifdef SSA_TRACE
#define SEL_PH(i) (ph ? (void)(ph[i] = clock64()) : (void)0)
#else
#define SEL_PH(i) ((void)0)
#endif
template <class Emit>
__device__ __forceinline__ void warp_select(const unsigned long long* sc, int n, int M, int k,
                                         int lane, unsigned long long* cand, uint32_t tau0,
                                         Emit emit, long long* ph = nullptr) {
    (void)ph;
    SEL_PH(0);
    uint32_t tau = tau0;
    if (tau == 0u) {
    const int r = k > 64 ? 4 : 2;
    // per-lane r largest keys; four keys per step in flight
    uint32_t t0 = 0u, t1 = 0u, t2 = 0u, t3 = 0u;
    for (int j0 = 0; j0 < n; j0 += 4) {
        uint32_t x[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) x[u] = lane_key(sc, n, M, lane, j0 + u);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            uint32_t xx = x[u], y;
            y = max(t0, xx); xx = min(t0, xx); t0 = y;
            y = max(t1, xx); xx = min(t1, xx); t1 = y;
            y = max(t2, xx); xx = min(t2, xx); t2 = y;
            t3 = max(t3, xx);
        }
    }
    uint32_t vl = r > 2 ? t3 : t1;
    // the q-th largest v_l: bitonic sort of the lanes' values, descending
    for (int kk = 2; kk <= 32; kk <<= 1)
        for (int jj = kk >> 1; jj > 0; jj >>= 1) {
            const uint32_t o = __shfl_xor_sync(0xffffffffu, vl, jj);
            const bool keep_max = ((lane & jj) == 0) == ((lane & kk) == 0);
            vl = keep_max ? max(vl, o) : min(vl, o);
        }
    tau = __shfl_sync(0xffffffffu, vl, (k + r - 1) / r - 1);
    }
    SEL_PH(1);
    int nc = 0;
    if (tau > 0u) {
        // this lane's candidates (a bit per column), then their place in
        // chunk order by a scan of the per-lane counts (branch-free loops
        // with warp-uniform bounds)
        unsigned long long bits = 0ull;
        for (int j = 0; j < n; ++j)
            bits |= (unsigned long long)(lane_key(sc, n, M, lane, j) >= tau) << j;
        const int mine = __popcll(bits);
        int at = warp_excl_scan(mine, lane, nc);
        if (nc <= kSelCand) {
            for (int j = 0; j < n; ++j) {
                const bool c = (bits >> j) & 1ull;
                const unsigned long long comp =
                    ((unsigned long long)lane_key(sc, n, M, lane, j) << 32) |
                    (uint32_t)~(uint32_t)(lane * n + j);
                if (c) cand[at] = comp;
                at += c;
            }
        }
        __syncwarp();
    }
    SEL_PH(2);
    if (tau > 0u && nc <= kSelCand) {
        const unsigned lt = (1u << lane) - 1u;
        // rank = number of larger composites (all distinct), every candidate
        // of this lane in one pass
        auto rank_emit = [&](auto per_tag) {
            constexpr int kPer = decltype(per_tag)::value;
            unsigned long long x[kPer];
            int rank[kPer];
#pragma unroll
            for (int u = 0; u < kPer; ++u) {
                const unsigned long long y = cand[lane + 32 * u];
                x[u] = lane + 32 * u < nc ? y : ~0ull;
                rank[u] = 0;
            }
            int m = 0;
            for (; m + 4 <= nc; m += 4) {
                const unsigned long long y0 = cand[m], y1 = cand[m + 1], y2 = cand[m + 2],
                                         y3 = cand[m + 3];
#pragma unroll
                for (int u = 0; u < kPer; ++u)
                    rank[u] += (y0 > x[u]) + (y1 > x[u]) + (y2 > x[u]) + (y3 > x[u]);
            }
            for (; m < nc; ++m) {
                const unsigned long long y = cand[m];
#pragma unroll
                for (int u = 0; u < kPer; ++u) rank[u] += y > x[u];
            }
            int ob = 0;
#pragma unroll
            for (int u = 0; u < kPer; ++u) {
                const bool take = lane + 32 * u < nc && rank[u] < k;
                const unsigned b = __ballot_sync(0xffffffffu, take);
                if (take) emit(ob + __popc(b & lt), (int)~(uint32_t)x[u]);
                ob += __popc(b);
            }
        };
        if (nc <= 64) rank_emit(std::integral_constant<int, 2>());
        else rank_emit(std::integral_constant<int, kSelCand / 32>());
        __syncwarp();
        SEL_PH(3);
        if (ph) ph[4] = nc;
        return;
    }
    // fallback: T = the k-th largest key; if some prefix already separates
    // exactly k keys, those are the selection and no tie needs breaking
    auto count_ge = [&](uint32_t x) {
        int c = 0;
        for (int j = 0; j < n; ++j) c += lane_key(sc, n, M, lane, j) >= x;
        return __reduce_add_sync(0xffffffffu, c);
    };
    uint32_t prefix = 0u;
    bool exact = false;
    for (int bit = 31; bit >= 0; --bit) {
        const uint32_t cnd = prefix | (1u << bit);
        const int c = count_ge(cnd);
        if (c >= k) {
            prefix = cnd;
            if (c == k) {
                exact = true;
                break;
            }
        }
    }
    // keys above T all, then keys equal to T in chunk order until k: each
    // lane's equal keys and selected keys are placed by scans of its counts
    const int need_eq = exact ? 0 : k - count_ge(prefix + 1u);
    int neq = 0;
    if (!exact)
        for (int j = 0; j < n; ++j) neq += lane * n + j < M && lane_key(sc, n, M, lane, j) == prefix;
    int tot;
    int eq_before = warp_excl_scan(neq, lane, tot);
    int nsel = 0;
    for (int j = 0, e = eq_before; j < n; ++j) {
        if (lane * n + j >= M) break;
        const uint32_t key = lane_key(sc, n, M, lane, j);
        const bool eq = !exact && key == prefix;
        nsel += (exact ? key >= prefix : key > prefix) || (eq && e < need_eq);
        e += eq;
    }
    int pos = warp_excl_scan(nsel, lane, tot);
    for (int j = 0, e = eq_before; j < n; ++j) {
        if (lane * n + j >= M) break;
        const uint32_t key = lane_key(sc, n, M, lane, j);
        const bool eq = !exact && key == prefix;
        if ((exact ? key >= prefix : key > prefix) || (eq && e < need_eq)) emit(pos++, lane * n + j);
        e += eq;
    }
    __syncwarp();
}

// --------------------------------------------------------------- kernel ---

__global__ void __launch_bounds__(kThreads, 1)
    stream_kernel(const __grid_constant__ Plan p, const __grid_constant__ CUtensorMap tm_kg,
                  const __grid_constant__ CUtensorMap tm_vg,
                  const __grid_constant__ CUtensorMap tm_kr,
                  const __grid_constant__ CUtensorMap tm_vr) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const Layout L = layout(p);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g8 = lane >> 2, tig = lane & 3;
    int* nb = reinterpret_cast<int*>(smem + L.plan);
    int* ps0 = nb + p.B;
    int* ps1 = ps0 + p.B + 1;
    unsigned* misc = reinterpret_cast<unsigned*>(smem + L.misc);
    const int G = p.G;

    // ---- prologue: the launch's epoch and the plan (the same in every block)
    if (threadIdx.x == 0) {
        prefetch_tensormap(&tm_kg);
        prefetch_tensormap(&tm_vg);
        prefetch_tensormap(&tm_kr);
        prefetch_tensormap(&tm_vr);
        unsigned e = ld_relaxed_u32(p.st_hdr) + 1u;
        misc[0] = e == 0u ? 1u : e;
    }
    for (int b = threadIdx.x; b < p.B; b += blockDim.x) {
        const int n = __ldg(p.seq_lens + b);
        const bool ok = n >= 1 && n <= p.n_max;
        if (!ok && blockIdx.x == 0) report_status(kStatusBadInput);
        nb[b] = ok ? n : 0;
    }
    __syncthreads();
    if (warp < 2) {  // warp L: exclusive prefix over sequences of list L
        int* out = warp ? ps1 : ps0;
        int carry = 0;
        for (int b0 = 0; b0 < p.B; b0 += 32) {
            const int b = b0 + lane;
            const int v = b < p.B ? p.Hkv * list_count(p, warp, nb[b]) : 0;
            int x = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            if (b < p.B) out[b] = carry + x - v;
            carry += __shfl_sync(0xffffffffu, x, 31);
        }
        if (lane == 0) out[p.B] = carry;
    }
    __syncthreads();
    const unsigned tag = misc[0];
    const View v{p, nb, ps0, ps1, (int)gridDim.x * kWorkers};
#ifdef SSA_TRACE
    int tr_n = 0;
#endif
    ST_TR(1, 0, 0);
    const long long lim = wait_cycles(p.wait_limit);
    const float scale = 0.125f;                        // 1/sqrt(64)
    const float scale_log2 = 0.125f * 1.4426950408889634f;
    const int tpc = (p.C + kRawRows - 1) / kRawRows;

    if (warp < kWorkers) {
        // ============================================================ worker
        const int w = blockIdx.x * kWorkers + warp;
        uint8_t* ring = smem + L.ring + warp * kStages * kSlotBytes;
        uint8_t* qs = smem + L.qs + warp * kStages * L.qbytes;
        uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars) + warp * kStages;
        Desc* desc = reinterpret_cast<Desc*>(smem + L.desc) + warp * kStages;
        float* lg = reinterpret_cast<float*>(smem + L.lg) + warp * G * L.lstride;
        float* rmax = reinterpret_cast<float*>(smem + L.rmax) + warp * p.st_rcap;
        uint32_t* bits = reinterpret_cast<uint32_t*>(smem + L.bits) + warp * L.bwords;
        int* selc = reinterpret_cast<int*>(smem + L.selc) + warp * 2 * L.kcap;
        if (lane == 0) {
            for (int s = 0; s < kStages; ++s) mbar_init(&full[s], 1);
            fence_barrier_init();
        }
        __syncwarp();
        const uint64_t pol = l2_policy_evict_first();
        const uint32_t ring_s = smem_u32(ring);

        // two-entry cache of published selections (entries in chunk order)
        int cpair[2] = {-1, -1}, ccount[2] = {0, 0};
        int pin = -1;  // pair whose raw tiles are being issued (kept cached)
        // Fetches the published selection of `pair` into a cache entry not
        // holding `keep`.  One round of loads per attempt; with `blocking`
        // polls until complete (bounded; on running out the entry holds no
        // chunk and a timeout is recorded).  Returns the entry or -1.
        auto fetch_sel = [&](int pair, int keep, bool blocking) -> int {
            if (cpair[0] == pair) return 0;
            if (cpair[1] == pair) return 1;
            const int e = (cpair[0] == keep && keep >= 0) ? 1 : 0;
            int* dst = selc + e * L.kcap;
            const int n = nb[pair / p.Hkv];
            const int k = min(p.topk, n / p.C);
            const unsigned long long* src = p.st_sel + (size_t)pair * p.st_sel_stride;
            const long long c0 = clock64();
            ST_TR(13, pair, blocking);
            for (;;) {
                bool ok = true;
                for (int i = lane; i < k; i += 32) {
                    const unsigned long long x = ld_relaxed_u64(src + i);
                    ok = ok && (unsigned)(x >> 32) == tag;
                    dst[i] = (int)(unsigned)x;
                }
                if (__all_sync(0xffffffffu, ok)) {
                    __syncwarp();
                    cpair[e] = pair;
                    ccount[e] = k;
                    ST_TR(14, pair, 1);
                    return e;
                }
                if (!blocking) {
                    ST_TR(14, pair, 0);
                    return -1;
                }
                if (clock64() - c0 > lim) {
                    if (lane == 0) report_status(kStatusTimeout);
                    __syncwarp();
                    cpair[e] = pair;
                    ccount[e] = 0;
                    return e;
                }
                __nanosleep(128);
            }
        };

        Gen gen;
        v.share(0, w, gen.x, gen.hi);
        int ni = 0, nc = 0;
        bool more = true, dead = false;

        // consumer state
        uint32_t qf[4][2];
        float acc[4][4];
        float m_run = -INFINITY, l_run = 0.f;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) qf[kk][0] = qf[kk][1] = 0u;
#pragma unroll
        for (int mt = 0; mt < 4; ++mt)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[mt][c] = 0.f;

        // Online-softmax update of head g8 with the logits x (log2 domain,
        // excluded = -inf): x becomes the probabilities, acc is rescaled.
        auto softmax_update = [&](auto& x) {
            constexpr int R = sizeof(x) / sizeof(x[0]);
            constexpr int Cn = sizeof(x[0]) / sizeof(float);
            float mx = -INFINITY;
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int c = 0; c < Cn; ++c) mx = fmaxf(mx, x[r][c]);
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            const float mnew = fmaxf(m_run, mx);
            const float ref = mnew == -INFINITY ? 0.f : mnew;
            float alpha = exp2f(m_run - ref);
            float ls = 0.f;
#pragma unroll
            for (int r = 0; r < R; ++r)
#pragma unroll
                for (int c = 0; c < Cn; ++c) {
                    x[r][c] = exp2f(x[r][c] - ref);
                    ls += x[r][c];
                }
            l_run = l_run * alpha + ls;
            m_run = mnew;
            if (g8 >= G) alpha = 1.f;
            if (__any_sync(0xffffffffu, alpha != 1.f)) {
                const float a0 = __shfl_sync(0xffffffffu, alpha, (2 * tig) << 2);
                const float a1 = __shfl_sync(0xffffffffu, alpha, (2 * tig + 1) << 2);
#pragma unroll
                for (int mt = 0; mt < 4; ++mt) {
                    acc[mt][0] *= a0;
                    acc[mt][2] *= a0;
                    acc[mt][1] *= a1;
                    acc[mt][3] *= a1;
                }
            }
        };
        // acc (dims as M, heads as N) += V^T (16 rows at r0 of a value box) . P^T
        auto pv16 = [&](uint32_t vbox, int r0, float p00, float p01, float p10, float p11) {
            uint32_t hi0, lo0, hi1, lo1;
            split_bf16(p00, p01, hi0, lo0);  // tokens 2 tig, 2 tig + 1
            split_bf16(p10, p11, hi1, lo1);  // tokens 2 tig + 8, 2 tig + 9
            const int row = r0 + (lane & 7) + ((lane >> 4) << 3);
            const int csel = (lane >> 3) & 1;
#pragma unroll
            for (int mt = 0; mt < 4; ++mt) {
                uint32_t a[4];
                ldsm_x4_trans(vbox + swz(row, 2 * mt + csel), a[0], a[1], a[2], a[3]);
                mma_bf16_16816(acc[mt], a, hi0, hi1);
                mma_bf16_16816(acc[mt], a, lo0, lo1);
            }
        };
        auto reset_state = [&]() {
            m_run = -INFINITY;
            l_run = 0.f;
#pragma unroll
            for (int mt = 0; mt < 4; ++mt)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[mt][c] = 0.f;
        };
        // One partial per query head of the segment (list Lp, pair); each
        // record's epoch word is written after its data.
        auto write_partial = [&](int Lp, int pair) {
            float l = l_run;
            l += __shfl_xor_sync(0xffffffffu, l, 1);
            l += __shfl_xor_sync(0xffffffffu, l, 2);
            if (tig == 0 && g8 < G)
                *reinterpret_cast<float2*>(part_rec(p, Lp, g8, w, pair) + 8) = make_float2(m_run, l);
            const int h0 = 2 * tig, h1 = 2 * tig + 1;
            float* o0 = reinterpret_cast<float*>(part_rec(p, Lp, h0 < G ? h0 : 0, w, pair) + 16);
            float* o1 = reinterpret_cast<float*>(part_rec(p, Lp, h1 < G ? h1 : 0, w, pair) + 16);
#pragma unroll
            for (int mt = 0; mt < 4; ++mt) {
                if (h0 < G) {
                    o0[16 * mt + g8] = acc[mt][0];
                    o0[16 * mt + g8 + 8] = acc[mt][2];
                }
                if (h1 < G) {
                    o1[16 * mt + g8] = acc[mt][1];
                    o1[16 * mt + g8 + 8] = acc[mt][3];
                }
            }
            __syncwarp();
            if (lane < G) {
                __threadfence();
                st_relaxed_u32(reinterpret_cast<unsigned*>(part_rec(p, Lp, lane, w, pair)), tag);
            }
        };

        for (;;) {
            // ---- issue ahead, up to kStages stages in flight
            while (more && !dead && ni < nc + kStages) {
                if (!gen.ready(v, w)) {
                    more = false;
                    break;
                }
                int y = 0;
                Desc d;
                d.kind = gen.phase;
                d.pair = gen.pair;
                if (gen.phase != K_RAW) {
                    const int rows_seg = (gen.i1 - gen.i0) * p.g;
                    const int nv = min(kGistRows, rows_seg - gen.off);
                    d.nvalid = nv;
                    d.flags = (gen.off == 0 ? (F_FIRST | (gen.phase == K_SCORE ? F_Q : 0)) : 0) |
                              (gen.off + kGistRows >= rows_seg ? F_LAST : 0);
                    d.lrow = gen.lbase + gen.off;
                    d.c0 = gen.i0;
                    d.nch = gen.i1 - gen.i0;
                    d.off = gen.off;
                    y = (gen.pair * p.M_max + gen.i0) * p.g + gen.off;
                    gen.off += kGistRows;
                    if (gen.off >= rows_seg) {
                        gen.in_seg = false;
                        gen.lbase += (rows_seg + 1) & ~1;  // keep segment rows even-aligned
                        gen.x = gen.first + gen.i1;
                    }
                } else {
                    const int pr = gen.pair;
                    const int n = nb[pr / p.Hkv];
                    const int M = n / p.C;
                    const int kc = min(p.topk, M);
                    const int u = gen.i0 + gen.off;
                    int r0, nv;
                    if (u < kc * tpc) {
                        // the selected chunk's tiles need the published selection
                        const int e = fetch_sel(pr, pin, ni == nc);
                        if (e < 0) break;  // not yet: consume what is in flight
                        pin = pr;
                        const int c = u / tpc, part = u - c * tpc;
                        if (c < ccount[e]) {
                            const int chunk = min(max(selc[e * L.kcap + c], 0), max(M - 1, 0));
                            r0 = chunk * p.C + part * kRawRows;
                            nv = min(kRawRows, p.C - part * kRawRows);
                        } else {
                            r0 = 0;
                            nv = 0;
                        }
                    } else {
                        const int t = u - kc * tpc;
                        r0 = M * p.C + t * kRawRows;
                        nv = min(kRawRows, n - r0);
                    }
                    d.nvalid = nv;
                    d.flags = (gen.off == 0 ? (F_FIRST | F_Q) : 0) | (u + 1 >= gen.i1 ? F_LAST : 0);
                    d.lrow = d.c0 = d.nch = d.off = 0;
                    y = pr * p.n_max + r0;
                    ++gen.off;
                    if (gen.i0 + gen.off >= gen.i1) {
                        gen.in_seg = false;
                        gen.x = gen.first + gen.i1;
                        pin = -1;
                    }
                }
                const int s = ni % kStages;
                ST_TR(12, d.kind, d.flags);
                __syncwarp();
                if (lane == 0) {
                    desc[s] = d;
                    fence_proxy_async_smem();
                    const bool wq = (d.flags & F_Q) != 0;
                    mbar_arrive_expect_tx(&full[s], (uint32_t)(kSlotBytes + (wq ? G * kD * 2 : 0)));
                    if (wq) {
                        const int b = d.pair / p.Hkv, j = d.pair - b * p.Hkv;
                        const __nv_bfloat16* src = static_cast<const __nv_bfloat16*>(p.q) +
                                                   ((size_t)b * p.Hq + (size_t)j * G) * kD;
                        bulk_load(qs + s * L.qbytes, src, (uint32_t)(G * kD * 2), &full[s]);
                    }
                    uint8_t* dst = ring + s * kSlotBytes;
                    if (d.kind == K_RAW) {
                        tma_load_2d_hint(dst, &tm_kr, 0, y, &full[s], pol);
                        tma_load_2d_hint(dst + kSlotBytes / 2, &tm_vr, 0, y, &full[s], pol);
                    } else {
                        tma_load_2d_hint(dst, d.kind == K_SCORE ? &tm_kg : &tm_vg, 0, y, &full[s],
                                         pol);
                    }
                }
                __syncwarp();
                ++ni;
            }
            if (nc == ni) {
                if (!more || dead) break;
                continue;  // the next stage waited for a selection: try again
            }

            // ---- consume the oldest stage
            const int s = nc % kStages;
            if (!mbar_wait(&full[s], (uint32_t)((nc / kStages) & 1), 8 * p.wait_limit)) {
                // a copy never landed: issue nothing more; later stages are
                // waited for (bounded) below
                dead = true;
                ++nc;
                continue;
            }
            const Desc d = desc[s];
            ST_TR(10, d.kind, d.flags);
            const uint32_t box = ring_s + s * kSlotBytes;
            const int nv = d.nvalid;
            if (d.flags & F_Q) {
                const uint8_t* qsm = qs + s * L.qbytes;
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    qf[kk][0] = g8 < G ? *reinterpret_cast<const uint32_t*>(
                                             qsm + (g8 * kD + 16 * kk + 2 * tig) * 2)
                                       : 0u;
                    qf[kk][1] = g8 < G ? *reinterpret_cast<const uint32_t*>(
                                             qsm + (g8 * kD + 16 * kk + 8 + 2 * tig) * 2)
                                       : 0u;
                }
            }
            if (d.kind == K_SCORE) {
                // ---- scoring: keys as the M rows, heads as N; the four 16-row
                // blocks are independent (rows past nvalid are computed from
                // whatever the slot holds and never stored)
                float st[4][4];
#pragma unroll
                for (int blk = 0; blk < 4; ++blk) {
                    st[blk][0] = st[blk][1] = st[blk][2] = st[blk][3] = 0.f;
                }
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
#pragma unroll
                    for (int blk = 0; blk < 4; ++blk) {
                        const int row = 16 * blk + (lane & 7) + (((lane >> 3) & 1) << 3);
                        uint32_t a[4];
                        ldsm_x4(box + swz(row, 2 * kk + (lane >> 4)), a[0], a[1], a[2], a[3]);
                        mma_bf16_16816(st[blk], a, qf[kk][0], qf[kk][1]);
                    }
                const int h0 = 2 * tig, h1 = h0 + 1;
                float* lg0 = lg + (h0 < G ? h0 : 0) * L.lstride + d.lrow;
                float* lg1 = lg + (h1 < G ? h1 : 0) * L.lstride + d.lrow;
#pragma unroll
                for (int blk = 0; blk < 4; ++blk) {
                    const int ra = 16 * blk + g8, rb = ra + 8;
                    if (h0 < G) {
                        if (ra < nv) lg0[ra] = st[blk][0] * scale_log2;
                        if (rb < nv) lg0[rb] = st[blk][2] * scale_log2;
                    }
                    if (h1 < G) {
                        if (ra < nv) lg1[ra] = st[blk][1] * scale_log2;
                        if (rb < nv) lg1[rb] = st[blk][3] * scale_log2;
                    }
                }
                float va[4], vb[4];
#pragma unroll
                for (int blk = 0; blk < 4; ++blk) {
                    va[blk] = h0 < G ? st[blk][0] : -INFINITY;
                    vb[blk] = h0 < G ? st[blk][2] : -INFINITY;
                    if (h1 < G) {
                        va[blk] = fmaxf(va[blk], st[blk][1]);
                        vb[blk] = fmaxf(vb[blk], st[blk][3]);
                    }
                }
#pragma unroll
                for (int o = 1; o <= 2; o <<= 1)
#pragma unroll
                    for (int blk = 0; blk < 4; ++blk) {
                        va[blk] = fmaxf(va[blk], __shfl_xor_sync(0xffffffffu, va[blk], o));
                        vb[blk] = fmaxf(vb[blk], __shfl_xor_sync(0xffffffffu, vb[blk], o));
                    }
                if (tig == 0) {
#pragma unroll
                    for (int blk = 0; blk < 4; ++blk) {
                        const int ra = 16 * blk + g8, rb = ra + 8;
                        if (ra < nv) rmax[d.lrow + ra] = va[blk] * scale;
                        if (rb < nv) rmax[d.lrow + rb] = vb[blk] * scale;
                    }
                }
                {
                    // the chunks whose last gist row this stage scored: their
                    // keys (max over the chunk's rows) go out now, so the
                    // selection can fold them in while scoring goes on
                    const int cb = p.g_shift >= 0 ? d.off >> p.g_shift : d.off / p.g;
                    const int ce = (d.flags & F_LAST) ? d.nch
                                   : (p.g_shift >= 0 ? (d.off + nv) >> p.g_shift : (d.off + nv) / p.g);
                    if (ce > cb) {
                        __syncwarp();
                        const int seg = d.lrow - d.off;
                        unsigned long long* dst =
                            p.st_scores + (size_t)d.pair * score_stride(p.M_max);
                        const int ncol = (nb[d.pair / p.Hkv] / p.C + 31) >> 5;
                        for (int c = cb + lane; c < ce; c += 32) {
                            const float* r = rmax + seg + c * p.g;
                            float m = r[0];
                            for (int t = 1; t < p.g; ++t) m = fmaxf(m, r[t]);
                            st_relaxed_u64(dst + score_pos(d.c0 + c, ncol), tagged(tag, score_key(m)));
                        }
                    }
                    if (d.flags & F_LAST) {
                        // the segment's second-largest chunk key (0 if it has
                        // one chunk): a bound the selection starts from
                        const int seg = d.lrow - d.off;
                        uint32_t t0 = 0u, t1 = 0u;
                        for (int c = lane; c < d.nch; c += 32) {
                            const float* r = rmax + seg + c * p.g;
                            float m = r[0];
                            for (int t = 1; t < p.g; ++t) m = fmaxf(m, r[t]);
                            const uint32_t x = score_key(m);
                            t1 = max(t1, min(t0, x));
                            t0 = max(t0, x);
                        }
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) {
                            const uint32_t u0 = __shfl_xor_sync(0xffffffffu, t0, o);
                            const uint32_t u1 = __shfl_xor_sync(0xffffffffu, t1, o);
                            t1 = max(max(t1, u1), min(t0, u0));
                            t0 = max(t0, u0);
                        }
                        if (lane == 0) st_relaxed_u64(p.st_sum + w + d.pair, tagged(tag, t1));
                    }
                }
            } else if (d.kind == K_GISTV) {
                // ---- gist values, masked by the pair's published selection
                if (d.flags & F_FIRST) {
                    reset_state();
                    const int e = fetch_sel(d.pair, pin, true);
                    const int words = (d.nch + 31) >> 5;
                    for (int i = lane; i < words; i += 32) bits[i] = 0u;
                    __syncwarp();
                    const int* ent = selc + e * L.kcap;
                    for (int i = lane; i < ccount[e]; i += 32) {
                        const int c = ent[i] - d.c0;
                        if (c >= 0 && c < d.nch) atomicOr(&bits[c >> 5], 1u << (c & 31));
                    }
                    __syncwarp();
                }
                // excluded rows of the stage: past the valid rows, or in a
                // selected chunk
                uint32_t ex[2];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int r = lane + 32 * hh;
                    const int sr = d.off + r;
                    const int c = min(p.g_shift >= 0 ? (sr >> p.g_shift) : sr / p.g, d.nch - 1);
                    const bool e = (r >= nv) | (((bits[c >> 5] >> (c & 31)) & 1u) != 0u);
                    ex[hh] = __ballot_sync(0xffffffffu, e);
                }
                float x[4][4];
                const float* lrow_p = lg + (g8 < G ? g8 : 0) * L.lstride + d.lrow + 2 * tig;
                // (branch-free: the kept-logit area is padded past the last
                // row, so every load is in bounds; exclusions are selects)
                const uint32_t hm = g8 < G ? 0u : 0xffffffffu;  // heads past G: all excluded
#pragma unroll
                for (int blk = 0; blk < 4; ++blk) {
                    const int r0 = 16 * blk;
                    const uint32_t eb = ((ex[blk >> 1] >> (16 * (blk & 1))) & 0xffffu) | hm;
                    const float2 a = *reinterpret_cast<const float2*>(lrow_p + r0);
                    const float2 b = *reinterpret_cast<const float2*>(lrow_p + r0 + 8);
                    x[blk][0] = ((eb >> (2 * tig)) & 1u) ? -INFINITY : a.x;
                    x[blk][1] = ((eb >> (2 * tig + 1)) & 1u) ? -INFINITY : a.y;
                    x[blk][2] = ((eb >> (2 * tig + 8)) & 1u) ? -INFINITY : b.x;
                    x[blk][3] = ((eb >> (2 * tig + 9)) & 1u) ? -INFINITY : b.y;
                }
                softmax_update(x);
#pragma unroll
                for (int blk = 0; blk < 4; ++blk) {
                    const uint32_t eb = (ex[blk >> 1] >> (16 * (blk & 1))) & 0xffffu;
                    if (16 * blk < nv && eb != 0xffffu)
                        pv16(box, 16 * blk, x[blk][0], x[blk][1], x[blk][2], x[blk][3]);
                }
                if (d.flags & F_LAST) {
                    write_partial(0, d.pair);
                    reset_state();
                }
            } else {
                // ---- raw tile: S = Q.K^T (heads as M), softmax, P.V
                if (d.flags & F_FIRST) reset_state();
                float s4[4][4];
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    s4[nt][0] = s4[nt][1] = s4[nt][2] = s4[nt][3] = 0.f;
#pragma unroll
                    for (int kq = 0; kq < 2; ++kq) {
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4(box + swz(8 * nt + (lane & 7), 4 * kq + (lane >> 3)), b0, b1, b2, b3);
                        const uint32_t a0[4] = {qf[2 * kq][0], 0u, qf[2 * kq][1], 0u};
                        const uint32_t a1[4] = {qf[2 * kq + 1][0], 0u, qf[2 * kq + 1][1], 0u};
                        mma_bf16_16816(s4[nt], a0, b0, b1);
                        mma_bf16_16816(s4[nt], a1, b2, b3);
                    }
                }
                float x[4][2];
#pragma unroll
                for (int nt = 0; nt < 4; ++nt) {
                    const int t0 = 8 * nt + 2 * tig;
                    x[nt][0] = (g8 < G && t0 < nv) ? s4[nt][0] * scale_log2 : -INFINITY;
                    x[nt][1] = (g8 < G && t0 + 1 < nv) ? s4[nt][1] * scale_log2 : -INFINITY;
                }
                softmax_update(x);
                const uint32_t vbox = box + kSlotBytes / 2;
#pragma unroll
                for (int ks = 0; ks < 2; ++ks)
                    if (16 * ks < nv)
                        pv16(vbox, 16 * ks, x[2 * ks][0], x[2 * ks][1], x[2 * ks + 1][0],
                             x[2 * ks + 1][1]);
                if (d.flags & F_LAST) {
                    write_partial(1, d.pair);
                    reset_state();
                }
            }
            __syncwarp();
            ST_TR(11, d.kind, d.flags);
            ++nc;
        }
        ST_TR(19, 0, 0);
        ST_TR(29, 0, 0);
        if (dead) {
            // every issued copy lands before the block exits (bounded)
            if (lane == 0)
                for (int i = max(0, ni - kStages); i < ni; ++i)
                    mbar_wait(&full[i % kStages], (uint32_t)((i / kStages) & 1), p.wait_limit);
            __syncwarp();
        }
    } else {
        // ====================================================== control warp
        const int N = gridDim.x, P = p.n_pairs;
        unsigned long long* cand = reinterpret_cast<unsigned long long*>(smem + L.cand);
        unsigned long long* sbuf = reinterpret_cast<unsigned long long*>(smem + L.sbuf);
        uint64_t* cbar = reinterpret_cast<uint64_t*>(smem + L.cbar);
        if (lane == 0) {
            mbar_init(cbar, 1);
            fence_barrier_init();
        }
        __syncwarp();
        uint32_t cpar = 0;
        const int sstride = score_stride(p.M_max);
        // ---- selections of the pairs this block owns: pair q is owned by
        // block floor(q * N / P)
        const int own_lo = (int)(((long long)blockIdx.x * P + N - 1) / N);
        const int own_hi = (int)(((long long)(blockIdx.x + 1) * P + N - 1) / N);
        for (int pr = own_lo; pr < own_hi; ++pr) {
            const int M = nb[pr / p.Hkv] / p.C;
            const int k = min(p.topk, M);
            unsigned long long* pub = p.st_sel + (size_t)pr * p.st_sel_stride;
            int32_t* user = p.sel_idx + (size_t)pr * p.topk;
            const bool publish = !(p.debug_flags & 1);
            ST_TR(20, pr, k);
            if (k == M) {
                // every complete chunk is selected (or none exists)
                for (int i = lane; i < p.topk; i += 32) {
                    user[i] = i < k ? i : -1;
                    if (i < k && publish) st_relaxed_u64(pub + i, tagged(tag, (unsigned)i));
                }
                continue;
            }
            // poll: one bulk copy of the pair's tagged chunk scores into
            // shared memory per round, until every word carries this launch's
            // epoch (bounded)
            const unsigned long long* src = p.st_scores + (size_t)pr * sstride;
            const int ncol = (M + 31) >> 5;
            const uint32_t bytes = (uint32_t)(ncol * 32 * 8);
            // the pair's scoring segments publish their second-largest keys:
            // lanes hold segments s and s + 32
            int w0, w1;
            v.pair_workers(0, pr, w0, w1);
            const int nseg = w1 - w0 + 1;
            const bool use_sum = nseg <= 64 && (k + 1) / 2 <= nseg;
            const unsigned long long* sums = p.st_sum + w0 + pr;
            uint32_t s2[2] = {0u, 0u};
            const long long c0 = clock64();
            for (;;) {
                __syncwarp();
                if (lane == 0) {
                    fence_proxy_async_smem();
                    mbar_arrive_expect_tx(cbar, bytes);
                    bulk_load(sbuf, src, bytes, cbar);
                }
                bool ok = true;
                if (use_sum) {
#pragma unroll
                    for (int r = 0; r < 2; ++r) {
                        const int sg = lane + 32 * r;
                        if (sg < nseg) {
                            const unsigned long long x = ld_relaxed_u64(sums + sg);
                            ok = ok && (unsigned)(x >> 32) == tag;
                            s2[r] = (uint32_t)x;
                        }
                    }
                }
                mbar_wait(cbar, cpar, p.wait_limit);
                cpar ^= 1u;
                for (int j = 0; j < ncol; ++j)
                    ok = ok && (lane * ncol + j >= M || (unsigned)(sbuf[j * 32 + lane] >> 32) == tag);
                ST_TR(23, pr, ok ? 1 : 0);
                if (__all_sync(0xffffffffu, ok)) break;
                if (clock64() - c0 > lim) {
                    if (lane == 0) report_status(kStatusTimeout);
                    break;
                }
                __nanosleep(100);
            }
            ST_TR(21, pr, 0);
            // tau: the ceil(k / 2)-th largest of the segments' second keys
            // (each of those segments holds two keys at least as large), or
            // 0 to let the top-k find its own bound
            uint32_t tau = 0u;
            if (use_sum) {
                if (nseg <= 32) {
                    uint32_t x = s2[0];
                    for (int kk = 2; kk <= 32; kk <<= 1)
                        for (int jj = kk >> 1; jj > 0; jj >>= 1) {
                            const uint32_t o = __shfl_xor_sync(0xffffffffu, x, jj);
                            const bool keep_max = ((lane & jj) == 0) == ((lane & kk) == 0);
                            x = keep_max ? max(x, o) : min(x, o);
                        }
                    tau = __shfl_sync(0xffffffffu, x, (k + 1) / 2 - 1);
                } else {
                    // the q-th largest of up to 64 values by counting
                    const int q = (k + 1) / 2;
                    uint32_t best = 0u;
                    for (int r = 0; r < 2; ++r) {
                        int above = 0, ties = 0;
                        for (int m = 0; m < 64; ++m) {
                            const uint32_t y = __shfl_sync(0xffffffffu, s2[m >> 5], m & 31);
                            above += y > s2[r];
                            ties += (y == s2[r]) && (m < 32 * r + lane);
                        }
                        if (above + ties == q - 1 && lane + 32 * r < 64) best = s2[r];
                    }
                    tau = __reduce_max_sync(0xffffffffu, best);
                }
            }
            long long ph[5] = {0, 0, 0, 0, 0};
            warp_select(sbuf, ncol, M, k, lane, cand, tau, [&](int pos, int c) {
                user[pos] = c;
                if (publish) st_relaxed_u64(pub + pos, tagged(tag, (unsigned)c));
            }, ph);
            ST_TR(24, pr, (unsigned)(ph[1] - ph[0]));
            ST_TR(25, pr, (unsigned)(ph[2] - ph[1]));
            ST_TR(26, pr, (unsigned)(ph[3] - ph[2]));
            ST_TR(27, (int)ph[4], 0);
            for (int i = k + lane; i < p.topk; i += 32) user[i] = -1;
            ST_TR(22, pr, 0);
        }

        // ---- combinations: task t = pair * G + head, t = block (mod N).
        // The partials of one (list, head, pair) are consecutive records; a
        // batch of up to 32 is waited for, then read with every load in
        // flight at once: lane l takes columns 4 (l & 15) .. + 3 of the
        // records 2 i + (l >> 4).
        for (int t = blockIdx.x; t < P * G; t += N) {
            const int pr = t / G, h = t - pr * G;
            const int b = pr / p.Hkv, j = pr - b * p.Hkv;
            float Mr = -INFINITY, Lr = 0.f;
            float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
            ST_TR(30, t, 0);
            for (int Lp = 0; Lp < 2; ++Lp) {
                int w0, w1;
                if (!v.pair_workers(Lp, pr, w0, w1)) continue;
                for (int base = w0; base <= w1; base += 32) {
                    const int cnt = min(32, w1 - base + 1);
                    const char* recs = part_rec(p, Lp, h, base, pr);
                    const char* mine = recs + (size_t)min(lane, cnt - 1) * kRecBytes;
                    const long long c0 = clock64();
                    for (;;) {
                        const bool ok =
                            lane >= cnt || ld_relaxed_u32(reinterpret_cast<const unsigned*>(mine)) == tag;
                        if (__all_sync(0xffffffffu, ok)) break;
                        if (clock64() - c0 > lim) {
                            if (lane == 0) report_status(kStatusTimeout);
                            break;
                        }
                        __nanosleep(128);
                    }
                    fence_acquire_gpu();
                    ST_TR(31, Lp, cnt);
                    float mi = -INFINITY, li = 0.f;
                    if (lane < cnt) {
                        const float2 ml = __ldcg(reinterpret_cast<const float2*>(mine + 8));
                        mi = ml.x;
                        li = ml.y;
                    }
                    float4 vals[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int rr = 2 * i + (lane >> 4);
                        vals[i] = rr < cnt ? __ldcg(reinterpret_cast<const float4*>(
                                                 recs + (size_t)rr * kRecBytes + 16) +
                                             (lane & 15))
                                           : make_float4(0.f, 0.f, 0.f, 0.f);
                    }
                    float mb = mi;
                    for (int off = 16; off > 0; off >>= 1)
                        mb = fmaxf(mb, __shfl_xor_sync(0xffffffffu, mb, off));
                    const float mn = fmaxf(Mr, mb);
                    const float ref = mn == -INFINITY ? 0.f : mn;
                    const float fo = exp2f(Mr - ref);
                    const float fi = exp2f(mi - ref);
                    float ls = li * fi;
                    for (int off = 16; off > 0; off >>= 1) ls += __shfl_xor_sync(0xffffffffu, ls, off);
                    // o is summed per half-warp; fo applies to both halves
                    Lr = Lr * fo + ls;
                    o.x *= fo;
                    o.y *= fo;
                    o.z *= fo;
                    o.w *= fo;
                    Mr = mn;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const float f = __shfl_sync(0xffffffffu, fi, 2 * i + (lane >> 4));
                        o.x += f * vals[i].x;
                        o.y += f * vals[i].y;
                        o.z += f * vals[i].z;
                        o.w += f * vals[i].w;
                    }
                }
            }
            // the two half-warps hold disjoint records of the same columns
            o.x += __shfl_xor_sync(0xffffffffu, o.x, 16);
            o.y += __shfl_xor_sync(0xffffffffu, o.y, 16);
            o.z += __shfl_xor_sync(0xffffffffu, o.z, 16);
            o.w += __shfl_xor_sync(0xffffffffu, o.w, 16);
            const float inv = Lr > 0.f ? 1.f / Lr : 0.f;
            if (lane < 16) {
                float4* dst = reinterpret_cast<float4*>(
                    p.out + (((size_t)b * p.Hq + (size_t)j * G + h) * kD));
                dst[lane] = make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
            }
            ST_TR(32, t, 0);
        }
        ST_TR(29, 0, 0);
    }

    // ---- the last block to finish moves the workspace's epoch on
    __syncthreads();
    if (threadIdx.x == 0) {
        __threadfence();
        const unsigned old = atomicInc(p.st_hdr + 1, gridDim.x - 1);
        if (old == gridDim.x - 1) {
            st_relaxed_u32(p.st_hdr, tag);
            __threadfence();
        }
    }
}

}  // namespace stream
}  // namespace ssa
