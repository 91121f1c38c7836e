// ssa_pipe.cuh -- the two-kernel decode pipeline: single level, bf16,
// d = 64, GQA groups of at most 8 query heads, at most 8192 chunks per
// sequence.
//
// "Simplified Sparse Attention via Gist Tokens": sec. 3.2 (each chunk is
// scored from its gist tokens only), sec. 3.3 (top-k chunks, then one
// attention pass over the unfolded context: gist K/V of the unselected
// chunks, raw K/V of the selected chunks, the raw tail), sec. 3.6 (split
// partial attention and a combination of the partials).
//
// One decode step is two kernels on one stream, the second launched with
// programmatic dependent launch so that it starts as the first drains:
//   score_kernel   every complete chunk's gist keys, 64 rows per stage: the
//                  per-head logits of each gist row (log2 domain) go to the
//                  workspace, and so does each chunk's score (the maximum over
//                  its gist rows and the group's heads of q.k / sqrt(d));
//   attend_kernel  the top-k of each (sequence, KV head) pair, run by the first
//                  four warps of the block that owns the pair (a deterministic
//                  top-k over the pair's chunk scores, or, for the App. A
//                  reading, one per query head over its own scores and their
//                  union; published to the workspace and written to sel_idx);
//                  then
//                  the unfolded context: the gist values of every chunk,
//                  weighted by the kept logits and masked by the selection
//                  (the selected chunks', or for the sec. 3.3 reading the
//                  unselected ones),
//                  and the raw K/V tiles of the selected chunks and of the
//                  tail; one partial (m, l, o) per query head and (list, pair)
//                  segment of a worker, combined into the output by the
//                  blocks' control warps.
// Every attention worker copies its first gist-value stages (values and kept
// logits) before the top-k runs, so those loads overlap it; what needs the
// selection (the mask, the raw tile addresses) polls the published,
// epoch-tagged entries (bounded).
//
// Both streaming kernels run one block per SM whose worker warps are
// independent: each fills its own ring of shared-memory stages with 2-D TMA
// copies (lane 0 issues, no multicast) and consumes them in order.  The work
// of a call is laid out as two lists, each the concatenation over pairs of
// that pair's elements: CHUNKS (complete chunks) and TILES (32-token raw
// tiles: the selected chunks', in chunk order, then the tail's); every
// worker takes an equal contiguous share of a list.
#pragma once

#include "ssa_device.cuh"
#include "ssa_internal.h"

namespace ssa {
namespace pipe {

constexpr int kD = 64;
constexpr int kSlotBytes = 8192;   // 64 gist rows, or 32 raw K + 32 raw V rows
constexpr int kGistRows = 64;
constexpr int kRawRows = 32;
constexpr int kMaxG = 8;           // query heads per KV head
constexpr int kMaxBlocks = 160;    // sizes the partial slots
constexpr int kRecBytes = 272;     // one partial: epoch, pad, m, l, o[64] (fp32)
// Published selection row (64-bit entries) of a pair: topk rounded up to 32, + 32.
__host__ __device__ inline int sel_stride(int topk) { return (topk + 31) / 32 * 32 + 32; }

enum : int { K_SCORE = 0, K_GISTV = 1, K_RAW = 2 };
enum : int { F_FIRST = 1, F_LAST = 2, F_Q = 4 };

// One ring stage, written by the worker when it issues the copies.
struct Desc {
    int kind, pair, nvalid, flags;
    int lrow;  // gist stages: logits row of the stage's first row
    int c0;    // gist stages: first chunk of the segment (index in the pair)
    int nch;   // gist stages: chunks of the segment
    int off;   // gist stages: row offset of the stage in the segment
};

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
// Whether a bounded wait that started at c0 has run out, decided once for
// the whole warp (lane 0's clock): every lane leaves a polling loop on the
// same round, so the warp-wide votes inside it stay converged.
__device__ __forceinline__ bool warp_expired(long long c0, long long lim) {
    return __shfl_sync(0xffffffffu, (int)(clock64() - c0 > lim), 0) != 0;
}
// A 64-bit word that carries the launch's epoch in its upper half.
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
    // selected chunks: k, or at most G k under the per-head union (unused
    // slots become empty tiles)
    return min(p.sel_stride, M) * tpc + (T + kRawRows - 1) / kRawRows;
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

// Timeline trace: builds compiled with SSA_TRACE record per warp (clock64,
// global timer, event | a << 8, b) into Plan::trace, laid out [block][16
// warps][trace_cap] (warps past 16 record nothing); the product build
// compiles these to nothing.
#ifdef SSA_TRACE
// events 1 (warp start) and 29 (warp end) also carry the global timer (ns)
#define ST_TR(ev, a, b)                                                                       \
    do {                                                                                      \
        if (p.trace && lane == 0 && tr_n < p.trace_cap && warp < 16) {                         \
            const unsigned long long c_ = clock64();                                           \
            const uint32_t g_ = ((ev) == 1 || (ev) == 29) ? (uint32_t)now_ns() : 0u;           \
            p.trace[((size_t)blockIdx.x * 16 + warp) * p.trace_cap + tr_n] =                   \
                make_uint4((uint32_t)c_, g_, (uint32_t)(ev) | ((uint32_t)(a) << 8), (uint32_t)(b)); \
        }                                                                                     \
        ++tr_n;                                                                               \
    } while (0)
#else
#define ST_TR(ev, a, b) ((void)0)
#endif

// -------------------------------------------------------------- pipeline ---

// Build-time shape of the two kernels: ring stages per worker warp and the
// thread bound each is compiled for (registers per thread follow from it),
// the most attention workers a block runs, whether P enters P.V as bf16 hi +
// lo parts (about 16 significant bits) or as bf16 alone, and whether the
// scoring kernel prefetches the gist values of the rows it scores into L2.
#ifndef SSA_SCORE_STAGES
#define SSA_SCORE_STAGES 3
#endif
#ifndef SSA_SCORE_THREADS
#define SSA_SCORE_THREADS 256
#endif
#ifndef SSA_ATTN_STAGES
#define SSA_ATTN_STAGES 2
#endif
#ifndef SSA_ATTN_THREADS
#define SSA_ATTN_THREADS 384
#endif
#ifndef SSA_ATTN_WORKERS
#define SSA_ATTN_WORKERS 11
#endif
#ifndef SSA_PIPE_PV_LO
#define SSA_PIPE_PV_LO 1
#endif
#ifndef SSA_PREFETCH_GISTV
#define SSA_PREFETCH_GISTV 0
#endif
constexpr int kScoreStages = SSA_SCORE_STAGES;  // ring stages per scoring worker
constexpr int kScoreThreads = SSA_SCORE_THREADS;
constexpr int kAttnStages = SSA_ATTN_STAGES;    // ring stages per attention worker
constexpr int kAttnThreads = SSA_ATTN_THREADS;
constexpr int kAttnWorkers = SSA_ATTN_WORKERS < SSA_ATTN_THREADS / 32 - 1 ? SSA_ATTN_WORKERS
                                                                           : SSA_ATTN_THREADS / 32 - 1;
constexpr int kMaxWorkers = kScoreThreads / 32;  // scoring worker warps per block

// Kept-logit row stride (floats): G rounded up to 4, so every row is a
// 16-byte unit and a stage's rows are one bulk copy.
__host__ __device__ inline int logit_stride(int G) { return (G + 3) & ~3; }
// Chunk-score row stride (floats) of a pair: M_max rounded up to 8, so each
// thread of the top-k reads its 8 chunks as two aligned 16-byte loads.
__host__ __device__ inline int score_row(int M_max) { return (M_max + 7) & ~7; }

// L2 prefetch of `bytes` (a multiple of 16) from a 16-byte aligned address.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes, uint64_t pol) {
    asm volatile("cp.async.bulk.prefetch.L2.global.L2::cache_hint [%0], %1, %2;"
                 ::"l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "l"(pol) : "memory");
}

__device__ __forceinline__ void launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void wait_prerequisites() {
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Lengths and per-list prefix sums over sequences, in shared memory (list 0;
// list 1 too when ps1 is given); invalid lengths count as 0 and are
// reported once.
__device__ __forceinline__ void build_plan(const Plan& p, int* nb, int* ps0, int* ps1, bool report) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    for (int b = threadIdx.x; b < p.B; b += blockDim.x) {
        const int n = __ldg(p.seq_lens + b);
        const bool ok = n >= 1 && n <= p.n_max;
        if (!ok && report) report_status(kStatusBadInput);
        nb[b] = ok ? n : 0;
    }
    __syncthreads();
    if (warp < (ps1 ? 2 : 1)) {
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
}

// A worker's place in one list: its share [x, hi) and the current segment.
struct Cursor {
    int x = 0, hi = 0;
    int pair = 0, first = 0, i0 = 0, i1 = 0, off = 0;
    bool in_seg = false;
    __device__ bool next_seg(const View& v, int L) {
        if (in_seg) return true;
        if (x >= hi) return false;
        int cnt;
        v.locate(L, x, pair, first, cnt);
        i0 = x - first;
        i1 = min(hi, first + cnt) - first;
        off = 0;
        in_seg = true;
        return true;
    }
    __device__ void end_seg() {
        in_seg = false;
        x = first + i1;
    }
};

// ---------------------------------------------------------------- layouts ---

struct ScoreLayout {
    int ring, qs, bars, desc, rmax, plan, total, qbytes;
};
__host__ __device__ inline ScoreLayout score_layout(const Plan& p, int workers) {
    ScoreLayout L;
    int o = 0;
    auto take = [&](int bytes) {
        const int at = o;
        o += (bytes + 15) / 16 * 16;
        return at;
    };
    L.ring = take(workers * kScoreStages * kSlotBytes);
    L.qbytes = (p.G * kD * 2 + 127) / 128 * 128;
    L.qs = take(workers * kScoreStages * L.qbytes);
    L.bars = take(workers * kScoreStages * 8);
    L.desc = take(workers * kScoreStages * (int)sizeof(Desc));
    L.rmax = take(workers * p.st_rcap * 4);
    L.plan = take((p.B + (p.B + 1)) * 4);
    L.total = o + 1024;
    return L;
}

struct AttnLayout {
    int ring, lgs, qs, bars, desc, bits, sel, tk, selout, ubits, plan, misc, total;
    int lgbytes, qbytes, bwords, kcap;
};
__host__ __device__ inline AttnLayout attn_layout(const Plan& p, int workers) {
    AttnLayout L;
    int o = 0;
    auto take = [&](int bytes) {
        const int at = o;
        o += (bytes + 15) / 16 * 16;
        return at;
    };
    L.ring = take(workers * kAttnStages * kSlotBytes);
    L.lgbytes = kGistRows * logit_stride(p.G) * 4;
    L.lgs = take(workers * kAttnStages * L.lgbytes);
    L.qbytes = (p.G * kD * 2 + 127) / 128 * 128;
    L.qs = take(workers * kAttnStages * L.qbytes);
    L.bars = take(workers * kAttnStages * 8);
    L.desc = take(workers * kAttnStages * (int)sizeof(Desc));
    L.bwords = (p.M_max + 31) / 32;
    L.bits = take(workers * L.bwords * 4);
    L.kcap = p.sel_stride > 0 ? p.sel_stride : 1;  // entries of a published selection
    L.sel = take(workers * 2 * L.kcap * 4);
    L.tk = take((int)sizeof(TopkScratch));
    L.selout = take(L.kcap * 4);
    L.ubits = take(p.sel_mode ? L.bwords * 4 : 0);  // per-head union: chunk bitmap
    L.plan = take((p.B + 2 * (p.B + 1)) * 4);
    L.misc = take(64);
    L.total = o + 1024;
    return L;
}

// ------------------------------------------------------------ score kernel ---

// Scoring on the CUDA cores (builds with SSA_SCORE_CUDA_CORES=1; the
// default build scores on the tensor cores).  Eight lanes share a gist row,
// each holding 8 of its 64 dims (one 16-byte load from the swizzled box) and
// the same 8 dims of every head's query in fp32; four rows per pass, 16
// passes per 64-row stage.  The 8 lanes' partial dot products are reduced
// and spread by a butterfly of warp shuffles, so lane c of the row ends with
// head c's logit; the row maximum over heads takes three more shuffles.
#ifndef SSA_SCORE_CUDA_CORES
#define SSA_SCORE_CUDA_CORES 0
#endif

__device__ __forceinline__ uint4 lds_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}
__device__ __forceinline__ float bf_lo(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf_hi(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }

// One 64-row stage: writes the kept logits of rows < nv (heads < G, log2
// domain) and their row maxima (q.k / sqrt(d)).  NG: 4 or 8 (G <= NG).
template <int NG>
__device__ __forceinline__ void score_stage_cuda_cores(const Plan& p, uint32_t box, const float (&qv)[8][8],
                                                       int nv, int G, int GP, float* lgrow,
                                                       float* rmax_seg, float scale, float scale_log2) {
    const int lane = threadIdx.x & 31, rq = lane >> 3, c = lane & 7;
#pragma unroll 2
    for (int t = 0; t < 16; ++t) {
        const int r = 4 * t + rq;
        const uint4 kw = lds_v4(box + swz(r, c));
        float k[8];
        k[0] = bf_lo(kw.x); k[1] = bf_hi(kw.x); k[2] = bf_lo(kw.y); k[3] = bf_hi(kw.y);
        k[4] = bf_lo(kw.z); k[5] = bf_hi(kw.z); k[6] = bf_lo(kw.w); k[7] = bf_hi(kw.w);
        float acc[NG];
#pragma unroll
        for (int h = 0; h < NG; ++h) {
            float a = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) a = fmaf(k[i], qv[h][i], a);
            acc[h] = a;
        }
        // butterfly reduce-scatter over the row's 8 lanes: lane c keeps head c
        // (NG = 8) or head c & 3 (NG = 4) with the sum over all 64 dims
        float x;
        if constexpr (NG == 8) {
            float v4[4], v2[2];
            const bool b4 = c & 4, b2 = c & 2, b1 = c & 1;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float keep = b4 ? acc[i + 4] : acc[i], send = b4 ? acc[i] : acc[i + 4];
                v4[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
            }
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const float keep = b2 ? v4[i + 2] : v4[i], send = b2 ? v4[i] : v4[i + 2];
                v2[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
            }
            const float keep = b1 ? v2[1] : v2[0], send = b1 ? v2[0] : v2[1];
            x = keep + __shfl_xor_sync(0xffffffffu, send, 1);
        } else {
            float v2[2];
            const bool b2 = c & 2, b1 = c & 1;
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const float keep = b2 ? acc[i + 2] : acc[i], send = b2 ? acc[i] : acc[i + 2];
                v2[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
            }
            const float keep = b1 ? v2[1] : v2[0], send = b1 ? v2[0] : v2[1];
            x = keep + __shfl_xor_sync(0xffffffffu, send, 1);
            x += __shfl_xor_sync(0xffffffffu, x, 4);
        }
        const int h = NG == 8 ? c : (c & 3);
        const bool valid = h < G && (NG == 8 || c < 4);
        if (valid && r < nv) lgrow[(size_t)r * GP + h] = x * scale_log2;
        float m = valid ? x : -INFINITY;
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
        if (c == 0 && r < nv) rmax_seg[r] = m * scale;
    }
}


// Grid: one block per SM, workers = blockDim.x / 32.  Each worker scores its
// share of the CHUNKS list: per 64-row stage of gist keys, S^T = K.Q^T on the
// tensor cores (keys as the M rows, the group's heads as N); each row's
// per-head logits q.k / sqrt(d) * log2(e) go to the workspace's kept logits,
// and the chunks whose last row the stage holds get their score (the
// maximum over their rows and heads of q.k / sqrt(d)).
__global__ void __launch_bounds__(kScoreThreads, 1)
    score_kernel(const __grid_constant__ Plan p, const __grid_constant__ CUtensorMap tm_kg) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int workers = blockDim.x >> 5;
    const ScoreLayout L = score_layout(p, workers);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g8 = lane >> 2, tig = lane & 3;
    const int G = p.G;
    int* nb = reinterpret_cast<int*>(smem + L.plan);
    int* ps0 = nb + p.B;
    // the selection kernel may start now (it waits for this grid to finish)
    launch_dependents();
    if (threadIdx.x == 0) prefetch_tensormap(&tm_kg);
    build_plan(p, nb, ps0, nullptr, blockIdx.x == 0);
    const View v{p, nb, ps0, ps0, (int)gridDim.x * workers};
    const int w = blockIdx.x * workers + warp;
#ifdef SSA_TRACE
    int tr_n = 0;
#endif
    ST_TR(1, 0, 0);
    const float scale = 0.125f;  // 1/sqrt(64)
    const float scale_log2 = 0.125f * 1.4426950408889634f;
    const int GP = logit_stride(G);

    uint8_t* ring = smem + L.ring + warp * kScoreStages * kSlotBytes;
    uint8_t* qs = smem + L.qs + warp * kScoreStages * L.qbytes;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars) + warp * kScoreStages;
    Desc* desc = reinterpret_cast<Desc*>(smem + L.desc) + warp * kScoreStages;
    float* rmax = reinterpret_cast<float*>(smem + L.rmax) + warp * p.st_rcap;
    if (lane == 0) {
        for (int s = 0; s < kScoreStages; ++s) mbar_init(&full[s], 1);
        fence_barrier_init();
    }
    __syncwarp();
    const uint64_t pol = l2_policy_evict_first();
    const uint64_t pol_keep = l2_policy_evict_last();
    const uint32_t ring_s = smem_u32(ring);

    Cursor cur;
    v.share(0, w, cur.x, cur.hi);
    int lbase = 0, ni = 0, nc = 0;
    bool more = true, dead = false;
#if SSA_SCORE_CUDA_CORES
    float qv[8][8];
#pragma unroll
    for (int h = 0; h < 8; ++h)
#pragma unroll
        for (int i = 0; i < 8; ++i) qv[h][i] = 0.f;
#else
    uint32_t qf[4][2];
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) qf[kk][0] = qf[kk][1] = 0u;
#endif

    for (;;) {
        while (more && !dead && ni < nc + kScoreStages) {
            if (!cur.next_seg(v, 0)) {
                more = false;
                break;
            }
            const int rows_seg = (cur.i1 - cur.i0) * p.g;
            Desc d;
            d.kind = K_SCORE;
            d.pair = cur.pair;
            d.nvalid = min(kGistRows, rows_seg - cur.off);
            d.flags = (cur.off == 0 ? (F_FIRST | F_Q) : 0) |
                      (cur.off + kGistRows >= rows_seg ? F_LAST : 0);
            d.lrow = lbase + cur.off;
            d.c0 = cur.i0;
            d.nch = cur.i1 - cur.i0;
            d.off = cur.off;
            const int y = (cur.pair * p.M_max + cur.i0) * p.g + cur.off;
            cur.off += kGistRows;
            if (cur.off >= rows_seg) {
                cur.end_seg();
                lbase += rows_seg;
            }
            const int s = ni % kScoreStages;
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
                tma_load_2d_hint(ring + s * kSlotBytes, &tm_kg, 0, y, &full[s], pol);
                if (SSA_PREFETCH_GISTV)
                    bulk_prefetch_l2(static_cast<const __nv_bfloat16*>(p.v_gist) + (size_t)y * kD,
                                     (uint32_t)d.nvalid * kD * 2, pol_keep);
            }
            __syncwarp();
            ++ni;
        }
        if (nc == ni) break;
        ST_TR(40, ni, nc);
        const int s = nc % kScoreStages;
        if (!mbar_wait(&full[s], (uint32_t)((nc / kScoreStages) & 1), 8 * p.wait_limit)) {
            dead = true;
            ++nc;
            continue;
        }
        const Desc d = desc[s];
        const uint32_t box = ring_s + s * kSlotBytes;
        const int nv = d.nvalid;
#if SSA_SCORE_CUDA_CORES
        if (d.flags & F_Q) {
            const __nv_bfloat16* qsm = reinterpret_cast<const __nv_bfloat16*>(qs + s * L.qbytes);
            const int c8 = 8 * (lane & 7);
#pragma unroll
            for (int h = 0; h < 8; ++h)
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    qv[h][i] = h < G ? __bfloat162float(qsm[h * kD + c8 + i]) : 0.f;
        }
        {
            float* lgrow = p.pp_logits + ((size_t)(d.pair * p.M_max + d.c0) * p.g + d.off) * GP;
            if (G <= 4)
                score_stage_cuda_cores<4>(p, box, qv, nv, G, GP, lgrow, rmax + d.lrow, scale, scale_log2);
            else
                score_stage_cuda_cores<8>(p, box, qv, nv, G, GP, lgrow, rmax + d.lrow, scale, scale_log2);
        }
#else
        if (d.flags & F_Q) {
            const uint8_t* qsm = qs + s * L.qbytes;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint32_t a = *reinterpret_cast<const uint32_t*>(qsm + (g8 * kD + 16 * kk + 2 * tig) * 2);
                const uint32_t b = *reinterpret_cast<const uint32_t*>(qsm + (g8 * kD + 16 * kk + 8 + 2 * tig) * 2);
                qf[kk][0] = g8 < G ? a : 0u;
                qf[kk][1] = g8 < G ? b : 0u;
            }
        }
        // the four 16-row blocks are independent (rows past nvalid are
        // computed from whatever the slot holds and never stored)
        float st[4][4];
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) st[blk][0] = st[blk][1] = st[blk][2] = st[blk][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
#pragma unroll
            for (int blk = 0; blk < 4; ++blk) {
                const int row = 16 * blk + (lane & 7) + (((lane >> 3) & 1) << 3);
                uint32_t a[4];
                ldsm_x4(box + swz(row, 2 * kk + (lane >> 4)), a[0], a[1], a[2], a[3]);
                mma_bf16_16816(st[blk], a, qf[kk][0], qf[kk][1]);
            }
        // kept logits: rows of the pair's gist list, GP floats per row; this
        // lane holds heads 2 tig, 2 tig + 1 of rows g8 and g8 + 8
        const int h0 = 2 * tig;
        float* lgrow = p.pp_logits + ((size_t)(d.pair * p.M_max + d.c0) * p.g + d.off) * GP + h0;
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
            const int ra = 16 * blk + g8, rb = ra + 8;
            if (h0 < G && ra < nv)
                *reinterpret_cast<float2*>(lgrow + (size_t)ra * GP) =
                    make_float2(st[blk][0] * scale_log2, st[blk][1] * scale_log2);
            if (h0 < G && rb < nv)
                *reinterpret_cast<float2*>(lgrow + (size_t)rb * GP) =
                    make_float2(st[blk][2] * scale_log2, st[blk][3] * scale_log2);
        }
        float va[4], vb[4];
#pragma unroll
        for (int blk = 0; blk < 4; ++blk) {
            va[blk] = h0 < G ? st[blk][0] : -INFINITY;
            vb[blk] = h0 < G ? st[blk][2] : -INFINITY;
            if (h0 + 1 < G) {
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
#endif
        // the chunks whose last gist row this stage scored
        const int cb = p.g_shift >= 0 ? d.off >> p.g_shift : d.off / p.g;
        const int ce = (d.flags & F_LAST) ? d.nch
                       : (p.g_shift >= 0 ? (d.off + nv) >> p.g_shift : (d.off + nv) / p.g);
        __syncwarp();
        const int seg = d.lrow - d.off;
        float* dst = p.pp_scores + (size_t)d.pair * score_row(p.M_max) + d.c0;
        for (int c = cb + lane; c < ce; c += 32) {
            const float* r = rmax + seg + c * p.g;
            float m = r[0];
            for (int t = 1; t < p.g; ++t) m = fmaxf(m, r[t]);
            dst[c] = m;
        }
        __syncwarp();
        ++nc;
    }
    ST_TR(29, ni, dead ? 1 : 0);
    if (dead) {
        if (lane == 0)
            for (int i = max(0, ni - kScoreStages); i < ni; ++i)
                mbar_wait(&full[i % kScoreStages], (uint32_t)((i / kScoreStages) & 1), p.wait_limit);
        __syncwarp();
    }
}

// The first four warps of a block run the library's deterministic block
// top-k together (a named barrier over their 128 threads).
struct Sync128 {
    __device__ void operator()() const { named_sync(1, 128); }
    __device__ bool or_(bool pred) const { return named_sync_or(1, 128, pred); }
};

// Exclusive prefix sum over the 128 threads of warps 0..3 (named barrier 1);
// sm holds 5 ints.  Returns this thread's prefix, and the total in `total`.
__device__ __forceinline__ int scan128(int v, int* sm, int& total) {
    const int lane = threadIdx.x & 31, wq = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sm[wq] = x;
    named_sync(1, 128);
    int base = 0, tot = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int si = sm[i];
        base += i < wq ? si : 0;
        tot += si;
    }
    named_sync(1, 128);
    total = tot;
    return base + x - v;
}

// Top-k of one pair by the 128 threads of warps 0..3 (sec. 3.3: the k =
// min(topk, M) chunks with the largest scores, ties to the lower chunk,
// ascending, then -1 up to topk, into out[0..topk)); M <= 1024.  Thread t
// owns chunks 8 t .. 8 t + 7.  A lower bound tau on the k-th largest key is
// the q-th largest (q = ceil(k / 2)) of the threads' second-largest keys:
// those q threads hold at least 2 q >= k keys that large.  The keys >= tau
// are compacted in chunk order (one block scan) and, if there are at most
// 128 of them, ranked exactly by counting larger composites (key, ~chunk);
// the selected ones are placed by a second scan.  Returns false (nothing
// written) when tau leaves more than 128 candidates; the caller then runs the
// general block top-k.  Straight-line code: every thread runs every step.
__device__ __forceinline__ bool fast_topk128(const float* scores, int M, int topk, int* out,
                                             TopkScratch& sc) {
    const int t = threadIdx.x;
    const int k = min(topk, M);
    if (k == 0) {
        for (int i = t; i < topk; i += 128) out[i] = -1;
        named_sync(1, 128);
        return true;
    }
    uint32_t key[8];
    {
        const float4* src = reinterpret_cast<const float4*>(scores);
        const float4 a = 8 * t < M ? __ldcg(src + 2 * t) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 b = 8 * t + 4 < M ? __ldcg(src + 2 * t + 1) : make_float4(0.f, 0.f, 0.f, 0.f);
        const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
        for (int i = 0; i < 8; ++i) key[i] = 8 * t + i < M ? score_key(v[i]) : 0u;
    }
    uint32_t t0 = 0u, t1 = 0u;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        t1 = max(t1, min(t0, key[i]));
        t0 = max(t0, key[i]);
    }
    uint32_t* v2 = sc.tmax;
    int* misc = sc.bcast;  // [0] tau
    v2[t] = t1;
    named_sync(1, 128);
    // rank of this thread's value among the 128 (ties to the lower thread)
    const int q = (k + 1) / 2;
    int rank = 0;
    for (int u = 0; u < 128; ++u) {
        const uint32_t y = v2[u];
        rank += (y > t1) | ((y == t1) & (u < t));
    }
    if (rank == q - 1) misc[0] = (int)t1;
    named_sync(1, 128);
    const uint32_t tau = (uint32_t)misc[0];
    int mine = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) mine += tau > 0u && key[i] >= tau;
    int nc;
    int at = scan128(mine, sc.scan, nc);
    if (tau == 0u || nc > 128) return false;  // uniform: every thread sees the same
    unsigned long long* cand = sc.ccomp;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const bool c = key[i] >= tau;
        if (c) cand[at] = ((unsigned long long)key[i] << 32) | (uint32_t)~(uint32_t)(8 * t + i);
        at += c;
    }
    named_sync(1, 128);
    const unsigned long long x = t < nc ? cand[t] : 0ull;
    int r = 0;
    for (int m = 0; m < nc; ++m) r += cand[m] > x;
    const bool take = t < nc && r < k;
    int ntake;
    const int pos = scan128(take ? 1 : 0, sc.scan, ntake);
    if (take) out[pos] = (int)~(uint32_t)x;
    for (int i = k + t; i < topk; i += 128) out[i] = -1;
    named_sync(1, 128);
    return true;
}

// --------------------------------------------------------- attend kernel ---

// Grid: one block per SM; the last warp of each block is its control warp,
// the others are workers.  A worker attends its share of the CHUNKS list
// (gist values weighted by the kept logits, rows of selected chunks masked)
// and then its share of the TILES list (raw K/V: S = Q.K^T, online softmax,
// P.V, all on the tensor cores), and writes one partial per query head for
// each (list, pair) it touches.  Partials carry the launch's epoch in their
// first word; a control warp combines the partials of its (pair, query
// head) tasks as they complete (every wait bounded); the last block to
// finish moves the epoch on.
// kUnion: the per-head union selection (a separate instantiation, so that
// its code does not weigh on the registers of the default one).
template <bool kUnion>
__global__ void __launch_bounds__(kAttnThreads, 1)
    attend_kernel(const __grid_constant__ Plan p, const __grid_constant__ CUtensorMap tm_vg,
                  const __grid_constant__ CUtensorMap tm_kr,
                  const __grid_constant__ CUtensorMap tm_vr) {
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const int workers = (blockDim.x >> 5) - 1;
    const AttnLayout L = attn_layout(p, workers);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g8 = lane >> 2, tig = lane & 3;
    const int G = p.G, GP = logit_stride(G);
    int* nb = reinterpret_cast<int*>(smem + L.plan);
    int* ps0 = nb + p.B;
    int* ps1 = ps0 + p.B + 1;
    unsigned* misc = reinterpret_cast<unsigned*>(smem + L.misc);
    if (threadIdx.x == 0) {
        prefetch_tensormap(&tm_vg);
        prefetch_tensormap(&tm_kr);
        prefetch_tensormap(&tm_vr);
        const unsigned e = ld_relaxed_u32(p.st_hdr) + 1u;
        misc[0] = e == 0u ? 1u : e;
    }
    build_plan(p, nb, ps0, ps1, false);
    // the scoring kernel's chunk scores and kept logits are read from here on
    wait_prerequisites();
    const unsigned tag = misc[0];
    const View v{p, nb, ps0, ps1, (int)gridDim.x * workers};
    const long long lim = wait_cycles(p.wait_limit);
#ifdef SSA_TRACE
    int tr_n = 32;  // the scoring kernel's events come first
#endif
    ST_TR(1, 0, 0);
    const float scale_log2 = 0.125f * 1.4426950408889634f;
    const int tpc = (p.C + kRawRows - 1) / kRawRows;

    if (warp < workers) {
        // ============================================================ worker
        const int w = blockIdx.x * workers + warp;
        uint8_t* ring = smem + L.ring + warp * kAttnStages * kSlotBytes;
        uint8_t* lgs = smem + L.lgs + warp * kAttnStages * L.lgbytes;
        uint8_t* qs = smem + L.qs + warp * kAttnStages * L.qbytes;
        uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars) + warp * kAttnStages;
        Desc* desc = reinterpret_cast<Desc*>(smem + L.desc) + warp * kAttnStages;
        uint32_t* bits = reinterpret_cast<uint32_t*>(smem + L.bits) + warp * L.bwords;
        // two-entry cache of published selections (entries in chunk order)
        int* selc = reinterpret_cast<int*>(smem + L.sel) + warp * 2 * L.kcap;
        if (lane == 0) {
            for (int s = 0; s < kAttnStages; ++s) mbar_init(&full[s], 1);
            fence_barrier_init();
        }
        __syncwarp();
        const uint64_t pol = l2_policy_evict_first();
        const uint32_t ring_s = smem_u32(ring);

        Cursor cg, cr;  // gist-value share (CHUNKS), raw share (TILES)
        v.share(0, w, cg.x, cg.hi);
        v.share(1, w, cr.x, cr.hi);
        int phase = K_GISTV, ni = 0, nc = 0, lbase = 0;
        bool dead = false;
        int cpair0 = -1, cpair1 = -1, ccount0 = 0, ccount1 = 0;
        int pin = -1;  // pair whose raw tiles are being issued (kept cached)
        // Fetches the published selection of `pair` into a cache entry not
        // holding `keep`.  One round of loads per attempt; with `blocking`
        // polls until every entry carries this launch's epoch (bounded; on
        // running out the entry holds no chunk and a timeout is recorded).
        // Returns the entry or -1; every lane gets the same answer.
        auto fetch_sel = [&](int pair, int keep, bool blocking) -> int {
            if (cpair0 == pair) return 0;
            if (cpair1 == pair) return 1;
            const int e = (cpair0 == keep && keep >= 0) ? 1 : 0;
            int* dst = selc + e * L.kcap;
            const int k = min(p.sel_stride, nb[pair / p.Hkv] / p.C);
            const unsigned long long* src = p.st_sel + (size_t)pair * p.st_sel_stride;
            const long long c0 = clock64();
            for (;;) {
                bool ok = true;
                for (int i = lane; i < k; i += 32) {
                    const unsigned long long x = ld_relaxed_u64(src + i);
                    ok = ok && (unsigned)(x >> 32) == tag;
                    dst[i] = (int)(unsigned)x;
                }
                const bool done = __all_sync(0xffffffffu, ok);
                const bool give_up = !done && warp_expired(c0, lim);
                if (done || give_up || !blocking) {
                    __syncwarp();
                    if (!done && !blocking) return -1;
                    if (give_up && lane == 0) report_status(kStatusTimeout);
                    // the chunks are the leading non-negative entries (a
                    // per-head union pads its slots with -1)
                    int cnt = 0;
                    for (int i = lane; i < k; i += 32) cnt += dst[i] >= 0;
#pragma unroll
                    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
                    if (e == 0) {
                        cpair0 = pair;
                        ccount0 = done ? cnt : 0;
                    } else {
                        cpair1 = pair;
                        ccount1 = done ? cnt : 0;
                    }
                    return e;
                }
                __nanosleep(64);
            }
        };
        auto sel_entries = [&](int e) -> const int* { return selc + e * L.kcap; };
        auto sel_count = [&](int e) { return e == 0 ? ccount0 : ccount1; };

        uint32_t qf[4][2];
        float acc[4][4];
        float m_run = -INFINITY, l_run = 0.f;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) qf[kk][0] = qf[kk][1] = 0u;
#pragma unroll
        for (int mt = 0; mt < 4; ++mt)
#pragma unroll
            for (int c = 0; c < 4; ++c) acc[mt][c] = 0.f;
        auto reset_state = [&]() {
            m_run = -INFINITY;
            l_run = 0.f;
#pragma unroll
            for (int mt = 0; mt < 4; ++mt)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[mt][c] = 0.f;
        };
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
#if SSA_PIPE_PV_LO
            split_bf16(p00, p01, hi0, lo0);
            split_bf16(p10, p11, hi1, lo1);
#else
            hi0 = pack_bf16(p00, p01);
            hi1 = pack_bf16(p10, p11);
            lo0 = lo1 = 0u;
#endif
            const int row = r0 + (lane & 7) + ((lane >> 4) << 3);
            const int csel = (lane >> 3) & 1;
#pragma unroll
            for (int mt = 0; mt < 4; ++mt) {
                uint32_t a[4];
                ldsm_x4_trans(vbox + swz(row, 2 * mt + csel), a[0], a[1], a[2], a[3]);
                mma_bf16_16816(acc[mt], a, hi0, hi1);
                if (SSA_PIPE_PV_LO) mma_bf16_16816(acc[mt], a, lo0, lo1);
            }
        };
        // One partial per query head of the segment (list Lp, pair); each
        // record's epoch word is written after its data.
        auto write_partial = [&](int Lp, int pair) {
            ST_TR(45, Lp, pair);
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

        // The top-k of the pairs this block owns (pair q is owned by block
        // q mod grid), by warps 0..3 with the library's block top-k; the
        // selection goes to sel_idx and, tagged with the epoch, to the
        // workspace for every worker that needs it.
        bool selected = false;
        int* selout = reinterpret_cast<int*>(smem + L.selout);
        TopkScratch& tks = *reinterpret_cast<TopkScratch*>(smem + L.tk);
        // Per-head union (App. A): each head of the group ranks the chunks by
        // its own score, the max over the chunk's gist rows of its kept logit
        // (log2 domain: the same order as q.k / sqrt(d)), written over the
        // pair's group-max scores one head at a time; the heads' top-k's are
        // ORed into a chunk bitmap and compacted in chunk order.
        uint32_t* ubits = reinterpret_cast<uint32_t*>(smem + L.ubits);
        auto union_selection = [&](int pr, int M) {
            const int t = threadIdx.x;
            float* hs = p.pp_scores + (size_t)pr * score_row(p.M_max);
            const int W = (M + 31) >> 5;
            for (int i = t; i < W; i += 128) ubits[i] = 0u;
            for (int h = 0; h < G; ++h) {
                const float* lg = p.pp_logits + (size_t)pr * p.M_max * p.g * GP + h;
                for (int m = t; m < M; m += 128) {
                    float best = -INFINITY;
                    for (int r = 0; r < p.g; ++r) best = fmaxf(best, __ldcg(lg + ((size_t)m * p.g + r) * GP));
                    hs[m] = best;
                }
                named_sync(1, 128);
                if (M > 1024 || !fast_topk128(hs, M, p.topk, selout, tks))
                    block_topk<128>(hs, M, p.topk, selout, tks, Sync128());
                named_sync(1, 128);
                for (int i = t; i < min(p.topk, M); i += 128)
                    atomicOr(&ubits[selout[i] >> 5], 1u << (selout[i] & 31));
                named_sync(1, 128);
            }
            const int per = (W + 127) / 128;
            const int w0 = t * per, w1 = min(w0 + per, W);
            int cnt = 0;
            for (int i = w0; i < w1; ++i) cnt += __popc(ubits[i]);
            int tot;
            int at = scan128(cnt, tks.scan, tot);
            for (int i = w0; i < w1; ++i)
                for (uint32_t x = ubits[i]; x; x &= x - 1) selout[at++] = i * 32 + __ffs(x) - 1;
            for (int i = tot + t; i < p.sel_stride; i += 128) selout[i] = -1;
            named_sync(1, 128);
        };
        auto run_selection = [&]() {
            if (warp >= 4 || p.topk <= 0 || (int)blockIdx.x >= p.n_pairs) return;
            for (int pr = blockIdx.x; pr < p.n_pairs; pr += gridDim.x) {
                const int M = nb[pr / p.Hkv] / p.C;
                const int k = min(p.sel_stride, M);  // published entries
                if constexpr (kUnion) {
                    union_selection(pr, M);
                } else {
                    const float* sc = p.pp_scores + (size_t)pr * score_row(p.M_max);
                    if (M > 1024 || !fast_topk128(sc, M, p.topk, selout, tks))
                        block_topk<128>(sc, M, p.topk, selout, tks, Sync128());
                    named_sync(1, 128);
                }
                unsigned long long* pub = p.st_sel + (size_t)pr * p.st_sel_stride;
                int32_t* user = p.sel_idx + (size_t)pr * p.sel_stride;
                for (int i = threadIdx.x; i < p.sel_stride; i += 128) {
                    const int c = selout[i];
                    user[i] = c;
                    if (i < k && !(p.debug_flags & 1))
                        st_relaxed_u64(pub + i, tagged(tag, (unsigned)c));
                }
                named_sync(1, 128);
            }
        };

        for (;;) {
            // ---- issue ahead; raw tiles only once the selection is known
            while (!dead && phase != 3 && ni < nc + kAttnStages) {
                Desc d;
                int y = 0;
                if (phase == K_GISTV) {
                    if (!cg.next_seg(v, 0)) {
                        phase = K_RAW;
                        continue;
                    }
                    const int rows_seg = (cg.i1 - cg.i0) * p.g;
                    d.kind = K_GISTV;
                    d.pair = cg.pair;
                    d.nvalid = min(kGistRows, rows_seg - cg.off);
                    d.flags = (cg.off == 0 ? F_FIRST : 0) | (cg.off + kGistRows >= rows_seg ? F_LAST : 0);
                    d.lrow = lbase + cg.off;
                    d.c0 = cg.i0;
                    d.nch = cg.i1 - cg.i0;
                    d.off = cg.off;
                    y = (cg.pair * p.M_max + cg.i0) * p.g + cg.off;
                    cg.off += kGistRows;
                    if (cg.off >= rows_seg) {
                        cg.end_seg();
                        lbase += rows_seg;
                    }
                } else {
                    if (!cr.next_seg(v, 1)) {
                        phase = 3;
                        break;
                    }
                    const int pr = cr.pair;
                    const int n = nb[pr / p.Hkv];
                    const int M = n / p.C;
                    const int kc = min(p.sel_stride, M);
                    const int u = cr.i0 + cr.off;
                    int r0, nv;
                    if (u < kc * tpc) {
                        // the selected chunk's tiles need the published
                        // selection (blocking only with nothing in flight, and
                        // only after this block's own top-k ran)
                        const int e = fetch_sel(pr, pin, selected && ni == nc);
                        if (e < 0) break;  // not yet: consume what is in flight
                        pin = pr;
                        const int c = u / tpc, part = u - c * tpc;
                        if (c < sel_count(e)) {
                            const int chunk = min(max(sel_entries(e)[c], 0), max(M - 1, 0));
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
                    d.kind = K_RAW;
                    d.pair = pr;
                    d.nvalid = nv;
                    d.flags = (cr.off == 0 ? (F_FIRST | F_Q) : 0) | (u + 1 >= cr.i1 ? F_LAST : 0);
                    d.lrow = d.c0 = d.nch = d.off = 0;
                    y = pr * p.n_max + r0;
                    ++cr.off;
                    if (cr.i0 + cr.off >= cr.i1) {
                        cr.end_seg();
                        pin = -1;
                    }
                }
                const int s = ni % kAttnStages;
                __syncwarp();
                if (lane == 0) {
                    desc[s] = d;
                    fence_proxy_async_smem();
                    uint8_t* dst = ring + s * kSlotBytes;
                    if (d.kind == K_GISTV) {
                        mbar_arrive_expect_tx(&full[s], (uint32_t)(kSlotBytes + L.lgbytes));
                        tma_load_2d_hint(dst, &tm_vg, 0, y, &full[s], pol);
                        bulk_load(lgs + s * L.lgbytes, p.pp_logits + (size_t)y * GP,
                                  (uint32_t)L.lgbytes, &full[s]);
                    } else {
                        // an empty tile (an unused slot of a per-head union)
                        // loads nothing but the query
                        const bool wq = (d.flags & F_Q) != 0;
                        const bool any = d.nvalid > 0;
                        mbar_arrive_expect_tx(&full[s], (uint32_t)((any ? kSlotBytes : 0) +
                                                                   (wq ? G * kD * 2 : 0)));
                        if (wq) {
                            const int b = d.pair / p.Hkv, j = d.pair - b * p.Hkv;
                            const __nv_bfloat16* src = static_cast<const __nv_bfloat16*>(p.q) +
                                                       ((size_t)b * p.Hq + (size_t)j * G) * kD;
                            bulk_load(qs + s * L.qbytes, src, (uint32_t)(G * kD * 2), &full[s]);
                        }
                        if (any) {
                            tma_load_2d_hint(dst, &tm_kr, 0, y, &full[s], pol);
                            tma_load_2d_hint(dst + kSlotBytes / 2, &tm_vr, 0, y, &full[s], pol);
                        }
                    }
                }
                __syncwarp();
                ++ni;
            }
            if (!selected) {
                // the first issue round is in flight: the pairs this block
                // owns get their top-k now
                ST_TR(41, ni, nc);
                run_selection();
                ST_TR(42, ni, nc);
                selected = true;
                continue;
            }
            if (nc == ni) {
                if (phase == 3 || dead) break;
                continue;  // the next raw tile waited for a selection: retry
            }
            ST_TR(43, phase, nc);

            // ---- consume the oldest stage
            const int s = nc % kAttnStages;
            if (!mbar_wait(&full[s], (uint32_t)((nc / kAttnStages) & 1), 8 * p.wait_limit)) {
                dead = true;
                ++nc;
                continue;
            }
            const Desc d = desc[s];
            ST_TR(46, d.kind, d.pair);
            const uint32_t box = ring_s + s * kSlotBytes;
            const int nv = d.nvalid;
            if (d.kind == K_GISTV) {
                if (d.flags & F_FIRST) {
                    reset_state();
                    // selected chunks of this segment (bit c: chunk c0 + c)
                    const int e = fetch_sel(d.pair, pin, true);
                    const int* ent = sel_entries(e);
                    const int k = sel_count(e);
                    const int words = (d.nch + 31) >> 5;
                    for (int i = lane; i < words; i += 32) bits[i] = 0u;
                    __syncwarp();
                    for (int i = lane; i < k; i += 32) {
                        const int c = ent[i] - d.c0;
                        if (c >= 0 && c < d.nch) atomicOr(&bits[c >> 5], 1u << (c & 31));
                    }
                    __syncwarp();
                }
                // excluded rows: past the valid rows, or in a selected chunk
                // (the selected-only context excludes the unselected ones)
                const bool keep_selected = p.ctx_mode == 1;
                uint32_t ex[2];
#pragma unroll
                for (int hh = 0; hh < 2; ++hh) {
                    const int r = lane + 32 * hh;
                    const int sr = d.off + r;
                    const int c = min(p.g_shift >= 0 ? (sr >> p.g_shift) : sr / p.g, d.nch - 1);
                    const bool in_sel = ((bits[c >> 5] >> (c & 31)) & 1u) != 0u;
                    const bool e = (r >= nv) | (in_sel != keep_selected);
                    ex[hh] = __ballot_sync(0xffffffffu, e);
                }
                // head g8's kept logits of rows r0 + 2 tig, + 1, + 8, + 9
                const float* lgst = reinterpret_cast<const float*>(lgs + s * L.lgbytes) + (g8 < G ? g8 : 0);
                const uint32_t hm = g8 < G ? 0u : 0xffffffffu;
                float x[4][4];
#pragma unroll
                for (int blk = 0; blk < 4; ++blk) {
                    const int r0 = 16 * blk + 2 * tig;
                    const uint32_t eb = ((ex[blk >> 1] >> (16 * (blk & 1))) & 0xffffu) | hm;
                    const float a0 = lgst[(r0)*GP], a1 = lgst[(r0 + 1) * GP];
                    const float b0 = lgst[(r0 + 8) * GP], b1 = lgst[(r0 + 9) * GP];
                    x[blk][0] = ((eb >> (2 * tig)) & 1u) ? -INFINITY : a0;
                    x[blk][1] = ((eb >> (2 * tig + 1)) & 1u) ? -INFINITY : a1;
                    x[blk][2] = ((eb >> (2 * tig + 8)) & 1u) ? -INFINITY : b0;
                    x[blk][3] = ((eb >> (2 * tig + 9)) & 1u) ? -INFINITY : b1;
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
                if (d.flags & F_FIRST) reset_state();
                if (d.flags & F_Q) {
                    const uint8_t* qsm = qs + s * L.qbytes;
#pragma unroll
                    for (int kk = 0; kk < 4; ++kk) {
                        const uint32_t a = *reinterpret_cast<const uint32_t*>(qsm + (g8 * kD + 16 * kk + 2 * tig) * 2);
                        const uint32_t b = *reinterpret_cast<const uint32_t*>(qsm + (g8 * kD + 16 * kk + 8 + 2 * tig) * 2);
                        qf[kk][0] = g8 < G ? a : 0u;
                        qf[kk][1] = g8 < G ? b : 0u;
                    }
                }
                // S = Q.K^T with the heads as M rows (rows 8..15 zero)
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
            ST_TR(47, d.kind, d.flags);
            __syncwarp();
            ++nc;
        }
        ST_TR(29, ni, dead ? 1 : 0);
        if (dead) {
            if (lane == 0)
                for (int i = max(0, ni - kAttnStages); i < ni; ++i)
                    mbar_wait(&full[i % kAttnStages], (uint32_t)((i / kAttnStages) & 1), p.wait_limit);
            __syncwarp();
        }
    } else {
        // ====================================================== control warp
        // Combinations: task t = pair * G + head, t = block (mod N).  The
        // partials of one (list, head, pair) are consecutive records; a batch
        // of up to 32 is waited for, then read with every load in flight at
        // once: lane l takes columns 4 (l & 15) .. + 3 of records 2 i + (l >> 4).
        const int N = gridDim.x, P = p.n_pairs;
        for (int t = blockIdx.x; t < P * G; t += N) {
            const int pr = t / G, h = t - pr * G;
            const int b = pr / p.Hkv, j = pr - b * p.Hkv;
            float Mr = -INFINITY, Lr = 0.f;
            float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int Lp = 0; Lp < 2; ++Lp) {
                int w0, w1;
                if (!v.pair_workers(Lp, pr, w0, w1)) continue;
                for (int base = w0; base <= w1; base += 32) {
                    const int cnt = min(32, w1 - base + 1);
                    const char* recs = part_rec(p, Lp, h, base, pr);
                    const char* mine = recs + (size_t)min(lane, cnt - 1) * kRecBytes;
                    const long long c0 = clock64();
                    ST_TR(44, t, base);
                    for (;;) {
                        const bool ok =
                            lane >= cnt || ld_relaxed_u32(reinterpret_cast<const unsigned*>(mine)) == tag;
                        if (__all_sync(0xffffffffu, ok)) break;
                        if (warp_expired(c0, lim)) {
                            if (lane == 0) report_status(kStatusTimeout);
                            break;
                        }
                        __nanosleep(128);
                    }
                    fence_acquire_gpu();
                    const float2 ml = __ldcg(reinterpret_cast<const float2*>(mine + 8));
                    const float mi = lane < cnt ? ml.x : -INFINITY;
                    const float li = lane < cnt ? ml.y : 0.f;
                    float4 vals[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int rr = min(2 * i + (lane >> 4), cnt - 1);
                        vals[i] = __ldcg(reinterpret_cast<const float4*>(recs + (size_t)rr * kRecBytes + 16) +
                                         (lane & 15));
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
                    Lr = Lr * fo + ls;
                    o.x *= fo;
                    o.y *= fo;
                    o.z *= fo;
                    o.w *= fo;
                    Mr = mn;
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        const int rr = 2 * i + (lane >> 4);
                        // every lane takes part in the shuffle (rr < 32)
                        const float fr = __shfl_sync(0xffffffffu, fi, rr);
                        const float f = rr < cnt ? fr : 0.f;
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
                float4* dst = reinterpret_cast<float4*>(p.out + (((size_t)b * p.Hq + (size_t)j * G + h) * kD));
                dst[lane] = make_float4(o.x * inv, o.y * inv, o.z * inv, o.w * inv);
            }
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

}  // namespace pipe
}  // namespace ssa
