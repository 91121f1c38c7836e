// ssa_api.cpp -- the C ABI of libssa (include/ssa.h): argument checks, work
// planning, workspace handling and dispatch to the kernels.  Never throws
// across the boundary; never synchronises the host in the hot calls.
#include "../../include/ssa.h"

#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <unordered_map>

#include "ssa_internal.h"

namespace ssa {
int fused_smem_bytes(const Plan& p);
}

namespace {

thread_local std::string g_err;
std::atomic<long long> g_wait_limit{0};
std::atomic<int> g_debug{0};
std::atomic<int> g_max_blocks{0};
#ifdef SSA_TRACE
std::atomic<void*> g_trace{nullptr};
std::atomic<int> g_trace_cap{0};
#endif
std::atomic<int> g_rows_per_score{0};

constexpr long long kDefaultWaitLimitNs = 2000000000ll;  // 2 s
constexpr int kMaxG = 16;
constexpr int kMaxTopk = 1024;
constexpr int kRowsPerScoreItem = 1024;

int rows_per_score_item() {
    int v = g_rows_per_score.load();
    return v > 0 ? v : kRowsPerScoreItem;
}
int max_blocks() { return g_max_blocks.load(); }

ssa_status fail(ssa_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
ssa_status fail(ssa_status s, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return s;
}

ssa_status cuda_fail(cudaError_t e, const char* what) {
    return fail(SSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int cdiv(long long a, long long b) { return (int)((a + b - 1) / b); }

// Common shape checks.  need_d: check d/dtype (not needed by top-k).
ssa_status check_shape(const ssa_shape* s, int C, bool need_d) {
    if (!s) return fail(SSA_ERR_INVALID_ARG, "shape is NULL");
    if (s->B < 1 || s->Hq < 1 || s->Hkv < 1 || s->n_max < 1)
        return fail(SSA_ERR_INVALID_ARG, "B, Hq, Hkv, n_max must be >= 1");
    if (s->Hq % s->Hkv) return fail(SSA_ERR_INVALID_ARG, "Hq (%d) not a multiple of Hkv (%d)",
                                    s->Hq, s->Hkv);
    if (s->Hq / s->Hkv > kMaxG)
        return fail(SSA_ERR_UNSUPPORTED, "group size Hq/Hkv = %d > %d", s->Hq / s->Hkv, kMaxG);
    if (C < 1) return fail(SSA_ERR_INVALID_ARG, "C must be >= 1");
    if (s->n_max % C) return fail(SSA_ERR_INVALID_ARG, "n_max (%d) not a multiple of C (%d)",
                                  s->n_max, C);
    if (need_d) {
        if (s->dtype == SSA_BF16) {
            if (s->d != 64 && s->d != 128)
                return fail(SSA_ERR_UNSUPPORTED, "bf16 needs d in {64, 128}, got %d", s->d);
        } else if (s->dtype == SSA_FP32) {
            if (s->d < 1 || s->d > 256)
                return fail(SSA_ERR_UNSUPPORTED, "fp32 needs 1 <= d <= 256, got %d", s->d);
        } else {
            return fail(SSA_ERR_INVALID_ARG, "unknown dtype %d", s->dtype);
        }
    }
    const long long P = (long long)s->B * s->Hkv;
    if (P * s->n_max >= (1ll << 31))
        return fail(SSA_ERR_UNSUPPORTED, "B*Hkv*n_max too large for 32-bit row indices");
    return SSA_OK;
}

// Fill shapes of a plan (no pointers).
void fill_shape(ssa::Plan& p, const ssa_shape* s, int C, int g, int topk) {
    p.dtype = s->dtype;
    p.B = s->B;
    p.Hq = s->Hq;
    p.Hkv = s->Hkv;
    p.G = s->Hq / s->Hkv;
    p.d = s->d;
    p.n_max = s->n_max;
    p.C = C;
    p.g = g;
    p.M_max = s->n_max / C;
    p.topk = topk;
    p.sel_stride = topk;
    p.n_pairs = s->B * s->Hkv;
    long long lim = g_wait_limit.load();
    p.wait_limit = lim > 0 ? lim : kDefaultWaitLimitNs;
    p.debug_flags = g_debug.load();
#ifdef SSA_TRACE
    p.trace = static_cast<uint4*>(g_trace.load());
    p.trace_cap = g_trace_cap.load();
#endif
}

bool fused_path(const ssa::Plan& p) {
    return p.dtype == SSA_BF16 && (p.d == 64 || p.d == 128) && p.B <= ssa::kFusedMaxB;
}

ssa_status check_sizes(const ssa::Plan& p) {
    const long long P = p.n_pairs;
    if (P * p.M_max * (long long)p.g >= (1ll << 31))
        return fail(SSA_ERR_UNSUPPORTED, "gist rows too large for 32-bit row indices");
    if (p.g > 1024) return fail(SSA_ERR_UNSUPPORTED, "g = %d > 1024", p.g);
    if (p.topk > kMaxTopk) return fail(SSA_ERR_UNSUPPORTED, "topk = %d > %d", p.topk, kMaxTopk);
    if (p.h2) {
        if (P * p.S_max * (long long)p.gm >= (1ll << 31))
            return fail(SSA_ERR_UNSUPPORTED, "meta rows too large for 32-bit row indices");
        if (p.gm > 1024) return fail(SSA_ERR_UNSUPPORTED, "gm = %d > 1024", p.gm);
        if ((long long)p.J * p.g > 1024)
            return fail(SSA_ERR_UNSUPPORTED, "J*g = %lld > 1024", (long long)p.J * p.g);
        if (p.topk_super > kMaxTopk)
            return fail(SSA_ERR_UNSUPPORTED, "topk_super = %d > %d", p.topk_super, kMaxTopk);
    }
    if (fused_path(p) && ssa::fused_smem_bytes(p) > 227 * 1024)
        return fail(SSA_ERR_UNSUPPORTED, "shared memory plan too large");
    return SSA_OK;
}

}  // namespace

namespace ssa {

void plan_decompose(Plan& p) {
    p.grid_cap = max_blocks();
    p.score_rows = rows_per_score_item();
    // counters line, published-count line, then the published selection(s)
    p.pair_ints = 64 + (p.topk + (p.h2 ? p.topk_super : 0) + 31) / 32 * 32;
    p.mask_words = (cdiv(p.M_max, 32) + 3) / 4 * 4;
    p.g_shift = -1;
    for (int sh = 0; sh < 11; ++sh)
        if (p.g == (1 << sh)) p.g_shift = sh;
    p.smask_words = p.h2 ? (cdiv(p.S_max, 32) + 3) / 4 * 4 : 0;
}

bool seg_lists(const Plan& p) {
    return fused_path(p) && p.topk <= kSegList && (!p.h2 || p.topk_super <= kSegList);
}

int ctrl_words(const Plan& p) { return 64 + p.pair_ints * p.n_pairs; }  // see ssa_fused.cuh

static WsLayout fused_layout(const Plan& p) {
    WsLayout L;
    size_t o = 0;
    auto take = [&](size_t bytes) {
        size_t at = o;
        o += (bytes + 255) / 256 * 256;
        return at;
    };
    const size_t P = (size_t)p.n_pairs;
    L.ctrl = take((size_t)ctrl_words(p) * 4);
    L.scores = take(P * p.M_max * 4);
    L.super_scores = take(p.h2 ? P * p.S_max * 4 : 0);
    L.cand_scores = take(p.h2 ? P * p.Mc_max * 4 : 0);
    L.chunk_mask = take(0);
    L.super_mask = take(0);
    // one set of segment lists per selection level
    L.cands = take(seg_lists(p) ? (p.h2 ? 2 : 1) * (ssa::kFusedMaxGrid + P) * ssa::kSegList * 8 : 0);
    // one partial per (attention list, segment slot, query head)
    L.partials =
        take(fused_path(p) ? 3 * (ssa::kFusedMaxGrid + P) * p.G * (size_t)(p.d + 2) * 4 : 0);
    L.total = o;
    return L;
}

// The pipeline's areas (p prepared by pipe_prepare); the epoch header sits
// at offset 0 in every size, so any two calls of this path agree on it.
static WsLayout pipe_layout(const Plan& p) {
    WsLayout L;
    size_t hdr, sc, lg, sel, part;
    pipe_ws_sizes(p, &hdr, &sc, &lg, &sel, &part);
    size_t o = 0;
    auto take = [&](size_t bytes) {
        size_t at = o;
        o += (bytes + 255) / 256 * 256;
        return at;
    };
    L.pipe = true;
    L.st_hdr = take(hdr);
    L.pp_scores = take(sc);
    L.pp_logits = take(lg);
    L.st_sel = take(sel);
    L.st_part = take(part);
    L.total = o;
    return L;
}

WsLayout plan_layout(const Plan& p) {
    Plan q = p;
    if (pipe_prepare(q)) return pipe_layout(q);
    return fused_layout(p);
}

size_t plan_bytes_any(const Plan& p) {
    size_t a = fused_layout(p).total;
    Plan q = p;
    q.mode = kModeFull;
    if (pipe_prepare(q)) {
        const size_t b = pipe_layout(q).total;
        if (b > a) a = b;
    }
    return a;
}

}  // namespace ssa

namespace {

void attach_ws(ssa::Plan& p, void* ws) {
    const ssa::WsLayout L = ssa::plan_layout(p);
    char* base = static_cast<char*>(ws);
    if (L.pipe) {
        p.st_hdr = reinterpret_cast<unsigned*>(base + L.st_hdr);
        p.pp_scores = reinterpret_cast<float*>(base + L.pp_scores);
        p.pp_logits = reinterpret_cast<float*>(base + L.pp_logits);
        p.st_sel = reinterpret_cast<unsigned long long*>(base + L.st_sel);
        p.st_part = base + L.st_part;
        return;
    }
    p.ctrl = reinterpret_cast<int*>(base + L.ctrl);
    p.scores = reinterpret_cast<float*>(base + L.scores);
    p.super_scores = p.h2 ? reinterpret_cast<float*>(base + L.super_scores) : nullptr;
    p.cand_scores = p.h2 ? reinterpret_cast<float*>(base + L.cand_scores) : nullptr;
    p.partials = reinterpret_cast<float*>(base + L.partials);
    p.cands = ssa::seg_lists(p) ? reinterpret_cast<unsigned long long*>(base + L.cands) : nullptr;
}

// A fused call leaves its control words and its score areas zero (the
// kernel clears what it used), but only for its own layout.  The library
// remembers, per workspace, what the last call left: all zero (after
// ssa_workspace_init, up to a size), a fused layout (control + score bytes
// that are zero), or unknown (a generic-path call).  Before a fused call whose
// layout is not already known to be zero, it zeroes that prefix
// (stream-ordered).
struct WsState {
    int kind = 0;      // 0: zero up to `bytes`; 1: fused layout; 2: unknown;
                       // 3: pipeline (up to `bytes`: zero or written by
                       //    that path, whose words carry an older epoch)
    size_t bytes = 0;  // kind 0: zeroed bytes; kind 1: zero prefix of the layout
    size_t ctrl = 0;   // kind 1: control bytes of the layout
};
std::mutex g_ws_mu;
std::unordered_map<const void*, WsState> g_ws;

void note_ws_zeroed(const void* ws, size_t bytes) {
    std::lock_guard<std::mutex> lk(g_ws_mu);
    WsState st;
    st.kind = 0;
    st.bytes = bytes;
    g_ws[ws] = st;
}

cudaError_t prepare_ws(void* ws, bool fused, size_t ctrl_bytes, size_t clean_bytes,
                       cudaStream_t stream) {
    bool zero = false;
    {
        std::lock_guard<std::mutex> lk(g_ws_mu);
        auto it = g_ws.find(ws);
        WsState next;
        next.kind = fused ? 1 : 2;
        next.bytes = clean_bytes;
        next.ctrl = ctrl_bytes;
        if (fused) {
            if (it == g_ws.end()) {
                zero = false;  // first use: the caller zeroed it
            } else if (it->second.kind == 0) {
                zero = it->second.bytes < clean_bytes;
            } else if (it->second.kind == 1) {
                zero = !(it->second.bytes == clean_bytes && it->second.ctrl == ctrl_bytes);
            } else {
                zero = true;
            }
        }
        g_ws[ws] = next;
    }
    return zero ? cudaMemsetAsync(ws, 0, clean_bytes, stream) : cudaSuccess;
}

// Before a pipeline call: its areas must hold zeros or words of an
// earlier launch of that path (whatever its sizes: the epoch header is at
// offset 0 and only grows), so the workspace is zeroed only when it comes
// from another path or is larger than what is known.
cudaError_t prepare_ws_pipe(void* ws, size_t need, cudaStream_t stream) {
    bool zero = false;
    {
        std::lock_guard<std::mutex> lk(g_ws_mu);
        auto it = g_ws.find(ws);
        WsState next;
        next.kind = 3;
        next.bytes = need;
        if (it != g_ws.end()) {
            const WsState& st = it->second;
            if ((st.kind == 0 || st.kind == 3) && st.bytes >= need)
                next.bytes = st.bytes;
            else
                zero = true;
        }
        g_ws[ws] = next;
    }
    return zero ? cudaMemsetAsync(ws, 0, need, stream) : cudaSuccess;
}

// After a device wait ran out, a fused-layout workspace may hold non-zero
// control words: its next call zeroes it.
void note_timeout() {
    std::lock_guard<std::mutex> lk(g_ws_mu);
    for (auto& kv : g_ws)
        if (kv.second.kind == 1) kv.second.kind = 2;
}

void note_ws_unknown(const void* ws) {
    std::lock_guard<std::mutex> lk(g_ws_mu);
    WsState st;
    st.kind = 2;
    g_ws[ws] = st;
}

cudaError_t launch_plan(const ssa::Plan& p, cudaStream_t stream) {
    if (p.pp_w3 > 0) return ssa::launch_pipe(p, stream);
    return fused_path(p) ? ssa::launch_fused(p, stream) : ssa::launch_generic(p, stream);
}

// Runs a workspace-using plan: caller workspace, or a stream-ordered one.
ssa_status run_with_ws(ssa::Plan& p, void* ws, size_t ws_bytes, cudaStream_t stream) {
    ssa::pipe_prepare(p);
    // a caller workspace must hold ssa_workspace_size() bytes, which cover
    // every path a call of these sizes can take
    const size_t need = p.h2 ? ssa::plan_layout(p).total : ssa::plan_bytes_any(p);
    void* own = nullptr;
    if (ws == nullptr) {
        if (ws_bytes != 0) return fail(SSA_ERR_WORKSPACE, "ws is NULL but ws_bytes != 0");
        cudaError_t e = cudaMallocAsync(&own, need, stream);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMallocAsync(workspace)");
        e = cudaMemsetAsync(own, 0, need, stream);
        if (e != cudaSuccess) {
            cudaFreeAsync(own, stream);
            return cuda_fail(e, "cudaMemsetAsync(workspace)");
        }
        ws = own;
    } else if (ws_bytes < need) {
        return fail(SSA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, need);
    } else if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) {
        return fail(SSA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
    }
    attach_ws(p, ws);
    if (!own) {
        const ssa::WsLayout L = ssa::plan_layout(p);
        cudaError_t e = L.pipe ? prepare_ws_pipe(ws, L.total, stream)
                                 : prepare_ws(ws, fused_path(p), (size_t)ssa::ctrl_words(p) * 4,
                                              L.partials, stream);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(control words)");
    }
    cudaError_t e = launch_plan(p, stream);
    if (own) cudaFreeAsync(own, stream);
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    return SSA_OK;
}

ssa_status check_tensors(const ssa::Plan& p, std::initializer_list<const void*> ptrs) {
    for (const void* q : ptrs)
        if (!q) return fail(SSA_ERR_INVALID_ARG, "a required pointer is NULL");
    if (fused_path(p))
        for (const void* q : ptrs)
            if (!aligned16(q)) return fail(SSA_ERR_UNSUPPORTED, "bf16 tensors must be 16-byte aligned");
    return SSA_OK;
}

ssa_status build_single(ssa::Plan& p, const ssa_shape* shape, int C, int g, int topk) {
    ssa_status st = check_shape(shape, C, true);
    if (st != SSA_OK) return st;
    if (g < 1) return fail(SSA_ERR_INVALID_ARG, "g must be >= 1");
    if (topk < 0) return fail(SSA_ERR_INVALID_ARG, "topk must be >= 0");
    fill_shape(p, shape, C, g, topk);
    ssa::plan_decompose(p);
    return check_sizes(p);
}

ssa_status build_h2(ssa::Plan& p, const ssa_shape* shape, int C, int g, int J, int gm,
                    int topk_super, int topk_chunk) {
    ssa_status st = check_shape(shape, C, true);
    if (st != SSA_OK) return st;
    if (g < 1 || J < 1 || gm < 1) return fail(SSA_ERR_INVALID_ARG, "g, J, gm must be >= 1");
    if (topk_super < 0 || topk_chunk < 0)
        return fail(SSA_ERR_INVALID_ARG, "topk_super, topk_chunk must be >= 0");
    fill_shape(p, shape, C, g, topk_chunk);
    p.h2 = 1;
    p.J = J;
    p.gm = gm;
    p.S_max = p.M_max / J;
    p.topk_super = topk_super;
    const int ks = topk_super < p.S_max ? topk_super : p.S_max;
    long long mc = (long long)ks * J + (J - 1);
    if (mc > p.M_max) mc = p.M_max;
    p.Mc_max = (int)(mc > 0 ? mc : 1);
    ssa::plan_decompose(p);
    return check_sizes(p);
}

// Variant step (generic kernels): layout = chunk scores (per head under the
// union reading) + the per-head selections.
static size_t variant_layout(const ssa::Plan& p, size_t* scores_off, size_t* head_sel_off) {
    size_t o = 0;
    auto take = [&](size_t bytes) {
        size_t at = o;
        o += (bytes + 255) / 256 * 256;
        return at;
    };
    const size_t rows = p.sel_mode ? (size_t)p.B * p.Hq : (size_t)p.n_pairs;
    *scores_off = take(rows * p.M_max * 4);
    *head_sel_off = take(p.sel_mode ? (size_t)p.B * p.Hq * (p.topk > 0 ? p.topk : 1) * 4 : 0);
    return o;
}

static ssa_status build_variant(ssa::Plan& p, const ssa_shape* shape, int C, int g, int topk,
                                int context, int select) {
    if (context != SSA_CONTEXT_UNSELECTED_GISTS && context != SSA_CONTEXT_SELECTED_ONLY)
        return fail(SSA_ERR_INVALID_ARG, "context = %d is not a context reading", context);
    if (select != SSA_SELECT_GROUP_MAX && select != SSA_SELECT_HEAD_UNION)
        return fail(SSA_ERR_INVALID_ARG, "select = %d is not a selection reading", select);
    ssa_status st = build_single(p, shape, C, g, topk);
    if (st != SSA_OK) return st;
    p.ctx_mode = context;
    p.sel_mode = select;
    p.sel_stride = select == SSA_SELECT_HEAD_UNION ? p.G * topk : topk;
    return SSA_OK;
}

// t-level plan: the single-level shape plus the levels' sizes (host arrays
// of levels - 1 summary token counts and levels top-k's).
static ssa_status build_hier(ssa::Plan& p, ssa::HierLevels& hl, const ssa_shape* shape, int C,
                             int g, int J, int levels, const int32_t* g_sum,
                             const int32_t* topk) {
    if (levels < 1 || levels > ssa::kMaxLevels)
        return fail(SSA_ERR_INVALID_ARG, "levels = %d outside [1, %d]", levels, ssa::kMaxLevels);
    if (J < 1) return fail(SSA_ERR_INVALID_ARG, "J must be >= 1");
    if (!topk || (levels > 1 && !g_sum)) return fail(SSA_ERR_INVALID_ARG, "topk or g_sum is NULL");
    ssa_status st = build_single(p, shape, C, g, topk[0]);
    if (st != SSA_OK) return st;
    p.J = J;
    hl.levels = levels;
    hl.mask_words = 0;
    for (int l = 0; l < levels; ++l) {
        if (topk[l] < 0 || topk[l] > kMaxTopk)
            return fail(topk[l] < 0 ? SSA_ERR_INVALID_ARG : SSA_ERR_UNSUPPORTED,
                        "topk[%d] = %d outside [0, %d]", l, topk[l], kMaxTopk);
        hl.topk[l] = topk[l];
        hl.umax[l] = l == 0 ? p.M_max : hl.umax[l - 1] / J;
        hl.gs[l] = l == 0 ? g : g_sum[l - 1];
        if (hl.gs[l] < 1 || hl.gs[l] > 1024)
            return fail(SSA_ERR_INVALID_ARG, "g_sum[%d] = %d outside [1, 1024]", l - 1, hl.gs[l]);
        if ((long long)p.n_pairs * hl.umax[l] * hl.gs[l] >= (1ll << 31))
            return fail(SSA_ERR_UNSUPPORTED, "level %d rows too large for 32-bit indices", l + 1);
        hl.mask_words += (hl.umax[l] + 31) / 32;
    }
    return SSA_OK;
}

// Workspace of a t-level step: each level's candidate scores.
static size_t hier_layout(const ssa::Plan& p, const ssa::HierLevels& hl, size_t* off) {
    size_t o = 0;
    for (int l = 0; l < hl.levels; ++l) {
        off[l] = o;
        o += ((size_t)p.n_pairs * (hl.umax[l] > 0 ? hl.umax[l] : 1) * 4 + 255) / 256 * 256;
    }
    return o;
}

}  // namespace

extern "C" {

ssa_status ssa_workspace_size_hier(const ssa_shape* shape, int32_t C, int32_t g, int32_t J,
                                   int32_t levels, const int32_t* g_sum, const int32_t* topk,
                                   size_t* bytes) {
    if (!bytes) return fail(SSA_ERR_INVALID_ARG, "bytes is NULL");
    ssa::Plan p;
    ssa::HierLevels hl;
    ssa_status st = build_hier(p, hl, shape, C, g, J, levels, g_sum, topk);
    if (st != SSA_OK) return st;
    size_t off[ssa::kMaxLevels];
    *bytes = hier_layout(p, hl, off);
    return SSA_OK;
}

ssa_status ssa_decode_hier(const ssa_shape* shape, const void* q, const void* k_raw,
                           const void* v_raw, const void* k_gist, const void* v_gist,
                           const int32_t* seq_lens, int32_t C, int32_t g, int32_t J,
                           int32_t levels, const void* const* k_sum, const void* const* v_sum,
                           const int32_t* g_sum, const int32_t* topk, float* out,
                           int32_t* const* sel, void* ws, size_t ws_bytes, cudaStream_t stream) {
    ssa::Plan p;
    ssa::HierLevels hl;
    ssa_status st = build_hier(p, hl, shape, C, g, J, levels, g_sum, topk);
    if (st != SSA_OK) return st;
    st = check_tensors(p, {q, k_raw, v_raw, k_gist, v_gist, seq_lens, out});
    if (st != SSA_OK) return st;
    if (!sel || (levels > 1 && (!k_sum || !v_sum)))
        return fail(SSA_ERR_INVALID_ARG, "sel, k_sum or v_sum is NULL");
    for (int l = 0; l < levels; ++l) {
        if (topk[l] > 0 && !sel[l]) return fail(SSA_ERR_INVALID_ARG, "sel[%d] is NULL", l);
        hl.sel[l] = sel[l];
        if (l > 0) {
            // a level with no unit at this capacity has an empty summary tensor
            if (hl.umax[l] > 0 && (!k_sum[l - 1] || !v_sum[l - 1]))
                return fail(SSA_ERR_INVALID_ARG, "k_sum[%d] or v_sum[%d] is NULL", l - 1, l - 1);
            hl.k_sum[l] = k_sum[l - 1];
            hl.v_sum[l] = v_sum[l - 1];
        }
    }
    p.mode = ssa::kModeFull;
    p.q = q;
    p.k_raw = k_raw;
    p.v_raw = v_raw;
    p.k_gist = k_gist;
    p.v_gist = v_gist;
    p.seq_lens = seq_lens;
    p.out = out;
    size_t off[ssa::kMaxLevels];
    const size_t need = hier_layout(p, hl, off);
    void* own = nullptr;
    if (ws == nullptr) {
        if (ws_bytes != 0) return fail(SSA_ERR_WORKSPACE, "ws is NULL but ws_bytes != 0");
        cudaError_t e = cudaMallocAsync(&own, need, stream);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMallocAsync(workspace)");
        ws = own;
    } else if (ws_bytes < need) {
        return fail(SSA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, need);
    } else if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) {
        return fail(SSA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
    } else {
        note_ws_unknown(ws);
    }
    for (int l = 0; l < levels; ++l)
        hl.cscore[l] = reinterpret_cast<float*>(static_cast<char*>(ws) + off[l]);
    cudaError_t e = ssa::launch_hier(p, hl, stream);
    if (own) cudaFreeAsync(own, stream);
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    return SSA_OK;
}

ssa_status ssa_score_gists(const ssa_shape* shape, const void* q, const void* k_gist,
                           const int32_t* seq_lens, int32_t C, int32_t g, float* scores,
                           cudaStream_t stream) {
    ssa::Plan p;
    ssa_status st = build_single(p, shape, C, g, 0);
    if (st != SSA_OK) return st;
    st = check_tensors(p, {q, k_gist, seq_lens, scores});
    if (st != SSA_OK) return st;
    p.mode = ssa::kModeScoreOnly;
    p.q = q;
    p.k_gist = k_gist;
    p.k_raw = k_gist;  // unused by scoring; any valid map base
    p.v_raw = k_gist;
    p.v_gist = k_gist;
    p.seq_lens = seq_lens;
    p.scores = scores;
    cudaError_t e = fused_path(p) ? ssa::launch_fused(p, stream) : ssa::launch_generic(p, stream);
    if (e != cudaSuccess) return cuda_fail(e, "ssa_score_gists launch");
    return SSA_OK;
}

ssa_status ssa_topk_chunks(const ssa_shape* shape, const float* scores, const int32_t* seq_lens,
                           int32_t C, int32_t topk, int32_t* sel_idx, cudaStream_t stream) {
    ssa_status st = check_shape(shape, C, false);
    if (st != SSA_OK) return st;
    if (topk < 0) return fail(SSA_ERR_INVALID_ARG, "topk must be >= 0");
    if (!scores || !seq_lens || !sel_idx) return fail(SSA_ERR_INVALID_ARG, "NULL pointer");
    if (topk == 0) return SSA_OK;
    ssa::Plan p;
    fill_shape(p, shape, C, 1, topk);
    p.seq_lens = seq_lens;
    p.sel_idx = sel_idx;
    cudaError_t e = ssa::launch_topk(p, scores, stream);
    if (e != cudaSuccess) return cuda_fail(e, "ssa_topk_chunks launch");
    return SSA_OK;
}

ssa_status ssa_sparse_decode(const ssa_shape* shape, const void* q, const void* k_raw,
                             const void* v_raw, const void* k_gist, const void* v_gist,
                             const int32_t* seq_lens, int32_t C, int32_t g, int32_t topk,
                             const int32_t* sel_idx, float* out, void* ws, size_t ws_bytes,
                             cudaStream_t stream) {
    ssa::Plan p;
    ssa_status st = build_single(p, shape, C, g, topk);
    if (st != SSA_OK) return st;
    st = check_tensors(p, {q, k_raw, v_raw, k_gist, v_gist, seq_lens, out});
    if (st != SSA_OK) return st;
    if (topk > 0 && !sel_idx) return fail(SSA_ERR_INVALID_ARG, "sel_idx is NULL");
    p.mode = ssa::kModeAttnOnly;
    p.q = q;
    p.k_raw = k_raw;
    p.v_raw = v_raw;
    p.k_gist = k_gist;
    p.v_gist = v_gist;
    p.seq_lens = seq_lens;
    p.sel_idx = const_cast<int32_t*>(sel_idx);
    p.out = out;
    return run_with_ws(p, ws, ws_bytes, stream);
}

ssa_status ssa_workspace_size_variant(const ssa_shape* shape, int32_t C, int32_t g, int32_t topk,
                                      int32_t context, int32_t select, size_t* bytes) {
    if (!bytes) return fail(SSA_ERR_INVALID_ARG, "bytes is NULL");
    ssa::Plan p;
    ssa_status st = build_variant(p, shape, C, g, topk, context, select);
    if (st != SSA_OK) return st;
    size_t a, b;
    *bytes = variant_layout(p, &a, &b);
    // the group-max selection may run on the two-kernel pipeline
    if (ssa::pipe_prepare(p)) {
        const size_t pb = ssa::plan_bytes_any(p);
        if (pb > *bytes) *bytes = pb;
    }
    return SSA_OK;
}

ssa_status ssa_decode_variant(const ssa_shape* shape, const void* q, const void* k_raw,
                              const void* v_raw, const void* k_gist, const void* v_gist,
                              const int32_t* seq_lens, int32_t C, int32_t g, int32_t topk,
                              int32_t context, int32_t select, float* out, int32_t* sel_idx,
                              void* ws, size_t ws_bytes, cudaStream_t stream) {
    ssa::Plan p;
    ssa_status st = build_variant(p, shape, C, g, topk, context, select);
    if (st != SSA_OK) return st;
    st = check_tensors(p, {q, k_raw, v_raw, k_gist, v_gist, seq_lens, out});
    if (st != SSA_OK) return st;
    if (topk > 0 && !sel_idx) return fail(SSA_ERR_INVALID_ARG, "sel_idx is NULL");
    p.mode = ssa::kModeFull;
    p.q = q;
    p.k_raw = k_raw;
    p.v_raw = v_raw;
    p.k_gist = k_gist;
    p.v_gist = v_gist;
    p.seq_lens = seq_lens;
    p.sel_idx = sel_idx;
    p.out = out;
    // a pipeline shape: the two-kernel path, whose attention kernel applies
    // either context's keep predicate and either selection
    if (ssa::pipe_prepare(p)) return run_with_ws(p, ws, ws_bytes, stream);
    size_t so, ho;
    const size_t need = variant_layout(p, &so, &ho);
    void* own = nullptr;
    if (ws == nullptr) {
        if (ws_bytes != 0) return fail(SSA_ERR_WORKSPACE, "ws is NULL but ws_bytes != 0");
        cudaError_t e = cudaMallocAsync(&own, need, stream);
        if (e != cudaSuccess) return cuda_fail(e, "cudaMallocAsync(workspace)");
        ws = own;
    } else if (ws_bytes < need) {
        return fail(SSA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, need);
    } else if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) {
        return fail(SSA_ERR_WORKSPACE, "workspace must be 256-byte aligned");
    } else {
        note_ws_unknown(ws);  // the generic kernels leave it holding scores
    }
    char* base = static_cast<char*>(ws);
    p.scores = reinterpret_cast<float*>(base + so);
    p.head_sel = p.sel_mode ? reinterpret_cast<int32_t*>(base + ho) : nullptr;
    cudaError_t e = ssa::launch_generic(p, stream);
    if (own) cudaFreeAsync(own, stream);
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    return SSA_OK;
}

ssa_status ssa_decode(const ssa_shape* shape, const void* q, const void* k_raw, const void* v_raw,
                      const void* k_gist, const void* v_gist, const int32_t* seq_lens, int32_t C,
                      int32_t g, int32_t topk, float* out, int32_t* sel_idx, void* ws,
                      size_t ws_bytes, cudaStream_t stream) {
    ssa::Plan p;
    ssa_status st = build_single(p, shape, C, g, topk);
    if (st != SSA_OK) return st;
    st = check_tensors(p, {q, k_raw, v_raw, k_gist, v_gist, seq_lens, out});
    if (st != SSA_OK) return st;
    if (topk > 0 && !sel_idx) return fail(SSA_ERR_INVALID_ARG, "sel_idx is NULL");
    p.mode = ssa::kModeFull;
    p.q = q;
    p.k_raw = k_raw;
    p.v_raw = v_raw;
    p.k_gist = k_gist;
    p.v_gist = v_gist;
    p.seq_lens = seq_lens;
    p.sel_idx = sel_idx;
    p.out = out;
    return run_with_ws(p, ws, ws_bytes, stream);
}

// Device copies of a host-buffer step's small tensors, after the decode's
// own workspace: q, seq_lens, out, sel_idx (256-byte aligned).
static size_t host_staging(const ssa::Plan& p, size_t base, size_t* off) {
    size_t o = (base + 255) / 256 * 256;
    auto take = [&](size_t bytes) {
        size_t at = o;
        o += (bytes + 255) / 256 * 256;
        return at;
    };
    const size_t e = p.dtype == SSA_BF16 ? 2 : 4;
    off[0] = take((size_t)p.B * p.Hq * p.d * e);
    off[1] = take((size_t)p.B * 4);
    off[2] = take((size_t)p.B * p.Hq * p.d * 4);
    off[3] = take((size_t)p.n_pairs * (p.topk > 0 ? p.topk : 1) * 4);
    return o;
}

ssa_status ssa_workspace_size_host(const ssa_shape* shape, int32_t C, int32_t g, int32_t topk,
                                   size_t* bytes) {
    if (!bytes) return fail(SSA_ERR_INVALID_ARG, "bytes is NULL");
    ssa::Plan p;
    ssa_status st = build_single(p, shape, C, g, topk);
    if (st != SSA_OK) return st;
    size_t off[4];
    *bytes = host_staging(p, ssa::plan_bytes_any(p), off);
    return SSA_OK;
}

ssa_status ssa_decode_host(const ssa_shape* shape, const void* q_host, const void* k_raw,
                           const void* v_raw, const void* k_gist, const void* v_gist,
                           const int32_t* seq_lens_host, int32_t C, int32_t g, int32_t topk,
                           float* out_host, int32_t* sel_idx_host, void* ws, size_t ws_bytes,
                           cudaStream_t stream) {
    ssa::Plan p;
    ssa_status st = build_single(p, shape, C, g, topk);
    if (st != SSA_OK) return st;
    if (!q_host || !seq_lens_host || !out_host || (topk > 0 && !sel_idx_host))
        return fail(SSA_ERR_INVALID_ARG, "a host buffer is NULL");
    if (!ws) return fail(SSA_ERR_WORKSPACE, "ssa_decode_host needs a workspace");
    const size_t base = ssa::plan_bytes_any(p);
    size_t off[4];
    const size_t need = host_staging(p, base, off);
    if (ws_bytes < need)
        return fail(SSA_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes, need);
    char* w = static_cast<char*>(ws);
    const size_t e = p.dtype == SSA_BF16 ? 2 : 4;
    const size_t qb = (size_t)p.B * p.Hq * p.d * e, ob = (size_t)p.B * p.Hq * p.d * 4;
    const size_t sb = (size_t)p.n_pairs * topk * 4;
    cudaError_t ce = cudaMemcpyAsync(w + off[0], q_host, qb, cudaMemcpyHostToDevice, stream);
    if (ce == cudaSuccess)
        ce = cudaMemcpyAsync(w + off[1], seq_lens_host, (size_t)p.B * 4, cudaMemcpyHostToDevice,
                             stream);
    if (ce != cudaSuccess) return cuda_fail(ce, "cudaMemcpyAsync(host to device)");
    st = ssa_decode(shape, w + off[0], k_raw, v_raw, k_gist, v_gist,
                    reinterpret_cast<const int32_t*>(w + off[1]), C, g, topk,
                    reinterpret_cast<float*>(w + off[2]), reinterpret_cast<int32_t*>(w + off[3]),
                    ws, base, stream);
    if (st != SSA_OK) return st;
    ce = cudaMemcpyAsync(out_host, w + off[2], ob, cudaMemcpyDeviceToHost, stream);
    if (ce == cudaSuccess && sb > 0)
        ce = cudaMemcpyAsync(sel_idx_host, w + off[3], sb, cudaMemcpyDeviceToHost, stream);
    if (ce != cudaSuccess) return cuda_fail(ce, "cudaMemcpyAsync(device to host)");
    return SSA_OK;
}

ssa_status ssa_decode_noalloc(const ssa_shape* shape, const void* q, const void* k_raw,
                              const void* v_raw, const void* k_gist, const void* v_gist,
                              const int32_t* seq_lens, int32_t C, int32_t g, int32_t topk,
                              float* out, int32_t* sel_idx, cudaStream_t stream) {
    ssa::Plan p;
    ssa_status st = build_single(p, shape, C, g, topk);
    if (st != SSA_OK) return st;
    st = check_tensors(p, {q, k_raw, v_raw, k_gist, v_gist, seq_lens, out});
    if (st != SSA_OK) return st;
    if (topk > 0 && !sel_idx) return fail(SSA_ERR_INVALID_ARG, "sel_idx is NULL");
    ssa::pipe_prepare(p);
    const ssa::WsLayout L = ssa::plan_layout(p);
    if (L.total > ssa::kBuiltinWsBytes)
        return fail(SSA_ERR_WORKSPACE,
                    "ssa_decode_noalloc: these sizes need %zu bytes of scratch, the built-in "
                    "area holds %zu; use ssa_decode with a workspace",
                    L.total, ssa::kBuiltinWsBytes);
    void* ws = nullptr;
    cudaError_t e = ssa::builtin_workspace(&ws);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(built-in scratch)");
    p.mode = ssa::kModeFull;
    p.q = q;
    p.k_raw = k_raw;
    p.v_raw = v_raw;
    p.k_gist = k_gist;
    p.v_gist = v_gist;
    p.seq_lens = seq_lens;
    p.sel_idx = sel_idx;
    p.out = out;
    attach_ws(p, ws);
    if (L.pipe) {
        // the pipeline's words carry the epoch of the launch that wrote
        // them: the area is cleared only when another path used it last
        e = prepare_ws_pipe(ws, L.total, stream);
    } else {
        // the area keeps whatever the previous call left: clear the part
        // that must start at zero (control words and scores), stream-ordered
        note_ws_unknown(ws);
        e = cudaMemsetAsync(ws, 0, L.partials, stream);
    }
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(built-in scratch)");
    e = launch_plan(p, stream);
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    return SSA_OK;
}

ssa_status ssa_decode_h2(const ssa_shape* shape, const void* q, const void* k_raw,
                         const void* v_raw, const void* k_gist, const void* v_gist,
                         const void* k_meta, const void* v_meta, const int32_t* seq_lens,
                         int32_t C, int32_t g, int32_t J, int32_t gm, int32_t topk_super,
                         int32_t topk_chunk, float* out, int32_t* sel_super, int32_t* sel_idx,
                         void* ws, size_t ws_bytes, cudaStream_t stream) {
    ssa::Plan p;
    ssa_status st = build_h2(p, shape, C, g, J, gm, topk_super, topk_chunk);
    if (st != SSA_OK) return st;
    st = check_tensors(p, {q, k_raw, v_raw, k_gist, v_gist, k_meta, v_meta, seq_lens, out});
    if (st != SSA_OK) return st;
    if ((topk_super > 0 && !sel_super) || (topk_chunk > 0 && !sel_idx))
        return fail(SSA_ERR_INVALID_ARG, "selection output is NULL");
    p.mode = ssa::kModeFull;
    p.q = q;
    p.k_raw = k_raw;
    p.v_raw = v_raw;
    p.k_gist = k_gist;
    p.v_gist = v_gist;
    p.k_meta = k_meta;
    p.v_meta = v_meta;
    p.seq_lens = seq_lens;
    p.sel_idx = sel_idx;
    p.sel_super = sel_super;
    p.out = out;
    return run_with_ws(p, ws, ws_bytes, stream);
}

ssa_status ssa_decode_path(const ssa_shape* shape, int32_t C, int32_t g, int32_t topk,
                           int32_t* path) {
    if (!path) return fail(SSA_ERR_INVALID_ARG, "path is NULL");
    ssa::Plan p;
    ssa_status st = build_single(p, shape, C, g, topk);
    if (st != SSA_OK) return st;
    p.mode = ssa::kModeFull;
    if (ssa::pipe_prepare(p))
        *path = SSA_PATH_PIPELINE;
    else
        *path = fused_path(p) ? SSA_PATH_FUSED : SSA_PATH_GENERIC;
    return SSA_OK;
}

ssa_status ssa_workspace_size(const ssa_shape* shape, int32_t C, int32_t g, int32_t topk,
                              size_t* bytes) {
    if (!bytes) return fail(SSA_ERR_INVALID_ARG, "bytes is NULL");
    ssa::Plan p;
    ssa_status st = build_single(p, shape, C, g, topk);
    if (st != SSA_OK) return st;
    *bytes = ssa::plan_bytes_any(p);
    return SSA_OK;
}

ssa_status ssa_workspace_size_h2(const ssa_shape* shape, int32_t C, int32_t g, int32_t J,
                                 int32_t gm, int32_t topk_super, int32_t topk_chunk,
                                 size_t* bytes) {
    if (!bytes) return fail(SSA_ERR_INVALID_ARG, "bytes is NULL");
    ssa::Plan p;
    ssa_status st = build_h2(p, shape, C, g, J, gm, topk_super, topk_chunk);
    if (st != SSA_OK) return st;
    *bytes = ssa::plan_layout(p).total;
    return SSA_OK;
}

ssa_status ssa_workspace_init(void* ws, size_t ws_bytes, cudaStream_t stream) {
    if (!ws) return fail(SSA_ERR_INVALID_ARG, "ws is NULL");
    cudaError_t e = cudaMemsetAsync(ws, 0, ws_bytes, stream);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(workspace)");
    note_ws_zeroed(ws, ws_bytes);
    return SSA_OK;
}

ssa_status ssa_get_device_status(int32_t* host_code, cudaStream_t stream) {
    if (!host_code) return fail(SSA_ERR_INVALID_ARG, "host_code is NULL");
    int v = 0;
    cudaError_t e = ssa::read_device_status(&v, stream);
    if (e != cudaSuccess) return cuda_fail(e, "reading the device status");
    if (v == SSA_ERR_DEVICE_TIMEOUT) note_timeout();
    *host_code = v;
    return SSA_OK;
}

void ssa_set_wait_limit(int64_t ns) { g_wait_limit.store(ns > 0 ? ns : 0); }

void ssa_set_debug_flags(int32_t flags) { g_debug.store(flags); }

void ssa_set_tuning(int32_t max_blocks, int32_t rows_per_score_item) {
    g_max_blocks.store(max_blocks > 0 ? max_blocks : 0);
    g_rows_per_score.store(rows_per_score_item > 0 ? rows_per_score_item : 0);
}

const char* ssa_status_string(ssa_status s) {
    switch (s) {
        case SSA_OK: return "ok";
        case SSA_ERR_INVALID_ARG: return "invalid argument";
        case SSA_ERR_UNSUPPORTED: return "unsupported configuration";
        case SSA_ERR_WORKSPACE: return "workspace missing or too small";
        case SSA_ERR_CUDA: return "CUDA error";
        case SSA_ERR_DEVICE_STATUS: return "device reported bad seq_lens or sel_idx";
        case SSA_ERR_DEVICE_TIMEOUT: return "a bounded device wait timed out";
    }
    return "unknown status";
}

const char* ssa_last_error(void) { return g_err.c_str(); }

int32_t ssa_version(void) { return 1; }

#ifdef SSA_TRACE
// Trace builds only: device buffer of blocks x cap x 16-byte events.
__attribute__((visibility("default"))) void ssa_set_trace(void* buf, int32_t cap) {
    g_trace.store(buf);
    g_trace_cap.store(cap);
}
#endif

}  // extern "C"
