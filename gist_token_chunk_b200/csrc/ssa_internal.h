// ssa_internal.h -- host-side plan and launcher interface between the C ABI
// (ssa_api.cpp) and the kernels (ssa_kernels.cu).  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime_api.h>
#include <stddef.h>
#include <stdint.h>

namespace ssa {

enum Mode : int { kModeFull = 0, kModeScoreOnly = 1, kModeAttnOnly = 2 };

// Upper bound on the fused kernel's grid (sizes the partials area).
constexpr int kFusedMaxGrid = 1024;
// Sequences the fused kernel's in-block plan holds.
constexpr int kFusedMaxB = 128;

// Everything a launch needs, resolved on the host.  Pointers are device
// pointers.  Sizes follow the public header's notation.
struct Plan {
    int mode = kModeFull;
    int h2 = 0;            // two-level (gist-of-gist) step
    int dtype = 0;         // 0 bf16, 1 fp32
    int B = 0, Hq = 0, Hkv = 0, G = 0, d = 0, n_max = 0, C = 0, g = 0, M_max = 0;
    int topk = 0;          // single level: topk; two level: topk_chunk
    int J = 0, gm = 0, S_max = 0, topk_super = 0, Mc_max = 0;
    int n_pairs = 0;

    // fused kernel: blocks (0: every co-resident block), summary rows per
    // scoring sub-item, control words per pair (counters + published selection)
    int grid_cap = 0;
    int score_rows = 1024;
    int pair_ints = 0;
    // ring stages of this launch; logits = 1: the scoring phase keeps the
    // per-row logits of its gist rows in shared memory ([head][logit_stride])
    // and the gist phase streams only the values of the same rows
    int stages = 0;
    int logits = 0;
    int logit_stride = 0;
    int mask_words = 0, smask_words = 0;
    int g_shift = -1;      // log2(g) when g is a power of two, else -1
    // topk (and topk_super) <= 32, single level in logits mode or two
    // level: every scoring segment publishes its 32 best slots (descending
    // composites key << 32 | ~slot) and the top-k merges those lists
    // instead of ranking every score
    int fastsel = 0;

    const void* q = nullptr;
    const void* k_raw = nullptr;
    const void* v_raw = nullptr;
    const void* k_gist = nullptr;
    const void* v_gist = nullptr;
    const void* k_meta = nullptr;
    const void* v_meta = nullptr;
    const int32_t* seq_lens = nullptr;
    float* scores = nullptr;        // [P, M_max]
    float* super_scores = nullptr;  // [P, S_max]
    float* cand_scores = nullptr;   // [P, Mc_max]
    int32_t* sel_idx = nullptr;     // [P, topk]
    int32_t* sel_super = nullptr;   // [P, topk_super]
    uint32_t* chunk_mask = nullptr; // [P, mask_words]
    uint32_t* super_mask = nullptr; // [P, smask_words]
    float* partials = nullptr;      // [3, kFusedMaxGrid + P, G, d + 2]
    unsigned long long* cands = nullptr;  // [levels, kFusedMaxGrid + P, 32] segment lists
    float* out = nullptr;           // [B, Hq, d]
    int* ctrl = nullptr;            // control words
    // two-kernel pipeline (ssa_pipe.cuh; pp_w3 > 0 when a call takes it):
    // workspace areas whose words carry the launch's epoch
    unsigned* st_hdr = nullptr;               // [0] epoch of the last launch, [1] blocks done
    unsigned long long* st_sel = nullptr;     // [P, st_sel_stride] epoch << 32 | chunk
    char* st_part = nullptr;                  // [2, G, st_part_slots] records of st_slot_bytes
    int st_sel_stride = 0, st_part_slots = 0, st_slot_bytes = 0;
    int st_rcap = 0;                          // kept-logit rows per scoring worker warp
    float* pp_scores = nullptr;               // [P, M_max rounded up to 8] chunk scores
    float* pp_logits = nullptr;               // [P * M_max * g + 64, logit stride] kept logits
    int pp_w1 = 0, pp_w3 = 0;                 // worker warps per block: scoring, attention
    // context / selection readings (ssa_decode_variant; 0, 0 everywhere else):
    // ctx_mode 1 = selected gists + selected raw + tail; sel_mode 1 = per-head
    // top-k, union over the group.  sel_stride = entries per pair in sel_idx.
    int ctx_mode = 0, sel_mode = 0, sel_stride = 0;
    int32_t* head_sel = nullptr;    // sel_mode 1: [B, Hq, topk] per-head selections
    long long wait_limit = 0;       // ns bound of every device-side wait
    int debug_flags = 0;
    // timeline trace (only written by builds compiled with SSA_TRACE)
    uint4* trace = nullptr;         // events: pipeline [gridDim.x][16][trace_cap], fused [gridDim.x][trace_cap]
    int trace_cap = 0;
};

// Coarse-to-fine selection over t levels (ssa_decode_hier): level 0 is the
// chunks (gists), level l >= 1 groups J level-(l-1) units and has gs[l]
// summary tokens in k_sum[l], v_sum[l] [B,Hkv,umax[l],gs[l],d].  cscore[l]
// holds each pair's candidate scores (umax[l] per pair), sel[l] the kept
// units [B,Hkv,topk[l]].
constexpr int kMaxLevels = 8;
struct HierLevels {
    int levels = 0;
    const void* k_sum[kMaxLevels] = {};
    const void* v_sum[kMaxLevels] = {};
    int gs[kMaxLevels] = {};
    int topk[kMaxLevels] = {};
    int umax[kMaxLevels] = {};
    float* cscore[kMaxLevels] = {};
    int32_t* sel[kMaxLevels] = {};
    int mask_words = 0;  // sum over levels of ceil(umax / 32)
};
cudaError_t launch_hier(const Plan& p, const HierLevels& hl, cudaStream_t stream);

// Workspace layout for a plan (byte offsets from the workspace base).
struct WsLayout {
    size_t ctrl = 0, scores = 0, super_scores = 0, cand_scores = 0, chunk_mask = 0,
           super_mask = 0, cands = 0, partials = 0, total = 0;
    // pipeline (pipe = true): epoch header, chunk scores, kept logits,
    // selections, partials
    bool pipe = false;
    size_t st_hdr = 0, st_sel = 0, st_part = 0;
    size_t pp_scores = 0, pp_logits = 0;
};

// Fills the decomposition fields of `p` (needs shapes) and the layout.  The
// layout is the pipeline's when the plan takes it, else the fused or
// generic path's.
void plan_decompose(Plan& p);
WsLayout plan_layout(const Plan& p);
// Bytes that cover every path a single-level call of these sizes can take.
size_t plan_bytes_any(const Plan& p);
int ctrl_words(const Plan& p);

// Segment candidate lists of the fused single-level top-k (entries per list).
constexpr int kSegList = 32;
// Whether a plan's layout holds the segment candidate lists.
bool seg_lists(const Plan& p);

// Two-kernel pipeline (single level, bf16, d = 64, G <= 8, topk <= 128):
// fills the pp_* and st_* sizes of `p` and returns true when the call takes
// it on the current device.
bool pipe_prepare(Plan& p);
cudaError_t launch_pipe(const Plan& p, cudaStream_t stream);
// Workspace bytes of the pipeline's areas for a prepared plan.
void pipe_ws_sizes(const Plan& p, size_t* hdr, size_t* scores, size_t* logits, size_t* sel,
                   size_t* part);

// Fast fused path: bf16, d in {64, 128}.  Returns a cudaError_t.
cudaError_t launch_fused(const Plan& p, cudaStream_t stream);
// Generic path: any d <= 256, bf16 or fp32, separate simple kernels.
cudaError_t launch_generic(const Plan& p, cudaStream_t stream);
// Standalone top-k over user scores (ssa_topk_chunks).
cudaError_t launch_topk(const Plan& p, const float* scores, cudaStream_t stream);

cudaError_t read_device_status(int* code, cudaStream_t stream);

// Built-in scratch of ssa_decode_noalloc: a fixed device array in the
// library's device code (no allocation).  Its device address for the current
// device, looked up once per device.
constexpr size_t kBuiltinWsBytes = size_t(16) << 20;
cudaError_t builtin_workspace(void** ptr);

// Query the SM count of the current device (cached per device).
int sm_count();

}  // namespace ssa
