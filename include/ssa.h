/*
 * ssa.h -- C ABI of libssa: the decode-time hot path of Simplified Sparse
 * Attention with gist tokens, for NVIDIA B200 (sm_100a).
 *
 * Method: "Simplified Sparse Attention via Gist Tokens" (Mao, Li, Fox).
 *   sec. 3.2  each chunk of C raw tokens carries g gist tokens whose keys
 *             score the chunk's relevance to the current query;
 *   sec. 3.3  the top-k chunks are unfolded back to their raw tokens and one
 *             softmax attention runs over the resulting hybrid context;
 *   sec. 3.5, App. B.2  gist-of-gist: meta-gists summarise J chunks and the
 *             selection runs coarse to fine;
 *   sec. 3.6  a decode step reads the chosen keys and a per-chunk index
 *             linear in the context, never the whole cache, and merges
 *             split partial attentions at the end.
 * Where the pages leave a step open this library fixes it as follows:
 *   - chunk score s[b,j,m] = max over the query heads h of KV head j and the
 *     chunk's g gist tokens t of  q[b,h] . k_gist[b,j,m,t] / sqrt(d);
 *   - one selection per (sequence, KV head), shared by its query heads;
 *     ties go to the lower chunk index; a NaN logit never wins a score
 *     maximum, and NaN scores given to ssa_topk_chunks rank as -inf;
 *   - the attended context of (b, j) is: the gist K/V of every UNselected
 *     complete chunk, the raw K/V of every token of the selected chunks, and
 *     the raw K/V of the tail tokens M_b*C .. n_b-1 (selected chunks' own
 *     gists are not attended);
 *   - seq_lens[b] = n_b counts every cached raw token (the current one
 *     included); M_b = floor(n_b / C) chunks are complete.
 * ssa_decode_variant offers the pages' other readings of the context and of
 * the selection, and ssa_decode_hier the coarse-to-fine selection over more
 * than two levels.  ssa_adaptive_topk gives App. A's selection budget, and
 * ssa_prefill_plan / ssa_prefill the block-sparse prefill under the gist
 * mask (sec. 3.1, 3.6).
 *
 * Notation and layouts (row-major, contiguous, all device memory unless said):
 *   B batch, Hq query heads, Hkv KV heads, G = Hq/Hkv, query head h reads KV
 *   head h / G; d head dim; n_max cache capacity (a multiple of C);
 *   M_max = n_max / C.
 *     q       [B, Hq, d]                 bf16 or fp32 (shape->dtype)
 *     k_raw   [B, Hkv, n_max, d]         same dtype
 *     v_raw   [B, Hkv, n_max, d]
 *     k_gist  [B, Hkv, M_max, g, d]
 *     v_gist  [B, Hkv, M_max, g, d]
 *     seq_lens int32 [B]                 (device)
 *     scores  fp32 [B, Hkv, M_max]
 *     sel_idx int32 [B, Hkv, topk]       selected chunks ascending, -1 padded
 *     out     fp32 [B, Hq, d]
 *   Two-level variant adds J (chunks per superchunk), gm (meta-gists per
 *   superchunk), S_max = M_max / J and
 *     k_meta, v_meta [B, Hkv, S_max, gm, d], sel_super int32 [B, Hkv, topk_super].
 *
 * Conventions for every call:
 *   - The caller owns every buffer; the library neither frees nor keeps any
 *     pointer beyond the call.  Calls are asynchronous on `stream` and never
 *     synchronise the host (except ssa_get_device_status).
 *   - Host-checkable errors (null pointer, topk < 0, C < 1, g < 1, n_max not a
 *     multiple of C, Hq not a multiple of Hkv, Hq/Hkv > 16, d not in
 *     {64, 128} for bf16 or not in [1, 256] for fp32, unknown dtype, a
 *     workspace that is too small) return an error code with nothing enqueued.
 *   - Errors only the device can see (n_b outside [1, n_max]; a sel_idx given
 *     to ssa_sparse_decode that is out of range, not strictly ascending, or not
 *     -1 padded) set the library's device status word and zero that
 *     sequence's outputs; read it with ssa_get_device_status.
 *   - CUDA launch errors return SSA_ERR_CUDA; ssa_last_error() gives the text.
 *     No C++ exception crosses this boundary.
 *   - topk > M_b selects every complete chunk; topk = 0 selects none.
 *
 * Workspace: the decode calls need device scratch of their
 * ssa_workspace_size*() bytes.  Pass ws = NULL, ws_bytes = 0 to let the
 * library allocate it stream-ordered (cudaMallocAsync) for that one call.  A
 * caller-owned workspace must be zeroed once with ssa_workspace_init() (or
 * cudaMemset 0) before its first use.  Every call leaves it reusable by later
 * calls on the same stream, for any sizes that fit, without re-initialising:
 * the two-kernel pipeline's words carry the launch's epoch, and the fused
 * kernel clears the state it used (control words, score scratch, the scoring
 * segments' candidate lists); when a call lays the workspace out differently
 * from its previous call, the library zeroes the part it needs stream-ordered
 * first.  After a call that reported SSA_ERR_DEVICE_TIMEOUT, initialise it
 * again.  Two calls that share a workspace must not run concurrently.
 */
#ifndef SSA_H_
#define SSA_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define SSA_API __attribute__((visibility("default")))
#else
#define SSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    SSA_OK = 0,
    SSA_ERR_INVALID_ARG = 1,   /* bad pointer, size or parameter            */
    SSA_ERR_UNSUPPORTED = 2,   /* valid but outside what the kernels handle */
    SSA_ERR_WORKSPACE = 3,     /* workspace missing or too small            */
    SSA_ERR_CUDA = 4,          /* a CUDA runtime call failed                */
    SSA_ERR_DEVICE_STATUS = 5, /* device saw bad seq_lens or sel_idx        */
    SSA_ERR_DEVICE_TIMEOUT = 6 /* a bounded device wait gave up             */
} ssa_status;

typedef enum { SSA_BF16 = 0, SSA_FP32 = 1 } ssa_dtype;

/* Shapes of one call.  dtype is an ssa_dtype. */
typedef struct {
    int32_t B, Hq, Hkv, d, n_max;
    int32_t dtype;
} ssa_shape;

/*
 * ssa_score_gists -- chunk relevance scores (sec. 3.2).
 *   scores[b,j,m] = max_{h in group j, t < g} q[b,h] . k_gist[b,j,m,t] / sqrt(d)
 *   for m < M_b, and -inf for M_b <= m < M_max.  Reads gist keys only.
 * In: q, k_gist, seq_lens.  Out: scores fp32 [B,Hkv,M_max].
 */
SSA_API ssa_status ssa_score_gists(const ssa_shape* shape, const void* q, const void* k_gist,
                           const int32_t* seq_lens, int32_t C, int32_t g, float* scores,
                           cudaStream_t stream);

/*
 * ssa_topk_chunks -- top-k chunk selection (sec. 3.3).
 * Per (b, j): the k_b = min(topk, M_b) chunks with the largest scores among
 * m < M_b, ties to the lower index, written ascending into sel_idx[b,j,0..k_b)
 * and -1 in sel_idx[b,j,k_b..topk).  Deterministic.
 * In: scores fp32 [B,Hkv,M_max], seq_lens.  Out: sel_idx int32 [B,Hkv,topk].
 * shape->d and shape->dtype are not used.
 */
SSA_API ssa_status ssa_topk_chunks(const ssa_shape* shape, const float* scores,
                           const int32_t* seq_lens, int32_t C, int32_t topk, int32_t* sel_idx,
                           cudaStream_t stream);

/*
 * ssa_sparse_decode -- hybrid attention over the unfolded context for a
 * GIVEN selection (sec. 3.3 attention, sec. 3.6 split partial passes plus
 * combination).  sel_idx[b,j,:] must hold strictly ascending chunk indices in
 * [0, M_b) followed only by -1 (at most topk entries); anything else sets the
 * device status and zeroes out[b,...].
 * Out: out fp32 [B,Hq,d].  Needs ssa_workspace_size() bytes of workspace.
 */
SSA_API ssa_status ssa_sparse_decode(const ssa_shape* shape, const void* q, const void* k_raw,
                             const void* v_raw, const void* k_gist, const void* v_gist,
                             const int32_t* seq_lens, int32_t C, int32_t g, int32_t topk,
                             const int32_t* sel_idx, float* out, void* ws, size_t ws_bytes,
                             cudaStream_t stream);

/*
 * ssa_decode -- the whole decode step: score, top-k, hybrid attention,
 * combination, in one stream-ordered call (sec. 3.2, 3.3, 3.6).
 * Out: out fp32 [B,Hq,d] and the selection sel_idx int32 [B,Hkv,topk].
 * Needs ssa_workspace_size() bytes of workspace.
 */
SSA_API ssa_status ssa_decode(const ssa_shape* shape, const void* q, const void* k_raw,
                      const void* v_raw, const void* k_gist, const void* v_gist,
                      const int32_t* seq_lens, int32_t C, int32_t g, int32_t topk, float* out,
                      int32_t* sel_idx, void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * ssa_decode_host -- ssa_decode with the step's small tensors in HOST memory:
 * q_host [B,Hq,d] (the shape's dtype) and seq_lens_host [B] are copied to the
 * device, the step runs, and out_host fp32 [B,Hq,d] and sel_idx_host int32
 * [B,Hkv,topk] are copied back, all stream-ordered on `stream` (one
 * cudaMemcpyAsync per tensor).  The KV cache (k_raw, v_raw, k_gist, v_gist)
 * is device memory, as in ssa_decode.  The device copies live in the
 * workspace, which must hold ssa_workspace_size_host() bytes (ws must not be
 * NULL).  Host buffers should be page-locked for the copies to be
 * asynchronous; pageable ones work, but their copies block the host.  The
 * host outputs are complete once the stream has passed this call
 * (synchronize, or wait on an event recorded after it).  A library
 * convenience for callers whose per-step tensors live on the host; the pages
 * have no counterpart.
 */
SSA_API ssa_status ssa_decode_host(const ssa_shape* shape, const void* q_host, const void* k_raw,
                                   const void* v_raw, const void* k_gist, const void* v_gist,
                                   const int32_t* seq_lens_host, int32_t C, int32_t g,
                                   int32_t topk, float* out_host, int32_t* sel_idx_host, void* ws,
                                   size_t ws_bytes, cudaStream_t stream);

/* Workspace bytes needed by ssa_decode_host for these sizes. */
SSA_API ssa_status ssa_workspace_size_host(const ssa_shape* shape, int32_t C, int32_t g,
                                           int32_t topk, size_t* bytes);

/*
 * ssa_decode_noalloc -- ssa_decode for callers that cannot allocate device
 * memory and cannot pass a workspace: for example an engine that reserves all
 * device memory for itself before serving, or a plugin interface that hands
 * over only the tensors.  The pages have no counterpart; this is a library
 * convenience, not a step of the method.
 * Same arguments and results as ssa_decode without ws / ws_bytes.  It
 * allocates nothing: its scratch is a fixed 16 MiB area inside the library's
 * device code (enough for the 32K, 128K and 512K batch workloads of this
 * library's tests; larger sizes return SSA_ERR_WORKSPACE with the byte count
 * in ssa_last_error(); use ssa_decode with a workspace then).
 * The first call on each device, with that device current, looks up the
 * area's device address (a CUDA runtime query); make that first call before
 * any stream capture.  Before the kernels run, a call clears what must start
 * at zero (a stream-ordered memset): on the two-kernel path only when the
 * area was last used by another path, or by a call that used less of it (its
 * words carry the launch's epoch and need no clearing), on the other paths
 * the control and score part every time.  All calls share the one area and it
 * keeps the last call's contents, so two calls whose work overlaps on the GPU
 * (different streams without ordering, several host threads) race on it:
 * order them on one stream.
 */
SSA_API ssa_status ssa_decode_noalloc(const ssa_shape* shape, const void* q, const void* k_raw,
                              const void* v_raw, const void* k_gist, const void* v_gist,
                              const int32_t* seq_lens, int32_t C, int32_t g, int32_t topk,
                              float* out, int32_t* sel_idx, cudaStream_t stream);

/*
 * ssa_decode_h2 -- two-level (gist-of-gist) decode step (sec. 3.5, App. B.2).
 * Level 2 scores the S_b = floor(M_b / J) complete superchunks with their gm
 * meta-gist keys (same max-over-heads-and-tokens score) and keeps the top
 * topk_super (ties to the lower index) -> sel_super.  The candidates are the J
 * chunks of each kept superchunk plus the remainder chunks S_b*J .. M_b-1;
 * level 1 scores the candidates with their gist keys and keeps the top
 * topk_chunk -> sel_idx.  The attended context is: meta-gist K/V of every
 * unselected complete superchunk, gist K/V of every unselected candidate
 * chunk, raw K/V of the selected chunks, and the raw tail.
 * Out: out, sel_super [B,Hkv,topk_super], sel_idx [B,Hkv,topk_chunk].
 * Needs ssa_workspace_size_h2() bytes of workspace.
 */
SSA_API ssa_status ssa_decode_h2(const ssa_shape* shape, const void* q, const void* k_raw,
                         const void* v_raw, const void* k_gist, const void* v_gist,
                         const void* k_meta, const void* v_meta, const int32_t* seq_lens,
                         int32_t C, int32_t g, int32_t J, int32_t gm, int32_t topk_super,
                         int32_t topk_chunk, float* out, int32_t* sel_super, int32_t* sel_idx,
                         void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * ssa_decode_variant -- the decode step under the pages' other readings of
 * the context and of the selection (the default readings are those of
 * ssa_decode):
 *   context SSA_CONTEXT_UNSELECTED_GISTS: gist K/V of the unselected complete
 *     chunks + raw K/V of the selected chunks + raw tail (ssa_decode);
 *   context SSA_CONTEXT_SELECTED_ONLY: gist K/V and raw K/V of the selected
 *     chunks + raw tail; unselected chunks contribute nothing (sec. 3.3
 *     read literally: a selected chunk brings its gists and its raw tokens,
 *     the other chunks are left out; |X| = k (C + g) + T);
 *   select SSA_SELECT_GROUP_MAX: one top-k per KV head over the max of its
 *     group's query heads (ssa_decode);
 *   select SSA_SELECT_HEAD_UNION: every query head scores the chunks with its
 *     own query (max over the chunk's g gists of q_h.k / sqrt(d)) and keeps
 *     its own top-k (ties to the lower index); the KV head's selection is the
 *     union over its group, and all heads of the group attend over the
 *     context it defines (App. A: the heads choose their chunks separately
 *     and the group unfolds their union).
 * Out: out fp32 [B,Hq,d]; sel_idx int32 [B,Hkv,cap], the selection ascending
 * and -1 padded, cap = topk (group max) or G * topk (head union).
 * On a shape the two-kernel pipeline takes (see ssa_decode_path) both
 * readings run there, when G * topk <= 1024; everything else runs on the
 * library's portable kernels (every dtype and head dim the library accepts).
 * Needs ssa_workspace_size_variant() bytes of workspace (ws = NULL:
 * allocated stream-ordered).  Errors as ssa_decode; an unknown context or
 * select value -> SSA_ERR_INVALID_ARG.
 */
#define SSA_CONTEXT_UNSELECTED_GISTS 0
#define SSA_CONTEXT_SELECTED_ONLY 1
#define SSA_SELECT_GROUP_MAX 0
#define SSA_SELECT_HEAD_UNION 1
SSA_API ssa_status ssa_decode_variant(const ssa_shape* shape, const void* q, const void* k_raw,
                                      const void* v_raw, const void* k_gist, const void* v_gist,
                                      const int32_t* seq_lens, int32_t C, int32_t g, int32_t topk,
                                      int32_t context, int32_t select, float* out,
                                      int32_t* sel_idx, void* ws, size_t ws_bytes,
                                      cudaStream_t stream);

/* Workspace bytes needed by ssa_decode_variant for these sizes and readings. */
SSA_API ssa_status ssa_workspace_size_variant(const ssa_shape* shape, int32_t C, int32_t g,
                                              int32_t topk, int32_t context, int32_t select,
                                              size_t* bytes);

/*
 * ssa_decode_hier -- coarse-to-fine selection over t = levels levels (sec.
 * 3.5: more levels of summaries as the context grows; App. B.2,
 * t = ceil(log_J M)), the two-level reading of ssa_decode_h2 applied
 * level by level.  Level 1 is the chunks with their g gists (k_gist,
 * v_gist).  A level-l unit (l >= 2) groups J level-(l-1) units and has
 * g_sum[l-2] summary tokens in k_sum[l-2], v_sum[l-2], bf16/fp32 like the
 * rest, laid out [B,Hkv,Umax(l),g_sum[l-2],d] with Umax(l) = (n_max / C) /
 * J^(l-1) (integer divisions, level by level).  A sequence has U_1 = M_b
 * complete chunks and U_l = floor(U_{l-1} / J) complete level-l units.
 * Selection, from the top: level t's candidates are its U_t units; level
 * l < t's are the J children of each unit kept at level l+1 (ascending),
 * then the remainder units U_{l+1} J .. U_l - 1, which lie in no complete
 * parent; each level keeps its topk[l-1] best candidates (score = max over
 * the group's query heads and the unit's summary tokens of q.k / sqrt(d),
 * ties to the lower index) into sel[l-1] [B,Hkv,topk[l-1]], ascending, -1
 * padded.  Context: the summary tokens of every unkept candidate at levels
 * >= 2, the gists of unkept candidate chunks, the raw tokens of kept chunks
 * and the raw tail.  levels = 1 is ssa_decode's step, levels = 2 is
 * ssa_decode_h2's.
 * k_sum, v_sum, g_sum (levels - 1 entries) and topk, sel (levels entries)
 * are HOST arrays; the tensors they point to are device memory (a level
 * with Umax(l) = 0 has no unit, and its k_sum, v_sum entries may be NULL).  1 <= levels
 * <= 8, J >= 1, 1 <= g_sum <= 1024, 0 <= topk <= 1024.  Runs on the
 * library's portable kernels.  Needs ssa_workspace_size_hier() bytes of
 * workspace (ws = NULL: allocated stream-ordered).
 */
SSA_API ssa_status ssa_decode_hier(const ssa_shape* shape, const void* q, const void* k_raw,
                                   const void* v_raw, const void* k_gist, const void* v_gist,
                                   const int32_t* seq_lens, int32_t C, int32_t g, int32_t J,
                                   int32_t levels, const void* const* k_sum,
                                   const void* const* v_sum, const int32_t* g_sum,
                                   const int32_t* topk, float* out, int32_t* const* sel, void* ws,
                                   size_t ws_bytes, cudaStream_t stream);

/* Workspace bytes needed by ssa_decode_hier for these sizes. */
SSA_API ssa_status ssa_workspace_size_hier(const ssa_shape* shape, int32_t C, int32_t g, int32_t J,
                                           int32_t levels, const int32_t* g_sum,
                                           const int32_t* topk, size_t* bytes);

/*
 * ssa_decode_path -- which kernels ssa_decode runs for these sizes on the
 * current device (a host-side query; nothing is launched):
 *   SSA_PATH_PIPELINE  two kernels on the stream: gist scoring, then top-k,
 *                      hybrid attention and combination (bf16, d = 64,
 *                      G <= 8, topk <= 128, M_max <= 8192, B <= 128);
 *   SSA_PATH_FUSED     one kernel for the whole step (other bf16 shapes with
 *                      d = 64 or 128 and B <= 128);
 *   SSA_PATH_GENERIC   the portable kernels (fp32, other d, larger B).
 * All three compute the same selection and output up to fp32 summation
 * order.  Errors: those of ssa_decode's size checks; path NULL ->
 * SSA_ERR_INVALID_ARG.
 */
#define SSA_PATH_GENERIC 0
#define SSA_PATH_FUSED 1
#define SSA_PATH_PIPELINE 2
SSA_API ssa_status ssa_decode_path(const ssa_shape* shape, int32_t C, int32_t g, int32_t topk,
                                   int32_t* path);

/* Workspace bytes needed by ssa_decode / ssa_sparse_decode for these sizes. */
SSA_API ssa_status ssa_workspace_size(const ssa_shape* shape, int32_t C, int32_t g, int32_t topk,
                              size_t* bytes);

/* Workspace bytes needed by ssa_decode_h2. */
SSA_API ssa_status ssa_workspace_size_h2(const ssa_shape* shape, int32_t C, int32_t g, int32_t J,
                                 int32_t gm, int32_t topk_super, int32_t topk_chunk,
                                 size_t* bytes);

/* Zero a caller-owned workspace (stream-ordered cudaMemsetAsync). */
SSA_API ssa_status ssa_workspace_init(void* ws, size_t ws_bytes, cudaStream_t stream);

/*
 * Synchronise `stream`, then return in *host_code the library's device status
 * word for the current device (SSA_OK, SSA_ERR_DEVICE_STATUS or
 * SSA_ERR_DEVICE_TIMEOUT; the first error since the last read wins) and clear
 * it.  For tests and diagnostics; the hot calls never read it.
 */
SSA_API ssa_status ssa_get_device_status(int32_t* host_code, cudaStream_t stream);

/*
 * Upper bound, in nanoseconds of GPU time, on every device-side wait (a flag
 * set by another block of the same launch, or a shared-memory barrier).  A
 * wait that runs out records SSA_ERR_DEVICE_TIMEOUT and the kernel carries on
 * without blocking.  The default (2 s) is far above any legal wait.  Values
 * < 1 restore the default.  Process-wide; affects later launches.
 */
SSA_API void ssa_set_wait_limit(int64_t ns);

/*
 * Work-splitting knobs of the fused kernel (process-wide, later launches):
 * max_blocks caps the blocks of the launch (every list of work is split into
 * that many equal shares; default: every block the device holds at once),
 * rows_per_score_item caps the summary rows a block scores before writing
 * chunk scores (at most 1024, the default).  Values < 1 restore the
 * defaults.  Results do not depend on them beyond fp32 summation order.
 */
SSA_API void ssa_set_tuning(int32_t max_blocks, int32_t rows_per_score_item);

/*
 * Test hooks (bit flags, process-wide, later launches; 0 disables all):
 * SSA_DEBUG_SKIP_PUBLISH: the selection step of ssa_sparse_decode never
 *   publishes its selection, so every attention worker waits until its wait
 *   limit and the call reports SSA_ERR_DEVICE_TIMEOUT through
 *   ssa_get_device_status.
 * SSA_DEBUG_FUSED_PATH: single-level bf16 calls that would take the
 *   two-kernel pipeline (d = 64, G <= 8, topk <= 128, M_max <= 8192) take the
 *   one-kernel fused path instead, so the two can be compared.  Both compute
 *   the same selection and the same output up to fp32 summation order.
 */
#define SSA_DEBUG_SKIP_PUBLISH 1
#define SSA_DEBUG_FUSED_PATH 2
SSA_API void ssa_set_debug_flags(int32_t flags);

SSA_API const char* ssa_status_string(ssa_status status);
/* Detail of the last error returned on this host thread ("" if none). */
SSA_API const char* ssa_last_error(void);
SSA_API int32_t ssa_version(void);

/*
 * ---------------------------------------------------------------- budget ---
 * ssa_adaptive_topk -- per-level selection budget (App. A): the chunks each
 * query head keeps, from the raw tokens in the cache n_kv, the chunk size L
 * (= C), the group size G and, for H-SSA, the chunks per meta-gist group J
 * (J = 1: single-level SSA).  With the effective compression L_eff = L * J:
 *     *k = floor(n_kv / (L_eff * G * L)) + 1,
 * so at least one chunk is kept, the group's union of unfolded raw tokens
 * G * k * L stays just above n_kv / L_eff, and both H-SSA levels use the
 * same k.  The pages name the inputs and the +1 but print no formula; this
 * one is the plainest reading.  Host only, no CUDA call.  Errors: n_kv < 0,
 * L, G or J < 1, k NULL -> SSA_ERR_INVALID_ARG; k above INT32_MAX ->
 * SSA_ERR_UNSUPPORTED.
 */
SSA_API ssa_status ssa_adaptive_topk(int64_t n_kv, int32_t L, int32_t G, int32_t J, int32_t* k);

/*
 * --------------------------------------------------------------- prefill ---
 * Prefill attention under the gist mask (sec. 3.1), run block-sparse over
 * permuted key columns (sec. 3.6).
 *
 * The mask: sequence b interleaves each complete chunk m < M_b = n_b / C of C
 * raw tokens with its g gist tokens (the gists follow the chunk and belong to
 * it); the raw tokens after M_b C form chunk M_b, without gists.  A token sees
 * an earlier-or-equal token of its own chunk, and every gist of an earlier
 * chunk; never an earlier chunk's raw tokens.
 *
 * Layout: the permutation puts every gist column (chunk-major) before every
 * raw column, which is how the decode cache already stores keys and values;
 * queries and outputs use the same two arrays per tensor:
 *   q_raw  [B,Hq,n_max,d]  bf16      q_gist [B,Hq,M_max,g,d]  bf16
 *   k_raw, v_raw [B,Hkv,n_max,d]      k_gist, v_gist [B,Hkv,M_max,g,d]
 *   o_raw  [B,Hq,n_max,d]  fp32      o_gist [B,Hq,M_max,g,d]  fp32
 * With raw row i of chunk m = i / C and gist row r = m g + t, the visible
 * columns of a row form one interval per part:
 *   raw row i:   gist columns [0, m g),       raw columns [m C, i + 1);
 *   gist row r:  gist columns [0, r + 1),     raw columns [m C, m C + C).
 *
 * The block plan (computed once per prefill on the host from the host copy of
 * seq_lens, then copied to the device by the caller and shared by every layer's
 * call): query tiles of SSA_PREFILL_BM consecutive rows of one part, key blocks of
 * SSA_PREFILL_BN consecutive columns of one part.  A tile lists every block
 * holding a visible pair, gist blocks first (ascending) then raw blocks; a
 * block is full when every valid row of the tile sees all of its columns
 * (the element mask is then skipped), else partial.  Per tile
 * SSA_PREFILL_TILE_INTS int32:
 *   [0] b  [1] part of the rows (0 raw, 1 gist)  [2] first row r0
 *   [3] valid rows (1 .. BM)  [4] n_b  [5] first entry  [6] entries  [7] 0
 * Tiles are ordered by decreasing entry count (ties: b, part, r0), so the
 * longest tiles start first.  Entry = (block << 2) | (part << 1) | full, with
 * part 0 = gist columns, 1 = raw columns and the block's first column
 * block * SSA_PREFILL_BN.
 */
#define SSA_PREFILL_BM 64
#define SSA_PREFILL_BN 64
#define SSA_PREFILL_TILE_INTS 8

/*
 * ssa_prefill_plan_size -- tile and entry counts of the plan for these
 * sizes.  seq_lens_host: B int32 in host memory.  Errors: B < 0, a NULL
 * pointer, C < 1, g < 1, n_max < 0 or not a multiple of C, an n_b outside
 * [0, n_max] -> SSA_ERR_INVALID_ARG; more than INT32_MAX entries ->
 * SSA_ERR_UNSUPPORTED.
 */
SSA_API ssa_status ssa_prefill_plan_size(int32_t B, const int32_t* seq_lens_host, int32_t n_max,
                                         int32_t C, int32_t g, int64_t* n_tiles,
                                         int64_t* n_entries);

/*
 * ssa_prefill_plan -- writes the plan into caller-owned HOST arrays tiles
 * [n_tiles * SSA_PREFILL_TILE_INTS] and entries [n_entries] (sizes from
 * ssa_prefill_plan_size; caps smaller than those -> SSA_ERR_INVALID_ARG,
 * with nothing written).  Same argument errors as ssa_prefill_plan_size.
 */
SSA_API ssa_status ssa_prefill_plan(int32_t B, const int32_t* seq_lens_host, int32_t n_max,
                                    int32_t C, int32_t g, int32_t* tiles, int64_t tiles_cap,
                                    int32_t* entries, int64_t entries_cap);

/*
 * ssa_prefill -- o = softmax(q k^T / sqrt(d) under the gist mask) v for every
 * row of every sequence, each (tile, query head) one CUDA block that streams
 * the tile's listed key blocks (tensor-core products, online softmax).
 * plan_tiles and plan_entries are the plan in device memory.  Rows at or past
 * n_b (raw) and M_b g (gist) of the outputs are not written.  bf16 inputs, d
 * in {64, 128}; every array pointer 16-byte aligned.  Errors (nothing
 * enqueued): NULL pointers (the gist arrays may be NULL when M_max g = 0),
 * C < 1, g < 1, n_max not a multiple of C, Hq not a multiple of Hkv, n_tiles
 * or n_entries < 0, misaligned pointers -> SSA_ERR_INVALID_ARG; fp32 or
 * another d, more than INT32_MAX blocks -> SSA_ERR_UNSUPPORTED; launch
 * failure -> SSA_ERR_CUDA.  n_tiles = 0 or B = 0 is SSA_OK with nothing
 * enqueued (checked before the pointers).  A plan that does not fit these arrays (a tile or
 * entry out of range) is caught on the device: the kernel skips that tile or
 * block, records SSA_ERR_DEVICE_STATUS for ssa_prefill_get_status, and reads
 * and writes nothing outside the arrays.
 */
SSA_API ssa_status ssa_prefill(const ssa_shape* shape, const void* q_raw, const void* q_gist,
                               const void* k_raw, const void* k_gist, const void* v_raw,
                               const void* v_gist, int32_t C, int32_t g,
                               const int32_t* plan_tiles, int64_t n_tiles,
                               const int32_t* plan_entries, int64_t n_entries, float* o_raw,
                               float* o_gist, cudaStream_t stream);

/*
 * Synchronise `stream`, return in *host_code the prefill's device status word
 * (SSA_OK or SSA_ERR_DEVICE_STATUS: the first plan error since the last read)
 * and clear it.  The prefill kernels keep their own word; ssa_get_device_status
 * does not see it.
 */
SSA_API ssa_status ssa_prefill_get_status(int32_t* host_code, cudaStream_t stream);

/* Detail of the last error a budget or prefill call returned on this host
 * thread ("" if none). */
SSA_API const char* ssa_prefill_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* SSA_H_ */
