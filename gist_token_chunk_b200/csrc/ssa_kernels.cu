// ssa_kernels.cu -- the one device translation unit of libssa: defines the
// device status word, instantiates the fused and generic kernels, and holds
// their host-side launchers (tensor-map encoding, grid sizing).
#include <cudaTypedefs.h>

#include <mutex>

#include "ssa_device.cuh"
#include "ssa_fused.cuh"
#include "ssa_generic.cuh"
#include "ssa_internal.h"
#include "ssa_pipe.cuh"

namespace ssa {

int sm_count() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 148;
    static int cached[64] = {0};
    if (dev < 64 && cached[dev] > 0) return cached[dev];
    int n = 0;
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
    if (dev < 64) cached[dev] = n;
    return n;
}

// The status word is taken (read and cleared) by one atomic exchange on the
// device, so a status that a kernel on another stream sets in between is
// either returned now or kept for the next read, never lost.
static __device__ int g_status_taken = 0;

__global__ void take_status_kernel() { g_status_taken = atomicExch(&g_device_status, 0); }

cudaError_t read_device_status(int* code, cudaStream_t stream) {
    take_status_kernel<<<1, 1, 0, stream>>>();
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    int v = 0;
    e = cudaMemcpyFromSymbolAsync(&v, g_status_taken, sizeof(int), 0, cudaMemcpyDeviceToHost,
                                  stream);
    if (e != cudaSuccess) return e;
    e = cudaStreamSynchronize(stream);
    *code = v;
    return e;
}

// ------------------------------------------------------- built-in scratch ---
// The scratch of ssa_decode_noalloc lives in the library's own device code, so
// that entry point never allocates.  Every call shares it.
static __device__ __align__(256) unsigned char g_builtin_ws[kBuiltinWsBytes];

// The driver's current context: the area's device address belongs to it (a
// device reset or a new primary context gives the area a new address).
static void* current_context() {
    using GetCtx = CUresult (*)(CUcontext*);
    static GetCtx fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void* f = nullptr;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<GetCtx>(f);
    });
    CUcontext c = nullptr;
    if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
    return c;
}

cudaError_t builtin_workspace(void** ptr) {
    static std::mutex mu;
    static void* ctx[64] = {nullptr};
    static void* addr[64] = {nullptr};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    void* c = current_context();
    std::lock_guard<std::mutex> lk(mu);
    if (!addr[dev] || c == nullptr || ctx[dev] != c) {
        // first use in this context (its device is current): look it up
        // (the query also makes the device's primary context current)
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_builtin_ws);
        if (e != cudaSuccess) return e;
        addr[dev] = p;
        ctx[dev] = current_context();
    }
    *ptr = addr[dev];
    return cudaSuccess;
}

// ------------------------------------------------------------- tensor maps ---

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        cudaDriverEntryPointQueryResult q;
        void* f = nullptr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// A [rows, d] bf16 row-major tensor as boxes of 64 columns x box_rows rows
// with the 128-byte swizzle.
// A descriptor is a pure function of (base, rows, d, box rows): each host
// thread keeps the last few it encoded, so a decode loop over the same
// buffers encodes none.
struct MapEntry {
    const void* base;
    uint64_t rows;
    int d, box_rows;
    CUtensorMap map;
};
constexpr int kMapCache = 16;
thread_local MapEntry t_maps[kMapCache];
thread_local int t_map_n = 0, t_map_next = 0;

static bool make_map(CUtensorMap* m, const void* base, uint64_t rows, int d,
                     int box_rows = fused::kBoxRows) {
    for (int i = 0; i < t_map_n; ++i) {
        const MapEntry& e = t_maps[i];
        if (e.base == base && e.rows == rows && e.d == d && e.box_rows == box_rows) {
            *m = e.map;
            return true;
        }
    }
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)d * 2};
    cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return false;
    MapEntry& e = t_maps[t_map_next];
    e.base = base;
    e.rows = rows;
    e.d = d;
    e.box_rows = box_rows;
    e.map = *m;
    t_map_next = (t_map_next + 1) % kMapCache;
    if (t_map_n < kMapCache) ++t_map_n;
    return true;
}

template <int D>
static cudaError_t launch_fused_d(const Plan& plan, cudaStream_t stream) {
    Plan p = plan;
    p.stages = fused::Cfg<D>::kStages;
    p.logits = 0;
    p.logit_stride = 0;
    // two levels: the merged segment lists at both selections
    p.fastsel = (p.cands != nullptr && p.h2 && p.mode == kModeFull && p.topk <= kSegList &&
                 p.topk_super <= kSegList)
                    ? 1
                    : 0;
    CUtensorMap m[6];
    const uint64_t P = (uint64_t)p.n_pairs;
    bool ok = make_map(&m[2], p.k_gist, P * p.M_max * p.g, D);
    if (ok && p.mode == kModeScoreOnly) {
        m[0] = m[1] = m[3] = m[2];  // scoring reads gist keys only
    } else if (ok) {
        ok = make_map(&m[0], p.k_raw, P * p.n_max, D) && make_map(&m[1], p.v_raw, P * p.n_max, D) &&
             make_map(&m[3], p.v_gist, P * p.M_max * p.g, D);
    }
    if (ok && p.h2) {
        ok = make_map(&m[4], p.k_meta, P * p.S_max * p.gm, D) &&
             make_map(&m[5], p.v_meta, P * p.S_max * p.gm, D);
    } else {
        m[4] = m[2];
        m[5] = m[3];
    }
    if (!ok) return cudaErrorInvalidValue;
    const fused::SmemLayout L = fused::smem_layout<D>(p);
    auto kern = fused::fused_kernel<D>;
    static int attr_done[64][2] = {{0}};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !attr_done[dev][D == 128]) {
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             227 * 1024);
        if (e != cudaSuccess) return e;
        attr_done[dev][D == 128] = 1;
    }
    int occ = 0;
    cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, fused::kThreads,
                                                                  (size_t)L.total);
    if (e != cudaSuccess) return e;
    if (occ < 1) return cudaErrorInvalidConfiguration;
    fused::SmemLayout Luse = L;
    // Logits mode (single level, whole step, d = 64): one ring stage less for
    // a shared-memory area that keeps the scored rows' logits, so the gist
    // phase streams only values.  Taken when every block's score share fits
    // and the blocks per SM stay the same.
    if (D == 64 && !p.h2 && p.mode == kModeFull && fused::logit_rows_cap(p.G) > 0) {
        Plan t = p;
        t.logits = 1;
        t.stages = fused::Cfg<D>::kStages - 1;
        t.logit_stride = fused::logit_rows_cap(p.G) + 8;
        const fused::SmemLayout Lt = fused::smem_layout<D>(t);
        int occ_t = 0;
        e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ_t, kern, fused::kThreads,
                                                          (size_t)Lt.total);
        if (e != cudaSuccess) return e;
        long long grid_t = (long long)sm_count() * occ_t;
        if (p.grid_cap > 0 && grid_t > p.grid_cap) grid_t = p.grid_cap;
        if (grid_t > kFusedMaxGrid) grid_t = kFusedMaxGrid;
        const long long chunks = (long long)p.n_pairs * p.M_max;
        if (grid_t > chunks) grid_t = chunks;
        const long long rows_max = grid_t > 0 ? (chunks + grid_t - 1) / grid_t * p.g : 0;
        if (occ_t >= occ && grid_t > 0 && rows_max <= fused::logit_rows_cap(p.G)) {
            // the merged segment lists replace the full top-k where a block's
            // segments are short (one sub-item each)
            t.fastsel = (p.cands != nullptr && p.topk <= kSegList) ? 1 : 0;
            p = t;
            occ = occ_t;
            Luse = Lt;
        }
    }
    // One block per co-resident slot: the static schedule waits across blocks,
    // so the launch is cooperative (all blocks resident at once).  Fewer
    // blocks when the call has little work (upper bound from n_max).
    const long long NP = p.n_pairs;
    const long long tpc = (p.C + fused::kBoxRows - 1) / fused::kBoxRows;
    long long work;
    if (p.mode == kModeScoreOnly) {
        work = NP * p.M_max;
    } else if (!p.h2) {
        const long long kc = p.topk < p.M_max ? p.topk : p.M_max;
        work = NP * (p.M_max + ((long long)p.M_max * p.g + 63) / 64 + kc * tpc + tpc + 1);
    } else {
        work = NP * (p.S_max + p.Mc_max + ((long long)p.S_max * p.gm + 63) / 64 +
                    ((long long)p.Mc_max * p.g + 63) / 64 + (long long)p.topk * tpc + tpc + 2);
    }
    long long grid = (long long)sm_count() * occ;
    if (p.grid_cap > 0 && grid > p.grid_cap) grid = p.grid_cap;
    if (grid > kFusedMaxGrid) grid = kFusedMaxGrid;
    if (grid > work) grid = work;
    if (grid < 1) grid = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(fused::kThreads);
    cfg.dynamicSmemBytes = (size_t)Luse.total;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, p, m[0], m[1], m[2], m[3], m[4], m[5]);
}

// -------------------------------------------------------------- pipeline ---

bool pipe_prepare(Plan& p) {
    p.pp_w1 = p.pp_w3 = 0;
    if (p.mode != kModeFull || p.h2 || p.dtype != 0 || p.d != pipe::kD) return false;
    if (p.G > pipe::kMaxG || p.topk > 128 || p.M_max > 8192 || p.B > kFusedMaxB) return false;
    if (p.sel_stride > 1024) return false;  // published selection entries
    if (p.debug_flags & 2) return false;  // the fused kernel, for comparisons
    const int nsm = sm_count();
    if (nsm > pipe::kMaxBlocks) return false;
    // scoring: 8 worker warps per block when the ring fits, else fewer; the
    // row maxima of the largest chunk share stay in shared memory
    const long long chunks = (long long)p.n_pairs * p.M_max;
    for (int w1 = pipe::kMaxWorkers; w1 >= 4; --w1) {
        const long long W = (long long)nsm * w1;
        const long long parts = chunks < W ? chunks : W;
        const long long per = parts > 0 ? (chunks + parts - 1) / parts : 1;
        const long long rows = (per * p.g + 31) / 32 * 32;
        if (rows > (1 << 16)) return false;
        p.st_rcap = (int)rows;
        if (pipe::score_layout(p, w1).total <= 227 * 1024) {
            p.pp_w1 = w1;
            break;
        }
    }
    // attention: as many worker warps as fit (at least the four that run a
    // block's top-k)
    for (int w3 = pipe::kAttnWorkers; w3 >= 4; --w3)
        if (pipe::attn_layout(p, w3).total <= 227 * 1024) {
            p.pp_w3 = w3;
            break;
        }
    if (p.pp_w1 == 0 || p.pp_w3 == 0) {
        p.pp_w1 = p.pp_w3 = 0;
        return false;
    }
    p.st_slot_bytes = pipe::kRecBytes;
    // one partial slot per (attention worker + pair) index of the launch
    p.st_part_slots = nsm * p.pp_w3 + p.n_pairs;
    p.st_sel_stride = pipe::sel_stride(p.sel_stride);
    return true;
}

void pipe_ws_sizes(const Plan& p, size_t* hdr, size_t* scores, size_t* logits, size_t* sel,
                   size_t* part) {
    const size_t P = (size_t)p.n_pairs;
    *hdr = 256;
    *scores = P * pipe::score_row(p.M_max) * 4;
    *logits = (P * p.M_max * p.g + 64) * pipe::logit_stride(p.G) * 4;
    *sel = P * p.st_sel_stride * 8;
    *part = 2 * (size_t)p.G * p.st_part_slots * p.st_slot_bytes;
}

cudaError_t launch_pipe(const Plan& p, cudaStream_t stream) {
    CUtensorMap m[4];
    const uint64_t P = (uint64_t)p.n_pairs;
    const bool ok = make_map(&m[0], p.k_gist, P * p.M_max * p.g, pipe::kD, pipe::kGistRows) &&
                    make_map(&m[1], p.v_gist, P * p.M_max * p.g, pipe::kD, pipe::kGistRows) &&
                    make_map(&m[2], p.k_raw, P * p.n_max, pipe::kD, pipe::kRawRows) &&
                    make_map(&m[3], p.v_raw, P * p.n_max, pipe::kD, pipe::kRawRows);
    if (!ok) return cudaErrorInvalidValue;
    static int attr_done[64] = {0};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 0 || dev >= 64 || !attr_done[dev]) {
        cudaError_t e = cudaFuncSetAttribute(pipe::score_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(pipe::attend_kernel<false>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(pipe::attend_kernel<true>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) attr_done[dev] = 1;
    }
    const unsigned nsm = (unsigned)sm_count();
    // scoring: an ordinary launch (it follows whatever came before on the
    // stream); attention: may start as scoring drains (programmatic
    // dependent launch) and waits for it on the device before it reads the
    // scoring results
    cudaLaunchConfig_t c1 = {};
    c1.gridDim = dim3(nsm);
    c1.blockDim = dim3(32 * p.pp_w1);
    c1.dynamicSmemBytes = (size_t)pipe::score_layout(p, p.pp_w1).total;
    c1.stream = stream;
    cudaError_t e = cudaLaunchKernelEx(&c1, pipe::score_kernel, p, m[0]);
    if (e != cudaSuccess) return e;
    cudaLaunchAttribute pdl[1];
    pdl[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t c3 = {};
    c3.gridDim = dim3(nsm);
    c3.blockDim = dim3(32 * (p.pp_w3 + 1));
    c3.dynamicSmemBytes = (size_t)pipe::attn_layout(p, p.pp_w3).total;
    c3.stream = stream;
    c3.attrs = pdl;
    c3.numAttrs = 1;
    return p.sel_mode == 1 ? cudaLaunchKernelEx(&c3, pipe::attend_kernel<true>, p, m[1], m[2], m[3])
                           : cudaLaunchKernelEx(&c3, pipe::attend_kernel<false>, p, m[1], m[2], m[3]);
}

cudaError_t launch_fused(const Plan& p, cudaStream_t stream) {
    if (p.d == 64) return launch_fused_d<64>(p, stream);
    if (p.d == 128) return launch_fused_d<128>(p, stream);
    return cudaErrorInvalidValue;
}

int fused_smem_bytes(const Plan& p) {
    if (p.d == 64) return fused::smem_layout<64>(p).total;
    return fused::smem_layout<128>(p).total;
}

// ----------------------------------------------------------------- generic ---

template <class T>
static cudaError_t launch_generic_t(const Plan& p, cudaStream_t stream) {
    const int P = p.n_pairs;
    // a given selection leaves the score area unused: it holds the flags of
    // rejected selections (the control words stay untouched, hence zero)
    int* bad = reinterpret_cast<int*>(p.scores);
    const size_t qsm = (size_t)p.G * p.d * sizeof(float);
    auto score = [&](int level, float* dst, int stride, int nslots) {
        const int per_block = 4;
        const int gx = (nslots + per_block - 1) / per_block;
        dim3 grid(gx > 0 ? gx : 1, P);
        gen::score_kernel<T><<<grid, 128, qsm, stream>>>(p, level, dst, stride, nslots);
    };
    if (p.mode == kModeScoreOnly) {
        score(0, p.scores, p.M_max, p.M_max);
        return cudaGetLastError();
    }
    if (p.mode == kModeAttnOnly) {
        gen::validate_kernel<<<(P + 127) / 128, 128, 0, stream>>>(p, bad);
    } else if (!p.h2 && p.sel_mode == 1) {
        // per-head scores and top-k, union over each group (App. A)
        const int rows = p.B * p.Hq;
        const int gx = (p.M_max + 3) / 4;
        gen::head_score_kernel<T><<<dim3(gx > 0 ? gx : 1, rows), 128, (size_t)p.d * sizeof(float),
                                    stream>>>(p, p.scores);
        gen::head_topk_kernel<<<rows, 128, 0, stream>>>(p, p.scores);
        gen::union_kernel<<<P, 128, (size_t)p.mask_words * sizeof(uint32_t), stream>>>(p);
    } else if (!p.h2) {
        score(0, p.scores, p.M_max, p.M_max);
        gen::topk_kernel<<<P, 128, 0, stream>>>(p, 0, p.scores, p.M_max);
    } else {
        score(1, p.super_scores, p.S_max, p.S_max);
        gen::topk_kernel<<<P, 128, 0, stream>>>(p, 1, p.super_scores, p.S_max);
        score(2, p.cand_scores, p.Mc_max, p.Mc_max);
        gen::topk_kernel<<<P, 128, 0, stream>>>(p, 2, p.cand_scores, p.Mc_max);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int nw = 8;
    const size_t sm = (size_t)(p.d + 2 * nw + nw * p.d) * sizeof(float) +
                      (size_t)(p.mask_words + p.smask_words) * sizeof(uint32_t);
    dim3 grid(p.Hq, p.B);
    gen::attend_kernel<T><<<grid, 32 * nw, sm, stream>>>(
        p, p.mode == kModeAttnOnly ? bad : nullptr);
    return cudaGetLastError();
}

template <class T>
static cudaError_t launch_hier_t(const Plan& p, const HierLevels& hl, cudaStream_t stream) {
    const int P = p.n_pairs;
    const size_t qsm = (size_t)p.G * p.d * sizeof(float);
    for (int l = hl.levels - 1; l >= 0; --l) {
        // candidates: every unit at the top; below, the kept parents'
        // children and fewer than J remainder units
        long long bound = hl.umax[l];
        if (l < hl.levels - 1) {
            const long long b2 = (long long)hl.topk[l + 1] * p.J + p.J;
            if (b2 < bound) bound = b2;
        }
        const int gx = (int)((bound + 3) / 4);
        gen::hier_score_kernel<T><<<dim3(gx > 0 ? gx : 1, P), 128, qsm, stream>>>(p, hl, l);
        gen::hier_topk_kernel<<<P, 128, 0, stream>>>(p, hl, l);
    }
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int nw = 8;
    int nsel = 0;
    for (int l = 0; l < hl.levels; ++l) nsel += hl.topk[l];
    const size_t sm = (size_t)(p.d + 2 * nw + nw * p.d) * sizeof(float) +
                      (size_t)hl.mask_words * sizeof(uint32_t) + (size_t)nsel * sizeof(int);
    if (sm > 48 * 1024) {
        e = cudaFuncSetAttribute(gen::hier_attend_kernel<T>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
    }
    gen::hier_attend_kernel<T><<<dim3(p.Hq, p.B), 32 * nw, sm, stream>>>(p, hl);
    return cudaGetLastError();
}

cudaError_t launch_hier(const Plan& p, const HierLevels& hl, cudaStream_t stream) {
    return p.dtype == 0 ? launch_hier_t<__nv_bfloat16>(p, hl, stream)
                        : launch_hier_t<float>(p, hl, stream);
}

cudaError_t launch_generic(const Plan& p, cudaStream_t stream) {
    if (p.dtype == 1) return launch_generic_t<float>(p, stream);
    return launch_generic_t<__nv_bfloat16>(p, stream);
}

cudaError_t launch_topk(const Plan& p, const float* scores, cudaStream_t stream) {
    gen::topk_kernel<<<p.n_pairs, 128, 0, stream>>>(p, 0, scores, p.M_max);
    return cudaGetLastError();
}

}  // namespace ssa
