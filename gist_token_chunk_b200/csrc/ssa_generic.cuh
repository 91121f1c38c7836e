// ssa_generic.cuh -- straightforward kernels for every dtype and head dim up
// to 256 (used for fp32 inputs and for head dims the fused path does not
// cover).  One warp per dot product, fp32 throughout, one block per query
// head for the attention.  Same semantics as the fused path; slow by design.
#pragma once

#include "ssa_device.cuh"
#include "ssa_internal.h"

namespace ssa {
namespace gen {

__device__ __forceinline__ float to_f(float x) { return x; }
__device__ __forceinline__ float to_f(__nv_bfloat16 x) { return __bfloat162float(x); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// Sequence length of b, or -1 (and a device status) when outside [1, n_max].
__device__ __forceinline__ int checked_len(const Plan& p, int b) {
    int n = p.seq_lens[b];
    if (n < 1 || n > p.n_max) {
        report_status(kStatusBadInput);
        return -1;
    }
    return n;
}

// Number of selected superchunks kept for (p): min(topk_super, S_b).
__device__ __forceinline__ int kept_super(const Plan& p, int S) {
    return p.topk_super < S ? p.topk_super : S;
}

// Candidate position c of pair `pr` -> chunk index (two-level step): the J
// children of each kept superchunk in ascending order, then the remainder.
__device__ __forceinline__ int cand_chunk(const Plan& p, int pr, int c, int ks, int S) {
    if (c < ks * p.J) return p.sel_super[(size_t)pr * p.topk_super + c / p.J] * p.J + c % p.J;
    return S * p.J + (c - ks * p.J);
}

// Slot scores: dst[pr*stride + s] = max over the group's heads and the
// slot's ntok summary rows of q.k/sqrt(d) for s < n_valid, -inf for
// n_valid <= s < n_slots.  level 0: gist slots of chunks (single level),
// 1: meta slots of superchunks, 2: candidate chunks (two level).
template <class T>
__global__ void score_kernel(Plan p, int level, float* dst, int stride, int n_slots_fixed) {
    extern __shared__ float qs[];  // [G][d]
    const int pr = blockIdx.y;
    const int b = pr / p.Hkv, j = pr % p.Hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const T* q = static_cast<const T*>(p.q) + ((size_t)b * p.Hq + (size_t)j * p.G) * p.d;
    for (int i = threadIdx.x; i < p.G * p.d; i += blockDim.x) qs[i] = to_f(q[i]);
    __syncthreads();
    const int n = checked_len(p, b);
    const int M = n > 0 ? n / p.C : 0;
    int n_valid, n_slots, ntok, ks = 0, S = 0;
    const T* keys;
    if (level == 0) {
        n_valid = M;
        n_slots = n_slots_fixed;
        ntok = p.g;
        keys = static_cast<const T*>(p.k_gist) + (size_t)pr * p.M_max * p.g * p.d;
    } else if (level == 1) {
        n_valid = M / p.J;
        n_slots = n_slots_fixed;
        ntok = p.gm;
        keys = static_cast<const T*>(p.k_meta) + (size_t)pr * p.S_max * p.gm * p.d;
    } else {
        S = M / p.J;
        ks = kept_super(p, S);
        n_valid = ks * p.J + (M - S * p.J);
        n_slots = n_valid;
        ntok = p.g;
        keys = static_cast<const T*>(p.k_gist) + (size_t)pr * p.M_max * p.g * p.d;
    }
    const float scale = rsqrtf((float)p.d);
    const int nw = blockDim.x >> 5;
    for (int s = blockIdx.x * nw + warp; s < n_slots; s += gridDim.x * nw) {
        float best = -INFINITY;
        if (s < n_valid) {
            const int slot = (level == 2) ? cand_chunk(p, pr, s, ks, S) : s;
            const T* kr = keys + (size_t)slot * ntok * p.d;
            for (int t = 0; t < ntok; ++t) {
                for (int h = 0; h < p.G; ++h) {
                    float acc = 0.f;
                    for (int i = lane; i < p.d; i += 32)
                        acc += qs[h * p.d + i] * to_f(kr[(size_t)t * p.d + i]);
                    acc = warp_sum(acc);
                    best = fmaxf(best, acc * scale);
                }
            }
        }
        if (lane == 0) dst[(size_t)pr * stride + s] = best;
    }
}

// q . k for one key row: 16-byte loads when the row allows them (each lane
// reads its own row, so wide loads keep the L1 requests per row few), else
// element loads.
__device__ __forceinline__ float bf_lo32(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf_hi32(uint32_t x) { return __uint_as_float(x & 0xffff0000u); }
template <class T>
__device__ __forceinline__ float dot_row(const float* qs, const T* kr, int d) {
    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
    int i = 0;
    if ((reinterpret_cast<uintptr_t>(kr) & 15u) == 0) {
        const uint4* k4 = reinterpret_cast<const uint4*>(kr);
        constexpr int per = 16 / (int)sizeof(T);
        for (; i + per <= d; i += per) {
            const uint4 w = k4[i / per];
            if constexpr (sizeof(T) == 2) {
                s0 += qs[i] * bf_lo32(w.x) + qs[i + 1] * bf_hi32(w.x);
                s1 += qs[i + 2] * bf_lo32(w.y) + qs[i + 3] * bf_hi32(w.y);
                s2 += qs[i + 4] * bf_lo32(w.z) + qs[i + 5] * bf_hi32(w.z);
                s3 += qs[i + 6] * bf_lo32(w.w) + qs[i + 7] * bf_hi32(w.w);
            } else {
                s0 += qs[i] * __uint_as_float(w.x);
                s1 += qs[i + 1] * __uint_as_float(w.y);
                s2 += qs[i + 2] * __uint_as_float(w.z);
                s3 += qs[i + 3] * __uint_as_float(w.w);
            }
        }
    }
    for (; i < d; ++i) s0 += qs[i] * to_f(kr[i]);
    return (s0 + s1) + (s2 + s3);
}

// Online softmax of one query (qs, fp32 in shared memory, log2-domain scale)
// over `rows` key/value rows, by one warp, 32 rows at a time: lane j takes
// the dot product of row r0 + j (its loads independent of the other lanes'),
// the warp shares one maximum and one sum per group, and each lane
// accumulates its dims (lane + 32 r) over the group's rows.  m_run, l_run,
// acc are the warp's running state (same values in every lane).
template <class T>
__device__ __forceinline__ void attend_rows(const float* qs, const T* kbase, const T* vbase,
                                            int rows, int d, float scale, float& m_run,
                                            float& l_run, float (&acc)[8]) {
    const int lane = threadIdx.x & 31;
    const int row_bytes = d * (int)sizeof(T);
    // L2 prefetch of row r's key and value lines (each lane one row)
    auto prefetch_row = [&](int r) {
        if (r >= rows) return;
        const char* kp = reinterpret_cast<const char*>(kbase + (size_t)r * d);
        const char* vp = reinterpret_cast<const char*>(vbase + (size_t)r * d);
        for (int o = 0; o < row_bytes; o += 128) {
            asm volatile("prefetch.global.L2 [%0];" ::"l"(kp + o));
            asm volatile("prefetch.global.L2 [%0];" ::"l"(vp + o));
        }
    };
    prefetch_row(lane);
    for (int r0 = 0; r0 < rows; r0 += 32) {
        const int r = r0 + lane;
        const int nr = min(32, rows - r0);
        prefetch_row(r + 32);  // the next group's rows, while this one computes
        float x = -INFINITY;
        if (r < rows) x = dot_row<T>(qs, kbase + (size_t)r * d, d) * scale;
        float mx = x;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        const float mn = fmaxf(m_run, mx);
        const float ref = mn == -INFINITY ? 0.f : mn;
        const float a = exp2f(m_run - ref);
        const float e = r < rows ? exp2f(x - ref) : 0.f;
        l_run = l_run * a + warp_sum(e);
        m_run = mn;
#pragma unroll
        for (int q = 0; q < 8; ++q) acc[q] *= a;
#pragma unroll 8
        for (int j = 0; j < nr; ++j) {
            const float ej = __shfl_sync(0xffffffffu, e, j);
            const T* vr = vbase + (size_t)(r0 + j) * d;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
                const int i = lane + 32 * q;
                if (i < d) acc[q] += ej * to_f(vr[i]);
            }
        }
    }
}

// Per-head chunk scores (selection reading "per head + union", App. A):
// dst[row * M_max + m] = max over the chunk's g gist rows of q_h.k/sqrt(d)
// for row = b * Hq + h, m < M_b; -inf for M_b <= m < M_max.
template <class T>
__global__ void head_score_kernel(Plan p, float* dst) {
    extern __shared__ float qs[];  // [d]
    const int row = blockIdx.y;
    const int b = row / p.Hq, h = row % p.Hq, j = h / p.G;
    const int pr = b * p.Hkv + j;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const T* q = static_cast<const T*>(p.q) + ((size_t)b * p.Hq + h) * p.d;
    for (int i = threadIdx.x; i < p.d; i += blockDim.x) qs[i] = to_f(q[i]);
    __syncthreads();
    const int n = checked_len(p, b);
    const int M = n > 0 ? n / p.C : 0;
    const T* keys = static_cast<const T*>(p.k_gist) + (size_t)pr * p.M_max * p.g * p.d;
    const float scale = rsqrtf((float)p.d);
    const int nw = blockDim.x >> 5;
    for (int m = blockIdx.x * nw + warp; m < p.M_max; m += gridDim.x * nw) {
        float best = -INFINITY;
        if (m < M) {
            const T* kr = keys + (size_t)m * p.g * p.d;
            for (int t = 0; t < p.g; ++t) {
                float acc = 0.f;
                for (int i = lane; i < p.d; i += 32) acc += qs[i] * to_f(kr[(size_t)t * p.d + i]);
                best = fmaxf(best, warp_sum(acc) * scale);
            }
        }
        if (lane == 0) dst[(size_t)row * p.M_max + m] = best;
    }
}

struct BlockSync {
    __device__ void operator()() const { __syncthreads(); }
    __device__ bool or_(bool pred) const { return __syncthreads_or(pred) != 0; }
};

// Top-k per pair (block of 128).  level 0: chunks over scores (single level
// or ssa_topk_chunks); 1: superchunks; 2: candidate chunks (positions are
// mapped to chunk ids afterwards; the map is increasing, so the order holds).
__global__ void topk_kernel(Plan p, int level, const float* vals, int stride) {
    __shared__ TopkScratch sc;
    const int pr = blockIdx.x;
    const int b = pr / p.Hkv;
    int n = p.seq_lens[b];
    if (n < 1 || n > p.n_max) n = 0;  // reported by the scoring kernel
    const int M = n / p.C;
    const float* v = vals + (size_t)pr * stride;
    if (level == 0) {
        block_topk<128>(v, M, p.topk, p.sel_idx + (size_t)pr * p.topk, sc, BlockSync());
    } else if (level == 1) {
        block_topk<128>(v, M / p.J, p.topk_super, p.sel_super + (size_t)pr * p.topk_super, sc,
                        BlockSync());
    } else {
        const int S = M / p.J;
        const int ks = kept_super(p, S);
        const int nc = ks * p.J + (M - S * p.J);
        int* out = p.sel_idx + (size_t)pr * p.topk;
        block_topk<128>(v, nc, p.topk, out, sc, BlockSync());
        __syncthreads();
        for (int c = threadIdx.x; c < p.topk; c += blockDim.x) {
            const int pos = out[c];
            if (pos >= 0) out[c] = cand_chunk(p, pr, pos, ks, S);
        }
    }
}

// Per-head top-k (block of 128 per row b * Hq + h) into head_sel.
__global__ void head_topk_kernel(Plan p, const float* vals) {
    __shared__ TopkScratch sc;
    const int row = blockIdx.x;
    const int b = row / p.Hq;
    int n = p.seq_lens[b];
    if (n < 1 || n > p.n_max) n = 0;  // reported by the scoring kernel
    block_topk<128>(vals + (size_t)row * p.M_max, n / p.C, p.topk,
                    p.head_sel + (size_t)row * p.topk, sc, BlockSync());
}

// Union of the group's per-head selections (App. A): sel_idx[pr] = the
// chunks any head of KV head j selected, ascending, then -1 up to sel_stride.
// One block of 128 per pair; a chunk bitmap in shared memory.
__global__ void union_kernel(Plan p) {
    extern __shared__ uint32_t bits[];  // [mask_words]
    __shared__ int base[129];
    const int pr = blockIdx.x;
    const int b = pr / p.Hkv, j = pr % p.Hkv;
    for (int i = threadIdx.x; i < p.mask_words; i += blockDim.x) bits[i] = 0u;
    __syncthreads();
    for (int e = threadIdx.x; e < p.G * p.topk; e += blockDim.x) {
        const int h = j * p.G + e / p.topk;
        const int m = p.head_sel[((size_t)b * p.Hq + h) * p.topk + e % p.topk];
        if (m >= 0) atomicOr(&bits[m >> 5], 1u << (m & 31));
    }
    __syncthreads();
    // thread t owns words [t * per, (t + 1) * per): count, scan, then write
    const int per = (p.mask_words + 127) / 128;
    const int w0 = threadIdx.x * per, w1 = min(w0 + per, p.mask_words);
    int cnt = 0;
    for (int w = w0; w < w1; ++w) cnt += __popc(bits[w]);
    base[threadIdx.x + 1] = cnt;
    __syncthreads();
    if (threadIdx.x == 0) {
        base[0] = 0;
        for (int t = 1; t <= 128; ++t) base[t] += base[t - 1];
    }
    __syncthreads();
    int32_t* out = p.sel_idx + (size_t)pr * p.sel_stride;
    int at = base[threadIdx.x];
    for (int w = w0; w < w1; ++w)
        for (uint32_t x = bits[w]; x; x &= x - 1) out[at++] = w * 32 + __ffs(x) - 1;
    for (int i = base[128] + threadIdx.x; i < p.sel_stride; i += blockDim.x) out[i] = -1;
}

// Checks a caller-given selection (ssa_sparse_decode): strictly ascending
// chunk indices in [0, M_b) followed only by -1.  Marks bad pairs in ctrl.
__global__ void validate_kernel(Plan p, int* bad) {
    const int pr = blockIdx.x * blockDim.x + threadIdx.x;
    if (pr >= p.n_pairs) return;
    const int b = pr / p.Hkv;
    int n = p.seq_lens[b];
    const int M = (n >= 1 && n <= p.n_max) ? n / p.C : 0;
    const int* s = p.sel_idx + (size_t)pr * p.topk;
    int ok = 1, prev = -1, ended = 0;
    for (int c = 0; c < p.topk; ++c) {
        int v = s[c];
        if (v < 0) {
            ended = 1;
            if (v != -1) ok = 0;
        } else {
            if (ended || v <= prev || v >= M) ok = 0;
            prev = v;
        }
    }
    bad[pr] = !ok;
    if (!ok) report_status(kStatusBadInput);
}

// One block per (query head, sequence): online softmax over the unfolded
// context, enumerated chunk by chunk; warps take units round-robin.
template <class T>
__global__ void attend_kernel(Plan p, const int* bad) {
    extern __shared__ float sm[];
    const int h = blockIdx.x, b = blockIdx.y;
    const int j = h / p.G;
    const int pr = b * p.Hkv + j;
    const int nw = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float* qs = sm;                                   // [d]
    float* wm = qs + p.d;                             // [nw]
    float* wl = wm + nw;                              // [nw]
    float* wacc = wl + nw;                            // [nw][d]
    uint32_t* cbits = reinterpret_cast<uint32_t*>(wacc + nw * p.d);  // [mask_words]
    uint32_t* sbits = cbits + p.mask_words;                          // [smask_words]
    float* outp = p.out + ((size_t)b * p.Hq + h) * p.d;

    int n = p.seq_lens[b];
    const bool bad_len = (n < 1 || n > p.n_max);
    const bool bad_sel = bad != nullptr && bad[pr];
    if (bad_len || bad_sel) {
        if (bad_len) report_status(kStatusBadInput);
        for (int i = threadIdx.x; i < p.d; i += blockDim.x) outp[i] = 0.f;
        return;
    }
    const T* qg = static_cast<const T*>(p.q) + ((size_t)b * p.Hq + h) * p.d;
    for (int i = threadIdx.x; i < p.d; i += blockDim.x) qs[i] = to_f(qg[i]);
    for (int i = threadIdx.x; i < p.mask_words; i += blockDim.x) cbits[i] = 0;
    for (int i = threadIdx.x; i < p.smask_words; i += blockDim.x) sbits[i] = 0;
    __syncthreads();
    const int M = n / p.C;
    const int S = p.h2 ? M / p.J : 0;
    const int ks = p.h2 ? kept_super(p, S) : 0;
    {
        const int ns = p.sel_stride > 0 ? p.sel_stride : p.topk;
        for (int c = threadIdx.x; c < ns; c += blockDim.x) {
            const int m = p.sel_idx[(size_t)pr * ns + c];
            if (m >= 0) atomicOr(&cbits[m >> 5], 1u << (m & 31));
        }
        for (int c = threadIdx.x; c < ks; c += blockDim.x) {
            const int x = p.sel_super[(size_t)pr * p.topk_super + c];
            atomicOr(&sbits[x >> 5], 1u << (x & 31));
        }
    }
    __syncthreads();
    const float scale = rsqrtf((float)p.d) * 1.4426950408889634f;  // log2 domain
    const T* kr = static_cast<const T*>(p.k_raw) + (size_t)pr * p.n_max * p.d;
    const T* vr = static_cast<const T*>(p.v_raw) + (size_t)pr * p.n_max * p.d;
    const T* kg = static_cast<const T*>(p.k_gist) + (size_t)pr * p.M_max * p.g * p.d;
    const T* vg = static_cast<const T*>(p.v_gist) + (size_t)pr * p.M_max * p.g * p.d;
    const T* km = p.h2 ? static_cast<const T*>(p.k_meta) + (size_t)pr * p.S_max * p.gm * p.d
                       : nullptr;
    const T* vm = p.h2 ? static_cast<const T*>(p.v_meta) + (size_t)pr * p.S_max * p.gm * p.d
                       : nullptr;
    float m_run = -INFINITY, l_run = 0.f;
    float acc[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) acc[r] = 0.f;

    // Every warp walks every unit in the same order and numbers its 32-row
    // groups the same way; warp w attends the groups numbered w mod (warps),
    // so the rows spread evenly whatever the unit sizes.
    int gi = 0;
    auto visit = [&](const T* kbase, const T* vbase, int rows) {
        for (int r0 = 0; r0 < rows; r0 += 32, ++gi)
            if (gi % nw == warp)
                attend_rows<T>(qs, kbase + (size_t)r0 * p.d, vbase + (size_t)r0 * p.d,
                               min(32, rows - r0), p.d, scale, m_run, l_run, acc);
    };
    // ctx_mode 0: a selected chunk contributes its raw tokens, an unselected
    // one its gists; ctx_mode 1: a selected chunk its gists and raw tokens,
    // an unselected one nothing
    auto chunk_unit = [&](int m) {
        const bool selected = cbits[m >> 5] >> (m & 31) & 1u;
        if (selected || p.ctx_mode == 0) {
            if (!selected || p.ctx_mode == 1)
                visit(kg + (size_t)m * p.g * p.d, vg + (size_t)m * p.g * p.d, p.g);
            if (selected) visit(kr + (size_t)m * p.C * p.d, vr + (size_t)m * p.C * p.d, p.C);
        }
    };
    // units: single level -> chunks 0..M-1 then the tail;
    // two level -> superchunks 0..S-1, remainder chunks, then the tail.
    const int n_units = p.h2 ? S + (M - S * p.J) + 1 : M + 1;
    for (int u = 0; u < n_units; ++u) {
        if (u == n_units - 1) {
            visit(kr + (size_t)M * p.C * p.d, vr + (size_t)M * p.C * p.d, n - M * p.C);
        } else if (!p.h2) {
            chunk_unit(u);
        } else if (u < S) {
            if (sbits[u >> 5] >> (u & 31) & 1u) {
                for (int i = 0; i < p.J; ++i) chunk_unit(u * p.J + i);
            } else {
                visit(km + (size_t)u * p.gm * p.d, vm + (size_t)u * p.gm * p.d, p.gm);
            }
        } else {
            chunk_unit(S * p.J + (u - S));
        }
    }
    if (lane == 0) {
        wm[warp] = m_run;
        wl[warp] = l_run;
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        int i = lane + 32 * r;
        if (i < p.d) wacc[warp * p.d + i] = acc[r];
    }
    __syncthreads();
    float mx = -INFINITY;
    for (int w = 0; w < nw; ++w) mx = fmaxf(mx, wm[w]);
    float L = 0.f;
    for (int w = 0; w < nw; ++w) L += (wm[w] == -INFINITY) ? 0.f : wl[w] * exp2f(wm[w] - mx);
    for (int i = threadIdx.x; i < p.d; i += blockDim.x) {
        float o = 0.f;
        for (int w = 0; w < nw; ++w)
            if (wm[w] != -INFINITY) o += wacc[w * p.d + i] * exp2f(wm[w] - mx);
        outp[i] = L > 0.f ? o / L : 0.f;
    }
}

// ------------------------------------------------------------- t levels ---

// Complete units of every level of pair `pr`'s sequence (U[0] = M).
__device__ __forceinline__ void hier_units(const Plan& p, const HierLevels& hl, int n, int* U) {
    U[0] = n > 0 ? n / p.C : 0;
    for (int l = 1; l < hl.levels; ++l) U[l] = U[l - 1] / p.J;
}

// Candidates of level l for pair pr: the top level's complete units; below,
// the J children of each unit kept one level up (ascending), then the
// remainder units U[l+1] J .. U[l] - 1.  Returns the count; cand_unit maps a
// candidate position to its unit (an increasing map).
// Every level keeps exactly min(topk, candidates) units, so the counts
// follow from the unit counts alone: no selection needs to be read.
__device__ __forceinline__ int hier_count(const HierLevels& hl, int l, int pr, const int* U,
                                          int J, int& nkept) {
    (void)pr;
    int nc = U[hl.levels - 1];
    nkept = 0;
    for (int m = hl.levels - 2; m >= l; --m) {
        nkept = min(hl.topk[m + 1], nc);
        nc = nkept * J + (U[m] - U[m + 1] * J);
    }
    return nc;
}
__device__ __forceinline__ int hier_unit(const HierLevels& hl, int l, int pr, const int* U, int J,
                                         int nkept, int c) {
    if (l == hl.levels - 1) return c;
    if (c < nkept * J) return hl.sel[l + 1][(size_t)pr * hl.topk[l + 1] + c / J] * J + c % J;
    return U[l + 1] * J + (c - nkept * J);
}

// Scores of level l's candidates: max over the group's heads and the unit's
// summary tokens (gists at level 0) of q.k/sqrt(d), into cscore[l].
template <class T>
__global__ void hier_score_kernel(Plan p, HierLevels hl, int l) {
    extern __shared__ float qs[];  // [G][d]
    const int pr = blockIdx.y;
    const int b = pr / p.Hkv, j = pr % p.Hkv;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const T* q = static_cast<const T*>(p.q) + ((size_t)b * p.Hq + (size_t)j * p.G) * p.d;
    for (int i = threadIdx.x; i < p.G * p.d; i += blockDim.x) qs[i] = to_f(q[i]);
    __syncthreads();
    int U[kMaxLevels];
    hier_units(p, hl, checked_len(p, b), U);
    int nkept;
    const int nc = hier_count(hl, l, pr, U, p.J, nkept);
    const int ntok = l == 0 ? p.g : hl.gs[l];
    const T* keys = l == 0 ? static_cast<const T*>(p.k_gist) + (size_t)pr * p.M_max * p.g * p.d
                           : static_cast<const T*>(hl.k_sum[l]) +
                                 (size_t)pr * hl.umax[l] * hl.gs[l] * p.d;
    const float scale = rsqrtf((float)p.d);
    const int nw = blockDim.x >> 5;
    for (int c = blockIdx.x * nw + warp; c < nc; c += gridDim.x * nw) {
        const T* kr = keys + (size_t)hier_unit(hl, l, pr, U, p.J, nkept, c) * ntok * p.d;
        float best = -INFINITY;
        for (int t = 0; t < ntok; ++t)
            for (int h = 0; h < p.G; ++h) {
                float acc = 0.f;
                for (int i = lane; i < p.d; i += 32) acc += qs[h * p.d + i] * to_f(kr[(size_t)t * p.d + i]);
                best = fmaxf(best, warp_sum(acc) * scale);
            }
        if (lane == 0) hl.cscore[l][(size_t)pr * hl.umax[l] + c] = best;
    }
}

// Level l's top-k over its candidates (ties to the lower position, which is
// the lower unit: the candidate map increases), mapped to unit ids.
__global__ void hier_topk_kernel(Plan p, HierLevels hl, int l) {
    __shared__ TopkScratch sc;
    const int pr = blockIdx.x;
    const int b = pr / p.Hkv;
    int n = p.seq_lens[b];
    if (n < 1 || n > p.n_max) n = 0;  // reported by the scoring kernel
    int U[kMaxLevels];
    hier_units(p, hl, n, U);
    int nkept;
    const int nc = hier_count(hl, l, pr, U, p.J, nkept);
    int* out = hl.sel[l] + (size_t)pr * hl.topk[l];
    block_topk<128>(hl.cscore[l] + (size_t)pr * hl.umax[l], nc, hl.topk[l], out, sc, BlockSync());
    __syncthreads();
    for (int c = threadIdx.x; c < hl.topk[l]; c += blockDim.x) {
        const int pos = out[c];
        if (pos >= 0) out[c] = hier_unit(hl, l, pr, U, p.J, nkept, pos);
    }
}

// Attention over the t-level context, one block per (query head, sequence):
// the summaries of every unkept candidate at levels >= 1, the gists of
// unkept candidate chunks, the raw tokens of kept chunks, the tail.  Every
// warp walks the same list of candidates (each level's selection is first
// copied to shared memory, so the walk reads no global memory) and numbers
// their 32-row groups in the same order; warp w attends the groups whose
// number is w mod (warps), so the rows spread evenly whatever the unit sizes.
template <class T>
__global__ void hier_attend_kernel(Plan p, HierLevels hl) {
    extern __shared__ float sm[];
    const int h = blockIdx.x, b = blockIdx.y;
    const int j = h / p.G;
    const int pr = b * p.Hkv + j;
    const int nw = blockDim.x >> 5;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    float* qs = sm;                                   // [d]
    float* wm = qs + p.d;                             // [nw]
    float* wl = wm + nw;                              // [nw]
    float* wacc = wl + nw;                            // [nw][d]
    uint32_t* bits = reinterpret_cast<uint32_t*>(wacc + nw * p.d);  // kept units, per level
    int* sels = reinterpret_cast<int*>(bits + hl.mask_words);        // every level's selection
    float* outp = p.out + ((size_t)b * p.Hq + h) * p.d;
    const int n = p.seq_lens[b];
    if (n < 1 || n > p.n_max) {
        report_status(kStatusBadInput);
        for (int i = threadIdx.x; i < p.d; i += blockDim.x) outp[i] = 0.f;
        return;
    }
    const T* qg = static_cast<const T*>(p.q) + ((size_t)b * p.Hq + h) * p.d;
    for (int i = threadIdx.x; i < p.d; i += blockDim.x) qs[i] = to_f(qg[i]);
    for (int i = threadIdx.x; i < hl.mask_words; i += blockDim.x) bits[i] = 0u;
    int off[kMaxLevels], soff[kMaxLevels];
    {
        int o = 0, so = 0;
        for (int l = 0; l < hl.levels; ++l) {
            off[l] = o;
            soff[l] = so;
            o += (hl.umax[l] + 31) / 32;
            so += hl.topk[l];
        }
    }
    for (int l = 0; l < hl.levels; ++l)
        for (int c = threadIdx.x; c < hl.topk[l]; c += blockDim.x)
            sels[soff[l] + c] = hl.sel[l][(size_t)pr * hl.topk[l] + c];
    __syncthreads();
    for (int l = 0; l < hl.levels; ++l)
        for (int c = threadIdx.x; c < hl.topk[l]; c += blockDim.x) {
            const int x = sels[soff[l] + c];
            if (x >= 0) atomicOr(&bits[off[l] + (x >> 5)], 1u << (x & 31));
        }
    __syncthreads();
    int U[kMaxLevels];
    hier_units(p, hl, n, U);
    const int M = U[0];
    const float scale = rsqrtf((float)p.d) * 1.4426950408889634f;  // log2 domain
    const T* kr = static_cast<const T*>(p.k_raw) + (size_t)pr * p.n_max * p.d;
    const T* vr = static_cast<const T*>(p.v_raw) + (size_t)pr * p.n_max * p.d;
    float m_run = -INFINITY, l_run = 0.f;
    float acc[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) acc[r] = 0.f;
    int gi = 0;  // number of the next 32-row group, the same in every warp
    // the warp's groups of `rows` rows at (kb, vb)
    auto rows_of = [&](const T* kb, const T* vb, int rows) {
        for (int r0 = 0; r0 < rows; r0 += 32, ++gi)
            if (gi % nw == warp)
                attend_rows<T>(qs, kb + (size_t)r0 * p.d, vb + (size_t)r0 * p.d,
                               min(32, rows - r0), p.d, scale, m_run, l_run, acc);
    };
    for (int l = hl.levels - 1; l >= 0; --l) {
        int nkept;
        const int nc = hier_count(hl, l, pr, U, p.J, nkept);
        const int ntok = l == 0 ? p.g : hl.gs[l];
        const T* ks = l == 0 ? static_cast<const T*>(p.k_gist) + (size_t)pr * p.M_max * p.g * p.d
                             : static_cast<const T*>(hl.k_sum[l]) + (size_t)pr * hl.umax[l] * ntok * p.d;
        const T* vs = l == 0 ? static_cast<const T*>(p.v_gist) + (size_t)pr * p.M_max * p.g * p.d
                             : static_cast<const T*>(hl.v_sum[l]) + (size_t)pr * hl.umax[l] * ntok * p.d;
        const int* up = l + 1 < hl.levels ? sels + soff[l + 1] : nullptr;
        for (int c = 0; c < nc; ++c) {
            int x;
            if (l == hl.levels - 1) x = c;
            else if (c < nkept * p.J) x = up[c / p.J] * p.J + c % p.J;
            else x = U[l + 1] * p.J + (c - nkept * p.J);
            const bool kept = bits[off[l] + (x >> 5)] >> (x & 31) & 1u;
            if (!kept)
                rows_of(ks + (size_t)x * ntok * p.d, vs + (size_t)x * ntok * p.d, ntok);
            else if (l == 0)
                rows_of(kr + (size_t)x * p.C * p.d, vr + (size_t)x * p.C * p.d, p.C);
        }
    }
    rows_of(kr + (size_t)M * p.C * p.d, vr + (size_t)M * p.C * p.d, n - M * p.C);
    if (lane == 0) {
        wm[warp] = m_run;
        wl[warp] = l_run;
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int i = lane + 32 * r;
        if (i < p.d) wacc[warp * p.d + i] = acc[r];
    }
    __syncthreads();
    float mx = -INFINITY;
    for (int w = 0; w < nw; ++w) mx = fmaxf(mx, wm[w]);
    float L = 0.f;
    for (int w = 0; w < nw; ++w) L += (wm[w] == -INFINITY) ? 0.f : wl[w] * exp2f(wm[w] - mx);
    for (int i = threadIdx.x; i < p.d; i += blockDim.x) {
        float o = 0.f;
        for (int w = 0; w < nw; ++w)
            if (wm[w] != -INFINITY) o += wacc[w * p.d + i] * exp2f(wm[w] - mx);
        outp[i] = L > 0.f ? o / L : 0.f;
    }
}

}  // namespace gen
}  // namespace ssa
