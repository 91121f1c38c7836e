// ssa_prefill.cu -- prefill attention under the gist mask ("Simplified Sparse
// Attention via Gist Tokens", sec. 3.1), run block-sparse over permuted key
// columns (sec. 3.6), with its host-side block plan, and the adaptive top-k
// budget (App. A).  A translation unit of its own: its device code (status
// word, PTX wrappers) shares nothing with the decode kernels' unit, which is
// compiled separately, so adding it changes none of their code.
//
// Kernel design (sm_100a, bf16, d in {64, 128}): one CUDA block of 4 warps per
// (query tile of 64 rows, query head); warp w owns rows 16 w .. 16 w + 15.  The
// block walks the tile's entry list; each key block (64 columns of one part)
// is brought into shared memory by cp.async (16-byte pieces, 128-byte rows
// XOR-swizzled so that ldmatrix reads are conflict-free, double-buffered so
// the next block's copy overlaps this block's math).  S = Q K^T and O += P V
// run on mma.sync m16n8k16 (bf16 in, fp32 accumulate); P enters the second
// product as a bf16 pair (value + rounding residue), so the output carries
// fp32-level accuracy.  The softmax is online (running maximum and sum per
// row, base 2).  The element mask is evaluated only in partial blocks: each
// row's visible columns are one interval per part (see include/ssa.h).
#include "../../include/ssa.h"

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdarg>
#include <cstdint>
#include <cmath>
#include <cstdio>
#include <string>
#include <vector>

namespace ssa_pf {

constexpr int kBM = SSA_PREFILL_BM;
constexpr int kBN = SSA_PREFILL_BN;
constexpr int kTileInts = SSA_PREFILL_TILE_INTS;
constexpr int kWarps = kBM / 16;
constexpr int kThreads = kWarps * 32;
static_assert(kBM == 64 && kBN == 64, "the kernel's fragment loops assume 64 x 64 tiles");

// ------------------------------------------------------------ device side ---

// First plan error since the last read (atomicCAS 0 -> code).
static __device__ int g_status = 0;
static __device__ int g_status_taken = 0;
static __global__ void take_status_kernel() { g_status_taken = atomicExch(&g_status, 0); }

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte global -> shared copy; src_bytes = 0 writes zeros and reads nothing.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_one() {
    asm volatile("cp.async.wait_group 1;" ::: "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t& r0, uint32_t& r1,
                                              uint32_t& r2, uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

// d += A (16 x 16, row) * B (16 x 8, col); bf16 in, fp32 accumulate.
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// (x0, x1) as a bf16 pair plus the bf16 pair of what rounding left out.
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
    __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
    __nv_bfloat162 l = __floats2bfloat162_rn(x0 - __bfloat162float(h.x),
                                             x1 - __bfloat162float(h.y));
    hi = *reinterpret_cast<uint32_t*>(&h);
    lo = *reinterpret_cast<uint32_t*>(&l);
}

// Shared address of 16-byte piece `u` of row `row` in a [kBN, D] bf16 block:
// D / 64 planes of kBN rows x 128 bytes, pieces XOR-swizzled by row & 7.
__device__ __forceinline__ uint32_t swz(uint32_t base, int row, int u) {
    return base + (u >> 3) * (kBN * 128) + row * 128 + (((u & 7) ^ (row & 7)) << 4);
}

struct Args {
    const __nv_bfloat16* q[2];  // [part]: 0 raw rows, 1 gist rows
    const __nv_bfloat16* k[2];  // [part]: 0 gist columns, 1 raw columns
    const __nv_bfloat16* v[2];
    float* o[2];                // [part of the rows]
    const int32_t* tiles;
    const int32_t* entries;
    long long n_tiles, n_entries;
    int B, Hq, Hkv, G, n_max, C, g;
    long long gr_max;           // M_max * g rows of the gist arrays
    float scale_log2;           // log2(e) / sqrt(d)
};

template <int D>
__global__ void __launch_bounds__(kThreads, D == 64 ? 3 : 1) prefill_kernel(Args a) {
    extern __shared__ __align__(128) unsigned char smem[];
    constexpr int kBlockBytes = kBN * D * 2;   // one K or V block
    constexpr int kPieces = kBN * (D / 8);     // 16-byte pieces per block
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g8 = lane >> 2, tig = lane & 3;

    const long long tile = blockIdx.x / a.Hq;
    const int h = int(blockIdx.x % a.Hq);
    const int j = h / a.G;
    const int32_t* T = a.tiles + tile * kTileInts;
    const int b = T[0], kind = T[1], r0 = T[2], rows = T[3], n = T[4];
    const long long begin = T[5];
    const int count = T[6];

    // The plan must fit the arrays; otherwise skip the tile (uniform branch).
    const long long M = (a.C > 0 && n >= 0) ? n / a.C : 0;
    const long long cnt_g = M * a.g, cnt_r = n;  // columns of part 0 (gist), 1 (raw)
    const long long row_cnt = kind == 0 ? cnt_r : cnt_g;
    const bool ok = b >= 0 && b < a.B && (kind == 0 || kind == 1) && n >= 0 && n <= a.n_max &&
                    r0 >= 0 && rows >= 1 && rows <= kBM && (long long)r0 + rows <= row_cnt &&
                    begin >= 0 && count >= 0 && begin + count <= a.n_entries;
    if (!ok) {
        if (threadIdx.x == 0) atomicCAS(&g_status, 0, (int)SSA_ERR_DEVICE_STATUS);
        return;
    }

    const long long q_rows = kind == 0 ? (long long)a.n_max : a.gr_max;
    const __nv_bfloat16* qb = (kind == 0 ? a.q[0] : a.q[1]) + ((long long)b * a.Hq + h) * q_rows * D;
    float* ob = (kind == 0 ? a.o[0] : a.o[1]) + ((long long)b * a.Hq + h) * q_rows * D;
    const long long kv_g = ((long long)b * a.Hkv + j) * a.gr_max * D;
    const long long kv_r = ((long long)b * a.Hkv + j) * (long long)a.n_max * D;

    // Q fragments of this warp's 16 rows (zeros past the valid rows).
    uint32_t qa[D / 16][4];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const int lr = 16 * warp + g8 + 8 * half;
        const bool v = lr < rows;
        const __nv_bfloat16* qr = qb + (long long)(r0 + (v ? lr : 0)) * D + 2 * tig;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
            qa[kk][half] = v ? *reinterpret_cast<const uint32_t*>(qr + 16 * kk) : 0u;
            qa[kk][2 + half] = v ? *reinterpret_cast<const uint32_t*>(qr + 16 * kk + 8) : 0u;
        }
    }

    // Visible interval of each of this thread's two rows in each column part
    // (the gist part's always starts at 0).
    long long hi_g[2], lo_r[2], hi_r[2];
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        const long long r = r0 + 16 * warp + g8 + 8 * half;
        if (kind == 0) {
            const long long m = r / a.C;
            hi_g[half] = m * a.g;
            lo_r[half] = m * a.C;
            hi_r[half] = r + 1;
        } else {
            const long long m = r / a.g;
            hi_g[half] = r + 1;
            lo_r[half] = m * a.C;
            hi_r[half] = m * a.C + a.C;
        }
    }

    const uint32_t sbase = smem_u32(smem);
    // Entry e of the list: its part, first column and whether it can be used.
    auto entry_of = [&](int e, int& part, long long& c0, bool& full) -> bool {
        const int32_t x = a.entries[begin + e];
        part = (x >> 1) & 1;
        c0 = (long long)(x >> 2) * kBN;
        const long long cnt = part ? cnt_r : cnt_g;
        full = (x & 1) && c0 + kBN <= cnt;
        return x >= 0 && c0 < cnt;
    };
    auto load = [&](int e, int stage) {
        int part;
        long long c0;
        bool full;
        if (!entry_of(e, part, c0, full)) return;
        const uint32_t ks = sbase + stage * 2 * kBlockBytes, vs = ks + kBlockBytes;
        const __nv_bfloat16* kr = part ? a.k[1] + kv_r : a.k[0] + kv_g;
        const __nv_bfloat16* vr = part ? a.v[1] + kv_r : a.v[0] + kv_g;
        const long long cnt = part ? cnt_r : cnt_g;
        for (int p = threadIdx.x; p < kPieces; p += kThreads) {
            const int row = p / (D / 8), u = p % (D / 8);
            const bool v = c0 + row < cnt;
            const long long off = (v ? (c0 + row) * D : 0) + u * 8;
            cp_async16(swz(ks, row, u), kr + off, v ? 16 : 0);
            cp_async16(swz(vs, row, u), vr + off, v ? 16 : 0);
        }
    };

    float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
    float acc[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[i][c] = 0.f;

    if (count > 0) load(0, 0);
    cp_async_commit();
    for (int e = 0; e < count; ++e) {
        if (e + 1 < count) load(e + 1, (e + 1) & 1);
        cp_async_commit();
        cp_async_wait_one();
        __syncthreads();

        int part;
        long long c0;
        bool full;
        const bool usable = entry_of(e, part, c0, full);
        if (!usable) {
            if (threadIdx.x == 0) atomicCAS(&g_status, 0, (int)SSA_ERR_DEVICE_STATUS);
        } else {
            const uint32_t ks = sbase + (e & 1) * 2 * kBlockBytes, vs = ks + kBlockBytes;
            // S = Q K^T: 8 tiles of 8 columns
            float s[8][4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
#pragma unroll
                for (int c = 0; c < 4; ++c) s[2 * i][c] = s[2 * i + 1][c] = 0.f;
                const int row = 16 * i + ((lane >> 4) << 3) + (lane & 7);
                const int csel = (lane >> 3) & 1;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(swz(ks, row, 2 * kk + csel), b0, b1, b2, b3);
                    mma16816(s[2 * i], qa[kk], b0, b1);
                    mma16816(s[2 * i + 1], qa[kk], b2, b3);
                }
            }
            // scale to base 2, mask partial blocks, online softmax
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const long long lo = part ? lo_r[half] : 0;
                const long long hi = part ? hi_r[half] : hi_g[half];
                float mx = -INFINITY;
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                    for (int c2 = 0; c2 < 2; ++c2) {
                        const int c = 2 * half + c2;
                        float x = s[nt][c] * a.scale_log2;
                        if (!full) {
                            const long long col = c0 + 8 * nt + 2 * tig + c2;
                            if (col < lo || col >= hi) x = -INFINITY;
                        }
                        s[nt][c] = x;
                        mx = fmaxf(mx, x);
                    }
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                const float m_new = fmaxf(m_run[half], mx);
                const float m_use = m_new == -INFINITY ? 0.f : m_new;
                const float alpha = exp2f(m_run[half] - m_use);
                m_run[half] = m_new;
                l_run[half] *= alpha;
#pragma unroll
                for (int dn = 0; dn < D / 8; ++dn) {
                    acc[dn][2 * half] *= alpha;
                    acc[dn][2 * half + 1] *= alpha;
                }
#pragma unroll
                for (int nt = 0; nt < 8; ++nt)
#pragma unroll
                    for (int c2 = 0; c2 < 2; ++c2) {
                        const float p = exp2f(s[nt][2 * half + c2] - m_use);
                        s[nt][2 * half + c2] = p;
                        l_run[half] += p;
                    }
            }
            // O += P V, P as value + residue
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                uint32_t ph[4], pl[4];
                split2(s[2 * i][0], s[2 * i][1], ph[0], pl[0]);
                split2(s[2 * i][2], s[2 * i][3], ph[1], pl[1]);
                split2(s[2 * i + 1][0], s[2 * i + 1][1], ph[2], pl[2]);
                split2(s[2 * i + 1][2], s[2 * i + 1][3], ph[3], pl[3]);
                const int row = 16 * i + (lane & 15);
                const int csel = lane >> 4;
#pragma unroll
                for (int mm = 0; mm < D / 16; ++mm) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_trans(swz(vs, row, 2 * mm + csel), b0, b1, b2, b3);
                    mma16816(acc[2 * mm], ph, b0, b1);
                    mma16816(acc[2 * mm], pl, b0, b1);
                    mma16816(acc[2 * mm + 1], ph, b2, b3);
                    mma16816(acc[2 * mm + 1], pl, b2, b3);
                }
            }
        }
        __syncthreads();
    }

    // o = acc / row sum, valid rows only
#pragma unroll
    for (int half = 0; half < 2; ++half) {
        float l = l_run[half];
        l += __shfl_xor_sync(0xffffffffu, l, 1);
        l += __shfl_xor_sync(0xffffffffu, l, 2);
        const int lr = 16 * warp + g8 + 8 * half;
        if (lr >= rows) continue;
        const float inv = l > 0.f ? 1.f / l : 0.f;
        float* orow = ob + (long long)(r0 + lr) * D + 2 * tig;
#pragma unroll
        for (int dn = 0; dn < D / 8; ++dn)
            *reinterpret_cast<float2*>(orow + 8 * dn) =
                make_float2(acc[dn][2 * half] * inv, acc[dn][2 * half + 1] * inv);
    }
}

// -------------------------------------------------------------- host side ---

thread_local std::string g_err;

ssa_status fail(ssa_status s, const char* fmt, ...) {
    char buf[256];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_err = buf;
    return s;
}

// Visible interval [lo, hi) of the tile's rows in one column part: the union
// (ulo, uhi) and the intersection (ilo, ihi) of the rows' intervals.
struct Span {
    long long ulo, uhi, ilo, ihi;
};

// Tile rows [r0, r1) of part `kind`; part 0 = gist columns, 1 = raw columns.
Span span_of(int kind, int part, long long r0, long long r1, long long C, long long g) {
    if (kind == 0) {  // raw rows i: gist [0, m g), raw [m C, i + 1)
        const long long m0 = r0 / C, m1 = (r1 - 1) / C;
        if (part == 0) return {0, m1 * g, 0, m0 * g};
        return {m0 * C, r1, m1 * C, r0 + 1};
    }
    // gist rows r = m g + t: gist [0, r + 1), raw [m C, m C + C)
    const long long m0 = r0 / g, m1 = (r1 - 1) / g;
    if (part == 0) return {0, r1, 0, r0 + 1};
    return {m0 * C, (m1 + 1) * C, m1 * C, m0 * C + C};
}

// Walks the plan; with out arrays given, writes it.  Returns the counts.
ssa_status build_plan(int32_t B, const int32_t* lens, int32_t n_max, int32_t C, int32_t g,
                      int64_t* n_tiles, int64_t* n_entries, int32_t* tiles, int32_t* entries) {
    if (B < 0 || !lens || C < 1 || g < 1 || n_max < 0 || n_max % C)
        return fail(SSA_ERR_INVALID_ARG, "prefill plan: bad B, C, g or n_max");
    for (int b = 0; b < B; ++b)
        if (lens[b] < 0 || lens[b] > n_max)
            return fail(SSA_ERR_INVALID_ARG, "prefill plan: seq_lens[%d] = %d outside [0, %d]",
                        b, lens[b], n_max);
    long long nt = 0, ne = 0;
    struct Key {
        int count, b, kind, r0;
        long long idx;
    };
    std::vector<Key> order;
    for (int b = 0; b < B; ++b) {
        const long long n = lens[b], M = n / C;
        const long long cnt[2] = {M * g, n};
        for (int kind = 0; kind < 2; ++kind) {
            const long long rows_total = kind == 0 ? n : M * g;
            for (long long r0 = 0; r0 < rows_total; r0 += kBM) {
                const long long r1 = std::min(rows_total, r0 + kBM);
                const long long first = ne;
                for (int part = 0; part < 2; ++part) {
                    const Span sp = span_of(kind, part, r0, r1, C, g);
                    if (sp.uhi <= sp.ulo) continue;
                    for (long long blk = sp.ulo / kBN; blk <= (sp.uhi - 1) / kBN; ++blk) {
                        const long long c0 = blk * kBN;
                        const bool full = c0 >= sp.ilo && c0 + kBN <= sp.ihi && c0 + kBN <= cnt[part];
                        if (entries) entries[ne] = (int32_t)((blk << 2) | (part << 1) | (full ? 1 : 0));
                        ++ne;
                        if (ne > INT32_MAX)
                            return fail(SSA_ERR_UNSUPPORTED, "prefill plan: more than 2^31 - 1 entries");
                    }
                }
                if (tiles) {
                    int32_t* t = tiles + nt * kTileInts;
                    t[0] = b;
                    t[1] = kind;
                    t[2] = (int32_t)r0;
                    t[3] = (int32_t)(r1 - r0);
                    t[4] = (int32_t)n;
                    t[5] = (int32_t)first;
                    t[6] = (int32_t)(ne - first);
                    t[7] = 0;
                    order.push_back({(int)(ne - first), b, kind, (int)r0, nt});
                }
                ++nt;
            }
        }
    }
    if (tiles && nt > 1) {
        // longest tiles first; ties by (b, part, r0)
        std::stable_sort(order.begin(), order.end(), [](const Key& x, const Key& y) {
            return x.count > y.count;
        });
        std::vector<int32_t> copy(tiles, tiles + nt * kTileInts);
        for (long long i = 0; i < nt; ++i)
            std::copy(copy.begin() + order[i].idx * kTileInts,
                      copy.begin() + (order[i].idx + 1) * kTileInts, tiles + i * kTileInts);
    }
    *n_tiles = nt;
    *n_entries = ne;
    return SSA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <int D>
cudaError_t launch(const Args& a, long long blocks, cudaStream_t stream) {
    const int smem = 2 * 2 * kBN * D * 2;
    // per device: set on every call (a host-side attribute write)
    cudaError_t e = cudaFuncSetAttribute(prefill_kernel<D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    prefill_kernel<D><<<(unsigned)blocks, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace ssa_pf

using namespace ssa_pf;

extern "C" {

SSA_API ssa_status ssa_adaptive_topk(int64_t n_kv, int32_t L, int32_t G, int32_t J, int32_t* k) {
    g_err.clear();
    if (!k || n_kv < 0 || L < 1 || G < 1 || J < 1)
        return fail(SSA_ERR_INVALID_ARG, "ssa_adaptive_topk: need n_kv >= 0, L, G, J >= 1");
    // floor(n_kv / (L J G L)) by successive divisions (no overflow of the product)
    const long long v = (long long)(n_kv / L / J / G / L) + 1;
    if (v > INT32_MAX) return fail(SSA_ERR_UNSUPPORTED, "ssa_adaptive_topk: k above 2^31 - 1");
    *k = (int32_t)v;
    return SSA_OK;
}

SSA_API ssa_status ssa_prefill_plan_size(int32_t B, const int32_t* seq_lens_host, int32_t n_max,
                                         int32_t C, int32_t g, int64_t* n_tiles,
                                         int64_t* n_entries) {
    g_err.clear();
    if (!n_tiles || !n_entries) return fail(SSA_ERR_INVALID_ARG, "ssa_prefill_plan_size: NULL output");
    return build_plan(B, seq_lens_host, n_max, C, g, n_tiles, n_entries, nullptr, nullptr);
}

SSA_API ssa_status ssa_prefill_plan(int32_t B, const int32_t* seq_lens_host, int32_t n_max,
                                    int32_t C, int32_t g, int32_t* tiles, int64_t tiles_cap,
                                    int32_t* entries, int64_t entries_cap) {
    g_err.clear();
    int64_t nt = 0, ne = 0;
    ssa_status s = build_plan(B, seq_lens_host, n_max, C, g, &nt, &ne, nullptr, nullptr);
    if (s != SSA_OK) return s;
    if ((nt > 0 && !tiles) || (ne > 0 && !entries) || tiles_cap < nt || entries_cap < ne)
        return fail(SSA_ERR_INVALID_ARG, "ssa_prefill_plan: need %lld tiles and %lld entries",
                    (long long)nt, (long long)ne);
    return build_plan(B, seq_lens_host, n_max, C, g, &nt, &ne, tiles, entries);
}

SSA_API ssa_status ssa_prefill(const ssa_shape* shape, const void* q_raw, const void* q_gist,
                               const void* k_raw, const void* k_gist, const void* v_raw,
                               const void* v_gist, int32_t C, int32_t g,
                               const int32_t* plan_tiles, int64_t n_tiles,
                               const int32_t* plan_entries, int64_t n_entries, float* o_raw,
                               float* o_gist, cudaStream_t stream) {
    g_err.clear();
    if (!shape) return fail(SSA_ERR_INVALID_ARG, "ssa_prefill: NULL shape");
    const ssa_shape& s = *shape;
    if (s.B < 0 || s.Hq < 1 || s.Hkv < 1 || s.Hq % s.Hkv || s.n_max < 0 || C < 1 || g < 1 ||
        s.n_max % C || n_tiles < 0 || n_entries < 0)
        return fail(SSA_ERR_INVALID_ARG, "ssa_prefill: bad sizes");
    if (s.dtype != SSA_BF16 || (s.d != 64 && s.d != 128))
        return fail(SSA_ERR_UNSUPPORTED, "ssa_prefill: bf16 with d in {64, 128} only");
    if (n_tiles == 0 || s.B == 0) return SSA_OK;
    const bool gists = (long long)(s.n_max / C) * g > 0;
    if (!q_raw || !k_raw || !v_raw || !o_raw || !plan_tiles || (n_entries > 0 && !plan_entries) ||
        (gists && (!q_gist || !k_gist || !v_gist || !o_gist)))
        return fail(SSA_ERR_INVALID_ARG, "ssa_prefill: NULL pointer");
    const void* ptrs[] = {q_raw, q_gist, k_raw, k_gist, v_raw, v_gist, o_raw, o_gist, plan_tiles};
    for (const void* p : ptrs)
        if (p && !aligned16(p)) return fail(SSA_ERR_INVALID_ARG, "ssa_prefill: pointer not 16-byte aligned");
    const long long blocks = (long long)n_tiles * s.Hq;
    if (blocks > INT32_MAX) return fail(SSA_ERR_UNSUPPORTED, "ssa_prefill: more than 2^31 - 1 blocks");

    Args a;
    a.q[0] = static_cast<const __nv_bfloat16*>(q_raw);
    a.q[1] = static_cast<const __nv_bfloat16*>(q_gist);
    a.k[0] = static_cast<const __nv_bfloat16*>(k_gist);
    a.k[1] = static_cast<const __nv_bfloat16*>(k_raw);
    a.v[0] = static_cast<const __nv_bfloat16*>(v_gist);
    a.v[1] = static_cast<const __nv_bfloat16*>(v_raw);
    a.o[0] = o_raw;
    a.o[1] = o_gist;
    a.tiles = plan_tiles;
    a.entries = plan_entries;
    a.n_tiles = n_tiles;
    a.n_entries = n_entries;
    a.B = s.B;
    a.Hq = s.Hq;
    a.Hkv = s.Hkv;
    a.G = s.Hq / s.Hkv;
    a.n_max = s.n_max;
    a.C = C;
    a.g = g;
    a.gr_max = (long long)(s.n_max / C) * g;
    a.scale_log2 = (float)(1.4426950408889634 / std::sqrt((double)s.d));
    cudaError_t e = s.d == 64 ? launch<64>(a, blocks, stream) : launch<128>(a, blocks, stream);
    if (e != cudaSuccess) return fail(SSA_ERR_CUDA, "ssa_prefill: %s", cudaGetErrorString(e));
    return SSA_OK;
}

SSA_API ssa_status ssa_prefill_get_status(int32_t* host_code, cudaStream_t stream) {
    g_err.clear();
    if (!host_code) return fail(SSA_ERR_INVALID_ARG, "ssa_prefill_get_status: NULL output");
    take_status_kernel<<<1, 1, 0, stream>>>();
    cudaError_t e = cudaGetLastError();
    int v = 0;
    if (e == cudaSuccess)
        e = cudaMemcpyFromSymbolAsync(&v, g_status_taken, sizeof(int), 0, cudaMemcpyDeviceToHost,
                                      stream);
    if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
    if (e != cudaSuccess)
        return fail(SSA_ERR_CUDA, "ssa_prefill_get_status: %s", cudaGetErrorString(e));
    *host_code = v;
    return SSA_OK;
}

SSA_API const char* ssa_prefill_last_error(void) { return g_err.c_str(); }

}  // extern "C"
