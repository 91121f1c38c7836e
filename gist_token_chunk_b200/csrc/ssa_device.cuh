// ssa_device.cuh -- device building blocks shared by the libssa kernels:
// PTX wrappers (mbarrier, TMA, ldmatrix, mma.sync), bounded flag waits, the
// device status word, an order-preserving float key, a block-wide exclusive
// scan and the deterministic block top-k used by chunk selection.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssa {

// Library-wide device status word (one per device that loads the library).
// Written with atomicCAS(0 -> code) so the first error since the last read
// wins; read and cleared from the host by ssa_get_device_status.  Defined
// here: this header belongs to the library's single device translation unit.
__device__ int g_device_status = 0;

constexpr int kStatusBadInput = 5;   // == SSA_ERR_DEVICE_STATUS
constexpr int kStatusTimeout = 6;    // == SSA_ERR_DEVICE_TIMEOUT

__device__ __forceinline__ void report_status(int code) {
    atomicCAS(&g_device_status, 0, code);
}

// ---------------------------------------------------------------- keys ---
// Order-preserving map of an fp32 score to uint32: a larger score gives a
// larger key; -0 is folded onto +0 and NaN onto -inf (NaN ranks as -inf).
__device__ __forceinline__ uint32_t score_key(float f) {
    uint32_t u = __float_as_uint(f);
    if ((u & 0x7fffffffu) > 0x7f800000u) u = 0xff800000u;  // NaN -> -inf
    if ((u << 1) == 0u) u = 0u;                            // -0 -> +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// ------------------------------------------------------------- memory ---
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release(int* p, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint64_t now_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Poll *p until it is >= target, for at most `limit_ns` nanoseconds.  On
// running out it records a timeout in the status word and returns false
// (never blocks for longer).
__device__ __forceinline__ bool wait_geq(const int* p, int target, long long limit_ns) {
    const uint64_t t0 = now_ns();
    for (;;) {
        if (ld_acquire(p) >= target) return true;
        if ((long long)(now_ns() - t0) > limit_ns) break;
        __nanosleep(128);
    }
    report_status(kStatusTimeout);
    return false;
}

// ----------------------------------------------------------- mbarrier ---
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete, for at most
// `limit_ns` nanoseconds (plus one hardware suspend interval).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, long long limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = now_ns();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((long long)(now_ns() - t0) > limit_ns) break;
    }
    report_status(kStatusTimeout);
    return false;
}

// ---------------------------------------------------------------- TMA ---
// 2-D tiled bulk tensor load global -> shared, completing on `bar`
// (no multicast; the destination is this CTA's shared memory).
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
        : "memory");
}

// 1-D bulk copy global -> shared (16-byte aligned addresses, size % 16 == 0).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------- tensor-core ops ---
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

// D += A(16x16 bf16, row) * B(16x8 bf16, col), fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

// Split (lo, hi) into a bf16 pair plus the bf16 pair of the rounding error,
// so that hi_part + lo_part carries ~16 significant bits of each value.
__device__ __forceinline__ void split_bf16(float x0, float x1, uint32_t& big, uint32_t& small) {
    __nv_bfloat162 b = __floats2bfloat162_rn(x0, x1);
    float r0 = x0 - __bfloat162float(b.x);
    float r1 = x1 - __bfloat162float(b.y);
    big = *reinterpret_cast<uint32_t*>(&b);
    small = pack_bf16(r0, r1);
}

// Named barrier over `nthreads` threads (a multiple of 32) with id `id`.
__device__ __forceinline__ void named_sync(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ------------------------------------------------------ block scan ---
// Exclusive prefix sum over the NT threads that call it together; `sync`
// synchronises exactly those threads; `sm` holds NT/32 + 1 ints.
template <int NT, class Sync>
__device__ __forceinline__ int block_exclusive_scan(int v, int* sm, int& total, Sync sync) {
    const int lane = threadIdx.x & 31;
    const int warp = (threadIdx.x & (NT - 1)) >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sm[warp] = x;
    sync();
    int base = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < NT / 32; ++w) {
        int s = sm[w];
        if (w < warp) base += s;
        tot += s;
    }
    sync();
    total = tot;
    return base + x - v;
}

// ---------------------------------------------------- block top-k ---
struct TopkScratch {
    int hist[256];
    int bcast[4];
    int scan[8];
};

// Deterministic top-k over vals[0..n) (sec. 3.3 "top-k chunks"): selects the
// k = min(topk, n) largest values, ties to the lower position, and writes
// map(i) for the selected positions i in ascending order of i to
// out[0..k), then -1 to out[k..topk).  If `mask` is not null, bit map(i) of
// `mask` is set for each selected i (the caller zeroes it beforehand).
// Runs on the NT threads that call it together; vals is read with
// L2-coherent loads so it may have been written by other blocks of the same
// launch.  Method: 4-pass MSB-first radix select on the order-preserving
// 32-bit key finds the k-th largest key tau and how many keys equal to tau
// are taken; a prefix count in index order then picks the lowest-index ties.
template <int NT, class Map, class Sync>
__device__ void block_topk(const float* vals, int n, int topk, int* out, uint32_t* mask, Map map,
                           TopkScratch& sc, Sync sync) {
    const int tid = threadIdx.x & (NT - 1);
    const int k = topk < n ? topk : n;
    if (k <= 0) {
        for (int c = tid; c < topk; c += NT) out[c] = -1;
        return;
    }
    if (k == n) {
        for (int c = tid; c < topk; c += NT) out[c] = c < n ? map(c) : -1;
        if (mask)
            for (int c = tid; c < n; c += NT) {
                int m = map(c);
                atomicOr(&mask[m >> 5], 1u << (m & 31));
            }
        return;
    }
    uint32_t prefix = 0, pmask = 0;
    int remaining = k;
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += NT) sc.hist[i] = 0;
        sync();
        for (int i = tid; i < n; i += NT) {
            uint32_t key = score_key(__ldcg(vals + i));
            if ((key & pmask) == prefix) atomicAdd(&sc.hist[(key >> shift) & 255u], 1);
        }
        sync();
        if (tid < 32) {
            const int lane = tid;
            int loc = 0;
#pragma unroll
            for (int b = 0; b < 8; ++b) loc += sc.hist[lane * 8 + b];
            int suf = loc;  // inclusive suffix over lanes >= lane
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                int y = __shfl_down_sync(0xffffffffu, suf, o);
                if (lane + o < 32) suf += y;
            }
            int running = suf - loc;  // keys in buckets above this lane's
#pragma unroll
            for (int b = 7; b >= 0; --b) {
                int c = sc.hist[lane * 8 + b];
                if (running < remaining && running + c >= remaining) {
                    sc.bcast[0] = lane * 8 + b;
                    sc.bcast[1] = running;
                }
                running += c;
            }
        }
        sync();
        const uint32_t digit = (uint32_t)sc.bcast[0];
        remaining -= sc.bcast[1];
        prefix |= digit << shift;
        pmask |= 0xffu << shift;
    }
    const uint32_t tau = prefix;
    const int need_eq = remaining;  // keys equal to tau that are taken

    const int per = (n + NT - 1) / NT;
    const int lo = tid * per;
    const int hi = min(lo + per, n);
    int n_eq = 0;
    for (int i = lo; i < hi; ++i) n_eq += (score_key(__ldcg(vals + i)) == tau);
    int tot;
    int eq_rank = block_exclusive_scan<NT>(n_eq, sc.scan, tot, sync);
    int n_sel = 0;
    {
        int r = eq_rank;
        for (int i = lo; i < hi; ++i) {
            uint32_t key = score_key(__ldcg(vals + i));
            if (key > tau) {
                ++n_sel;
            } else if (key == tau) {
                n_sel += (r < need_eq);
                ++r;
            }
        }
    }
    int pos = block_exclusive_scan<NT>(n_sel, sc.scan, tot, sync);
    {
        int r = eq_rank;
        for (int i = lo; i < hi; ++i) {
            uint32_t key = score_key(__ldcg(vals + i));
            bool take = false;
            if (key > tau) {
                take = true;
            } else if (key == tau) {
                take = (r < need_eq);
                ++r;
            }
            if (take) {
                int m = map(i);
                out[pos++] = m;
                if (mask) atomicOr(&mask[m >> 5], 1u << (m & 31));
            }
        }
    }
    for (int c = k + tid; c < topk; c += NT) out[c] = -1;
}

}  // namespace ssa
