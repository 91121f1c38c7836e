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

__device__ __forceinline__ int ld_relaxed(const int* p) {
    int v;
    asm volatile("ld.relaxed.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void fence_acquire_gpu() {
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
}

__device__ __forceinline__ int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

// Release increment without a returned value (fire and forget).
__device__ __forceinline__ void red_release_add(int* p, int v) {
    asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void st_release(int* p, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ uint64_t now_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

// Wait bounds count SM clock cycles (clock64 is a cheap per-SM counter; the
// global timer is not polled in hot loops).  2 cycles per ns covers SM clocks
// up to 2 GHz, so a bound of N ns never ends a wait earlier than N ns.
__device__ __forceinline__ long long wait_cycles(long long limit_ns) { return 2 * limit_ns; }

// Poll *p until it is >= target, for at most `limit_ns` nanoseconds, then
// acquire.  Relaxed polls with a capped exponential back-off keep many
// waiting blocks from saturating the L2 slice that holds the word.  On
// running out it records a timeout in the status word and returns false
// (never blocks for longer).
__device__ __forceinline__ bool wait_geq(const int* p, int target, long long limit_ns) {
    if (ld_relaxed(p) >= target) {
        fence_acquire_gpu();
        return true;
    }
    const long long c0 = clock64(), lim = wait_cycles(limit_ns);
    unsigned sleep_ns = 32;
    for (;;) {
        __nanosleep(sleep_ns);
        if (sleep_ns < 128) sleep_ns *= 2;
        if (ld_relaxed(p) >= target) {
            fence_acquire_gpu();
            return true;
        }
        if (clock64() - c0 > lim) break;
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

// try_wait with a suspend-time hint: the warp sleeps in hardware until the
// phase completes or `hint_ns` passes, instead of re-polling shared memory
// (polling warps would compete with the neighbour block for the SM's
// shared-memory pipe).
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity,
                                                    uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Non-blocking test of phase completion (never suspends the warp).
__device__ __forceinline__ bool mbar_test_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete, for at most
// `limit_ns` nanoseconds (plus one suspend interval).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, long long limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const long long c0 = clock64(), lim = wait_cycles(limit_ns);
    for (;;) {
        if (mbar_test_wait(bar, parity)) return true;
        __nanosleep(20);
        if (clock64() - c0 > lim) break;
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

// The same with an L2 eviction-priority policy (from l2_policy_*).
__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* map, int x, int y,
                                                 uint64_t* bar, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

// L2 policies: keep lines that are read again soon; drop single-use lines first.
__device__ __forceinline__ uint64_t l2_policy_evict_last() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}
__device__ __forceinline__ uint64_t l2_policy_evict_first() {
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
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

// Barrier over `nthreads` threads that also ORs a predicate across them.
__device__ __forceinline__ bool named_sync_or(int id, int nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "barrier.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
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
struct NoProbe {
    __device__ void operator()(int) const {}
};

// ------------------------------------------------- warp-level ranking ---
// Entries are 64-bit composites key << 32 | ~position (score_key order, ties
// to the lower position: a larger composite ranks first).  A composite with a
// zero key part (e.g. 1) is a placeholder below every real entry; 0 itself
// means "not written yet" wherever entries are published.

__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* p) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ unsigned long long cmax_u64(unsigned long long a, unsigned long long b) {
    return a > b ? a : b;
}
__device__ __forceinline__ unsigned long long cmin_u64(unsigned long long a, unsigned long long b) {
    return a < b ? a : b;
}

// Bitonic sort of the warp's 32 entries (one per lane) into descending order
// (lane 0 holds the largest).
__device__ __forceinline__ unsigned long long warp_sort_desc(unsigned long long x, int lane) {
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1)
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            const unsigned long long o = __shfl_xor_sync(0xffffffffu, x, j);
            // runs with (lane & k) == 0 descend, the others ascend; the final
            // run (k = 32) descends
            const bool keep_max = ((lane & j) == 0) == ((lane & k) == 0);
            x = keep_max ? cmax_u64(x, o) : cmin_u64(x, o);
        }
    return x;
}

// The 32 largest of two descending 32-entry lists a and b, descending: the
// elementwise maximum of a and reversed b is a bitonic sequence holding them,
// which one bitonic merge pass sorts.
__device__ __forceinline__ unsigned long long warp_merge_desc(unsigned long long a,
                                                              unsigned long long b, int lane) {
    const unsigned long long br = __shfl_sync(0xffffffffu, b, 31 - lane);
    unsigned long long x = cmax_u64(a, br);
#pragma unroll
    for (int j = 16; j > 0; j >>= 1) {
        const unsigned long long o = __shfl_xor_sync(0xffffffffu, x, j);
        x = (lane & j) == 0 ? cmax_u64(x, o) : cmin_u64(x, o);
    }
    return x;
}

// Bitonic sort of the warp's 32 ints into ascending order.
__device__ __forceinline__ int warp_sort_asc(int x, int lane) {
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1)
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            const int o = __shfl_xor_sync(0xffffffffu, x, j);
            const bool keep_min = ((lane & j) == 0) == ((lane & k) == 0);
            x = keep_min ? min(x, o) : max(x, o);
        }
    return x;
}

constexpr int kTopkCandCap = 512;  // candidates the filtered selection ranks directly
constexpr int kTopkRegPer = 16;    // values per thread the filtered selection holds

struct TopkScratch {
    int hist[256];
    int bcast[4];
    int scan[8];
    alignas(16) uint32_t tmax[128];           // per-thread key maxima (NT <= 128)
    // candidates: key << 32 | ~position (a larger value ranks first)
    alignas(16) unsigned long long ccomp[kTopkCandCap];
};

// Deterministic top-k over vals[0..n) (sec. 3.3 "top-k chunks"): selects the
// k = min(topk, n) largest values, ties to the lower position, and writes the
// selected positions in ascending order to out[0..k), then -1 to
// out[k..topk).  Runs on the NT (<= 128) threads that call it together.
// vals is read with L2-coherent loads (it may have been written by other
// blocks of the same launch), in batches so that many loads are in flight.
//
// Filtered path (k <= NT, n <= NT * kTopkRegPer): one round of loads puts
// every value in registers (strided, coalesced); each thread takes its
// maximum key; the k-th largest of those NT maxima is a lower bound tau on
// the k-th largest key (k distinct keys reach it), so every selected key --
// ties at the boundary included -- is >= tau.  The keys >= tau go to shared
// memory as (key, position) pairs and are ranked exactly by counting (larger
// key first, then lower position); the k best are then ordered by position.
// Fallback (k > NT, larger n, or more than kTopkCandCap keys >= tau):
// MSB-first radix select on the order-preserving 32-bit key, reading vals
// from L2 per pass.
// If `pub` is not null, each selected position i is also written there as
// pub[rank] = i + 1 (a published copy that is never 0 once written).
// With poll_ns > 0, vals may still be being written by other blocks: a value
// whose bits are all zero is not written yet (writers store +0 as -0), and
// the loads repeat (for at most poll_ns) until every value is present.
// Sync must provide or_(bool): a barrier that ORs a predicate.
template <int NT, class Sync, class Probe = NoProbe>
__device__ __noinline__ void block_topk(const float* vals, int n, int topk, int* out, TopkScratch& sc,
                           Sync sync, Probe probe = Probe(), int* pub = nullptr,
                           long long poll_ns = 0) {
    const int tid = threadIdx.x & (NT - 1);
    const int k = topk < n ? topk : n;
    // polling: wait until every value is present (the filtered path below
    // does this in its own loads)
    auto poll_all = [&]() {
        const int* iv = reinterpret_cast<const int*>(vals);
        const long long c0 = clock64(), lim = wait_cycles(poll_ns);
        for (;;) {
            bool missing = false;
            for (int i = tid; i < n; i += NT) missing |= ld_relaxed(iv + i) == 0;
            // every thread takes the same branch: the vote decides
            const bool expired = clock64() - c0 > lim;
            if (!sync.or_(missing && !expired)) {
                if (missing) report_status(kStatusTimeout);
                break;
            }
            __nanosleep(128);
        }
    };
    const bool filtered = k > 0 && k < n && k <= NT && n <= NT * kTopkRegPer;
    if (poll_ns > 0 && !filtered && n > 0) poll_all();
    if (k <= 0) {
        for (int c = tid; c < topk; c += NT) out[c] = -1;
        return;
    }
    if (k == n) {
        for (int c = tid; c < topk; c += NT) {
            out[c] = c < n ? c : -1;
            if (pub && c < n) pub[c] = c + 1;
        }
        return;
    }
    if (filtered) {
        // one round of loads: every value of the range, held in registers
        uint32_t key[kTopkRegPer];
        if (poll_ns <= 0) {
#pragma unroll
            for (int u = 0; u < kTopkRegPer; ++u) {
                const int i = u * NT + tid;
                key[u] = i < n ? score_key(__ldcg(vals + i)) : 0u;  // 0: below every real key
            }
        } else {
            const int* iv = reinterpret_cast<const int*>(vals);
            const long long c0 = clock64(), lim = wait_cycles(poll_ns);
            unsigned sleep_ns = 32;
            for (;;) {
                bool missing = false;
#pragma unroll
                for (int u = 0; u < kTopkRegPer; ++u) {
                    const int i = u * NT + tid;
                    const int b = i < n ? ld_relaxed(iv + i) : 1;
                    missing |= (b == 0);
                    key[u] = i < n ? score_key(__int_as_float(b)) : 0u;
                }
                // every thread takes the same branch: the vote decides
                const bool expired = clock64() - c0 > lim;
                if (!sync.or_(missing && !expired)) {
                    if (missing) report_status(kStatusTimeout);
                    break;
                }
                __nanosleep(sleep_ns);
                if (sleep_ns < 256) sleep_ns *= 2;
            }
        }
        uint32_t mx = 0u;
#pragma unroll
        for (int u = 0; u < kTopkRegPer; ++u) mx = max(mx, key[u]);
        sc.tmax[tid] = mx;
        if (tid == 0) sc.bcast[2] = 0;
        probe(1);
        sync();
        // tau: the k-th largest of the NT maxima (ties by thread), reached by
        // at least k distinct values, so every selected value is >= tau
        int r0 = 0, r1 = 0, r2 = 0, r3 = 0;  // independent partial counts
        const uint4* tm4 = reinterpret_cast<const uint4*>(sc.tmax);
#pragma unroll
        for (int j4 = 0; j4 < NT / 4; ++j4) {
            const uint4 o = tm4[j4];
            const int j = 4 * j4;
            r0 += int(o.x > mx) | (int(o.x == mx) & int(j < tid));
            r1 += int(o.y > mx) | (int(o.y == mx) & int(j + 1 < tid));
            r2 += int(o.z > mx) | (int(o.z == mx) & int(j + 2 < tid));
            r3 += int(o.w > mx) | (int(o.w == mx) & int(j + 3 < tid));
        }
        const int rank = (r0 + r1) + (r2 + r3);
        probe(7);
        if (rank == k - 1) sc.bcast[3] = (int)mx;
        sync();
        probe(8);
        const uint32_t tau = (uint32_t)sc.bcast[3];
        // candidates (key >= tau) into shared memory, in any order: the
        // ranking below compares (key, position) pairs, never slots.  Each
        // warp reserves room for its candidates with one shared atomic.
        int mine = 0;
#pragma unroll
        for (int u = 0; u < kTopkRegPer; ++u) mine += (key[u] >= tau && key[u] != 0u);
        const int lane = threadIdx.x & 31;
        int incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        int base = 0;
        if (lane == 31 && incl > 0) base = atomicAdd(&sc.bcast[2], incl);
        base = __shfl_sync(0xffffffffu, base, 31) + incl - mine;
#pragma unroll
        for (int u = 0; u < kTopkRegPer; ++u) {
            if (key[u] >= tau && key[u] != 0u) {
                if (base < kTopkCandCap)
                    sc.ccomp[base] = ((unsigned long long)key[u] << 32) |
                                     (uint32_t)~(uint32_t)(u * NT + tid);
                ++base;
            }
        }
        probe(5);
        sync();
        probe(9);
        const int total = sc.bcast[2];
        if (total <= kTopkCandCap - 1) {
            // exact rank of each candidate (pairs of entries per load; an
            // odd count is padded with 0, below every candidate); the k best
            // land in sel[rank]
            int* sel = sc.hist;
            const int total2 = (total + 1) >> 1;
            if (tid == 0 && (total & 1)) sc.ccomp[total] = 0ull;
            if (tid < 4 - (k & 3) && (k & 3)) sel[k + tid] = 0x7fffffff;  // pad for the placement
            sync();
            const ulonglong2* cc2 = reinterpret_cast<const ulonglong2*>(sc.ccomp);
            for (int c = tid; c < total; c += NT) {
                const unsigned long long mine = sc.ccomp[c];
                int ra = 0, rb = 0;
#pragma unroll 4
                for (int o = 0; o < total2; ++o) {
                    const ulonglong2 v = cc2[o];
                    ra += v.x > mine;
                    rb += v.y > mine;
                }
                const int r = ra + rb;
                if (r < k) sel[r] = (int)~(uint32_t)mine;
            }
            sync();
            // ascending positions: place each selected one by counting smaller ones
            if (tid < k) {
                const int mine = sel[tid];
                int pa = 0, pb = 0, pc = 0, pd = 0;
                const int4* s4 = reinterpret_cast<const int4*>(sel);
                for (int j = 0; j < (k + 3) >> 2; ++j) {
                    const int4 v = s4[j];
                    pa += v.x < mine;
                    pb += v.y < mine;
                    pc += v.z < mine;
                    pd += v.w < mine;
                }
                const int pos = (pa + pb) + (pc + pd);
                out[pos] = mine;
                if (pub) pub[pos] = mine + 1;
            }
            for (int c = k + tid; c < topk; c += NT) out[c] = -1;
            probe(3);
            sync();  // sel (the histogram area) is free again
            return;
        }
        // too many keys >= tau (e.g. many equal scores): exact radix path
    }
    uint32_t prefix = 0, pmask = 0;
    int remaining = k;
#pragma unroll 1
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int i = tid; i < 256; i += NT) sc.hist[i] = 0;
        sync();
        for (int i = tid; i < n; i += NT) {
            const uint32_t key = score_key(__ldcg(vals + i));
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
        remaining -= sc.bcast[1];
        prefix |= (uint32_t)sc.bcast[0] << shift;
        pmask |= 0xffu << shift;
    }
    // prefix is now the k-th largest key; `remaining` keys equal to it are taken
    const int need_eq = remaining;
    const int per = (n + NT - 1) / NT;
    const int lo = min(tid * per, n), hi = min(lo + per, n);
    int n_eq = 0;
    for (int i = lo; i < hi; ++i) n_eq += (score_key(__ldcg(vals + i)) == prefix);
    int tot;
    const int eq_rank = block_exclusive_scan<NT>(n_eq, sc.scan, tot, sync);
    int n_sel = 0;
    {
        int r = eq_rank;
        for (int i = lo; i < hi; ++i) {
            const uint32_t key = score_key(__ldcg(vals + i));
            if (key > prefix) {
                ++n_sel;
            } else if (key == prefix) {
                n_sel += (r < need_eq);
                ++r;
            }
        }
    }
    int pos = block_exclusive_scan<NT>(n_sel, sc.scan, tot, sync);
    {
        int r = eq_rank;
        for (int i = lo; i < hi; ++i) {
            const uint32_t key = score_key(__ldcg(vals + i));
            bool take = false;
            if (key > prefix) {
                take = true;
            } else if (key == prefix) {
                take = (r < need_eq);
                ++r;
            }
            if (take) {
                if (pub) pub[pos] = i + 1;
                out[pos++] = i;
            }
        }
    }
    for (int c = k + tid; c < topk; c += NT) out[c] = -1;
    probe(3);
}

}  // namespace ssa
