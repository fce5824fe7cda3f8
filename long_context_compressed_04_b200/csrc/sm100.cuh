// Thin wrappers over the sm_100a instructions the tensor-core kernels use: mbarriers,
// TMA tiled loads (no multicast), tcgen05 MMA / commit / TMEM allocation and loads.
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "common.cuh"

namespace csa {
namespace sm100 {

// A wait gives up after this many SM clocks (~2 s at 1.9 GHz), marks the CTA aborted and
// reports CSA_DEV_TIMEOUT, so a broken pipeline ends the kernel instead of hanging it.
constexpr long long kWaitLimitCycles = 4000000000LL;

// The limit the bounded waits below use, in SM clocks.  Every kernel file that includes
// this header holds its own copy (internal linkage); csa_debug_set_wait_limit sets all of
// them.  The drains of a CTA's own copies and MMAs keep kWaitLimitCycles whatever this is,
// so a lowered limit never lets a CTA leave with asynchronous work still in flight.
namespace {
__device__ long long g_wait_limit_cycles = kWaitLimitCycles;
}

__device__ __forceinline__ long long wait_limit_cycles() {
    return *reinterpret_cast<volatile long long*>(&g_wait_limit_cycles);
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
                 : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_addr(bar)) : "memory");
}

// Non-blocking: true when the phase of the given parity has completed (never suspends).
__device__ __forceinline__ bool mbar_ready(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// True when the phase of the given parity has completed; a thread whose phase is not complete
// is first suspended in hardware until it completes or about `hint_ns` nanoseconds pass:
// waiting roles then take no issue slots from the ones doing work.
__device__ __forceinline__ bool mbar_test_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Suspend limit of one try_wait inside the bounded waits (the abort flag and the clock are
// checked between them).
constexpr uint32_t kSleepHintNs = 20000;

// Limits below this many clocks make the waits poll (test_wait, never suspending) instead
// of suspending in try_wait: a suspended thread may sleep until the phase completes, so a
// short limit would otherwise never be reached.
constexpr long long kPollBelowCycles = 1000000;

// Bounded wait.  Returns false when the CTA has been aborted by another role or this wait
// ran out of time (then it aborts the CTA and flags CSA_DEV_TIMEOUT).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int32_t* dev_status) {
    if (mbar_ready(bar, parity)) return true;
    const long long limit = wait_limit_cycles();
    const bool poll = limit < kPollBelowCycles;
    const long long t0 = clock64();
    for (;;) {
        if (poll ? mbar_ready(bar, parity) : mbar_test_sleep(bar, parity, kSleepHintNs))
            return true;
        if (*abort_flag) return false;
        if (clock64() - t0 > limit) {
            *abort_flag = 1;
            flag(dev_status, CSA_DEV_TIMEOUT);
            return false;
        }
    }
}

// Bounded wait that ignores the abort flag: used to drain this CTA's own asynchronous
// copies and MMAs before it releases shared memory and tensor memory.
__device__ __forceinline__ bool mbar_drain(uint64_t* bar, uint32_t parity, int32_t* dev_status) {
    const long long t0 = clock64();
    while (!mbar_test_sleep(bar, parity, kSleepHintNs)) {
        if (clock64() - t0 > kWaitLimitCycles) {
            flag(dev_status, CSA_DEV_TIMEOUT);
            return false;
        }
    }
    return true;
}

// Bounded wait whose result is the same for every lane of the calling warp (all lanes
// must call it): a warp never splits between a collective and an abort path.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity,
                                               volatile int* abort_flag, int32_t* dev_status) {
    const bool ok = mbar_wait(bar, parity, abort_flag, dev_status);
    return __all_sync(0xffffffffu, ok);
}

// ---- thread-block clusters (distributed shared memory) ----------------------------------
__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Address in the cluster's shared window of `local` as it lies in CTA `rank`'s memory.
__device__ __forceinline__ uint32_t mapa(const void* local, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr(local)), "r"(rank));
    return r;
}

__device__ __forceinline__ uint32_t cluster_nctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t cluster_addr) {
    uint32_t v;
    asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(cluster_addr) : "memory");
    return v;
}

__device__ __forceinline__ uint4 ld_cluster_u4(uint32_t cluster_addr) {
    uint4 v;
    asm volatile("ld.shared::cluster.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(cluster_addr)
                 : "memory");
    return v;
}

// Release-arrive (cluster scope) on an mbarrier of any CTA of the cluster.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
                 : "memory");
}

// Orders this thread's prior shared-memory accesses before later cluster-visible operations.
__device__ __forceinline__ void fence_cluster() {
    asm volatile("fence.acq_rel.cluster;" ::: "memory");
}

// Non-blocking test with acquire at cluster scope.
__device__ __forceinline__ bool mbar_ready_cluster(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait with acquire at cluster scope (arrivals come from other CTAs of the cluster);
// the result is the same for every lane of the calling warp (all lanes must call it).  It
// polls rather than suspending in try_wait: a thread suspended there was seen to resume
// microseconds after the phase had been completed by arrivals from other CTAs.
__device__ __forceinline__ bool mbar_wait_cluster_warp(uint64_t* bar, uint32_t parity,
                                                       volatile int* abort_flag,
                                                       int32_t* dev_status) {
    bool ok = true;
    if (!mbar_ready_cluster(bar, parity)) {
        const long long t0 = clock64();
        for (;;) {
            if (mbar_ready_cluster(bar, parity)) break;
            if (*abort_flag) {
                ok = false;
                break;
            }
            if (clock64() - t0 > wait_limit_cycles()) {
                *abort_flag = 1;
                flag(dev_status, CSA_DEV_TIMEOUT);
                ok = false;
                break;
            }
        }
    }
    return __all_sync(0xffffffffu, ok);
}

__device__ __forceinline__ float4 ld_cluster_f4(uint32_t cluster_addr) {
    float4 v;
    asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "r"(cluster_addr)
                 : "memory");
    return v;
}

__device__ __forceinline__ float ld_cluster_f32(uint32_t cluster_addr) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(cluster_addr) : "memory");
    return v;
}

__device__ __forceinline__ void st_cluster_f4(uint32_t cluster_addr, float4 v) {
    asm volatile("st.shared::cluster.v4.f32 [%0], {%1, %2, %3, %4};" ::"r"(cluster_addr), "f"(v.x),
                 "f"(v.y), "f"(v.z), "f"(v.w)
                 : "memory");
}

__device__ __forceinline__ void st_cluster_f32(uint32_t cluster_addr, float v) {
    asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(cluster_addr), "f"(v) : "memory");
}

// Every thread of every CTA of the cluster (release / acquire).
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// AND of `v` over the `nthreads` threads meeting at named barrier `id` (all must arrive).
__device__ __forceinline__ bool named_barrier_and(int id, int nthreads, bool v) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred pi, po;\n\t"
        "setp.ne.u32 pi, %1, 0;\n\t"
        "bar.red.and.pred po, %2, %3, pi;\n\t"
        "selp.u32 %0, 1, 0, po;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)v), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

// 2^x by the PTX approximate base-2 exponential (flush-to-zero; 2^-inf = +0), for softmax
// weights that are rounded to bf16 afterwards.
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// L2 prefetch of `bytes` contiguous bytes (16-byte aligned address, multiple of 16 bytes).
__device__ __forceinline__ void prefetch_l2_bulk(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2D tiled TMA load into this CTA's shared memory, completing on `bar` (no multicast).
// x is the innermost coordinate in elements; it must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t x, int32_t y) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%3, %4}], [%2];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(x), "r"(y)
        : "memory");
}

// L2 policy of a load: for data read once (read_once), its lines are the first the cache
// evicts, so the lines that later kernels read stay; otherwise the lines' priority is left
// as a plain load leaves it.
__device__ __forceinline__ uint64_t l2_policy(bool read_once) {
    uint64_t p;
    if (read_once)
        asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    else
        asm volatile("createpolicy.fractional.L2::evict_unchanged.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// tma_load_2d with an L2 cache policy (l2_policy) for the lines it brings in.
__device__ __forceinline__ void tma_load_2d_hint(void* dst, const CUtensorMap* map, uint64_t* bar,
                                                 int32_t x, int32_t y, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint "
        "[%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(x), "r"(y), "l"(policy)
        : "memory");
}

// Bulk copy of `bytes` contiguous bytes global -> shared (16-byte aligned addresses, a
// multiple of 16 bytes), completing on `bar` with its byte count.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

// TMA gather of 4 rows (row coordinates r0..r3, each may be out of range -> zero fill) of a
// 2D tensor map whose box is one row high; the rows land consecutively at dst.
__device__ __forceinline__ void tma_gather4(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int32_t x, int32_t r0, int32_t r1, int32_t r2,
                                            int32_t r3) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_addr(bar)), "r"(x), "r"(r0), "r"(r1),
        "r"(r2), "r"(r3)
        : "memory");
}

// ---- tcgen05 ----------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_addr(dst_smem)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] x B[smem]^T, e4m3 x e4m3 -> fp32, shape from the instruction descriptor.
__device__ __forceinline__ void mma_f8f6f4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[smem] x B[smem]^T, bf16 x bf16 -> fp32.
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrives once on `bar` when every tcgen05 operation this thread issued so far completes.
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// 32 lanes x 16 / 32 / 64 consecutive 32-bit columns: thread i of the warp gets row
// (lane base + i), columns [col, col + N).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* r) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t* r) {
    tmem_ld16(taddr, r);
    tmem_ld16(taddr + 16, r + 16);
}

__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t* r) {
    tmem_ld32(taddr, r);
    tmem_ld32(taddr + 32, r + 32);
}

// Stores 32 lanes x 16 consecutive 32-bit columns (thread i: row lane base + i).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* r) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}

__device__ __forceinline__ void tmem_st_wait() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major tile stored with the 128-byte swizzle
// (rows of 128 bytes, 8-row groups 1024 bytes apart; tile base 1024-byte aligned).
// Advancing along K inside the 128-byte row adds (bytes >> 4) to the start address.
__device__ __forceinline__ uint64_t smem_desc_k_sw128(const void* tile) {
    const uint64_t addr = smem_addr(tile);
    uint64_t d = 0;
    d |= (addr >> 4) & 0x3FFFull;          // start address
    d |= 1ull << 16;                       // leading-dim byte offset (unused with swizzle)
    d |= (uint64_t)(1024 >> 4) << 32;      // stride-dim byte offset: 8 rows x 128 B
    d |= 1ull << 46;                       // descriptor version for sm_100
    d |= 2ull << 61;                       // 128-byte swizzle
    return d;
}

// K-major tile with the 64-byte swizzle (rows of 64 bytes, 8-row groups 512 bytes apart;
// tile base 512-byte aligned).  Advancing along K inside the row adds (bytes >> 4).
__device__ __forceinline__ uint64_t smem_desc_k_sw64(const void* tile) {
    const uint64_t addr = smem_addr(tile);
    uint64_t d = 0;
    d |= (addr >> 4) & 0x3FFFull;          // start address
    d |= 1ull << 16;                       // leading-dim byte offset (unused with swizzle)
    d |= (uint64_t)(512 >> 4) << 32;       // stride-dim byte offset: 8 rows x 64 B
    d |= 1ull << 46;                       // descriptor version for sm_100
    d |= 4ull << 61;                       // 64-byte swizzle
    return d;
}

// 32 rows x 16 bytes stored contiguously (no swizzle: 8-row core matrices 128 bytes apart),
// the source of a tcgen05.cp of shape 32x128b.
__device__ __forceinline__ uint64_t smem_desc_rows16(const void* p) {
    const uint64_t addr = smem_addr(p);
    uint64_t d = 0;
    d |= (addr >> 4) & 0x3FFFull;
    d |= (uint64_t)(128 >> 4) << 16;
    d |= (uint64_t)(128 >> 4) << 32;
    d |= 1ull << 46;
    return d;
}

// Copies 32 rows x 128 bits of shared memory into TMEM columns [col, col + 4) of all four
// 32-lane quarters (row r to lanes r, 32 + r, 64 + r, 96 + r).
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
                 : "memory");
}

// Orders this thread's generic-proxy shared-memory writes before later async-proxy reads
// (TMA, tcgen05.cp, tcgen05.mma).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// D[tmem] (+)= (A x SFA)[smem] x (B x SFB)[smem]^T, MXFP4: packed e2m1 A and B (K = 64 per
// instruction), one UE8M0 scale per 32 elements from TMEM (sfa / sfb: column addresses;
// the instruction descriptor selects the bytes).
__device__ __forceinline__ void mma_mxf4(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                         uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%5], [%6], "
        "p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
        : "memory");
}

// Instruction descriptor of kind::mxf4 with UE8M0 scales: e2m1 A and B, K-major, M x N,
// dense K = 64; sf_a / sf_b: the byte of each 32-bit TMEM scale column this instruction's
// first 32-element block reads (0 or 2: two blocks per instruction).
__host__ __device__ constexpr uint32_t instr_desc_mxf4(int M, int N, uint32_t sf_a,
                                                       uint32_t sf_b) {
    return (sf_b << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | (1u << 23) |
           ((uint32_t)(M >> 4) << 24) | (sf_a << 29);
}

// Instruction descriptor: fp32 accumulate, A/B K-major, shape M x N.
// a_fmt / b_fmt: e4m3 = 0 (kind::f8f6f4); bf16 = 1 (kind::f16).
__host__ __device__ constexpr uint32_t instr_desc(uint32_t a_fmt, uint32_t b_fmt, int M, int N,
                                                  uint32_t b_major_mn = 0) {
    return (1u << 4) | (a_fmt << 7) | (b_fmt << 10) | (b_major_mn << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

}  // namespace sm100

// Host side of the wait limit: each kernel file registers a setter of its own copy of
// g_wait_limit_cycles when the library loads (csa_debug_set_wait_limit calls them all).
void register_wait_limit_setter(cudaError_t (*set)(long long cycles));
namespace {
cudaError_t set_wait_limit_of_this_file(long long cycles) {
    return cudaMemcpyToSymbol(sm100::g_wait_limit_cycles, &cycles, sizeof(cycles));
}
const bool g_wait_limit_setter_registered =
    (register_wait_limit_setter(&set_wait_limit_of_this_file), true);
}  // namespace
}  // namespace csa
