// sm100.cuh -- thin inline-PTX wrappers for the Blackwell (sm_100a) features the
// triangle-multiplication kernels use: mbarriers with bounded waits, TMA tensor
// copies, tcgen05 tensor-memory allocation, MMA, commit and loads.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace trimul {

// Device-wide error word; read and cleared by tri_mul_check_device_status().
extern __device__ unsigned int g_device_error;

enum : unsigned int {
    kErrTimeoutProducer = 1u << 0,
    kErrTimeoutMma = 1u << 1,
    kErrTimeoutEpilogue = 1u << 2,
    kErrTimeoutDrain = 1u << 3,
    kErrRange = 1u << 4,            // a non-finite fp16 intermediate
};

// About one second at the B200 boost clock.
constexpr long long kWaitLimitCycles = 2000000000LL;
constexpr long long kDrainLimitCycles = 200000000LL;

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbarrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                     smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Like mbar_try_wait, but a thread whose phase is not complete is suspended by the
// hardware until the phase completes (or about `hint_ns` passes) instead of returning at
// once; waiting warps then stop re-issuing shared-memory polls that compete with the
// tensor cores' and the other warps' shared-memory traffic.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t *bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity to complete. Returns false
// (after raising the CTA's abort flag and the device error word) if the phase
// does not complete within the limit, or if another warp of the CTA aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                          unsigned int err_code) {
    if (mbar_try_wait(bar, parity)) return true;
    long long start = clock64();
    uint32_t spins = 0;
    while (true) {
        if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
        if ((++spins & 15u) == 0) {
            if (*abort_flag) return false;
            if (clock64() - start > kWaitLimitCycles) {
                *abort_flag = 1;
                atomicOr(&g_device_error, err_code);
                return false;
            }
        }
    }
}

// ------------------------------------------------------------------ CTA pairs (clusters of two)

__device__ __forceinline__ uint32_t cluster_ctarank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// The shared::cluster address of the object at `p` (in this CTA's shared memory) in cluster CTA
// `rank`: the same offset in that CTA's shared memory.
__device__ __forceinline__ uint32_t mapa_shared(const void *p, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
    return r;
}

// Asynchronous 4-byte store into the shared memory of a cluster CTA (shared::cluster address
// `addr`) that completes 4 bytes of the transaction count of that CTA's mbarrier at `bar`: a
// thread waiting on the barrier then sees the data, with no fence on the storing side.
__device__ __forceinline__ void st_async_u32(uint32_t addr, uint32_t v, uint32_t bar) {
    asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.u32 [%0], %1, [%2];" ::"r"(addr), "r"(v),
                 "r"(bar)
                 : "memory");
}

// Arrive on the mbarrier at shared::cluster address `addr` (this CTA's or the peer's) with the
// default semantics (release at CTA scope): enough where the waiter needs no data from this thread
// (a buffer freed after this thread's loads of it returned, tensor memory read after
// tcgen05.fence::before_thread_sync), and much cheaper than a cluster-scope release, which waits
// for the thread's outstanding memory traffic.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t addr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(addr) : "memory");
}

// Arrive on the mbarrier at shared::cluster address `addr` (this CTA's or the peer's), releasing
// this thread's earlier memory operations at cluster scope.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(addr) : "memory");
}

// (With the suspend-time hint of mbar_try_wait_sleep.)
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t *bar, uint32_t parity, uint32_t hint_ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

// mbar_wait for a barrier that the peer CTA arrives on: acquires at cluster scope, so that what
// the peer released with its arrival (its stores into this CTA's shared memory, the data it saw
// land) is visible. Same bound and abort protocol; a waiting thread is suspended like mbar_wait's.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                                  unsigned int err_code) {
    long long start = clock64();
    uint32_t spins = 0;
    while (!mbar_try_wait_cluster(bar, parity, 20000u)) {
        if ((++spins & 15u) == 0) {
            if (*abort_flag) return false;
            if (clock64() - start > kWaitLimitCycles) {
                *abort_flag = 1;
                atomicOr(&g_device_error, err_code);
                return false;
            }
        }
    }
    return true;
}

// Every thread of both CTAs arrives, then waits for all (release / acquire at cluster scope). Each
// kernel that uses it calls it from every thread at the same two points (after the barrier
// initialisation and before the exit), with every role's loop bounded before it.
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// Short bounded wait used only on the abort path to let copies in flight land.
__device__ __forceinline__ void mbar_drain(uint64_t *bar, uint32_t parity) {
    long long start = clock64();
    while (!mbar_try_wait(bar, parity)) {
        if (clock64() - start > kDrainLimitCycles) {
            atomicOr(&g_device_error, (unsigned int)kErrTimeoutDrain);
            return;
        }
    }
}

// ------------------------------------------------------------------ programmatic dependent launch

// Lets the next kernel in the stream start its prologue on SMs this grid leaves free.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Waits until the previous kernel in the stream has completed and its memory operations
// are visible (returns at once for a launch without the programmatic-serialization attribute).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ------------------------------------------------------------------ persistent tile walk

// Visits the tiles first, first + step, ... of a [batch][tiles_per_batch] grid as (batch b,
// tile t within the batch) without a division per tile.
struct TileWalk {
    int b, t;
    __device__ __forceinline__ TileWalk(int first, int tiles_per_batch)
        : b(first / tiles_per_batch), t(first - (first / tiles_per_batch) * tiles_per_batch) {}
    __device__ __forceinline__ void advance(int step, int tiles_per_batch) {
        t += step;
        while (t >= tiles_per_batch) {
            t -= tiles_per_batch;
            ++b;
        }
    }
};

// ------------------------------------------------------------------ ragged masks

// x / d for x < 2^32 and d >= 1 through the host-computed multiplier m = floor(2^64 / d) + 1
// (m = 0 stands for d = 1): x m / 2^64 = x / d + x e / (d 2^64) with 0 < e <= d, an excess
// below 2^-32 that never reaches the next multiple of 1 / d, so the high word is exact.
__device__ __forceinline__ uint32_t div_by_magic(uint32_t x, uint64_t m) {
    return m ? (uint32_t)__umul64hi((uint64_t)x, m) : x;
}

// Whether every pair of the TP-pair tile (128 by default) starting at pair p0 of batch element b
// is masked, from the mask's extents ext[2b] = R_b (1 + the last row holding a nonzero mask
// entry) and ext[2b + 1] = C_b (1 + the last such column): the tile lies in rows >= R_b, or
// within one row at columns >= C_b. ext = null: no extents, nothing is skipped. rowdiv divides
// by N / 8 (p0 and N are multiples of 8).
template <int TP = 128>
__device__ __forceinline__ bool tile_masked_out(const int *ext, int b, long long p0, int N, long long NN,
                                                uint64_t rowdiv) {
    if (!ext) return false;
    const int R = __ldg(ext + 2 * b), C = __ldg(ext + 2 * b + 1);
    const int i0 = (int)div_by_magic((uint32_t)(p0 >> 3), rowdiv);
    if (i0 >= R) return true;
    const long long last = (p0 + TP - 1 < NN - 1) ? p0 + TP - 1 : NN - 1;
    const int i1 = (int)div_by_magic((uint32_t)(last >> 3), rowdiv);
    return i1 == i0 && (int)(p0 - (long long)i0 * N) >= C;
}

// ------------------------------------------------------------------ named barriers

__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// All `nthreads` threads using named barrier `id` learn whether every one of them
// passed `ok`; used so that a warpgroup leaves its loop together after a failed wait.
__device__ __forceinline__ bool group_all(bool ok, uint32_t id, uint32_t nthreads) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.and.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"((uint32_t)ok), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0;
}

// ------------------------------------------------------------------ TMA

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int32_t c0, int32_t c1) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}

__device__ __forceinline__ void tma_load_3d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int32_t c0, int32_t c1, int32_t c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

// A CTA pair's copy (cta_group::2, no multicast): the box lands in this CTA's shared memory and
// completes its bytes on the mbarrier at shared::cluster address `bar`, which may be the peer's.
__device__ __forceinline__ void tma_load_3d_pair(void *dst, const CUtensorMap *map, uint32_t bar, int32_t c0,
                                                 int32_t c1, int32_t c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, "
        "%5}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

__device__ __forceinline__ void tma_load_4d(void *dst, const CUtensorMap *map, uint64_t *bar,
                                            int32_t c0, int32_t c1, int32_t c2, int32_t c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

__device__ __forceinline__ void tma_store_3d(const CUtensorMap *map, const void *src, int32_t c0,
                                             int32_t c1, int32_t c2) {
    asm volatile(
        "cp.async.bulk.tensor.3d.global.shared::cta.tile.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(smem_u32(src)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

__device__ __forceinline__ void tma_store_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until at most N committed store groups still read shared memory.
template <int N>
__device__ __forceinline__ void tma_store_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

template <int N>
__device__ __forceinline__ void tma_store_wait_all() {
    asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// 16-byte global -> shared copy through L2 (cp.async, generic proxy); the first `bytes` of the
// 16 are read and the rest are zero-filled, so 0 writes zeros and reads nothing.
__device__ __forceinline__ void cp_async_16(void *dst, const void *src, uint32_t bytes = 16) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_u32(dst)), "l"(src), "r"(bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
// This thread's copies have landed (other threads see them after a barrier).
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }

// Make generic-proxy shared-memory writes visible to the async proxy (TMA store).
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ------------------------------------------------------------------ tcgen05

// Allocate `ncols` TMEM columns (power of two >= 32); whole warp executes.
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(dst_smem)),
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

// The same for a CTA pair (cta_group::2): one warp of each CTA, with the same warp index and the
// same destination offset, allocates together; both CTAs get the same column address.
__device__ __forceinline__ void tmem_alloc_pair(uint32_t *dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 inputs, fp32 accumulation).
__device__ __forceinline__ void tc_mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                            uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` when all previously issued tcgen05.mma of this thread complete.
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// CTA-pair MMA, issued by one thread of CTA 0: D (M = 256) = A * B^T with A's rows 0-127 from CTA
// 0's and rows 128-255 from CTA 1's shared memory, B's first N/2 rows from CTA 0's and the rest
// from CTA 1's (each at the descriptors' offsets), D's rows 0-127 into CTA 0's TMEM and 128-255 into
// CTA 1's, both at `tmem_d`.
__device__ __forceinline__ void tc_mma_bf16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                 uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on the mbarrier at this offset in every CTA of `cta_mask` when this thread's
// earlier CTA-pair MMAs complete.
__device__ __forceinline__ void tc_commit_pair_mc(uint64_t *bar, uint16_t cta_mask) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"(cta_mask)
        : "memory");
}

// The same, on this CTA's barrier only.
__device__ __forceinline__ void tc_commit_pair(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// tcgen05.wait::ld tied to the destinations of the loads it waits for: the loads write their
// registers asynchronously, so every use of them must stay after the wait; listing them as
// read-write operands of the wait makes the compiler keep it so (a plain wait orders memory
// accesses only).
__device__ __forceinline__ void tc_wait_ld_regs(float (&a)[16], float (&b)[16]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+f"(a[0]), "+f"(a[1]), "+f"(a[2]), "+f"(a[3]), "+f"(a[4]), "+f"(a[5]), "+f"(a[6]), "+f"(a[7]),
                   "+f"(a[8]), "+f"(a[9]), "+f"(a[10]), "+f"(a[11]), "+f"(a[12]), "+f"(a[13]), "+f"(a[14]), "+f"(a[15]),
                   "+f"(b[0]), "+f"(b[1]), "+f"(b[2]), "+f"(b[3]), "+f"(b[4]), "+f"(b[5]), "+f"(b[6]), "+f"(b[7]),
                   "+f"(b[8]), "+f"(b[9]), "+f"(b[10]), "+f"(b[11]), "+f"(b[12]), "+f"(b[13]), "+f"(b[14]), "+f"(b[15])
                 :
                 : "memory");
}

// 32 lanes x 32 consecutive fp32 columns: thread t of the warp gets lane (base lane + t).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 lanes x 16 consecutive fp32 columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// 32 lanes x 8 consecutive fp32 columns.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

// tc_wait_ld_regs for two 8-column loads.
__device__ __forceinline__ void tc_wait_ld_regs8(float (&a)[8], float (&b)[8]) {
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+f"(a[0]), "+f"(a[1]), "+f"(a[2]), "+f"(a[3]), "+f"(a[4]), "+f"(a[5]), "+f"(a[6]), "+f"(a[7]),
                   "+f"(b[0]), "+f"(b[1]), "+f"(b[2]), "+f"(b[3]), "+f"(b[4]), "+f"(b[5]), "+f"(b[6]), "+f"(b[7])
                 :
                 : "memory");
}

// Shared-memory matrix descriptor for tcgen05.mma with the 128-byte swizzle.
//   K-major tile: rows of 64 bf16 (128 B) at 128 B stride, 8-row groups at
//                 `sbo` bytes (1024 for a dense tile); the leading offset is unused.
//   MN-major tile: 64 MN-elements per 128 B row; K rows at 128 B, 8-row K groups
//                 at `sbo` bytes, successive 64-element MN blocks at `lbo` bytes.
__device__ __forceinline__ uint64_t smem_desc_sw128(const void *smem_ptr, uint32_t lbo,
                                                    uint32_t sbo) {
    uint64_t addr = smem_u32(smem_ptr);
    uint64_t d = 0;
    d |= (addr >> 4) & 0x3FFFull;                 // start address, bits [0,14)
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;  // leading byte offset, bits [16,30)
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;  // stride byte offset, bits [32,46)
    d |= 1ull << 46;                              // descriptor version for sm_100
    d |= 2ull << 61;                              // layout: 128-byte swizzle
    return d;
}

// Instruction descriptor: kind::f16, fp32 D, dense; A and B both f16 (f16 = true) or
// both bf16 (the two operands of one MMA always share their type).
__host__ __device__ constexpr uint32_t idesc_f32acc(int M, int N, bool a_mn_major, bool b_mn_major,
                                                    bool f16) {
    return (1u << 4)                              // D format: f32
           | ((f16 ? 0u : 1u) << 7)               // A format: f16 = 0, bf16 = 1
           | ((f16 ? 0u : 1u) << 10)              // B format: f16 = 0, bf16 = 1
           | ((a_mn_major ? 1u : 0u) << 15)       // A major-ness
           | ((b_mn_major ? 1u : 0u) << 16)       // B major-ness
           | ((uint32_t)(N >> 3) << 17)           // N / 8
           | ((uint32_t)(M >> 4) << 24);          // M / 16
}

// ------------------------------------------------------------------ math helpers

// Logistic function through the hardware tanh: sigma(v) = 0.5 + 0.5 tanh(v / 2).
__device__ __forceinline__ float sigmoid_tanh(float v) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(0.5f * v));
    return fmaf(0.5f, t, 0.5f);
}

// Logistic function through exp and a reciprocal (more accurate than the tanh form).
__device__ __forceinline__ float sigmoid_exp(float v) { return __fdividef(1.0f, 1.0f + __expf(-v)); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
    __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&h);
}

// Packed two-lane fp32 arithmetic (the sm_100 f32x2 forms, through the compiler's own
// intrinsics so that it places the two lanes in register pairs itself): one instruction, two
// independent results, each rounded exactly as the scalar instruction would round it.
__device__ __forceinline__ float2 f2_fma(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 f2_add(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 f2_mul(float2 a, float2 b) { return __fmul2_rn(a, b); }

// Hardware tanh approximation (one special-function instruction).
__device__ __forceinline__ float tanh_approx(float v) {
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(v));
    return t;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Byte offset of 16-byte unit `u` of row `r` in a 128-byte-swizzled tile (rows of 128 B).
__device__ __forceinline__ uint32_t sw128_offset(uint32_t r, uint32_t u) {
    return r * 128u + ((u ^ (r & 7u)) << 4);
}

// Byte offset of 16-byte unit `u` (0..3) of row `r` in a 64-byte-swizzled tile (rows of 64 B;
// address bits 4-5 are XORed with bits 7-8, so the pattern repeats every 512 bytes).
__device__ __forceinline__ uint32_t sw64_offset(uint32_t r, uint32_t u) {
    return r * 64u + ((u ^ ((r >> 1) & 3u)) << 4);
}

}  // namespace trimul
