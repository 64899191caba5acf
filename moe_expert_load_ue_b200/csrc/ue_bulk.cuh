// Bulk-copy (TMA, no tensor maps) and mbarrier helpers of the weight-sync
// kernels: cp.async.bulk global->shared completing on an mbarrier with a byte
// count, cp.async.bulk shared->global in bulk groups, and the global timer for
// bounded waits.  No multicast form is used anywhere.
#pragma once

#include <cstdint>

namespace ue {
namespace {

constexpr int kSyncThreads = 128;
constexpr int kSyncStages = 4;
constexpr int kSyncTile = 48 * 1024;                       // bytes per stage
constexpr unsigned long long kWaitLimitNs = 2000000000ull; // default bound of one wait: 2 s

__device__ __forceinline__ uint32_t smem_addr(const void *p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ unsigned long long global_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, unsigned count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t *bar, unsigned bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, unsigned parity)
{
    unsigned ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Waits until the mbarrier completes the given phase or limit_ns passes on the
// global timer; false if it gave up.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, unsigned parity, unsigned long long limit_ns)
{
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = global_ns();
    while (!mbar_try_wait(bar, parity))
        if (global_ns() - t0 > limit_ns) return false;
    return true;
}

// The ring's way out after a wait gave up: record the error, then wait (each
// wait bounded again) for the loads this thread issued into stages it has not
// consumed - items first .. issued-1 of the ring - so that no copy lands in
// shared memory after the CTA exits, and drain its bulk stores.  A load that
// never completes is abandoned after its bound; the device state is then
// undefined, which the status word reports.
__device__ __forceinline__ void ring_give_up(int32_t *dev_err, uint64_t *bar, int stages, int64_t first,
                                             int64_t issued, unsigned long long limit_ns)
{
    atomicOr(dev_err, 1);
    for (int64_t k = first; k < issued; ++k)
        mbar_wait_bounded(&bar[k % stages], (unsigned)((k / stages) & 1), limit_ns);
    asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

__device__ __forceinline__ void bulk_load(void *dst_smem, const void *src, unsigned bytes, uint64_t *bar)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            smem_addr(dst_smem)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar))
        : "memory");
}

__device__ __forceinline__ void bulk_store(void *dst, const void *src_smem, unsigned bytes)
{
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
                 "r"(smem_addr(src_smem)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
// Until at most n (0..3, clamped) committed bulk groups still read shared memory.
__device__ __forceinline__ void bulk_wait_read_n(int n)
{
    switch (n) {
    case 0: asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); break;
    case 1: asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); break;
    case 2: asm volatile("cp.async.bulk.wait_group.read 2;" ::: "memory"); break;
    default: asm volatile("cp.async.bulk.wait_group.read 3;" ::: "memory"); break;
    }
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

}  // namespace
}  // namespace ue
