// Step 4 - replica weight sync: home slot -> every redundant slot of the expert.
//
// "Replica weight sync" (csrc/kernels/weight_sync.cu in "How dots-infra/ultraep
// works"; the news summary describes the transfers of expert states as
// persistent tile streaming with a relay mechanism against fan-out overload).
//
// Design (sm_100a): a persistent grid, one CTA per SM.  Work items are
// (replicated expert m, tile t) pairs, dealt round-robin to the CTAs.  One
// elected thread per CTA streams them through a ring of shared-memory stages
// with the Tensor Memory Accelerator's bulk copies (no tensor maps):
//   cp.async.bulk global->shared  (completion on an mbarrier, expect_tx)
//   cp.async.bulk shared->global  once per replica of the expert (bulk_group)
// so each home tile is read from HBM once and fanned out to all of its
// replicas - the one-GPU form of the pages' relay against fan-out overload.
// Stage reuse waits on cp.async.bulk.wait_group.read.  No multicast anywhere.
// Every mbarrier wait is bounded by the global timer (the context's wait
// limit); on timeout the kernel records an error in the context's status
// word, waits (bounded again) for the loads it issued into the other stages,
// drains its stores and exits.
//
// Incremental form: given the previous microbatch's slot_expert, a redundant
// slot that already held its expert is not copied (the expert weights do not
// change between the microbatches of one training step), and experts left
// with nothing to copy produce no work items.
#include "ue_internal.cuh"
#include "ue_bulk.cuh"

namespace ue {
namespace {

struct SyncItem {
    const uint8_t *src;
    unsigned bytes;
    int m;
    int64_t offset;
};

__global__ void __launch_bounds__(kSyncThreads, 1)
k_sync(uint8_t *__restrict__ W, int64_t slot_bytes, int E, int S, int cap,
       const int32_t *__restrict__ rep_off, const int32_t *__restrict__ rep_slot,
       const int32_t *__restrict__ rep_experts, const int32_t *__restrict__ info,
       const int32_t *__restrict__ prev, int32_t *__restrict__ dev_err, unsigned long long wait_ns, int stall)
{
    extern __shared__ __align__(128) uint8_t sm_sync[];
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm_sync);                 // [stages + 1]; the last one: see stall
    uint8_t *stage = sm_sync + 128;                                        // [stages][tile]
    int32_t *x_home = reinterpret_cast<int32_t *>(stage + (size_t)kSyncStages * kSyncTile);  // [E]
    int32_t *x_first = x_home + E;                                         // [E] first redundant entry
    int32_t *x_cnt = x_first + E;                                          // [E] redundant replicas
    int32_t *x_slot = x_cnt + E;                                           // [cap] slots to write
    int32_t *x_act = x_slot + cap;                                         // [E+1] experts with work; count

    // Per replicated expert: its home slot and the redundant slots to write
    // (all of them, or those whose expert changed since the previous plan).
    const int M = clampi(__ldg(info + 3), 0, E);
    for (int m = threadIdx.x; m < M; m += blockDim.x) {
        const int e = clampi(__ldg(rep_experts + m), 0, E - 1);
        const int off = clampi(__ldg(rep_off + e), 0, cap - 1);
        const int end = clampi(__ldg(rep_off + e + 1), off + 1, cap);
        x_home[m] = clampi(__ldg(rep_slot + off), 0, S - 1);
        x_first[m] = off + 1;
        int c = 0;
        for (int p = off + 1; p < end; ++p) {
            const int slot = clampi(__ldg(rep_slot + p), 0, S - 1);
            if (prev == nullptr || __ldg(prev + slot) != e) x_slot[off + 1 + c++] = slot;
        }
        x_cnt[m] = c;
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i <= kSyncStages; ++i) mbar_init(&bar[i], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x < 32) {                  // compact the experts that have slots to write
        const int lane = threadIdx.x;
        int n = 0;
        for (int m0 = 0; m0 < M; m0 += 32) {
            const int m = m0 + lane;
            const bool a = m < M && x_cnt[m] > 0;
            const unsigned b = __ballot_sync(0xffffffffu, a);
            if (a) x_act[n + __popc(b & lanemask_lt())] = m;
            n += __popc(b);
        }
        if (lane == 0) x_act[E] = n;
    }
    __syncthreads();
    const int MA = x_act[E];
    if (threadIdx.x != 0 || MA == 0) return;

    const int64_t ntiles = (slot_bytes + kSyncTile - 1) / kSyncTile;
    const int64_t total = (int64_t)MA * ntiles;
    if ((int64_t)blockIdx.x >= total) return;
    const int64_t nmy = (total - 1 - blockIdx.x) / gridDim.x + 1;

    auto item = [&](int64_t k) {
        const int64_t i = (int64_t)blockIdx.x + k * gridDim.x;
        SyncItem it;
        it.m = x_act[(int)(i % MA)];
        const int64_t t = i / MA;
        it.offset = t * kSyncTile;
        const int64_t left = slot_bytes - it.offset;
        it.bytes = (unsigned)(left < kSyncTile ? left : kSyncTile);
        it.src = W + (int64_t)x_home[it.m] * slot_bytes + it.offset;
        return it;
    };
    auto issue_load = [&](int64_t k) {
        const SyncItem it = item(k);
        const int b = (int)(k % kSyncStages);
        mbar_expect_tx(&bar[b], it.bytes);
        bulk_load(stage + (size_t)b * kSyncTile, it.src, it.bytes, &bar[b]);
    };

    // Store groups left reading shared memory before a stage is refilled: with
    // many tiles, kSyncStages - 1 (more writes in flight, the next load issued
    // one tile ahead); a CTA with few tiles keeps its loads ahead instead (its
    // ring would otherwise wait on each load while filling).
    const int keep = nmy >= 16 ? kSyncStages - 1 : 1;
    int64_t issued = 0;      // tiles whose load was issued; tile i goes to stage i % kSyncStages
    for (; issued < nmy && issued < kSyncStages; ++issued) issue_load(issued);
    // Diagnostic: CTA 0 waits once, with its first loads in flight, on the
    // extra barrier, on which nothing ever arrives: the wait runs out and the
    // kernel takes its way out (exercised by a test through the context).
    if (stall && blockIdx.x == 0 && !mbar_wait_bounded(&bar[kSyncStages], 0, wait_ns)) {
        ring_give_up(dev_err, bar, kSyncStages, 0, issued, wait_ns);
        return;
    }
    for (int64_t k = 0; k < nmy; ++k) {
        const int b = (int)(k % kSyncStages);
        if (!mbar_wait_bounded(&bar[b], (unsigned)((k / kSyncStages) & 1), wait_ns)) {
            ring_give_up(dev_err, bar, kSyncStages, k + 1, issued, wait_ns);
            return;
        }
        const SyncItem it = item(k);
        const uint8_t *src = stage + (size_t)b * kSyncTile;
        const int first = x_first[it.m], cnt = x_cnt[it.m];
        for (int j = 0; j < cnt; ++j)
            bulk_store(W + (int64_t)x_slot[first + j] * slot_bytes + it.offset, src, it.bytes);
        bulk_commit();
        // Stages are refilled oldest first, each once its stores have read it
        // (tile issued - kSyncStages is the oldest not yet refilled), leaving
        // up to `keep` store groups still reading.
        if (issued < nmy && k + 1 - (issued - kSyncStages) > keep) {
            bulk_wait_read_n(keep);
            while (issued < nmy && k + 1 - (issued - kSyncStages) > keep) {
                issue_load(issued);
                ++issued;
            }
        }
    }
    bulk_wait_all();
}

}  // namespace

size_t sync_smem_bytes(const Shape &sh)
{
    return 128 + (size_t)kSyncStages * kSyncTile + (size_t)(3 * sh.E + sh.E + sh.NR + sh.E + 1) * sizeof(int32_t);
}

cudaError_t launch_sync(const Shape &sh, const Launch &ln, uint8_t *weights, int64_t slot_bytes,
                        const PlanDev &plan, const int32_t *prev_slot_expert, int32_t *dev_err, cudaStream_t st,
                        const WaitBound &wb)
{
    k_sync<<<ln.sms, kSyncThreads, sync_smem_bytes(sh), st>>>(weights, slot_bytes, sh.E, sh.S, sh.E + sh.NR,
                                                               plan.rep_off, plan.rep_slot, plan.rep_experts,
                                                               plan.info, prev_slot_expert, dev_err, wb.ns,
                                                               wb.stall);
    return cudaGetLastError();
}

cudaError_t set_sync_attributes(size_t max_smem)
{
    return allow_smem(k_sync, max_smem);
}

}  // namespace ue
