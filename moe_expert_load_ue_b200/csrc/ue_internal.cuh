// Internal declarations shared by the kernels of libue.so (sm_100a only).
#pragma once

#include <cstdint>
#include <utility>

#include <cuda_runtime.h>

#include "ue.h"

namespace ue {

// Limits of the C ABI (also stated in ue.h).
constexpr int kMaxE = 1024;
constexpr int kMaxN = 1024;
constexpr int kMaxNR = 4096;
constexpr int kMaxCluster = 8;        // portable cluster size
constexpr int kMaxGpus = 128;         // GPUs of one NVLink domain for the calls across GPUs

// Device-side view of the plan (same arrays as ue_plan_buffers).
struct PlanDev {
    int32_t *slot_expert, *slot_quota, *rep_off, *rep_slot, *rep_cum, *rep_experts;
    int32_t *load, *rank_off, *rank_load_before, *rank_load_after, *info;
};

inline PlanDev to_dev(const ue_plan_buffers &p)
{
    return PlanDev{p.slot_expert, p.slot_quota, p.rep_off, p.rep_slot, p.rep_cum, p.rep_experts,
                   p.load, p.rank_off, p.rank_load_before, p.rank_load_after, p.info};
}

// Per-GPU base pointers as mapped on the calling GPU (passed by value).
struct PeerTable {
    const void *p[kMaxGpus];
};

// Shape derived from ue_config.
struct Shape {
    int E, N, R, K, H, HR, S, NR;
    int64_t T, per_rank;   // per_rank = (T / N) * K ids of each source rank
};

// Per-launch choices made on the host.
struct Launch {
    int sms;               // SM count of the device
    int cluster;           // CTAs per simulated rank for load / reroute
    size_t max_smem;       // opt-in shared memory per block
};

// Outputs of the dispatch layout (ue_dispatch_buffers without the caller's struct).
struct DispatchOut {
    const float *gates;
    int32_t *slot_off, *src_index;
    float *gates_out;
};

// Cut of each rank's ids into B pieces of zp ids for the persistent reroute
// kernel (NP = N * B pieces; NP = 0: the rank-per-cluster kernel is used).
// The load kernel writes to the workspace, per rank, B + 1 rows of E + 1 ints
// (rows [N][B + 1][E + 1]): row b holds the occurrences of each expert (column
// E: of ids outside [0, E)) in the rank's ids before piece b, row B the rank's
// totals.
struct Pieces {
    int B;          // pieces per rank
    int64_t zp;     // ids per piece (a multiple of 32; the last piece of a rank may be shorter)
    int NP;         // N * B, or 0
    int grid;       // CTAs of the persistent reroute kernel
};

// Host launchers (one per kernel file).  Each returns cudaGetLastError().
// With pc (NP > 0) the load kernel also writes the piece rows; counts may then
// be nullptr (the rows alone, for a reroute without a preceding load).  With
// lv it also adds every rank's counts into lv[0..E) (which must hold zeros):
// the expert loads, for a planner launched with the same lv right after it.
cudaError_t launch_load(const Shape &sh, const Launch &ln, const int32_t *ids, int32_t *counts,
                        int32_t *bad, cudaStream_t st, const Pieces *pc = nullptr, int32_t *rows = nullptr,
                        int32_t *lv = nullptr);
// Shared memory of the load kernel; ppc = pieces per CTA (0: no piece rows).
size_t load_smem_bytes(const Shape &sh, int ppc);

// variant: bit 0 re-queues partly placed overflow, bit 1 spreads stuck
// remainders over the expert's replicas (0 = the stated rule).  lv: the expert
// loads summed by the preceding load grid (launch_load with lv), read instead
// of summing counts and set back to zeros; nullptr: the loads from counts.
cudaError_t launch_plan(const Shape &sh, const int32_t *counts, const PlanDev &plan, cudaStream_t st,
                        bool pdl, int variant, int32_t *lv = nullptr);
size_t plan_smem_bytes(const Shape &sh);
int plan_cluster(const Shape &sh);

cudaError_t launch_reroute(const Shape &sh, const Launch &ln, const int32_t *ids, const PlanDev &plan,
                           int32_t *phys, cudaStream_t st, bool pdl);
cudaError_t launch_dispatch(const Shape &sh, const Launch &ln, const int32_t *ids, const PlanDev &plan,
                            int32_t *phys, const DispatchOut &out, int32_t *dev_err, cudaStream_t st, bool pdl);
// Shared memory of the reroute kernel (dispatch variant or not) with a
// staging buffer of stage_cap ids (0: ids are read twice from memory), and as
// many gates when the dispatch variant carries them.
size_t reroute_smem_bytes(const Shape &sh, bool dispatch, int stage_cap, bool gates);

// The persistent reroute over the pieces whose rows the load kernel wrote.
// ctr: two ints of the workspace, 0 before the launch (the kernel leaves them 0).
cudaError_t launch_reroute_pieces(const Shape &sh, const Pieces &pc, const int32_t *ids, const PlanDev &plan,
                                  const int32_t *rows, int32_t *ctr, int32_t *phys, cudaStream_t st, bool pdl);
size_t reroute_pieces_smem_bytes(const Shape &sh);
int reroute_pieces_blocks_per_sm(size_t smem);
cudaError_t set_reroute_pieces_attributes(size_t max_smem);

// Bound of the weight-sync kernels' mbarrier waits (ns on the global timer)
// and the diagnostic stall (CTA 0 waits once on a barrier nothing completes).
struct WaitBound {
    unsigned long long ns;
    int stall;
};

// The gradient reduction streamed through a ring of bulk copies (one CTA per
// SM, sms CTAs); dev_err: bit 0 when a bounded wait gives up.
cudaError_t launch_grad_reduce_bulk(const Shape &sh, int sms, float *master, const void *grads, int grad_dtype,
                                    int64_t P, const PlanDev &plan, int32_t *dev_err, cudaStream_t st,
                                    const WaitBound &wb);
// The same across G GPUs on GPU g: its home experts' master rows, replica
// gradient rows pulled through the peer table (plain bulk loads).
cudaError_t launch_grad_reduce_bulk_shard(const Shape &sh, int sms, float *master, const PeerTable &grads, int G,
                                          int g, int grad_dtype, int64_t P, const PlanDev &plan, int32_t *dev_err,
                                          cudaStream_t st, const WaitBound &wb);

// prev_slot_expert: the previous plan's slot_expert for the incremental form, or nullptr.
cudaError_t launch_sync(const Shape &sh, const Launch &ln, uint8_t *weights, int64_t slot_bytes,
                        const PlanDev &plan, const int32_t *prev_slot_expert, int32_t *dev_err, cudaStream_t st,
                        const WaitBound &wb);
size_t sync_smem_bytes(const Shape &sh);

cudaError_t launch_grad_reduce(const Shape &sh, const Launch &ln, float *master, const void *grads,
                               int grad_dtype, int64_t P, const PlanDev &plan, cudaStream_t st);
size_t grad_smem_bytes(const Shape &sh);
size_t grad_bulk_smem_bytes(const Shape &sh);

// Calls across G GPUs (GPU g holds ranks [g*N/G, (g+1)*N/G)).  round >= 0 is
// a relay round (0: scatter of the parts from the home slot, 1: all-gather
// among the consumer GPUs), -1 the direct form; relay_rounds(G) = 1 when
// G <= 2, else 2.
int relay_rounds(int G);
cudaError_t launch_sync_shard(const Shape &sh, const Launch &ln, const PeerTable &base, uint8_t *local, int G,
                              int g, int round, int64_t slot_bytes, const PlanDev &plan, int32_t *dev_err,
                              cudaStream_t st, const WaitBound &wb);
size_t sync_shard_smem_bytes(const Shape &sh);
cudaError_t launch_grad_reduce_shard(const Shape &sh, const Launch &ln, float *master, const PeerTable &grads,
                                     int G, int g, int grad_dtype, int64_t P, const PlanDev &plan, cudaStream_t st);
size_t grad_shard_smem_bytes(const Shape &sh);

// Launch with an optional thread-block cluster (cluster > 1) and optional
// programmatic dependent launch (pdl: the kernel may start while the previous
// kernel on the stream finishes; it must griddepcontrol.wait before reading
// that kernel's outputs).
template <typename... KArgs, typename... Args>
cudaError_t launch_ex(void (*kernel)(KArgs...), unsigned grid, unsigned block, size_t smem, cudaStream_t st,
                      unsigned cluster, bool pdl, Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(block);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[2];
    unsigned n = 0;
    if (cluster > 1) {
        attr[n].id = cudaLaunchAttributeClusterDimension;
        attr[n].val.clusterDim.x = cluster;
        attr[n].val.clusterDim.y = 1;
        attr[n].val.clusterDim.z = 1;
        ++n;
    }
    if (pdl) {
        attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[n].val.programmaticStreamSerializationAllowed = 1;
        ++n;
    }
    cfg.attrs = attr;
    cfg.numAttrs = n;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Opt a kernel into `max_smem` bytes of shared memory per block in total
// (dynamic plus the kernel's static shared memory).
template <typename... KArgs>
cudaError_t allow_smem(void (*kernel)(KArgs...), size_t max_smem)
{
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, kernel);
    if (e != cudaSuccess) return e;
    const size_t dyn = max_smem > fa.sharedSizeBytes ? max_smem - fa.sharedSizeBytes : 0;
    return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dyn);
}

// ---- device helpers ---------------------------------------------------------

__device__ __forceinline__ int lane_id() { return threadIdx.x & 31; }

__device__ __forceinline__ unsigned lanemask_lt()
{
    unsigned m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

__device__ __forceinline__ int clampi(int v, int lo, int hi) { return v < lo ? lo : (v > hi ? hi : v); }

// Shared-memory increment as one native reduction (red.shared.add), so that
// the compiler does not rewrite it into a per-address warp aggregation loop.
__device__ __forceinline__ void smem_add(int32_t *p, int v)
{
    asm volatile("red.shared.add.u32 [%0], %1;" ::"r"((uint32_t)__cvta_generic_to_shared(p)), "r"(v) : "memory");
}

// Programmatic dependent launch: wait for the previous grid on the stream to
// complete (and its writes to be visible); allow the next grid to launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Split cluster barrier (release on arrive, acquire on wait).
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }
// Arrive without release semantics: only says "this CTA is done reading its
// peers' shared memory", so it does not wait for the CTA's own global stores.
__device__ __forceinline__ void cluster_arrive_relaxed()
{
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}

}  // namespace ue
