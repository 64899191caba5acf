// Step 1 - load computation: exact per-source-rank histogram of the top-k ids.
//
// "Load computation" (csrc/kernels/load_compute.cu in the component list of
// "How dots-infra/ultraep works"; the arXiv abstract calls UltraEP an
// "exact-load" balancer).  counts[r][e] = #{(t, k) : t in rank r, ids[t][k] = e}.
//
// Design (sm_100a): one thread-block cluster per simulated rank.  Each CTA of
// the cluster histograms a contiguous share of the rank's ids with 16-byte
// (int4) loads into shared-memory histograms (one copy per warp, so that
// shared atomics on a popular expert collide only inside a warp), sums the
// copies, and the cluster then reduces its CTA histograms over distributed
// shared memory, each CTA summing a slice of the E columns.  The rank's row
// of counts is written with plain stores: no global atomics, no pre-zeroing,
// no workspace.
#include <cooperative_groups.h>

#include "ue_internal.cuh"

namespace cg = cooperative_groups;

namespace ue {
namespace {

constexpr int kLoadWarps = 16;
constexpr int kCopies = 16;      // shared-memory histogram copies per CTA (one per warp)

__device__ __forceinline__ void count_id(int32_t *h, int id, int E, int &nbad)
{
    if ((unsigned)id < (unsigned)E) smem_add(h + id, 1);
    else ++nbad;
}

__global__ void __launch_bounds__(kLoadWarps * 32)
k_load(const int32_t *__restrict__ ids, int64_t per_rank, int E,
       int32_t *__restrict__ counts, int32_t *__restrict__ bad)
{
    extern __shared__ __align__(16) int32_t sm_load[];
    int32_t *hist = sm_load;                     // [kCopies][E] counts
    int32_t *tot = hist + kCopies * E;           // [E]    CTA counts (read by the cluster)
    int32_t *sbad = tot + E;                     // [1]

    // The planner (launched with programmatic dependent launch) may start
    // now; it waits for this grid's completion before reading counts.
    pdl_trigger();

    cg::cluster_group cluster = cg::this_cluster();
    const int C = (int)cluster.num_blocks();
    const int c = (int)cluster.block_rank();
    const int r = blockIdx.x / C;
    const int lane = lane_id(), warp = threadIdx.x >> 5;

    // This CTA's share [lo, hi) of rank r's flat id range, 32-id aligned shares.
    const int64_t share = ((per_rank + C - 1) / C + 31) / 32 * 32;
    const int64_t base = (int64_t)r * per_rank;
    const int64_t lo = base + min(per_rank, (int64_t)c * share);
    const int64_t hi = base + min(per_rank, (int64_t)(c + 1) * share);
    // int4 body [vlo, vhi) on 16-byte boundaries (ids is 16-byte aligned).
    const int64_t vlo = min(hi, (lo + 3) / 4 * 4);
    const int64_t vhi = max(vlo, hi / 4 * 4);
    const int4 *vec = reinterpret_cast<const int4 *>(ids + vlo);
    const int64_t nvec = (vhi - vlo) / 4;
    const int64_t stride = (int64_t)blockDim.x;
    // The first four vectors of every thread are in flight while the
    // histograms are cleared.
    int4 q0[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int64_t v = threadIdx.x + k * stride;
        q0[k] = v < nvec ? __ldg(vec + v) : make_int4(-1, -1, -1, -1);
    }
    for (int i = threadIdx.x; i < kCopies * E; i += blockDim.x) hist[i] = 0;
    if (threadIdx.x == 0) *sbad = 0;
    __syncthreads();
    int32_t *h = hist + (warp % kCopies) * E;
    int nbad = 0;

    // Ragged head (< 4 ids) and tail (< 4 ids).
    if (warp == 0) {
        int64_t i = -1;
        if (lane < vlo - lo) i = lo + lane;
        else if (lane >= 4 && lane - 4 < hi - vhi) i = vhi + (lane - 4);
        if (i >= 0) count_id(h, __ldg(ids + i), E, nbad);
    }
    // Body: every thread walks int4 vectors, four in flight.
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        if (threadIdx.x + k * stride < nvec) {
            count_id(h, q0[k].x, E, nbad); count_id(h, q0[k].y, E, nbad);
            count_id(h, q0[k].z, E, nbad); count_id(h, q0[k].w, E, nbad);
        }
    }
    int64_t v = threadIdx.x + 4 * stride;
    for (; v + 3 * stride < nvec; v += 4 * stride) {
        int4 q[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) q[k] = __ldg(vec + v + k * stride);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            count_id(h, q[k].x, E, nbad); count_id(h, q[k].y, E, nbad);
            count_id(h, q[k].z, E, nbad); count_id(h, q[k].w, E, nbad);
        }
    }
    for (; v < nvec; v += stride) {
        const int4 a = __ldg(vec + v);
        count_id(h, a.x, E, nbad); count_id(h, a.y, E, nbad); count_id(h, a.z, E, nbad); count_id(h, a.w, E, nbad);
    }
    if (nbad) atomicAdd(sbad, nbad);
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int s = 0;
#pragma unroll
        for (int w = 0; w < kCopies; ++w) s += hist[w * E + e];
        tot[e] = s;
    }

    // Cluster reduction over distributed shared memory.
    cluster.sync();
    const int cols = (E + C - 1) / C;
    const int e0 = c * cols, e1 = min(E, e0 + cols);
    for (int e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
        int part[kMaxCluster];
#pragma unroll
        for (int q = 0; q < kMaxCluster; ++q) part[q] = q < C ? cluster.map_shared_rank(tot, q)[e] : 0;
        int s = 0;
#pragma unroll
        for (int q = 0; q < kMaxCluster; ++q) s += part[q];
        counts[(int64_t)r * E + e] = s;
    }
    if (bad != nullptr && c == 0 && threadIdx.x == 0) {
        int s = 0;
        for (int q = 0; q < C; ++q) s += *cluster.map_shared_rank(sbad, q);
        bad[r] = s;
    }
    cluster_arrive_relaxed();   // done reading the peers; they may still read this CTA's totals
    cluster_wait();
}

}  // namespace

size_t load_smem_bytes(const Shape &sh) { return (size_t)((kCopies + 1) * sh.E + 4) * sizeof(int32_t); }

cudaError_t launch_load(const Shape &sh, const Launch &ln, const int32_t *ids, int32_t *counts,
                        int32_t *bad, cudaStream_t st)
{
    return launch_ex(k_load, (unsigned)(sh.N * ln.cluster), kLoadWarps * 32, load_smem_bytes(sh), st,
                     (unsigned)ln.cluster, false, ids, sh.per_rank, sh.E, counts, bad);
}

cudaError_t set_load_attributes(size_t max_smem)
{
    return allow_smem(k_load, max_smem);
}

}  // namespace ue
