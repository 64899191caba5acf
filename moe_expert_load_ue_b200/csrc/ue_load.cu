// Step 1 - load computation: exact per-source-rank histogram of the top-k ids.
//
// "Load computation" (csrc/kernels/load_compute.cu in the component list of
// "How dots-infra/ultraep works"; the arXiv abstract calls UltraEP an
// "exact-load" balancer).  counts[r][e] = #{(t, k) : t in rank r, ids[t][k] = e}.
//
// Design (sm_100a): one thread-block cluster per simulated rank.  Each CTA of
// the cluster histograms a contiguous share of the rank's ids into shared
// memory with 16-byte (int4) loads and warp-aggregated shared atomics
// (__match_any_sync groups equal ids so each distinct id in a warp does one
// atomic).  The cluster then reduces its CTA histograms over distributed
// shared memory, each CTA summing a slice of the E columns, and writes its
// rank's row of counts with plain stores: no global atomics, no pre-zeroing,
// no workspace.
#include <cooperative_groups.h>

#include "ue_internal.cuh"

namespace cg = cooperative_groups;

namespace ue {
namespace {

constexpr int kLoadWarps = 16;

// One warp step: every lane offers `key` (-1 = nothing); each group of equal
// keys adds its size to hist[key] once, from its lowest lane.
__device__ __forceinline__ void warp_hist_add(int32_t *hist, int key)
{
    const unsigned m = __match_any_sync(0xffffffffu, key);
    if (key >= 0 && (lanemask_lt() & m) == 0) atomicAdd(&hist[key], __popc(m));
}

__device__ __forceinline__ int valid_key(int id, int E, bool in_range, int &nbad)
{
    if (!in_range) return -1;
    if ((unsigned)id < (unsigned)E) return id;
    ++nbad;
    return -1;
}

__global__ void __launch_bounds__(kLoadWarps * 32)
k_load(const int32_t *__restrict__ ids, int64_t per_rank, int E,
       int32_t *__restrict__ counts, int32_t *__restrict__ bad)
{
    extern __shared__ __align__(16) int32_t sm_load[];
    int32_t *hist = sm_load;          // [E]
    int32_t *sbad = sm_load + E;      // [1]

    cg::cluster_group cluster = cg::this_cluster();
    const int C = (int)cluster.num_blocks();
    const int c = (int)cluster.block_rank();
    const int r = blockIdx.x / C;
    const int lane = lane_id(), warp = threadIdx.x >> 5;

    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
    if (threadIdx.x == 0) *sbad = 0;
    __syncthreads();

    // This CTA's share [lo, hi) of rank r's flat id range, 32-id aligned shares.
    const int64_t share = ((per_rank + C - 1) / C + 31) / 32 * 32;
    const int64_t base = (int64_t)r * per_rank;
    const int64_t lo = base + min(per_rank, (int64_t)c * share);
    const int64_t hi = base + min(per_rank, (int64_t)(c + 1) * share);
    // int4 body [vlo, vhi) on 16-byte boundaries (ids is 16-byte aligned).
    const int64_t vlo = min(hi, (lo + 3) / 4 * 4);
    const int64_t vhi = max(vlo, hi / 4 * 4);
    int nbad = 0;

    // Ragged head (< 4 ids) and tail (< 4 ids), one warp step.
    if (warp == 0) {
        int64_t i = -1;
        if (lane < vlo - lo) i = lo + lane;
        else if (lane >= 4 && lane - 4 < hi - vhi) i = vhi + (lane - 4);
        const int id = i >= 0 ? __ldg(ids + i) : -1;
        warp_hist_add(hist, valid_key(id, E, i >= 0, nbad));
    }

    // Body: each warp walks int4 vectors; two vectors in flight per lane.
    const int4 *vec = reinterpret_cast<const int4 *>(ids + vlo);
    const int64_t nvec = (vhi - vlo) / 4;
    constexpr int kStride = kLoadWarps * 32;
    for (int64_t w0 = (int64_t)warp * 32; w0 < nvec; w0 += 2 * kStride) {
        const int64_t i0 = w0 + lane, i1 = w0 + kStride + lane;
        const bool v0 = i0 < nvec, v1 = i1 < nvec;
        int4 a = v0 ? __ldg(vec + i0) : make_int4(0, 0, 0, 0);
        int4 b = v1 ? __ldg(vec + i1) : make_int4(0, 0, 0, 0);
        warp_hist_add(hist, valid_key(a.x, E, v0, nbad));
        warp_hist_add(hist, valid_key(a.y, E, v0, nbad));
        warp_hist_add(hist, valid_key(a.z, E, v0, nbad));
        warp_hist_add(hist, valid_key(a.w, E, v0, nbad));
        if (w0 + kStride < nvec) {   // warp-uniform
            warp_hist_add(hist, valid_key(b.x, E, v1, nbad));
            warp_hist_add(hist, valid_key(b.y, E, v1, nbad));
            warp_hist_add(hist, valid_key(b.z, E, v1, nbad));
            warp_hist_add(hist, valid_key(b.w, E, v1, nbad));
        }
    }
    if (nbad) atomicAdd(sbad, nbad);

    // Cluster reduction over distributed shared memory.
    cluster.sync();
    const int cols = (E + C - 1) / C;
    const int e0 = c * cols, e1 = min(E, e0 + cols);
    for (int e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
        int s = 0;
        for (int q = 0; q < C; ++q) s += cluster.map_shared_rank(hist, q)[e];
        counts[(int64_t)r * E + e] = s;
    }
    if (bad != nullptr && c == 0 && threadIdx.x == 0) {
        int s = 0;
        for (int q = 0; q < C; ++q) s += *cluster.map_shared_rank(sbad, q);
        bad[r] = s;
    }
    cluster.sync();   // peers may still read this CTA's histogram
}

}  // namespace

size_t load_smem_bytes(const Shape &sh) { return (size_t)(sh.E + 4) * sizeof(int32_t); }

cudaError_t launch_load(const Shape &sh, const Launch &ln, const int32_t *ids, int32_t *counts,
                        int32_t *bad, cudaStream_t st)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(sh.N * ln.cluster));
    cfg.blockDim = dim3(kLoadWarps * 32);
    cfg.dynamicSmemBytes = load_smem_bytes(sh);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)ln.cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_load, ids, sh.per_rank, sh.E, counts, bad);
}

cudaError_t set_load_attributes(size_t max_smem)
{
    return cudaFuncSetAttribute(k_load, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)max_smem);
}

}  // namespace ue
