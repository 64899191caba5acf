// Step 3 - routing expansion: logical expert id -> physical replica slot.
//
// "Routing expansion" (csrc/kernels/reroute.cu; "Routing expansion -> Token
// dispatch: physical routing" in "How dots-infra/ultraep works").  The j-th
// occurrence (0-based, token-major (t, k) order) of expert e goes to the
// replica i of e whose cumulative-quota range [rep_cum[i], rep_cum[i] + q_i)
// holds j.
//
// Design (sm_100a): the same rank-per-cluster decomposition as the load
// kernel.  j = (occurrences of e in earlier ranks: plan.rank_off[r][e])
//           + (occurrences in earlier CTAs of this rank's cluster, read from
//              the peers' shared-memory histograms over DSMEM)
//           + (occurrences in earlier warps of this CTA: exclusive scan of
//              per-warp histograms)
//           + (running count inside the warp: __match_any_sync groups equal
//              ids, the rank inside a group is popc(group & lanemask_lt)).
// The replica tables of the plan sit in shared memory; the lookup scans the
// (typically 1-3) replicas of e from the last one down.
#include <cooperative_groups.h>

#include "ue_internal.cuh"

namespace cg = cooperative_groups;

namespace ue {
namespace {

constexpr int kRerouteWarps = 16;
constexpr int kUnroll = 4;

struct RerouteSmem {
    int32_t *hist;   // [W][E]  per-warp counts, then per-warp base occurrence index
    int32_t *tot;    // [E]     this CTA's counts (read by later CTAs of the cluster)
    int32_t *roff;   // [E+1]
    int32_t *rslot;  // [cap]
    int32_t *rcum;   // [cap]
};

__device__ __forceinline__ RerouteSmem carve(int32_t *base, int E, int cap)
{
    RerouteSmem s;
    s.hist = base;
    s.tot = s.hist + kRerouteWarps * E;
    s.roff = s.tot + E;
    s.rslot = s.roff + E + 1;
    s.rcum = s.rslot + cap;
    return s;
}

__global__ void __launch_bounds__(kRerouteWarps * 32)
k_reroute(const int32_t *__restrict__ ids, int64_t per_rank, int E, int cap,
          const int32_t *__restrict__ rep_off, const int32_t *__restrict__ rep_slot,
          const int32_t *__restrict__ rep_cum, const int32_t *__restrict__ rank_off,
          int32_t *__restrict__ phys)
{
    extern __shared__ __align__(16) int32_t sm_rr[];
    const RerouteSmem s = carve(sm_rr, E, cap);

    cg::cluster_group cluster = cg::this_cluster();
    const int C = (int)cluster.num_blocks();
    const int c = (int)cluster.block_rank();
    const int r = blockIdx.x / C;
    const int lane = lane_id(), warp = threadIdx.x >> 5;

    // Plan tables -> shared memory (clamped so a malformed plan cannot index out of bounds).
    for (int i = threadIdx.x; i <= E; i += blockDim.x) s.roff[i] = clampi(__ldg(rep_off + i), 0, cap);
    for (int i = threadIdx.x; i < cap; i += blockDim.x) {
        s.rslot[i] = __ldg(rep_slot + i);
        s.rcum[i] = __ldg(rep_cum + i);
    }
    for (int i = threadIdx.x; i < kRerouteWarps * E; i += blockDim.x) s.hist[i] = 0;
    __syncthreads();

    // CTA share [lo, hi) of rank r's ids, and this warp's part [wlo, whi).
    const int64_t share = ((per_rank + C - 1) / C + 31) / 32 * 32;
    const int64_t base = (int64_t)r * per_rank;
    const int64_t lo = base + min(per_rank, (int64_t)c * share);
    const int64_t hi = base + min(per_rank, (int64_t)(c + 1) * share);
    const int64_t wpart = ((hi - lo) + kRerouteWarps - 1) / kRerouteWarps;
    const int64_t wshare = (wpart + 31) / 32 * 32;
    const int64_t wlo = min(hi, lo + warp * wshare);
    const int64_t whi = min(hi, wlo + wshare);
    int32_t *h = s.hist + warp * E;

    // Pass 1: per-warp histogram of the warp's part (warp-private: no atomics).
    for (int64_t x0 = wlo; x0 < whi; x0 += 32 * kUnroll) {
        int key[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = x0 + u * 32 + lane;
            const int id = i < whi ? __ldg(ids + i) : -1;
            key[u] = (unsigned)id < (unsigned)E ? id : -1;
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const unsigned m = __match_any_sync(0xffffffffu, key[u]);
            if (key[u] >= 0 && (lanemask_lt() & m) == 0) h[key[u]] += __popc(m);
            __syncwarp();
        }
    }
    __syncthreads();

    // Exclusive scan over warps per expert; CTA totals for the cluster peers.
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int run = 0;
#pragma unroll
        for (int w = 0; w < kRerouteWarps; ++w) {
            const int t = s.hist[w * E + e];
            s.hist[w * E + e] = run;
            run += t;
        }
        s.tot[e] = run;
    }
    cluster.sync();
    // Base occurrence index of this CTA = earlier ranks + earlier CTAs of this rank.
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int b = __ldg(rank_off + (int64_t)r * E + e);
        for (int q = 0; q < c; ++q) b += cluster.map_shared_rank(s.tot, q)[e];
#pragma unroll
        for (int w = 0; w < kRerouteWarps; ++w) s.hist[w * E + e] += b;
    }
    cluster_arrive();          // done reading peers; they may exit once all arrive
    __syncthreads();

    // Pass 2: stable occurrence index and replica lookup.
    for (int64_t x0 = wlo; x0 < whi; x0 += 32 * kUnroll) {
        int key[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = x0 + u * 32 + lane;
            const int id = i < whi ? __ldg(ids + i) : -1;
            key[u] = (unsigned)id < (unsigned)E ? id : -1;
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = x0 + u * 32 + lane;
            const int k = key[u];
            const unsigned m = __match_any_sync(0xffffffffu, k);
            const int before = __popc(m & lanemask_lt());
            int out = -1;
            int j = 0;
            if (k >= 0) {
                j = h[k] + before;
                const int off = min(s.roff[k], cap - 1);
                int i_rep = clampi(s.roff[k + 1] - off, 1, cap - off) - 1;
                while (i_rep > 0 && s.rcum[off + i_rep] > j) --i_rep;
                out = s.rslot[off + i_rep];
            }
            __syncwarp();
            if (k >= 0 && before == 0) h[k] += __popc(m);
            __syncwarp();
            if (i < whi) phys[i] = out;
        }
    }
    cluster_wait();            // keep this CTA's shared memory alive for its peers
}

}  // namespace

size_t reroute_smem_bytes(const Shape &sh)
{
    const int cap = sh.E + sh.NR;
    return (size_t)(kRerouteWarps * sh.E + sh.E + sh.E + 1 + 2 * cap) * sizeof(int32_t);
}

cudaError_t launch_reroute(const Shape &sh, const Launch &ln, const int32_t *ids, const PlanDev &plan,
                           int32_t *phys, cudaStream_t st)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(sh.N * ln.cluster));
    cfg.blockDim = dim3(kRerouteWarps * 32);
    cfg.dynamicSmemBytes = reroute_smem_bytes(sh);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)ln.cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_reroute, ids, sh.per_rank, sh.E, sh.E + sh.NR, plan.rep_off,
                              plan.rep_slot, plan.rep_cum, plan.rank_off, phys);
}

cudaError_t set_reroute_attributes(size_t max_smem)
{
    return cudaFuncSetAttribute(k_reroute, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)max_smem);
}

}  // namespace ue
