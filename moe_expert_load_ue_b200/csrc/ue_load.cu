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
// of counts is written with plain stores: no global atomics, no pre-zeroing.
// For microbatches routed by the persistent reroute kernel (many ranks or
// many tokens per rank) the kernel also writes the histogram of every piece
// of a rank's ids to the context's workspace; otherwise it uses none.
#include <cooperative_groups.h>

#include "ue_internal.cuh"

namespace cg = cooperative_groups;

namespace ue {
namespace {

constexpr int kLoadWarps = 16;
constexpr int kCopies = 16;      // shared-memory histogram copies per CTA (one per warp)

using HistRef = uint32_t;        // shared-state-space address of a histogram copy
__device__ __forceinline__ HistRef hist_ref(int32_t *h) { return (uint32_t)__cvta_generic_to_shared(h); }

// One id into a histogram copy of E + 1 bins at shared address h: an id
// outside [0, E) lands in bin E, so that the count is one unsigned min, one
// address and one shared reduction, with no branch.
__device__ __forceinline__ void count_id(HistRef h, int id, int E)
{
    const uint32_t bin = min((uint32_t)id, (uint32_t)E);
    asm volatile("red.shared.add.u32 [%0], 1;" ::"r"(h + 4u * bin) : "memory");
}

__device__ __forceinline__ void count4(HistRef h, int4 q, int E)
{
    count_id(h, q.x, E); count_id(h, q.y, E); count_id(h, q.z, E); count_id(h, q.w, E);
}

// The first four int4 vectors of every thread for the range [lo, hi) (its
// 16-byte aligned body), loaded before the histograms are cleared or reduced.
struct Head {
    int4 q[4];
};

__device__ __forceinline__ Head load_head(const int32_t *__restrict__ ids, int64_t lo, int64_t hi)
{
    const int64_t vlo = min(hi, (lo + 3) / 4 * 4);
    const int64_t vhi = max(vlo, hi / 4 * 4);
    const int4 *vec = reinterpret_cast<const int4 *>(ids + vlo);
    const int64_t nvec = (vhi - vlo) / 4;
    Head hd;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int64_t v = threadIdx.x + k * (int64_t)blockDim.x;
        hd.q[k] = v < nvec ? __ldg(vec + v) : make_int4(-1, -1, -1, -1);
    }
    return hd;
}

// Counts the ids of [lo, hi) into this warp's histogram copy h: a ragged head
// and tail (< 4 ids each) by warp 0, the body as int4 vectors, four in flight
// per thread (the first four already in hd).
__device__ __forceinline__ void count_range(const int32_t *__restrict__ ids, int64_t lo, int64_t hi, int E,
                                            HistRef h, const Head &hd)
{
    const int lane = lane_id(), warp = threadIdx.x >> 5;
    const int64_t vlo = min(hi, (lo + 3) / 4 * 4);
    const int64_t vhi = max(vlo, hi / 4 * 4);
    const int4 *vec = reinterpret_cast<const int4 *>(ids + vlo);
    const int nvec = (int)((vhi - vlo) / 4);
    const int stride = (int)blockDim.x;
    if (warp == 0) {
        int64_t i = -1;
        if (lane < vlo - lo) i = lo + lane;
        else if (lane >= 4 && lane - 4 < hi - vhi) i = vhi + (lane - 4);
        if (i >= 0) count_id(h, __ldg(ids + i), E);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k)
        if ((int)threadIdx.x + k * stride < nvec) count4(h, hd.q[k], E);
    int v = (int)threadIdx.x + 4 * stride;
    for (; v + 3 * stride < nvec; v += 4 * stride) {
        int4 q[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) q[k] = __ldg(vec + v + k * stride);
#pragma unroll
        for (int k = 0; k < 4; ++k) count4(h, q[k], E);
    }
    for (; v < nvec; v += stride) count4(h, __ldg(vec + v), E);
}

// Every histogram row below has E + 1 columns: the E experts, then the ids
// outside [0, E).
//
// PIECES: the CTA's share is cut into pieces of zp ids (piece b of the rank is
// [b*zp, (b+1)*zp), pieces c*ppc .. c*ppc+ppc-1 in CTA c of the cluster).
// Row b of rank r, rows[(r*(B+1) + b)][0..E], receives the occurrences of
// every expert in the rank's ids before piece b (an exclusive prefix over the
// pieces), and row B the rank's totals.  The persistent reroute kernel takes
// each piece's starting occurrence indices and its counts from two
// consecutive rows.
template <bool PIECES>
__global__ void __launch_bounds__(kLoadWarps * 32)
k_load(const int32_t *__restrict__ ids, int64_t per_rank, int E,
       int32_t *__restrict__ counts, int32_t *__restrict__ bad,
       int32_t *__restrict__ rows, int64_t zp, int B, int32_t *__restrict__ lv)
{
    extern __shared__ __align__(16) int32_t sm_load[];
    const int E1 = E + 1;
    int32_t *hist = sm_load;                     // [kCopies][E1] counts
    int32_t *tot = hist + kCopies * E1;          // [E1]  CTA counts (read by the cluster)
    int32_t *pcnt = tot + E1;                    // PIECES: [ppc][E1] counts of the CTA's pieces

    // The planner (launched with programmatic dependent launch) may start
    // now; it waits for this grid's completion before reading counts.
    pdl_trigger();

    cg::cluster_group cluster = cg::this_cluster();
    const int C = (int)cluster.num_blocks();
    const int c = (int)cluster.block_rank();
    const int r = blockIdx.x / C;
    const int warp = threadIdx.x >> 5;

    // This CTA's share [lo, hi) of rank r's flat id range (32-id aligned
    // shares, or whole pieces).
    const int ppc = PIECES ? (B + C - 1) / C : 1;
    const int64_t share = PIECES ? (int64_t)ppc * zp : ((per_rank + C - 1) / C + 31) / 32 * 32;
    const int64_t base = (int64_t)r * per_rank;
    const int64_t lo = base + min(per_rank, (int64_t)c * share);
    const int64_t hi = base + min(per_rank, (int64_t)(c + 1) * share);
    const int64_t len = PIECES ? zp : share;
    const HistRef h = hist_ref(hist + (warp % kCopies) * E1);

    Head hd = load_head(ids, lo, min(hi, lo + len));
    for (int i = threadIdx.x; i < kCopies * E1; i += blockDim.x) hist[i] = 0;
    if (PIECES)
        for (int e = threadIdx.x; e < E1; e += blockDim.x) tot[e] = 0;
    __syncthreads();

    if constexpr (!PIECES) {
        count_range(ids, lo, hi, E, h, hd);
        __syncthreads();
        for (int e = threadIdx.x; e < E1; e += blockDim.x) {
            int s = 0;
#pragma unroll
            for (int w = 0; w < kCopies; ++w) s += hist[w * E1 + e];
            tot[e] = s;
        }
    } else {
        for (int64_t plo = lo; plo < hi; plo += len) {
            const int64_t phi = min(hi, plo + len);
            count_range(ids, plo, phi, E, h, hd);
            // The next piece's first vectors load while this one is reduced.
            if (phi < hi) hd = load_head(ids, phi, min(hi, phi + len));
            __syncthreads();
            int32_t *pc = pcnt + (int)((plo - lo) / zp) * E1;
            for (int e = threadIdx.x; e < E1; e += blockDim.x) {
                int s = 0;
#pragma unroll
                for (int w = 0; w < kCopies; ++w) {
                    s += hist[w * E1 + e];
                    hist[w * E1 + e] = 0;
                }
                tot[e] += s;
                pc[e] = s;
            }
            __syncthreads();
        }
    }

    // Cluster reduction over distributed shared memory; column E is the
    // rank's count of ids outside [0, E).
    cluster.sync();
    const int cols = (E1 + C - 1) / C;
    const int e0 = c * cols, e1 = min(E1, e0 + cols);
    for (int e = e0 + threadIdx.x; e < e1; e += blockDim.x) {
        int part[kMaxCluster];
#pragma unroll
        for (int q = 0; q < kMaxCluster; ++q) part[q] = q < C ? cluster.map_shared_rank(tot, q)[e] : 0;
        int s = 0;
#pragma unroll
        for (int q = 0; q < kMaxCluster; ++q) s += part[q];
        if (e < E) {
            if (counts != nullptr) counts[(int64_t)r * E + e] = s;
            if (lv != nullptr && s != 0) atomicAdd(lv + e, s);
        } else if (bad != nullptr) {
            bad[r] = s;
        }
    }
    if constexpr (PIECES) {
        // The prefix rows of this CTA's pieces: the earlier CTAs' totals
        // (peers' shared memory), then the pieces in order; the CTA holding
        // the rank's last piece also writes the totals row B.
        const int b0 = c * ppc, nq = min(ppc, B - b0);
        for (int e = threadIdx.x; e < E1; e += blockDim.x) {
            int run = 0;
            for (int q = 0; q < c; ++q) run += cluster.map_shared_rank(tot, q)[e];
            for (int q = 0; q < nq; ++q) {
                rows[((int64_t)r * (B + 1) + b0 + q) * E1 + e] = run;
                run += pcnt[q * E1 + e];
            }
            if (nq > 0 && b0 + nq == B) rows[((int64_t)r * (B + 1) + B) * E1 + e] = run;
        }
    }
    cluster_arrive_relaxed();   // done reading the peers; they may still read this CTA's totals
    cluster_wait();
}

}  // namespace

size_t load_smem_bytes(const Shape &sh, int ppc)
{
    return (size_t)((kCopies + 1) + (size_t)ppc) * (sh.E + 1) * sizeof(int32_t);
}

cudaError_t launch_load(const Shape &sh, const Launch &ln, const int32_t *ids, int32_t *counts,
                        int32_t *bad, cudaStream_t st, const Pieces *pc, int32_t *rows, int32_t *lv)
{
    if (pc != nullptr && pc->NP > 0) {
        const int ppc = (pc->B + ln.cluster - 1) / ln.cluster;
        return launch_ex(k_load<true>, (unsigned)(sh.N * ln.cluster), kLoadWarps * 32, load_smem_bytes(sh, ppc), st,
                         (unsigned)ln.cluster, false, ids, sh.per_rank, sh.E, counts, bad, rows, pc->zp, pc->B, lv);
    }
    return launch_ex(k_load<false>, (unsigned)(sh.N * ln.cluster), kLoadWarps * 32, load_smem_bytes(sh, 0), st,
                     (unsigned)ln.cluster, false, ids, sh.per_rank, sh.E, counts, bad, (int32_t *)nullptr,
                     (int64_t)0, 0, lv);
}

cudaError_t set_load_attributes(size_t max_smem)
{
    cudaError_t e = allow_smem(k_load<false>, max_smem);
    if (e == cudaSuccess) e = allow_smem(k_load<true>, max_smem);
    return e;
}

}  // namespace ue
