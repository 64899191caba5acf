// Step 3 - routing expansion: logical expert id -> physical replica slot.
//
// "Routing expansion" (csrc/kernels/reroute.cu; "Routing expansion -> Token
// dispatch: physical routing" in "How dots-infra/ultraep works").  The j-th
// occurrence (0-based, token-major (t, k) order) of expert e goes to the
// replica i of e whose cumulative-quota range [rep_cum[i], rep_cum[i] + q_i)
// holds j.
//
// Design (sm_100a): the rank-per-cluster decomposition of the load kernel.
// Each warp owns a contiguous part of its CTA's ids, and the occurrence index
// of the warp's first occurrence of e is
//     rank_off[r][e]                         (earlier ranks, from the plan)
//   + totals of e in earlier CTAs of the rank's cluster (peers' shared memory, DSMEM)
//   + counts of e in earlier warps of this CTA (exclusive scan of per-warp histograms).
// Pass 1 (per-warp histograms) needs only the ids, so it runs before
// griddepcontrol.wait: launched with programmatic dependent launch, it
// overlaps the planner.  Pass 1 also keeps the CTA's ids in shared memory
// (when they fit), so pass 2 does not read them from memory again; both passes
// move four ids per lane with 16-byte accesses when the share is aligned.  From the counts and the bases each warp then knows,
// per expert, whether all its occurrences fall into one replica's quota range
// ("uniform": almost every (warp, expert) pair of a replicated expert; an
// expert with one replica always is).  Pass 2 is then one or two shared-memory
// lookups per id; only ids of an expert whose quota boundary falls inside the
// warp's part are ranked exactly, by ballots over the bits of the expert's
// compact index in plan.rep_experts.
#include <cooperative_groups.h>

#include "ue_internal.cuh"

namespace cg = cooperative_groups;

namespace ue {
namespace {

constexpr int kRerouteWarps = 16;
constexpr int kUnroll = 4;
constexpr int kStageIds = 8192;   // ids of a CTA share kept in shared memory between the passes

struct RerouteSmem {
    int32_t *hist;   // [W][E] per-warp counts, then their exclusive scan over the warps
    int32_t *code;   // [W][M] per warp and replicated expert: ~slot (uniform) or running occurrence index
    int32_t *tot;    // [E]    this CTA's counts (read by later CTAs of the cluster)
    int32_t *base;   // [E]    occurrences of e before this CTA's ids
    int32_t *rexp;   // [E]    replicated experts (plan.rep_experts)
    int2 *tab;       // [E]    {home slot if one replica, else first replica entry; (compact index << 16) | count}
    int2 *rc;        // [cap]  {cumulative quota, slot} of each replica entry
    int32_t *stage;  // [kStageIds] the CTA's ids, read once from HBM in pass 1 (when they fit)
};

__host__ __device__ inline size_t reroute_smem_words(int E, int cap)
{
    return (size_t)2 * kRerouteWarps * E + 3 * (size_t)E + 2 * (size_t)E + 2 * (size_t)cap + 8 + kStageIds;
}

// Word offsets are computed as integers from the (16-byte aligned) base of the
// dynamic shared memory, so every pointer stays visibly derived from it and
// compiles to shared-memory instructions.
__device__ __forceinline__ RerouteSmem carve(int32_t *base, int E, int cap)
{
    RerouteSmem s;
    int o = 0;
    s.hist = base + o;   o += kRerouteWarps * E;
    s.code = base + o;   o += kRerouteWarps * E;
    s.tot = base + o;    o += E;
    s.base = base + o;   o += E;
    s.rexp = base + o;   o += E;
    o = (o + 1) & ~1;                       // 8-byte alignment for the int2 tables
    s.tab = reinterpret_cast<int2 *>(base + o);
    o += 2 * E;
    s.rc = reinterpret_cast<int2 *>(base + o);
    o += 2 * cap;
    o = (o + 3) & ~3;                       // 16-byte alignment for the staged ids
    s.stage = base + o;
    return s;
}

// Lanes of the warp holding the same key as this lane (keys in [0, 2^nb), or -1).
__device__ __forceinline__ unsigned match_key(int key, int nb)
{
    const unsigned none = __ballot_sync(0xffffffffu, key < 0);
    unsigned m = key < 0 ? none : ~none;
    for (int b = 0; b < nb; ++b) {
        const bool bit = (key >> b) & 1;
        const unsigned v = __ballot_sync(0xffffffffu, bit);
        m &= bit ? v : ~v;
    }
    return m;
}

__global__ void __launch_bounds__(kRerouteWarps * 32)
k_reroute(const int32_t *__restrict__ ids, int64_t per_rank, int E, int cap,
          const int32_t *__restrict__ rep_off, const int32_t *__restrict__ rep_slot,
          const int32_t *__restrict__ rep_cum, const int32_t *__restrict__ rep_experts,
          const int32_t *__restrict__ info, const int32_t *__restrict__ rank_off,
          int32_t *__restrict__ phys)
{
    extern __shared__ __align__(16) int32_t sm_rr[];
    const RerouteSmem s = carve(sm_rr, E, cap);

    cg::cluster_group cluster = cg::this_cluster();
    const int C = (int)cluster.num_blocks();
    const int c = (int)cluster.block_rank();
    const int r = blockIdx.x / C;
    const int lane = lane_id(), warp = threadIdx.x >> 5;

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
    const bool staged = hi - lo <= kStageIds;     // then pass 2 reads the ids from shared memory
    // Vector mode: 16-byte loads and stores, four ids per lane, when the CTA's
    // share and phys are 16-byte aligned and the share fits in shared memory.
    const bool vec = staged && (lo % 4) == 0 && ((hi - lo) % 4) == 0 &&
                     (reinterpret_cast<uintptr_t>(phys) & 15) == 0;

    // Pass 1: per-warp histogram of the warp's part (ids only; overlaps the planner).
    if (vec) {
        for (int64_t v0 = wlo; v0 < whi; v0 += 128 * kUnroll) {
            int4 q[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t i = v0 + 128 * u + 4 * lane;
                q[u] = i < whi ? __ldg(reinterpret_cast<const int4 *>(ids + i)) : make_int4(-1, -1, -1, -1);
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t i = v0 + 128 * u + 4 * lane;
                if (i < whi) *reinterpret_cast<int4 *>(s.stage + (i - lo)) = q[u];
                if ((unsigned)q[u].x < (unsigned)E) smem_add(h + q[u].x, 1);
                if ((unsigned)q[u].y < (unsigned)E) smem_add(h + q[u].y, 1);
                if ((unsigned)q[u].z < (unsigned)E) smem_add(h + q[u].z, 1);
                if ((unsigned)q[u].w < (unsigned)E) smem_add(h + q[u].w, 1);
            }
        }
    } else
    for (int64_t x0 = wlo; x0 < whi; x0 += 32 * kUnroll) {
        int id[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = x0 + u * 32 + lane;
            id[u] = i < whi ? __ldg(ids + i) : -1;
        }
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            const int64_t i = x0 + u * 32 + lane;
            if (staged && i < whi) s.stage[i - lo] = id[u];
            if ((unsigned)id[u] < (unsigned)E) smem_add(h + id[u], 1);
        }
    }
    __syncthreads();
    // Exclusive scan over the warps per expert (in place) and CTA totals.
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

    // The plan (and rank_off) of the preceding planner grid: every global load
    // of the plan is issued in one round.
    pdl_wait();
    const int M = clampi(__ldg(info + 3), 0, E);
    for (int i = threadIdx.x; i < cap; i += blockDim.x) s.rc[i] = make_int2(__ldg(rep_cum + i), __ldg(rep_slot + i));
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const int o0 = __ldg(rep_off + e), o1 = __ldg(rep_off + e + 1);
        int b = __ldg(rank_off + (int64_t)r * E + e);
        int peer[kMaxCluster];
#pragma unroll
        for (int q = 0; q < kMaxCluster; ++q) peer[q] = q < c ? cluster.map_shared_rank(s.tot, q)[e] : 0;
        const int off = clampi(o0, 0, cap - 1);
        const int n = clampi(o1 - off, 1, min(cap - off, 0xffff));
        s.tab[e] = make_int2(off, n);
#pragma unroll
        for (int q = 0; q < kMaxCluster; ++q) b += peer[q];
        s.base[e] = b;            // occurrences of e before this CTA's ids
    }
    for (int m = threadIdx.x; m < M; m += blockDim.x) s.rexp[m] = clampi(__ldg(rep_experts + m), 0, E - 1);
    cluster_arrive_relaxed();  // done reading peers; they may exit once all have arrived
    __syncthreads();
    // Replicated experts get their compact index; every other expert's table
    // entry becomes its home slot (its only replica).
    for (int m = threadIdx.x; m < M; m += blockDim.x) s.tab[s.rexp[m]].y |= m << 16;
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        if ((s.tab[e].y & 0xffff) == 1) s.tab[e].x = s.rc[s.tab[e].x].y;
    __syncthreads();
    // Per (warp, replicated expert): ~slot when all the warp's occurrences of
    // the expert share one replica, else the warp's first occurrence index.
    for (int i = threadIdx.x; i < kRerouteWarps * M; i += blockDim.x) {
        const int w = i / M, m = i - w * M;
        const int e = s.rexp[m];
        const int2 t = s.tab[e];
        const int n = t.y & 0xffff;
        const int excl = s.hist[w * E + e];
        const int cnt = (w + 1 < kRerouteWarps ? s.hist[(w + 1) * E + e] : s.tot[e]) - excl;
        const int j0 = s.base[e] + excl;
        int lo = 0, hi = n - 1;                         // largest k with cum[k] <= j0
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s.rc[t.x + mid].x <= j0) lo = mid;
            else hi = mid - 1;
        }
        const bool uniform = lo == n - 1 || j0 + cnt <= s.rc[t.x + lo + 1].x;
        s.code[w * M + m] = uniform ? ~s.rc[t.x + lo].y : j0;
    }
    const int nb = M > 1 ? 32 - __clz(M - 1) : 0;   // bits of the compact index
    __syncthreads();

    // Replica of one id; rank_it when its expert's quota boundary falls inside
    // this warp's part (the occurrence index j is then needed).
    auto lookup = [&](int id, int &out, int &v, int2 &t, bool &rank_it) {
        const bool valid = (unsigned)id < (unsigned)E;
        t = valid ? s.tab[id] : make_int2(-1, 1);
        out = t.x;                                     // the home slot (a single replica); -1 for a bad id
        v = 0;
        if ((t.y & 0xffff) > 1) {
            v = s.code[warp * M + (t.y >> 16)];
            out = ~v;                                  // the warp's uniform replica, if v < 0
        }
        rank_it = (t.y & 0xffff) > 1 && v >= 0;
    };
    // One scalar step of 32 consecutive ids (lane order = token-major order).
    auto step = [&](int id, int64_t i) {
        int out, v;
        int2 t;
        bool rank_it;
        lookup(id, out, v, t, rank_it);
        if (__any_sync(0xffffffffu, rank_it)) {
            const int cm = t.y >> 16;
            const unsigned m = match_key(rank_it ? cm : -1, nb);
            const int before = __popc(m & lanemask_lt());
            if (rank_it) {
                const int j = v + before;
                int k = (t.y & 0xffff) - 1;
                while (k > 0 && s.rc[t.x + k].x > j) --k;
                out = s.rc[t.x + k].y;
            }
            __syncwarp();
            if (rank_it && before == 0) s.code[warp * M + cm] = v + __popc(m);
            __syncwarp();
        }
        if (i < whi) phys[i] = out;
    };

    // Pass 2: replica of every (t, k).
    if (vec) {
        // Blocks of 128 ids, four per lane: when no id of the block needs its
        // occurrence index, one 16-byte store per lane; otherwise the block is
        // replayed as four ordered scalar steps.
        for (int64_t v0 = wlo; v0 < whi; v0 += 128) {
            const int64_t i = v0 + 4 * lane;
            const int4 q = i < whi ? *reinterpret_cast<const int4 *>(s.stage + (i - lo)) : make_int4(-1, -1, -1, -1);
            int o0, o1, o2, o3, v;
            int2 t;
            bool r0, r1, r2, r3;
            lookup(q.x, o0, v, t, r0);
            lookup(q.y, o1, v, t, r1);
            lookup(q.z, o2, v, t, r2);
            lookup(q.w, o3, v, t, r3);
            if (!__any_sync(0xffffffffu, r0 || r1 || r2 || r3)) {
                if (i < whi) *reinterpret_cast<int4 *>(phys + i) = make_int4(o0, o1, o2, o3);
            } else {
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int64_t iu = v0 + 32 * u + lane;
                    step(iu < whi ? s.stage[iu - lo] : -1, iu);
                }
            }
        }
    } else {
        for (int64_t x0 = wlo; x0 < whi; x0 += 32 * kUnroll) {
            int id[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int64_t i = x0 + u * 32 + lane;
                id[u] = i >= whi ? -1 : (staged ? s.stage[i - lo] : __ldg(ids + i));
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) step(id[u], x0 + u * 32 + lane);
        }
    }
    cluster_wait();            // keep this CTA's shared memory alive for its peers
}

}  // namespace

size_t reroute_smem_bytes(const Shape &sh) { return reroute_smem_words(sh.E, sh.E + sh.NR) * sizeof(int32_t); }

cudaError_t launch_reroute(const Shape &sh, const Launch &ln, const int32_t *ids, const PlanDev &plan,
                           int32_t *phys, cudaStream_t st, bool pdl)
{
    return launch_ex(k_reroute, (unsigned)(sh.N * ln.cluster), kRerouteWarps * 32, reroute_smem_bytes(sh), st,
                     (unsigned)ln.cluster, pdl, ids, sh.per_rank, sh.E, sh.E + sh.NR, plan.rep_off, plan.rep_slot,
                     plan.rep_cum, plan.rep_experts, plan.info, plan.rank_off, phys);
}

cudaError_t set_reroute_attributes(size_t max_smem)
{
    cudaError_t e = allow_smem(k_reroute, max_smem);
    // The largest shared-memory split, so that two CTAs per SM fit and the grid
    // runs in one wave beside the planner (the default split may leave room for one).
    if (e == cudaSuccess) e = cudaFuncSetAttribute(k_reroute, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    return e;
}

}  // namespace ue
