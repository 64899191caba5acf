// Step 2 - quota-driven placement planning.
//
// "Placement planning" (csrc/kernels/placement.cu in "How dots-infra/ultraep
// works"; the news summary's quota-driven scheduler that reacts to the load
// right after gating).  The rule:
//   load[e] = sum_r counts[r][e];  L = sum_e load[e];  Q = ceil(L / N)
//   home pass (increasing e):   take = min(load[e], Q - cur[home]); ovf = load - take
//   overflow experts, largest overflow first (ties: lower id), each placed
//   fully before the next: every chunk goes to the rank with the most spare
//   Q - cur (ties: lowest rank) among ranks with a free redundant slot and
//   spare > 0; chunk = min(remaining, spare); if no rank is eligible the
//   remainder stays on the home slot (flag bit 0).
//   Replica list of e: home slot, then redundant slots in allocation order;
//   rep_cum = exclusive prefix of their quotas.
//
// Design (sm_100a): one thread-block cluster of up to 8 CTAs x 1024 threads.
//   Peer CTAs (cluster rank >= 1) own 32-expert column groups of counts: they
//     sum their columns (loads) and arrive on the cluster barrier, then - off
//     the critical path, while CTA 0 plans - write the exclusive column scan
//     over ranks, rank_off[r][e], that the reroute kernel needs.
//   CTA 0 pulls the loads over DSMEM and plans:
//     * home pass in closed form from a block-wide prefix sum: the home rank's
//       load before e is min(Q, in-rank prefix), so
//       take = min(Q, prefix + load) - min(Q, prefix);
//     * overflow order by a rank-by-counting sort of packed (overflow, id) keys;
//     * R = 1: a rank can be chosen at most once and its spare never changes
//       before that, so the greedy visits the eligible ranks in the order of
//       their initial spare (descending, lowest rank first).  The ranks are
//       sorted once, their spares prefix-summed, and each overflow expert takes
//       the next run of ranks whose spares cover it: one warp-wide search per
//       expert instead of one argmax per chunk;
//     * R > 1: the chunk-by-chunk greedy in one warp, each rank's spare and
//       used slots in the registers of lane r % 32, the argmax as two
//       redux.sync (largest spare, then lowest rank holding it);
//     * once no rank is eligible none becomes eligible again (spares only
//       shrink, used slots only grow): the rest of the overflow stays home;
//     * then all 1024 threads write the tables.
#include <climits>

#include <cooperative_groups.h>

#include "ue_internal.cuh"

namespace cg = cooperative_groups;

namespace ue {
namespace {

constexpr int kPlanThreads = 1024;
constexpr int kPlanWarps = kPlanThreads / 32;

// Shared-memory layout of a planner CTA (all 4-byte words unless noted).
struct PlanSmem {
    int32_t *part;        // [32][33] column-group partial sums
    int32_t *ws;          // [96] scan / reduction scratch
    int32_t *misc;        // [8]  assignments, stop position, remainder at the stop
    int32_t *sload;       // [E]  loads (peers: of their own column groups)
    int32_t *pre;         // [E]  exclusive prefix of load over experts
    int32_t *qh;          // [E]  home quota (plus any residual)
    int32_t *ovf;         // [E]
    int32_t *order;       // [E]  overflow order
    int32_t *afirst;      // [E]  first assignment of e
    int32_t *acnt;        // [E]  number of assignments of e
    int32_t *before;      // [N]
    int32_t *spare;       // [N]
    int32_t *extra;       // [N]  residual overflow kept home
    int32_t *rsorted;     // [N]  R = 1: eligible ranks by initial spare
    int32_t *rsum;        // [N+1] R = 1: exclusive prefix of their spares
    int32_t *ar;          // [NR] assignment rank
    int32_t *au;          // [NR] assignment redundant index on that rank
    int32_t *ac;          // [NR] assignment quota
    int32_t *ae;          // [NR] assignment expert
    int32_t *sasg;        // [NR] (rank, redundant index) -> assignment or -1
    unsigned long long *key;   // [max(E, N)] packed sort keys (8-byte aligned)
};

__host__ __device__ inline size_t plan_smem_words(int E, int N, int NR)
{
    const int K = E > N ? E : N;
    return (size_t)32 * 33 + 96 + 8 + (size_t)7 * E + (size_t)5 * N + 1 + (size_t)5 * NR + 2 + (size_t)2 * K;
}

__device__ __forceinline__ PlanSmem carve(int32_t *p, int E, int N, int NR)
{
    PlanSmem s;
    s.part = p;      p += 32 * 33;
    s.ws = p;        p += 96;
    s.misc = p;      p += 8;
    s.sload = p;     p += E;
    s.pre = p;       p += E;
    s.qh = p;        p += E;
    s.ovf = p;       p += E;
    s.order = p;     p += E;
    s.afirst = p;    p += E;
    s.acnt = p;      p += E;
    s.before = p;    p += N;
    s.spare = p;     p += N;
    s.extra = p;     p += N;
    s.rsorted = p;   p += N;
    s.rsum = p;      p += N + 1;
    s.ar = p;        p += NR;
    s.au = p;        p += NR;
    s.ac = p;        p += NR;
    s.ae = p;        p += NR;
    s.sasg = p;      p += NR;
    p += (reinterpret_cast<uintptr_t>(p) & 7) ? 1 : 0;
    s.key = reinterpret_cast<unsigned long long *>(p);
    return s;
}

// Block-wide exclusive prefix sum of one value per thread (all 1024 threads call it).
__device__ int block_excl_scan(int v, int32_t *ws, int *total)
{
    const int lane = lane_id(), warp = threadIdx.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) ws[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = ws[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        ws[32 + lane] = w;   // inclusive prefix of warp sums
    }
    __syncthreads();
    const int r = (warp ? ws[32 + warp - 1] : 0) + x - v;
    *total = ws[32 + kPlanWarps - 1];
    __syncthreads();
    return r;
}

// Sum of counts[r][g*32 + lane] over this thread's rows [r0, r1).
__device__ __forceinline__ int column_part(const int32_t *__restrict__ counts, int E, int g, int r0, int r1)
{
    const int e = g * 32 + lane_id();
    int sum = 0;
    if (e < E)
        for (int r = r0; r < r1; ++r) sum += __ldg(counts + (int64_t)r * E + e);
    return sum;
}

// Column totals of group g from part[row group][column]; writes sload and the plan's load.
__device__ __forceinline__ void column_totals(int E, int g, const int32_t *part, int32_t *sload, int32_t *load_out)
{
    const int tid = threadIdx.x;
    if (tid < 32) {
        const int e = g * 32 + tid;
        int t = 0;
#pragma unroll 8
        for (int w = 0; w < 32; ++w) t += part[w * 33 + tid];
        if (e < E) {
            sload[e] = t;
            load_out[e] = t;
        }
    }
}

// Exclusive scan of column group g over the row groups (part[row group][column]),
// then rank_off[r][e] for this thread's rows [r0, r1).
__device__ void column_rank_off(const int32_t *__restrict__ counts, int E, int g, int r0, int r1, int32_t *part,
                                int32_t *rank_off)
{
    const int lane = lane_id(), warp = threadIdx.x >> 5;
    __syncthreads();   // column_totals has read part
    {   // warp w scans column w of the group over the row groups (lane = row group)
        const int v = part[lane * 33 + warp];
        int x = v;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        part[lane * 33 + warp] = x - v;
    }
    __syncthreads();
    const int e = g * 32 + lane;
    int run = part[warp * 33 + lane];
    if (e < E)
        for (int r = r0; r < r1; ++r) {
            rank_off[(int64_t)r * E + e] = run;
            run += __ldg(counts + (int64_t)r * E + e);
        }
    __syncthreads();
}

// R > 1: the chunk-by-chunk greedy, run by warp 0.
template <int NRL>
__device__ void greedy_chunks(const PlanSmem &s, int N, int R, int M1)
{
    const int lane = lane_id();
    unsigned sp[NRL];
    int us[NRL];
#pragma unroll
    for (int i = 0; i < NRL; ++i) {
        const int r = lane + 32 * i;
        sp[i] = r < N ? (unsigned)s.spare[r] : 0u;
        us[i] = 0;
    }
    unsigned bs;
    int br;
    auto lane_best = [&]() {
        bs = 0;
        br = INT_MAX;
#pragma unroll
        for (int i = 0; i < NRL; ++i) {
            const bool better = us[i] < R && sp[i] > bs;    // strict: lowest rank on ties
            bs = better ? sp[i] : bs;
            br = better ? lane + 32 * i : br;
        }
    };
    lane_best();

    int na = 0, stop_pos = M1, stop_rem = 0;
    for (int m0 = 0; m0 < M1 && stop_pos == M1; m0 += 32) {
        const int idx = m0 + lane;
        const int e_l = idx < M1 ? s.order[idx] : 0;
        const int o_l = idx < M1 ? s.ovf[e_l] : 0;
        const int cnt = min(32, M1 - m0);
        for (int j = 0; j < cnt; ++j) {
            const int e = __shfl_sync(0xffffffffu, e_l, j);
            int rem = __shfl_sync(0xffffffffu, o_l, j);
            const int first = na;
            while (rem > 0) {
                const unsigned mx = __reduce_max_sync(0xffffffffu, bs);
                if (mx == 0u) break;                             // no eligible rank left
                const int rs = __reduce_min_sync(0xffffffffu, bs == mx ? br : INT_MAX);
                const int c = rem < (int)mx ? rem : (int)mx;
                const bool own = lane == (rs & 31);
                const int si = rs >> 5;
                int u = 0;
#pragma unroll
                for (int i = 0; i < NRL; ++i) {
                    const bool hit = own && i == si;
                    u = hit ? us[i] : u;
                    us[i] += hit ? 1 : 0;
                    sp[i] -= hit ? (unsigned)c : 0u;
                }
                lane_best();
                u = __shfl_sync(0xffffffffu, u, rs & 31);
                if (lane == 0) {
                    s.ar[na] = rs;
                    s.au[na] = u;
                    s.ac[na] = c;
                    s.ae[na] = e;
                    s.sasg[rs * R + u] = na;
                }
                rem -= c;
                ++na;
            }
            if (lane == 0) {
                s.afirst[e] = first;
                s.acnt[e] = na - first;
            }
            if (rem > 0) {                                       // ran out at this expert
                stop_pos = m0 + j;
                stop_rem = rem;
                break;
            }
        }
    }
#pragma unroll
    for (int i = 0; i < NRL; ++i) {
        const int r = lane + 32 * i;
        if (r < N) s.spare[r] = (int)sp[i];
    }
    if (lane == 0) {
        s.misc[0] = na;
        s.misc[1] = stop_pos;
        s.misc[2] = stop_rem;
    }
}

// R = 1: walk the eligible ranks in sorted order (s.rsorted, exclusive prefix
// s.rsum, K of them); run by warp 0.  Assignment a is sorted position a.
__device__ void greedy_sorted(const PlanSmem &s, int K, int M1)
{
    const int lane = lane_id();
    int p = 0, stop_pos = M1, stop_rem = 0;
    for (int m = 0; m < M1; ++m) {
        const int e = s.order[m];
        const int rem = s.ovf[e];
        const long long target = (long long)s.rsum[p] + rem;   // smallest q > p with rsum[q] >= target
        int q = -1;
        for (int base = p + 1; base <= K; base += 32) {
            const int cand = base + lane;
            const bool hit = cand <= K && (long long)s.rsum[cand] >= target;
            const unsigned b = __ballot_sync(0xffffffffu, hit);
            if (b) {
                q = base + __ffs(b) - 1;
                break;
            }
        }
        const int end = q < 0 ? K : q;            // ranks [p, end) go to e
        for (int a = p + lane; a < end; a += 32) {
            const int r = s.rsorted[a];
            const int full = s.rsum[a + 1] - s.rsum[a];
            s.ar[a] = r;
            s.au[a] = 0;
            s.ac[a] = (q >= 0 && a == end - 1) ? rem - (s.rsum[a] - s.rsum[p]) : full;
            s.ae[a] = e;
            s.sasg[r] = a;
        }
        if (lane == 0) {
            s.afirst[e] = p;
            s.acnt[e] = end - p;
        }
        if (q < 0) {                              // every remaining rank used: the rest stays home
            stop_pos = m;
            stop_rem = rem - (s.rsum[K] - s.rsum[p]);
            p = K;
            break;
        }
        p = q;
    }
    __syncwarp();
    for (int a = lane; a < p; a += 32) s.spare[s.ar[a]] -= s.ac[a];
    if (lane == 0) {
        s.misc[0] = p;
        s.misc[1] = stop_pos;
        s.misc[2] = stop_rem;
    }
}

template <int NRL>
__global__ void __launch_bounds__(kPlanThreads, 1)
k_plan(const int32_t *__restrict__ counts, int E, int N, int R, PlanDev plan)
{
    extern __shared__ __align__(16) int32_t sm_plan[];
    const int H = E / N, HR = H + R, S = N * HR, NR = N * R, cap = E + NR;
    const PlanSmem s = carve(sm_plan, E, N, NR);

    cg::cluster_group cluster = cg::this_cluster();
    const int C = (int)cluster.num_blocks();
    const int c = (int)cluster.block_rank();
    const int tid = threadIdx.x, warp = tid >> 5;
    const int groups = (E + 31) / 32;
    const int rpg = (N + 31) / 32;                 // ranks per row group
    const int r0 = min(N, warp * rpg), r1 = min(N, r0 + rpg);

    // The reroute grid may launch now (its first pass needs only the ids);
    // the counts of the load grid are read after it completes.
    pdl_trigger();
    pdl_wait();

    if (C > 1 && c != 0) {
        // Peer: loads of the own column groups, then (off the critical path) rank_off.
        for (int g = c - 1; g < groups; g += C - 1) {
            s.part[warp * 33 + lane_id()] = column_part(counts, E, g, r0, r1);
            __syncthreads();
            column_totals(E, g, s.part, s.sload, plan.load);
            __syncthreads();
        }
        cluster_arrive();      // #1: loads ready for CTA 0
        for (int g = c - 1; g < groups; g += C - 1) {
            s.part[warp * 33 + lane_id()] = column_part(counts, E, g, r0, r1);
            __syncthreads();
            column_rank_off(counts, E, g, r0, r1, s.part, plan.rank_off);
        }
        cluster_wait();
        cluster_arrive();      // #2: completes once CTA 0 has pulled the loads
        cluster_wait();
        return;
    }
    if (C == 1) {
        for (int g = 0; g < groups; ++g) {
            s.part[warp * 33 + lane_id()] = column_part(counts, E, g, r0, r1);
            __syncthreads();
            column_totals(E, g, s.part, s.sload, plan.load);
            column_rank_off(counts, E, g, r0, r1, s.part, plan.rank_off);
        }
    }
    cluster_arrive();
    cluster_wait();
    const int e = tid;
    const bool ve = e < E;
    const int ld = !ve ? 0 : (C == 1 ? s.sload[e] : cluster.map_shared_rank(s.sload, 1 + (e >> 5) % (C - 1))[e]);
    cluster_arrive();          // #2; the matching wait is at the end of the kernel

    // ---- the plan ---------------------------------------------------------------
    int L;
    const int pre = block_excl_scan(ld, s.ws, &L);
    const int Q = L == 0 ? 0 : (L - 1) / N + 1;
    if (ve) s.pre[e] = pre;
    for (int r = tid; r < N; r += kPlanThreads) s.extra[r] = 0;
    for (int i = tid; i < NR; i += kPlanThreads) s.sasg[i] = -1;
    __syncthreads();

    // Home pass in closed form.
    int my_ovf = 0;
    if (ve) {
        const int h = e / H;
        const int pin = pre - s.pre[h * H];      // load of earlier experts of the same home rank
        const int take = min(Q, pin + ld) - min(Q, pin);
        my_ovf = ld - take;
        s.qh[e] = take;
        s.ovf[e] = my_ovf;
        s.acnt[e] = 0;
        s.afirst[e] = 0;
        if (e % H == H - 1) {
            const int rank_sum = pin + ld;
            s.before[h] = rank_sum;
            s.spare[h] = Q - min(Q, rank_sum);
        }
    }
    // Overflow experts as packed keys: larger overflow first, then lower id.
    int M1;
    const int pos = block_excl_scan(my_ovf > 0 ? 1 : 0, s.ws, &M1);
    if (my_ovf > 0) s.key[pos] = ((unsigned long long)(unsigned)my_ovf << 32) | (0xffffffffu - (unsigned)e);
    __syncthreads();
    if (tid < M1) {
        const unsigned long long mine = s.key[tid];
        int rank = 0;
#pragma unroll 8
        for (int k = 0; k < M1; ++k) rank += s.key[k] > mine ? 1 : 0;
        s.order[rank] = (int)(0xffffffffu - (unsigned)(mine & 0xffffffffu));
    }
    __syncthreads();

    if (R == 1) {
        // Eligible ranks (spare > 0) sorted by spare descending, lowest rank first.
        const int sp_r = tid < N ? s.spare[tid] : 0;
        int K;
        const int kpos = block_excl_scan(sp_r > 0 ? 1 : 0, s.ws, &K);
        if (sp_r > 0) s.key[kpos] = ((unsigned long long)(unsigned)sp_r << 32) | (0xffffffffu - (unsigned)tid);
        __syncthreads();
        int my_rank = 0, my_sp = 0;
        if (tid < K) {
            const unsigned long long mine = s.key[tid];
            int rank = 0;
#pragma unroll 8
            for (int k = 0; k < K; ++k) rank += s.key[k] > mine ? 1 : 0;
            my_rank = rank;
            my_sp = (int)(mine >> 32);
            s.rsorted[rank] = (int)(0xffffffffu - (unsigned)(mine & 0xffffffffu));
        }
        __syncthreads();
        if (tid < K) s.rsum[my_rank] = my_sp;   // spares in sorted order
        __syncthreads();
        const int sp_sorted = tid < K ? s.rsum[tid] : 0;
        int tot;
        const int ex = block_excl_scan(sp_sorted, s.ws, &tot);
        if (tid < K) s.rsum[tid] = ex;
        if (tid == 0) s.rsum[K] = tot;
        __syncthreads();
        if (warp == 0) greedy_sorted(s, K, M1);
    } else if (warp == 0) {
        greedy_chunks<NRL>(s, N, R, M1);
    }
    __syncthreads();
    const int n_asg = s.misc[0], stop_pos = s.misc[1], stop_rem = s.misc[2];
    const int flags = stop_pos < M1 ? 1 : 0;
    // Slots ran out at overflow position stop_pos: that expert's remainder and
    // the whole overflow of every later expert stay on their home slots.
    for (int p = stop_pos + tid; p < M1; p += kPlanThreads) {
        const int ep = s.order[p];
        const int res = p == stop_pos ? stop_rem : s.ovf[ep];
        s.qh[ep] += res;
        atomicAdd(&s.extra[ep / H], res);
        if (p != stop_pos) {
            s.afirst[ep] = 0;
            s.acnt[ep] = 0;
        }
    }
    __syncthreads();

    // Replica lists (CSR) and the replicated-expert list from one packed scan:
    // the low 16 bits count replica entries, the high bits replicated experts.
    const int na_e = ve ? s.acnt[e] : 0;
    const int packed = ve ? (1 + na_e) | ((na_e > 0 ? 1 : 0) << 16) : 0;
    int tot_packed;
    const int pk = block_excl_scan(packed, s.ws, &tot_packed);
    const int off = pk & 0xffff, mpos = pk >> 16;
    const int tot_rep = tot_packed & 0xffff, M = tot_packed >> 16;
    if (ve) {
        const int h = e / H;
        plan.rep_off[e] = off;
        plan.rep_slot[off] = h * HR + e % H;
        plan.rep_cum[off] = 0;
        int cum = s.qh[e];
        const int a0 = s.afirst[e];
        for (int i = 0; i < na_e; ++i) {
            const int a = a0 + i;
            plan.rep_slot[off + 1 + i] = s.ar[a] * HR + H + s.au[a];
            plan.rep_cum[off + 1 + i] = cum;
            cum += s.ac[a];
        }
        if (na_e > 0) plan.rep_experts[mpos] = e;
    }
    if (tid == 0) plan.rep_off[E] = tot_rep;
    for (int p = tot_rep + tid; p < cap; p += kPlanThreads) {
        plan.rep_slot[p] = -1;
        plan.rep_cum[p] = -1;
    }
    for (int p = M + tid; p < E; p += kPlanThreads) plan.rep_experts[p] = -1;

    // Slot table.
    for (int sl = tid; sl < S; sl += kPlanThreads) {
        const int r = sl / HR, u = sl % HR;
        int se, sq;
        if (u < H) {
            se = r * H + u;
            sq = s.qh[se];
        } else {
            const int a = s.sasg[r * R + (u - H)];
            se = a >= 0 ? s.ae[a] : -1;
            sq = a >= 0 ? s.ac[a] : 0;
        }
        plan.slot_expert[sl] = se;
        plan.slot_quota[sl] = sq;
    }

    // Rank loads before / after and their maxima.
    int mb = 0, ma = 0;
    for (int r = tid; r < N; r += kPlanThreads) {
        const int after = Q - s.spare[r] + s.extra[r];
        plan.rank_load_before[r] = s.before[r];
        plan.rank_load_after[r] = after;
        mb = max(mb, s.before[r]);
        ma = max(ma, after);
    }
    mb = __reduce_max_sync(0xffffffffu, mb);
    ma = __reduce_max_sync(0xffffffffu, ma);
    if (lane_id() == 0) {
        s.ws[warp] = mb;
        s.ws[32 + warp] = ma;
    }
    __syncthreads();
    if (tid == 0) {
        for (int w = 1; w < kPlanWarps; ++w) {
            mb = max(mb, s.ws[w]);
            ma = max(ma, s.ws[32 + w]);
        }
        plan.info[0] = Q;
        plan.info[1] = L;
        plan.info[2] = flags;
        plan.info[3] = M;
        plan.info[4] = n_asg;
        plan.info[5] = mb;
        plan.info[6] = ma;
        plan.info[7] = 0;
    }
    cluster_wait();
}

}  // namespace

size_t plan_smem_bytes(const Shape &sh) { return plan_smem_words(sh.E, sh.N, sh.NR) * sizeof(int32_t); }

int plan_cluster(const Shape &sh)
{
    const int groups = (sh.E + 31) / 32;
    if (groups <= 1) return 1;
    return groups + 1 < kMaxCluster ? groups + 1 : kMaxCluster;   // CTA 0 plans, peers own column groups
}

cudaError_t launch_plan(const Shape &sh, const int32_t *counts, const PlanDev &plan, cudaStream_t st, bool pdl)
{
    const unsigned C = (unsigned)plan_cluster(sh);
    const int nrl = (sh.N + 31) / 32;
    const size_t smem = plan_smem_bytes(sh);
#define UE_PLAN_LAUNCH(V) launch_ex(k_plan<V>, C, kPlanThreads, smem, st, C, pdl, counts, sh.E, sh.N, sh.R, plan)
    if (nrl <= 1) return UE_PLAN_LAUNCH(1);
    if (nrl <= 2) return UE_PLAN_LAUNCH(2);
    if (nrl <= 4) return UE_PLAN_LAUNCH(4);
    if (nrl <= 8) return UE_PLAN_LAUNCH(8);
    if (nrl <= 16) return UE_PLAN_LAUNCH(16);
    return UE_PLAN_LAUNCH(32);
#undef UE_PLAN_LAUNCH
}

cudaError_t set_plan_attributes(size_t max_smem)
{
    const int m = (int)max_smem;
    const cudaFuncAttribute a = cudaFuncAttributeMaxDynamicSharedMemorySize;
    cudaError_t e = cudaFuncSetAttribute(k_plan<1>, a, m);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(k_plan<2>, a, m);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(k_plan<4>, a, m);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(k_plan<8>, a, m);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(k_plan<16>, a, m);
    if (e == cudaSuccess) e = cudaFuncSetAttribute(k_plan<32>, a, m);
    return e;
}

}  // namespace ue
