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
//   Phase A (all CTAs, column blocks of 32 experts): column sums of counts
//     give load[e]; the exclusive column scan over ranks gives rank_off[r][e]
//     (what the reroute kernel needs).  CTA 0 then pulls every expert's load
//     from the owning CTA's shared memory over DSMEM.
//   Phase B (CTA 0): the home pass in closed form from a block-wide prefix
//     sum (the home rank's load before e is min(Q, in-rank prefix), so
//     take = min(Q, prefix + load) - min(Q, prefix)); the overflow order by
//     a rank-by-counting sort; the greedy in one warp, each rank's spare and
//     used-slot count held in the registers of lane r % 32, the argmax with
//     two redux.sync instructions per chunk (max spare, then min rank among
//     the lanes holding it); then all 1024 threads write the tables.
#include <climits>

#include <cooperative_groups.h>

#include "ue_internal.cuh"

namespace cg = cooperative_groups;

namespace ue {
namespace {

constexpr int kPlanThreads = 1024;
constexpr int kPlanWarps = kPlanThreads / 32;

// Shared-memory layout of the planner CTA (all int32).
struct PlanSmem {
    int32_t *part;      // [32][33] phase-A partial sums
    int32_t *ws;        // [64] scan / reduction scratch
    int32_t *misc;      // [8]  n_asg, flags
    int32_t *sload;     // [E]  loads of this CTA's column groups (CTA 0: all of them)
    int32_t *pre;       // [E]  exclusive prefix of load over experts
    int32_t *qh;        // [E]  home quota (plus any residual)
    int32_t *ovf;       // [E]
    int32_t *cl;        // [E]  experts with overflow (compacted)
    int32_t *order;     // [E]  overflow order
    int32_t *afirst;    // [E]  first assignment of e
    int32_t *acnt;      // [E]  number of assignments of e
    int32_t *before;    // [N]
    int32_t *spare;     // [N]
    int32_t *extra;     // [N]  residual overflow kept home
    int32_t *ar;        // [NR] assignment rank
    int32_t *au;        // [NR] assignment redundant index on that rank
    int32_t *ac;        // [NR] assignment quota
    int32_t *ae;        // [NR] assignment expert
    int32_t *sasg;      // [NR] (rank, redundant index) -> assignment or -1
};

__host__ __device__ inline size_t plan_smem_words(int E, int N, int NR)
{
    return (size_t)32 * 33 + 64 + 8 + (size_t)8 * E + (size_t)3 * N + (size_t)5 * NR;
}

__device__ __forceinline__ PlanSmem carve(int32_t *p, int E, int N, int NR)
{
    PlanSmem s;
    s.part = p;            p += 32 * 33;
    s.ws = p;              p += 64;
    s.misc = p;            p += 8;
    s.sload = p;           p += E;
    s.pre = p;             p += E;
    s.qh = p;              p += E;
    s.ovf = p;             p += E;
    s.cl = p;              p += E;
    s.order = p;           p += E;
    s.afirst = p;          p += E;
    s.acnt = p;            p += E;
    s.before = p;          p += N;
    s.spare = p;           p += N;
    s.extra = p;           p += N;
    s.ar = p;              p += NR;
    s.au = p;              p += NR;
    s.ac = p;              p += NR;
    s.ae = p;              p += NR;
    s.sasg = p;
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

__device__ int block_max(int v, int32_t *ws)
{
    const int lane = lane_id(), warp = threadIdx.x >> 5;
    v = __reduce_max_sync(0xffffffffu, v);
    if (lane == 0) ws[warp] = v;
    __syncthreads();
    int m = ws[0];
    for (int w = 1; w < kPlanWarps; ++w) m = max(m, ws[w]);
    __syncthreads();
    return m;
}

// The greedy overflow placement, run by warp 0.  Lane l owns ranks l, l+32, ...
// (NRL per lane), keeping spare capacity and used redundant slots in registers.
template <int NRL>
__device__ void greedy(const PlanSmem &s, int N, int R, int H, int M1)
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
    unsigned bs = 0;
    int br = INT_MAX;
    auto lane_best = [&]() {
        bs = 0;
        br = INT_MAX;
#pragma unroll
        for (int i = 0; i < NRL; ++i) {
            const int r = lane + 32 * i;
            const bool eligible = r < N && us[i] < R && sp[i] > 0u;
            if (eligible && sp[i] > bs) { bs = sp[i]; br = r; }   // strict: lowest rank on ties
        }
    };
    lane_best();

    int na = 0, flags = 0;
    for (int m = 0; m < M1; ++m) {
        const int e = s.order[m];
        int rem = s.ovf[e];
        const int first = na;
        while (rem > 0) {
            const unsigned mx = __reduce_max_sync(0xffffffffu, bs);
            if (mx == 0u) {                       // slots ran out: remainder stays home
                if (lane == 0) {
                    s.qh[e] += rem;
                    s.extra[e / H] += rem;
                }
                flags |= 1;
                break;
            }
            const int rs = __reduce_min_sync(0xffffffffu, bs == mx ? br : INT_MAX);
            const int c = rem < (int)mx ? rem : (int)mx;
            if (lane == (rs & 31)) {
                const int slot_i = rs >> 5;
                int u = 0;
#pragma unroll
                for (int i = 0; i < NRL; ++i) {
                    if (i == slot_i) {
                        u = us[i];
                        us[i] += 1;
                        sp[i] -= (unsigned)c;
                    }
                }
                s.ar[na] = rs;
                s.au[na] = u;
                s.ac[na] = c;
                s.ae[na] = e;
                s.sasg[rs * R + u] = na;
                lane_best();
            }
            rem -= c;
            ++na;
        }
        if (lane == 0) {
            s.afirst[e] = first;
            s.acnt[e] = na - first;
        }
    }
#pragma unroll
    for (int i = 0; i < NRL; ++i) {
        const int r = lane + 32 * i;
        if (r < N) s.spare[r] = (int)sp[i];
    }
    if (lane == 0) {
        s.misc[0] = na;
        s.misc[1] = flags;
    }
}

__global__ void __launch_bounds__(kPlanThreads, 1)
k_plan(const int32_t *__restrict__ counts, int E, int N, int R, PlanDev plan)
{
    extern __shared__ __align__(16) int32_t sm_plan[];
    const int H = E / N, HR = H + R, S = N * HR, NR = N * R, cap = E + NR;
    const PlanSmem s = carve(sm_plan, E, N, NR);

    cg::cluster_group cluster = cg::this_cluster();
    const int C = (int)cluster.num_blocks();
    const int c = (int)cluster.block_rank();
    const int tid = threadIdx.x, lane = lane_id(), warp = tid >> 5;

    // ---- phase A: loads and rank offsets, 32-expert column groups ----------
    const int rpg = (N + 31) / 32;               // ranks per row group
    const int r0 = min(N, warp * rpg), r1 = min(N, r0 + rpg);
    for (int g = c; g * 32 < E; g += C) {
        const int e = g * 32 + lane;
        const bool ve = e < E;
        int sum = 0;
        if (ve)
            for (int r = r0; r < r1; ++r) sum += __ldg(counts + (int64_t)r * E + e);
        s.part[warp * 33 + lane] = sum;
        __syncthreads();
        {   // warp w scans column w of the group over the 32 row groups (lane = row group)
            const int col = warp;
            const int v = s.part[lane * 33 + col];
            int x = v;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            s.part[lane * 33 + col] = x - v;
            const int ec = g * 32 + col;
            if (lane == 31 && ec < E) {
                plan.load[ec] = x;
                s.sload[ec] = x;          // pulled by CTA 0 after the cluster barrier
            }
        }
        __syncthreads();
        int run = s.part[warp * 33 + lane];
        if (ve)
            for (int r = r0; r < r1; ++r) {
                plan.rank_off[(int64_t)r * E + e] = run;
                run += __ldg(counts + (int64_t)r * E + e);
            }
        __syncthreads();
    }
    cluster.sync();
    if (c != 0) {              // keep this CTA's loads readable until CTA 0 has pulled them
        cluster_arrive();
        cluster_wait();
        return;
    }

    // ---- phase B: the plan, CTA 0 ---------------------------------------------
    const int e = tid;
    const bool ve = e < E;
    const int ld = ve ? cluster.map_shared_rank(s.sload, (e >> 5) % C)[e] : 0;
    cluster_arrive();
    cluster_wait();
    int L;
    const int pre = block_excl_scan(ld, s.ws, &L);
    const int Q = L == 0 ? 0 : (L - 1) / N + 1;
    if (ve) s.pre[e] = pre;
    for (int r = tid; r < N; r += kPlanThreads) s.extra[r] = 0;
    __syncthreads();

    // Home pass in closed form.
    if (ve) {
        const int h = e / H;
        const int pin = pre - s.pre[h * H];      // load of earlier experts of the same home rank
        const int take = min(Q, pin + ld) - min(Q, pin);
        s.qh[e] = take;
        s.ovf[e] = ld - take;
        s.acnt[e] = 0;
        s.afirst[e] = 0;
        if (e % H == H - 1) {
            const int rank_sum = pin + ld;
            s.before[h] = rank_sum;
            s.spare[h] = Q - min(Q, rank_sum);
        }
    }
    for (int i = tid; i < NR; i += kPlanThreads) s.sasg[i] = -1;

    // Overflow experts, then their order: overflow descending, lower id first.
    const int has_ovf = (ve && s.ovf[e] > 0) ? 1 : 0;   // read after the scan's barriers
    int M1;
    const int pos = block_excl_scan(has_ovf, s.ws, &M1);
    if (has_ovf) s.cl[pos] = e;
    __syncthreads();
    if (tid < M1) {
        const int ei = s.cl[tid], oi = s.ovf[ei];
        int rank = 0;
        for (int k = 0; k < M1; ++k) {
            const int ek = s.cl[k], ok = s.ovf[ek];
            rank += (ok > oi) || (ok == oi && ek < ei);
        }
        s.order[rank] = ei;
    }
    __syncthreads();

    // Greedy placement in warp 0.
    if (warp == 0) {
        const int nrl = (N + 31) / 32;
        if (nrl <= 1) greedy<1>(s, N, R, H, M1);
        else if (nrl <= 2) greedy<2>(s, N, R, H, M1);
        else if (nrl <= 4) greedy<4>(s, N, R, H, M1);
        else if (nrl <= 8) greedy<8>(s, N, R, H, M1);
        else if (nrl <= 16) greedy<16>(s, N, R, H, M1);
        else greedy<32>(s, N, R, H, M1);
    }
    __syncthreads();
    const int n_asg = s.misc[0], flags = s.misc[1];

    // Replica lists (CSR): home first, then allocation order.
    const int nrep = ve ? 1 + s.acnt[e] : 0;
    int tot_rep;
    const int off = block_excl_scan(nrep, s.ws, &tot_rep);
    if (ve) {
        const int h = e / H;
        plan.rep_off[e] = off;
        plan.rep_slot[off] = h * HR + e % H;
        plan.rep_cum[off] = 0;
        int cum = s.qh[e];
        const int a0 = s.afirst[e];
        for (int i = 0; i < s.acnt[e]; ++i) {
            const int a = a0 + i;
            plan.rep_slot[off + 1 + i] = s.ar[a] * HR + H + s.au[a];
            plan.rep_cum[off + 1 + i] = cum;
            cum += s.ac[a];
        }
    }
    if (tid == 0) plan.rep_off[E] = tot_rep;
    for (int p = tot_rep + tid; p < cap; p += kPlanThreads) {
        plan.rep_slot[p] = -1;
        plan.rep_cum[p] = -1;
    }

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

    // Experts holding redundant replicas, increasing id.
    const int rep_flag = (ve && s.acnt[e] > 0) ? 1 : 0;
    int M;
    const int mpos = block_excl_scan(rep_flag, s.ws, &M);
    if (rep_flag) plan.rep_experts[mpos] = e;
    for (int p = M + tid; p < E; p += kPlanThreads) plan.rep_experts[p] = -1;

    // Rank loads before / after.
    int mb = 0, ma = 0;
    for (int r = tid; r < N; r += kPlanThreads) {
        const int after = Q - s.spare[r] + s.extra[r];
        plan.rank_load_before[r] = s.before[r];
        plan.rank_load_after[r] = after;
        mb = max(mb, s.before[r]);
        ma = max(ma, after);
    }
    mb = block_max(mb, s.ws);
    ma = block_max(ma, s.ws);
    if (tid == 0) {
        plan.info[0] = Q;
        plan.info[1] = L;
        plan.info[2] = flags;
        plan.info[3] = M;
        plan.info[4] = n_asg;
        plan.info[5] = mb;
        plan.info[6] = ma;
        plan.info[7] = 0;
    }
}

}  // namespace

size_t plan_smem_bytes(const Shape &sh) { return plan_smem_words(sh.E, sh.N, sh.NR) * sizeof(int32_t); }

int plan_cluster(const Shape &sh)
{
    const int groups = (sh.E + 31) / 32;
    return groups < kMaxCluster ? groups : kMaxCluster;
}

cudaError_t launch_plan(const Shape &sh, const int32_t *counts, const PlanDev &plan, cudaStream_t st)
{
    const int C = plan_cluster(sh);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)C);
    cfg.blockDim = dim3(kPlanThreads);
    cfg.dynamicSmemBytes = plan_smem_bytes(sh);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = (unsigned)C;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, k_plan, counts, sh.E, sh.N, sh.R, plan);
}

cudaError_t set_plan_attributes(size_t max_smem)
{
    return cudaFuncSetAttribute(k_plan, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)max_smem);
}

}  // namespace ue
