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
// Design (sm_100a): one thread-block cluster of up to 8 CTAs.  Every
//   CTA other than CTA 0 sums a slice of the rank rows of counts into a partial
//   load vector in shared memory and arrives on the cluster barrier.  CTA 0
//   adds the partial vectors over DSMEM (the loads) and plans; meanwhile - off
//   the critical path - the other CTAs write the exclusive scan over ranks of
//   their row slices, rank_off[r][e], that the reroute kernel needs (the
//   partial vectors of the earlier slices give each slice its starting
//   offsets).  CTA 0 plans:
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

constexpr int kPlanMaxThreads = 1024;

// Shared-memory layout of a planner CTA (all 4-byte words unless noted).
struct PlanSmem {
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
    int32_t *rem;         // [E]  variants: remaining overflow of order[p]
    int32_t *alast;       // [E]  requeue: last assignment of e
    int32_t *anext;       // [NR] requeue: next assignment of the same expert, -1 at the end
    int32_t *stuck;       // [E]  experts left with overflow when slots ran out, in visit order
    int32_t *srem;        // [E]  their remainders
    int32_t *tmp;         // [NR+1] spread: the assignments of the expert being spread
    unsigned long long *key;   // [max(E, N)] packed sort keys (8-byte aligned)
    unsigned long long *key2;  // [N] R = 1: packed keys of the eligible ranks
};

__host__ __device__ inline size_t plan_smem_words(int E, int N, int NR)
{
    const int K = E > N ? E : N;
    return (size_t)96 + 8 + (size_t)11 * E + (size_t)5 * N + 1 + (size_t)7 * NR + 1 + 2 + (size_t)2 * K +
           (size_t)2 * N;
}

// Word offsets are computed as integers from the (16-byte aligned) base of the
// dynamic shared memory, so every pointer stays visibly derived from it and
// compiles to shared-memory instructions.
__device__ __forceinline__ PlanSmem carve(int32_t *p, int E, int N, int NR)
{
    PlanSmem s;
    int o = 0;
    s.ws = p + o;        o += 96;
    s.misc = p + o;      o += 8;
    s.sload = p + o;     o += E;
    s.pre = p + o;       o += E;
    s.qh = p + o;        o += E;
    s.ovf = p + o;       o += E;
    s.order = p + o;     o += E;
    s.afirst = p + o;    o += E;
    s.acnt = p + o;      o += E;
    s.before = p + o;    o += N;
    s.spare = p + o;     o += N;
    s.extra = p + o;     o += N;
    s.rsorted = p + o;   o += N;
    s.rsum = p + o;      o += N + 1;
    s.ar = p + o;        o += NR;
    s.au = p + o;        o += NR;
    s.ac = p + o;        o += NR;
    s.ae = p + o;        o += NR;
    s.sasg = p + o;      o += NR;
    s.rem = p + o;       o += E;
    s.alast = p + o;     o += E;
    s.anext = p + o;     o += NR;
    s.stuck = p + o;     o += E;
    s.srem = p + o;      o += E;
    s.tmp = p + o;       o += NR + 1;
    o = (o + 1) & ~1;                       // 8-byte alignment for the keys
    s.key = reinterpret_cast<unsigned long long *>(p + o);
    s.key2 = s.key + (E > N ? E : N);
    return s;
}

// Block-wide exclusive prefix sum of one value per thread (every thread of the
// block calls it; blockDim.x is a multiple of 32).
__device__ __forceinline__ int block_excl_scan(int v, int32_t *ws, int *total)
{
    const int lane = lane_id(), warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) ws[warp] = x;
    __syncthreads();
    if (warp == 0) {
        int w = lane < nw ? ws[lane] : 0;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, w, o);
            if (lane >= o) w += y;
        }
        ws[32 + lane] = w;   // inclusive prefix of warp sums
    }
    __syncthreads();
    const int r = (warp ? ws[32 + warp - 1] : 0) + x - v;
    *total = ws[32 + nw - 1];
    __syncthreads();
    return r;
}

constexpr int kRowBatch = 16;  // rows of counts loaded per batch (all loads in flight together)

// Row slice [r0, r1) of counts summed per expert into part[e].
__device__ __forceinline__ void slice_sums(const int32_t *__restrict__ counts, int E, int r0, int r1, int32_t *part)
{
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int acc = 0;
        for (int rb = r0; rb < r1; rb += kRowBatch) {
            int v[kRowBatch];
#pragma unroll
            for (int k = 0; k < kRowBatch; ++k) v[k] = rb + k < r1 ? __ldg(counts + (int64_t)(rb + k) * E + e) : 0;
#pragma unroll
            for (int k = 0; k < kRowBatch; ++k) acc += v[k];
        }
        part[e] = acc;
    }
}

// rank_off[r][e] for the rows [r0, r1), starting from the occurrences in the
// rows before r0: the partial vectors of the CTAs q0 <= q < c (over DSMEM).
__device__ __forceinline__ void slice_rank_off(cg::cluster_group &cluster, const int32_t *__restrict__ counts, int E,
                                               int r0, int r1, int c, int q0, int32_t *part,
                                               int32_t *__restrict__ rank_off)
{
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int prev[kMaxCluster];
#pragma unroll
        for (int q = 0; q < kMaxCluster; ++q) prev[q] = (q >= q0 && q < c) ? cluster.map_shared_rank(part, q)[e] : 0;
        int run = 0;
#pragma unroll
        for (int q = 0; q < kMaxCluster; ++q) run += prev[q];
        for (int rb = r0; rb < r1; rb += kRowBatch) {
            int v[kRowBatch];
#pragma unroll
            for (int k = 0; k < kRowBatch; ++k) v[k] = rb + k < r1 ? __ldg(counts + (int64_t)(rb + k) * E + e) : 0;
#pragma unroll
            for (int k = 0; k < kRowBatch; ++k) {
                if (rb + k < r1) rank_off[(int64_t)(rb + k) * E + e] = run;
                run += v[k];
            }
        }
    }
}

// R > 1: the chunk-by-chunk greedy, run by warp 0.
template <int NRL>
__device__ __forceinline__ void greedy_chunks(const PlanSmem &s, int N, int R, int M1)
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

// The two sorts of the planner as ranks (keys are unique; larger first):
// order[rank] of the M1 overflow keys s.key[0..M1), and for the K eligible
// ranks s.key2[0..K) their sorted position, rsorted[rank], and the sum of the
// spares (high words) of the keys above, rsum[rank] (rsum[K]: the total).  A
// group of g consecutive lanes shares one key, each lane comparing it with
// every g-th key of its array, four loads in flight; the group then adds its
// lanes' counts.  Both arrays are ranked in the same pass over the block.
__device__ __forceinline__ void rank_keys(const PlanSmem &s, int M1, int K)
{
    const int n = M1 + K, nt = blockDim.x;
    int g = 1;
    while (g < 32 && 2 * g * n <= nt) g *= 2;
    const int groups = nt / g, sub = threadIdx.x & (g - 1);
    const int off2 = (int)(s.key2 - s.key);
    for (int i0 = 0; i0 < n; i0 += groups) {       // the same trip count in every thread
        const int i = i0 + (int)threadIdx.x / g;
        const bool valid = i < n, first = i < M1;
        const int base = first ? 0 : off2, na = first ? M1 : K;
        const unsigned long long mine = valid ? s.key[base + (first ? i : i - M1)] : 0ull;
        int rank = 0;
        unsigned above = 0;                        // (overflow keys: unused)
        if (valid) {
            int k = sub;
            for (; k + 3 * g < na; k += 4 * g) {
                unsigned long long o[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) o[u] = s.key[base + k + u * g];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    rank += o[u] > mine ? 1 : 0;
                    above += o[u] > mine ? (unsigned)(o[u] >> 32) : 0u;
                }
            }
            for (; k < na; k += g) {
                const unsigned long long o = s.key[base + k];
                rank += o > mine ? 1 : 0;
                above += o > mine ? (unsigned)(o >> 32) : 0u;
            }
        }
        for (int x = 1; x < g; x <<= 1) {
            rank += __shfl_xor_sync(0xffffffffu, rank, x);
            above += __shfl_xor_sync(0xffffffffu, above, x);
        }
        if (valid && sub == 0) {
            const int id = (int)(0xffffffffu - (unsigned)(mine & 0xffffffffu));
            if (first) {
                s.order[rank] = id;
            } else {
                s.rsorted[rank] = id;
                s.rsum[rank] = (int)above;
                if (rank == K - 1) s.rsum[K] = (int)(above + (unsigned)(mine >> 32));
            }
        }
    }
}

// R = 1: walk the eligible ranks in sorted order (exclusive spare prefix
// s.rsum over K ranks); run by warp 0.  Expert m of the overflow order takes
// the sorted positions [cut[m], cut[m+1]) (recorded in s.afirst / s.acnt);
// assignment a is sorted position a, filled in by the whole block afterwards.
// The prefix values are held in registers, a window of 32 at a time, and the
// cuts of a batch of 32 experts are kept by their lanes and stored together,
// so each expert costs a compare, a ballot and two shuffles.
__device__ __forceinline__ void greedy_sorted(const PlanSmem &s, int K, int M1)
{
    const int lane = lane_id();
    int p = 0, stop_pos = M1, stop_rem = 0;
    unsigned rsum_p = 0;                              // s.rsum[p]
    int wbase = 1;                                    // window: lane holds s.rsum[wbase + lane]
    unsigned wv = wbase + lane <= K ? (unsigned)s.rsum[wbase + lane] : UINT_MAX;
    for (int m0 = 0; m0 < M1 && stop_pos == M1; m0 += 32) {
        const int idx = m0 + lane;
        const int e_l = idx < M1 ? s.order[idx] : 0;
        const int o_l = idx < M1 ? s.ovf[e_l] : 0;
        const int cnt = min(32, M1 - m0);
        int my_first = 0, my_end = 0;                 // the cut of expert m0 + lane
        int j = 0;
        for (; j < cnt; ++j) {
            const int rem = __shfl_sync(0xffffffffu, o_l, j);
            // The cut ends at the smallest q > p with rsum[q] >= target.  The
            // prefix is strictly increasing (spares > 0) and rem > 0, so that q
            // is the first position of the window at or above the target and
            // rsum[q] is the window's smallest value at or above it: one
            // redux.sync on the critical path; the position by a ballot beside
            // it.  Values stay below 2^32: a spare sum and an overflow are each
            // below 2^31.
            const unsigned target = rsum_p + (unsigned)rem;
            unsigned rq = __reduce_min_sync(0xffffffffu, wv >= target ? wv : UINT_MAX);
            while (rq == UINT_MAX && wbase + 32 <= K) {   // the whole window is below the target
                wbase += 32;
                wv = wbase + lane <= K ? (unsigned)s.rsum[wbase + lane] : UINT_MAX;
                rq = __reduce_min_sync(0xffffffffu, wv >= target ? wv : UINT_MAX);
            }
            if (rq == UINT_MAX) {                     // every remaining rank used: the rest stays home
                my_first = lane == j ? p : my_first;
                my_end = lane == j ? K : my_end;
                stop_pos = m0 + j;
                stop_rem = rem - (s.rsum[K] - (int)rsum_p);
                p = K;
                ++j;
                break;
            }
            const int q = wbase + __popc(__ballot_sync(0xffffffffu, wv < target));
            my_first = lane == j ? p : my_first;
            my_end = lane == j ? q : my_end;
            p = q;
            rsum_p = rq;
        }
        if (lane < j) {
            s.afirst[e_l] = my_first;
            s.acnt[e_l] = my_end - my_first;
            s.rem[m0 + lane] = my_first;          // cut start by overflow position
        }
    }
    if (lane == 0) {
        s.misc[0] = p;
        s.misc[1] = stop_pos;
        s.misc[2] = stop_rem;
    }
}

// Variant REQUEUE: after every chunk the expert with the largest remaining
// overflow (ties: lower id) is placed next; run by warp 0.  Lane l owns the
// overflow-order positions l, l + 32, ... (rem[p] = what order[p] still has to
// place) and keeps the best of them as one 32-bit key (remaining << 10 |
// 1023 - id, so that one redux.sync max picks the expert, ties to the lower id)
// while every overflow is below 2^22; otherwise the pick takes two redux.sync.
// Only the owner of the expert just served rescans its positions.  Ranks: with
// R = 1 a rank is chosen at most once and its spare does not change before, so
// the k-th chunk goes to the k-th rank of the ranks sorted by initial spare
// (rsorted, K of them); with R > 1 the argmax of greedy_chunks.  An expert's
// assignments are chained in allocation order through afirst / anext.
template <int NRL>
__device__ __forceinline__ void greedy_requeue(const PlanSmem &s, int N, int R, int M1, int K)
{
    const int lane = lane_id();
    unsigned sp[NRL];
    int us[NRL];
    unsigned bs = 0;
    int br = INT_MAX;
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
    if (R > 1) {
#pragma unroll
        for (int i = 0; i < NRL; ++i) {
            const int r = lane + 32 * i;
            sp[i] = r < N ? (unsigned)s.spare[r] : 0u;
            us[i] = 0;
        }
        lane_best();
    }
    int omax = 0;
    for (int p = lane; p < M1; p += 32) {
        const int o = s.ovf[s.order[p]];
        s.rem[p] = o;
        omax = max(omax, o);
    }
    const bool packed = __reduce_max_sync(0xffffffffu, omax) < (1 << 22);
    __syncwarp();
    unsigned bkey;                 // packed: the lane's best key
    int brem, bid, bpos;
    auto expert_best = [&]() {
        brem = 0;
        bid = INT_MAX;
        bpos = 0;
        for (int p = lane; p < M1; p += 32) {
            const int r = s.rem[p], e = s.order[p];
            if (r > brem || (r == brem && r > 0 && e < bid)) {
                brem = r;
                bid = e;
                bpos = p;
            }
        }
        bkey = brem > 0 ? ((unsigned)brem << 10) | (1023u - (unsigned)bid) : 0u;
    };
    expert_best();
    int na = 0;
    bool ran_out = false;
    for (;;) {
        int mx, e, el;
        if (packed) {
            const unsigned k = __reduce_max_sync(0xffffffffu, bkey);
            if (k == 0u) break;                                  // every overflow placed
            mx = (int)(k >> 10);
            e = 1023 - (int)(k & 1023u);
            el = __ffs(__ballot_sync(0xffffffffu, bkey == k)) - 1;
        } else {
            mx = __reduce_max_sync(0xffffffffu, brem);
            if (mx == 0) break;
            e = __reduce_min_sync(0xffffffffu, brem == mx ? bid : INT_MAX);
            el = __ffs(__ballot_sync(0xffffffffu, brem == mx && bid == e)) - 1;
        }
        int rs, spare_rs, u = 0;
        if (R == 1) {
            if (na >= K) {                                       // every eligible rank used
                ran_out = true;
                break;
            }
            rs = s.rsorted[na];
            spare_rs = s.rsum[na + 1] - s.rsum[na];
        } else {
            const unsigned ms = __reduce_max_sync(0xffffffffu, bs);
            if (ms == 0u) {                                      // no eligible rank left
                ran_out = true;
                break;
            }
            rs = __reduce_min_sync(0xffffffffu, bs == ms ? br : INT_MAX);
            spare_rs = (int)ms;
        }
        const int c = mx < spare_rs ? mx : spare_rs;
        if (R > 1) {
            const bool own = lane == (rs & 31);
            const int si = rs >> 5;
#pragma unroll
            for (int i = 0; i < NRL; ++i) {
                const bool hit = own && i == si;
                u = hit ? us[i] : u;
                us[i] += hit ? 1 : 0;
                sp[i] -= hit ? (unsigned)c : 0u;
            }
            lane_best();
            u = __shfl_sync(0xffffffffu, u, rs & 31);
        }
        if (lane == el) {                                        // the owner of e records the chunk
            s.ar[na] = rs;
            s.au[na] = u;
            s.ac[na] = c;
            s.ae[na] = e;
            s.sasg[rs * R + u] = na;
            s.anext[na] = -1;
            const int last = s.alast[e];
            if (last >= 0) s.anext[last] = na;
            else s.afirst[e] = na;
            s.alast[e] = na;
            s.acnt[e] += 1;
            s.rem[bpos] = mx - c;
            if (R == 1) s.spare[rs] -= c;
            expert_best();
        }
        ++na;
    }
    if (R > 1) {
#pragma unroll
        for (int i = 0; i < NRL; ++i) {
            const int r = lane + 32 * i;
            if (r < N) s.spare[r] = (int)sp[i];
        }
    }
    if (lane == 0) {
        s.misc[0] = na;
        s.misc[1] = ran_out ? 0 : M1;
        s.misc[2] = 0;
    }
}

// Variant SPREAD, run by warp 0 over the ns stuck experts in visit order:
// each remainder goes token by token to the replica whose rank has the lowest
// load (ties: the earlier replica, home first).  In closed form: the replicas
// are filled up to the level lam with f(lam) = sum_i max(0, lam - l_i) <= res
// < f(lam + 1), and the t = res - f(lam) tokens left go one each to the first
// t replicas (in replica order) whose load is then lam.  Rank load =
// Q - spare + extra.  chained: assignments linked through anext (REQUEUE),
// else contiguous from afirst.  With at most 32 replicas and res < 2^26 the
// loads stay in registers and f is one redux.sync add of terms clamped to
// res + 1 (the sum then fits 32 bits); otherwise a 64-bit shuffle sum.
__device__ __forceinline__ void spread_stuck(const PlanSmem &s, int ns, int Q, int H, bool chained)
{
    const int lane = lane_id();
    for (int k = 0; k < ns; ++k) {
        const int e = s.stuck[k], h = e / H, res = s.srem[k];
        const int nred = s.acnt[e];
        if (nred == 0 || res == 0) {
            if (lane == 0) {
                s.qh[e] += res;
                s.extra[h] += res;
            }
            __syncwarp();
            continue;
        }
        if (lane == 0) {
            int a = s.afirst[e];
            for (int i = 0; i < nred; ++i) {
                s.tmp[i] = a;
                a = chained ? s.anext[a] : a + 1;
            }
        }
        __syncwarp();
        const int n = 1 + nred;
        auto rank_of = [&](int i) { return i == 0 ? h : s.ar[s.tmp[i - 1]]; };
        auto load_of = [&](int i) {
            const int r = rank_of(i);
            return Q - s.spare[r] + s.extra[r];
        };
        int lam;
        if (n <= 32 && res < (1 << 26)) {
            const int my = lane < n ? load_of(lane) : INT_MAX;
            const int minl = __reduce_min_sync(0xffffffffu, my);
            int lo = minl, hi = minl + res;
            while (lo < hi) {
                const int mid = lo + (hi - lo + 1) / 2;
                const unsigned term = lane < n && mid > my ? (unsigned)min(mid - my, res + 1) : 0u;
                if (__reduce_add_sync(0xffffffffu, term) <= (unsigned)res) lo = mid;
                else hi = mid - 1;
            }
            lam = lo;
        } else {
            int minl = INT_MAX;
            for (int i = lane; i < n; i += 32) minl = min(minl, load_of(i));
            minl = __reduce_min_sync(0xffffffffu, minl);
            auto fill = [&](int x) {
                long long f = 0;
                for (int i = lane; i < n; i += 32) f += max(0, x - load_of(i));
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) f += __shfl_xor_sync(0xffffffffu, f, o);
                return f;
            };
            int lo = minl, hi = minl + res;
            while (lo < hi) {
                const int mid = lo + (hi - lo + 1) / 2;
                if (fill(mid) <= res) lo = mid;
                else hi = mid - 1;
            }
            lam = lo;
        }
        // f(lam) and the replicas at or below lam, in replica order.
        long long f = 0;
        for (int i = lane; i < n; i += 32) f += max(0, lam - load_of(i));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) f += __shfl_xor_sync(0xffffffffu, f, o);
        const int t = res - (int)f;           // < number of replicas at or below lam
        int seen = 0;
        for (int i0 = 0; i0 < n; i0 += 32) {
            const int i = i0 + lane;
            const int l = i < n ? load_of(i) : INT_MAX;
            const bool at = i < n && l <= lam;
            const unsigned b = __ballot_sync(0xffffffffu, at);
            const int add = at ? (lam - l) + ((seen + __popc(b & lanemask_lt())) < t ? 1 : 0) : 0;
            __syncwarp();                     // every load of the batch read before any update
            if (add > 0) {
                const int r = rank_of(i);
                if (i == 0) s.qh[e] += add;
                else s.ac[s.tmp[i - 1]] += add;
                s.extra[r] += add;            // replicas of one expert sit on distinct ranks
            }
            seen += __popc(b);
            __syncwarp();
        }
    }
}

// The plan's slot table, and (loads) the rank loads before / after with their
// maxima (info[5], info[6]), from CTA 0's final plan state read over DSMEM:
// the part of a cluster's output its helper CTAs write while CTA 0 writes the
// replica lists.  Helper hc of nh takes every nh-th run of blockDim.x slots.
__device__ __forceinline__ void plan_tail(cg::cluster_group &cluster, const PlanSmem &s, const PlanDev &plan, int hc,
                                          int nh, int N, int R, int H, int HR, int S, bool loads)
{
    const int32_t *qh = cluster.map_shared_rank(s.qh, 0);
    const int32_t *sasg = cluster.map_shared_rank(s.sasg, 0);
    const int32_t *ae = cluster.map_shared_rank(s.ae, 0);
    const int32_t *ac = cluster.map_shared_rank(s.ac, 0);
    for (int sl = hc * (int)blockDim.x + (int)threadIdx.x; sl < S; sl += nh * (int)blockDim.x) {
        const int r = sl / HR, u = sl % HR;
        int se, sq;
        if (u < H) {
            se = r * H + u;
            sq = qh[se];
        } else {
            const int a = sasg[r * R + (u - H)];
            se = a >= 0 ? ae[a] : -1;
            sq = a >= 0 ? ac[a] : 0;
        }
        plan.slot_expert[sl] = se;
        plan.slot_quota[sl] = sq;
    }
    if (!loads) return;
    const int32_t *spare = cluster.map_shared_rank(s.spare, 0);
    const int32_t *extra = cluster.map_shared_rank(s.extra, 0);
    const int32_t *before = cluster.map_shared_rank(s.before, 0);
    const int Q = cluster.map_shared_rank(s.misc, 0)[4];
    const int warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
    int mb = 0, ma = 0;
    for (int r = threadIdx.x; r < N; r += blockDim.x) {
        const int b = before[r], after = Q - spare[r] + extra[r];
        plan.rank_load_before[r] = b;
        plan.rank_load_after[r] = after;
        mb = max(mb, b);
        ma = max(ma, after);
    }
    mb = __reduce_max_sync(0xffffffffu, mb);
    ma = __reduce_max_sync(0xffffffffu, ma);
    if (lane_id() == 0) {
        s.ws[warp] = mb;
        s.ws[32 + warp] = ma;
    }
    __syncthreads();
    if (warp == 0) {
        mb = __reduce_max_sync(0xffffffffu, lane_id() < nw ? s.ws[lane_id()] : 0);
        ma = __reduce_max_sync(0xffffffffu, lane_id() < nw ? s.ws[32 + lane_id()] : 0);
        if (threadIdx.x == 0) {
            plan.info[5] = mb;
            plan.info[6] = ma;
        }
    }
}

// kVariants = false compiles the stated rule alone (variant is ignored), so
// the default planner carries none of the variants' code.
template <int NRL, bool kVariants>
__global__ void __launch_bounds__(kPlanMaxThreads, 1)
k_plan(const int32_t *__restrict__ counts, int E, int N, int R, int variant, PlanDev plan, int32_t *lv)
{
    extern __shared__ __align__(16) int32_t sm_plan[];
    const int H = E / N, HR = H + R, S = N * HR, NR = N * R, cap = E + NR;
    const PlanSmem s = carve(sm_plan, E, N, NR);

    cg::cluster_group cluster = cg::this_cluster();
    const int C = (int)cluster.num_blocks();
    const int c = (int)cluster.block_rank();
    const int tid = threadIdx.x, nt = blockDim.x, warp = tid >> 5;
    // This CTA's slice of the rank rows of counts.  With a cluster, CTA 0 holds
    // no rows (it only plans) and the other CTAs split them.
    const int slices = C > 1 ? C - 1 : 1, sl_id = C > 1 ? c - 1 : 0;
    const int rows = (N + slices - 1) / slices;
    const int r0 = (C > 1 && c == 0) ? N : min(N, sl_id * rows);
    const int r1 = (C > 1 && c == 0) ? N : min(N, r0 + rows);

    // The reroute grid may launch now (its first pass needs only the ids);
    // the counts of the load grid are read after it completes.
    pdl_trigger();
    pdl_wait();

    // direct: the load grid summed the expert loads into lv, which CTA 0 reads
    // (and sets back to zeros) without waiting for the slices, whose partial
    // vectors then serve rank_off alone.
    const bool direct = lv != nullptr && c == 0;
    if (!direct && (C == 1 || c != 0)) slice_sums(counts, E, r0, r1, s.sload);
    // #1: this slice's partial loads are ready (CTA 0 of a cluster publishes none).
    if (c == 0 && C > 1) cluster_arrive_relaxed();
    else cluster_arrive();
    if (!direct) cluster_wait();
    if (c != 0) {
        // Off the critical path: rank_off for this slice (the slices of the
        // lower peers give its start), then stay resident until every CTA has
        // read this CTA's partial vector.
        slice_rank_off(cluster, counts, E, r0, r1, c, 1, s.sload, plan.rank_off);
        cluster_arrive_relaxed();   // #2: done reading the lower peers
        cluster_wait();             // #2: CTA 0's plan state is final (it arrived with release)
        plan_tail(cluster, s, plan, c - 1, C - 1, N, R, H, HR, S, c == 1);
        cluster_arrive_relaxed();   // #3: done reading CTA 0
        cluster_wait();
        return;
    }
    const int e = tid;
    const bool ve = e < E;
    int ld = 0;
    if (ve) {
        if (direct) {
            ld = __ldcg(lv + e);
            lv[e] = 0;
        } else if (C == 1) {
            ld = s.sload[e];
        } else {
            int part[kMaxCluster];
#pragma unroll
            for (int q = 1; q < kMaxCluster; ++q) part[q] = q < C ? cluster.map_shared_rank(s.sload, q)[e] : 0;
#pragma unroll
            for (int q = 1; q < kMaxCluster; ++q) ld += part[q];
        }
        plan.load[e] = ld;
    }
    if (!direct && C == 1) cluster_arrive_relaxed();  // #2 (a cluster of one)

    // ---- the plan (CTA 0; blockDim >= max(E, N)) ---------------------------------
    int L;
    const int pre = block_excl_scan(ld, s.ws, &L);
    const int Q = L == 0 ? 0 : (L - 1) / N + 1;
    if (ve) s.pre[e] = pre;
    if (tid == 0) s.misc[4] = Q;                  // for the rank loads (plan_tail)
    for (int r = tid; r < N; r += nt) s.extra[r] = 0;
    for (int i = tid; i < NR; i += nt) s.sasg[i] = -1;
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
        s.alast[e] = -1;
    }
    // Rank tid's home load and spare, from the prefix of the loads.
    int my_spare = 0;
    if (tid < N) {
        const int rank_sum = (tid + 1 < N ? s.pre[(tid + 1) * H] : L) - s.pre[tid * H];
        my_spare = Q - min(Q, rank_sum);
        s.before[tid] = rank_sum;
        s.spare[tid] = my_spare;
    }
    // Overflow experts (larger overflow first, then lower id) and, for R = 1,
    // the eligible ranks (spare > 0; larger spare first, then lower rank) as
    // packed keys, both compacted by one scan (experts in the low 16 bits).
    const bool eligible = R == 1 && my_spare > 0;
    int packed_tot;
    const int pk0 = block_excl_scan((my_ovf > 0 ? 1 : 0) | (eligible ? 1 << 16 : 0), s.ws, &packed_tot);
    const int M1 = packed_tot & 0xffff, K = packed_tot >> 16;
    if (my_ovf > 0) s.key[pk0 & 0xffff] = ((unsigned long long)(unsigned)my_ovf << 32) | (0xffffffffu - (unsigned)e);
    if (eligible) s.key2[pk0 >> 16] = ((unsigned long long)(unsigned)my_spare << 32) | (0xffffffffu - (unsigned)tid);
    if (tid == 0 && K == 0) s.rsum[0] = 0;        // no eligible rank: an empty prefix
    __syncthreads();
    rank_keys(s, M1, K);
    __syncthreads();

    const bool requeue = kVariants && (variant & 1) != 0, spread = kVariants && (variant & 2) != 0;
    if (R == 1) {
        if (requeue) {
            if (warp == 0) greedy_requeue<NRL>(s, N, R, M1, K);
        } else {
            if (warp == 0) greedy_sorted(s, K, M1);
            __syncthreads();
            // Fill the assignments: expert m of the overflow order owns the sorted
            // positions of its cut; every rank is full except the last rank of an
            // expert that was placed completely (m before the stop), which takes
            // what is left of the expert's overflow.
            // One thread per assignment: its expert is the last overflow
            // position (among those the walk reached) whose cut starts at or
            // before it (s.rem holds the cut starts by position).
            const int n_a = s.misc[0], stop = s.misc[1];
            const int nproc = stop < M1 ? stop + 1 : M1;
            for (int a = tid; a < n_a; a += nt) {
                int lo = 0, hi = nproc - 1;
                while (lo < hi) {
                    const int mid = (lo + hi + 1) >> 1;
                    if (s.rem[mid] <= a) lo = mid;
                    else hi = mid - 1;
                }
                const int em = s.order[lo];
                const int a0 = s.rem[lo], na = s.acnt[em];
                const int r = s.rsorted[a];
                int q = s.rsum[a + 1] - s.rsum[a];
                if (lo < stop && a == a0 + na - 1) q = s.ovf[em] - (s.rsum[a] - s.rsum[a0]);
                s.ar[a] = r;
                s.au[a] = 0;
                s.ac[a] = q;
                s.ae[a] = em;
                s.sasg[r] = a;
                s.spare[r] -= q;
            }
        }
    } else if (requeue) {
        if (warp == 0) greedy_requeue<NRL>(s, N, R, M1, 0);
    } else if (warp == 0) {
        greedy_chunks<NRL>(s, N, R, M1);
    }
    __syncthreads();
    const int n_asg = s.misc[0], stop_pos = s.misc[1], stop_rem = s.misc[2];
    const int flags = stop_pos < M1 ? 1 : 0;
    if (!requeue) {
        // Slots ran out at overflow position stop_pos: that expert's remainder
        // and the whole overflow of every later expert are stuck, in this order.
        for (int p = stop_pos + tid; p < M1; p += nt) {
            const int ep = s.order[p];
            const int res = p == stop_pos ? stop_rem : s.ovf[ep];
            if (p != stop_pos) {
                s.afirst[ep] = 0;
                s.acnt[ep] = 0;
            }
            if (spread) {
                s.stuck[p - stop_pos] = ep;
                s.srem[p - stop_pos] = res;
            } else {                      // the stated rule: the remainder stays home
                s.qh[ep] += res;
                atomicAdd(&s.extra[ep / H], res);
            }
        }
        if (spread) {
            __syncthreads();
            if (warp == 0) spread_stuck(s, M1 - stop_pos, Q, H, false);
        }
    } else if (flags) {
        // Re-queued overflow: the stuck experts are those with overflow left,
        // visited largest remainder first (ties: lower id).
        const int rp = tid < M1 ? s.rem[tid] : 0;
        const int ep = tid < M1 ? s.order[tid] : 0;
        int ns;
        const int kp = block_excl_scan(rp > 0 ? 1 : 0, s.ws, &ns);
        if (rp > 0) s.key[kp] = ((unsigned long long)(unsigned)rp << 32) | (0xffffffffu - (unsigned)ep);
        __syncthreads();
        if (tid < ns) {
            const unsigned long long mine = s.key[tid];
            int rank = 0;
            for (int k = 0; k < ns; ++k) rank += s.key[k] > mine ? 1 : 0;
            const int ek = (int)(0xffffffffu - (unsigned)(mine & 0xffffffffu));
            const int rk = (int)(mine >> 32);
            s.stuck[rank] = ek;
            s.srem[rank] = rk;
            if (!spread) {
                s.qh[ek] += rk;
                atomicAdd(&s.extra[ek / H], rk);
            }
        }
        if (spread) {
            __syncthreads();
            if (warp == 0) spread_stuck(s, ns, Q, H, true);
        }
    }
    __syncthreads();
    if (C > 1) {
        // #2: the plan state the helpers read (qh, sasg, ae, ac, spare, extra,
        // before, Q) is final; they write the slot table and the rank loads.
        if (direct) cluster_wait();     // #1, skipped above
        cluster_arrive();
    }

    // Replica lists (CSR) and the replicated-expert list from one packed scan:
    // the low 16 bits count replica entries, the high bits replicated experts.
    const int na_e = ve ? s.acnt[e] : 0;
    const int packed = ve ? (1 + na_e) | ((na_e > 0 ? 1 : 0) << 16) : 0;
    int tot_packed;
    const int pk = block_excl_scan(packed, s.ws, &tot_packed);
    const int off = pk & 0xffff, mpos = pk >> 16;
    const int tot_rep = tot_packed & 0xffff, M = tot_packed >> 16;
    // R = 1 under the stated rule: an expert's assignments are consecutive
    // sorted positions and all but its last are full ranks, so the cumulative
    // quota before assignment a is qh + rsum[a] - rsum[first]: one thread per
    // assignment writes its entry.
    const bool sorted_csr = R == 1 && !requeue && !spread;
    if (ve) {
        const int h = e / H;
        plan.rep_off[e] = off;
        plan.rep_slot[off] = h * HR + e % H;
        plan.rep_cum[off] = 0;
        if (sorted_csr) {
            s.pre[e] = off;                       // (reused) replica-list offset of e
        } else {
            int cum = s.qh[e];
            int a = s.afirst[e];
            for (int i = 0; i < na_e; ++i) {
                plan.rep_slot[off + 1 + i] = s.ar[a] * HR + H + s.au[a];
                plan.rep_cum[off + 1 + i] = cum;
                cum += s.ac[a];
                a = requeue ? s.anext[a] : a + 1;
            }
        }
        if (na_e > 0) plan.rep_experts[mpos] = e;
    }
    if (sorted_csr) {
        __syncthreads();
        for (int a = tid; a < n_asg; a += nt) {
            const int ea = s.ae[a], a0 = s.afirst[ea];
            const int entry = s.pre[ea] + 1 + (a - a0);
            plan.rep_slot[entry] = s.ar[a] * HR + H;
            plan.rep_cum[entry] = s.qh[ea] + s.rsum[a] - s.rsum[a0];
        }
    }
    if (tid == 0) plan.rep_off[E] = tot_rep;
    for (int p = tot_rep + tid; p < cap; p += nt) {
        plan.rep_slot[p] = -1;
        plan.rep_cum[p] = -1;
    }
    for (int p = M + tid; p < E; p += nt) plan.rep_experts[p] = -1;

    if (C == 1) {
        plan_tail(cluster, s, plan, 0, 1, N, R, H, HR, S, true);
        if (tid == 0) {
            plan.info[0] = Q;
            plan.info[1] = L;
            plan.info[2] = flags;
            plan.info[3] = M;
            plan.info[4] = n_asg;
            plan.info[7] = 0;
        }
        slice_rank_off(cluster, counts, E, r0, r1, 0, 0, s.sload, plan.rank_off);
        if (direct) {          // the barrier phases CTA 0 skipped above
            cluster_wait();    // #1
            cluster_arrive_relaxed();   // #2
        }
        cluster_wait();        // #2
        return;
    }
    if (tid == 0) {            // info[5], info[6]: the rank loads' maxima, by helper CTA 1
        plan.info[0] = Q;
        plan.info[1] = L;
        plan.info[2] = flags;
        plan.info[3] = M;
        plan.info[4] = n_asg;
        plan.info[7] = 0;
    }
    cluster_wait();                // #2
    cluster_arrive_relaxed();      // #3
    cluster_wait();                // #3: the helpers have read this CTA's plan state
}

}  // namespace

size_t plan_smem_bytes(const Shape &sh) { return plan_smem_words(sh.E, sh.N, sh.NR) * sizeof(int32_t); }

// Threads of a planner CTA: one per expert and one per rank at least; more
// when counts is large so that each thread sums at most ~8 values per slice.
int plan_threads(const Shape &sh)
{
    int t = sh.E > sh.N ? sh.E : sh.N;
    t = (t + 31) / 32 * 32;
    if (t < 64) t = 64;
    const int64_t cells = (int64_t)sh.N * sh.E;
    while (t < kPlanMaxThreads && cells > (int64_t)8 * kMaxCluster * t) t *= 2;
    return t < kPlanMaxThreads ? t : kPlanMaxThreads;
}

// CTAs of the planner cluster: enough row slices that each thread sums at most ~8 rows.
int plan_cluster(const Shape &sh)
{
    const int64_t per_cta = (int64_t)8 * plan_threads(sh);
    int C = 1;
    while (C < kMaxCluster && (int64_t)sh.N * sh.E > per_cta * C) C *= 2;
    return C < sh.N ? C : (sh.N < 1 ? 1 : sh.N);
}

cudaError_t launch_plan(const Shape &sh, const int32_t *counts, const PlanDev &plan, cudaStream_t st, bool pdl,
                        int variant, int32_t *lv)
{
    const unsigned C = (unsigned)plan_cluster(sh);
    const unsigned threads = (unsigned)plan_threads(sh);
    const int nrl = (sh.N + 31) / 32;
    const size_t smem = plan_smem_bytes(sh);
#define UE_PLAN_LAUNCH(V)                                                                                       \
    (variant ? launch_ex(k_plan<V, true>, C, threads, smem, st, C, pdl, counts, sh.E, sh.N, sh.R, variant, plan, lv) \
             : launch_ex(k_plan<V, false>, C, threads, smem, st, C, pdl, counts, sh.E, sh.N, sh.R, 0, plan, lv))
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
    for (auto k : {k_plan<1, false>, k_plan<2, false>, k_plan<4, false>, k_plan<8, false>, k_plan<16, false>,
                   k_plan<32, false>, k_plan<1, true>, k_plan<2, true>, k_plan<4, true>, k_plan<8, true>,
                   k_plan<16, true>, k_plan<32, true>}) {
        const cudaError_t e = allow_smem(k, max_smem);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace ue
