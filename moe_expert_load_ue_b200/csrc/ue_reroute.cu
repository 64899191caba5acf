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
// move four ids per lane with 16-byte accesses when the share is aligned.
// From the counts and the bases each warp then knows, per expert, whether all
// of its occurrences fall into one replica's quota range (an expert with one
// replica always does; so does almost every (warp, expert) pair of a
// replicated one), and a per-warp table maps every expert to that slot, or
// marks it with the warp's running occurrence index.  Pass 2 is one shared
// load per id; a block of 128 ids whose marked ids all belong to one expert
// and stay inside one replica range advances the running index by their
// count; only a block that straddles a quota boundary ranks its ids exactly,
// by ballots over the bits of the expert id.
//
// Dispatch layout (token dispatch consumes the physical routing: "Routing
// expansion -> Token dispatch: physical routing", "Token dispatch -> Expert
// compute: dispatches tokens").  The dispatch variant of the kernel also groups
// the assignments by slot: with slot_off the exclusive prefix of the plan's
// slot quotas, the assignment with occurrence index j that replica entry p
// (slot rep_slot[p], cumulative quota rep_cum[p]) serves lands at position
//     slot_off[rep_slot[p]] + j - rep_cum[p]
// of src_index (its flat index t*K + k) and gates_out (its gate), i.e. a
// stable grouping by slot computed in the same pass.  Every valid id then
// needs its occurrence index, so this variant ranks every id of a warp step
// by ballots over the bits of the expert id.
#include <climits>

#include <cooperative_groups.h>

#include "ue_internal.cuh"

namespace cg = cooperative_groups;

namespace ue {
namespace {

constexpr int kRerouteWarps = 16;
constexpr int kUnroll = 4;
constexpr int kStageIds = 8192;   // ids of a CTA share kept in shared memory between the passes
constexpr int kRepCache = 64;     // replicated experts whose current replica each warp caches

// Kernel-side view of the dispatch outputs (unused by the plain variant).
struct DispatchArgs {
    const float *gates;            // [T*K] or nullptr
    const int32_t *slot_quota;     // [S] the plan's slot quotas
    int32_t *slot_off;             // [S+1] out (written by CTA 0)
    int32_t *src_index;            // [T*K] out
    float *gates_out;              // [T*K] out when gates != nullptr
    int32_t *err;                  // device status word: bit 1 = ids do not match the plan's quotas
    int64_t L;                     // T*K: capacity of src_index / gates_out
    int S;
};

struct RerouteSmem {
    int32_t *hist;   // [W][E] per-warp counts, then their exclusive scan over the warps
    int32_t *code;   // [W][E] per warp and expert: its slot, or -2 - the warp's next occurrence index
                     //        (dispatch variant: [32] partial sums of the slot-offset scan)
    int2 *cc;        // [W][kRepCache] plain: per warp and replicated expert (list position), the slot of
                     //        the replica holding the warp's next occurrence and where that replica ends
    int32_t *tot;    // [E]    this CTA's counts (read by later CTAs of the cluster)
    int32_t *base;   // [E]    occurrences of e before this CTA's ids
    int32_t *rexp;   // [E+1]  plain: the replicated experts and their count; dispatch variant:
                     //        exclusive prefix of this CTA's per-expert counts
    int2 *tab;       // [E]    {home slot if one replica, else first replica entry; (compact index << 16) | count}
    int2 *rc;        // [cap]  {cumulative quota, slot} of each replica entry
    int32_t *soff;   // [S+1]  dispatch only: exclusive prefix of the slot quotas
    uint8_t *tag;    // [W][E] dispatch only: per warp and expert, a lane of the current step holding it
    int32_t *stage;  // [stage_cap] the CTA's ids, read once from HBM in pass 1 (when they fit)
    float *gstage;   // [stage_cap] dispatch with gates: the CTA's gates, read in pass 1 likewise
    uint16_t *oli;   // [stage_cap] dispatch: local indices of the CTA's assignments in (expert, j) order
};

// Words of code[]: per (warp, replicated expert) for the plain variant; the
// dispatch variant keeps only the warps' partial sums there.
__host__ __device__ inline int code_words(int E, int S_disp)
{
    return S_disp > 0 ? 32 : kRerouteWarps * E + 2 * kRerouteWarps * kRepCache;
}

// Shared-memory words; S_disp = S for the dispatch variant, else 0; the
// gates are staged beside the ids (gstage_cap = stage_cap) when carried.
__host__ __device__ inline size_t reroute_smem_words(int E, int cap, int S_disp, int stage_cap, int gstage_cap)
{
    const size_t dwords = S_disp > 0 ? (size_t)S_disp + 1 + ((size_t)kRerouteWarps * E + 3) / 4 : 0;
    const size_t oli_words = S_disp > 0 ? ((size_t)stage_cap + 1) / 2 : 0;
    return (size_t)kRerouteWarps * E + code_words(E, S_disp) + 3 * (size_t)E + 1 + 2 * (size_t)E + 2 * (size_t)cap +
           dwords + 8 + (size_t)stage_cap + (size_t)gstage_cap + oli_words;
}

// Word offsets are computed as integers from the (16-byte aligned) base of the
// dynamic shared memory, so every pointer stays visibly derived from it and
// compiles to shared-memory instructions.
__device__ __forceinline__ RerouteSmem carve(int32_t *base, int E, int cap, int S_disp, int stage_cap,
                                             int gstage_cap)
{
    RerouteSmem s;
    int o = 0;
    s.hist = base + o;   o += kRerouteWarps * E;
    s.code = base + o;   o += code_words(E, S_disp);
    s.cc = reinterpret_cast<int2 *>(s.code + kRerouteWarps * E);   // plain variant (8-byte aligned)
    s.tot = base + o;    o += E;
    s.base = base + o;   o += E;
    s.rexp = base + o;   o += E + 1;
    o = (o + 1) & ~1;                       // 8-byte alignment for the int2 tables
    s.tab = reinterpret_cast<int2 *>(base + o);
    o += 2 * E;
    s.rc = reinterpret_cast<int2 *>(base + o);
    o += 2 * cap;
    s.soff = base + o;   o += S_disp > 0 ? S_disp + 1 : 0;
    s.tag = reinterpret_cast<uint8_t *>(base + o);
    o += S_disp > 0 ? (kRerouteWarps * E + 3) / 4 : 0;
    o = (o + 3) & ~3;                       // 16-byte alignment for the staged ids and gates
    s.stage = base + o;  o += (stage_cap + 3) & ~3;
    s.gstage = reinterpret_cast<float *>(base + o);
    o += (gstage_cap + 3) & ~3;
    s.oli = reinterpret_cast<uint16_t *>(base + o);
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

// Largest k in [0, n) with rc[k].x <= j (rc[0].x = 0 <= j): the replica entry
// whose cumulative-quota range holds occurrence j.  A replica with quota 0 has
// an empty range and is skipped, since the next entry has the same cum.
__device__ __forceinline__ int covering_entry(const int2 *rc, int n, int j)
{
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (rc[mid].x <= j) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Exclusive prefix of get(0..n-1) into out[0..n] (out[n] = the total), each
// thread a contiguous run; tmp holds 32 words.  Every thread of the block
// calls it; out may be written while get reads other memory.
template <class Get>
__device__ __forceinline__ void runs_excl_scan(Get get, int n, int32_t *out, int32_t *tmp)
{
    const int lane = lane_id(), warp = threadIdx.x >> 5;
    const int per = (n + (int)blockDim.x - 1) / (int)blockDim.x;
    const int a0 = min(n, (int)threadIdx.x * per), a1 = min(n, a0 + per);
    int sum = 0;
    for (int a = a0; a < a1; ++a) {
        const int q = get(a);
        out[a] = q;
        sum += q;
    }
    int x = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    __syncthreads();                       // tmp may still be read by a previous call
    if (lane == 31) tmp[warp] = x;
    __syncthreads();
    int run = x - sum;
    for (int w = 0; w < warp; ++w) run += tmp[w];
    for (int a = a0; a < a1; ++a) {
        const int q = out[a];
        out[a] = run;
        run += q;
    }
    if (a0 < n && a1 == n) out[n] = run;   // the thread owning the last entry
    if (n == 0 && threadIdx.x == 0) out[0] = 0;
    __syncthreads();
}

template <bool kDispatch>
__global__ void __launch_bounds__(kRerouteWarps * 32)
k_reroute(const int32_t *__restrict__ ids, int64_t per_rank, int E, int cap,
          const int32_t *__restrict__ rep_off, const int32_t *__restrict__ rep_slot,
          const int32_t *__restrict__ rep_cum, const int32_t *__restrict__ rank_off,
          int32_t *__restrict__ phys, int H, int HR, int stage_cap, DispatchArgs da)
{
    extern __shared__ __align__(16) int32_t sm_rr[];
    const RerouteSmem s = carve(sm_rr, E, cap, kDispatch ? da.S : 0, stage_cap,
                                (kDispatch && da.gates != nullptr) ? stage_cap : 0);

    cg::cluster_group cluster = cg::this_cluster();
    const int C = (int)cluster.num_blocks();
    const int c = (int)cluster.block_rank();
    const int r = blockIdx.x / C;
    const int lane = lane_id(), warp = threadIdx.x >> 5;

    for (int i = threadIdx.x; i < kRerouteWarps * E; i += blockDim.x) s.hist[i] = 0;
    if (!kDispatch && threadIdx.x == 0) s.rexp[E] = 0;   // count of the replicated-expert list
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
    const bool staged = hi - lo <= stage_cap;     // then pass 2 reads the ids from shared memory
    // Vector mode: 16-byte loads and stores, four ids per lane, when the CTA's
    // share and phys are 16-byte aligned (ids is); the ids come from shared
    // memory in pass 2 when the share was staged, else from memory again.
    const bool vec = (lo % 4) == 0 && ((hi - lo) % 4) == 0 && (reinterpret_cast<uintptr_t>(phys) & 15) == 0;

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
                if (staged && i < whi) *reinterpret_cast<int4 *>(s.stage + (i - lo)) = q[u];
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
    // Dispatch with gates: the warp's gates are staged beside its ids.
    const bool gstaged = kDispatch && da.gates != nullptr && staged;
    if (gstaged) {
        if ((lo % 4) == 0 && ((hi - lo) % 4) == 0 && (reinterpret_cast<uintptr_t>(da.gates) & 15) == 0) {
            for (int64_t v0 = wlo; v0 < whi; v0 += 128 * kUnroll) {
                float4 g[kUnroll];
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    const int64_t i = v0 + 128 * u + 4 * lane;
                    if (i < whi) g[u] = __ldg(reinterpret_cast<const float4 *>(da.gates + i));
                }
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    const int64_t i = v0 + 128 * u + 4 * lane;
                    if (i < whi) *reinterpret_cast<float4 *>(s.gstage + (i - lo)) = g[u];
                }
            }
        } else {
            for (int64_t x0 = wlo; x0 < whi; x0 += 32 * kUnroll) {
                float g[kUnroll];
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    const int64_t i = x0 + u * 32 + lane;
                    g[u] = i < whi ? __ldg(da.gates + i) : 0.0f;
                }
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    const int64_t i = x0 + u * 32 + lane;
                    if (i < whi) s.gstage[i - lo] = g[u];
                }
            }
        }
    }
    __syncthreads();
    // Exclusive scan over the warps per expert (in place) and CTA totals; the
    // 16 counts of an expert are loaded together before any is overwritten.
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int c[kRerouteWarps];
#pragma unroll
        for (int w = 0; w < kRerouteWarps; ++w) c[w] = s.hist[w * E + e];
        int run = 0;
#pragma unroll
        for (int w = 0; w < kRerouteWarps; ++w) {
            s.hist[w * E + e] = run;
            run += c[w];
        }
        s.tot[e] = run;
    }
    cluster.sync();

    // Still before the plan: the occurrences of e in the earlier CTAs of the
    // cluster (peers' totals over DSMEM) and, for the plain variant, each
    // warp's table row filled with the home slots (the plan never moves them).
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        int peer[kMaxCluster];
#pragma unroll
        for (int q = 0; q < kMaxCluster; ++q) peer[q] = q < c ? cluster.map_shared_rank(s.tot, q)[e] : 0;
        int b = 0;
#pragma unroll
        for (int q = 0; q < kMaxCluster; ++q) b += peer[q];
        s.base[e] = b;
    }
    if (!kDispatch) {
        int32_t *row = s.code + warp * E;
        for (int e = lane; e < E; e += 32) {
            const int hr = e / H;
            row[e] = hr * HR + (e - hr * H);
        }
    }
    cluster_arrive_relaxed();  // done reading peers; they may exit once all have arrived

    // The plan (and rank_off) of the preceding planner grid: every global load
    // of the plan is issued in one round.
    pdl_wait();
    for (int i = threadIdx.x; i < cap; i += blockDim.x) s.rc[i] = make_int2(__ldg(rep_cum + i), __ldg(rep_slot + i));
    for (int e = threadIdx.x; e < E; e += blockDim.x) {
        const int o0 = __ldg(rep_off + e), o1 = __ldg(rep_off + e + 1);
        const int b = __ldg(rank_off + (int64_t)r * E + e);
        const int off = clampi(o0, 0, cap - 1);
        const int n = clampi(o1 - off, 1, min(cap - off, 0xffff));
        int packed = n;
        if (!kDispatch && n > 1) {               // plain: list the replicated experts (any order)
            const int pos = atomicAdd(&s.rexp[E], 1);
            s.rexp[pos] = e;
            packed |= pos << 16;                  // the expert's position in the list
        }
        s.tab[e] = make_int2(off, packed);
        s.base[e] += b;           // occurrences of e before this CTA's ids
    }
    if constexpr (kDispatch) {
        // Slot offsets (exclusive prefix of the slot quotas; CTA 0 writes
        // them out) and, for the local grouping below, the exclusive prefix
        // of this CTA's per-expert counts (in rexp[], unused by this variant).
        runs_excl_scan([&](int a) { return __ldg(da.slot_quota + a); }, da.S, s.soff, s.code);
        runs_excl_scan([&](int e) { return s.tot[e]; }, E, s.rexp, s.code);
        const int S = da.S;
        if (blockIdx.x == 0)
            for (int a = threadIdx.x; a <= S; a += blockDim.x) da.slot_off[a] = s.soff[a];
        // Running occurrence index of each (warp, expert): base + earlier warps.
        for (int w = 0; w < kRerouteWarps; ++w)
            for (int e = threadIdx.x; e < E; e += blockDim.x) s.hist[w * E + e] += s.base[e];
        // An expert whose occurrences in this CTA, [base, base + tot), all fall
        // into one replica's range gets its slot and position offset directly:
        // tab[e] = {soff[slot] - rep_cum, -1 - slot}; it is taken only when that
        // whole range of positions lies inside the slot's segment and below
        // T*K, so no per-id check is needed.  Others keep {entry, count}.  The
        // local grouping index becomes rexp[e] + j (j the occurrence index).
        for (int e = threadIdx.x; e < E; e += blockDim.x) {
            const int b = s.base[e], nt = s.tot[e];
            const int2 t = s.tab[e];
            if (b >= 0 && nt > 0) {
                const int k = covering_entry(s.rc + t.x, t.y & 0xffff, b);
                const int2 q = s.rc[t.x + k];
                if (q.y >= 0 && q.y < S) {
                    const int lo = s.soff[q.y], hi = s.soff[q.y + 1];
                    if (lo >= 0 && hi >= lo && (int64_t)hi <= da.L && b >= q.x &&
                        (int64_t)b + nt <= (int64_t)q.x + (hi - lo))
                        s.tab[e] = make_int2(lo - q.x, -1 - q.y);
                }
            }
            s.rexp[e] -= b;
        }
        __syncthreads();

        // Pass 2: every valid id is ranked among the warp's equal ids (lane
        // order = token-major order) to get its occurrence index j; the
        // replica entry p covering j is the slot, and the assignment lands at
        // soff[slot] + j - rep_cum[p].  Equal ids of a step are found by a
        // per-warp tag table: each lane writes its lane number at its expert,
        // one lane per expert wins, and the winning lane number is a 5-bit key
        // that is equal exactly for equal ids.  With the ids staged, the
        // position replaces the id in stage[] and the CTA orders its
        // assignments by (expert, j) in oli[] (local indices), so that each
        // slot's run of this CTA is written out contiguously below; otherwise
        // every assignment is stored where it lands.
        uint8_t *tag = s.tag + warp * E;
        int32_t *wh = s.hist + warp * E;
        const unsigned lt = lanemask_lt();
        const int nloc = (int)(whi - wlo);       // this warp's ids, local index lbase + k
        const int lbase = (int)(wlo - lo);
        for (int k00 = 0; k00 < nloc; k00 += 32 * kUnroll) {
            int idv[kUnroll];                // the ids of four steps in flight together
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int k = k00 + 32 * u + lane;
                idv[u] = k < nloc ? (staged ? s.stage[lbase + k] : __ldg(ids + lo + lbase + k)) : -1;
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int k0 = k00 + 32 * u;
                if (k0 >= nloc) break;
                const int k = k0 + lane;
                const int li = lbase + k;
                const int id = idv[u];
                const bool valid = (unsigned)id < (unsigned)E;
                if (valid) tag[id] = (uint8_t)lane;
                __syncwarp();
                const int key = valid ? tag[id] : 0;
                unsigned m = __ballot_sync(0xffffffffu, valid);
#pragma unroll
                for (int b = 0; b < 5; ++b) {
                    const unsigned v = __ballot_sync(0xffffffffu, (key >> b) & 1);
                    m &= ((key >> b) & 1) ? v : ~v;
                }
                const int before = __popc(m & lt);
                int out = -1;
                if (valid) {
                    const int j = wh[id] + before;
                    const int2 t = s.tab[id];
                    int pos = -1;
                    if (t.y < 0) {                       // one replica for all of this CTA's ids
                        out = -1 - t.y;
                        pos = j + t.x;
                    } else {
                        const int2 q = s.rc[t.x + covering_entry(s.rc + t.x, t.y & 0xffff, j)];
                        out = q.y;
                        // Inside the slot's segment whenever the ids are the ones the
                        // plan was computed from; anything else is reported, not written.
                        if (out >= 0 && out < S) {
                            pos = s.soff[out] + (j - q.x);
                            if (pos < s.soff[out] || pos >= s.soff[out + 1] || (int64_t)pos >= da.L) pos = -1;
                        }
                        if (pos < 0) atomicOr(da.err, 2);
                    }
                    if (staged) {
                        s.stage[li] = pos;
                        s.oli[s.rexp[id] + j] = (uint16_t)li;
                    } else if (pos >= 0) {
                        da.src_index[pos] = (int32_t)(lo + li);
                        if (da.gates != nullptr) da.gates_out[pos] = __ldg(da.gates + lo + li);
                    }
                }
                __syncwarp();
                if (valid && before == 0) wh[id] += __popc(m);
                __syncwarp();
                if (k < nloc) phys[lo + li] = out;
            }
        }
        if (staged) {
            // Write-out in (expert, j) order: consecutive threads take
            // consecutive positions of one slot's run.
            __syncthreads();
            const int nvalid = s.rexp[E];
            for (int lp = threadIdx.x; lp < nvalid; lp += blockDim.x) {
                const int li = s.oli[lp];
                const int pos = s.stage[li];
                if (pos < 0) continue;
                da.src_index[pos] = (int32_t)(lo + li);
                if (gstaged) da.gates_out[pos] = s.gstage[li];
                else if (da.gates != nullptr) da.gates_out[pos] = __ldg(da.gates + lo + li);
            }
        }
    } else {
        __syncthreads();
        // Per-warp direct table code[w][e] (each warp its own row): the slot of
        // every id of e in warp w's part when they all fall into one replica
        // (an expert with one replica always does: its home slot, filled in
        // before the plan), else -2 - j with j the occurrence index of the
        // warp's next occurrence of e (updated as the warp goes).  Only the
        // replicated experts' entries are computed here.
        int32_t *tb = s.code + warp * E;
        const int nrep = s.rexp[E];
        for (int i = lane; i < nrep; i += 32) {
            const int e = s.rexp[i];
            const int2 t = s.tab[e];
            const int n = t.y & 0xffff;
            const int excl = s.hist[warp * E + e];
            const int cnt = (warp + 1 < kRerouteWarps ? s.hist[(warp + 1) * E + e] : s.tot[e]) - excl;
            const int j0 = s.base[e] + excl;
            const int k = covering_entry(s.rc + t.x, n, j0);
            const bool uniform = k == n - 1 || j0 + cnt <= s.rc[t.x + k + 1].x;
            tb[e] = uniform ? s.rc[t.x + k].y : -2 - j0;
            if (!uniform && i < kRepCache)
                s.cc[warp * kRepCache + i] = make_int2(s.rc[t.x + k].y, s.rc[t.x + k + 1].x);
        }
        const int nbe = E > 1 ? 32 - __clz(E - 1) : 0;   // bits of an expert id
        __syncwarp();

        // Table entry of one id: its slot (>= 0), -1 for a bad id, or -2 - j
        // (<= -2) when the id must be ranked to find its replica.
        auto lookup = [&](int id) { return (unsigned)id < (unsigned)E ? tb[id] : -1; };
        // One scalar step of 32 consecutive ids (lane order = token-major order).
        auto step = [&](int id, int64_t i) {
            const int c = lookup(id);
            int out = c;
            if (__any_sync(0xffffffffu, c <= -2)) {
                const unsigned m = match_key(c <= -2 ? id : -1, nbe);
                const int before = __popc(m & lanemask_lt());
                if (c <= -2) {
                    const int j = -2 - c + before;
                    const int2 t = s.tab[id];
                    out = s.rc[t.x + covering_entry(s.rc + t.x, t.y & 0xffff, j)].y;
                }
                __syncwarp();
                if (c <= -2 && before == 0) tb[id] = c - __popc(m);
                __syncwarp();
            }
            if (i < whi) phys[i] = out;
        };

        // Pass 2: replica of every (t, k).
        if (vec) {
            // Blocks of 128 ids, four per lane: when no id of the block needs
            // ranking, one 16-byte store per lane; otherwise the marked ids are
            // ranked expert by expert with a warp scan of the lanes' counts
            // (no search when an expert's occurrences here stay in one
            // replica), then stored the same way.
            for (int64_t v00 = wlo; v00 < whi; v00 += 128 * kUnroll) {
                int4 qs[kUnroll];            // every block's ids in flight together
#pragma unroll
                for (int u = 0; u < kUnroll; ++u) {
                    const int64_t i = v00 + 128 * u + 4 * lane;
                    qs[u] = i >= whi ? make_int4(-1, -1, -1, -1)
                            : staged ? *reinterpret_cast<const int4 *>(s.stage + (i - lo))
                                     : __ldg(reinterpret_cast<const int4 *>(ids + i));
                }
#pragma unroll
                for (int ub = 0; ub < kUnroll; ++ub) {
                    const int64_t v0 = v00 + 128 * ub;
                    if (v0 >= whi) break;
                    const int64_t i = v0 + 4 * lane;
                    const int4 q = qs[ub];
                    const int o0 = lookup(q.x), o1 = lookup(q.y), o2 = lookup(q.z), o3 = lookup(q.w);
                    const bool r0 = o0 <= -2, r1 = o1 <= -2, r2 = o2 <= -2, r3 = o3 <= -2;
                    if (!__any_sync(0xffffffffu, r0 || r1 || r2 || r3)) {
                        if (i < whi) *reinterpret_cast<int4 *>(phys + i) = make_int4(o0, o1, o2, o3);
                        continue;
                    }
                    // Rank the marked ids expert by expert (the smallest expert
                    // id first): an expert's occurrences in the block, in
                    // token-major order, are lane by lane and x, y, z, w within
                    // a lane, so an exclusive scan of the lanes' counts gives
                    // each its occurrence index.
                    int p0 = o0, p1 = o1, p2 = o2, p3 = o3;
                    bool m0 = r0, m1 = r1, m2 = r2, m3 = r3;   // still to rank
                    while (__any_sync(0xffffffffu, m0 || m1 || m2 || m3)) {
                        int emn = INT_MAX;
                        if (m0) emn = min(emn, q.x);
                        if (m1) emn = min(emn, q.y);
                        if (m2) emn = min(emn, q.z);
                        if (m3) emn = min(emn, q.w);
                        const int ex = __reduce_min_sync(0xffffffffu, emn);
                        const bool h0 = m0 && q.x == ex, h1 = m1 && q.y == ex;
                        const bool h2 = m2 && q.z == ex, h3 = m3 && q.w == ex;
                        const int cnt = __popc(__ballot_sync(0xffffffffu, h0)) + __popc(__ballot_sync(0xffffffffu, h1)) +
                                        __popc(__ballot_sync(0xffffffffu, h2)) + __popc(__ballot_sync(0xffffffffu, h3));
                        const int2 te = s.tab[ex];
                        const int n = te.y & 0xffff, ci = te.y >> 16;
                        const int vv = -2 - tb[ex];          // the warp's next occurrence index of ex
                        const int2 cur = ci < kRepCache ? s.cc[warp * kRepCache + ci] : make_int2(-1, 0);
                        if (cur.x >= 0 && vv + cnt < cur.y) {
                            // All of them, and the next occurrence, in the cached replica.
                            p0 = h0 ? cur.x : p0;
                            p1 = h1 ? cur.x : p1;
                            p2 = h2 ? cur.x : p2;
                            p3 = h3 ? cur.x : p3;
                        } else {
                            const int mine = h0 + h1 + h2 + h3;
                            int incl = mine;
#pragma unroll
                            for (int o = 1; o < 32; o <<= 1) {
                                const int y = __shfl_up_sync(0xffffffffu, incl, o);
                                if (lane >= o) incl += y;
                            }
                            const int k1 = covering_entry(s.rc + te.x, n, vv);
                            const int k2 = covering_entry(s.rc + te.x, n, vv + cnt - 1);
                            if (k1 == k2) {                  // one replica for all of them
                                const int sl = s.rc[te.x + k1].y;
                                p0 = h0 ? sl : p0;
                                p1 = h1 ? sl : p1;
                                p2 = h2 ? sl : p2;
                                p3 = h3 ? sl : p3;
                            } else {
                                int j = vv + incl - mine;
                                if (h0) p0 = s.rc[te.x + covering_entry(s.rc + te.x, n, j++)].y;
                                if (h1) p1 = s.rc[te.x + covering_entry(s.rc + te.x, n, j++)].y;
                                if (h2) p2 = s.rc[te.x + covering_entry(s.rc + te.x, n, j++)].y;
                                if (h3) p3 = s.rc[te.x + covering_entry(s.rc + te.x, n, j++)].y;
                            }
                            if (lane == 0 && ci < kRepCache) {   // the replica of the next occurrence
                                const int k3 = covering_entry(s.rc + te.x, n, vv + cnt);
                                s.cc[warp * kRepCache + ci] =
                                    make_int2(s.rc[te.x + k3].y, k3 + 1 < n ? s.rc[te.x + k3 + 1].x : INT_MAX);
                            }
                        }
                        __syncwarp();
                        if (lane == 0) tb[ex] = -2 - (vv + cnt);
                        __syncwarp();
                        m0 = m0 && !h0;
                        m1 = m1 && !h1;
                        m2 = m2 && !h2;
                        m3 = m3 && !h3;
                    }
                    if (i < whi) *reinterpret_cast<int4 *>(phys + i) = make_int4(p0, p1, p2, p3);
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
    }
    cluster_wait();            // keep this CTA's shared memory alive for its peers
}

}  // namespace

size_t reroute_smem_bytes(const Shape &sh, bool dispatch, int stage_cap, bool gates)
{
    const int cap = sh.E + sh.NR;
    return reroute_smem_words(sh.E, cap, dispatch ? sh.S : 0, stage_cap, dispatch && gates ? stage_cap : 0) *
           sizeof(int32_t);
}

namespace {
// The ids of a CTA are kept in shared memory between the passes when the
// staging buffer fits beside the tables.
int stage_cap_for(const Shape &sh, const Launch &ln, bool dispatch, bool gates)
{
    return reroute_smem_bytes(sh, dispatch, kStageIds, gates) <= ln.max_smem ? kStageIds : 0;
}
}  // namespace

cudaError_t launch_reroute(const Shape &sh, const Launch &ln, const int32_t *ids, const PlanDev &plan,
                           int32_t *phys, cudaStream_t st, bool pdl)
{
    const int stage = stage_cap_for(sh, ln, false, false);
    return launch_ex(k_reroute<false>, (unsigned)(sh.N * ln.cluster), kRerouteWarps * 32,
                     reroute_smem_bytes(sh, false, stage, false), st, (unsigned)ln.cluster, pdl, ids, sh.per_rank, sh.E,
                     sh.E + sh.NR, plan.rep_off, plan.rep_slot, plan.rep_cum, plan.rank_off, phys, sh.H, sh.HR, stage,
                     DispatchArgs{});
}

cudaError_t launch_dispatch(const Shape &sh, const Launch &ln, const int32_t *ids, const PlanDev &plan,
                            int32_t *phys, const DispatchOut &out, int32_t *dev_err, cudaStream_t st, bool pdl)
{
    const bool gates = out.gates != nullptr;
    const int stage = stage_cap_for(sh, ln, true, gates);
    const DispatchArgs da{out.gates, plan.slot_quota, out.slot_off, out.src_index, out.gates_out, dev_err,
                          sh.N * sh.per_rank, sh.S};
    return launch_ex(k_reroute<true>, (unsigned)(sh.N * ln.cluster), kRerouteWarps * 32,
                     reroute_smem_bytes(sh, true, stage, gates), st, (unsigned)ln.cluster, pdl, ids, sh.per_rank, sh.E,
                     sh.E + sh.NR, plan.rep_off, plan.rep_slot, plan.rep_cum, plan.rank_off, phys, sh.H, sh.HR, stage, da);
}

cudaError_t set_reroute_attributes(size_t max_smem)
{
    // The largest shared-memory split, so that two CTAs per SM fit and the grid
    // runs in one wave beside the planner (the default split may leave room for one).
    for (auto k : {k_reroute<false>, k_reroute<true>}) {
        cudaError_t e = allow_smem(k, max_smem);
        if (e == cudaSuccess) e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

}  // namespace ue
