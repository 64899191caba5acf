// Step 3 - routing expansion for large microbatches: a persistent kernel over
// pieces of each rank's ids.
//
// "Routing expansion" (csrc/kernels/reroute.cu; "Routing expansion -> Token
// dispatch: physical routing" in "How dots-infra/ultraep works").  The j-th
// occurrence (0-based, token-major order) of expert e goes to the replica of e
// whose cumulative-quota range [rep_cum[i], rep_cum[i] + q_i) holds j.
//
// When a rank's ids do not fit the rank-per-cluster kernel in one wave with
// its ids kept on chip (many ranks, or many tokens per rank), each rank's ids
// are cut into B pieces of zp ids and the load kernel writes, per rank, the
// occurrences of every expert before each piece, rows[(r*(B+1) + b)][e], and
// the rank's totals in row B.  For piece (r, b) the occurrence index of its
// first occurrence of e is then
//     base[e] = rank_off[r][e] + rows(r, b)[e],
// and the piece holds rows(r, b+1)[e] - rows(r, b)[e] occurrences of e.  An expert whose
// occurrences in the piece, [base, base + count), all fall into one replica's
// range - every expert with a single replica, and all but a handful of the
// replicated ones - is routed by one shared-memory table lookup per id: the
// piece needs no ranking and no histogram pass, so every id is read from
// memory once and written once.  Only the "boundary" experts of a piece (a
// quota boundary inside it) are ranked: per 8192-id sub-chunk, each warp
// counts their ids, a scan over the warps gives each warp's starting
// occurrence index, and inside a warp the ids are ranked by ballots in
// token-major order (lane order, then the four ids of a lane).
//
// Pieces are claimed by the CTAs of a resident grid from a counter, so the
// CTAs finish together whatever a piece costs; the next piece's ids and rows
// are copied into shared memory while the current one streams.
#include <climits>

#include "ue_internal.cuh"

namespace ue {
namespace {

constexpr int kRpWarps = 16;
constexpr int kRpThreads = kRpWarps * 32;
constexpr int kRpPerLane = 16;                        // ids per lane per sub-chunk
constexpr int kRpSub = kRpThreads * kRpPerLane;       // 8192 ids per sub-chunk
constexpr int kRpNB = 64;                             // boundary experts ranked per round

// Largest k in [0, n) with rc[k].x <= j (rc[0].x <= j): the replica entry
// whose cumulative-quota range holds occurrence j.
__device__ __forceinline__ int covering(const int2 *rc, int n, int j)
{
    int lo = 0, hi = n - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (rc[mid].x <= j) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

struct PieceSmem {
    int2 *rc;        // [cap]  {cumulative quota, slot} of each replica entry
    int2 *tab;       // [E]    {first replica entry, replicas}
    int32_t *pslot;  // [E]    piece table: slot, or -2 - (boundary index)
    int32_t *bexp;   // [E]    boundary experts of the piece
    int32_t *bj;     // [E]    their running occurrence index
    int32_t *wcnt;   // [kRpWarps][kRpNB] per-warp counts, then per-warp starting index
    int32_t *wslot;  // [kRpWarps][kRpNB] per warp: the boundary expert's slot when its ids stay in one replica
    int32_t *misc;   // [8]    boundary counts (2), this CTA's first piece, its next piece (2)
    int32_t *f;      // [3][E] rank_off row, rows (r, b) and (r, b + 1) of the next piece
    int32_t *stage;  // [2][kRpSub] ids of the current and the next sub-chunk (thread-private slots)
};

__host__ __device__ inline size_t piece_smem_words(int E, int cap)
{
    const size_t tables = 2 * (size_t)cap + 8 * (size_t)E + 2 * (size_t)kRpWarps * kRpNB + 8;
    return (tables + 3) / 4 * 4 + 2 * (size_t)kRpSub;
}

// The expert ids a lane holds for one block: V consecutive ids (V = 4: one
// 16-byte load; V = 1: scalar).  Positions past the piece hold kNone.
constexpr int kNone = INT_MIN;

template <int V>
struct Ids {
    int v[V];
};

template <int V>
__device__ __forceinline__ Ids<V> load_ids(const int32_t *__restrict__ ids, int x, int end)
{
    Ids<V> q;
    if constexpr (V == 4) {
        if (x < end) {
            const int4 a = __ldcs(reinterpret_cast<const int4 *>(ids + x));
            q.v[0] = a.x; q.v[1] = a.y; q.v[2] = a.z; q.v[3] = a.w;
        } else {
            q.v[0] = q.v[1] = q.v[2] = q.v[3] = kNone;
        }
    } else {
        q.v[0] = x < end ? __ldcs(ids + x) : kNone;
    }
    return q;
}

template <int V>
__device__ __forceinline__ void store_out(int32_t *__restrict__ phys, int x, int end, const int (&o)[V])
{
    if (x >= end) return;
    if constexpr (V == 4) __stcs(reinterpret_cast<int4 *>(phys + x), make_int4(o[0], o[1], o[2], o[3]));
    else __stcs(phys + x, o[0]);
}

// Asynchronous copies global -> shared (cp.async, completion per thread).
template <int V>
__device__ __forceinline__ void cp_async(int32_t *dst, const int32_t *src)
{
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
    if constexpr (V == 4) asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
    else asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(d), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// V ids per lane and block; a warp's part of a sub-chunk is kRpPerLane / V
// blocks of 32 * V consecutive ids (block, then lane, then the lane's V ids is
// token-major order).
template <int V>
__global__ void __launch_bounds__(kRpThreads, 2)
k_reroute_pieces(const int32_t *__restrict__ ids, int per_rank, int E, int cap, int B, int zp, int NP,
                 const int32_t *__restrict__ rep_off, const int32_t *__restrict__ rep_slot,
                 const int32_t *__restrict__ rep_cum, const int32_t *__restrict__ rank_off,
                 const int32_t *__restrict__ rows, int32_t *__restrict__ phys, int32_t *__restrict__ ctr)
{
    constexpr int kBlocks = kRpPerLane / V;           // blocks per warp and sub-chunk
    extern __shared__ __align__(16) int32_t sm_rp[];
    PieceSmem s;
    {
        int o = 0;
        s.rc = reinterpret_cast<int2 *>(sm_rp + o);  o += 2 * cap;
        s.tab = reinterpret_cast<int2 *>(sm_rp + o); o += 2 * E;
        s.pslot = sm_rp + o;                          o += E;
        s.bexp = sm_rp + o;                           o += E;
        s.bj = sm_rp + o;                             o += E;
        s.wcnt = sm_rp + o;                           o += kRpWarps * kRpNB;
        s.wslot = sm_rp + o;                          o += kRpWarps * kRpNB;
        s.misc = sm_rp + o;                           o += 8;
        s.f = sm_rp + o;                              o += 3 * E;
        s.stage = sm_rp + (o + 3) / 4 * 4;            // 16-byte aligned
    }
    const int lane = lane_id(), warp = threadIdx.x >> 5;
    const int stride_row = E + 1;

    // The rows a piece's table needs - rank_off[r][e], rows(r, b)[e] and
    // rows(r, b + 1)[e] - copied asynchronously into f[3][E] (each thread its
    // experts), so that they arrive while the previous piece streams.
    // Claim p routes piece b = B - 1 - p / Nr of rank r = p % Nr: the load pass
    // walks every rank's pieces first to last, so the pieces it read last (the
    // ones still in L2) are routed first.
    const int Nr = NP / B;
    auto piece_of = [&](int p, int &r, int &b) {
        const int q = p / Nr;
        r = p - q * Nr;
        b = B - 1 - q;
    };
    auto fetch_issue = [&](int p) {
        int r, b;
        piece_of(p, r, b);
        const int32_t *row = rows + ((size_t)r * (B + 1) + b) * stride_row;
        for (int e = threadIdx.x; e < E; e += kRpThreads) {
            cp_async<1>(s.f + e, rank_off + (size_t)r * E + e);
            cp_async<1>(s.f + E + e, row + e);
            cp_async<1>(s.f + 2 * E + e, row + stride_row + e);
        }
    };

    // This thread's 16 ids of a sub-chunk in its own slots of stage[buf]
    // (cp.async: no registers held, no barrier, since each thread reads back
    // only what it copied).
    auto stage_at = [&](int buf, int u) { return s.stage + buf * kRpSub + (u * kRpThreads + threadIdx.x) * V; };
    auto sub_issue = [&](int s0, int end, int buf) {
        const int wlo = s0 + (int)warp * (kRpSub / kRpWarps);
#pragma unroll
        for (int u = 0; u < kBlocks; ++u) {
            const int x = wlo + u * 32 * V + V * lane;
            if (x < end) cp_async<V>(stage_at(buf, u), ids + x);
        }
        cp_async_commit();
    };
    auto sub_read = [&](int s0, int end, int buf, Ids<V> (&q)[kBlocks]) {
        const int wlo = s0 + (int)warp * (kRpSub / kRpWarps);
#pragma unroll
        for (int u = 0; u < kBlocks; ++u) {
            const int x = wlo + u * 32 * V + V * lane;
            if constexpr (V == 4) {
                if (x < end) {
                    const int4 a = *reinterpret_cast<const int4 *>(stage_at(buf, u));
                    q[u].v[0] = a.x; q[u].v[1] = a.y; q[u].v[2] = a.z; q[u].v[3] = a.w;
                } else {
                    q[u].v[0] = q[u].v[1] = q[u].v[2] = q[u].v[3] = kNone;
                }
            } else {
                q[u].v[0] = x < end ? *stage_at(buf, u) : kNone;
            }
        }
    };
    auto piece_range = [&](int p, int &lo, int &hi) {
        int r, b;
        piece_of(p, r, b);
        lo = (int)r * per_rank + (int)b * zp;
        hi = min(lo + zp, (int)(r + 1) * per_rank);
    };

    // Pieces are claimed from the counter ctr[0], each CTA one piece ahead
    // (ctr[1] counts finished CTAs; the last one resets both for the next
    // launch, so they start at 0 without a memset).  The first sub-chunk's ids
    // load while the planner finishes.
    if (threadIdx.x == 0) s.misc[2] = atomicAdd(ctr, 1);
    __syncthreads();
    int p = s.misc[2];
    int buf = 0;
    if (p < NP) {
        int lo, hi;
        piece_range(p, lo, hi);
        sub_issue(lo, hi, 0);
    }

    // The plan tables (the same for every piece), after the planner's grid.
    pdl_wait();
    for (int i = threadIdx.x; i < cap; i += kRpThreads) s.rc[i] = make_int2(__ldg(rep_cum + i), __ldg(rep_slot + i));
    for (int e = threadIdx.x; e < E; e += kRpThreads) {
        const int o0 = __ldg(rep_off + e), o1 = __ldg(rep_off + e + 1);
        const int off = clampi(o0, 0, cap - 1);
        s.tab[e] = make_int2(off, clampi(o1 - off, 1, cap - off));
    }
    if (p < NP) fetch_issue(p);
    cp_async_commit();
    if (threadIdx.x == 0) s.misc[0] = s.misc[1] = 0;

    auto lookup = [&](int id) { return (unsigned)id < (unsigned)E ? s.pslot[id] : -1; };

    // Route one sub-chunk whose ids this thread holds in q.  Boundary experts
    // r0 .. r0+nact-1 are ranked (nact = 0: none); round0 writes every id,
    // a later round only its boundary experts' ids.
    auto route = [&](const Ids<V> (&q)[kBlocks], int s0, int end, int r0, int nact, bool round0) {
        const int wlo = s0 + (int)warp * (kRpSub / kRpWarps);
        if (nact <= 0) {
            // No boundary expert in this piece: table lookups only.
#pragma unroll
            for (int u = 0; u < kBlocks; ++u) {
                int o[V];
#pragma unroll
                for (int k = 0; k < V; ++k) o[k] = lookup(q[u].v[k]);
                store_out<V>(phys, wlo + u * 32 * V + V * lane, end, o);
            }
            return;
        }
        // Count this warp's ids of the active boundary experts.
        for (int i = threadIdx.x; i < kRpWarps * kRpNB; i += kRpThreads) s.wcnt[i] = 0;
        __syncthreads();
#pragma unroll
        for (int u = 0; u < kBlocks; ++u)
#pragma unroll
            for (int k = 0; k < V; ++k) {
                const int c = lookup(q[u].v[k]);
                const int a = -2 - c - r0;
                if (c <= -2 && a >= 0 && a < nact) smem_add(s.wcnt + warp * kRpNB + a, 1);
            }
        __syncthreads();
        if (threadIdx.x < nact) {        // each warp's starting occurrence index
            int run = s.bj[r0 + threadIdx.x];
#pragma unroll
            for (int w = 0; w < kRpWarps; ++w) {
                const int c = s.wcnt[w * kRpNB + threadIdx.x];
                s.wcnt[w * kRpNB + threadIdx.x] = run;
                run += c;
            }
            s.bj[r0 + threadIdx.x] = run;
        }
        __syncthreads();
        // A warp whose occurrences of a boundary expert stay in one replica
        // takes its slot; only the warp holding a quota boundary ranks.
        int32_t *wj = s.wcnt + warp * kRpNB;
        int32_t *ws = s.wslot + warp * kRpNB;
        for (int i = lane; i < nact; i += 32) {
            const int j0 = wj[i];
            const int c = (warp + 1 < kRpWarps ? s.wcnt[(warp + 1) * kRpNB + i] : s.bj[r0 + i]) - j0;
            const int2 t = s.tab[s.bexp[r0 + i]];
            const int k = covering(s.rc + t.x, t.y, j0);
            const bool one = c <= 0 || k == t.y - 1 || (int)j0 + c <= (int)s.rc[t.x + k + 1].x;
            ws[i] = one ? s.rc[t.x + k].y : -1;
        }
        __syncwarp();
#pragma unroll
        for (int u = 0; u < kBlocks; ++u) {
            const int x = wlo + u * 32 * V + V * lane;
            int o[V], a[V];
            bool m[V];
            bool any = false;
#pragma unroll
            for (int k = 0; k < V; ++k) {
                o[k] = lookup(q[u].v[k]);
                a[k] = -2 - o[k] - r0;
                const bool act = o[k] <= -2 && a[k] >= 0 && a[k] < nact;
                const int v = act ? ws[a[k]] : -1;
                if (v >= 0) o[k] = v;
                m[k] = act && v < 0;
                any |= m[k];
            }
            // Rank the remaining ids boundary expert by boundary expert: lanes
            // in order, a lane's ids in order.
            while (__any_sync(0xffffffffu, any)) {
                int amin = INT_MAX;
#pragma unroll
                for (int k = 0; k < V; ++k)
                    if (m[k]) amin = min(amin, a[k]);
                const int ax = __reduce_min_sync(0xffffffffu, amin);
                int mine = 0;
#pragma unroll
                for (int k = 0; k < V; ++k) mine += (m[k] && a[k] == ax) ? 1 : 0;
                int incl = mine;
#pragma unroll
                for (int d = 1; d < 32; d <<= 1) {
                    const int y = __shfl_up_sync(0xffffffffu, incl, d);
                    if (lane >= d) incl += y;
                }
                const int total = __shfl_sync(0xffffffffu, incl, 31);
                const int2 t = s.tab[s.bexp[r0 + ax]];
                int j = wj[ax] + incl - mine;
#pragma unroll
                for (int k = 0; k < V; ++k)
                    if (m[k] && a[k] == ax) {
                        o[k] = s.rc[t.x + covering(s.rc + t.x, t.y, j)].y;
                        ++j;
                        m[k] = false;
                    }
                __syncwarp();
                if (lane == 0) wj[ax] += total;
                __syncwarp();
                any = false;
#pragma unroll
                for (int k = 0; k < V; ++k) any |= m[k];
            }
            if (round0) {
                // Boundary experts of later rounds are written then.
#pragma unroll
                for (int k = 0; k < V; ++k)
                    if (o[k] <= -2) o[k] = -1;
                store_out<V>(phys, x, end, o);
            } else {
#pragma unroll
                for (int k = 0; k < V; ++k)     // only this round's boundary ids
                    if (x + k < end && a[k] >= 0 && a[k] < nact) phys[x + k] = o[k];
            }
        }
        __syncthreads();                  // wcnt and wslot are rewritten for the next sub-chunk
    };

    for (int it = 0; p < NP; ++it) {
        int plo, phi;
        piece_range(p, plo, phi);
        // Boundary counters alternate between pieces: the one of the previous
        // piece is cleared only after every thread has read it.
        int32_t *nbp = s.misc + (it & 1);

        // Piece table: the slot of every expert whose occurrences here stay in
        // one replica, else a boundary index (its running index in bj[]).
        // Every copy issued so far has landed (the piece's rows in f[] and
        // its first staged sub-chunk).
        cp_async_wait<0>();
        __syncthreads();               // f[] of all threads; tab/rc; the previous piece is done with pslot, bexp, bj
        if (threadIdx.x == 0) {
            s.misc[(it + 1) & 1] = 0;
            s.misc[3 + (it & 1)] = atomicAdd(ctr, 1);     // the next piece, read after the next barrier
        }
        for (int e = threadIdx.x; e < E; e += kRpThreads) {
            const int2 t = s.tab[e];
            const int j0 = s.f[e] + s.f[E + e], c = s.f[2 * E + e] - s.f[E + e];
            int out;
            if (t.y == 1) {
                out = s.rc[t.x].y;
            } else {
                const int k = covering(s.rc + t.x, t.y, j0);
                if (c <= 0 || k == t.y - 1 || (int)j0 + c <= (int)s.rc[t.x + k + 1].x) {
                    out = s.rc[t.x + k].y;
                } else {
                    const int idx = atomicAdd(nbp, 1);
                    s.bexp[idx] = e;
                    s.bj[idx] = j0;
                    out = -2 - idx;
                }
            }
            s.pslot[e] = out;
        }
        __syncthreads();               // pslot, bexp, bj written; f[] read
        const int nb = *nbp;
        const int pn = s.misc[3 + (it & 1)];

        // Round 0 from the staged ids, one sub-chunk ahead (the next piece's
        // first sub-chunk after this piece's last).
        for (int s0 = plo; s0 < phi; s0 += kRpSub) {
            if (s0 + kRpSub < phi) {
                sub_issue(s0 + kRpSub, phi, buf ^ 1);
                cp_async_wait<1>();
            } else if (pn < NP) {
                // The next piece's rows and first sub-chunk.
                int nlo, nhi;
                piece_range(pn, nlo, nhi);
                fetch_issue(pn);
                sub_issue(nlo, nhi, buf ^ 1);
                cp_async_wait<1>();
            } else {
                cp_async_wait<0>();
            }
            Ids<V> q[kBlocks];
            sub_read(s0, phi, buf, q);
            buf ^= 1;
            route(q, s0, phi, 0, min(kRpNB, nb), true);
        }
        // Boundary experts past the first kRpNB: further rounds, ids read again.
        for (int r0 = kRpNB; r0 < nb; r0 += kRpNB)
            for (int s0 = plo; s0 < phi; s0 += kRpSub) {
                const int wlo = s0 + (int)warp * (kRpSub / kRpWarps);
                Ids<V> q[kBlocks];
#pragma unroll
                for (int u = 0; u < kBlocks; ++u) q[u] = load_ids<V>(ids, wlo + u * 32 * V + V * lane, phi);
                route(q, s0, phi, r0, min(kRpNB, nb - r0), false);
            }
        p = pn;
    }
    cp_async_wait<0>();
    if (threadIdx.x == 0 && atomicAdd(ctr + 1, 1) == (int)gridDim.x - 1) {
        atomicExch(ctr, 0);
        atomicExch(ctr + 1, 0);
    }
}

}  // namespace

size_t reroute_pieces_smem_bytes(const Shape &sh)
{
    return piece_smem_words(sh.E, sh.E + sh.NR) * sizeof(int32_t);
}

cudaError_t launch_reroute_pieces(const Shape &sh, const Pieces &pc, const int32_t *ids, const PlanDev &plan,
                                  const int32_t *rows, int32_t *ctr, int32_t *phys, cudaStream_t st, bool pdl)
{
    const int cap = sh.E + sh.NR;
    const bool vec = sh.per_rank % 4 == 0 && (reinterpret_cast<uintptr_t>(phys) & 15) == 0;
    const unsigned grid = (unsigned)min(pc.NP, pc.grid);
    if (grid == 0) return cudaSuccess;
    const size_t smem = reroute_pieces_smem_bytes(sh);
    if (vec)
        return launch_ex(k_reroute_pieces<4>, grid, kRpThreads, smem, st, 1u, pdl, ids, (int)sh.per_rank, sh.E, cap,
                         pc.B, (int)pc.zp, pc.NP, plan.rep_off, plan.rep_slot, plan.rep_cum, plan.rank_off, rows, phys, ctr);
    return launch_ex(k_reroute_pieces<1>, grid, kRpThreads, smem, st, 1u, pdl, ids, (int)sh.per_rank, sh.E, cap,
                     pc.B, (int)pc.zp, pc.NP, plan.rep_off, plan.rep_slot, plan.rep_cum, plan.rank_off, rows, phys, ctr);
}

int reroute_pieces_blocks_per_sm(size_t smem)
{
    int a = 0, b = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&a, k_reroute_pieces<4>, kRpThreads, smem) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&b, k_reroute_pieces<1>, kRpThreads, smem) != cudaSuccess)
        return 1;
    const int n = a < b ? a : b;
    return n > 0 ? n : 1;
}

cudaError_t set_reroute_pieces_attributes(size_t max_smem)
{
    cudaError_t e = allow_smem(k_reroute_pieces<4>, max_smem);
    if (e == cudaSuccess) e = allow_smem(k_reroute_pieces<1>, max_smem);
    return e;
}

}  // namespace ue
