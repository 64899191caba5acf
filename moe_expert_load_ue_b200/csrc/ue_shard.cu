// Steps 4 and 5 across the GPUs of one NVLink domain.
//
// Replica weight sync and replica gradient reduction when the N ranks are
// spread over G GPUs: GPU g holds ranks [g*N/G, (g+1)*N/G), hence slots
// [g*SG, (g+1)*SG) (SG = S / G), the experts homed on those ranks and the
// replica-gradient rows of their redundant slots.  Transfers between GPUs use
// the relay mechanism against fan-out overload (UltraEP news summary,
// "Comment fonctionne l'équilibrage en 300 microsecondes"), read as a scatter
// then an all-gather: an expert's consumers c_0 < c_1 < ... < c_{f-1} are the
// GPUs other than its home GPU holding a filled redundant slot of it; its
// bytes are cut into f parts of q = 16 * ceil(slot_bytes / (16 f)) bytes;
//   round 0: c_j pulls part j from the home slot (and the home GPU fills its
//            own redundant slots of the expert);
//   round 1: c_i pulls every other part j from c_j's lowest slot of it.
// So the home sends each byte once, not once per consumer: with every peer at
// full bandwidth through NVSwitch, the busiest GPU's traffic, not the number
// of hops, sets the time.  Round -1 is the direct form (every consumer pulls
// the whole slot from the home slot).
//
// Design (sm_100a).  Sync: the single-GPU sync kernel's persistent ring of
// TMA bulk copies, run on each GPU over the byte ranges it receives in the
// round.  The CTAs flatten (expert, part, 48 KiB tile) into one item list (a
// prefix over the experts, a binary search per item); the global->shared bulk
// load reads the source GPU's slot through the caller's peer mapping (no
// tensor map, no multicast), and the shared->global bulk stores write the
// range into every local slot of the expert, so a byte crosses NVLink once
// per receiving GPU however many of its ranks hold the expert.
// Gradient reduction: the home GPU of each replicated expert pulls every
// replica's gradient row from the GPU holding it, in replica order, with the
// single-GPU kernel's fp32 adds, so its result is bit-identical to it.
// Peer pointers are plain arguments; on one GPU the G "GPUs" may be parts of
// one allocation.  No kernel here waits on another GPU: the caller orders the
// rounds (a barrier across GPUs between them).
#include <climits>

#include "ue_internal.cuh"
#include "ue_bulk.cuh"
#include "ue_grad.cuh"

namespace ue {
namespace {

// A set of GPU ids < kMaxGpus kept in registers (every index is unrolled).
struct GpuSet {
    uint32_t w[kMaxGpus / 32];

    __device__ __forceinline__ void clear()
    {
#pragma unroll
        for (int i = 0; i < kMaxGpus / 32; ++i) w[i] = 0;
    }
    __device__ __forceinline__ void add(int x)
    {
#pragma unroll
        for (int i = 0; i < kMaxGpus / 32; ++i)
            if ((x >> 5) == i) w[i] |= 1u << (x & 31);
    }
    // Members below x.
    __device__ __forceinline__ int count_below(int x) const
    {
        int n = 0;
#pragma unroll
        for (int i = 0; i < kMaxGpus / 32; ++i) {
            const int lo = i * 32;
            if (x >= lo + 32) n += __popc(w[i]);
            else if (x > lo) n += __popc(w[i] & ((1u << (x - lo)) - 1u));
        }
        return n;
    }
};

__global__ void __launch_bounds__(kSyncThreads, 1)
k_sync_shard(PeerTable base, uint8_t *__restrict__ local, int64_t slot_bytes, int E, int S, int SG, int G, int g,
             int round, int cap, const int32_t *__restrict__ rep_off, const int32_t *__restrict__ rep_slot,
             const int32_t *__restrict__ rep_experts, const int32_t *__restrict__ info,
             int32_t *__restrict__ dev_err, unsigned long long wait_ns, int stall)
{
    extern __shared__ __align__(128) uint8_t sm_sync[];
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm_sync);                 // [stages + 1]; the last one: see stall
    uint8_t *stage = sm_sync + 128;                                        // [stages][tile]
    const uint8_t **x_base = reinterpret_cast<const uint8_t **>(stage + (size_t)kSyncStages * kSyncTile);  // [G]
    int64_t *x_q = reinterpret_cast<int64_t *>(x_base + kMaxGpus);        // [E] part length
    int32_t *x_first = reinterpret_cast<int32_t *>(x_q + E);               // [E] first replica entry (off + 1)
    int32_t *x_cnt = x_first + E;                                          // [E] destinations on this GPU
    int32_t *x_j0 = x_cnt + E;                                             // [E] first part index
    int32_t *x_pn = x_j0 + E;                                              // [E] part indices (before the skip)
    int32_t *x_skip = x_pn + E;                                            // [E] part left out (-1: none)
    int32_t *x_pt = x_skip + E;                                            // [E] tiles per full part
    int32_t *x_home = x_pt + E;                                            // [E] home slot, or -1: parts from consumers
    int32_t *x_ipre = x_home + E;                                          // [E+1] exclusive prefix of items
    int32_t *x_slot = x_ipre + E + 1;                                      // [cap] local destination slots
    int32_t *x_src = x_slot + cap;                                         // [cap] lowest slot of consumer j

    for (int i = threadIdx.x; i < G; i += blockDim.x) x_base[i] = static_cast<const uint8_t *>(base.p[i]);
    // Per replicated expert: this GPU's slots of it, its consumers (the GPUs
    // other than the home one holding it) and, for this round, which parts of
    // the slot this GPU receives and from where.
    const int M = clampi(__ldg(info + 3), 0, E);
    for (int m = threadIdx.x; m < M; m += blockDim.x) {
        const int e = clampi(__ldg(rep_experts + m), 0, E - 1);
        const int off = clampi(__ldg(rep_off + e), 0, cap - 1);
        const int end = clampi(__ldg(rep_off + e + 1), off + 1, cap);
        const int home = clampi(__ldg(rep_slot + off), 0, S - 1);
        const int hg = home / SG;
        GpuSet cons;
        cons.clear();
        int c = 0;
        for (int p = off + 1; p < end; ++p) {
            const int s = clampi(__ldg(rep_slot + p), 0, S - 1);
            const int gp = s / SG;
            if (gp != hg) cons.add(gp);
            if (gp == g) x_slot[off + 1 + c++] = s - g * SG;
        }
        const int f = cons.count_below(kMaxGpus);
        int64_t q = slot_bytes;
        int j0 = 0, pn = 1, skip = -1, src_home = home;
        bool active = c > 0;
        if (active) {
            if (g == hg) {
                active = round <= 0;                 // the home GPU's own replicas: round 0 (or direct)
            } else if (round >= 0) {
                const int i = cons.count_below(g);   // this GPU's consumer index
                q = 16 * ((slot_bytes + 16 * (int64_t)f - 1) / (16 * (int64_t)f));
                if (round == 0) {
                    j0 = i;                          // scatter: its own part, from the home slot
                } else {
                    pn = f;                          // all-gather: every other part, from its consumer
                    skip = i;
                    src_home = -1;
                    for (int j = 0; j < f; ++j) x_src[off + 1 + j] = INT_MAX;
                    for (int p = off + 1; p < end; ++p) {
                        const int s = clampi(__ldg(rep_slot + p), 0, S - 1);
                        const int gp = s / SG;
                        if (gp == hg) continue;
                        const int j = cons.count_below(gp);
                        if (s < x_src[off + 1 + j]) x_src[off + 1 + j] = s;
                    }
                }
            }
        }
        int items = 0;
        const int pt = (int)((q + kSyncTile - 1) / kSyncTile);
        if (active)
            for (int j = j0; j < j0 + pn; ++j) {
                if (j == skip) continue;
                const int64_t lo = (int64_t)j * q;
                const int64_t len = lo < slot_bytes ? (slot_bytes - lo < q ? slot_bytes - lo : q) : 0;
                items += (int)((len + kSyncTile - 1) / kSyncTile);
            }
        x_q[m] = q;
        x_first[m] = off + 1;
        x_cnt[m] = c;
        x_j0[m] = j0;
        x_pn[m] = pn;
        x_skip[m] = skip;
        x_pt[m] = pt;
        x_home[m] = src_home;
        x_ipre[m] = items;                           // turned into the exclusive prefix below
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i <= kSyncStages; ++i) mbar_init(&bar[i], 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x < 32) {                  // exclusive prefix of the items over the experts
        const int lane = threadIdx.x;
        int run = 0;
        for (int m0 = 0; m0 < M; m0 += 32) {
            const int m = m0 + lane;
            const int v = m < M ? x_ipre[m] : 0;
            int x = v;
#pragma unroll
            for (int d = 1; d < 32; d <<= 1) {
                const int y = __shfl_up_sync(0xffffffffu, x, d);
                if (lane >= d) x += y;
            }
            if (m < M) x_ipre[m] = run + x - v;
            run += __shfl_sync(0xffffffffu, x, 31);
        }
        if (lane == 0) x_ipre[M] = run;
    }
    __syncthreads();
    const int total = x_ipre[M];
    if (threadIdx.x != 0 || total == 0 || (int)blockIdx.x >= total) return;
    const int64_t nmy = (total - 1 - (int)blockIdx.x) / (int)gridDim.x + 1;

    struct Item {
        int m;
        unsigned bytes;
        int64_t offset;
        const uint8_t *src;
    };
    auto item = [&](int64_t k) {
        const int idx = (int)blockIdx.x + (int)(k * gridDim.x);
        int lo = 0, hi = M - 1;                      // last m with x_ipre[m] <= idx
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (x_ipre[mid] <= idx) lo = mid;
            else hi = mid - 1;
        }
        Item it;
        it.m = lo;
        const int l = idx - x_ipre[lo];
        const int pt = x_pt[lo];
        const int ord = l / pt;                      // ordinal among the parts received
        const int sk = x_skip[lo];
        const int j = x_j0[lo] + ord + (sk >= 0 && x_j0[lo] + ord >= sk ? 1 : 0);
        const int64_t q = x_q[lo];
        const int64_t pend = ((int64_t)j + 1) * q < slot_bytes ? ((int64_t)j + 1) * q : slot_bytes;
        it.offset = (int64_t)j * q + (int64_t)(l - ord * pt) * kSyncTile;
        const int64_t left = pend - it.offset;
        it.bytes = (unsigned)(left < kSyncTile ? left : kSyncTile);
        const int src = x_home[lo] >= 0 ? x_home[lo] : x_src[x_first[lo] + j];
        const int sg = src / SG;
        it.src = x_base[sg] + (int64_t)(src - sg * SG) * slot_bytes + it.offset;
        return it;
    };
    auto issue_load = [&](int64_t k) {
        const Item it = item(k);
        const int b = (int)(k % kSyncStages);
        mbar_expect_tx(&bar[b], it.bytes);
        bulk_load(stage + (size_t)b * kSyncTile, it.src, it.bytes, &bar[b]);
    };

    int64_t issued = 0;
    for (; issued < nmy && issued < kSyncStages; ++issued) issue_load(issued);
    // Diagnostic: CTA 0 waits once, with its first loads in flight, on the
    // extra barrier, on which nothing ever arrives (see k_sync).
    if (stall && blockIdx.x == 0 && !mbar_wait_bounded(&bar[kSyncStages], 0, wait_ns)) {
        ring_give_up(dev_err, bar, kSyncStages, 0, issued, wait_ns);
        return;
    }
    for (int64_t k = 0; k < nmy; ++k) {
        const int b = (int)(k % kSyncStages);
        if (!mbar_wait_bounded(&bar[b], (unsigned)((k / kSyncStages) & 1), wait_ns)) {
            ring_give_up(dev_err, bar, kSyncStages, k + 1, issued, wait_ns);
            return;
        }
        const Item it = item(k);
        const uint8_t *src = stage + (size_t)b * kSyncTile;
        const int first = x_first[it.m], cnt = x_cnt[it.m];
        for (int j = 0; j < cnt; ++j)
            bulk_store(local + (int64_t)x_slot[first + j] * slot_bytes + it.offset, src, it.bytes);
        bulk_commit();
        if (k >= 1 && k - 1 + kSyncStages < nmy) {
            bulk_wait_read_1();
            issue_load(k - 1 + kSyncStages);
            ++issued;
        }
    }
    bulk_wait_all();
}

template <bool BF16>
__global__ void __launch_bounds__(kGradThreads)
k_grad_reduce_shard(float *__restrict__ master, PeerTable grads, int64_t P, int E, int S, int H, int HR, int R,
                    int NG, int G, int g, int cap, const int32_t *__restrict__ rep_off,
                    const int32_t *__restrict__ rep_slot, const int32_t *__restrict__ rep_experts,
                    const int32_t *__restrict__ info)
{
    extern __shared__ __align__(16) uint8_t sm_grs[];
    const void **x_base = reinterpret_cast<const void **>(sm_grs);            // [G]
    int32_t *x_e = reinterpret_cast<int32_t *>(x_base + kMaxGpus);            // [E] local master row of m
    int32_t *x_first = x_e + E;                                               // [E]
    int32_t *x_cnt = x_first + E;                                             // [E]
    int32_t *x_act = x_cnt + E;                                               // [E+1]
    int32_t *x_loc = x_act + E + 1;                                           // [cap] gpu << 16 | local row

    for (int i = threadIdx.x; i < G; i += blockDim.x) x_base[i] = grads.p[i];
    const int EG = E / G;
    const int M = R > 0 ? clampi(__ldg(info + 3), 0, E) : 0;
    for (int m = threadIdx.x; m < M; m += blockDim.x) {
        const int e = clampi(__ldg(rep_experts + m), 0, E - 1);
        const int off = clampi(__ldg(rep_off + e), 0, cap - 1);
        const int end = clampi(__ldg(rep_off + e + 1), off + 1, cap);
        x_e[m] = e - g * EG;
        x_first[m] = off + 1;
        x_cnt[m] = e / EG == g ? end - off - 1 : 0;   // reduced on its home GPU only
    }
    for (int p = threadIdx.x; p < cap; p += blockDim.x) {
        const int s = clampi(__ldg(rep_slot + p), 0, S - 1);
        const int r = s / HR, u = s % HR - H;          // u < 0 for home slots
        const int h = r / NG;
        x_loc[p] = u >= 0 ? (h << 16) | ((r - h * NG) * R + u) : 0;
    }
    __syncthreads();
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        int n = 0;
        for (int m0 = 0; m0 < M; m0 += 32) {
            const int m = m0 + lane;
            const bool a = m < M && x_cnt[m] > 0;
            const unsigned b = __ballot_sync(0xffffffffu, a);
            if (a) x_act[n + __popc(b & lanemask_lt())] = m;
            n += __popc(b);
        }
        if (lane == 0) x_act[E] = n;
    }
    __syncthreads();
    const int MA = x_act[E];

    const int64_t nchunks = (P + kChunk - 1) / kChunk;
    const int64_t total = (int64_t)MA * nchunks;
    for (int64_t it = blockIdx.x; it < total; it += gridDim.x) {
        const int m = x_act[(int)(it / nchunks)];
        const int64_t x = (it % nchunks) * kChunk + (int64_t)threadIdx.x * kElemsPerThread;
        if (x >= P) continue;
        float4 *mp = reinterpret_cast<float4 *>(master + (int64_t)x_e[m] * P + x);
        const float4 a = __ldcs(mp), b = __ldcs(mp + 1);
        F8 acc;
        acc.v[0] = a.x; acc.v[1] = a.y; acc.v[2] = a.z; acc.v[3] = a.w;
        acc.v[4] = b.x; acc.v[5] = b.y; acc.v[6] = b.z; acc.v[7] = b.w;
        const int first = x_first[m], cnt = x_cnt[m];
        for (int j0 = 0; j0 < cnt; j0 += kBatch) {
            F8 gv[kBatch];
#pragma unroll
            for (int j = 0; j < kBatch; ++j)
                if (j0 + j < cnt) {
                    const int loc = x_loc[first + j0 + j];
                    gv[j] = load8<BF16>(x_base[loc >> 16], (int64_t)(loc & 0xffff) * P + x);
                }
#pragma unroll
            for (int j = 0; j < kBatch; ++j)
                if (j0 + j < cnt) add8(acc, gv[j]);
        }
        __stcs(mp, make_float4(acc.v[0], acc.v[1], acc.v[2], acc.v[3]));
        __stcs(mp + 1, make_float4(acc.v[4], acc.v[5], acc.v[6], acc.v[7]));
    }
}

}  // namespace

int relay_rounds(int G) { return G <= 2 ? 1 : 2; }

size_t sync_shard_smem_bytes(const Shape &sh)
{
    const int cap = sh.E + sh.NR;
    return 128 + (size_t)kSyncStages * kSyncTile + kMaxGpus * sizeof(void *) + (size_t)sh.E * sizeof(int64_t) +
           (size_t)(8 * sh.E + 1 + 2 * cap) * sizeof(int32_t);
}

size_t grad_shard_smem_bytes(const Shape &sh)
{
    return kMaxGpus * sizeof(void *) + (size_t)(4 * sh.E + 1 + sh.E + sh.NR) * sizeof(int32_t);
}

cudaError_t launch_sync_shard(const Shape &sh, const Launch &ln, const PeerTable &base, uint8_t *local, int G,
                              int g, int round, int64_t slot_bytes, const PlanDev &plan, int32_t *dev_err,
                              cudaStream_t st, const WaitBound &wb)
{
    k_sync_shard<<<ln.sms, kSyncThreads, sync_shard_smem_bytes(sh), st>>>(
        base, local, slot_bytes, sh.E, sh.S, sh.S / G, G, g, round, sh.E + sh.NR, plan.rep_off, plan.rep_slot,
        plan.rep_experts, plan.info, dev_err, wb.ns, wb.stall);
    return cudaGetLastError();
}

int grad_shard_blocks_per_sm(int grad_dtype, size_t smem);

cudaError_t launch_grad_reduce_shard(const Shape &sh, const Launch &ln, float *master, const PeerTable &grads,
                                     int G, int g, int grad_dtype, int64_t P, const PlanDev &plan, cudaStream_t st)
{
    const size_t smem = grad_shard_smem_bytes(sh);
    const int cap = sh.E + sh.NR, NG = sh.N / G;
    const unsigned grid = (unsigned)(ln.sms * grad_shard_blocks_per_sm(grad_dtype, smem));
    if (grad_dtype == 1)
        k_grad_reduce_shard<true><<<grid, kGradThreads, smem, st>>>(master, grads, P, sh.E, sh.S, sh.H, sh.HR,
                                                                      sh.R, NG, G, g, cap, plan.rep_off,
                                                                      plan.rep_slot, plan.rep_experts, plan.info);
    else
        k_grad_reduce_shard<false><<<grid, kGradThreads, smem, st>>>(master, grads, P, sh.E, sh.S, sh.H, sh.HR,
                                                                       sh.R, NG, G, g, cap, plan.rep_off,
                                                                       plan.rep_slot, plan.rep_experts, plan.info);
    return cudaGetLastError();
}

// Resident CTAs per SM with the shared memory one launch uses.
int grad_shard_blocks_per_sm(int grad_dtype, size_t smem)
{
    int n = 0;
    const cudaError_t e =
        grad_dtype == 1
            ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_grad_reduce_shard<true>, kGradThreads, smem)
            : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_grad_reduce_shard<false>, kGradThreads, smem);
    return (e == cudaSuccess && n > 0) ? n : 1;
}

cudaError_t set_shard_attributes(size_t max_smem)
{
    cudaError_t e = allow_smem(k_sync_shard, max_smem);
    if (e == cudaSuccess) e = allow_smem(k_grad_reduce_shard<true>, max_smem);
    if (e == cudaSuccess) e = allow_smem(k_grad_reduce_shard<false>, max_smem);
    return e;
}

}  // namespace ue
