// Step 5 - replica gradient reduction into the fp32 master gradient.
//
// "Replica gradient reduction" (csrc/kernels/grad_reduce.cu in "How
// dots-infra/ultraep works"; "Expert compute -> Replica gradient reduction:
// replica gradients" and "Replica gradient reduction -> MoE framework: master
// gradients").  For every expert e holding redundant replicas, in replica
// order i = 1, 2, ...:
//     master[e][x] = master[e][x] + float(grad[row(i)][x])
// one fp32 round-to-nearest add per replica (bf16 widened exactly), so the
// result is bit-identical to a sequential loop in that order.
//
// Design (sm_100a): HBM-bound streaming.  A persistent grid-stride loop over
// (replicated expert, 2048-element chunk) items; each thread owns 8
// consecutive elements: two 16-byte fp32 loads of the master, one 16-byte
// load per bf16 replica row (two for fp32), all replica loads of a batch of
// four issued before the adds.  Loads and stores use the streaming
// (evict-first) cache operators: every byte is touched once.
#include <cuda_bf16.h>

#include "ue_internal.cuh"
#include "ue_grad.cuh"

namespace ue {
namespace {

template <bool BF16>
__global__ void __launch_bounds__(kGradThreads)
k_grad_reduce(float *__restrict__ master, const void *__restrict__ grads, int64_t P, int E, int S, int H,
              int HR, int R, int cap, const int32_t *__restrict__ rep_off, const int32_t *__restrict__ rep_slot,
              const int32_t *__restrict__ rep_experts, const int32_t *__restrict__ info)
{
    extern __shared__ __align__(16) int32_t sm_gr[];
    int32_t *x_e = sm_gr;            // [E] expert of item group m
    int32_t *x_first = x_e + E;      // [E] first redundant entry
    int32_t *x_cnt = x_first + E;    // [E]
    int32_t *x_row = x_cnt + E;      // [cap] replica-gradient row of each replica entry

    const int M = R > 0 ? clampi(__ldg(info + 3), 0, E) : 0;   // no replica rows when R == 0
    for (int m = threadIdx.x; m < M; m += blockDim.x) {
        const int e = clampi(__ldg(rep_experts + m), 0, E - 1);
        const int off = clampi(__ldg(rep_off + e), 0, cap - 1);
        const int end = clampi(__ldg(rep_off + e + 1), off + 1, cap);
        x_e[m] = e;
        x_first[m] = off + 1;
        x_cnt[m] = end - off - 1;
    }
    for (int p = threadIdx.x; p < cap; p += blockDim.x) {
        const int s = clampi(__ldg(rep_slot + p), 0, S - 1);
        const int u = s % HR - H;             // redundant index on its rank (< 0 for home slots)
        x_row[p] = u >= 0 ? (s / HR) * R + u : 0;
    }
    __syncthreads();

    const int64_t nchunks = (P + kChunk - 1) / kChunk;
    const int64_t total = (int64_t)M * nchunks;
    for (int64_t it = blockIdx.x; it < total; it += gridDim.x) {
        const int m = (int)(it / nchunks);
        const int64_t x = (it - (int64_t)m * nchunks) * kChunk + (int64_t)threadIdx.x * kElemsPerThread;
        if (x >= P) continue;
        float4 *mp = reinterpret_cast<float4 *>(master + (int64_t)x_e[m] * P + x);
        const float4 a = __ldcs(mp), b = __ldcs(mp + 1);
        F8 acc;
        acc.v[0] = a.x; acc.v[1] = a.y; acc.v[2] = a.z; acc.v[3] = a.w;
        acc.v[4] = b.x; acc.v[5] = b.y; acc.v[6] = b.z; acc.v[7] = b.w;
        const int first = x_first[m], cnt = x_cnt[m];
        for (int j0 = 0; j0 < cnt; j0 += kBatch) {
            F8 g[kBatch];
#pragma unroll
            for (int j = 0; j < kBatch; ++j)
                if (j0 + j < cnt) g[j] = load8<BF16>(grads, (int64_t)x_row[first + j0 + j] * P + x);
#pragma unroll
            for (int j = 0; j < kBatch; ++j)
                if (j0 + j < cnt) add8(acc, g[j]);
        }
        __stcs(mp, make_float4(acc.v[0], acc.v[1], acc.v[2], acc.v[3]));
        __stcs(mp + 1, make_float4(acc.v[4], acc.v[5], acc.v[6], acc.v[7]));
    }
}

// ---- the same reduction on the Tensor Memory Accelerator's bulk copies ----------
//
// One persistent CTA per SM.  A producer lane streams each item's row chunks
// - the master chunk, then every replica's chunk in replica order - with
// cp.async.bulk into a ring of shared-memory slots (completion on an mbarrier
// per slot); eight consumer warps add them, in that order, into registers (the
// same fp32 round-to-nearest adds as k_grad_reduce, so the result is the same
// bits) and release each slot on its "empty" mbarrier; the sum goes back to
// the master row with one bulk store per item from a double-buffered output
// tile.  A slot holds a master chunk or kGbSlotBytes of replica chunks (one
// fp32 chunk, two bf16 ones), so the ring holds the same bytes whatever the
// gradient type.  Every wait is bounded by the global timer; on expiry the kernel
// records bit 0 in the status word, the producer lets its loads in flight land,
// and the CTA returns.
constexpr int kGbConsumers = 256;                 // 8 consumer warps
constexpr int kGbThreads = kGbConsumers + 32;     // + 1 producer warp
constexpr int kGbChunk = 8192;                    // elements per item
constexpr int kGbPer = kGbChunk / kGbConsumers;   // 32 elements per consumer thread
constexpr int kGbWarpElems = kGbChunk / (kGbConsumers / 32);   // 1024 elements per consumer warp
constexpr int kGbSlots = 4;
constexpr int kGbSlotBytes = kGbChunk * 4;        // a master chunk (fp32); a replica chunk fits too
__device__ __forceinline__ uint32_t gb_smem(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

// Waits for the mbarrier phase, at most limit_ns on the global timer.
__device__ __forceinline__ bool gb_wait(uint64_t *bar, unsigned parity, unsigned long long limit_ns)
{
    unsigned ok;
    asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(gb_smem(bar)), "r"(parity) : "memory");
    if (ok) return true;
    unsigned long long t0, t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
    for (;;) {
        asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                     "selp.u32 %0, 1, 0, p;\n\t}"
                     : "=r"(ok) : "r"(gb_smem(bar)), "r"(parity) : "memory");
        if (ok) return true;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
        if (t - t0 > limit_ns) return false;
    }
}

// SHARD: the same reduction across G GPUs on GPU g: only the experts homed on
// GPU g (master holds their rows, e - g * E/G), each replica's chunk pulled
// from the GPU holding its gradient row through the peer table (GPU h =
// rank / (N/G), local row (rank - h * N/G) * R + u) with plain bulk loads.
template <bool BF16, bool SHARD>
__global__ void __launch_bounds__(kGbThreads, 1)
k_grad_reduce_bulk(float *__restrict__ master, const void *__restrict__ grads, PeerTable peers, int G, int g,
                   int64_t P, int E, int S, int H, int HR, int R, int cap, const int32_t *__restrict__ rep_off,
                   const int32_t *__restrict__ rep_slot, const int32_t *__restrict__ rep_experts,
                   const int32_t *__restrict__ info, int32_t *__restrict__ dev_err, unsigned long long wait_ns,
                   int stall)
{
    extern __shared__ __align__(128) uint8_t sm_gb[];
    uint64_t *full = reinterpret_cast<uint64_t *>(sm_gb);           // [kGbSlots]
    uint64_t *empty = full + kGbSlots;                                // [kGbSlots]
    uint64_t *never = empty + kGbSlots;                               // diagnostic: nothing arrives on it
    int32_t *abort_flag = reinterpret_cast<int32_t *>(never + 1);
    uint8_t *slot = sm_gb + 1024;                                     // [kGbSlots][kGbSlotBytes]
    float *outb = reinterpret_cast<float *>(slot + kGbSlots * kGbSlotBytes);   // [warps][2][kGbWarpElems]
    int32_t *x_e = reinterpret_cast<int32_t *>(outb + 2 * kGbChunk);  // [E]
    int32_t *x_first = x_e + E;                                       // [E]
    int32_t *x_cnt = x_first + E;                                     // [E]
    int32_t *x_row = x_cnt + E;                                       // [cap] replica row (SHARD: gpu << 16 | local row)
    int32_t *x_act = x_row + cap;                                     // [E + 1] SHARD: experts with work; count
    const uint8_t **x_base = reinterpret_cast<const uint8_t **>(
        (reinterpret_cast<uintptr_t>(x_act + E + 1) + 7) & ~static_cast<uintptr_t>(7));   // [kMaxGpus] SHARD

    const int M = R > 0 ? clampi(__ldg(info + 3), 0, E) : 0;
    const int EG = SHARD ? E / G : E, NG = SHARD ? (S / HR) / G : 1;
    for (int m = threadIdx.x; m < M; m += blockDim.x) {
        const int e = clampi(__ldg(rep_experts + m), 0, E - 1);
        const int off = clampi(__ldg(rep_off + e), 0, cap - 1);
        const int end = clampi(__ldg(rep_off + e + 1), off + 1, cap);
        x_e[m] = SHARD ? e - g * EG : e;
        x_first[m] = off + 1;
        x_cnt[m] = (!SHARD || e / EG == g) ? end - off - 1 : 0;     // across GPUs: reduced on its home GPU
    }
    for (int p = threadIdx.x; p < cap; p += blockDim.x) {
        const int sl = clampi(__ldg(rep_slot + p), 0, S - 1);
        const int r = sl / HR, u = sl % HR - H;
        if constexpr (SHARD) {
            const int h = r / NG;
            x_row[p] = u >= 0 ? (h << 16) | ((r - h * NG) * R + u) : 0;
        } else {
            x_row[p] = u >= 0 ? r * R + u : 0;
        }
    }
    if constexpr (SHARD) {
        for (int h = threadIdx.x; h < G; h += blockDim.x) x_base[h] = static_cast<const uint8_t *>(peers.p[h]);
        __syncthreads();
        if (threadIdx.x < 32) {                  // the experts homed here that have replicas
            int n = 0;
            for (int m0 = 0; m0 < M; m0 += 32) {
                const int m = m0 + threadIdx.x;
                const bool a = m < M && x_cnt[m] > 0;
                const unsigned bal = __ballot_sync(0xffffffffu, a);
                if (a) x_act[n + __popc(bal & lanemask_lt())] = m;
                n += __popc(bal);
            }
            if (threadIdx.x == 0) x_act[E] = n;
        }
    }
    if (threadIdx.x == 0) {
        for (int i = 0; i < kGbSlots; ++i) {
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(gb_smem(&full[i])) : "memory");
            asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(gb_smem(&empty[i])), "r"(kGbConsumers / 32)
                         : "memory");
        }
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(gb_smem(never)) : "memory");
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();

    const int64_t nchunks = (P + kGbChunk - 1) / kGbChunk;
    const int MA = SHARD ? x_act[E] : M;                  // work groups: SHARD lists them in x_act
    const int64_t total = (int64_t)MA * nchunks;
    auto group = [&](int64_t it) { return SHARD ? x_act[(int)(it / nchunks)] : (int)(it / nchunks); };
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int kElem = BF16 ? 2 : 4;
    constexpr int kRepPerSlot = kGbSlotBytes / (kGbChunk * kElem);   // bf16: two replica chunks per slot

    if (warp == kGbConsumers / 32) {
        // Producer: one lane walks the segments (master, then replicas) of this
        // CTA's items in order, one ring slot per segment.
        if (lane != 0) return;
        int64_t seg = 0;
        for (int64_t it = blockIdx.x; it < total; it += gridDim.x) {
            const int m = group(it);
            const int64_t x0 = (it % nchunks) * kGbChunk;
            const int n = (int)min((int64_t)kGbChunk, P - x0);
            const int cnt = x_cnt[m];
            const int nseg = 1 + (cnt + kRepPerSlot - 1) / kRepPerSlot;
            for (int j = 0; j < nseg; ++j, ++seg) {
                const int b = (int)(seg % kGbSlots);
                if (seg >= kGbSlots && !gb_wait(&empty[b], (unsigned)(((seg / kGbSlots) - 1) & 1), wait_ns)) {
                    atomicOr(dev_err, 1);
                    *reinterpret_cast<volatile int32_t *>(abort_flag) = 1;
                    // Let the loads already issued into the other slots land.
                    for (int64_t k = seg - kGbSlots + 1; k < seg; ++k)
                        gb_wait(&full[k % kGbSlots], (unsigned)((k / kGbSlots) & 1), wait_ns);
                    return;
                }
                // Segment 0: the master chunk; segment j >= 1: replicas
                // (j - 1) * kRepPerSlot + 1 .. (at most kRepPerSlot, each in
                // its kGbChunk * kElem bytes of the slot).
                const int r0 = (j - 1) * kRepPerSlot + 1;
                const int nr = j == 0 ? 1 : min(kRepPerSlot, cnt - r0 + 1);
                const unsigned bytes = j == 0 ? (unsigned)n * 4u : (unsigned)n * (unsigned)kElem;
                asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(gb_smem(&full[b])),
                             "r"(bytes * (unsigned)nr) : "memory");
                for (int q = 0; q < nr; ++q) {
                    const void *src;
                    if (j == 0) {
                        src = master + (int64_t)x_e[m] * P + x0;
                    } else {
                        const int loc = x_row[x_first[m] + r0 - 1 + q];
                        const uint8_t *gb = SHARD ? x_base[loc >> 16] : static_cast<const uint8_t *>(grads);
                        const int64_t row = SHARD ? (loc & 0xffff) : loc;
                        src = gb + (row * P + x0) * kElem;
                    }
                    asm volatile(
                        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
                        ::"r"(gb_smem(slot + (size_t)b * kGbSlotBytes + (size_t)q * kGbChunk * kElem)), "l"(src),
                        "r"(bytes), "r"(gb_smem(&full[b]))
                        : "memory");
                }
            }
        }
        // Drain: the consumers wait for the last loads; the producer leaves.
        return;
    }

    // Consumers: warp w owns the chunk's elements [w * kGbWarpElems, (w + 1) *
    // kGbWarpElems), lane l the float4 groups i * 32 + l of them; each warp
    // writes its part back from its own double-buffered output tile with its
    // own bulk stores, so no consumer waits on another (only on the ring's
    // mbarriers, each wait bounded).
    // Diagnostic: consumer warp 0 of CTA 0 waits once on a barrier nothing
    // completes; its wait runs out, it leaves, and the producer's wait for it
    // runs out in turn (the way out exercised by a test through the context).
    if (stall && blockIdx.x == 0 && warp == 0 && !gb_wait(never, 0, wait_ns)) {
        if (lane == 0) atomicOr(dev_err, 1);
        return;
    }
    int64_t seg = 0;
    int ob = 0;
    float *tile = outb + warp * (2 * kGbWarpElems);
    for (int64_t it = blockIdx.x; it < total; it += gridDim.x, ob ^= 1) {
        const int m = group(it);
        const int64_t x0 = (it % nchunks) * kGbChunk;
        const int n = (int)min((int64_t)kGbChunk, P - x0);
        const int cnt = x_cnt[m];
        const int w0 = warp * kGbWarpElems;                  // this warp's first element of the chunk
        const int nseg = 1 + (cnt + kRepPerSlot - 1) / kRepPerSlot;
        float acc[kGbPer];
        bool ok = true;
        for (int j = 0; j < nseg; ++j, ++seg) {
            const int b = (int)(seg % kGbSlots);
            if (!gb_wait(&full[b], (unsigned)((seg / kGbSlots) & 1), wait_ns)) {
                ok = false;
                break;
            }
            const uint8_t *src = slot + (size_t)b * kGbSlotBytes;
            const int nr = j == 0 ? 1 : min(kRepPerSlot, cnt - (j - 1) * kRepPerSlot);
            for (int q = 0; q < nr; ++q) {                     // replicas in order
                const uint8_t *sq = src + (size_t)q * kGbChunk * kElem;
#pragma unroll
                for (int i = 0; i < kGbPer / 4; ++i) {
                    const int x = w0 + 4 * (i * 32 + lane);
                    if (x >= n) continue;
                    float v[4];
                    if (j == 0 || !BF16) {
                        const float4 f = *reinterpret_cast<const float4 *>(sq + (size_t)x * 4);
                        v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
                    } else {
                        const uint2 u = *reinterpret_cast<const uint2 *>(sq + (size_t)x * 2);
                        v[0] = __uint_as_float(u.x << 16);
                        v[1] = __uint_as_float(u.x & 0xffff0000u);
                        v[2] = __uint_as_float(u.y << 16);
                        v[3] = __uint_as_float(u.y & 0xffff0000u);
                    }
#pragma unroll
                    for (int k = 0; k < 4; ++k) acc[4 * i + k] = j == 0 ? v[k] : __fadd_rn(acc[4 * i + k], v[k]);
                }
            }
            __syncwarp();
            if (lane == 0)
                asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(gb_smem(&empty[b])) : "memory");
        }
        if (!ok || *reinterpret_cast<volatile int32_t *>(abort_flag)) {
            if (lane == 0) {
                atomicOr(dev_err, 1);
                asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
            }
            return;
        }
        const int wn = min(kGbWarpElems, n - w0);            // elements of this warp's part (may be <= 0)
        if (wn <= 0) continue;
        // This warp's output tile is free once its store of two items ago has read it.
        float *out = tile + ob * kGbWarpElems;
        if (lane == 0) asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
        __syncwarp();
#pragma unroll
        for (int i = 0; i < kGbPer / 4; ++i) {
            const int x = 4 * (i * 32 + lane);
            if (x < wn) *reinterpret_cast<float4 *>(out + x) = make_float4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2],
                                                                         acc[4 * i + 3]);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) {
            asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(master +
                                                                                        (int64_t)x_e[m] * P + x0 + w0),
                         "r"(gb_smem(out)), "r"((unsigned)wn * 4u)
                         : "memory");
            asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        }
    }
    if (lane == 0) asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}

}  // namespace

size_t grad_bulk_smem_bytes(const Shape &sh)
{
    return 1024 + (size_t)kGbSlots * kGbSlotBytes + 2 * (size_t)kGbChunk * 4 +
           (size_t)(5 * sh.E + sh.NR + 1) * sizeof(int32_t) + 8 + (size_t)kMaxGpus * sizeof(void *);
}

namespace {
template <bool SHARD>
cudaError_t launch_bulk(const Shape &sh, int sms, float *master, const void *grads, const PeerTable &peers, int G,
                        int g, int grad_dtype, int64_t P, const PlanDev &plan, int32_t *dev_err, cudaStream_t st,
                        const WaitBound &wb)
{
    const size_t smem = grad_bulk_smem_bytes(sh);
    const int cap = sh.E + sh.NR;
    if (grad_dtype == 1)
        k_grad_reduce_bulk<true, SHARD><<<sms, kGbThreads, smem, st>>>(
            master, grads, peers, G, g, P, sh.E, sh.S, sh.H, sh.HR, sh.R, cap, plan.rep_off, plan.rep_slot,
            plan.rep_experts, plan.info, dev_err, wb.ns, wb.stall);
    else
        k_grad_reduce_bulk<false, SHARD><<<sms, kGbThreads, smem, st>>>(
            master, grads, peers, G, g, P, sh.E, sh.S, sh.H, sh.HR, sh.R, cap, plan.rep_off, plan.rep_slot,
            plan.rep_experts, plan.info, dev_err, wb.ns, wb.stall);
    return cudaGetLastError();
}
}  // namespace

cudaError_t launch_grad_reduce_bulk(const Shape &sh, int sms, float *master, const void *grads, int grad_dtype,
                                    int64_t P, const PlanDev &plan, int32_t *dev_err, cudaStream_t st,
                                    const WaitBound &wb)
{
    PeerTable none;
    none.p[0] = nullptr;
    return launch_bulk<false>(sh, sms, master, grads, none, 1, 0, grad_dtype, P, plan, dev_err, st, wb);
}

cudaError_t launch_grad_reduce_bulk_shard(const Shape &sh, int sms, float *master, const PeerTable &grads, int G,
                                          int g, int grad_dtype, int64_t P, const PlanDev &plan, int32_t *dev_err,
                                          cudaStream_t st, const WaitBound &wb)
{
    return launch_bulk<true>(sh, sms, master, nullptr, grads, G, g, grad_dtype, P, plan, dev_err, st, wb);
}

cudaError_t set_grad_bulk_attributes(size_t max_smem)
{
    cudaError_t e = allow_smem(k_grad_reduce_bulk<true, false>, max_smem);
    if (e == cudaSuccess) e = allow_smem(k_grad_reduce_bulk<false, false>, max_smem);
    if (e == cudaSuccess) e = allow_smem(k_grad_reduce_bulk<true, true>, max_smem);
    if (e == cudaSuccess) e = allow_smem(k_grad_reduce_bulk<false, true>, max_smem);
    return e;
}

// Resident CTAs per SM of the vector kernel with the shared memory one launch
// uses (its tables grow with E and N*R).
int grad_blocks_per_sm(int grad_dtype, size_t smem)
{
    int n = 0;
    const cudaError_t e =
        grad_dtype == 1
            ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_grad_reduce<true>, kGradThreads, smem)
            : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_grad_reduce<false>, kGradThreads, smem);
    return (e == cudaSuccess && n > 0) ? n : 1;
}

size_t grad_smem_bytes(const Shape &sh) { return (size_t)(3 * sh.E + sh.E + sh.NR) * sizeof(int32_t); }

cudaError_t launch_grad_reduce(const Shape &sh, const Launch &ln, float *master, const void *grads,
                               int grad_dtype, int64_t P, const PlanDev &plan, cudaStream_t st)
{
    const size_t smem = grad_smem_bytes(sh);
    const dim3 grid((unsigned)(ln.sms * grad_blocks_per_sm(grad_dtype, smem)));   // one wave of resident CTAs
    const int cap = sh.E + sh.NR;
    if (grad_dtype == 1)
        k_grad_reduce<true><<<grid, kGradThreads, smem, st>>>(master, grads, P, sh.E, sh.S, sh.H, sh.HR, sh.R, cap,
                                                              plan.rep_off, plan.rep_slot, plan.rep_experts, plan.info);
    else
        k_grad_reduce<false><<<grid, kGradThreads, smem, st>>>(master, grads, P, sh.E, sh.S, sh.H, sh.HR, sh.R, cap,
                                                               plan.rep_off, plan.rep_slot, plan.rep_experts, plan.info);
    return cudaGetLastError();
}

}  // namespace ue
