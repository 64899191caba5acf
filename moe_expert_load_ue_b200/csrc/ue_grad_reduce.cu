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

}  // namespace

int grad_blocks_per_sm(int grad_dtype)
{
    int n = 0;
    const cudaError_t e =
        grad_dtype == 1
            ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_grad_reduce<true>, kGradThreads, 32 * 1024)
            : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_grad_reduce<false>, kGradThreads, 32 * 1024);
    return (e == cudaSuccess && n > 0) ? n : 1;
}

size_t grad_smem_bytes(const Shape &sh) { return (size_t)(3 * sh.E + sh.E + sh.NR) * sizeof(int32_t); }

cudaError_t launch_grad_reduce(const Shape &sh, const Launch &ln, float *master, const void *grads,
                               int grad_dtype, int64_t P, const PlanDev &plan, cudaStream_t st)
{
    const dim3 grid((unsigned)ln.sms);   // resident CTAs: SMs x blocks per SM
    const size_t smem = grad_smem_bytes(sh);
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
