// Element helpers of the gradient-reduction kernels: eight consecutive
// elements per thread, fp32 adds in round-to-nearest, bf16 widened exactly,
// streaming (evict-first) loads.
#pragma once

#include <cstdint>

#include <cuda_bf16.h>

namespace ue {
namespace {

constexpr int kGradThreads = 256;
constexpr int kElemsPerThread = 8;
constexpr int kChunk = kGradThreads * kElemsPerThread;
constexpr int kBatch = 4;

struct F8 {
    float v[8];
};

__device__ __forceinline__ void add8(F8 &acc, const F8 &g)
{
#pragma unroll
    for (int i = 0; i < 8; ++i) acc.v[i] = __fadd_rn(acc.v[i], g.v[i]);
}

template <bool BF16>
__device__ __forceinline__ F8 load8(const void *base, int64_t elem)
{
    F8 r;
    if constexpr (BF16) {
        const uint4 u = __ldcs(reinterpret_cast<const uint4 *>(static_cast<const __nv_bfloat16 *>(base) + elem));
        const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {   // bf16 -> fp32 is exact: the 16 bits become the high half
            r.v[2 * i] = __uint_as_float(w[i] << 16);
            r.v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    } else {
        const float4 *p = reinterpret_cast<const float4 *>(static_cast<const float *>(base) + elem);
        const float4 a = __ldcs(p), b = __ldcs(p + 1);
        r.v[0] = a.x; r.v[1] = a.y; r.v[2] = a.z; r.v[3] = a.w;
        r.v[4] = b.x; r.v[5] = b.y; r.v[6] = b.z; r.v[7] = b.w;
    }
    return r;
}

}  // namespace
}  // namespace ue
