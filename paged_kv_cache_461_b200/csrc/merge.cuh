// merge.cuh -- merge of attention states over disjoint key ranges (the flash-decoding
// second pass): for one (row, head) with parts s = 0..n-1 holding normalised outputs o_s
// and natural-log LSEs, LSE = ln sum exp(lse_s) and out = sum exp(lse_s - LSE) o_s, one
// warp per (row, head), fp32 throughout, bf16 output.
#pragma once

#include <math_constants.h>

#include <type_traits>

#include "pa_internal.cuh"

namespace pa {

// Global loads that bypass L1 (kFresh): states written by other CTAs of the same grid.
template <bool kFresh, typename T>
__device__ __forceinline__ T ld_state(const T *p)
{
    if constexpr (kFresh)
        return __ldcg(p);
    else
        return *p;
}

// One warp merges the n parts of one (row, head).  o points at part 0's D floats (parts
// o_stride floats apart), lse at part 0 (lse_stride apart).
template <int D, bool kFresh = false>
__device__ __forceinline__ void merge_one(const float *__restrict__ o, int64_t o_stride, const float *__restrict__ lse,
                                          int lse_stride, int n, __nv_bfloat16 *__restrict__ out, float *lse_out)
{
    constexpr int kPer = D / 32; // 4 (D=128) or 2 (D=64) consecutive floats per lane
    using Vec = typename std::conditional<kPer == 4, float4, float2>::type;
    const int lane = threadIdx.x & 31;
    float mx = -CUDART_INF_F;
    for (int s = lane; s < n; s += 32)
        mx = fmaxf(mx, ld_state<kFresh>(lse + (int64_t)s * lse_stride));
#pragma unroll
    for (int o2 = 16; o2; o2 >>= 1)
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o2));
    float acc[kPer];
#pragma unroll
    for (int i = 0; i < kPer; ++i)
        acc[i] = 0.f;
    float z = 0.f;
    if (mx != -CUDART_INF_F) {
        for (int s0 = 0; s0 < n; s0 += 32) {
            const int s = s0 + lane;
            const float w = s < n ? __expf(ld_state<kFresh>(lse + (int64_t)s * lse_stride) - mx) : 0.f;
            z += w;
            const int cnt = min(32, n - s0);
            // four parts' loads in flight before their products are accumulated
            int k = 0;
            for (; k + 4 <= cnt; k += 4) {
                Vec v[4];
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    v[u] = ld_state<kFresh>(reinterpret_cast<const Vec *>(o + (int64_t)(s0 + k + u) * o_stride +
                                                                          lane * kPer));
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float wk = __shfl_sync(0xffffffffu, w, k + u);
                    acc[0] += wk * v[u].x;
                    acc[1] += wk * v[u].y;
                    if constexpr (kPer == 4) {
                        acc[2] += wk * reinterpret_cast<const float4 &>(v[u]).z;
                        acc[3] += wk * reinterpret_cast<const float4 &>(v[u]).w;
                    }
                }
            }
            for (; k < cnt; ++k) {
                const float wk = __shfl_sync(0xffffffffu, w, k);
                const Vec v =
                    ld_state<kFresh>(reinterpret_cast<const Vec *>(o + (int64_t)(s0 + k) * o_stride + lane * kPer));
                acc[0] += wk * v.x;
                acc[1] += wk * v.y;
                if constexpr (kPer == 4) {
                    acc[2] += wk * reinterpret_cast<const float4 &>(v).z;
                    acc[3] += wk * reinterpret_cast<const float4 &>(v).w;
                }
            }
        }
#pragma unroll
        for (int o2 = 16; o2; o2 >>= 1)
            z += __shfl_xor_sync(0xffffffffu, z, o2);
    }
    const float inv = z > 0.f ? 1.f / z : 0.f;
    __nv_bfloat16 *dst = out + lane * kPer;
    if constexpr (kPer == 4) {
        __nv_bfloat162 a = __floats2bfloat162_rn(acc[0] * inv, acc[1] * inv);
        __nv_bfloat162 b = __floats2bfloat162_rn(acc[2] * inv, acc[3] * inv);
        uint2 v;
        v.x = *reinterpret_cast<uint32_t *>(&a);
        v.y = *reinterpret_cast<uint32_t *>(&b);
        *reinterpret_cast<uint2 *>(dst) = v;
    } else {
        *reinterpret_cast<__nv_bfloat162 *>(dst) = __floats2bfloat162_rn(acc[0] * inv, acc[1] * inv);
    }
    if (lse_out && lane == 0)
        *lse_out = z > 0.f ? mx + logf(z) : -CUDART_INF_F;
}

} // namespace pa
