// route.cuh -- per-token mask routing ("Masked Gated Linear Unit", "Measured
// effects": route each token to 1 or 2 of its 4 masks instead of summing all
// of them; the page defines no router, the reading here is one linear map of
// the token and top-k, after the mixture-of-experts routers it builds on).
//
// One warp per token: the n_m router scores r_i = sum_k x[k] W_r[i][k] in
// fp32 (lane-strided partial sums, then a fixed butterfly), then lane 0
// keeps the k highest scores (of equal scores the lower mask index; a NaN
// score never beats a number) and writes the token's mask weights: 1 for
// each kept mask ("hard"), or the softmax of all n_m scores for each kept
// mask ("softmax"); 0 for the others.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

namespace mglu {

enum { ROUTE_HARD = 0, ROUTE_SOFTMAX = 1 };

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename E>
__global__ void __launch_bounds__(256) route_kernel(const E *__restrict__ x, int64_t T, int64_t d,
                                                    const E *__restrict__ Wr, int n_m, int k, int mode,
                                                    float *__restrict__ weights, float *__restrict__ scores)
{
    const int lane = threadIdx.x & 31;
    const int64_t t = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (t >= T)
        return;
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
        acc[i] = 0.0f;
    const E *xr = x + t * d;
    for (int64_t kk = lane; kk < d; kk += 32) {
        const float xv = to_f32(xr[kk]);
#pragma unroll
        for (int i = 0; i < 8; ++i)
            if (i < n_m)
                acc[i] = fmaf(xv, to_f32(Wr[(int64_t)i * d + kk]), acc[i]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
#pragma unroll
        for (int i = 0; i < 8; ++i)
            acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], off);
    if (lane != 0)
        return;
    uint32_t sel = 0;
    for (int r = 0; r < k; ++r) {
        int best = -1;
        for (int i = 0; i < n_m; ++i)
            if (!((sel >> i) & 1u) && (best < 0 || acc[i] > acc[best]))
                best = i;
        sel |= 1u << best;
    }
    float m = -INFINITY, den = 0.0f;
    if (mode == ROUTE_SOFTMAX) {
        for (int i = 0; i < n_m; ++i)
            m = fmaxf(m, acc[i]);
        for (int i = 0; i < n_m; ++i)
            den += expf(acc[i] - m);
    }
    for (int i = 0; i < n_m; ++i) {
        const bool kept = (sel >> i) & 1u;
        const float w = !kept ? 0.0f : mode == ROUTE_SOFTMAX ? expf(acc[i] - m) / den : 1.0f;
        weights[t * n_m + i] = w;
        if (scores)
            scores[t * n_m + i] = acc[i];
    }
}

}  // namespace mglu
