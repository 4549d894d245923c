// route.cuh -- per-token mask routing ("Masked Gated Linear Unit", "Measured
// effects": route each token to 1 or 2 of its 4 masks instead of summing all
// of them; the page defines no router, the reading here is one linear map of
// the token and top-k, after the mixture-of-experts routers it builds on).
//
// One CTA of 256 threads per token: the n_m router scores
// r_i = sum_k x[k] W_r[i][k] in fp32 (each thread a strided share of k, 16-byte
// loads where the rows allow them, then a fixed reduction tree over the
// threads), then thread 0 keeps the k highest scores (of equal scores the
// lower mask index; a NaN score never beats a number) and writes the token's
// mask weights: 1 for each kept mask ("hard"), or the softmax of all n_m
// scores for each kept mask ("softmax"); 0 for the others.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace mglu {

enum { ROUTE_HARD = 0, ROUTE_SOFTMAX = 1 };

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

__device__ __forceinline__ void acc8(float (&acc)[8], int n_m, const float (&xv)[8], const uint4 *w, int64_t stride)
{
#pragma unroll
    for (int i = 0; i < 8; ++i)
        if (i < n_m) {
            const uint4 v = __ldg(w + i * stride);
            const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                acc[i] = fmaf(xv[2 * e], __uint_as_float(u[e] << 16), acc[i]);
                acc[i] = fmaf(xv[2 * e + 1], __uint_as_float(u[e] & 0xFFFF0000u), acc[i]);
            }
        }
}

// The n_m partial scores of one token held by thread tid of a group of 256
// (tid = 0..255; thread tid takes k8 = tid, tid + 256, ... of the 8-value
// chunks, or k = tid, tid + 256, ... of single values), each summed
// over the 32 lanes of its warp by a fixed xor tree (every lane ends with
// its warp's sums).  The callers keep this order so that every copy of the
// router gives the same scores bit for bit.
template <typename E>
__device__ __forceinline__ void route_partial(const E *__restrict__ xr, int64_t d, const E *__restrict__ Wr, int n_m,
                                              int vec, int tid, float (&acc)[8])
{
#pragma unroll
    for (int i = 0; i < 8; ++i)
        acc[i] = 0.0f;
    if constexpr (sizeof(E) == 2) {
        if (vec) {  // d % 8 == 0 and 16-byte aligned rows: 8 values per load
            for (int64_t k8 = tid; k8 < d / 8; k8 += 256) {
                const uint4 v = __ldg(reinterpret_cast<const uint4 *>(xr) + k8);
                const uint32_t u[4] = {v.x, v.y, v.z, v.w};
                float xv[8];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    xv[2 * e] = __uint_as_float(u[e] << 16);
                    xv[2 * e + 1] = __uint_as_float(u[e] & 0xFFFF0000u);
                }
                acc8(acc, n_m, xv, reinterpret_cast<const uint4 *>(Wr) + k8, d / 8);
            }
        } else {
            for (int64_t kk = tid; kk < d; kk += 256) {
                const float xv = to_f32(xr[kk]);
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (i < n_m)
                        acc[i] = fmaf(xv, to_f32(Wr[(int64_t)i * d + kk]), acc[i]);
            }
        }
    } else {
        for (int64_t kk = tid; kk < d; kk += 256) {
            const float xv = to_f32(xr[kk]);
#pragma unroll
            for (int i = 0; i < 8; ++i)
                if (i < n_m)
                    acc[i] = fmaf(xv, to_f32(Wr[(int64_t)i * d + kk]), acc[i]);
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
#pragma unroll
        for (int i = 0; i < 8; ++i)
            acc[i] += __shfl_xor_sync(0xffffffffu, acc[i], off);
}

// From the 8 warps' sums part[w][i] of one token: the scores (summed over
// the warps in order), the k kept masks and the token's mask weights w[i]
// (scores into sc_out when not NULL).
__device__ __forceinline__ void route_select(const float (*part)[8], int n_m, int k, int mode, float *w,
                                             float *sc_out)
{
    float sc[8];
    for (int i = 0; i < 8; ++i) {
        float v = 0.0f;
        for (int ww = 0; ww < 8; ++ww)
            v += part[ww][i];
        sc[i] = v;
    }
    uint32_t sel = 0;
    for (int r = 0; r < k; ++r) {
        int best = -1;
        for (int i = 0; i < n_m; ++i)
            if (!((sel >> i) & 1u) && (best < 0 || sc[i] > sc[best]))
                best = i;
        sel |= 1u << best;
    }
    float m = -INFINITY, den = 0.0f;
    if (mode == ROUTE_SOFTMAX) {
        for (int i = 0; i < n_m; ++i)
            m = fmaxf(m, sc[i]);
        for (int i = 0; i < n_m; ++i)
            den += expf(sc[i] - m);
    }
    for (int i = 0; i < n_m; ++i) {
        const bool kept = (sel >> i) & 1u;
        w[i] = !kept ? 0.0f : mode == ROUTE_SOFTMAX ? expf(sc[i] - m) / den : 1.0f;
        if (sc_out)
            sc_out[i] = sc[i];
    }
}

template <typename E>
__global__ void __launch_bounds__(256) route_kernel(const E *__restrict__ x, int64_t T, int64_t d,
                                                    const E *__restrict__ Wr, int n_m, int k, int mode, int vec,
                                                    float *__restrict__ weights, float *__restrict__ scores)
{
    __shared__ float part[8][8];  // [warp][mask]
    // The next kernel in the stream (the routed forward) may launch and set
    // up now; it waits for this grid to complete before it reads anything.
    // This grid in turn waits for the previous kernel before reading x.
    pdl_launch_dependents();
    pdl_wait();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int64_t t = blockIdx.x;
    float acc[8];
    route_partial<E>(x + t * d, d, Wr, n_m, vec, tid, acc);
    if (lane == 0)
#pragma unroll
        for (int i = 0; i < 8; ++i)
            part[warp][i] = acc[i];
    __syncthreads();
    if (tid != 0)
        return;
    route_select(part, n_m, k, mode, weights + t * n_m, scores ? scores + t * n_m : nullptr);
}

}  // namespace mglu
