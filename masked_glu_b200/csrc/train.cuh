// train.cuh -- elementwise kernels of the training path ("Masked Gated Linear
// Unit", "Limitations": masks are learned, held as FP16 logits while
// training; the page lists the straight-through estimator among the works it
// builds on).  With a_i = dL/dg_i and c_i = dL/dv_i per token and column, the
// gradients regroup into products with n_m + 1 operands each:
//     dx    = sum_i (a_i - c_i) (M_i . W) + (sum_i c_i) W
//     E_i   = (a_i - c_i)^T x,   F = (sum_i c_i)^T x
//     dW    = sum_i M_i . E_i + F
//     dM_i  = W . E_i            (straight through: the logit gets dL/dM_i)
// The products are plain GEMMs over materialised operands; these kernels
// build the masked operand [M_1.W; ...; M_n.W; W] and combine the E_i.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "common.cuh"

namespace mglu {
namespace tr {

// Mask bits of the 8-weight chunk at (row j, k) as the lo/hi words of
// pair_mask (NM bytes at byte offset (j*d + k)*NM/8; k % 8 == 0).
template <int NM>
__device__ __forceinline__ void chunk_bits(const uint8_t *packed, int64_t j, int64_t d, int64_t k, uint32_t &lo,
                                           uint32_t &hi)
{
    const uint8_t *p = packed + (j * d + k) * NM / 8;
    if constexpr (NM == 8) {
        const uint2 v = __ldg(reinterpret_cast<const uint2 *>(p));
        lo = v.x;
        hi = v.y;
    } else if constexpr (NM == 4) {
        lo = __ldg(reinterpret_cast<const unsigned int *>(p));
        hi = 0;
    } else if constexpr (NM == 2) {
        lo = __ldg(reinterpret_cast<const unsigned short *>(p));
        hi = 0;
    } else {
        lo = __ldg(p);
        hi = 0;
    }
}

template <int NM, int I>
__device__ __forceinline__ void store_masked(uint4 *dst, int64_t plane, uint4 w, uint32_t lo, uint32_t hi)
{
    if constexpr (I < NM) {
        uint4 m;
        m.x = w.x & pair_mask<NM, 0, I>(lo, hi);
        m.y = w.y & pair_mask<NM, 1, I>(lo, hi);
        m.z = w.z & pair_mask<NM, 2, I>(lo, hi);
        m.w = w.w & pair_mask<NM, 3, I>(lo, hi);
        dst[I * plane] = m;
        store_masked<NM, I + 1>(dst, plane, w, lo, hi);
    }
}

// B [(NM + 1)][h][d] bf16: plane i < NM is M_i . W, plane NM is W.  One
// thread per 8-weight chunk (d % 8 == 0).
template <int NM>
__global__ void __launch_bounds__(256) masked_weights_kernel(const __nv_bfloat16 *__restrict__ W,
                                                             const uint8_t *__restrict__ packed, int64_t h, int64_t d,
                                                             __nv_bfloat16 *__restrict__ B)
{
    const int64_t chunk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t cpr = d / 8;  // chunks per row
    if (chunk >= h * cpr)
        return;
    const int64_t j = chunk / cpr, k = (chunk - j * cpr) * 8;
    const uint4 w = __ldg(reinterpret_cast<const uint4 *>(W + j * d + k));
    uint32_t lo, hi;
    chunk_bits<NM>(packed, j, d, k, lo, hi);
    uint4 *dst = reinterpret_cast<uint4 *>(B + j * d + k);
    const int64_t plane = h * d / 8;  // uint4 per plane
    store_masked<NM, 0>(dst, plane, w, lo, hi);
    dst[NM * plane] = w;
}

// dW [h][d] = sum_i M_i . E_i + E_NM, and dM_i [h][d] = W . E_i (if dM is not
// NULL), from E [(NM + 1)][h][d] fp32.  One thread per 4 consecutive k.
template <int NM>
__global__ void __launch_bounds__(256) combine_kernel(const float *__restrict__ E, const __nv_bfloat16 *__restrict__ W,
                                                      const uint8_t *__restrict__ packed, int64_t h, int64_t d,
                                                      float *__restrict__ dW, float *__restrict__ dM)
{
    const int64_t q = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;  // index of 4 weights
    const int64_t hd = h * d;
    if (q * 4 >= hd)
        return;
    const int64_t e0 = q * 4;  // d % 8 == 0, so the 4 weights share a row
    const int64_t j = e0 / d, k = e0 - j * d;
    float wv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
        wv[e] = __bfloat162float(W[e0 + e]);
    float acc[4];
    {
        const float4 f = __ldg(reinterpret_cast<const float4 *>(E + NM * hd + e0));
        acc[0] = f.x, acc[1] = f.y, acc[2] = f.z, acc[3] = f.w;
    }
#pragma unroll
    for (int i = 0; i < NM; ++i) {
        const float4 f = __ldg(reinterpret_cast<const float4 *>(E + i * hd + e0));
        const float ev[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int64_t pos = (j * d + k + e) * NM + i;  // the packed bit of mask i, weight (j, k + e)
            const float m = (float)((packed[pos >> 3] >> (pos & 7)) & 1u);
            acc[e] = fmaf(m, ev[e], acc[e]);
        }
        if (dM)
            *reinterpret_cast<float4 *>(dM + i * hd + e0) =
                make_float4(wv[0] * ev[0], wv[1] * ev[1], wv[2] * ev[2], wv[3] * ev[3]);
    }
    *reinterpret_cast<float4 *>(dW + e0) = make_float4(acc[0], acc[1], acc[2], acc[3]);
}

}  // namespace tr
}  // namespace mglu
