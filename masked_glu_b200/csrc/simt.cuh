// simt.cuh -- fp32 MGLU forward and fp32 dense product on CUDA cores.
//
// The fp32 path exists for full-precision inputs: plain fp32 multiply-add,
// never TF32.  One warp owns one output column j (a row of W) and up to four
// tokens; its lanes split k, then reduce with shuffles.
#pragma once
#include <cstdint>

#include "common.cuh"

namespace mglu {

constexpr int kSimtTokens = 4;

// NM = 0: dense product out[b][j] = sum_k x[b][k] * W[j][k] (the down-projection).
// NM > 0: out[b][j] = sum_i w_i act(g_i) * (D - g_i) with g_i the gate part
// of mask i and w_i the token's mask weight (mw [T][NM]; NULL: 1).
template <int NM>
__global__ void __launch_bounds__(256) simt_f32_kernel(const float *__restrict__ x, int64_t T, int64_t d,
                                                       const float *__restrict__ W, int64_t h,
                                                       const uint8_t *__restrict__ packed, int act,
                                                       float *__restrict__ out, const float *__restrict__ mw)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int64_t j = (int64_t)blockIdx.x * 8 + warp;
    const int64_t t0 = (int64_t)blockIdx.y * kSimtTokens;
    if (j >= h)
        return;
    const int nt = (int)(T - t0 < kSimtTokens ? T - t0 : kSimtTokens);
    float dense[kSimtTokens] = {0.f, 0.f, 0.f, 0.f};
    float gate[NM > 0 ? NM : 1][kSimtTokens];
#pragma unroll
    for (int i = 0; i < (NM > 0 ? NM : 1); ++i)
#pragma unroll
        for (int t = 0; t < kSimtTokens; ++t)
            gate[i][t] = 0.f;

    const float *wrow = W + j * d;
    for (int64_t k = lane; k < d; k += 32) {
        const float w = wrow[k];
        uint32_t bits = 0;
        if (NM > 0) {
            const int64_t pos = (j * d + k) * NM;  // first bit of weight (j, k)
            bits = (uint32_t)(packed[pos >> 3] >> (pos & 7));
        }
#pragma unroll
        for (int t = 0; t < kSimtTokens; ++t) {
            if (t < nt) {
                const float p = x[(t0 + t) * d + k] * w;
                dense[t] += p;
#pragma unroll
                for (int i = 0; i < NM; ++i)
                    if ((bits >> i) & 1u)
                        gate[i][t] += p;
            }
        }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
#pragma unroll
        for (int t = 0; t < kSimtTokens; ++t) {
            dense[t] += __shfl_xor_sync(0xffffffffu, dense[t], off);
#pragma unroll
            for (int i = 0; i < NM; ++i)
                gate[i][t] += __shfl_xor_sync(0xffffffffu, gate[i][t], off);
        }
    }
    if (lane < nt) {
        float D = 0.f, o = 0.f;
#pragma unroll
        for (int t = 0; t < kSimtTokens; ++t)
            if (t == lane)
                D = dense[t];
        if (NM == 0) {
            o = D;
        } else {
#pragma unroll
            for (int i = 0; i < NM; ++i) {
                float g = 0.f;
#pragma unroll
                for (int t = 0; t < kSimtTokens; ++t)
                    if (t == lane)
                        g = gate[i][t];
                const float wi = mw ? mw[(t0 + lane) * NM + i] : 1.0f;
                o += wi * (act_fn(act & ACT_MASK, (act & GATE_DENSE) ? D : g) * (D - g));
            }
        }
        out[(t0 + lane) * h + j] = o;
    }
}

}  // namespace mglu
