// common.cuh -- pieces shared by the MGLU kernels: the gating activation and
// the expansion of packed mask bits into bf16x2 lane masks.
#pragma once
#include <cstdint>

#ifdef __CUDACC__
#define MGLU_HD __host__ __device__ __forceinline__
#else
#define MGLU_HD inline
#endif

namespace mglu {

enum { ACT_SWISH = 0, ACT_GELU = 1, ACT_RELU = 2 };

#ifdef __CUDACC__
// Gating activation ("Masked Gated Linear Unit", "Measured effects": Swish
// for SwiMGLU; GELU and ReLU as the ablation variants).  Swish uses beta = 1;
// GELU is the exact form z * Phi(z) with CUDA's erff.
__device__ __forceinline__ float act_fn(int act, float z)
{
    if (act == ACT_SWISH)
        return __fdividef(z, 1.0f + __expf(-z));
    if (act == ACT_GELU)
        return 0.5f * z * (1.0f + erff(z * 0.70710678118654752440f));
    return fmaxf(z, 0.0f);
}
#endif

// prmt in default mode; on the host an emulation of the PTX definition so the
// lane-mask expansion below can be checked without a GPU.
MGLU_HD uint32_t prmt_any(uint32_t a, uint32_t b, uint32_t sel)
{
#if defined(__CUDA_ARCH__)
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
#else
    const uint64_t src = (uint64_t)a | ((uint64_t)b << 32);
    uint32_t d = 0;
    for (int n = 0; n < 4; ++n) {
        const uint32_t s = (sel >> (4 * n)) & 0xF;
        uint32_t byte = (uint32_t)(src >> (8 * (s & 7))) & 0xFF;
        if (s & 8)
            byte = (byte & 0x80) ? 0xFF : 0x00;
        d |= byte << (8 * n);
    }
    return d;
#endif
}

// Lane mask for one bf16x2 register of W.
//
// An 8-weight chunk of one row of W (16 bytes) owns NM*8 consecutive mask
// bits in the packed format: bit (w*NM + i) is mask i of weight w of the
// chunk, w = 0..7, counted from the least significant bit of the chunk's
// first mask byte.  `lo` holds mask bytes 0..3 of the chunk (little endian),
// `hi` bytes 4..7 (used only when NM = 8).
//
// Register Q (0..3) of the chunk holds weights 2Q (low half) and 2Q+1 (high
// half).  The result is 0xFFFF in each half whose weight has mask I set, else
// 0x0000, so `reg & pair_mask` keeps exactly the weights in the gate of mask
// I.  Each bit is shifted to bit 7 of its byte and prmt's sign-replicate
// selector copies it across the byte pair: two shifts and one prmt.
template <int NM, int Q, int I>
MGLU_HD uint32_t pair_mask(uint32_t lo, uint32_t hi)
{
    constexpr int p0 = (2 * Q) * NM + I;      // bit of weight 2Q
    constexpr int p1 = (2 * Q + 1) * NM + I;  // bit of weight 2Q+1
    constexpr int byte0 = p0 / 8, byte1 = p1 / 8;
    constexpr int sh0 = 7 - (p0 % 8), sh1 = 7 - (p1 % 8);
    const uint32_t v0 = (byte0 < 4 ? lo : hi) << sh0;
    const uint32_t v1 = (byte1 < 4 ? lo : hi) << sh1;
    constexpr uint32_t s0 = 0x8u | (uint32_t)(byte0 & 3);  // sign of a byte of v0 (first operand)
    constexpr uint32_t s1 = 0xCu | (uint32_t)(byte1 & 3);  // sign of a byte of v1 (second operand)
    constexpr uint32_t sel = s0 | (s0 << 4) | (s1 << 8) | (s1 << 12);
    return prmt_any(v0, v1, sel);
}

}  // namespace mglu
