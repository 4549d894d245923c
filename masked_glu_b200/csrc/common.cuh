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
// Flag OR-ed into act: the dense-gate ablation ("Masked Gated Linear Unit",
// "Measured effects", last row, "Remove the gate mask (dense gate)"): every
// gate is the whole product x W, each value keeps its mask.
enum { GATE_DENSE = 16, ACT_MASK = 15 };

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

// Its derivative, for the training path: Swish sigma(z) + z sigma(z) (1 -
// sigma(z)); GELU Phi(z) + z phi(z); ReLU 1 for z > 0, else 0 (the subgradient
// 0 at 0).
__device__ __forceinline__ float act_grad_fn(int act, float z)
{
    if (act == ACT_SWISH) {
        const float s = __fdividef(1.0f, 1.0f + __expf(-z));
        return s + z * s * (1.0f - s);
    }
    if (act == ACT_GELU)
        return 0.5f * (1.0f + erff(z * 0.70710678118654752440f)) + z * 0.39894228040143267794f * __expf(-0.5f * z * z);
    return z > 0.0f ? 1.0f : 0.0f;
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

// ---------------------------------------------------------------- mask logits
// Mask bit of an IEEE binary16 mask logit ("Masked Gated Linear Unit",
// "Limitations": masks are held as FP16 logits while training): 1 where the
// logit is greater than zero, i.e. for the bit patterns 0x0001 (the smallest
// subnormal) through 0x7C00 (+infinity); +0, -0, every negative value and
// every NaN give 0.
MGLU_HD uint32_t logit_bit(uint32_t h16) { return ((h16 - 1u) & 0xFFFFu) < 0x7C00u ? 1u : 0u; }

// ---------------------------------------------------------------- sign flips
// The decode kernel applies mask i to a bf16 pair by flipping signs: it
// accumulates h_i = x (S_i . W) with S_i = +1 where mask i is set and -1
// where it is clear, so g_i = (D + h_i) / 2 and v_i = (D - h_i) / 2 with the
// dense product D = x W.  One LOP3 per pair and mask builds the operand.
//
// group_bits<NM, S>: the mask bits of weights 4S .. 4S+3 of an 8-weight
// chunk (lo/hi as for pair_mask), rearranged so that mask I of weight 4S
// sits at bit I, of weight 4S+2 at bit 8+I, of weight 4S+1 at bit 16+I and
// of weight 4S+3 at bit 24+I.  Shifting the result left by 15-I then puts
// mask I of the pair (4S, 4S+1) at bits 15 and 31 (the pair's sign bits),
// shifting by 7-I does so for the pair (4S+2, 4S+3).
template <int NM, int S>
MGLU_HD uint32_t group_bits(uint32_t lo, uint32_t hi)
{
    static_assert(S == 0 || S == 1, "two groups of four weights per chunk");
    if constexpr (NM == 8) {
        // one byte per weight: bytes [b0 b1 b2 b3] -> [b0 b2 b1 b3]
        return prmt_any(S == 0 ? lo : hi, 0u, 0x3120u);
    } else {
        uint32_t n = lo;  // one nibble per weight, weight w in nibble w
        if constexpr (NM == 2) {
            // 2-bit fields -> nibbles
            n = (n | (n << 8)) & 0x00FF00FFu;
            n = (n | (n << 4)) & 0x0F0F0F0Fu;
            n = (n | (n << 2)) & 0x33333333u;
        } else if constexpr (NM == 1) {
            // bits -> nibbles
            n = (n | (n << 12)) & 0x000F000Fu;
            n = (n | (n << 6)) & 0x03030303u;
            n = (n | (n << 3)) & 0x11111111u;
        }
        const uint32_t even = n & 0x0F0F0F0Fu;         // weights 0 2 4 6, one per byte
        const uint32_t odd = (n >> 4) & 0x0F0F0F0Fu;   // weights 1 3 5 7
        return prmt_any(even, odd, S == 0 ? 0x5410u : 0x7632u);
    }
}

// A bf16 pair with the sign of each half flipped where the matching bit of
// m (bit 15 for the low half, bit 31 for the high half) is clear.
MGLU_HD uint32_t flip_pair(uint32_t w, uint32_t m) { return w ^ (~m & 0x80008000u); }

}  // namespace mglu
