// pack.cuh -- mask bit-packing and unpacking kernels.
//
// Packed format ("Approach" of "Masked Gated Linear Unit": binary masks that
// the fused kernel unpacks; the bit layout is this library's own): weight
// (j, k) owns n_m bits starting at bit (j*d + k)*n_m of a little-endian byte
// stream, bit i = mask i.  With d % 8 == 0 every packed byte holds whole
// weights of one row, so a k-range of a row of W maps to a contiguous byte
// range of the same row of the packed stream.
#pragma once
#include <cstdint>

#include "common.cuh"

namespace mglu {

// One thread writes one 16-byte chunk of the packed stream (128 / NM
// weights, every mask plane read once).  `vec` selects 16-byte loads of the
// mask planes (needs (h*d) % 16 == 0 and a 16-byte aligned `masks`).  The
// last byte may be partial when h*d*NM is not a multiple of 8; its unused
// high bits are written as 0.
template <int NM>
__global__ void __launch_bounds__(256) pack_kernel(const uint8_t *__restrict__ masks, int64_t hd, int64_t nbytes,
                                                   uint8_t *__restrict__ packed, int vec)
{
    constexpr int WPB = 8 / NM;  // weights per packed byte
    const int64_t chunk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t b0 = chunk * 16;
    if (b0 >= nbytes)
        return;
    const int nb = (int)(nbytes - b0 < 16 ? nbytes - b0 : 16);
    const int64_t w0 = b0 * WPB;
    const int nw = (int)(hd - w0 < (int64_t)nb * WPB ? hd - w0 : (int64_t)nb * WPB);
    uint32_t word[4] = {0u, 0u, 0u, 0u};
    if (vec && nb == 16) {
#pragma unroll
        for (int i = 0; i < NM; ++i) {
            const uint4 *plane = reinterpret_cast<const uint4 *>(masks + (int64_t)i * hd + w0);
#pragma unroll
            for (int q = 0; q < 8 / NM; ++q) {  // (128 / NM) weights = 8 / NM loads of 16
                const uint4 v = __ldg(plane + q);
                const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const uint32_t byte = (wv[e >> 2] >> (8 * (e & 3))) & 0xFFu;
                    const int bit = (q * 16 + e) * NM + i;
                    word[bit >> 5] |= (byte != 0u ? 1u : 0u) << (bit & 31);
                }
            }
        }
    } else {
        for (int i = 0; i < NM; ++i) {
            const uint8_t *plane = masks + (int64_t)i * hd + w0;
            for (int w = 0; w < nw; ++w) {
                const int bit = w * NM + i;
                word[bit >> 5] |= (plane[w] != 0 ? 1u : 0u) << (bit & 31);
            }
        }
    }
    if (nb == 16) {
        *reinterpret_cast<uint4 *>(packed + b0) = make_uint4(word[0], word[1], word[2], word[3]);
    } else {
        for (int b = 0; b < nb; ++b)
            packed[b0 + b] = (uint8_t)(word[b >> 2] >> (8 * (b & 3)));
    }
}

// The same packing from FP16 mask logits [NM][h][d] (bit = logit > 0, see
// logit_bit): one thread writes one 16-byte chunk of the packed stream.
// `vec` selects 16-byte loads of the logit planes (needs (h*d) % 8 == 0 and
// a 16-byte aligned `logits`).
template <int NM>
__global__ void __launch_bounds__(256) pack_logits_kernel(const uint16_t *__restrict__ logits, int64_t hd,
                                                          int64_t nbytes, uint8_t *__restrict__ packed, int vec)
{
    constexpr int WPB = 8 / NM;
    const int64_t chunk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t b0 = chunk * 16;
    if (b0 >= nbytes)
        return;
    const int nb = (int)(nbytes - b0 < 16 ? nbytes - b0 : 16);
    const int64_t w0 = b0 * WPB;
    const int nw = (int)(hd - w0 < (int64_t)nb * WPB ? hd - w0 : (int64_t)nb * WPB);
    uint32_t word[4] = {0u, 0u, 0u, 0u};
    if (vec && nb == 16) {
#pragma unroll
        for (int i = 0; i < NM; ++i) {
            const uint4 *plane = reinterpret_cast<const uint4 *>(logits + (int64_t)i * hd + w0);
#pragma unroll
            for (int q = 0; q < 16 / NM; ++q) {  // (128 / NM) logits = 16 / NM loads of 8
                const uint4 v = __ldg(plane + q);
                const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int bit = (q * 8 + e) * NM + i;
                    word[bit >> 5] |= logit_bit((wv[e >> 1] >> (16 * (e & 1))) & 0xFFFFu) << (bit & 31);
                }
            }
        }
    } else {
        for (int i = 0; i < NM; ++i) {
            const uint16_t *plane = logits + (int64_t)i * hd + w0;
            for (int w = 0; w < nw; ++w) {
                const int bit = w * NM + i;
                word[bit >> 5] |= logit_bit(plane[w]) << (bit & 31);
            }
        }
    }
    if (nb == 16) {
        *reinterpret_cast<uint4 *>(packed + b0) = make_uint4(word[0], word[1], word[2], word[3]);
    } else {
        for (int b = 0; b < nb; ++b)
            packed[b0 + b] = (uint8_t)(word[b >> 2] >> (8 * (b & 3)));
    }
}

// Inverse: one thread reads one 16-byte chunk and writes its 128 / NM weights
// in every mask plane as bytes 0 / 1.
template <int NM>
__global__ void __launch_bounds__(256) unpack_kernel(const uint8_t *__restrict__ packed, int64_t hd, int64_t nbytes,
                                                     uint8_t *__restrict__ masks, int vec)
{
    constexpr int WPB = 8 / NM;
    const int64_t chunk = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t b0 = chunk * 16;
    if (b0 >= nbytes)
        return;
    const int nb = (int)(nbytes - b0 < 16 ? nbytes - b0 : 16);
    const int64_t w0 = b0 * WPB;
    const int nw = (int)(hd - w0 < (int64_t)nb * WPB ? hd - w0 : (int64_t)nb * WPB);
    uint32_t word[4] = {0u, 0u, 0u, 0u};
    if (nb == 16) {
        const uint4 v = *reinterpret_cast<const uint4 *>(packed + b0);
        word[0] = v.x;
        word[1] = v.y;
        word[2] = v.z;
        word[3] = v.w;
    } else {
        for (int b = 0; b < nb; ++b)
            word[b >> 2] |= (uint32_t)packed[b0 + b] << (8 * (b & 3));
    }
    if (vec && nb == 16) {
#pragma unroll
        for (int i = 0; i < NM; ++i) {
            uint4 *plane = reinterpret_cast<uint4 *>(masks + (int64_t)i * hd + w0);
#pragma unroll
            for (int q = 0; q < 8 / NM; ++q) {
                uint32_t out[4] = {0u, 0u, 0u, 0u};
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int bit = (q * 16 + e) * NM + i;
                    out[e >> 2] |= ((word[bit >> 5] >> (bit & 31)) & 1u) << (8 * (e & 3));
                }
                plane[q] = make_uint4(out[0], out[1], out[2], out[3]);
            }
        }
    } else {
        for (int i = 0; i < NM; ++i) {
            uint8_t *plane = masks + (int64_t)i * hd + w0;
            for (int w = 0; w < nw; ++w) {
                const int bit = w * NM + i;
                plane[w] = (uint8_t)((word[bit >> 5] >> (bit & 31)) & 1u);
            }
        }
    }
}

}  // namespace mglu
