// decode.cuh -- MGLU up-projection for few tokens (T <= 16), and the dense
// product (NM = 0) used as the decode-time down-projection.
//
// Memory-bound design ("Masked Gated Linear Unit", "Problem" and "Approach":
// decoding is bound by reading the weights, so each weight and its mask bits
// are read once and the masks are unpacked inside the kernel):
//
//  * A CTA owns ROWS = 16 rows of W (16 output columns j) and a contiguous
//    range of k.  When the row block is split along k over a thread-block
//    cluster, partial sums are combined through distributed shared memory.
//  * One producer thread streams stages of KS = 256 k through a ring of
//    shared-memory buffers with TMA: the W tile (4 boxes of 16 x 64 bf16,
//    128-byte swizzle), the matching packed-mask tile (16 rows x KS*NM/8
//    bytes) and the x tile (8*NT tokens x 64 bf16, zero-filled past T).
//  * Four consumer warps each take 64 k of a stage.  A lane loads 8
//    consecutive weights of two rows, turns each mask's bits into bf16x2 lane
//    masks (pair_mask), and feeds W and the NM masked copies of W as the A
//    operand of mma.sync m16n8k16 with the tokens as B.  One dense product D
//    and NM gate products g_i accumulate in fp32; the value of mask i is
//    D - g_i.  The tensor cores only reduce here: the kernel is bound by HBM.
//  * Epilogue: cross-warp and cross-CTA sums in a fixed order, then
//    out = sum_i act(g_i) * (D - g_i) rounded once to bf16.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"

namespace mglu {
namespace dec {

constexpr int ROWS = 16;
constexpr int KS = 256;
constexpr int SUBK = 64;
constexpr int NSUB = KS / SUBK;  // 4
constexpr int NCW = NSUB;        // consumer warps, one sub-tile each
constexpr int NTHREADS = (NCW + 1) * 32;
constexpr int STAGES = 4;

template <int NM, int NT>
struct Layout {
    static constexpr int W_SUB = ROWS * SUBK * 2;   // 2048 B
    static constexpr int X_ROWS = 8 * NT;
    static constexpr int X_SUB = X_ROWS * SUBK * 2;  // 1024 * NT B
    static constexpr int M_ROW = KS * NM / 8;        // mask bytes per row per stage
    static constexpr int M_BYTES = ROWS * M_ROW;
    static constexpr int W_OFF = 0;
    static constexpr int X_OFF = NSUB * W_SUB;
    static constexpr int M_OFF = X_OFF + NSUB * X_SUB;
    static constexpr int STAGE = (M_OFF + M_BYTES + 1023) / 1024 * 1024;
    static constexpr uint32_t TX = NSUB * W_SUB + NSUB * X_SUB + M_BYTES;
    static constexpr int ACC = (NM + 1) * NT * 128;  // floats of one warp's accumulators
    static constexpr int RING = STAGES * STAGE;
    static constexpr int PART_OFF = RING;
    static constexpr int BAR_OFF = PART_OFF + ACC * 4;
    static constexpr int SMEM = BAR_OFF + 2 * STAGES * 8 + 1024;  // + slack for 1024-B alignment
    static_assert(NCW * ACC * 4 <= RING, "cross-warp reduction must fit in the ring");
};

template <int NM, int NT>
__device__ __forceinline__ void load_mask_chunk(const uint8_t *p, uint32_t &lo, uint32_t &hi)
{
    if constexpr (NM == 8) {
        const uint2 v = *reinterpret_cast<const uint2 *>(p);
        lo = v.x;
        hi = v.y;
    } else if constexpr (NM == 4) {
        lo = *reinterpret_cast<const uint32_t *>(p);
        hi = 0;
    } else if constexpr (NM == 2) {
        lo = *reinterpret_cast<const uint16_t *>(p);
        hi = 0;
    } else if constexpr (NM == 1) {
        lo = *p;
        hi = 0;
    } else {
        lo = hi = 0;
    }
}

// Masked copies of the A fragment for mask I, k16 sub-step S.
template <int NM, int S, int I>
__device__ __forceinline__ void masked_fragment(const uint32_t (&wa)[4], const uint32_t (&wb)[4], uint32_t alo,
                                                uint32_t ahi, uint32_t blo, uint32_t bhi, uint32_t (&a)[4])
{
    a[0] = wa[2 * S] & pair_mask<NM, 2 * S, I>(alo, ahi);
    a[1] = wb[2 * S] & pair_mask<NM, 2 * S, I>(blo, bhi);
    a[2] = wa[2 * S + 1] & pair_mask<NM, 2 * S + 1, I>(alo, ahi);
    a[3] = wb[2 * S + 1] & pair_mask<NM, 2 * S + 1, I>(blo, bhi);
}

template <int NM, int NT, int S, int I>
struct MaskLoop {
    static __device__ __forceinline__ void run(float (&acc)[NM + 1][NT][4], const uint32_t (&wa)[4],
                                               const uint32_t (&wb)[4], const uint32_t (&xb)[NT][4],
                                               uint32_t alo, uint32_t ahi, uint32_t blo, uint32_t bhi)
    {
        if constexpr (I < NM) {
            uint32_t a[4];
            masked_fragment<NM, S, I>(wa, wb, alo, ahi, blo, bhi, a);
#pragma unroll
            for (int t = 0; t < NT; ++t)
                mma_bf16_16816(acc[1 + I][t], a[0], a[1], a[2], a[3], xb[t][2 * S], xb[t][2 * S + 1]);
            MaskLoop<NM, NT, S, I + 1>::run(acc, wa, wb, xb, alo, ahi, blo, bhi);
        }
    }
};

// One unit: 16 rows x 32 k.  Lane (g, c) holds weights [8c, 8c+8) of rows g
// and g+8; k16 sub-step S uses its pairs 2S and 2S+1.  The k order inside the
// MMA is a permutation of the physical k that depends only on c and S, so the
// same permutation applied to x (operand B) leaves every sum unchanged.
template <int NM, int NT, int S>
__device__ __forceinline__ void unit_step(float (&acc)[NM + 1][NT][4], const uint32_t (&wa)[4],
                                          const uint32_t (&wb)[4], const uint32_t (&xb)[NT][4], uint32_t alo,
                                          uint32_t ahi, uint32_t blo, uint32_t bhi)
{
#pragma unroll
    for (int t = 0; t < NT; ++t)
        mma_bf16_16816(acc[0][t], wa[2 * S], wb[2 * S], wa[2 * S + 1], wb[2 * S + 1], xb[t][2 * S],
                       xb[t][2 * S + 1]);
    MaskLoop<NM, NT, S, 0>::run(acc, wa, wb, xb, alo, ahi, blo, bhi);
}

template <int NM, int NT>
__global__ void __launch_bounds__(NTHREADS) decode_kernel(const __grid_constant__ CUtensorMap tm_w,
                                                          const __grid_constant__ CUtensorMap tm_x,
                                                          const __grid_constant__ CUtensorMap tm_m, int T,
                                                          int rows, int d, int ksplit, int act,
                                                          __nv_bfloat16 *__restrict__ out)
{
    using L = Layout<NM, NT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::BAR_OFF);
    uint64_t *empty = full + STAGES;
    float *part = reinterpret_cast<float *>(smem + L::PART_OFF);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rb = blockIdx.x / ksplit;
    const int kr = blockIdx.x % ksplit;  // == rank in the cluster when ksplit > 1
    const int row0 = rb * ROWS;
    const int nst = (d + KS - 1) / KS;
    const int st0 = (int)((int64_t)kr * nst / ksplit);
    const int nmy = (int)((int64_t)(kr + 1) * nst / ksplit) - st0;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NCW);
        }
        fence_mbar_init();
    }
    __syncthreads();

    float acc[NM + 1][NT][4];
#pragma unroll
    for (int v = 0; v <= NM; ++v)
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int r = 0; r < 4; ++r)
                acc[v][t][r] = 0.f;

    if (warp == NCW) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            prefetch_tensormap(&tm_w);
            prefetch_tensormap(&tm_x);
            if (NM > 0)
                prefetch_tensormap(&tm_m);
            for (int it = 0; it < nmy; ++it) {
                const int s = it % STAGES;
                const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
                if (!mbar_wait(&empty[s], ph ^ 1u))
                    break;
                uint8_t *st = smem + s * L::STAGE;
                mbar_arrive_expect_tx(&full[s], L::TX);
                const int k0 = (st0 + it) * KS;
#pragma unroll
                for (int sub = 0; sub < NSUB; ++sub) {
                    tma_load_2d(st + L::W_OFF + sub * L::W_SUB, &tm_w, &full[s], k0 + sub * SUBK, row0);
                    tma_load_2d(st + L::X_OFF + sub * L::X_SUB, &tm_x, &full[s], k0 + sub * SUBK, 0);
                }
                if (NM > 0)
                    tma_load_2d(st + L::M_OFF, &tm_m, &full[s], k0 * NM / 8, row0);
            }
        }
    } else {
        // ---------------------------------------------------------- consumers
        const int g = lane >> 2, c = lane & 3;
        for (int it = 0; it < nmy; ++it) {
            const int s = it % STAGES;
            const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
            if (!mbar_wait(&full[s], ph))
                break;
            const uint8_t *st = smem + s * L::STAGE;
            const uint8_t *wsub = st + L::W_OFF + warp * L::W_SUB;
            const uint8_t *xsub = st + L::X_OFF + warp * L::X_SUB;
            const uint8_t *msub = st + L::M_OFF + warp * (SUBK * NM / 8);
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int ch = ((4 * u + c) ^ g) << 4;  // 128-byte swizzle: chunk ^ (row & 7)
                uint32_t wa[4], wb[4], xb[NT][4];
                {
                    const uint4 va = *reinterpret_cast<const uint4 *>(wsub + g * 128 + ch);
                    const uint4 vb = *reinterpret_cast<const uint4 *>(wsub + (g + 8) * 128 + ch);
                    wa[0] = va.x, wa[1] = va.y, wa[2] = va.z, wa[3] = va.w;
                    wb[0] = vb.x, wb[1] = vb.y, wb[2] = vb.z, wb[3] = vb.w;
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        const uint4 vx = *reinterpret_cast<const uint4 *>(xsub + (8 * t + g) * 128 + ch);
                        xb[t][0] = vx.x, xb[t][1] = vx.y, xb[t][2] = vx.z, xb[t][3] = vx.w;
                    }
                }
                uint32_t alo = 0, ahi = 0, blo = 0, bhi = 0;
                if constexpr (NM > 0) {
                    const int mo = (32 * u + 8 * c) * NM / 8;
                    load_mask_chunk<NM, NT>(msub + g * L::M_ROW + mo, alo, ahi);
                    load_mask_chunk<NM, NT>(msub + (g + 8) * L::M_ROW + mo, blo, bhi);
                }
                unit_step<NM, NT, 0>(acc, wa, wb, xb, alo, ahi, blo, bhi);
                unit_step<NM, NT, 1>(acc, wa, wb, xb, alo, ahi, blo, bhi);
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&empty[s]);
        }
    }

    // ------------------------------------------------------------ reductions
    __syncthreads();  // every issued stage was consumed: the ring is free
    float *red = reinterpret_cast<float *>(smem);
    if (warp < NCW) {
#pragma unroll
        for (int v = 0; v <= NM; ++v)
#pragma unroll
            for (int t = 0; t < NT; ++t)
#pragma unroll
                for (int r = 0; r < 4; ++r)
                    red[warp * L::ACC + ((v * NT + t) * 4 + r) * 32 + lane] = acc[v][t][r];
    }
    __syncthreads();
    for (int e = threadIdx.x; e < L::ACC; e += NTHREADS) {
        float sum = 0.f;
#pragma unroll
        for (int w = 0; w < NCW; ++w)
            sum += red[w * L::ACC + e];
        part[e] = sum;
    }
    __syncthreads();
    if (ksplit > 1)
        cluster_sync();
    if (kr == 0) {
        const uint32_t part_addr = smem_u32(part);
        for (int e = threadIdx.x; e < NT * 128; e += NTHREADS) {
            const int t = e >> 7, r = (e >> 5) & 3, ln = e & 31;
            const int row = (ln >> 2) + 8 * (r >> 1);
            const int tok = 8 * t + 2 * (ln & 3) + (r & 1);
            float vals[NM + 1];
#pragma unroll
            for (int v = 0; v <= NM; ++v) {
                const int idx = ((v * NT + t) * 4 + r) * 32 + ln;
                float sum = part[idx];
                for (int q = 1; q < ksplit; ++q) {
                    float pv;
                    asm volatile("ld.shared::cluster.f32 %0, [%1];"
                                 : "=f"(pv)
                                 : "r"(mapa_shared(part_addr + idx * 4, (uint32_t)q))
                                 : "memory");
                    sum += pv;
                }
                vals[v] = sum;
            }
            if (row0 + row < rows && tok < T) {
                float o;
                if constexpr (NM == 0) {
                    o = vals[0];
                } else {
                    o = 0.f;
#pragma unroll
                    for (int i = 0; i < NM; ++i)
                        o += act_fn(act, vals[1 + i]) * (vals[0] - vals[1 + i]);
                }
                out[(int64_t)tok * rows + row0 + row] = __float2bfloat16_rn(o);
            }
        }
    }
    if (ksplit > 1)
        cluster_sync();  // peers keep their partials alive until rank 0 has read them
}

}  // namespace dec
}  // namespace mglu
