// decode.cuh -- MGLU up-projection for few tokens (T <= 16), and the dense
// product (NM = 0) used as the decode-time down-projection.
//
// Memory-bound design ("Masked Gated Linear Unit", "Problem" and "Approach":
// decoding is bound by reading the weights, so each weight and its mask bits
// are read exactly once and the masks are unpacked inside the kernel):
//
//  * Work is the flattened list of units (row block of ROWS = 16 rows of W,
//    k-stage of KS = 256).  A persistent grid (one or two CTAs per SM) gives
//    every CTA an equal contiguous share of the list, so all SMs stream the
//    same number of bytes and finish together.
//  * One producer thread streams the CTA's units through a deep ring of
//    shared-memory stages with TMA, without pausing at row-block boundaries:
//    the W tile (4 boxes of 16 x 64 bf16, 128-byte swizzle), the packed-mask
//    tile of the same rows and k (128- or 64-byte swizzle) and the x tile
//    (8*NT tokens x 64 bf16, zero-filled past T).
//  * Eight consumer warps each take 32 k of a stage.  A lane loads 8
//    consecutive weights of two rows, turns each mask's bits into bf16x2 lane
//    masks (pair_mask: two shifts and one prmt per register) and feeds W and
//    the NM masked copies of W as the A operand of mma.sync m16n8k16, with
//    the tokens as B.  One dense product D and NM gate products g_i
//    accumulate in fp32; the value of mask i is D - g_i.  The tensor cores
//    only do the k reduction here; HBM bandwidth bounds the kernel.
//  * At the end of a row block the eight warps reduce through shared memory
//    (fixed tree order).  A row block whose k range lies inside one CTA is
//    finished there: out = sum_i act(g_i) (D - g_i), rounded once to bf16.
//    A row block split between CTAs (at most at the two ends of a CTA's
//    share) is finished by whichever of its CTAs arrives last: the others'
//    partial sums come from a small global workspace, added in CTA order, so
//    the result does not depend on arrival order.  The arrival counter is
//    reset by the finishing CTA, leaving the workspace zeroed.
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
constexpr int NSUB = KS / SUBK;  // 4 W / x boxes per stage
constexpr int NCW = 8;           // consumer warps: one 32-k unit of a stage each
constexpr int NTHREADS = (NCW + 1) * 32;
constexpr int MAX_CTAS = 320;    // grid cap; sizes the split-row-block workspace
constexpr int BAR_CONSUMERS = 1; // named barrier id for the consumer warps

template <int NM, int NT>
struct Layout {
    static constexpr int CPS = (NT == 1 && NM < 8) ? 2 : 1;  // CTAs per SM (register budget)
    static constexpr int W_SUB = ROWS * SUBK * 2;     // 2048 B
    static constexpr int X_SUB = 8 * NT * SUBK * 2;   // 1024 * NT B
    static constexpr int M_ROW = KS * NM / 8;         // mask bytes of one row per stage
    static constexpr int M_BOX = M_ROW > 128 ? 128 : M_ROW;  // inner bytes of one mask box
    static constexpr int M_NBOX = NM == 0 ? 0 : M_ROW / M_BOX;
    static constexpr int M_BOXB = (ROWS * M_BOX + 1023) / 1024 * 1024;
    static constexpr int W_OFF = 0;
    static constexpr int X_OFF = NSUB * W_SUB;
    static constexpr int M_OFF = X_OFF + NSUB * X_SUB;
    static constexpr int STAGE = M_OFF + M_NBOX * M_BOXB;
    static constexpr uint32_t TX = NSUB * W_SUB + NSUB * X_SUB + M_NBOX * ROWS * M_BOX;
    static constexpr int ACC = (NM + 1) * NT * 128;   // floats of one warp's accumulators
    static constexpr int RED_OFF_BYTES = 0;
    static constexpr int BUDGET = CPS == 2 ? 110 * 1024 : 214 * 1024;
    static constexpr int RED = 4 * ACC * 4;           // four reduction slots
    static constexpr int STAGES_FIT = (BUDGET - RED - 1024 - 256) / STAGE;
    static constexpr int STAGES = STAGES_FIT > 12 ? 12 : STAGES_FIT;
    static constexpr int RING = STAGES * STAGE;
    static constexpr int RED_OFF = RING;
    static constexpr int BAR_OFF = RED_OFF + RED;
    static constexpr int SMEM = BAR_OFF + 2 * STAGES * 8 + 1024;
    static_assert(STAGES >= 3, "ring too shallow");
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

// Swizzled byte offset inside a mask box with inner size M_BOX bytes.
template <int M_BOX>
__device__ __forceinline__ int mask_swz(int row, int o)
{
    if constexpr (M_BOX == 128)
        return row * 128 + ((((o >> 4) ^ (row & 7)) << 4) | (o & 15));
    else if constexpr (M_BOX == 64)
        return row * 64 + ((((o >> 4) ^ ((row >> 1) & 3)) << 4) | (o & 15));
    else
        return row * M_BOX + o;
}

template <int M_BOX>
constexpr CUtensorMapSwizzle mask_swizzle_mode()
{
    return M_BOX == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : M_BOX == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                                                   : CU_TENSOR_MAP_SWIZZLE_NONE;
}

template <int NM>
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

template <int NM, int NT, int S, int I>
struct MaskLoop {
    static __device__ __forceinline__ void run(float (&acc)[NM + 1][NT][4], const uint32_t (&wa)[4],
                                               const uint32_t (&wb)[4], const uint32_t (&xb)[NT][4],
                                               uint32_t alo, uint32_t ahi, uint32_t blo, uint32_t bhi)
    {
        if constexpr (I < NM) {
            const uint32_t a0 = wa[2 * S] & pair_mask<NM, 2 * S, I>(alo, ahi);
            const uint32_t a1 = wb[2 * S] & pair_mask<NM, 2 * S, I>(blo, bhi);
            const uint32_t a2 = wa[2 * S + 1] & pair_mask<NM, 2 * S + 1, I>(alo, ahi);
            const uint32_t a3 = wb[2 * S + 1] & pair_mask<NM, 2 * S + 1, I>(blo, bhi);
#pragma unroll
            for (int t = 0; t < NT; ++t)
                mma_bf16_16816(acc[1 + I][t], a0, a1, a2, a3, xb[t][2 * S], xb[t][2 * S + 1]);
            MaskLoop<NM, NT, S, I + 1>::run(acc, wa, wb, xb, alo, ahi, blo, bhi);
        }
    }
};

// One 16-row x 32-k unit.  Lane (g, c) holds weights [8c, 8c+8) of rows g
// and g+8; k16 sub-step S uses its bf16 pairs 2S and 2S+1.  The k order
// inside the MMA is a permutation of the physical k that depends only on c
// and S; x (operand B) is loaded with the same permutation, so every sum is
// unchanged.
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

__device__ __forceinline__ void consumer_bar() { asm volatile("bar.sync %0, %1;" ::"n"(BAR_CONSUMERS), "n"(NCW * 32) : "memory"); }

// CTA whose share contains unit u (shares are [c*U/G, (c+1)*U/G)).
__device__ __forceinline__ int cta_of(int64_t u, int64_t U, int G) { return (int)(((u + 1) * G + U - 1) / U) - 1; }
__device__ __forceinline__ int64_t share_begin(int c, int64_t U, int G) { return (int64_t)c * U / G; }

template <int NM, int NT>
__device__ __forceinline__ float out_value(int act, const float (&acc)[NM + 1][NT][4], int t, int r)
{
    if constexpr (NM == 0) {
        return acc[0][t][r];
    } else {
        const float D = acc[0][t][r];
        float o = 0.f;
#pragma unroll
        for (int i = 0; i < NM; ++i)
            o += act_fn(act, acc[1 + i][t][r]) * (D - acc[1 + i][t][r]);
        return o;
    }
}

// Workspace (global, caller-provided): partial sums of split row blocks, two
// slots per CTA (first and last row block of its share), then one arrival
// counter per row block.  Counters must be zero on entry and are zero again
// when the kernel completes.
template <int NM, int NT>
__global__ void __launch_bounds__(NTHREADS, Layout<NM, NT>::CPS) decode_kernel(const __grid_constant__ CUtensorMap tm_w,
                                                             const __grid_constant__ CUtensorMap tm_x,
                                                             const __grid_constant__ CUtensorMap tm_m, int T,
                                                             int rows, int d, int act, float *__restrict__ ws_part,
                                                             int *__restrict__ ws_count,
                                                             __nv_bfloat16 *__restrict__ out)
{
    using L = Layout<NM, NT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::BAR_OFF);
    uint64_t *empty = full + L::STAGES;
    float *red = reinterpret_cast<float *>(smem + L::RED_OFF);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int G = gridDim.x;
    const int nst = (d + KS - 1) / KS;
    const int64_t RB = (rows + ROWS - 1) / ROWS;
    const int64_t U = RB * nst;
    const int64_t u_begin = share_begin(blockIdx.x, U, G);
    const int64_t u_end = share_begin(blockIdx.x + 1, U, G);

    if (threadIdx.x == 0) {
        for (int s = 0; s < L::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], NCW);
        }
        fence_mbar_init();
    }
    __syncthreads();
    if (u_begin >= u_end)
        return;

    if (warp == NCW) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            prefetch_tensormap(&tm_w);
            prefetch_tensormap(&tm_x);
            if (NM > 0)
                prefetch_tensormap(&tm_m);
            int it = 0;
            for (int64_t u = u_begin; u < u_end; ++u, ++it) {
                const int s = it % L::STAGES;
                const uint32_t ph = (uint32_t)(it / L::STAGES) & 1u;
                if (!mbar_wait(&empty[s], ph ^ 1u))
                    break;
                const int row0 = (int)(u / nst) * ROWS;
                const int k0 = (int)(u % nst) * KS;
                uint8_t *st = smem + s * L::STAGE;
                mbar_arrive_expect_tx(&full[s], L::TX);
#pragma unroll
                for (int sub = 0; sub < NSUB; ++sub) {
                    tma_load_2d(st + L::W_OFF + sub * L::W_SUB, &tm_w, &full[s], k0 + sub * SUBK, row0);
                    tma_load_2d(st + L::X_OFF + sub * L::X_SUB, &tm_x, &full[s], k0 + sub * SUBK, 0);
                }
#pragma unroll
                for (int b = 0; b < L::M_NBOX; ++b)
                    tma_load_2d(st + L::M_OFF + b * L::M_BOXB, &tm_m, &full[s], k0 * NM / 8 + b * L::M_BOX, row0);
            }
        }
        return;
    }

    // -------------------------------------------------------------- consumers
    const int g = lane >> 2, c = lane & 3;
    const int sub = warp >> 1, uu = warp & 1;
    const int ch = ((4 * uu + c) ^ g) << 4;  // 128-byte swizzle: 16-byte chunk ^ (row & 7)
    // this warp's 32 k inside the stage, as a byte offset into the stage's mask rows
    const int mo = (warp * 32 + 8 * c) * NM / 8;
    const int mbox = NM > 0 ? mo / L::M_BOX : 0;
    const int mo_in = NM > 0 ? mo % L::M_BOX : 0;
    const int moff_a = mask_swz<L::M_BOX>(g, mo_in);
    const int moff_b = mask_swz<L::M_BOX>(g + 8, mo_in);

    float acc[NM + 1][NT][4];
#pragma unroll
    for (int v = 0; v <= NM; ++v)
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int r = 0; r < 4; ++r)
                acc[v][t][r] = 0.f;

    // A timed-out wait (status recorded by mbar_wait) stops the waiting and
    // the math, but every warp still runs the same sequence of named
    // barriers, so no warp can be left waiting at one.
    bool ok = true;
    int it = 0;
    for (int64_t u = u_begin; u < u_end; ++u, ++it) {
        const int s = it % L::STAGES;
        const uint32_t ph = (uint32_t)(it / L::STAGES) & 1u;
        if (ok && !mbar_wait(&full[s], ph))
            ok = false;
        if (ok) {
            const uint8_t *st = smem + s * L::STAGE;
            const uint8_t *wsub = st + L::W_OFF + sub * L::W_SUB;
            const uint8_t *xsub = st + L::X_OFF + sub * L::X_SUB;
            uint32_t wa[4], wb[4], xb[NT][4];
            const uint4 va = *reinterpret_cast<const uint4 *>(wsub + g * 128 + ch);
            const uint4 vb = *reinterpret_cast<const uint4 *>(wsub + (g + 8) * 128 + ch);
            wa[0] = va.x, wa[1] = va.y, wa[2] = va.z, wa[3] = va.w;
            wb[0] = vb.x, wb[1] = vb.y, wb[2] = vb.z, wb[3] = vb.w;
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const uint4 vx = *reinterpret_cast<const uint4 *>(xsub + (8 * t + g) * 128 + ch);
                xb[t][0] = vx.x, xb[t][1] = vx.y, xb[t][2] = vx.z, xb[t][3] = vx.w;
            }
            uint32_t alo = 0, ahi = 0, blo = 0, bhi = 0;
            if constexpr (NM > 0) {
                const uint8_t *mb = st + L::M_OFF + mbox * L::M_BOXB;
                load_mask_chunk<NM>(mb + moff_a, alo, ahi);
                load_mask_chunk<NM>(mb + moff_b, blo, bhi);
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&empty[s]);  // operands are in registers: the stage can be refilled
            unit_step<NM, NT, 0>(acc, wa, wb, xb, alo, ahi, blo, bhi);
            unit_step<NM, NT, 1>(acc, wa, wb, xb, alo, ahi, blo, bhi);
        }

        const int ks = (int)(u % nst);
        if (ks != nst - 1 && u != u_end - 1)
            continue;

        // ---------------------------------------------------- row block done here
        const int64_t rb = u / nst;
        // tree reduction of the 8 warps' accumulators into warp 0 (fixed order)
        float *slot = red + (warp & 3) * L::ACC;
        if (warp >= 4) {
#pragma unroll
            for (int v = 0; v <= NM; ++v)
#pragma unroll
                for (int t = 0; t < NT; ++t)
                    *reinterpret_cast<float4 *>(slot + ((v * NT + t) * 32 + lane) * 4) =
                        make_float4(acc[v][t][0], acc[v][t][1], acc[v][t][2], acc[v][t][3]);
        }
        consumer_bar();
        if (warp < 4) {
#pragma unroll
            for (int v = 0; v <= NM; ++v)
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    const float4 o = *reinterpret_cast<const float4 *>(slot + ((v * NT + t) * 32 + lane) * 4);
                    acc[v][t][0] += o.x, acc[v][t][1] += o.y, acc[v][t][2] += o.z, acc[v][t][3] += o.w;
                }
        }
        consumer_bar();
        if (warp >= 1 && warp < 4) {
#pragma unroll
            for (int v = 0; v <= NM; ++v)
#pragma unroll
                for (int t = 0; t < NT; ++t)
                    *reinterpret_cast<float4 *>(slot + ((v * NT + t) * 32 + lane) * 4) =
                        make_float4(acc[v][t][0], acc[v][t][1], acc[v][t][2], acc[v][t][3]);
        }
        consumer_bar();
        if (warp == 0) {
#pragma unroll
            for (int q = 1; q < 4; ++q)
#pragma unroll
                for (int v = 0; v <= NM; ++v)
#pragma unroll
                    for (int t = 0; t < NT; ++t) {
                        const float4 o =
                            *reinterpret_cast<const float4 *>(red + q * L::ACC + ((v * NT + t) * 32 + lane) * 4);
                        acc[v][t][0] += o.x, acc[v][t][1] += o.y, acc[v][t][2] += o.z, acc[v][t][3] += o.w;
                    }
        }
        consumer_bar();

        if (warp == 0 && ok) {
            const int c_first = cta_of(rb * nst, U, G);
            const int c_last = cta_of(rb * nst + nst - 1, U, G);
            bool finish = true;
            if (c_first != c_last) {
                // split row block: publish this CTA's partial, the last arriver finishes
                const int my_slot = 2 * blockIdx.x + (rb == share_begin(blockIdx.x, U, G) / nst ? 0 : 1);
                float *mine = ws_part + (int64_t)my_slot * L::ACC;
#pragma unroll
                for (int v = 0; v <= NM; ++v)
#pragma unroll
                    for (int t = 0; t < NT; ++t)
                        __stcg(reinterpret_cast<float4 *>(mine + ((v * NT + t) * 32 + lane) * 4),
                               make_float4(acc[v][t][0], acc[v][t][1], acc[v][t][2], acc[v][t][3]));
                __threadfence();
                __syncwarp();
                int prev = 0;
                if (lane == 0)
                    prev = atomicAdd(ws_count + rb, 1);
                prev = __shfl_sync(0xffffffffu, prev, 0);
                finish = prev == c_last - c_first;
                if (finish) {
                    // every partial, this CTA's included, read back in CTA order
                    __threadfence();
#pragma unroll
                    for (int v = 0; v <= NM; ++v)
#pragma unroll
                        for (int t = 0; t < NT; ++t)
#pragma unroll
                            for (int r = 0; r < 4; ++r)
                                acc[v][t][r] = 0.f;
                    for (int cc = c_first; cc <= c_last; ++cc) {
                        const int sl = 2 * cc + (rb == share_begin(cc, U, G) / nst ? 0 : 1);
                        const float *p = ws_part + (int64_t)sl * L::ACC;
#pragma unroll
                        for (int v = 0; v <= NM; ++v)
#pragma unroll
                            for (int t = 0; t < NT; ++t) {
                                const float4 o = __ldcg(reinterpret_cast<const float4 *>(p + ((v * NT + t) * 32 + lane) * 4));
                                acc[v][t][0] += o.x, acc[v][t][1] += o.y, acc[v][t][2] += o.z, acc[v][t][3] += o.w;
                            }
                    }
                    if (lane == 0)
                        ws_count[rb] = 0;  // leave the workspace zeroed for the next call
                }
            }
            if (finish) {
                const int row0 = (int)rb * ROWS;
#pragma unroll
                for (int t = 0; t < NT; ++t)
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const int row = g + 8 * (r >> 1);
                        const int tok = 8 * t + 2 * c + (r & 1);
                        if (row0 + row < rows && tok < T)
                            out[(int64_t)tok * rows + row0 + row] = __float2bfloat16_rn(out_value<NM, NT>(act, acc, t, r));
                    }
            }
        }
#pragma unroll
        for (int v = 0; v <= NM; ++v)
#pragma unroll
            for (int t = 0; t < NT; ++t)
#pragma unroll
                for (int r = 0; r < 4; ++r)
                    acc[v][t][r] = 0.f;
    }
}

// Workspace bytes of the decode kernel: partial slots for the largest grid,
// then one counter per row block of `rows` (256-byte aligned pieces).
__host__ __device__ constexpr int64_t part_bytes() { return (int64_t)2 * MAX_CTAS * 9 * 2 * 128 * 4; }
__host__ __device__ constexpr int64_t workspace_bytes(int64_t rows)
{
    return part_bytes() + ((rows + ROWS - 1) / ROWS * 4 + 255) / 256 * 256;
}

}  // namespace dec
}  // namespace mglu
