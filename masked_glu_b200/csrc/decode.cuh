// decode.cuh -- MGLU up-projection for few tokens (T <= 16), and the dense
// product (NM = 0) used as the decode-time down-projection.
//
// Memory-bound design ("Masked Gated Linear Unit", "Problem" and "Approach":
// decoding is bound by reading the weights, so each weight and its mask bits
// are read exactly once and the masks are unpacked inside the kernel):
//
//  * Work is made of units (row block of ROWS = 16 rows of W, k-stage of
//    KS = 512 (256 for 9..16 tokens)).  A persistent grid of one CTA per SM
//    splits it evenly: every CTA gets the same number of whole row blocks
//    (data-parallel part) plus an equal contiguous share of the units of the
//    remaining row blocks (stream-K part), so all SMs stream the same number
//    of bytes.  Each CTA does its stream-K share first, so the combining of
//    row blocks split between CTAs overlaps the data-parallel part instead of
//    trailing the kernel.
//  * A producer warp streams the CTA's share through a deep ring of
//    shared-memory stages with three TMA loads per stage, issued together by
//    three lanes: the W tile (16 rows x KS, as KS/64 boxes of 64 k with the
//    128-byte swizzle), the x tile (the T token rows x KS) and
//    the packed-mask tile of the same rows and k.  It does not pause at
//    row-block boundaries.
//  * Sixteen consumer warps (eight for 9..16 tokens) each take 32 k of a stage.  A lane loads 8
//    consecutive weights of two rows, turns each mask's bits into bf16x2 lane
//    masks (pair_mask: two shifts and one prmt per register) and feeds W and
//    the NM masked copies of W as the A operand of mma.sync m16n8k16, with
//    the tokens as B.  One dense product D and NM gate products g_i
//    accumulate in fp32; the value of mask i is D - g_i.  The tensor cores
//    only do the k reduction here; HBM bandwidth bounds the kernel.
//  * At the end of a row block the consumers drop their accumulators into
//    shared-memory slots and carry on; a finisher warp adds the slots in a
//    fixed order.  A row block whose k range lies inside one CTA is
//    finished there: out = sum_i act(g_i) (D - g_i), rounded once to bf16.
//    A row block split between CTAs (only at the two ends of a stream-K
//    share) is finished by whichever of its CTAs arrives last: the others' partial
//    sums come from a small global scratch, added in CTA order, so the result
//    does not depend on arrival order.  The arrival counter is reset by the
//    finishing CTA, leaving the scratch zeroed.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"

namespace mglu {
namespace dec {

constexpr int ROWS = 16;
constexpr int MAX_CTAS = 320;         // grid cap; sizes the split-row-block scratch
constexpr int BAR_SLOTS_FULL = 1;     // consumers arrive, finisher waits
constexpr int BAR_SLOTS_FREE = 2;     // finisher arrives, consumers wait
constexpr int MASK_K = 128;           // k covered by one row of a mask box

template <int NM, int NT>
struct Layout {
    // consumer warps: as many as the register file allows (a quadrant holds
    // 16K registers, so 4 warps of 128 or 5 of 96 registers)
    static constexpr int NCW = NT == 2 ? 8 : NM == 8 ? 12 : 16;
    static constexpr int PRODUCER_WARP = NCW;
    static constexpr int FINISHER_WARP = NCW + 1;
    static constexpr int NTHREADS = (NCW + 2) * 32;
    static constexpr int BAR_COUNT = (NCW + 1) * 32;   // consumers + finisher
    static constexpr int KS = NCW * 32;                // k per stage: 32 per consumer warp
    static constexpr int NKC = KS / 64;                // 64-k chunks per stage
    static constexpr int XR = 8 * NT;                  // token rows of the x tile
    static constexpr int W_CHUNK = ROWS * 128;         // bytes of one 16 x 64 bf16 chunk
    static constexpr int X_CHUNK = XR * 128;
    static constexpr int M_BOX = 16 * NM;              // bytes of one row of a mask box (128 k)
    static constexpr int M_CHUNKS = KS / MASK_K;
    static constexpr int W_OFF = 0;
    static constexpr int X_OFF = NKC * W_CHUNK;
    static constexpr int M_OFF = X_OFF + NKC * X_CHUNK;
    static constexpr int M_BYTES = NM == 0 ? 0 : M_CHUNKS * ROWS * M_BOX;
    static constexpr int STAGE = (M_OFF + M_BYTES + 1023) / 1024 * 1024;
    // bytes one stage receives when the x box has xr token rows
    static __device__ __forceinline__ uint32_t tx(int xr) { return (uint32_t)(NKC * W_CHUNK + NKC * xr * 128 + M_BYTES); }
    static constexpr int ACC = (NM + 1) * NT * 128;    // floats of one warp's accumulators
    static constexpr int SLOTS = NCW * ACC * 4;
    static constexpr int BUDGET = 220 * 1024;
    static constexpr int STAGES_FIT = (BUDGET - SLOTS - 1024 - 256) / STAGE;
    static constexpr int STAGES = STAGES_FIT > 12 ? 12 : STAGES_FIT;
    static constexpr int SLOT_OFF = STAGES * STAGE;
    static constexpr int BAR_OFF = SLOT_OFF + SLOTS;
    static constexpr int SMEM = BAR_OFF + 2 * STAGES * 8 + 1024;
    static_assert(STAGES >= 3, "ring too shallow");
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

// Byte offset of (row, o) inside one mask box (rows of M_BOX bytes) under the
// swizzle the tensor map uses for that width.
template <int M_BOX>
__device__ __forceinline__ int mask_swz(int row, int o)
{
    if constexpr (M_BOX == 128)
        return row * 128 + ((((o >> 4) ^ (row & 7)) << 4) | (o & 15));
    else if constexpr (M_BOX == 64)
        return row * 64 + ((((o >> 4) ^ ((row >> 1) & 3)) << 4) | (o & 15));
    else if constexpr (M_BOX == 32)
        return row * 32 + ((((o >> 4) ^ ((row >> 2) & 1)) << 4) | (o & 15));
    else
        return row * M_BOX + o;
}

template <int M_BOX>
constexpr CUtensorMapSwizzle mask_swizzle_mode()
{
    return M_BOX == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
         : M_BOX == 64  ? CU_TENSOR_MAP_SWIZZLE_64B
         : M_BOX == 32  ? CU_TENSOR_MAP_SWIZZLE_32B
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

__device__ __forceinline__ uint32_t hmul2_bf16(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

template <int S>
__device__ __forceinline__ uint32_t shift_signed(uint32_t v)
{
    if constexpr (S >= 0)
        return v << S;
    else
        return v >> (-S);
}

// n_m = 8 path.  The ALU pipe is the scarce one here, so masks are applied
// with a bf16 multiply on the FMA pipe: the chunk's mask bytes are reordered
// [w0 w2 w1 w3] so the bits of mask I for the weight pair (w0, w1) sit at I
// and I+16 (pair (w2, w3): I+8 and I+24); one shift moves mask I to the
// exponent MSBs 14/30 and mask I-1 to 13/29 of the two bf16 halves, and an
// AND leaves 2.0 (bit 14), 2^-63 (bit 13) or 0 per half.  Multiplying W by it
// is exact, so mask 2P+1 accumulates 2*g and mask 2P accumulates 2^-63*g;
// out_value undoes the powers of two.
template <int NT, int S, int P>
struct ExpMaskLoop {
    static __device__ __forceinline__ void run(float (&acc)[9][NT][4], const uint32_t (&wa)[4],
                                               const uint32_t (&wb)[4], const uint32_t (&xb)[NT][4], uint32_t ra,
                                               uint32_t rb)
    {
        if constexpr (P < 4) {
            constexpr int I = 2 * P + 1;
            const uint32_t ae = shift_signed<14 - I>(ra), ao = shift_signed<6 - I>(ra);
            const uint32_t be = shift_signed<14 - I>(rb), bo = shift_signed<6 - I>(rb);
            {
                const uint32_t a0 = hmul2_bf16(wa[2 * S], ae & 0x40004000u);
                const uint32_t a1 = hmul2_bf16(wb[2 * S], be & 0x40004000u);
                const uint32_t a2 = hmul2_bf16(wa[2 * S + 1], ao & 0x40004000u);
                const uint32_t a3 = hmul2_bf16(wb[2 * S + 1], bo & 0x40004000u);
#pragma unroll
                for (int t = 0; t < NT; ++t)
                    mma_bf16_16816(acc[1 + I][t], a0, a1, a2, a3, xb[t][2 * S], xb[t][2 * S + 1]);
            }
            {
                const uint32_t a0 = hmul2_bf16(wa[2 * S], ae & 0x20002000u);
                const uint32_t a1 = hmul2_bf16(wb[2 * S], be & 0x20002000u);
                const uint32_t a2 = hmul2_bf16(wa[2 * S + 1], ao & 0x20002000u);
                const uint32_t a3 = hmul2_bf16(wb[2 * S + 1], bo & 0x20002000u);
#pragma unroll
                for (int t = 0; t < NT; ++t)
                    mma_bf16_16816(acc[I][t], a0, a1, a2, a3, xb[t][2 * S], xb[t][2 * S + 1]);
            }
            ExpMaskLoop<NT, S, P + 1>::run(acc, wa, wb, xb, ra, rb);
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
    if constexpr (NM == 8) {
        const uint32_t ra = prmt(S == 0 ? alo : ahi, 0u, 0x3120u);
        const uint32_t rb = prmt(S == 0 ? blo : bhi, 0u, 0x3120u);
        ExpMaskLoop<NT, S, 0>::run(acc, wa, wb, xb, ra, rb);
    } else {
        MaskLoop<NM, NT, S, 0>::run(acc, wa, wb, xb, alo, ahi, blo, bhi);
    }
}

template <int NM, int NT>
__device__ __forceinline__ float out_value(int act, const float (&acc)[NM + 1][NT][4], int t, int r)
{
    if constexpr (NM == 0) {
        return acc[0][t][r];
    } else {
        const float D = acc[0][t][r];
        float o = 0.f;
#pragma unroll
        for (int i = 0; i < NM; ++i) {
            // n_m = 8 accumulates mask i scaled by 2 (odd i) or 2^-63 (even i)
            const float scale = NM == 8 ? ((i & 1) ? 0.5f : 9.223372036854775808e18f) : 1.0f;
            const float gi = acc[1 + i][t][r] * scale;
            o += act_fn(act, gi) * (D - gi);
        }
        return o;
    }
}

template <int NM, int NT>
__device__ __forceinline__ void zero_acc(float (&acc)[NM + 1][NT][4])
{
#pragma unroll
    for (int v = 0; v <= NM; ++v)
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int r = 0; r < 4; ++r)
                acc[v][t][r] = 0.f;
}

// Accumulators are stored lane-major: float4 (v, t, lane) at ((v*NT + t)*32 + lane)*4.
template <int NM, int NT>
__device__ __forceinline__ void add_slot(float (&acc)[NM + 1][NT][4], const float *p, int lane, bool global)
{
#pragma unroll
    for (int v = 0; v <= NM; ++v)
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            const float4 *q = reinterpret_cast<const float4 *>(p + ((v * NT + t) * 32 + lane) * 4);
            const float4 o = global ? __ldcg(q) : *q;
            acc[v][t][0] += o.x, acc[v][t][1] += o.y, acc[v][t][2] += o.z, acc[v][t][3] += o.w;
        }
}

// The work of one CTA: first its stream-K share (units of the last RB_sk row
// blocks, split evenly over the grid), then its whole row blocks.  Every
// role of the CTA walks the same sequence with the same counters; no
// division happens per unit.
struct Sched {
    // 32-bit arithmetic throughout (the host keeps d < 2^22 and rows < 2^27,
    // so every product below fits): the integer divisions run once per CTA.
    int nst;          // k-stages per row block
    int G, cta;       // grid size, this CTA
    int RB;           // row blocks
    int q;            // whole row blocks per CTA
    int rb_sk0;       // first stream-K row block
    uint32_t U_sk;    // stream-K units
    uint32_t sk_b;    // first stream-K unit of this CTA
    int n_sk, n;      // units of this CTA: stream-K, all

    __device__ __forceinline__ void init(int rows, int d, int ks_width)
    {
        nst = (d + ks_width - 1) / ks_width;
        G = gridDim.x;
        cta = blockIdx.x;
        RB = (rows + ROWS - 1) / ROWS;
        q = RB / G;
        rb_sk0 = q * G;
        U_sk = (uint32_t)(RB - rb_sk0) * (uint32_t)nst;
        sk_b = sk_begin(cta);
        n_sk = (int)(sk_begin(cta + 1) - sk_b);
        n = n_sk + q * nst;
    }
    // (row block, stage) of the first unit of this CTA
    __device__ __forceinline__ void start(int &rb, int &ks) const
    {
        if (n_sk > 0) {
            rb = rb_sk0 + (int)(sk_b / (uint32_t)nst);
            ks = (int)(sk_b % (uint32_t)nst);
        } else {
            rb = cta * q;
            ks = 0;
        }
    }
    // advance after unit i (0-based) of this CTA
    __device__ __forceinline__ void next(int i, int &rb, int &ks) const
    {
        if (i + 1 == n_sk) {
            rb = cta * q;
            ks = 0;
        } else if (++ks == nst) {
            ks = 0;
            ++rb;
        }
    }
    // does unit i end this CTA's part of its row block?
    __device__ __forceinline__ bool flush_at(int i, int ks) const
    {
        return ks == nst - 1 || i == n_sk - 1 || i == n - 1;
    }
    // CTA whose stream-K share holds stream-K unit v
    __device__ __forceinline__ int sk_owner(uint32_t v) const
    {
        return (int)(((v + 1) * (uint32_t)G + U_sk - 1) / U_sk) - 1;
    }
    __device__ __forceinline__ uint32_t sk_begin(int c) const { return (uint32_t)c * U_sk / (uint32_t)G; }
};

// Scratch (global, caller-provided): partial sums of split row blocks, two
// slots per CTA (first and last row block of its stream-K share), then one
// arrival counter per row block.  Counters must be zero on entry and are
// zero again when the kernel completes.
template <int NM, int NT>
__global__ void __launch_bounds__(Layout<NM, NT>::NTHREADS, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                  const __grid_constant__ CUtensorMap tm_m, int T, int xr, int rows, int d, int act,
                  float *__restrict__ ws_part, int *__restrict__ ws_count, __nv_bfloat16 *__restrict__ out)
{
    using L = Layout<NM, NT>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::BAR_OFF);
    uint64_t *empty = full + L::STAGES;
    float *slots = reinterpret_cast<float *>(smem + L::SLOT_OFF);

    // The next kernel in the stream may start its prologue now; every access
    // to global memory below waits for the previous kernel to finish.
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    Sched sc;
    sc.init(rows, d, L::KS);

    if (threadIdx.x == 0) {
        for (int s = 0; s < L::STAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], L::NCW);
        }
        fence_mbar_init();
    }
    __syncthreads();
    if (sc.n == 0)
        return;
    pdl_wait();

    if (warp == L::PRODUCER_WARP) {
        // ------------------------------------------------------------- producer
        constexpr int NTMA = NM > 0 ? 3 : 2;
        const CUtensorMap *map = lane == 0 ? &tm_w : lane == 1 ? &tm_x : &tm_m;
        if (lane < NTMA)
            prefetch_tensormap(map);
        const int dst_off = lane == 0 ? L::W_OFF : lane == 1 ? L::X_OFF : L::M_OFF;
        int rb, ks;
        sc.start(rb, ks);
        for (int i = 0; i < sc.n; ++i) {
            const int s = i % L::STAGES;
            const uint32_t ph = (uint32_t)(i / L::STAGES) & 1u;
            int ok = 1;
            if (lane == 0) {
                ok = mbar_wait(&empty[s], ph ^ 1u);
                if (ok)
                    mbar_arrive_expect_tx(&full[s], L::tx(xr));
            }
            if (!__shfl_sync(0xffffffffu, ok, 0))
                break;
            __syncwarp();
            const int row0 = rb * ROWS;
            const int k0 = ks * L::KS;
            // lane 0: W (0, row0, k0/64); lane 1: x (0, 0, k0/64); lane 2: masks (0, row0, k0/128)
            if (lane < NTMA)
                tma_load_3d(smem + s * L::STAGE + dst_off, map, &full[s], 0, lane == 1 ? 0 : row0,
                            lane == 2 ? k0 / MASK_K : k0 / 64);
            sc.next(i, rb, ks);
        }
        return;
    }

    if (warp == L::FINISHER_WARP) {
        // ------------------------------------------------------------- finisher
        const int g = lane >> 2, c = lane & 3;
        float acc[NM + 1][NT][4];
        int rb, ks;
        sc.start(rb, ks);
        for (int i = 0; i < sc.n; sc.next(i, rb, ks), ++i) {
            if (!sc.flush_at(i, ks))
                continue;
            named_bar_sync(BAR_SLOTS_FULL, L::BAR_COUNT);  // the consumers' slots are written
            zero_acc<NM, NT>(acc);
            for (int w = 0; w < L::NCW; ++w)
                add_slot<NM, NT>(acc, slots + w * L::ACC, lane, false);
            if (i != sc.n - 1)
                named_bar_arrive(BAR_SLOTS_FREE, L::BAR_COUNT);

            bool finish = true;
            if (i < sc.n_sk) {
                const uint32_t v0 = (uint32_t)(rb - sc.rb_sk0) * (uint32_t)sc.nst;  // its first stream-K unit
                const int c_first = sc.sk_owner(v0);
                const int c_last = sc.sk_owner(v0 + (uint32_t)sc.nst - 1);
                if (c_first != c_last) {
                    // split row block: publish this CTA's partial, the last arriver finishes
                    const int my_slot = 2 * sc.cta + (v0 <= sc.sk_b ? 0 : 1);
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
                        zero_acc<NM, NT>(acc);
                        for (int cc = c_first; cc <= c_last; ++cc) {
                            const int sl = 2 * cc + (v0 <= sc.sk_begin(cc) ? 0 : 1);
                            add_slot<NM, NT>(acc, ws_part + (int64_t)sl * L::ACC, lane, true);
                        }
                        if (lane == 0)
                            ws_count[rb] = 0;  // leave the scratch zeroed for the next call
                    }
                }
            }
            if (finish) {
                const int row0 = rb * ROWS;
#pragma unroll
                for (int t = 0; t < NT; ++t)
#pragma unroll
                    for (int r = 0; r < 4; ++r) {
                        const int row = g + 8 * (r >> 1);
                        const int tok = 8 * t + 2 * c + (r & 1);
                        if (row0 + row < rows && tok < T)
                            out[(int64_t)tok * rows + row0 + row] =
                                __float2bfloat16_rn(out_value<NM, NT>(act, acc, t, r));
                    }
            }
        }
        return;
    }

    // ----------------------------------------------------------------- consumers
    const int g = lane >> 2, c = lane & 3;
    const int kc = warp >> 1, uu = warp & 1;     // this warp's 32 k: chunk kc, half uu
    const int ch = ((4 * uu + c) ^ g) << 4;      // 128-byte swizzle: 16-byte chunk ^ (row & 7)
    const int mc = warp >> 2;                    // mask box holding this warp's k
    const int mo = ((warp & 3) * 32 + 8 * c) * NM / 8;
    const int moff_a = L::M_OFF + mc * ROWS * L::M_BOX + mask_swz<L::M_BOX>(g, mo);
    const int moff_b = L::M_OFF + mc * ROWS * L::M_BOX + mask_swz<L::M_BOX>(g + 8, mo);
    const int woff = L::W_OFF + kc * L::W_CHUNK + g * 128 + ch;
    // the x box holds xr token rows per 64-k chunk (rows past xr read other
    // data; they only feed the MMA columns of tokens >= T, never stored)
    int xoff[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t) {
        const int xrow = kc * xr + 8 * t + g;
        xoff[t] = L::X_OFF + xrow * 128 + (((4 * uu + c) ^ (xrow & 7)) << 4);
    }
    float acc[NM + 1][NT][4];
    zero_acc<NM, NT>(acc);

    // A timed-out wait (status recorded by mbar_wait) stops the waiting and
    // the math, but every consumer still runs the same sequence of named
    // barriers with the finisher, so no warp can be left waiting at one.
    bool ok = true;
    int nflush = 0;
    int rb, ks;
    sc.start(rb, ks);
    for (int i = 0; i < sc.n; sc.next(i, rb, ks), ++i) {
        const int s = i % L::STAGES;
        const uint32_t ph = (uint32_t)(i / L::STAGES) & 1u;
        if (ok && !mbar_wait(&full[s], ph))
            ok = false;
        if (ok) {
            const uint8_t *st = smem + s * L::STAGE;
            uint32_t wa[4], wb[4], xb[NT][4];
            const uint4 va = *reinterpret_cast<const uint4 *>(st + woff);
            const uint4 vb = *reinterpret_cast<const uint4 *>(st + woff + 8 * 128);
            wa[0] = va.x, wa[1] = va.y, wa[2] = va.z, wa[3] = va.w;
            wb[0] = vb.x, wb[1] = vb.y, wb[2] = vb.z, wb[3] = vb.w;
#pragma unroll
            for (int t = 0; t < NT; ++t) {
                const uint4 vx = *reinterpret_cast<const uint4 *>(st + xoff[t]);
                xb[t][0] = vx.x, xb[t][1] = vx.y, xb[t][2] = vx.z, xb[t][3] = vx.w;
            }
            uint32_t alo = 0, ahi = 0, blo = 0, bhi = 0;
            if constexpr (NM > 0) {
                load_mask_chunk<NM>(st + moff_a, alo, ahi);
                load_mask_chunk<NM>(st + moff_b, blo, bhi);
            }
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&empty[s]);  // operands are in registers: the stage can be refilled
            unit_step<NM, NT, 0>(acc, wa, wb, xb, alo, ahi, blo, bhi);
            unit_step<NM, NT, 1>(acc, wa, wb, xb, alo, ahi, blo, bhi);
        }
        if (!sc.flush_at(i, ks))
            continue;
        // ---------------------------------------------------- row block done here
        if (nflush > 0)
            named_bar_sync(BAR_SLOTS_FREE, L::BAR_COUNT);  // finisher has read the previous slots
        float *slot = slots + warp * L::ACC;
#pragma unroll
        for (int v = 0; v <= NM; ++v)
#pragma unroll
            for (int t = 0; t < NT; ++t)
                *reinterpret_cast<float4 *>(slot + ((v * NT + t) * 32 + lane) * 4) =
                    make_float4(acc[v][t][0], acc[v][t][1], acc[v][t][2], acc[v][t][3]);
        named_bar_arrive(BAR_SLOTS_FULL, L::BAR_COUNT);
        ++nflush;
        zero_acc<NM, NT>(acc);
    }
}

// Scratch bytes of the decode kernel: partial slots for the largest grid,
// then one counter per row block of `rows` (256-byte aligned pieces).
__host__ __device__ constexpr int64_t part_bytes() { return (int64_t)2 * MAX_CTAS * 9 * 2 * 128 * 4; }
__host__ __device__ constexpr int64_t workspace_bytes(int64_t rows)
{
    return part_bytes() + ((rows + ROWS - 1) / ROWS * 4 + 255) / 256 * 256;
}

}  // namespace dec
}  // namespace mglu
