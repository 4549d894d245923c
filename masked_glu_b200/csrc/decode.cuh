// decode.cuh -- MGLU up-projection for few tokens (T <= 16), and the dense
// product (NM = 0) used as the decode-time down-projection.
//
// Memory-bound design ("Masked Gated Linear Unit", "Problem" and "Approach":
// decoding is bound by reading the weights, so each weight and its mask bits
// are read exactly once and the masks are unpacked inside the kernel):
//
//  * Work is made of units (row block of ROWS = 16 rows of W, k-stage of
//    KS k: 1024 for n_m <= 4, 768 for n_m = 8, 512 for 9..16 tokens).  A
//    persistent grid of one CTA per SM splits it evenly: every CTA gets the
//    same number of whole row blocks (data-parallel part) plus an equal
//    contiguous share of the units of the remaining row blocks (stream-K
//    part), so all SMs stream the same number of bytes.  Each CTA does its
//    stream-K share first, so the combining of row blocks split between CTAs
//    overlaps the data-parallel part instead of trailing the kernel.
//  * One producer thread streams the CTA's share through a ring of
//    shared-memory stages: per stage a W box (16 rows x KS, 128-byte
//    swizzle), an x box (the token rows x KS) and a packed-mask box of the
//    same rows and k, each completing on an mbarrier of its own.
//  * The consumer warps (4 for n_m <= 4, 12 for n_m = 8, 8 for 9..16 tokens)
//    each take 32 * UPW k of a stage.  A lane loads 8 consecutive weights of
//    two rows, turns each mask's bits into bf16x2 masks (AND masks for
//    n_m <= 4, exponent-bit scales for n_m = 8) and feeds W and the NM masked
//    copies of W as the A operand of mma.sync m16n8k16, with the tokens as
//    B.  One dense product D and NM gate products g_i accumulate in fp32;
//    the value of mask i is D - g_i.  The SM's instruction issue (mask
//    building plus the HMMAs) and the per-stage synchronization bound the
//    kernel; every weight and mask byte is read once.
//  * At the end of a row block the consumers drop their accumulators into
//    shared-memory slots and carry on; a finisher warp adds the slots in a
//    fixed order.  A row block whose k range lies inside one CTA is
//    finished there: out = sum_i act(g_i) (D - g_i), rounded once to bf16.
//    A row block split between CTAs (only at the two ends of a stream-K
//    share) is finished by whichever of its CTAs arrives last: the others'
//    partial sums come from a small global scratch, added in CTA order, so
//    the result does not depend on arrival order.  The arrival counter is
//    reset by the finishing CTA, leaving the scratch zeroed.
//  * The synchronization follows rules found necessary on B200 (each is
//    stated where it applies): one TMA load per mbarrier, one producer
//    thread, one polling lane per consumer warp, a proxy fence before
//    ordinary loads of a TMA-written stage, and release of a stage only once
//    its loads have returned.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"
#include "sched.cuh"

namespace mglu {
namespace dec {

constexpr int MAX_CTAS = 320;         // grid cap; sizes the split-row-block scratch
constexpr int BAR_SLOTS_FULL = 1;     // consumers arrive, finisher waits
constexpr int BAR_SLOTS_FREE = 2;     // finisher arrives, consumers wait
constexpr int MASK_K = 128;           // k covered by one row of a mask box

// Default consumer warps / 32-k units per warp and stage, chosen by timing on
// B200.  The math of a unit is bound by instruction issue, so more warps help
// only by hiding the per-stage wait and load latency, while fewer warps leave
// fewer accumulator slots to reduce and more shared memory for the ring:
// four warps with eight units (1024 k per stage) for n_m <= 4, twelve with two
// (768 k) for n_m = 8, eight with two (512 k) for two token blocks.  (Eight
// warps with four units was 5 % faster for n_m = 4 but gave wrong rows at
// T = 8 in repeated runs; it is not used.)
template <int NM, int NT>
struct DefaultShape {
    static constexpr int NCW = NT == 2 ? 8 : NM == 8 ? 12 : 4;
    static constexpr int UPW = NT == 2 ? 2 : NM == 8 ? 2 : 8;
};

constexpr int MAX_STAGES = 12;

template <int NM, int NT, int NCW_ = DefaultShape<NM, NT>::NCW, int UPW_ = DefaultShape<NM, NT>::UPW>
struct Layout {
    static constexpr int NCW = NCW_;
    static constexpr int UPW = UPW_;                   // 32-k units per consumer warp per stage
    static constexpr int W_WARP = NCW;                 // producer warp (one thread issues every load)
    static constexpr int FINISHER_WARP = NCW + 1;
    static constexpr int NTHREADS = (NCW + 2) * 32;
    static constexpr int BAR_COUNT = (NCW + 1) * 32;   // consumers + finisher
    static constexpr int KS = NCW * 32 * UPW;          // k per stage
    static constexpr int NKC = KS / 64;                // 64-k chunks per stage
    static constexpr int XR = 8 * NT;                  // most token rows of the x tile
    static constexpr int W_BYTES = ROWS * NKC * 128;   // W tile [16 rows][NKC chunks of 64 k]
    static constexpr int M_BOX = 16 * NM;              // mask bytes of one row per 128 k
    static constexpr int M_CHUNKS = KS / MASK_K;
    static constexpr int M_BYTES = NM == 0 ? 0 : M_CHUNKS * ROWS * M_BOX;
    static constexpr int M_OFF = W_BYTES;
    static constexpr int X_OFF = M_OFF + (M_BYTES + 1023) / 1024 * 1024;
    static constexpr int ACC = (NM + 1) * NT * 128;    // floats of one warp's accumulators
    static constexpr int SLOTS = NCW * ACC * 4;
    // shared memory: barriers, consumer slots, then the ring of stages
    static constexpr int BAR_OFF = 0;                  // full, xfull, mfull, empty: MAX_STAGES each
    static constexpr int SLOT_OFF = 1024;
    static constexpr int RING_OFF = (SLOT_OFF + SLOTS + 1023) / 1024 * 1024;
    static constexpr int SMEM = 227 * 1024;            // includes 1 KB of alignment slack
    static constexpr int RING_BYTES = SMEM - 1024 - RING_OFF;
    // a stage with xr token rows of x (x boxes hold only the T rows loaded)
    static __host__ __device__ constexpr int x_bytes(int xr) { return (NKC * xr * 128 + 1023) / 1024 * 1024; }
    static __host__ __device__ constexpr int stage_bytes(int xr) { return X_OFF + x_bytes(xr); }
    static __host__ __device__ constexpr int stages(int xr)
    {
        return RING_BYTES / stage_bytes(xr) > MAX_STAGES ? MAX_STAGES : RING_BYTES / stage_bytes(xr);
    }
    static_assert(RING_BYTES / (X_OFF + (NKC * XR * 128 + 1023) / 1024 * 1024) >= 3, "ring too shallow");
};

// Byte offset of a linear position inside a staged tile under the tensor
// map's swizzle: the 16-byte unit index (address bits 4 and up) is XORed with
// the 128-byte line index (address bits 7 and up) over 3, 2 or 1 bits for the
// 128-, 64- and 32-byte swizzles; narrower tiles are not swizzled.  Every
// tile starts on a 1024-byte boundary, so tile offsets and addresses agree.
template <int SPAN>
__host__ __device__ constexpr int swz(int lin)
{
    return SPAN == 128 ? lin ^ (((lin >> 7) & 7) << 4)
         : SPAN == 64  ? lin ^ (((lin >> 7) & 3) << 4)
         : SPAN == 32  ? lin ^ (((lin >> 7) & 1) << 4)
                       : lin;
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

// v << S (S >= 0) or v >> -S, written as an integer multiply so it can run on
// the FMA pipe instead of the busier ALU pipe.
template <int S>
__device__ __forceinline__ uint32_t shift_signed(uint32_t v)
{
    uint32_t r;
    if constexpr (S == 0)
        r = v;
    else if constexpr (S > 0)
        asm("mul.lo.u32 %0, %1, %2;" : "=r"(r) : "r"(v), "n"(1u << S));
    else
        asm("mul.hi.u32 %0, %1, %2;" : "=r"(r) : "r"(v), "n"(1u << (32 + S)));
    return r;
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

// Scratch (global, caller-provided): partial sums of split row blocks, two
// slots per CTA (first and last row block of its stream-K share), then one
// arrival counter per row block.  Counters must be zero on entry and are
// zero again when the kernel completes.
template <int NM, int NT, int NCW_ = DefaultShape<NM, NT>::NCW, int UPW_ = DefaultShape<NM, NT>::UPW>
__global__ void __launch_bounds__(Layout<NM, NT, NCW_, UPW_>::NTHREADS, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tm_w, const __grid_constant__ CUtensorMap tm_x,
                  const __grid_constant__ CUtensorMap tm_m, int T, int xr, int rows, int d, int act,
                  float *__restrict__ ws_part, int *__restrict__ ws_count, __nv_bfloat16 *__restrict__ out)
{
    using L = Layout<NM, NT, NCW_, UPW_>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *full = reinterpret_cast<uint64_t *>(smem + L::BAR_OFF);
    uint64_t *xfull = full + MAX_STAGES;
    uint64_t *mfull = xfull + MAX_STAGES;
    uint64_t *empty = mfull + MAX_STAGES;
    float *slots = reinterpret_cast<float *>(smem + L::SLOT_OFF);
    uint8_t *ring = smem + L::RING_OFF;
    const int STAGE = L::stage_bytes(xr);
    const int NSTAGES = L::stages(xr);

    // The next kernel in the stream may start its prologue now; every access
    // to global memory below waits for the previous kernel to finish.
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    Sched sc;
    sc.init(rows, d, L::KS, gridDim.x, blockIdx.x);

    if (threadIdx.x == 0) {
        for (int s = 0; s < NSTAGES; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&xfull[s], 1);
            mbar_init(&mfull[s], 1);
            mbar_init(&empty[s], L::NCW);
        }
        fence_mbar_init();
    }
    __syncthreads();
    if (sc.n == 0)
        return;
    pdl_wait();

    if (warp == L::W_WARP) {
        // ------------------------------------------------------------- producer
        // One thread issues the W, x and mask boxes of a stage, each completing
        // on a barrier of its own.  (Loads from several producer warps, or
        // several loads completing on one barrier, gave occasional wrong
        // operands on B200; one load per barrier from one thread did not.)
        if (lane == 0) {
            const uint32_t xbytes = (uint32_t)(L::NKC * xr * 128);
            prefetch_tensormap(&tm_w);
            prefetch_tensormap(&tm_x);
            if (NM > 0)
                prefetch_tensormap(&tm_m);
            int rb, ks;
            sc.start(rb, ks);
            for (int i = 0; i < sc.n; sc.next(i, rb, ks), ++i) {
                const int s = i % NSTAGES;
                const uint32_t ph = (uint32_t)(i / NSTAGES) & 1u;
                if (!mbar_wait(&empty[s], ph ^ 1u))
                    break;
                uint8_t *st = ring + s * STAGE;
                const int k0 = ks * L::KS;
                // boxes: W (0, k0/64, row0), x (0, k0/64, 0), masks (0, k0/128, row0)
                mbar_arrive_expect_tx(&full[s], (uint32_t)L::W_BYTES);
                tma_load_3d(st, &tm_w, &full[s], 0, k0 / 64, rb * ROWS);
                mbar_arrive_expect_tx(&xfull[s], xbytes);
                tma_load_3d(st + L::X_OFF, &tm_x, &xfull[s], 0, k0 / 64, 0);
                if constexpr (NM > 0) {
                    mbar_arrive_expect_tx(&mfull[s], (uint32_t)L::M_BYTES);
                    tma_load_3d(st + L::M_OFF, &tm_m, &mfull[s], 0, k0 / MASK_K, rb * ROWS);
                }
            }
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
            if (i != sc.n - 1) {
                __threadfence_block();  // the slot reads above are done before the consumers may overwrite
                named_bar_arrive(BAR_SLOTS_FREE, L::BAR_COUNT);
            }

            bool finish = true;
            if (i < sc.n_sk) {
                int c_first, c_last;
                const int nparts = sc.contributors(rb, c_first, c_last);
                if (c_first != c_last) {
                    // publish this CTA's partial; the last arriver finishes
                    float *mine = ws_part + (int64_t)sc.slot(sc.cta, rb) * L::ACC;
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
                    finish = prev == nparts - 1;
                    if (finish) {
                        // every partial, this CTA's included, read back in CTA order
                        __threadfence();
                        zero_acc<NM, NT>(acc);
                        for (int cc = c_first; cc <= c_last; ++cc)
                            if (sc.contributes(cc))
                                add_slot<NM, NT>(acc, ws_part + (int64_t)sc.slot(cc, rb) * L::ACC, lane, true);
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
    // shared-memory offsets of this warp's operands inside a stage, per unit
    int woff[L::UPW], moff_a[L::UPW], moff_b[L::UPW], xoff[L::UPW][NT];
#pragma unroll
    for (int uw = 0; uw < L::UPW; ++uw) {
        const int un = warp * L::UPW + uw;   // 32-k unit of the stage
        const int kc = un >> 1, uu = un & 1; // 64-k chunk, half of it
        // W tile [row][chunk][64 k]: lane (g, c) reads 16 bytes of row g; row
        // g + 8 is 8 * NKC lines on, the same swizzle phase
        woff[uw] = swz<128>((g * L::NKC + kc) * 128 + (4 * uu + c) * 16);
        // x tile [token][chunk][64 k] holds xr tokens; lanes of tokens >= xr
        // read token xr - 1 (their MMA columns are never stored)
#pragma unroll
        for (int t = 0; t < NT; ++t) {
            const int tr = 8 * t + g < xr ? 8 * t + g : xr - 1;
            xoff[uw][t] = L::X_OFF + swz<128>((tr * L::NKC + kc) * 128 + (4 * uu + c) * 16);
        }
        // mask tile [row][128-k chunk][M_BOX bytes]
        const int mc = un >> 2;
        const int mo = ((un & 3) * 32 + 8 * c) * NM / 8;
        moff_a[uw] = L::M_OFF + swz<L::M_BOX>((g * L::M_CHUNKS + mc) * L::M_BOX + mo);
        moff_b[uw] = L::M_OFF + swz<L::M_BOX>(((g + 8) * L::M_CHUNKS + mc) * L::M_BOX + mo);
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
        const int s = i % NSTAGES;
        const uint32_t ph = (uint32_t)(i / NSTAGES) & 1u;
        if (ok && !mbar_wait_warp3(&xfull[s], &full[s], NM > 0 ? &mfull[s] : nullptr, ph))
            ok = false;
        // The stage was written through the async proxy (TMA) and is read
        // below with ordinary loads: order the two proxies for this thread.
        // (Without this fence, reads right after the wait occasionally saw
        // stale operands on B200.)
        fence_proxy_async_smem();
        if (ok) {
            const uint8_t *st = ring + s * STAGE;
            uint32_t wa[L::UPW][4], wb[L::UPW][4], xb[L::UPW][NT][4];
            uint32_t alo[L::UPW], ahi[L::UPW], blo[L::UPW], bhi[L::UPW];
#pragma unroll
            for (int uw = 0; uw < L::UPW; ++uw) {
                const uint4 va = *reinterpret_cast<const uint4 *>(st + woff[uw]);
                const uint4 vb = *reinterpret_cast<const uint4 *>(st + woff[uw] + 8 * L::NKC * 128);
                wa[uw][0] = va.x, wa[uw][1] = va.y, wa[uw][2] = va.z, wa[uw][3] = va.w;
                wb[uw][0] = vb.x, wb[uw][1] = vb.y, wb[uw][2] = vb.z, wb[uw][3] = vb.w;
#pragma unroll
                for (int t = 0; t < NT; ++t) {
                    const uint4 vx = *reinterpret_cast<const uint4 *>(st + xoff[uw][t]);
                    xb[uw][t][0] = vx.x, xb[uw][t][1] = vx.y, xb[uw][t][2] = vx.z, xb[uw][t][3] = vx.w;
                }
                alo[uw] = ahi[uw] = blo[uw] = bhi[uw] = 0;
                if constexpr (NM > 0) {
                    load_mask_chunk<NM>(st + moff_a[uw], alo[uw], ahi[uw]);
                    load_mask_chunk<NM>(st + moff_b[uw], blo[uw], bhi[uw]);
                }
            }
            // Release the stage only once every lane's loads have returned:
            // folding all loaded words into one value makes each lane wait for
            // its own loads before the warp synchronizes and lane 0 arrives.
            // (Releasing right after issuing the loads let a refill overwrite
            // operands still being read, now and then, on B200.)
            uint32_t dep = 0;
#pragma unroll
            for (int uw = 0; uw < L::UPW; ++uw) {
                dep ^= wa[uw][0] ^ wa[uw][1] ^ wa[uw][2] ^ wa[uw][3] ^ wb[uw][0] ^ wb[uw][1] ^ wb[uw][2] ^ wb[uw][3];
#pragma unroll
                for (int t = 0; t < NT; ++t)
                    dep ^= xb[uw][t][0] ^ xb[uw][t][1] ^ xb[uw][t][2] ^ xb[uw][t][3];
                dep ^= alo[uw] ^ ahi[uw] ^ blo[uw] ^ bhi[uw];
            }
            consume(dep);
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&empty[s]);
#pragma unroll
            for (int uw = 0; uw < L::UPW; ++uw) {
                unit_step<NM, NT, 0>(acc, wa[uw], wb[uw], xb[uw], alo[uw], ahi[uw], blo[uw], bhi[uw]);
                unit_step<NM, NT, 1>(acc, wa[uw], wb[uw], xb[uw], alo[uw], ahi[uw], blo[uw], bhi[uw]);
            }
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
        __threadfence_block();  // the slot writes are visible before the finisher reads them
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
