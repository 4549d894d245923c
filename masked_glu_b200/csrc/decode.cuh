// decode.cuh -- MGLU up-projection for few tokens (T <= 16), and the dense
// product (NM = 0) used as the decode-time down-projection.
//
// Memory-bound design ("Masked Gated Linear Unit", "Problem" and "Approach":
// decoding is bound by reading the weights, so each weight and its mask bits
// are read exactly once and the masks are unpacked inside the kernel):
//
//  * Work is made of stages (row block of ROWS = 16 rows of W, k-stage of
//    KS = 32 * NW k, one 32-k unit per consumer warp).  A persistent grid of
//    one CTA per SM splits the stages evenly: every CTA gets the same number
//    of whole row blocks (data-parallel part) plus an equal contiguous share
//    of the stages of the remaining row blocks (stream-K part), so all SMs
//    stream the same number of bytes.  Each CTA does its stream-K share
//    first, so the combining of row blocks split between CTAs overlaps the
//    data-parallel part instead of trailing the kernel.
//  * Each warp streams its own unit of every stage through a private ring of
//    P stages in shared memory: lane (g, c) copies (cp.async) 16 bytes of W
//    rows g and g + 8 (eight weights each), their mask bits and 16 bytes of
//    each token block's x, P - 1 stages ahead of the one it multiplies, and
//    reads back only what it copied itself.  The copies are tracked by
//    cp.async groups, not registers, so the ring can be deep (about 100 KB in
//    flight per SM); no staged operand passes from one thread to another, so
//    the weight stream needs no barrier.
//  * Masks are applied by sign flips (see group_bits / flip_pair): the warp
//    accumulates the dense product D = x W and h_i = x (S_i . W) with
//    S_i = +1 where mask i is set and -1 where it is clear, on mma.sync
//    m16n8k16 with the 16 rows as M and the tokens as N; one LOP3 and one
//    shift per bf16 pair and mask build the operand.  Then g_i = (D + h_i)/2
//    and v_i = (D - h_i)/2 = D - g_i.
//  * At the end of a row block's part in this CTA each warp drops its
//    accumulators into a shared-memory slot (one or two slot sets, used in
//    turn)
//    and carries on, except the part's finisher: the warps take that role in
//    turn (part f: warp f mod NW), wait for every slot of the part, add them
//    in a fixed order and finish the part.  Before a set is written again
//    every warp, that part's finisher included, meets on a barrier.  A row block whose k range lies
//    inside one CTA is finished there:
//    out = sum_i act(g_i) v_i, rounded once to bf16.  A row block split
//    between CTAs (only at the two ends of a stream-K share) is finished by
//    whichever of its CTAs arrives last: the others' partial sums come from
//    a small global scratch, added in CTA order, so the result does not
//    depend on arrival order.  The arrival counter is reset by the finishing
//    CTA, leaving the scratch zeroed.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"
#include "sched.cuh"

namespace mglu {
namespace dec {

constexpr int MAX_CTAS = 320;  // grid cap; sizes the split-row-block scratch
// named barriers: slot set b is full (writers arrive, the part's finisher
// waits) / free again (every warp waits: the finisher reaches it after
// reading the set)
constexpr int BAR_FULL0 = 1;
constexpr int BAR_FREE0 = 3;

// Warps by n_m and token blocks.  Registers are allocated to warps in groups
// of four, so NW is a multiple of four: 16 warps get 128 registers a thread,
// 12 get 168, 8 get 255.
template <int NM, int NT>
struct DefaultShape {
    static constexpr int NW = NT == 1 ? 16 : NM == 8 ? 8 : NM == 4 ? 12 : 16;
};

template <int NM, int NT, int NW_ = DefaultShape<NM, NT>::NW>
struct Layout {
    static constexpr int NW = NW_;                     // warps, each a consumer and in turn a finisher
    static constexpr int NTHREADS = NW * 32;
    static constexpr int BAR_COUNT = NW * 32;
    static constexpr int KS = NW * 32;                 // k per stage
    static constexpr int ACC = (NM + 1) * NT * 128;    // floats of one warp's accumulators
    static constexpr int SLOT_SET = NW * ACC;          // floats of one slot set
    // one stage of a warp's ring, per lane: W rows g and g + 8 (16 bytes
    // each), their mask bytes (n_m >= 4; narrower masks go through
    // registers), 16 bytes of x per token block; laid out lane-contiguous per
    // row so that each 16-byte read of a warp is conflict-free
    static constexpr int MB = NM >= 4 ? NM : 0;         // mask bytes per lane and row in the ring
    static constexpr int W_A = 0, W_B = 512;
    static constexpr int M_A = 1024, M_B = 1024 + 32 * MB;
    static constexpr int X_OFF = (1024 + 64 * MB + 15) / 16 * 16;
    static constexpr int STG = (X_OFF + 512 * NT + 127) / 128 * 128;
    static constexpr int BUDGET = 227 * 1024;
    static constexpr int ring_depth(int sets) { return (BUDGET - sets * SLOT_SET * 4) / (NW * STG); }
    // two slot sets when the ring stays at least 5 deep with them, else one
    static constexpr int SETS = ring_depth(2) >= 5 ? 2 : 1;
    static constexpr int P = ring_depth(SETS) > 8 ? 8 : ring_depth(SETS);
    static constexpr int RING_OFF = SETS * SLOT_SET * 4;
    static constexpr int SMEM = RING_OFF + NW * P * STG;
    static_assert(NW % 4 == 0, "warps are allocated registers in groups of four");
    static_assert(P >= 3, "ring too shallow");
    static_assert(SMEM <= BUDGET, "shared memory");
};

// ---------------------------------------------------------------- loads
// Narrow mask bits (n_m <= 2: one or two bytes per lane and row) are loaded
// into registers one stage ahead: read-only path, not kept in L1.
__device__ __forceinline__ uint2 ld_stream_8(const void *p)
{
    uint2 v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ld_stream_4(const void *p)
{
    uint32_t v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.u32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ld_stream_2(const void *p)
{
    unsigned short v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.u16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ uint32_t ld_stream_1(const void *p)
{
    unsigned short v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::256B.u8 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

// Mask bits of an 8-weight chunk: NM bytes at byte offset (j*d + k)*NM/8.
template <int NM>
__device__ __forceinline__ uint2 ld_mask_chunk(const uint8_t *p)
{
    if constexpr (NM == 8)
        return ld_stream_8(p);
    else if constexpr (NM == 4)
        return make_uint2(ld_stream_4(p), 0u);
    else if constexpr (NM == 2)
        return make_uint2(ld_stream_2(p), 0u);
    else if constexpr (NM == 1)
        return make_uint2(ld_stream_1(p), 0u);
    else
        return make_uint2(0u, 0u);
}

// One stage's operands of one lane: 8 weights of rows g and g + 8, their
// mask bits, and 8 values of x for each token block.
template <int NM, int NT>
struct Operands {
    uint4 wa, wb;
    uint2 ma, mb;
    uint4 xv[NT];
};

// v << S for a constant S >= 0, as an integer multiply so that it issues to
// the FMA pipe (the ALU pipe takes the LOP3s of the sign flips).
template <int S>
__device__ __forceinline__ uint32_t shl_fma(uint32_t v)
{
    if constexpr (S == 0) {
        return v;
    } else {
        uint32_t r;
        asm("mul.lo.u32 %0, %1, %2;" : "=r"(r) : "r"(v), "n"(1u << S));
        return r;
    }
}

__device__ __forceinline__ uint32_t u4(const uint4 &v, int q)
{
    return q == 0 ? v.x : q == 1 ? v.y : q == 2 ? v.z : v.w;
}

// h_I += x (S_I . W) for k16 sub-step S of the unit, then the next mask.
// With ROUTED, masks whose bit in `used` is clear (no token of the call
// gives them a nonzero weight) skip their products.
template <int NM, int NT, bool ROUTED, int S, int I>
struct FlipLoop {
    static __device__ __forceinline__ void run(float (&acc)[NM + 1][NT][4], const Operands<NM, NT> &o, uint32_t ra,
                                               uint32_t rb, uint32_t used)
    {
        if constexpr (I < NM) {
            if (!ROUTED || ((used >> I) & 1u)) {
                const uint32_t a0 = flip_pair(u4(o.wa, 2 * S), shl_fma<15 - I>(ra));
                const uint32_t a1 = flip_pair(u4(o.wb, 2 * S), shl_fma<15 - I>(rb));
                const uint32_t a2 = flip_pair(u4(o.wa, 2 * S + 1), shl_fma<7 - I>(ra));
                const uint32_t a3 = flip_pair(u4(o.wb, 2 * S + 1), shl_fma<7 - I>(rb));
#pragma unroll
                for (int t = 0; t < NT; ++t)
                    mma_bf16_16816(acc[1 + I][t], a0, a1, a2, a3, u4(o.xv[t], 2 * S), u4(o.xv[t], 2 * S + 1));
            }
            FlipLoop<NM, NT, ROUTED, S, I + 1>::run(acc, o, ra, rb, used);
        }
    }
};

// One 16-row x 32-k unit.  Lane (g, c) holds weights [8c, 8c+8) of rows g
// and g+8; k16 sub-step S uses its bf16 pairs 2S and 2S+1.  The k order
// inside the MMA is a permutation of the physical k that depends only on c
// and S; x (operand B) is loaded with the same permutation, so every sum is
// unchanged.
template <int NM, int NT, bool ROUTED, int S>
__device__ __forceinline__ void unit_step(float (&acc)[NM + 1][NT][4], const Operands<NM, NT> &o, uint32_t used)
{
#pragma unroll
    for (int t = 0; t < NT; ++t)
        mma_bf16_16816(acc[0][t], u4(o.wa, 2 * S), u4(o.wb, 2 * S), u4(o.wa, 2 * S + 1), u4(o.wb, 2 * S + 1),
                       u4(o.xv[t], 2 * S), u4(o.xv[t], 2 * S + 1));
    if constexpr (NM > 0) {
        const uint32_t ra = group_bits<NM, S>(o.ma.x, o.ma.y);
        const uint32_t rb = group_bits<NM, S>(o.mb.x, o.mb.y);
        FlipLoop<NM, NT, ROUTED, S, 0>::run(acc, o, ra, rb, used);
    }
}

// The output of one (row, token) from its sums (D, h_1, ..., h_NM):
// sum_i w_i act(g_i) v_i, with the token's mask weights w (NULL: every
// weight 1).
template <int NM>
__device__ __forceinline__ float out_value(int act, const float (&sums)[NM + 1], const float *__restrict__ w)
{
    if constexpr (NM == 0) {
        return sums[0];
    } else {
        const float D = sums[0];
        const bool dense_gate = (act & GATE_DENSE) != 0;
        const int a = act & ACT_MASK;
        float o = 0.f;
#pragma unroll
        for (int i = 0; i < NM; ++i) {
            const float h = sums[1 + i];
            const float g = 0.5f * (D + h);  // x (M_i . W)
            const float v = 0.5f * (D - h);  // x ((1 - M_i) . W)
            o += (w ? w[i] : 1.0f) * (act_fn(a, dense_gate ? D : g) * v);
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
// One float4 is loaded and added at a time (an empty asm with a memory
// clobber keeps the compiler from hoisting all loads ahead): the finisher
// runs while the warp's prefetched operands occupy registers.
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
            asm volatile("" ::: "memory");
        }
}

// Finish row-block part f (the calling warp is its finisher) from the NW
// slots of its set: add them in warp order, then either write the outputs or, for a row block split between
// CTAs, publish this CTA's partial sum and let the last CTA to arrive add all
// partials in CTA order and write them.  Not inlined: it runs once per part,
// and keeping its registers out of the streaming loop leaves that loop
// without spills.
template <int NM, int NT, bool ROUTED, int NW>
__device__ __noinline__ void finish_part(float *__restrict__ set_base, int rb, bool stream_k,
                                         const Sched sc, int act, int T, int rows, float *__restrict__ ws_part,
                                         int *__restrict__ ws_count, __nv_bfloat16 *__restrict__ out,
                                         const float *__restrict__ mw)
{
    constexpr int ACC = (NM + 1) * NT * 128;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    float acc[NM + 1][NT][4];
    zero_acc<NM, NT>(acc);
#pragma unroll 1
    for (int w = 0; w < NW; ++w)
        add_slot<NM, NT>(acc, set_base + w * ACC, lane, false);
    bool finish = true;
    if (stream_k) {
        int c_first, c_last;
        const int nparts = sc.contributors(rb, c_first, c_last);
        if (c_first != c_last) {
            float *mine = ws_part + (int64_t)sc.slot(sc.cta, rb) * ACC;
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
#pragma unroll 1
                for (int cc = c_first; cc <= c_last; ++cc)
                    if (sc.contributes(cc))
                        add_slot<NM, NT>(acc, ws_part + (int64_t)sc.slot(cc, rb) * ACC, lane, true);
                if (lane == 0)
                    ws_count[rb] = 0;  // leave the scratch zeroed for the next call
            }
        }
    }
    if (finish) {
        // Park the sums in this warp's own slot of the set (already read;
        // no other warp writes it) and form the outputs one (token, row) at a
        // time from there.
        float *own = set_base + warp * ACC;
#pragma unroll
        for (int v = 0; v <= NM; ++v)
#pragma unroll
            for (int t = 0; t < NT; ++t)
                *reinterpret_cast<float4 *>(own + ((v * NT + t) * 32 + lane) * 4) =
                    make_float4(acc[v][t][0], acc[v][t][1], acc[v][t][2], acc[v][t][3]);
        const int row0 = rb * ROWS;
#pragma unroll 1
        for (int tr = 0; tr < NT * 4; ++tr) {
            const int t = tr >> 2, r = tr & 3;
            const int row = g + 8 * (r >> 1);
            const int tok = 8 * t + 2 * c + (r & 1);
            float sums[NM + 1];
#pragma unroll
            for (int v = 0; v <= NM; ++v)
                sums[v] = own[((v * NT + t) * 32 + lane) * 4 + r];
            if (row0 + row < rows && tok < T)
                out[(int64_t)tok * rows + row0 + row] =
                    __float2bfloat16_rn(out_value<NM>(act, sums, ROUTED ? mw + (int64_t)tok * NM : nullptr));
        }
    }
}

// Scratch (global, caller-provided): partial sums of split row blocks, two
// slots per CTA (first and last row block of its stream-K share), then one
// arrival counter per row block.  Counters must be zero on entry and are
// zero again when the kernel completes.
//
// ROUTED: per-token mask weights mw [T][NM] scale each mask's term, and a
// mask that no token of the call weights (all its weights zero) skips its
// products (the weight stream is read in full either way).
template <int NM, int NT, bool ROUTED = false, int NW_ = DefaultShape<NM, NT>::NW>
__global__ void __launch_bounds__(Layout<NM, NT, NW_>::NTHREADS, 1)
    decode_kernel(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ W,
                  const uint8_t *__restrict__ packed, int T, int rows, int d, int act, float *__restrict__ ws_part,
                  int *__restrict__ ws_count, __nv_bfloat16 *__restrict__ out, const float *__restrict__ mw)
{
    using L = Layout<NM, NT, NW_>;
    extern __shared__ __align__(128) float slots[];  // L::SETS sets of NW slots, then the warps' rings

    // The next kernel in the stream may start its prologue now; every access
    // to global memory below waits for the previous kernel to finish.
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    Sched sc;
    sc.init(rows, d, L::KS, gridDim.x, blockIdx.x);
    if (sc.n == 0)
        return;
    pdl_wait();

    // masks some token of the call weights
    uint32_t used = (1u << NM) - 1u;
    if constexpr (ROUTED) {
        uint32_t u = 0;
        for (int e = lane; e < T * NM; e += 32)
            u |= (mw[e] != 0.0f ? 1u : 0u) << (e % NM);
        used = __reduce_or_sync(0xffffffffu, u);
    }

    // ----------------------------------------------------------------- consumers
    // This warp's 32-k unit of stage ks starts at k = ks * KS + 32 * warp;
    // this lane's 8 weights at k = that + 8 * c.
    const int kl = 32 * warp + 8 * c;
    const int64_t mrow = (int64_t)d * NM / 8;  // mask bytes per row of W
    int xrow[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t)
        xrow[t] = 8 * t + g < T ? 8 * t + g : T - 1;  // lanes of absent tokens repeat the last one
    uint8_t *ring = reinterpret_cast<uint8_t *>(slots) + L::RING_OFF + warp * L::P * L::STG;
    const uint32_t ring_s = smem_u32(ring);

    // Copies of stage (rb, ks) into ring stage ss; lanes outside the matrix
    // copy zeros (a d % 8 == 0 row keeps a lane's 8 weights all in or out).
    auto issue = [&](int ss, int rb, int ks) {
        const uint32_t st = ring_s + (uint32_t)(ss * L::STG);
        const int k = ks * L::KS + kl;
        const int ra = rb * ROWS + g, rbb = ra + 8;
        const bool kin = k < d, va = kin && ra < rows, vb = kin && rbb < rows;
        cp_async_cg16(st + L::W_A + lane * 16, va ? W + (int64_t)ra * d + k : W, va ? 16u : 0u);
        cp_async_cg16(st + L::W_B + lane * 16, vb ? W + (int64_t)rbb * d + k : W, vb ? 16u : 0u);
        if constexpr (L::MB > 0) {
            cp_async_ca<L::MB>(st + L::M_A + lane * L::MB, va ? packed + (int64_t)ra * mrow + (int64_t)k * NM / 8 : packed,
                               va ? (uint32_t)L::MB : 0u);
            cp_async_ca<L::MB>(st + L::M_B + lane * L::MB, vb ? packed + (int64_t)rbb * mrow + (int64_t)k * NM / 8 : packed,
                               vb ? (uint32_t)L::MB : 0u);
        }
#pragma unroll
        for (int t = 0; t < NT; ++t)
            cp_async_ca<16>(st + L::X_OFF + t * 512 + lane * 16, kin ? x + (int64_t)xrow[t] * d + k : x,
                            kin ? 16u : 0u);
    };
    // n_m <= 2: a lane's mask bits (1 or 2 bytes a row) come through registers
    auto load_small_masks = [&](uint2 &ma, uint2 &mb, int rb, int ks) {
        const int k = ks * L::KS + kl;
        const int ra = rb * ROWS + g, rbb = ra + 8;
        ma = mb = make_uint2(0u, 0u);
        if (k < d) {
            if (ra < rows)
                ma = ld_mask_chunk<NM>(packed + (int64_t)ra * mrow + (int64_t)k * NM / 8);
            if (rbb < rows)
                mb = ld_mask_chunk<NM>(packed + (int64_t)rbb * mrow + (int64_t)k * NM / 8);
        }
    };

    float acc[NM + 1][NT][4];
    zero_acc<NM, NT>(acc);

    // the copy cursor runs P - 1 stages ahead of the compute cursor
    int rb_c, ks_c, rb_l, ks_l;
    sc.start(rb_c, ks_c);
    rb_l = rb_c, ks_l = ks_c;
    for (int b = 0; b < L::P - 1; ++b) {
        if (b < sc.n)
            issue(b, rb_l, ks_l);
        cp_async_commit();  // one group per stage, empty past the end
        sc.next(b, rb_l, ks_l);
    }
    uint2 sm_a = make_uint2(0u, 0u), sm_b = make_uint2(0u, 0u);  // next stage's narrow masks
    if constexpr (NM > 0 && L::MB == 0)
        load_small_masks(sm_a, sm_b, rb_c, ks_c);

    int nflush = 0;
    for (int i = 0; i < sc.n; ++i) {
        const int il = i + L::P - 1;
        if (il < sc.n)
            issue(il % L::P, rb_l, ks_l);
        cp_async_commit();
        sc.next(il, rb_l, ks_l);
        cp_async_wait<L::P - 1>();  // this lane's copies of stage i have landed

        Operands<NM, NT> o;
        const uint8_t *st = ring + (i % L::P) * L::STG;
        o.wa = *reinterpret_cast<const uint4 *>(st + L::W_A + lane * 16);
        o.wb = *reinterpret_cast<const uint4 *>(st + L::W_B + lane * 16);
#pragma unroll
        for (int t = 0; t < NT; ++t)
            o.xv[t] = *reinterpret_cast<const uint4 *>(st + L::X_OFF + t * 512 + lane * 16);
        if constexpr (L::MB == 8) {
            o.ma = *reinterpret_cast<const uint2 *>(st + L::M_A + lane * 8);
            o.mb = *reinterpret_cast<const uint2 *>(st + L::M_B + lane * 8);
        } else if constexpr (L::MB == 4) {
            o.ma = make_uint2(*reinterpret_cast<const uint32_t *>(st + L::M_A + lane * 4), 0u);
            o.mb = make_uint2(*reinterpret_cast<const uint32_t *>(st + L::M_B + lane * 4), 0u);
        } else {
            o.ma = sm_a;
            o.mb = sm_b;
        }
        if constexpr (NM > 0 && L::MB == 0) {
            if (i + 1 < sc.n) {
                int rb_n = rb_c, ks_n = ks_c;
                sc.next(i, rb_n, ks_n);
                load_small_masks(sm_a, sm_b, rb_n, ks_n);
            }
        }
        if (ks_c * L::KS + 32 * warp < d) {
            unit_step<NM, NT, ROUTED, 0>(acc, o, used);
            unit_step<NM, NT, ROUTED, 1>(acc, o, used);
        }
        if (sc.flush_at(i, ks_c)) {
            // ---------------------------------------------- row-block part done here
            const int f = nflush++, set = f % L::SETS;
            // this set was last used by part f - SETS: all warps meet here, the
            // finisher of that part among them once it has read the set
            if (f >= L::SETS)
                named_bar_sync(BAR_FREE0 + set, L::BAR_COUNT);
            float *slot = slots + set * L::SLOT_SET + warp * L::ACC;
#pragma unroll
            for (int v = 0; v <= NM; ++v)
#pragma unroll
                for (int t = 0; t < NT; ++t)
                    *reinterpret_cast<float4 *>(slot + ((v * NT + t) * 32 + lane) * 4) =
                        make_float4(acc[v][t][0], acc[v][t][1], acc[v][t][2], acc[v][t][3]);
            zero_acc<NM, NT>(acc);
            if (warp == f % L::NW) {
                named_bar_sync(BAR_FULL0 + set, L::BAR_COUNT);  // every slot of part f is written
                finish_part<NM, NT, ROUTED, L::NW>(slots + set * L::SLOT_SET, rb_c, i < sc.n_sk, sc, act, T, rows,
                                                   ws_part, ws_count, out, mw);
            } else {
                __threadfence_block();  // the slot writes are visible before the finisher reads them
                named_bar_arrive(BAR_FULL0 + set, L::BAR_COUNT);
            }
        }
        sc.next(i, rb_c, ks_c);
    }
    cp_async_wait<0>();  // no copy outlives the kernel
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
