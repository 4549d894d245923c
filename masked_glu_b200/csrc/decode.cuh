// decode.cuh -- MGLU up-projection for few tokens (T <= 16), and the dense
// product (NM = 0) used as the decode-time down-projection.
//
// Memory-bound design ("Masked Gated Linear Unit", "Problem" and "Approach":
// decoding is bound by reading the weights, so each weight and its mask bits
// are read exactly once and the masks are unpacked inside the kernel):
//
//  * Work is made of units (row block of ROWS = 16 rows of W, step of
//    STEP = 64 k: two 32-k MMA units).  A persistent grid of one CTA per
//    SM gives every warp of the grid an equal contiguous range of units
//    (warp-level stream-K, see sched.cuh), so all warps stream the same
//    number of bytes and none ever waits for another while it streams.
//  * Each warp streams its units through a private ring of P stages in
//    shared memory: lane (g, c) copies (cp.async) 16 bytes of W rows g and
//    g + 8 per MMA unit (eight weights each) and their mask bits, P - 1 units
//    ahead of the one it multiplies, and reads back only what it copied
//    itself; x (small, read by every CTA) comes from L1 at the top of each
//    unit.  The copies are tracked by cp.async groups, not registers, so the
//    ring can be deep; no staged operand passes from one thread to another,
//    so the weight stream needs no barrier.
//  * Masks are applied by sign flips (see group_bits / flip_pair): the warp
//    accumulates the dense product D = x W and h_i = x (S_i . W) with
//    S_i = +1 where mask i is set and -1 where it is clear, on mma.sync
//    m16n8k16 with the 16 rows as M and the tokens as N; one LOP3 and one
//    shift per bf16 pair and mask build the operand.  Then g_i = (D + h_i)/2
//    and v_i = (D - h_i)/2 = D - g_i.
//  * A warp's range meets each row block in one segment.  A segment that
//    covers the whole row block is finished by the warp at once: each lane
//    holds every sum of its (row, token) pairs, so out = sum_i act(g_i) v_i,
//    rounded once to bf16, needs no exchange.  The range's first and last
//    segments may be partial: the first is dropped into a shared-memory head
//    slot, the last stays in registers.  After the stream (one __syncthreads,
//    no fences while copies are in flight) the CTA adds the partial segments
//    of each of its row blocks in warp order.  The first and last row block
//    of a CTA's range may also have units in other CTAs: their CTA sums go to
//    a small global scratch, and split_kernel, launched right after on the
//    same stream, adds them in CTA order.  Every sum is therefore formed in
//    a fixed order: results do not depend on timing.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"
#include "route.cuh"
#include "sched.cuh"

namespace mglu {
namespace dec {

constexpr int MAX_CTAS = 320;  // grid cap; sizes the split-row-block scratch
// floats of one CTA's partial of a split row block: the largest slot (n_m = 8,
// 16 tokens)
constexpr int PART_FLOATS = 9 * ROWS * 16;

// Token capacity TT of an instance (2, 8 or 16 tokens) and its 8-token
// MMA column blocks.
template <int TT>
constexpr int token_blocks()
{
    static_assert(TT == 2 || TT == 8 || TT == 16, "token capacity");
    return TT > 8 ? 2 : 1;
}

// Warps by n_m and token capacity.  Registers are allocated to warps in
// groups of four, so NW is a multiple of four: 16 warps get 128 registers a
// thread, 12 get 168, 8 get 255.
template <int NM, int TT>
struct DefaultShape {
    // n_m = 8 with 3 to 8 tokens: 8 warps of 255 registers, four MMA units
    // per unit of work (measured faster there; not at 1 or 2 tokens)
    static constexpr int NW = token_blocks<TT>() == 1 ? (NM == 8 && TT == 8 ? 8 : 16) : NM == 8 ? 8 : NM == 4 ? 12 : 16;
    static constexpr int UPW = NM == 8 && TT == 8 ? 4 : 2;  // 32-k MMA units a warp takes per unit of work
};

// A warp's slot holds its sums of a part compactly: float (v, row, tok) at
// (v * ROWS + row) * TT + tok for the instance's token capacity TT (v = 0 the
// dense product, 1 + i mask i).  Only the call's T tokens are written and
// added, so writing, adding and finishing a part cost in proportion to the
// tokens the call has, not to the MMA's 8 columns; the constant stride keeps
// every slot address a fixed offset from the lane's base.
template <int NM, int TT>
constexpr int slot_floats()
{
    return (NM + 1) * ROWS * TT;
}

template <int NM, int TT, int NW_ = DefaultShape<NM, TT>::NW>
struct Layout {
    static constexpr int NT = token_blocks<TT>();
    static constexpr int NW = NW_;                     // warps, each streaming its own unit range
    static constexpr int UPW = DefaultShape<NM, TT>::UPW;  // 32-k MMA units per unit of work
    static constexpr int STEP = 32 * UPW;              // k per unit of work
    static constexpr int NTHREADS = NW * 32;
    static constexpr int ACC = slot_floats<NM, TT>();  // floats of one warp's slot
    static constexpr int HEADS = NW * ACC;             // the warps' head slots
    // one stage of a warp's ring, per 32-k MMA unit u and lane: W rows g and
    // g + 8 (16 bytes each) and their mask bytes (n_m >= 4; narrower masks
    // go through registers), laid out lane-contiguous per row so that each
    // 16-byte read of a warp is conflict-free; x comes from L1 (its rows are
    // small and every warp of every CTA reads them)
    static constexpr int MB = NM >= 4 ? NM : 0;         // mask bytes per lane and row in the ring
    static constexpr int W_BYTES = 1024, M_BYTES = 64 * MB;
    static __host__ __device__ constexpr int w_a(int u) { return u * W_BYTES; }
    static __host__ __device__ constexpr int w_b(int u) { return u * W_BYTES + 512; }
    static __host__ __device__ constexpr int m_a(int u) { return UPW * W_BYTES + u * M_BYTES; }
    static __host__ __device__ constexpr int m_b(int u) { return UPW * W_BYTES + u * M_BYTES + 32 * MB; }
    static constexpr int STG = (UPW * (W_BYTES + M_BYTES) + 127) / 128 * 128;
    static constexpr int BUDGET = 227 * 1024;
    static constexpr int DEPTH = (BUDGET - HEADS * 4) / (NW * STG);
    static constexpr int P = DEPTH > 8 ? 8 : DEPTH;    // ring stages per warp
    static constexpr int RING_OFF = HEADS * 4;
    static constexpr int SMEM = RING_OFF + NW * P * STG;
    static_assert(NW % 4 == 0, "warps are allocated registers in groups of four");
    static_assert(P >= 3, "ring too shallow");
    static_assert(SMEM <= BUDGET, "shared memory");
    static_assert(HEADS <= NW * P * STG / 4, "the tail slots reuse the rings after the stream");
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

__device__ __forceinline__ uint4 ld_cached_16(const void *p)
{
    uint4 v;
    asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
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

// The shifts of the sign flips, v << (15 - I) for mask I, as integer
// multiplies by powers of two held in registers.  The value 1 they are made
// from is not known to the compiler, which would otherwise turn a constant
// shift into an ALU instruction: the ALU pipe already takes one LOP3 per
// flipped bf16 pair, so the shifts go to the FMA pipe instead.
template <int NM>
struct Shifts {
    uint32_t m[NM > 0 ? NM : 1];
    __device__ __forceinline__ void init(uint32_t one)
    {
#pragma unroll
        for (int i = 0; i < NM; ++i)
            m[i] = one << (15 - i);
    }
};

__device__ __forceinline__ uint32_t mul_u32(uint32_t v, uint32_t m)
{
    uint32_t r;
    asm("mul.lo.u32 %0, %1, %2;" : "=r"(r) : "r"(v), "r"(m));
    return r;
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
    // ra, rb: the group bits of rows g and g + 8 (mask I of the pair (4S, 4S+1)
    // at bits I and 16 + I); ra8, rb8 the same words shifted right by 8 (mask
    // I of the pair (4S+2, 4S+3) at those bits).  Shifting left by 15 - I puts
    // the bits at 15 and 31, the pairs' sign bits.
    static __device__ __forceinline__ void run(float (&acc)[NM + 1][NT][4], const Operands<NM, NT> &o, uint32_t ra,
                                               uint32_t rb, uint32_t ra8, uint32_t rb8, uint32_t used,
                                               const Shifts<NM> &sh)
    {
        if constexpr (I < NM) {
            if (!ROUTED || ((used >> I) & 1u)) {
                const uint32_t a0 = flip_pair(u4(o.wa, 2 * S), mul_u32(ra, sh.m[I]));
                const uint32_t a1 = flip_pair(u4(o.wb, 2 * S), mul_u32(rb, sh.m[I]));
                const uint32_t a2 = flip_pair(u4(o.wa, 2 * S + 1), mul_u32(ra8, sh.m[I]));
                const uint32_t a3 = flip_pair(u4(o.wb, 2 * S + 1), mul_u32(rb8, sh.m[I]));
#pragma unroll
                for (int t = 0; t < NT; ++t)
                    mma_bf16_16816(acc[1 + I][t], a0, a1, a2, a3, u4(o.xv[t], 2 * S), u4(o.xv[t], 2 * S + 1));
            }
            FlipLoop<NM, NT, ROUTED, S, I + 1>::run(acc, o, ra, rb, ra8, rb8, used, sh);
        }
    }
};

// One 16-row x 32-k unit.  Lane (g, c) holds weights [8c, 8c+8) of rows g
// and g+8; k16 sub-step S uses its bf16 pairs 2S and 2S+1.  The k order
// inside the MMA is a permutation of the physical k that depends only on c
// and S; x (operand B) is loaded with the same permutation, so every sum is
// unchanged.
template <int NM, int NT, bool ROUTED, int S>
__device__ __forceinline__ void unit_step(float (&acc)[NM + 1][NT][4], const Operands<NM, NT> &o, uint32_t used,
                                          const Shifts<NM> &sh)
{
#pragma unroll
    for (int t = 0; t < NT; ++t)
        mma_bf16_16816(acc[0][t], u4(o.wa, 2 * S), u4(o.wb, 2 * S), u4(o.wa, 2 * S + 1), u4(o.wb, 2 * S + 1),
                       u4(o.xv[t], 2 * S), u4(o.xv[t], 2 * S + 1));
    if constexpr (NM > 0) {
        const uint32_t ra = group_bits<NM, S>(o.ma.x, o.ma.y);
        const uint32_t rb = group_bits<NM, S>(o.mb.x, o.mb.y);
        FlipLoop<NM, NT, ROUTED, S, 0>::run(acc, o, ra, rb, ra >> 8, rb >> 8, used, sh);
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

// The partial sums of one (row, token) as float32 planes [2 NM + 1][T][rows]:
// D, then g_i and v_i for each mask i (the checking entry point's output).
template <int NM>
__device__ __forceinline__ void write_partials(float *__restrict__ gv, int64_t plane, int64_t at,
                                               const float (&sums)[NM + 1])
{
    const float D = sums[0];
    gv[at] = D;
#pragma unroll
    for (int i = 0; i < NM; ++i) {
        gv[(1 + 2 * i) * plane + at] = 0.5f * (D + sums[1 + i]);
        gv[(2 + 2 * i) * plane + at] = 0.5f * (D - sums[1 + i]);
    }
}

// The output of one (row, token) of row block rb from its NM + 1 sums (or,
// for the checking entry point, its partial sums).
template <int NM, bool ROUTED>
__device__ __forceinline__ void write_output(const float (&sums)[NM + 1], int rb, int row, int tok, int act, int T,
                                             int rows, __nv_bfloat16 *__restrict__ out,
                                             const float *__restrict__ mw, float *__restrict__ gv)
{
    const int r = rb * ROWS + row;
    if (r >= rows)
        return;
    const int64_t at = (int64_t)tok * rows + r;
    if (gv)
        write_partials<NM>(gv, (int64_t)T * rows, at, sums);
    else
        out[at] = __float2bfloat16_rn(out_value<NM>(act, sums, ROUTED ? mw + (int64_t)tok * NM : nullptr));
}

// After the stream, one warp per row block of its CTA's range: add the
// partial segments this CTA's warps hold of row block rb, in warp order (a
// warp's first segment sits in its head slot, its last in its tail slot),
// then write the outputs, or, if other CTAs also hold units of rb, store
// this CTA's sums for split_kernel.  A row block that one warp covered whole
// was finished by that warp already.
template <int NM, int TT, bool ROUTED>
__device__ __noinline__ void combine_cta(int rb, const Plan pl, const float *__restrict__ heads,
                                         const float *__restrict__ tails, int act, int T, int rows,
                                         float *__restrict__ ws_part, __nv_bfloat16 *__restrict__ out,
                                         const float *__restrict__ mw, float *__restrict__ gv)
{
    constexpr int ACC = slot_floats<NM, TT>();
    const int lane = threadIdx.x & 31;
    const int cta = blockIdx.x, w0 = cta * pl.NW;
    const uint32_t ub = (uint32_t)rb * (uint32_t)pl.nsw, ue = ub + (uint32_t)pl.nsw;
    int w_lo = pl.owner(ub), w_hi = pl.owner(ue - 1u);
    if (w_lo == w_hi)
        return;  // one warp covered it whole
    w_lo = w_lo > w0 ? w_lo : w0;
    w_hi = w_hi < w0 + pl.NW - 1 ? w_hi : w0 + pl.NW - 1;
    int c_first, c_last;
    pl.ctas_of(rb, c_first, c_last);
    float *mine = c_first != c_last ? ws_part + (int64_t)pl.slot(cta, rb) * PART_FLOATS : nullptr;
#pragma unroll 1
    for (int p = lane; p < ROWS * T; p += 32) {
        const int row = p / T, tok = p - row * T;
        float sums[NM + 1];
#pragma unroll
        for (int v = 0; v <= NM; ++v)
            sums[v] = 0.f;
#pragma unroll 1
        for (int w = w_lo; w <= w_hi; ++w) {
            const uint32_t b = pl.begin(w), e = pl.begin(w + 1);
            if (b == e)
                continue;  // an empty range (more warps than units) holds nothing
            // warp w's first row block is its head segment unless it is also its last
            const int first = (int)(b / (uint32_t)pl.nsw), last = (int)((e - 1u) / (uint32_t)pl.nsw);
            const float *src = (rb == first && first != last ? heads : tails) + (w - w0) * ACC;
#pragma unroll
            for (int v = 0; v <= NM; ++v)
                sums[v] += src[(v * ROWS + row) * TT + tok];
        }
        if (mine) {
#pragma unroll
            for (int v = 0; v <= NM; ++v)
                mine[(v * ROWS + row) * TT + tok] = sums[v];
        } else {
            write_output<NM, ROUTED>(sums, rb, row, tok, act, T, rows, out, mw, gv);
        }
    }
}

// Row blocks whose units several CTAs hold: the first CTA of each (for which
// it is the last row block of its range) adds every CTA's stored sums in CTA
// order and writes the outputs.  Launched after the decode kernel on the same
// stream (its stores are visible once it has completed); one warp per CTA of
// that grid, most of which have nothing to do.
template <int NM, int TT, bool ROUTED>
__global__ void __launch_bounds__(32) split_kernel(int rows, int d, int step, int grid, int nw, int T, int act,
                                                   const float *__restrict__ ws_part,
                                                   __nv_bfloat16 *__restrict__ out, const float *__restrict__ mw,
                                                   float *__restrict__ gv)
{
    pdl_launch_dependents();
    Plan pl;
    pl.init(rows, d, step, grid, nw);
    const int c = blockIdx.x;
    if (!pl.cta_has_units(c))
        return;
    const int rb = pl.last_rb(c);
    int c_first, c_last;
    pl.ctas_of(rb, c_first, c_last);
    if (c_first == c_last || c_first != c)
        return;
    pdl_wait();  // the decode kernel has completed
    const int lane = threadIdx.x;
#pragma unroll 1
    for (int p = lane; p < ROWS * T; p += 32) {
        const int row = p / T, tok = p - row * T;
        float sums[NM + 1];
#pragma unroll
        for (int v = 0; v <= NM; ++v)
            sums[v] = 0.f;
#pragma unroll 1
        for (int cc = c_first; cc <= c_last; ++cc) {
            if (!pl.cta_has_units(cc))
                continue;
            const float *src = ws_part + (int64_t)pl.slot(cc, rb) * PART_FLOATS;
#pragma unroll
            for (int v = 0; v <= NM; ++v)
                sums[v] += src[(v * ROWS + row) * TT + tok];
        }
        write_output<NM, ROUTED>(sums, rb, row, tok, act, T, rows, out, mw, gv);
    }
}

// In-kernel routing (ROUTED instances).  When Wr is not NULL the kernel
// scores and routes every token itself, with the arithmetic of route_kernel
// (route_partial / route_select, so the weights equal mglu_route_topk's bit
// for bit), before its stream starts; every CTA keeps its own copy of the
// weights in shared memory, and CTA 0 also stores them (and the scores) for
// the caller and for split_kernel.
struct Router {
    const __nv_bfloat16 *Wr;  // [NM][d]; NULL: the weights come in mw
    int k, mode, vec;         // kept masks, ROUTE_HARD / ROUTE_SOFTMAX, 16-byte rows
    float *weights, *scores;  // [T][NM] outputs (scores may be NULL)
};

// The decode kernel.  Scratch (global, caller-provided): this CTA's sums of
// the first and the last row block of its range when other CTAs also hold
// units of them (read by split_kernel); it needs no initialization.
//
// ROUTED: per-token mask weights mw [T][NM] scale each mask's term, and a
// mask that no token of the call weights (all its weights zero) skips its
// products (the weight stream is read in full either way).
// gv (not NULL): write the partial sums D, g_i, v_i instead of outputs.
template <int NM, int TT, bool ROUTED = false, int NW_ = DefaultShape<NM, TT>::NW>
__global__ void __launch_bounds__(Layout<NM, TT, NW_>::NTHREADS, 1)
    decode_kernel(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ W,
                  const uint8_t *__restrict__ packed, int T, int rows, int d, int act, float *__restrict__ ws_part,
                  __nv_bfloat16 *__restrict__ out, const float *__restrict__ mw, float *__restrict__ gv, Router ro)
{
    using L = Layout<NM, TT, NW_>;
    constexpr int NT = L::NT;
    extern __shared__ __align__(128) float slots[];  // the warps' head slots, then their rings

    // The next kernel in the stream may start its prologue now; every access
    // to global memory below waits for the previous kernel to finish.
    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, c = lane & 3;
    Plan pl;
    pl.init(rows, d, L::STEP, gridDim.x, L::NW);
    if (!pl.cta_has_units(blockIdx.x))
        return;
    const int gw = blockIdx.x * L::NW + warp;
    const uint32_t u0 = pl.begin(gw), u1 = pl.begin(gw + 1);
    const int n = (int)(u1 - u0);  // this warp's units
    const int nsw = pl.nsw;
    pdl_wait();

    Shifts<NM> sh;
    sh.init(1u + ((uint32_t)act >> 16));  // act < 2^16: the value is 1

    // the mask weights the epilogue reads: mw, or the kernel's own routing
    // (computed below, after the first copies of the stream are issued)
    __shared__ float s_mw[ROUTED ? 16 * (NM > 0 ? NM : 1) : 1];
    const float *mwk = mw;
    // masks some token of the call weights
    uint32_t used = (1u << NM) - 1u;

    // Unit (rb, s) covers k = s * STEP + 32 u + [0, 32) for MMA units u of
    // rows rb * ROWS + [0, 16); this lane's 8 weights of MMA unit u start at
    // k = s * STEP + 32 u + 8 c.
    const int kl = 8 * c;
    const int64_t mrow = (int64_t)d * NM / 8;  // mask bytes per row of W
    int xrow[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t)
        xrow[t] = 8 * t + g < T ? 8 * t + g : T - 1;  // lanes of absent tokens repeat the last one
    uint8_t *ring = reinterpret_cast<uint8_t *>(slots) + L::RING_OFF + warp * L::P * L::STG;
    const uint32_t ring_s = smem_u32(ring);

    // The copy cursor: the unit it copies next and this lane's source
    // pointers for it (rows g and g + 8 of the row block).  Inside a row
    // block the pointers advance by one unit; a new row block recomputes them.
    struct Cursor {
        int rb, s;
        bool rows_in;  // all 16 rows of the row block exist
        const __nv_bfloat16 *wa, *wb;
        const uint8_t *ma, *mb;
    };
    const int kfull = d / L::STEP;  // units that lie wholly inside the row
    auto place = [&](Cursor &cu) {
        const int ra = cu.rb * ROWS + g;
        const int k = cu.s * L::STEP + kl;
        cu.rows_in = cu.rb * ROWS + ROWS <= rows;
        cu.wa = W + (int64_t)ra * d + k;
        cu.wb = cu.wa + 8 * (int64_t)d;
        cu.ma = packed + (int64_t)ra * mrow + (int64_t)k * NM / 8;
        cu.mb = cu.ma + 8 * mrow;
    };
    auto advance = [&](Cursor &cu) {
        if (++cu.s < nsw) {
            cu.wa += L::STEP, cu.wb += L::STEP;
            cu.ma += L::STEP * NM / 8, cu.mb += L::STEP * NM / 8;
        } else {
            cu.s = 0;
            ++cu.rb;
            place(cu);
        }
    };
    // Copies of the cursor's unit into ring stage ss.  A unit wholly inside
    // the matrix copies without checks; otherwise lanes outside it copy
    // zeros (a d % 8 == 0 row keeps a lane's 8 weights all in or out).
    // Mask bytes (n_m >= 4): the four lanes of a group g hold 4 * MB
    // contiguous bytes per row and MMA unit, so when the packed rows are
    // 16-byte strided the group copies them in 16-byte pieces (lane c takes
    // pieces c, c + 4, ...), a quarter (n_m = 4) or half (n_m = 8) as many
    // copies as one per lane; the lanes then read each other's bytes after a
    // __syncwarp.  Otherwise every lane copies its own MB bytes.
    constexpr int MH = L::MB / 4 > 0 ? L::MB / 4 : 1;  // 16-byte pieces per row and MMA unit
    constexpr int MPL = 2 * L::UPW * MH / 4;           // pieces per lane
    const bool mask16 = L::MB > 0 && mrow % 16 == 0;
    auto issue_masks16 = [&](uint32_t stage, const Cursor &cu, bool checked) {
        const uint8_t *ma0 = cu.ma - c * L::MB, *mb0 = cu.mb - c * L::MB;  // the group's first bytes
        const int ra = cu.rb * ROWS + g;
#pragma unroll
        for (int j = 0; j < MPL; ++j) {
            const int q = c + 4 * j;
            const int row = q / (L::UPW * MH), u = (q / MH) % L::UPW, half = q % MH;
            const uint8_t *src = (row ? mb0 : ma0) + u * (32 * NM / 8) + half * 16;
            const uint32_t dst = stage + (row ? L::m_b(u) : L::m_a(u)) + g * 4 * L::MB + half * 16;
            if (!checked) {
                cp_async_cg16(dst, src);
            } else {
                constexpr int PW = 128 / (NM > 0 ? NM : 1);  // weights per 16-byte piece
                const int kp = cu.s * L::STEP + 32 * u + half * PW;  // first weight of the piece
                const int wts = d - kp < PW ? d - kp : PW;
                const bool ok = wts > 0 && ra + 8 * row < rows;
                cp_async_cg16(dst, ok ? src : packed, ok ? (uint32_t)(wts * NM / 8) : 0u);
            }
        }
    };
    // Copies of the cursor's unit into ring stage ss.  A unit wholly inside
    // the matrix copies without checks; otherwise lanes outside it copy
    // zeros (a d % 8 == 0 row keeps a lane's 8 weights all in or out).
    auto issue = [&](int ss, const Cursor &cu) {
        const uint32_t stage = ring_s + (uint32_t)(ss * L::STG);
        const uint32_t st = stage + lane * 16;
        const uint32_t sm = stage + lane * L::MB;
        if (cu.rows_in && cu.s < kfull) {
#pragma unroll
            for (int u = 0; u < L::UPW; ++u) {
                cp_async_cg16(st + L::w_a(u), cu.wa + 32 * u);
                cp_async_cg16(st + L::w_b(u), cu.wb + 32 * u);
            }
            if constexpr (L::MB > 0) {
                if (mask16) {
                    issue_masks16(stage, cu, false);
                } else {
#pragma unroll
                    for (int u = 0; u < L::UPW; ++u) {
                        cp_async_ca<L::MB>(sm + L::m_a(u), cu.ma + 32 * u * NM / 8);
                        cp_async_ca<L::MB>(sm + L::m_b(u), cu.mb + 32 * u * NM / 8);
                    }
                }
            }
        } else {
            const int ra = cu.rb * ROWS + g;
#pragma unroll
            for (int u = 0; u < L::UPW; ++u) {
                const bool kin = cu.s * L::STEP + kl + 32 * u < d;
                const bool va = kin && ra < rows, vb = kin && ra + 8 < rows;
                cp_async_cg16(st + L::w_a(u), va ? cu.wa + 32 * u : W, va ? 16u : 0u);
                cp_async_cg16(st + L::w_b(u), vb ? cu.wb + 32 * u : W, vb ? 16u : 0u);
                if constexpr (L::MB > 0) {
                    if (!mask16) {
                        cp_async_ca<L::MB>(sm + L::m_a(u), va ? cu.ma + 32 * u * NM / 8 : packed,
                                           va ? (uint32_t)L::MB : 0u);
                        cp_async_ca<L::MB>(sm + L::m_b(u), vb ? cu.mb + 32 * u * NM / 8 : packed,
                                           vb ? (uint32_t)L::MB : 0u);
                    }
                }
            }
            if constexpr (L::MB > 0) {
                if (mask16)
                    issue_masks16(stage, cu, true);
            }
        }
    };
    // x of a unit comes from L1 (its rows are small and every warp reads
    // them), loaded at the top of the unit's iteration; for n_m <= 2 the
    // narrow mask bits (one or two bytes a lane and row) stream from memory
    // into registers one unit ahead.
    const __nv_bfloat16 *xl[NT];  // this lane's x rows at its k offset
#pragma unroll
    for (int t = 0; t < NT; ++t)
        xl[t] = x + (int64_t)xrow[t] * d + kl;
    auto load_x = [&](uint4 (&xv)[L::UPW][NT], int s) {
        const int k0 = s * L::STEP;
        if (s < kfull) {
#pragma unroll
            for (int u = 0; u < L::UPW; ++u)
#pragma unroll
                for (int t = 0; t < NT; ++t)
                    xv[u][t] = ld_cached_16(xl[t] + k0 + 32 * u);
        } else {
#pragma unroll
            for (int u = 0; u < L::UPW; ++u)
#pragma unroll
                for (int t = 0; t < NT; ++t)
                    xv[u][t] = k0 + kl + 32 * u < d ? ld_cached_16(xl[t] + k0 + 32 * u) : make_uint4(0u, 0u, 0u, 0u);
        }
    };
    struct NarrowMasks {
        uint2 a[L::UPW], b[L::UPW];
    };
    auto load_narrow = [&](NarrowMasks &nm, int rb, int s) {
        const int ra = rb * ROWS + g, rbb = ra + 8;
#pragma unroll
        for (int u = 0; u < L::UPW; ++u) {
            const int k = s * L::STEP + kl + 32 * u;
            const bool kin = k < d;
            nm.a[u] = nm.b[u] = make_uint2(0u, 0u);
            if (kin && ra < rows)
                nm.a[u] = ld_mask_chunk<NM>(packed + (int64_t)ra * mrow + (int64_t)k * NM / 8);
            if (kin && rbb < rows)
                nm.b[u] = ld_mask_chunk<NM>(packed + (int64_t)rbb * mrow + (int64_t)k * NM / 8);
        }
    };
    constexpr bool NARROW = NM > 0 && L::MB == 0;

    float acc[NM + 1][NT][4];
    zero_acc<NM, NT>(acc);
    // a warp's sums of a segment into a slot, compactly (see slot_floats)
    auto write_slot = [&](float *slot) {
#pragma unroll
        for (int v = 0; v <= NM; ++v)
#pragma unroll
            for (int t = 0; t < NT; ++t)
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int tok = 8 * t + 2 * c + (r & 1), row = g + 8 * (r >> 1);
                    if (tok < T)
                        slot[(v * ROWS + row) * TT + tok] = acc[v][t][r];
                }
    };
    // a row block this warp covered whole: every lane holds all NM + 1 sums
    // of its (row, token) pairs, so it writes their outputs directly
    auto finish_whole = [&](int rb) {
#pragma unroll
        for (int t = 0; t < NT; ++t)
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const int tok = 8 * t + 2 * c + (r & 1), row = g + 8 * (r >> 1);
                if (tok < T) {
                    float sums[NM + 1];
#pragma unroll
                    for (int v = 0; v <= NM; ++v)
                        sums[v] = acc[v][t][r];
                    write_output<NM, ROUTED>(sums, rb, row, tok, act, T, rows, out, mwk, gv);
                }
            }
    };

    // the copy cursor runs P - 1 units ahead of the compute cursor
    int rb_c = (int)(u0 / (uint32_t)nsw), s_c = (int)(u0 % (uint32_t)nsw);
    int seg_start = s_c;  // first unit of the current segment
    Cursor cl;
    cl.rb = rb_c, cl.s = s_c;
    place(cl);
    for (int b = 0; b < L::P - 1; ++b) {
        if (b < n)
            issue(b, cl);
        cp_async_commit();  // one group per unit, empty past the end
        if (b + 1 < n)
            advance(cl);
    }
    NarrowMasks nmask;
    if constexpr (NARROW) {
        if (n > 0)
            load_narrow(nmask, rb_c, s_c);
    }

    // routing in the kernel, while the first copies are in flight
    if constexpr (ROUTED) {
        if (ro.Wr) {
            // the token groups' warp sums go to the head slots, which no warp
            // writes before its first segment ends (T * 64 floats; the slots
            // hold NW * (NM + 1) * 16 * TT >= 256 * TT of them)
            float(*part)[8][8] = reinterpret_cast<float(*)[8][8]>(slots);
            constexpr int G = L::NTHREADS / 256;  // groups of 256 threads, one token each at a time
            const int vt = threadIdx.x & 255, grp = threadIdx.x >> 8;
            if (grp < G) {
#pragma unroll 1
                for (int t = grp; t < T; t += G) {
                    float a8[8];
                    route_partial<__nv_bfloat16>(x + (int64_t)t * d, d, ro.Wr, NM, ro.vec, vt, a8);
                    if ((vt & 31) == 0)
#pragma unroll
                        for (int i = 0; i < 8; ++i)
                            part[t][vt >> 5][i] = a8[i];
                }
            }
            __syncthreads();
            if (threadIdx.x < T) {
                const int t = threadIdx.x;
                route_select(part[t], NM, ro.k, ro.mode, &s_mw[t * NM],
                             blockIdx.x == 0 && ro.scores ? ro.scores + (int64_t)t * NM : nullptr);
                if (blockIdx.x == 0)
#pragma unroll
                    for (int i = 0; i < NM; ++i)
                        ro.weights[(int64_t)t * NM + i] = s_mw[t * NM + i];
            }
            __syncthreads();
            mwk = s_mw;
        }
    }

    if constexpr (ROUTED) {
        uint32_t u = 0;
        for (int e = lane; e < T * NM; e += 32)
            u |= (mwk[e] != 0.0f ? 1u : 0u) << (e % NM);
        used = __reduce_or_sync(0xffffffffu, u);
    }
    bool tail = false;  // the last segment is partial: its sums stay in acc
    for (int i = 0; i < n; ++i) {
        uint4 xv[L::UPW][NT];
        load_x(xv, s_c);
        const int il = i + L::P - 1;
        if (il < n)
            issue(il % L::P, cl);
        cp_async_commit();
        if (il + 1 < n)
            advance(cl);
        int rb_n = rb_c, s_n = s_c + 1;
        if (s_n == nsw)
            s_n = 0, ++rb_n;
        NarrowMasks cur;
        if constexpr (NARROW) {
            cur = nmask;
            if (i + 1 < n)
                load_narrow(nmask, rb_n, s_n);
        }
        cp_async_wait<L::P - 1>();  // this lane's copies of unit i have landed
        if constexpr (L::MB > 0)
            __syncwarp();  // and, for the shared mask pieces, every lane's

        // Units past the end of the row (a ragged last unit) hold zeros in
        // the ring and in x, so they add nothing.
        const uint8_t *st = ring + (i % L::P) * L::STG;
#pragma unroll
        for (int u = 0; u < L::UPW; ++u) {
            Operands<NM, NT> o;
            o.wa = *reinterpret_cast<const uint4 *>(st + L::w_a(u) + lane * 16);
            o.wb = *reinterpret_cast<const uint4 *>(st + L::w_b(u) + lane * 16);
#pragma unroll
            for (int t = 0; t < NT; ++t)
                o.xv[t] = xv[u][t];
            if constexpr (L::MB == 8) {
                o.ma = *reinterpret_cast<const uint2 *>(st + L::m_a(u) + lane * 8);
                o.mb = *reinterpret_cast<const uint2 *>(st + L::m_b(u) + lane * 8);
            } else if constexpr (L::MB == 4) {
                o.ma = make_uint2(*reinterpret_cast<const uint32_t *>(st + L::m_a(u) + lane * 4), 0u);
                o.mb = make_uint2(*reinterpret_cast<const uint32_t *>(st + L::m_b(u) + lane * 4), 0u);
            } else if constexpr (NARROW) {
                o.ma = cur.a[u];
                o.mb = cur.b[u];
            } else {
                o.ma = o.mb = make_uint2(0u, 0u);
            }
            unit_step<NM, NT, ROUTED, 0>(acc, o, used, sh);
            unit_step<NM, NT, ROUTED, 1>(acc, o, used, sh);
        }
        if (s_c == nsw - 1 || i == n - 1) {
            // ---------------------------------------------- a segment ends here
            if (seg_start == 0 && s_c == nsw - 1) {
                finish_whole(rb_c);
                zero_acc<NM, NT>(acc);
            } else if (i < n - 1) {
                write_slot(slots + warp * L::ACC);  // the head: the range's first segment
                zero_acc<NM, NT>(acc);
            } else {
                tail = true;
            }
            seg_start = 0;
        }
        rb_c = rb_n, s_c = s_n;
    }
    cp_async_wait<0>();  // no copy outlives the stream

    // After the stream: the partial segments of the CTA's row blocks.
    float *tails = slots + L::HEADS;  // the rings are free once every warp is here
    __syncthreads();
    if (tail)
        write_slot(tails + warp * L::ACC);
    __syncthreads();
    const int rb_last = pl.last_rb(blockIdx.x);
#pragma unroll 1
    for (int rb = pl.first_rb(blockIdx.x) + warp; rb <= rb_last; rb += L::NW)
        combine_cta<NM, TT, ROUTED>(rb, pl, slots, tails, act, T, rows, ws_part, out, mwk, gv);
}

// Scratch bytes of the decode kernel: two partial slots per CTA.
__host__ __device__ constexpr int64_t part_bytes() { return (int64_t)2 * MAX_CTAS * PART_FLOATS * 4; }
__host__ __device__ constexpr int64_t workspace_bytes(int64_t) { return part_bytes(); }

}  // namespace dec
}  // namespace mglu
