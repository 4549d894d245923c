// decode.cuh -- MGLU up-projection for few tokens (T <= 16), and the dense
// product (NM = 0) used as the decode-time down-projection.
//
// Memory-bound design ("Masked Gated Linear Unit", "Problem" and "Approach":
// decoding is bound by reading the weights, so each weight and its mask bits
// are read exactly once and the masks are unpacked inside the kernel):
//
//  * Work is made of stages (row block of ROWS = 16 rows of W, k-stage of
//    KS = 64 * NW k: two 32-k units per warp).  A persistent grid of
//    one CTA per SM splits the stages evenly: every CTA gets the same number
//    of whole row blocks (data-parallel part) plus an equal contiguous share
//    of the stages of the remaining row blocks (stream-K part), so all SMs
//    stream the same number of bytes.  Each CTA does its stream-K share
//    first, so the combining of row blocks split between CTAs overlaps the
//    data-parallel part instead of trailing the kernel.
//  * Each warp streams its own units of every stage through a private ring of
//    P stages in shared memory: lane (g, c) copies (cp.async) 16 bytes of W
//    rows g and g + 8 per unit (eight weights each) and their mask bits,
//    P - 1 stages ahead of the one it multiplies, and reads back only what
//    it copied itself; x (small, read by every CTA) comes from L1 one stage
//    ahead.  The copies are tracked by
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
//    in a fixed order and finish the part.  It releases the set as soon as
//    it has read it.  A row block whose k range lies
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
// floats of one CTA's partial of a split row block: the largest slot (n_m = 8,
// 16 tokens)
constexpr int PART_FLOATS = 9 * ROWS * 16;
// named barriers: slot set b is full (writers arrive, the part's finisher
// waits); a set is free again for part f (the finisher of part f - SETS
// arrives once it has read it, the other warps wait) on FREE0 + f % 2
constexpr int BAR_FULL0 = 1;
constexpr int BAR_FREE0 = 3;
// cooperative finishing (token capacity 8 or 16): the reducer warps' own
// barrier
constexpr int BAR_READ = 5;

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
    static constexpr int NW = token_blocks<TT>() == 1 ? 16 : NM == 8 ? 8 : NM == 4 ? 12 : 16;
};

// A warp's slot holds its sums of a part compactly: float (v, row, tok) at
// (v * ROWS + row) * T + tok for the call's T tokens (v = 0 the dense
// product, 1 + i mask i), so writing, adding and finishing a part cost in
// proportion to the tokens the call has, not to the MMA's 8 columns.
template <int NM, int TT>
constexpr int slot_floats()
{
    return (NM + 1) * ROWS * TT;
}

template <int NM, int TT, int NW_ = DefaultShape<NM, TT>::NW>
struct Layout {
    static constexpr int NT = token_blocks<TT>();
    static constexpr int NW = NW_;                     // warps, each a consumer and in turn a finisher
    static constexpr int UPW = 2;                      // 32-k units per warp and stage
    static constexpr int NTHREADS = NW * 32;
    static constexpr int BAR_COUNT = NW * 32;
    static constexpr int KS = NW * 32 * UPW;           // k per stage
    static constexpr int ACC = slot_floats<NM, TT>();  // floats of one warp's slot
    static constexpr int SLOT_SET = NW * ACC;          // floats of one slot set
    // one stage of a warp's ring, per unit u and lane: W rows g and g + 8
    // (16 bytes each) and their mask bytes (n_m >= 4; narrower masks go
    // through registers), laid out lane-contiguous per row so that each
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
    static constexpr int ring_depth(int sets) { return (BUDGET - sets * SLOT_SET * 4) / (NW * STG); }
    // two slot sets when a set is small (an eighth of shared memory at
    // most), so a part's finisher never holds up the next part; else one,
    // leaving the room to the ring
    static constexpr int SETS = TT <= 2 && SLOT_SET * 4 <= BUDGET / 8 ? 2 : 1;
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

// Finish row-block part f (the calling warp is its finisher) from the NW
// slots of its set (compact, see slot_floats): add them element by element
// in warp order into the warp's own slot, arrive on FREE barrier free_bar (if
// not 0: a later part reuses the set; the own slot is written again only by
// this warp), then either write the outputs or, for a row block split
// between CTAs, publish this CTA's partial sums and let the last CTA to
// arrive add all partials in CTA order and write them.  Not inlined: it runs
// once per part, and keeping its registers out of the streaming loop leaves
// that loop without spills.
template <int NM, bool ROUTED, int NW>
__device__ __noinline__ void finish_part(float *__restrict__ set_base, int slot_cap, int rb, bool stream_k,
                                         int free_bar, const Sched sc, int act, int T, int rows,
                                         float *__restrict__ ws_part, int *__restrict__ ws_count,
                                         __nv_bfloat16 *__restrict__ out, const float *__restrict__ mw,
                                         float *__restrict__ gv)
{
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int E = (NM + 1) * ROWS * T;  // sums of the part
    float *own = set_base + warp * slot_cap;
#pragma unroll 1
    for (int e = lane; e < E; e += 32) {
        float v[NW];
#pragma unroll
        for (int w = 0; w < NW; ++w)
            v[w] = set_base[w * slot_cap + e];
        float s = v[0];
#pragma unroll
        for (int w = 1; w < NW; ++w)
            s += v[w];
        own[e] = s;  // element e of the own slot was read above, by this lane
    }
    if (free_bar) {
        __threadfence_block();  // the slot reads above come before the set is written again
        named_bar_arrive(free_bar, NW * 32);  // the other warps may write this set again
    }
    bool finish = true;
    if (stream_k) {
        int c_first, c_last;
        const int nparts = sc.contributors(rb, c_first, c_last);
        if (c_first != c_last) {
            float *mine = ws_part + (int64_t)sc.slot(sc.cta, rb) * PART_FLOATS;
#pragma unroll 1
            for (int e = lane; e < E; e += 32)
                __stcg(mine + e, own[e]);
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
#pragma unroll 1
                for (int e = lane; e < E; e += 32) {
                    float s = 0.f;
#pragma unroll 1
                    for (int cc = c_first; cc <= c_last; ++cc)
                        if (sc.contributes(cc))
                            s += __ldcg(ws_part + (int64_t)sc.slot(cc, rb) * PART_FLOATS + e);
                    own[e] = s;
                }
                if (lane == 0)
                    ws_count[rb] = 0;  // leave the scratch zeroed for the next call
            }
        }
    }
    if (finish) {
        __syncwarp();  // every lane's sums are in the own slot
        const int row0 = rb * ROWS;
        const int64_t plane = (int64_t)T * rows;
#pragma unroll 1
        for (int p = lane; p < ROWS * T; p += 32) {
            const int row = p / T, tok = p - row * T;
            if (row0 + row >= rows)
                continue;
            float sums[NM + 1];
#pragma unroll
            for (int v = 0; v <= NM; ++v)
                sums[v] = own[(v * ROWS + row) * T + tok];
            const int64_t at = (int64_t)tok * rows + row0 + row;
            if (gv)
                write_partials<NM>(gv, plane, at, sums);
            else
                out[at] = __float2bfloat16_rn(out_value<NM>(act, sums, ROUTED ? mw + (int64_t)tok * NM : nullptr));
        }
    }
}

// Cooperative finishing of part f for token capacities 8 and 16, run by the
// reducer warps (the first R = ceil(16 T / 32) warps), one thread per
// (row, token) of the row block: it adds that output's NM + 1 sums over the
// NW slots in warp order, the reducers meet on BAR_READ (every slot is read)
// and, if a later part exists and some warps are not reducers, arrive on
// FREE so those warps may write the set again.  A row block split between
// CTAs is finished as in finish_part, by whichever CTA arrives last.
template <int NM, bool ROUTED, int NW>
__device__ __noinline__ void finish_coop(const float *__restrict__ set_base, int slot_cap, int rb, bool stream_k,
                                         int R, bool free_arrive, const Sched sc, int act, int T, int rows,
                                         float *__restrict__ ws_part, int *__restrict__ ws_count,
                                         __nv_bfloat16 *__restrict__ out, const float *__restrict__ mw,
                                         float *__restrict__ gv)
{
    __shared__ int s_last;
    const int p = threadIdx.x;  // (row, token) of this thread
    const bool has = p < ROWS * T;
    const int row = has ? p / T : 0, tok = has ? p - row * T : 0;
    float sums[NM + 1];
#pragma unroll
    for (int v = 0; v <= NM; ++v) {
        float acc = 0.f;
        if (has) {
            const float *q = set_base + (v * ROWS + row) * T + tok;
            acc = q[0];
#pragma unroll
            for (int w = 1; w < NW; ++w)
                acc += q[w * slot_cap];
        }
        sums[v] = acc;
    }
    named_bar_sync(BAR_READ, R * 32);  // every reducer has read the set
    if (free_arrive) {
        __threadfence_block();
        named_bar_arrive(BAR_FREE0, NW * 32);
    }
    bool finish = true;
    if (stream_k) {
        int c_first, c_last;
        const int nparts = sc.contributors(rb, c_first, c_last);
        if (c_first != c_last) {
            float *mine = ws_part + (int64_t)sc.slot(sc.cta, rb) * PART_FLOATS;
            if (has) {
#pragma unroll
                for (int v = 0; v <= NM; ++v)
                    __stcg(mine + (v * ROWS + row) * T + tok, sums[v]);
            }
            __threadfence();
            named_bar_sync(BAR_READ, R * 32);  // this CTA's partial is published
            if (p == 0)
                s_last = atomicAdd(ws_count + rb, 1) == nparts - 1;
            named_bar_sync(BAR_READ, R * 32);
            finish = s_last != 0;
            if (finish) {
                // every partial, this CTA's included, read back in CTA order
                __threadfence();
                if (has) {
#pragma unroll
                    for (int v = 0; v <= NM; ++v) {
                        float acc = 0.f;
#pragma unroll 1
                        for (int cc = c_first; cc <= c_last; ++cc)
                            if (sc.contributes(cc))
                                acc += __ldcg(ws_part + (int64_t)sc.slot(cc, rb) * PART_FLOATS +
                                              (v * ROWS + row) * T + tok);
                        sums[v] = acc;
                    }
                }
                if (p == 0)
                    ws_count[rb] = 0;  // leave the scratch zeroed for the next call
            }
        }
    }
    const int row0 = rb * ROWS;
    if (finish && has && row0 + row < rows) {
        const int64_t at = (int64_t)tok * rows + row0 + row;
        if (gv)
            write_partials<NM>(gv, (int64_t)T * rows, at, sums);
        else
            out[at] = __float2bfloat16_rn(out_value<NM>(act, sums, ROUTED ? mw + (int64_t)tok * NM : nullptr));
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
template <int NM, int TT, bool ROUTED = false, int NW_ = DefaultShape<NM, TT>::NW>
__global__ void __launch_bounds__(Layout<NM, TT, NW_>::NTHREADS, 1)
    decode_kernel(const __nv_bfloat16 *__restrict__ x, const __nv_bfloat16 *__restrict__ W,
                  const uint8_t *__restrict__ packed, int T, int rows, int d, int act, float *__restrict__ ws_part,
                  int *__restrict__ ws_count, __nv_bfloat16 *__restrict__ out, const float *__restrict__ mw,
                  float *__restrict__ gv)
{
    using L = Layout<NM, TT, NW_>;
    constexpr int NT = L::NT;
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
    // This warp's units of stage ks start at k = ks * KS + 32 * (UPW * warp + u);
    // this lane's 8 weights of unit u at k = that + 8 * c.
    const int kl = 32 * L::UPW * warp + 8 * c;
    const int64_t mrow = (int64_t)d * NM / 8;  // mask bytes per row of W
    int xrow[NT];
#pragma unroll
    for (int t = 0; t < NT; ++t)
        xrow[t] = 8 * t + g < T ? 8 * t + g : T - 1;  // lanes of absent tokens repeat the last one
    uint8_t *ring = reinterpret_cast<uint8_t *>(slots) + L::RING_OFF + warp * L::P * L::STG;
    const uint32_t ring_s = smem_u32(ring);

    // The copy cursor: the stage it copies next and this lane's source
    // pointers for it (rows g and g + 8 of the row block, k of the lane's
    // piece of the warp's first unit).  Inside a row block the pointers
    // advance by one stage; a new row block recomputes them.
    struct Cursor {
        int rb, ks;
        bool rows_in;  // all 16 rows of the row block exist
        const __nv_bfloat16 *wa, *wb;
        const uint8_t *ma, *mb;
    };
    const int kfull = d / L::KS;  // k-stages that lie wholly inside the row
    auto place = [&](Cursor &cu) {
        const int ra = cu.rb * ROWS + g;
        const int k = cu.ks * L::KS + kl;
        cu.rows_in = cu.rb * ROWS + ROWS <= rows;
        cu.wa = W + (int64_t)ra * d + k;
        cu.wb = cu.wa + 8 * (int64_t)d;
        cu.ma = packed + (int64_t)ra * mrow + (int64_t)k * NM / 8;
        cu.mb = cu.ma + 8 * mrow;
    };
    auto advance = [&](int i, Cursor &cu) {  // past unit i of this CTA
        sc.next(i, cu.rb, cu.ks);
        if (cu.ks != 0) {
            cu.wa += L::KS, cu.wb += L::KS;
            cu.ma += L::KS * NM / 8, cu.mb += L::KS * NM / 8;
        } else {
            place(cu);
        }
    };
    // Copies of the cursor's stage into ring stage ss.  A stage wholly inside
    // the matrix copies without checks; otherwise lanes outside it copy
    // zeros (a d % 8 == 0 row keeps a lane's 8 weights all in or out).
    auto issue = [&](int ss, const Cursor &cu) {
        const uint32_t st = ring_s + (uint32_t)(ss * L::STG) + lane * 16;
        const uint32_t sm = ring_s + (uint32_t)(ss * L::STG) + lane * L::MB;
        if (cu.rows_in && cu.ks < kfull) {
#pragma unroll
            for (int u = 0; u < L::UPW; ++u) {
                cp_async_cg16(st + L::w_a(u), cu.wa + 32 * u);
                cp_async_cg16(st + L::w_b(u), cu.wb + 32 * u);
                if constexpr (L::MB > 0) {
                    cp_async_ca<L::MB>(sm + L::m_a(u), cu.ma + 32 * u * NM / 8);
                    cp_async_ca<L::MB>(sm + L::m_b(u), cu.mb + 32 * u * NM / 8);
                }
            }
        } else {
            const int ra = cu.rb * ROWS + g;
#pragma unroll
            for (int u = 0; u < L::UPW; ++u) {
                const bool kin = cu.ks * L::KS + kl + 32 * u < d;
                const bool va = kin && ra < rows, vb = kin && ra + 8 < rows;
                cp_async_cg16(st + L::w_a(u), va ? cu.wa + 32 * u : W, va ? 16u : 0u);
                cp_async_cg16(st + L::w_b(u), vb ? cu.wb + 32 * u : W, vb ? 16u : 0u);
                if constexpr (L::MB > 0) {
                    cp_async_ca<L::MB>(sm + L::m_a(u), va ? cu.ma + 32 * u * NM / 8 : packed,
                                       va ? (uint32_t)L::MB : 0u);
                    cp_async_ca<L::MB>(sm + L::m_b(u), vb ? cu.mb + 32 * u * NM / 8 : packed,
                                       vb ? (uint32_t)L::MB : 0u);
                }
            }
        }
    };
    // x of a stage comes from L1 (its rows are small and every warp reads
    // them), loaded at the top of the stage's iteration; for n_m <= 2 the
    // narrow mask bits (one or two bytes a lane and row) stream from memory
    // into registers one stage ahead.
    const __nv_bfloat16 *xl[NT];  // this lane's x rows at its k offset
#pragma unroll
    for (int t = 0; t < NT; ++t)
        xl[t] = x + (int64_t)xrow[t] * d + kl;
    auto load_x = [&](uint4 (&xv)[L::UPW][NT], int ks) {
        const int k0 = ks * L::KS;
        if (ks < kfull) {
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
    auto load_narrow = [&](NarrowMasks &nm, int rb, int ks) {
        const int ra = rb * ROWS + g, rbb = ra + 8;
#pragma unroll
        for (int u = 0; u < L::UPW; ++u) {
            const int k = ks * L::KS + kl + 32 * u;
            const bool kin = k < d;
            nm.a[u] = nm.b[u] = make_uint2(0u, 0u);
            if (kin && ra < rows)
                nm.a[u] = ld_mask_chunk<NM>(packed + (int64_t)ra * mrow + (int64_t)k * NM / 8);
            if (kin && rbb < rows)
                nm.b[u] = ld_mask_chunk<NM>(packed + (int64_t)rbb * mrow + (int64_t)k * NM / 8);
        }
    };
    constexpr bool NARROW = NM > 0 && L::MB == 0;

    const int nflushes = sc.flushes();
    float acc[NM + 1][NT][4];
    zero_acc<NM, NT>(acc);
    // a warp's sums of a part into its slot, compactly (see slot_floats)
    auto write_slot = [&](float *slot, const float (&a)[NM + 1][NT][4]) {
#pragma unroll
        for (int v = 0; v <= NM; ++v)
#pragma unroll
            for (int t = 0; t < NT; ++t)
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    const int tok = 8 * t + 2 * c + (r & 1), row = g + 8 * (r >> 1);
                    if (tok < T)
                        slot[(v * ROWS + row) * T + tok] = a[v][t][r];
                }
    };

    // the copy cursor runs P - 1 stages ahead of the compute cursor
    int rb_c, ks_c;
    sc.start(rb_c, ks_c);
    Cursor cl;
    cl.rb = rb_c, cl.ks = ks_c;
    place(cl);
    for (int b = 0; b < L::P - 1; ++b) {
        if (b < sc.n)
            issue(b, cl);
        cp_async_commit();  // one group per stage, empty past the end
        if (b + 1 < sc.n)
            advance(b, cl);
    }
    NarrowMasks nmask;
    if constexpr (NARROW)
        load_narrow(nmask, rb_c, ks_c);

    int nflush = 0;
    for (int i = 0; i < sc.n; ++i) {
        uint4 xv[L::UPW][NT];
        load_x(xv, ks_c);
        const int il = i + L::P - 1;
        if (il < sc.n)
            issue(il % L::P, cl);
        cp_async_commit();
        if (il + 1 < sc.n)
            advance(il, cl);
        int rb_n = rb_c, ks_n = ks_c;
        sc.next(i, rb_n, ks_n);
        NarrowMasks cur;
        if constexpr (NARROW) {
            cur = nmask;
            if (i + 1 < sc.n)
                load_narrow(nmask, rb_n, ks_n);
        }
        cp_async_wait<L::P - 1>();  // this lane's copies of stage i have landed

        const uint8_t *st = ring + (i % L::P) * L::STG;
#pragma unroll
        for (int u = 0; u < L::UPW; ++u) {
            if (ks_c * L::KS + 32 * (L::UPW * warp + u) >= d)
                continue;  // the whole unit lies past the end of the row
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
            unit_step<NM, NT, ROUTED, 0>(acc, o, used);
            unit_step<NM, NT, ROUTED, 1>(acc, o, used);
        }
        if (sc.flush_at(i, ks_c)) {
            // ---------------------------------------------- row-block part done here
            const int f = nflush++;
            if constexpr (TT <= 2) {
                const int set = f % L::SETS;
                // this set was last used by part f - SETS: wait until its
                // finisher has read it (that finisher arrived as soon as it
                // had, and does not wait here); the FREE barrier alternates by
                // part
                if (f >= L::SETS && warp != (f - L::SETS) % L::NW)
                    named_bar_sync(BAR_FREE0 + (f & 1), L::BAR_COUNT);
                write_slot(slots + set * L::SLOT_SET + warp * L::ACC, acc);
                zero_acc<NM, NT>(acc);
                if (warp == f % L::NW) {
                    named_bar_sync(BAR_FULL0 + set, L::BAR_COUNT);  // every slot of part f is written
                    finish_part<NM, ROUTED, L::NW>(slots + set * L::SLOT_SET, L::ACC, rb_c, i < sc.n_sk,
                                                   f + L::SETS < nflushes ? BAR_FREE0 + ((f + L::SETS) & 1) : 0,
                                                   sc, act, T, rows, ws_part, ws_count, out, mw, gv);
                } else {
                    __threadfence_block();  // the slot writes are visible before the finisher reads them
                    named_bar_arrive(BAR_FULL0 + set, L::BAR_COUNT);
                }
            } else {
                // one slot set; the reducers read part f - 1 before anyone
                // writes part f (the reducers met on BAR_READ after reading,
                // the others wait on FREE, on which the reducers arrived)
                const int R = (ROWS * T + 31) / 32;
                if (f >= 1 && warp >= R)
                    named_bar_sync(BAR_FREE0, L::BAR_COUNT);
                write_slot(slots + warp * L::ACC, acc);
                zero_acc<NM, NT>(acc);
                named_bar_sync(BAR_FULL0, L::BAR_COUNT);  // every slot of part f is written
                if (warp < R)
                    finish_coop<NM, ROUTED, L::NW>(slots, L::ACC, rb_c, i < sc.n_sk, R,
                                                   f + 1 < nflushes && R < L::NW, sc, act, T, rows, ws_part,
                                                   ws_count, out, mw, gv);
            }
        }
        rb_c = rb_n, ks_c = ks_n;
    }
    cp_async_wait<0>();  // no copy outlives the kernel
}

// Scratch bytes of the decode kernel: partial slots for the largest grid,
// then one counter per row block of `rows` (256-byte aligned pieces).
__host__ __device__ constexpr int64_t part_bytes() { return (int64_t)2 * MAX_CTAS * PART_FLOATS * 4; }
__host__ __device__ constexpr int64_t workspace_bytes(int64_t rows)
{
    return part_bytes() + ((rows + ROWS - 1) / ROWS * 4 + 255) / 256 * 256;
}

}  // namespace dec
}  // namespace mglu
