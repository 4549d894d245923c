// prefill.cuh -- MGLU up-projection for many tokens on the 5th-generation
// tensor cores (tcgen05, accumulators in TMEM), and the dense product
// (NM = 0) used as the prefill down-projection.
//
// For many tokens the MGLU forward is a dense contraction: for every token b
// and column j it needs D = x W and the NM gate products g_i = x (M_i . W).
// The kernel computes them as ONE matrix product per tile whose B operand is
// the stack [W; M_1.W; ...; M_NM.W] of NJ weight rows each, so one MMA per
// k16 step yields every accumulator of the tile and the x tile is read once
// per step ("Approach" of "Masked Gated Linear Unit": one shared weight
// matrix, masks split it into gate and value parts; values are D - g_i).
//
// Warp roles of the persistent CTA (one per SM):
//   warp 0      TMA producer: x tile (128 tokens x 64 k), W tile (NJ x 64),
//               packed-mask tile, into a ring of STAGES shared-memory stages
//   warp 1      TMEM allocator and the single thread that issues tcgen05.mma
//   warps 2..    builders (6 to 12 warps by n_m): write the NM masked copies of the W tile next to
//               it in shared memory (same 128-byte swizzle), then signal
//   last 4 warps epilogue: tcgen05.ld the accumulators, out = sum_i
//               act(g_i)(D - g_i), bf16 stores; overlaps the next tile's
//               MMAs through a double-buffered accumulator
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "common.cuh"
#include "ptx.cuh"

namespace mglu {
namespace pf {

constexpr int BM = 128;  // tokens per tile (UMMA M)
constexpr int BK = 64;   // k per stage: one 128-byte swizzle atom of bf16
constexpr int TMEM_COLS = 512;
constexpr int ACC_STRIDE = 256;  // TMEM columns between the two accumulator buffers

template <int NM>
struct Cfg {
    // Weight rows per tile: the stacked operand has N = (NM+1)*NJ rows with
    // N <= 256 and N % 16 == 0 (UMMA shape rule for M = 128); NJ % 8 == 0 so
    // every variant block starts on an 8-row swizzle boundary.
    static constexpr int NJ = NM == 0 ? 256 : NM == 1 ? 128 : NM == 2 ? 80 : NM == 4 ? 48 : 16;
    static constexpr int N = (NM + 1) * NJ;
    static constexpr int STAGES = NM == 8 ? 5 : 4;
    static constexpr int A_BYTES = BM * BK * 2;  // 16 KB
    static constexpr int B_BYTES = N * BK * 2;
    static constexpr int MB = NM == 0 ? 0 : (BK * NM / 8 < 16 ? 16 : BK * NM / 8);  // mask bytes per row per stage
    static constexpr int M_BYTES = NJ * MB;
    static constexpr int STAGE = (A_BYTES + B_BYTES + M_BYTES + 1023) / 1024 * 1024;
    static constexpr uint32_t W_TX = NJ * BK * 2;  // bytes of one W box (the variant rows are built here)
    static constexpr int BAR_OFF = STAGES * STAGE;
    static constexpr int SMEM = BAR_OFF + 512 + 1024;
    // warps: 0 TMA, 1 TMEM + MMA, then NBW builders, then 4 epilogue warps.
    // A stage has NJ * 8 build items (16-byte pieces of the W tile); builder
    // counts that split them into whole rounds were fastest on B200 (n_m = 4:
    // 384 items, 12 warps, 966 TFLOP/s against 842 with 4 warps); the dense
    // kernel has nothing to build.
    static constexpr int NBW = NM == 0 ? 4 : NM == 8 ? 6 : NM == 4 ? 12 : NM == 2 ? 10 : 8;
    // builder groups: group b builds the stages with it % BG == b, so each
    // builder has BG stages' time to hide its loads, stores and fence
    static constexpr int BG = 1;
    static constexpr int GW = NBW / BG;  // builder warps per group
    static_assert(NBW % BG == 0, "builder groups");
    // epilogue columns per TMEM load round (8 where the register budget of the
    // larger block is tight)
    static constexpr int EC = NM >= 4 ? 8 : 16;
    static constexpr int NTHREADS = (2 + NBW + 4) * 32;
    static_assert(N <= 256 && N % 16 == 0 && NJ % 8 == 0, "bad tile shape");
    static_assert(NJ % EC == 0, "epilogue chunking");
    static_assert(SMEM <= 227 * 1024, "shared memory");
};

template <int NM>
__device__ __forceinline__ void load_mask_bytes(const uint8_t *p, uint32_t &lo, uint32_t &hi)
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
    } else {
        lo = *p;
        hi = 0;
    }
}

template <int NM, int I>
__device__ __forceinline__ void build_variants(uint8_t *B, int off, uint4 w, uint32_t lo, uint32_t hi)
{
    if constexpr (I < NM) {
        uint4 m;
        m.x = w.x & pair_mask<NM, 0, I>(lo, hi);
        m.y = w.y & pair_mask<NM, 1, I>(lo, hi);
        m.z = w.z & pair_mask<NM, 2, I>(lo, hi);
        m.w = w.w & pair_mask<NM, 3, I>(lo, hi);
        *reinterpret_cast<uint4 *>(B + (1 + I) * Cfg<NM>::NJ * 128 + off) = m;
        build_variants<NM, I + 1>(B, off, w, lo, hi);
    }
}

// Store 8 floats as bf16 at p[0..8) (n valid; 16-byte store when all 8 are
// valid and p is 16-byte aligned).
__device__ __forceinline__ void store8_bf16(__nv_bfloat16 *p, const float (&v)[8], int n, bool vec)
{
    if (vec && n == 8) {
        uint4 pk;
        __nv_bfloat162 p0 = __floats2bfloat162_rn(v[0], v[1]);
        __nv_bfloat162 p1 = __floats2bfloat162_rn(v[2], v[3]);
        __nv_bfloat162 p2 = __floats2bfloat162_rn(v[4], v[5]);
        __nv_bfloat162 p3 = __floats2bfloat162_rn(v[6], v[7]);
        pk.x = *reinterpret_cast<uint32_t *>(&p0);
        pk.y = *reinterpret_cast<uint32_t *>(&p1);
        pk.z = *reinterpret_cast<uint32_t *>(&p2);
        pk.w = *reinterpret_cast<uint32_t *>(&p3);
        *reinterpret_cast<uint4 *>(p) = pk;
    } else {
#pragma unroll
        for (int e = 0; e < 8; ++e)
            if (e < n)
                p[e] = __float2bfloat16_rn(v[e]);
    }
}

// The training path's epilogue for one token (one TMEM lane) of a tile: for
// every column j of the tile, with D = x W and g_i from the accumulators,
// v_i = D - g_i:
//   block i < NM of gout:  dout (act'(g_i) v_i - act(g_i))
//   block NM of gout:      sum_i dout act(g_i)
// One mask at a time, 8 columns at a time, to keep registers low.  The tile's
// NC columns start at weight row n0; block i of the accumulator starts BS
// TMEM columns after block i - 1.
template <int NM, int BS = Cfg<NM>::NJ, int NC = Cfg<NM>::NJ>
__device__ __forceinline__ void grad_epilogue(uint32_t tbase, int tok, int T, int rows, int n0, int act,
                                              const __nv_bfloat16 *__restrict__ dout, __nv_bfloat16 *__restrict__ gout)
{
    static_assert(NC % 8 == 0, "eight columns at a time");
    const int a = act & ACT_MASK;
    const int64_t gstride = (int64_t)(NM + 1) * rows;
    for (int jc = 0; jc < NC; jc += 8) {
        const int j = n0 + jc;
        const int nv = tok < T ? (rows - j < 8 ? (rows - j > 0 ? rows - j : 0) : 8) : 0;
        const bool vec = (rows & 7) == 0;
        uint32_t dv[8];
        tmem_ld_x8(tbase + jc, dv);
        float go[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
            go[e] = e < nv ? __bfloat162float(dout[(int64_t)tok * rows + j + e]) : 0.0f;
        tmem_wait_ld();
        float cs[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
            cs[e] = 0.0f;
#pragma unroll 1
        for (int i = 0; i < NM; ++i) {
            uint32_t gv[8];
            tmem_ld_x8(tbase + (1 + i) * BS + jc, gv);
            tmem_wait_ld();
            float ai[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float g = __uint_as_float(gv[e]);
                const float v = __uint_as_float(dv[e]) - g;
                const float av = act_fn(a, g);
                ai[e] = go[e] * (act_grad_fn(a, g) * v - av);
                cs[e] += go[e] * av;
            }
            if (nv > 0)
                store8_bf16(gout + (int64_t)tok * gstride + (int64_t)i * rows + j, ai, nv, vec);
        }
        if (nv > 0)
            store8_bf16(gout + (int64_t)tok * gstride + (int64_t)NM * rows + j, cs, nv, vec);
    }
}

// Mask bits of an 8-weight chunk read straight from global memory (NM bytes
// at byte offset (row * d + k) * NM / 8; zero outside the matrix).
template <int NM>
__device__ __forceinline__ uint2 load_mask_global(const uint8_t *packed, int row, int k, int rows, int d)
{
    if (row >= rows || k >= d)
        return make_uint2(0u, 0u);
    const uint8_t *p = packed + ((int64_t)row * d + k) * NM / 8;
    if constexpr (NM == 8)
        return __ldg(reinterpret_cast<const uint2 *>(p));
    else if constexpr (NM == 4)
        return make_uint2(__ldg(reinterpret_cast<const unsigned int *>(p)), 0u);
    else if constexpr (NM == 2)
        return make_uint2(__ldg(reinterpret_cast<const unsigned short *>(p)), 0u);
    else
        return make_uint2(__ldg(p), 0u);
}

// mw: per-token mask weights [T][NM] that scale each mask's term (NULL:
// every weight 1).
// mask_direct != 0: the packed rows are not 16-byte strided (d * NM / 8 is
// not a multiple of 16), so no tensor map can describe them; the builders
// then read each chunk's mask bits from global memory (issued before they
// wait for the W tile, so the two latencies overlap) instead of a staged
// mask tile.
//
// GRAD: the epilogue of the training path instead of the forward's.  With
// the loss gradient dout [T][rows] it writes, for every token b and column
// j, the n_m + 1 coefficients of the backward's products into
// gout [T][(NM + 1) * rows]: block i < NM holds dout * (act'(g_i) v_i -
// act(g_i)) (the gradient of g_i minus that of v_i), block NM holds
// sum_i dout * act(g_i) (the gradient of every v_i); rounded to bf16.
template <int NM, bool GRAD = false>
__global__ void __launch_bounds__(Cfg<NM>::NTHREADS, 1) prefill_kernel(const __grid_constant__ CUtensorMap tm_x,
                                                              const __grid_constant__ CUtensorMap tm_w,
                                                              const __grid_constant__ CUtensorMap tm_m, int T,
                                                              int rows, int d, int act,
                                                              __nv_bfloat16 *__restrict__ out,
                                                              const uint8_t *__restrict__ packed, int mask_direct,
                                                              const float *__restrict__ mw,
                                                              const __nv_bfloat16 *__restrict__ dout,
                                                              __nv_bfloat16 *__restrict__ gout)
{
    using C = Cfg<NM>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // one barrier per TMA load of a stage: x (A), W, masks
    uint64_t *xfull = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
    uint64_t *full = xfull + C::STAGES;
    uint64_t *mfull = full + C::STAGES;
    uint64_t *built = mfull + C::STAGES;
    uint64_t *empty = built + C::STAGES;
    uint64_t *acc_full = empty + C::STAGES;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *drain = acc_empty + 2;  // the MMA issuer's last commit: every MMA has completed
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);

    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_m = (T + BM - 1) / BM;
    const int num_n = (rows + C::NJ - 1) / C::NJ;
    const int num_tiles = num_m * num_n;
    const int nkb = (d + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&xfull[s], 1);
            mbar_init(&full[s], 1);
            mbar_init(&mfull[s], 1);
            mbar_init(&built[s], C::GW);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);
        }
        mbar_init(drain, 1);
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_wait();  // the previous kernel's outputs (x) are complete from here on

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            prefetch_tensormap(&tm_x);
            prefetch_tensormap(&tm_w);
            if (NM > 0)
                prefetch_tensormap(&tm_m);
            int it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                const int m0 = (tile % num_m) * BM;
                const int n0 = (tile / num_m) * C::NJ;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
#ifdef MGLU_TEST_HOOKS
                    if (it >= 1 && *(volatile int *)&g_test_stall_producer) {
                        ok = false;  // stop issuing: the consumers' waits run out
                        break;
                    }
#endif
                    const int s = it % C::STAGES;
                    const uint32_t ph = (uint32_t)(it / C::STAGES) & 1u;
                    if (!mbar_wait(&empty[s], ph ^ 1u)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = smem + s * C::STAGE;
                    // each load completes on a barrier of its own
                    mbar_arrive_expect_tx(&xfull[s], C::A_BYTES);
                    tma_load_2d(st, &tm_x, &xfull[s], kb * BK, m0);
                    mbar_arrive_expect_tx(&full[s], C::W_TX);
                    tma_load_2d(st + C::A_BYTES, &tm_w, &full[s], kb * BK, n0);
                    if constexpr (NM > 0) {
                        if (!mask_direct) {
                            const int mc = (kb * BK * NM / 8) / C::MB * C::MB;  // 16-byte aligned column
                            mbar_arrive_expect_tx(&mfull[s], C::M_BYTES);
                            tma_load_2d(st + C::A_BYTES + C::B_BYTES, &tm_m, &mfull[s], mc, n0);
                        }
                    }
                }
            }
            // Before the CTA may exit, every load issued must have landed: the
            // last STAGES iterations' barriers have completed their phase (at
            // once when the consumers took them; after a timeout, bounded).
            for (int j = it - C::STAGES < 0 ? 0 : it - C::STAGES; j < it; ++j) {
                const int s = j % C::STAGES;
                const uint32_t ph = (uint32_t)(j / C::STAGES) & 1u;
                mbar_wait(&xfull[s], ph);
                mbar_wait(&full[s], ph);
                if (NM > 0 && !mask_direct)
                    mbar_wait(&mfull[s], ph);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_bf16(BM, C::N);
            int it = 0, acc_it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++acc_it) {
                const int b = acc_it & 1;
                const uint32_t aph = (uint32_t)(acc_it >> 1) & 1u;
                if (!mbar_wait(&acc_empty[b], aph ^ 1u))
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(b * ACC_STRIDE);
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % C::STAGES;
                    const uint32_t ph = (uint32_t)(it / C::STAGES) & 1u;
                    if (!mbar_wait(NM > 0 ? &built[s] : &full[s], ph) || !mbar_wait(&xfull[s], ph)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + s * C::STAGE);
                    const uint32_t b_addr = a_addr + C::A_BYTES;
#pragma unroll
                    for (int k16 = 0; k16 < BK / 16; ++k16)
                        umma_f16_ss(d_tmem, sw128_kmajor_desc(a_addr + k16 * 32), sw128_kmajor_desc(b_addr + k16 * 32),
                                    idesc, (kb | k16) != 0 ? 1u : 0u);
                    umma_commit(&empty[s]);
                }
                if (ok)
                    umma_commit(&acc_full[b]);
            }
            // every MMA issued has completed before TMEM is released
            umma_commit(drain);
            mbar_wait(drain, 0);
        }
    } else if (warp < 2 + C::NBW) {
        // ---------------------------------------------------------- builders
        if constexpr (NM > 0) {
            const int grp = (warp - 2) / C::GW;                   // builder group
            const int bt = threadIdx.x - 64 - grp * 32 * C::GW;   // 0 .. 32 * GW - 1
            constexpr int ITEMS = C::NJ * 8;   // 16-byte pieces of a W tile
            constexpr int MAXI = (ITEMS + 32 * C::GW - 1) / (32 * C::GW);
            int it = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                const int n0 = (tile / num_m) * C::NJ;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    if (C::BG > 1 && it % C::BG != grp)
                        continue;
                    const int s = it % C::STAGES;
                    const uint32_t ph = (uint32_t)(it / C::STAGES) & 1u;
                    uint2 mg[MAXI];
                    if (mask_direct) {
#pragma unroll
                        for (int q = 0; q < MAXI; ++q) {
                            const int item = bt + q * 32 * C::GW;
                            mg[q] = item < ITEMS ? load_mask_global<NM>(packed, n0 + (item >> 3), kb * BK + 8 * (item & 7),
                                                                        rows, d)
                                                 : make_uint2(0u, 0u);
                        }
                    }
                    if (!mbar_wait_warp3(&full[s], mask_direct ? nullptr : &mfull[s], nullptr, ph)) {
                        ok = false;
                        break;
                    }
                    fence_proxy_async_smem();  // TMA-written tiles are read with ordinary loads below
                    uint8_t *B = smem + s * C::STAGE + C::A_BYTES;
                    const uint8_t *Mt = B + C::B_BYTES;
                    const int moff = (kb * BK * NM / 8) % C::MB;  // nonzero only when NM = 1
#pragma unroll
                    for (int q = 0; q < MAXI; ++q) {
                        const int item = bt + q * 32 * C::GW;
                        if (item < ITEMS) {
                            const int r = item >> 3, c = item & 7;
                            const int off = r * 128 + ((c ^ (r & 7)) << 4);
                            const uint4 w = *reinterpret_cast<const uint4 *>(B + off);
                            uint32_t lo, hi;
                            if (mask_direct) {
                                lo = mg[q].x;
                                hi = mg[q].y;
                            } else {
                                load_mask_bytes<NM>(Mt + r * C::MB + moff + c * NM, lo, hi);
                            }
                            build_variants<NM, 0>(B, off, w, lo, hi);
                        }
                    }
                    fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&built[s]);
                }
            }
        }
    } else {
        // ---------------------------------------------------------- epilogue
        const int q = warp & 3;  // TMEM lane quadrant this warp may access
        int acc_it = 0;
        for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++acc_it) {
            const int b = acc_it & 1;
            const uint32_t aph = (uint32_t)(acc_it >> 1) & 1u;
            if (!mbar_wait_warp(&acc_full[b], aph))
                break;
            tc_fence_after();
            const int m0 = (tile % num_m) * BM;
            const int n0 = (tile / num_m) * C::NJ;
            const int tok = m0 + 32 * q + lane;
            float wt[NM > 0 ? NM : 1];
#pragma unroll
            for (int i = 0; i < (NM > 0 ? NM : 1); ++i)
                wt[i] = mw && tok < T ? mw[(int64_t)tok * NM + i] : 1.0f;
            const uint32_t tbase = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * ACC_STRIDE);
            if constexpr (GRAD && NM > 0) {
                grad_epilogue<NM>(tbase, tok, T, rows, n0, act, dout, gout);
            } else {
            __nv_bfloat16 *orow = out + (int64_t)tok * rows;
            for (int jc = 0; jc < C::NJ; jc += C::EC) {
                float o[C::EC];
                {
                    uint32_t dv[C::EC];
#pragma unroll
                    for (int h8 = 0; h8 < C::EC / 8; ++h8)
                        tmem_ld_x8(tbase + jc + 8 * h8, *reinterpret_cast<uint32_t(*)[8]>(&dv[8 * h8]));
                    if constexpr (NM == 0) {
                        tmem_wait_ld();
#pragma unroll
                        for (int e = 0; e < C::EC; ++e)
                            o[e] = __uint_as_float(dv[e]);
                    } else {
                        uint32_t gv[NM][C::EC];
#pragma unroll
                        for (int i = 0; i < NM; ++i)
#pragma unroll
                            for (int h8 = 0; h8 < C::EC / 8; ++h8)
                                tmem_ld_x8(tbase + (1 + i) * C::NJ + jc + 8 * h8,
                                           *reinterpret_cast<uint32_t(*)[8]>(&gv[i][8 * h8]));
                        tmem_wait_ld();
                        const bool dense_gate = (act & GATE_DENSE) != 0;
                        const int a = act & ACT_MASK;
#pragma unroll
                        for (int e = 0; e < C::EC; ++e) {
                            const float D = __uint_as_float(dv[e]);
                            float acc = 0.f;
#pragma unroll
                            for (int i = 0; i < NM; ++i) {
                                const float gi = __uint_as_float(gv[i][e]);
                                acc += wt[i] * (act_fn(a, dense_gate ? D : gi) * (D - gi));
                            }
                            o[e] = acc;
                        }
                    }
                }
                if (tok < T) {
                    const int j = n0 + jc;
                    if ((rows & 7) == 0 && j + C::EC <= rows) {
#pragma unroll
                        for (int e = 0; e < C::EC; e += 8) {
                            uint4 pk;
                            __nv_bfloat162 p0 = __floats2bfloat162_rn(o[e + 0], o[e + 1]);
                            __nv_bfloat162 p1 = __floats2bfloat162_rn(o[e + 2], o[e + 3]);
                            __nv_bfloat162 p2 = __floats2bfloat162_rn(o[e + 4], o[e + 5]);
                            __nv_bfloat162 p3 = __floats2bfloat162_rn(o[e + 6], o[e + 7]);
                            pk.x = *reinterpret_cast<uint32_t *>(&p0);
                            pk.y = *reinterpret_cast<uint32_t *>(&p1);
                            pk.z = *reinterpret_cast<uint32_t *>(&p2);
                            pk.w = *reinterpret_cast<uint32_t *>(&p3);
                            *reinterpret_cast<uint4 *>(orow + j + e) = pk;
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < C::EC; ++e)
                            if (j + e < rows)
                                orow[j + e] = __float2bfloat16_rn(o[e]);
                    }
                }
            }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&acc_empty[b]);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}

}  // namespace pf
}  // namespace mglu
