// prefill_pair.cuh -- the many-token MGLU up-projection (and the dense
// product of the down-projection, NM = 0) on CTA pairs (tcgen05
// cta_group::2): one MMA of 256 tokens x N columns per k16 step, issued by
// the pair's first CTA.
//
// The 1-CTA kernel (prefill.cuh) is bound by shared-memory bandwidth: per
// k-stage every CTA writes the x tile and the W tile by TMA, its builder warps
// read W and write the n_m masked copies, and the MMA reads the x tile and all
// n_m + 1 blocks of the stacked B operand.  In a pair each CTA keeps its own
// 128 tokens of x but only HALF of every block of the stacked B operand (the
// first or the second NJ/2 weight rows of the column tile): it loads, builds
// and lends the MMA half the B bytes, so the shared-memory traffic per FLOP
// drops by about a third ("Masked Gated Linear Unit", "Approach": one shared
// W and n_m masks; the products are D = x W and g_i = x (M_i . W), v_i =
// D - g_i).
//
// The MMA's N columns are CTA 0's half-blocks followed by CTA 1's:
//   [D_a, g_1a, ..., g_NMa, D_b, g_1b, ..., g_NMb],  a / b = rows n0 + [0, NJ/2)
// and n0 + [NJ/2, NJ) of W (each half padded with zero rows to whole 8-row
// swizzle atoms); each CTA's TMEM holds those N columns for its 128 tokens,
// and its epilogue writes its tokens' outputs for all NJ columns.
//
// Roles per CTA (warp 0 TMA producer, warp 1 TMEM and, in CTA 0, the MMA
// issuer, NBW builder warps, 4 epilogue warps).  Barriers that both CTAs
// signal live in CTA 0: the x tiles' bytes (xfull, armed by CTA 0 for both),
// the built stages (built, one arrival per builder warp of both CTAs) and the
// drained accumulators (acc_empty, one arrival per epilogue warp of both).
// The MMA's commits arrive on both CTAs' stage and accumulator barriers.
// The dense instance (NM = 0) has no builders: both CTAs' W halves, like the
// x tiles, come by the 2-SM TMA form onto CTA 0's barrier.  The GRAD instance
// runs the training path's gradient epilogue on each half of the tile.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "common.cuh"
#include "prefill.cuh"
#include "ptx.cuh"

namespace mglu {
namespace pf {

template <int NM, bool GRAD = false>
struct PairCfg {
    // weight rows of a column tile (both CTAs).  At n_m = 8 the forward takes
    // 28: nine blocks of 14 rows per CTA, padded by two zero rows, fill
    // N = 256.  With the 1-CTA kernel's 16 rows the MMA is only N = 144 wide
    // and the x tile, whose shared-memory writes and reads are fixed per k16
    // step, dominates the shared-memory traffic.  The gradient epilogue reads
    // 8-column blocks and keeps 16.
    static constexpr int NJ = NM == 8 && !GRAD ? 28 : Cfg<NM>::NJ;
    static constexpr int NJH = NJ / 2;           // this CTA's half
    static constexpr int NH = (NM + 1) * NJH;    // B rows in this CTA
    static constexpr int NHP = (NH + 7) / 8 * 8; // ... padded to whole 8-row swizzle atoms
    static constexpr int N = 2 * NHP;            // MMA columns
    // the variant blocks do not start on 8-column (TMEM) / 8-row boundaries
    static constexpr bool RAGGED = NJH % 8 != 0;
    static constexpr int BM2 = 2 * BM;           // tokens of a pair tile
    static constexpr int A_BYTES = BM * BK * 2;  // 16 KB
    static constexpr int B_BYTES = NHP * BK * 2;
    static constexpr int MB = Cfg<NM>::MB;       // mask bytes per row per stage (0: the dense product)
    static constexpr int M_BYTES = NJH * MB;
    static constexpr int STAGE = (A_BYTES + B_BYTES + M_BYTES + 1023) / 1024 * 1024;
    static constexpr int STAGES = (227 * 1024 - 2048) / STAGE > 8 ? 8 : (227 * 1024 - 2048) / STAGE;
    static constexpr uint32_t W_TX = NJH * BK * 2;
    static constexpr int BAR_OFF = STAGES * STAGE;
    static constexpr int SMEM = BAR_OFF + 1024 + 1024;
    // builders: NJH * 8 16-byte pieces of this CTA's W half per stage (none
    // for the dense product)
    static constexpr int ITEMS = NM == 0 ? 0 : NJH * 8;
    // one item per builder thread where that takes at most 10 warps, else two
    static constexpr int NBW = (ITEMS + 31) / 32 <= 10 ? (ITEMS + 31) / 32 : 8;
    static constexpr int EC = NJH % Cfg<NM>::EC == 0 ? Cfg<NM>::EC : 8;
    static constexpr int NTHREADS = (2 + NBW + 4) * 32;
    static_assert(!RAGGED || (NM > 0 && !GRAD), "only the forward act-sum epilogue reads ragged blocks");
    static_assert(RAGGED || NJH % EC == 0, "epilogue chunking");
    static_assert(N <= 256 && N % 16 == 0, "UMMA shape for M = 256");
    static_assert(STAGES >= 3, "ring too shallow");
    static_assert(SMEM <= 227 * 1024, "shared memory");
    static_assert(ITEMS <= 2 * 32 * NBW, "builder items");
    // the dense product's W tiles, like the x tiles, complete on CTA 0's
    // barrier: the MMA waits for nothing else
    static constexpr uint32_t LEADER_TX = NM == 0 ? 2u * (A_BYTES + W_TX) : 2u * A_BYTES;
};

// Variant I of W piece (r, c) goes to stacked row (1 + I) * NJH + r, at the
// 16-byte column its row's 128-byte swizzle gives (the stage is 1024-byte
// aligned, so the swizzle row is the stacked row mod 8).
template <int NM, int NJH, int I>
__device__ __forceinline__ void build_variants_pair(uint8_t *B, int r, int c, uint4 w, uint32_t lo, uint32_t hi)
{
    if constexpr (I < NM) {
        uint4 m;
        m.x = w.x & pair_mask<NM, 0, I>(lo, hi);
        m.y = w.y & pair_mask<NM, 1, I>(lo, hi);
        m.z = w.z & pair_mask<NM, 2, I>(lo, hi);
        m.w = w.w & pair_mask<NM, 3, I>(lo, hi);
        const int R = (1 + I) * NJH + r;
        *reinterpret_cast<uint4 *>(B + R * 128 + ((c ^ (R & 7)) << 4)) = m;
        build_variants_pair<NM, NJH, I + 1>(B, r, c, w, lo, hi);
    }
}

// mw: per-token mask weights [T][NM] (NULL: every weight 1).  The packed
// rows must be 16-byte strided (a tensor map describes the mask tiles).
// GRAD: the training path's epilogue (see grad_epilogue) into gout from the
// loss gradient dout, instead of the forward's output.
template <int NM, bool GRAD = false>
__global__ void __launch_bounds__(PairCfg<NM, GRAD>::NTHREADS, 1)
    prefill_pair_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                        const __grid_constant__ CUtensorMap tm_m, int T, int rows, int d, int act,
                        __nv_bfloat16 *__restrict__ out, const float *__restrict__ mw,
                        const __nv_bfloat16 *__restrict__ dout, __nv_bfloat16 *__restrict__ gout)
{
    using C = PairCfg<NM, GRAD>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *xfull = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);  // CTA 0's: both x tiles landed
    uint64_t *wfull = xfull + C::STAGES;                                // own W half landed
    uint64_t *mfull = wfull + C::STAGES;                                // own mask half landed
    uint64_t *built = mfull + C::STAGES;                                // CTA 0's: both CTAs built
    uint64_t *empty = built + C::STAGES;                                // own: the MMA has read the stage
    uint64_t *acc_full = empty + C::STAGES;                             // own: accumulator ready
    uint64_t *acc_empty = acc_full + 2;                                 // CTA 0's: both epilogues drained
    uint64_t *drain = acc_empty + 2;                                    // own: every MMA has completed
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);

    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int num_m = (T + C::BM2 - 1) / C::BM2;
    const int num_n = (rows + C::NJ - 1) / C::NJ;
    const int num_tiles = num_m * num_n;
    const int nkb = (d + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(&xfull[s], 1);
            mbar_init(&wfull[s], 1);
            mbar_init(&mfull[s], 1);
            mbar_init(&built[s], C::NBW > 0 ? 2 * C::NBW : 1);  // unused by the dense product
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 8);
        }
        mbar_init(drain, 1);
        fence_mbar_init();
    }
    if constexpr (C::NHP > C::NH) {
        // the pad rows of the stacked operand are never loaded or built:
        // zero them once, for the tensor core (async proxy) to read
        constexpr int PIECES = (C::NHP - C::NH) * 8;
        for (int i = threadIdx.x; i < C::STAGES * PIECES; i += C::NTHREADS) {
            uint8_t *B = smem + (i / PIECES) * C::STAGE + C::A_BYTES;
            *reinterpret_cast<uint4 *>(B + (C::NH + (i % PIECES) / 8) * 128 + (i % 8) * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, TMEM_COLS);
        tmem_relinquish_pair();
    }
    __syncwarp();
    tc_fence_before();
    cluster_sync();  // both CTAs' barriers and TMEM exist before any remote arrival or MMA
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_wait();

    if (warp == 0) {
        // ---------------------------------------------------------- producer (both CTAs)
        if (lane == 0) {
            prefetch_tensormap(&tm_x);
            prefetch_tensormap(&tm_w);
            prefetch_tensormap(&tm_m);
            int it = 0;
            bool ok = true;
            for (int tile = pair; tile < num_tiles && ok; tile += npairs) {
                const int m0 = (tile % num_m) * C::BM2 + (int)rank * BM;
                const int n0 = (tile / num_m) * C::NJ + (int)rank * C::NJH;
                for (int kb = 0; kb < nkb; ++kb, ++it) {
#ifdef MGLU_TEST_HOOKS
                    if (it >= 1 && *(volatile int *)&g_test_stall_producer) {
                        ok = false;  // stop issuing: every other wait of the pair runs out
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
                    if (rank == 0)
                        mbar_arrive_expect_tx(&xfull[s], C::LEADER_TX);  // both CTAs' x (and dense W) tiles
                    tma_load_2d_pair(st, &tm_x, cluster_addr(&xfull[s], 0), kb * BK, m0);
                    if constexpr (NM == 0) {
                        tma_load_2d_pair(st + C::A_BYTES, &tm_w, cluster_addr(&xfull[s], 0), kb * BK, n0);
                    } else {
                        mbar_arrive_expect_tx(&wfull[s], C::W_TX);
                        tma_load_2d(st + C::A_BYTES, &tm_w, &wfull[s], kb * BK, n0);
                        const int mc = (kb * BK * NM / 8) / C::MB * C::MB;  // 16-byte aligned column
                        mbar_arrive_expect_tx(&mfull[s], C::M_BYTES);
                        tma_load_2d(st + C::A_BYTES + C::B_BYTES, &tm_m, &mfull[s], mc, n0);
                    }
                }
            }
            // Before the CTA may exit, every load issued has landed: its own W
            // and mask tiles, and (counted on CTA 0's barrier, which CTA 0
            // waits for before the closing cluster barrier) the pair-form loads.
            for (int j = it - C::STAGES < 0 ? 0 : it - C::STAGES; j < it; ++j) {
                const int s = j % C::STAGES;
                const uint32_t ph = (uint32_t)(j / C::STAGES) & 1u;
                if constexpr (NM > 0) {
                    mbar_wait(&wfull[s], ph);
                    mbar_wait(&mfull[s], ph);
                }
                if (rank == 0)
                    mbar_wait(&xfull[s], ph);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer (CTA 0)
        if (rank == 0 && lane == 0) {
            constexpr uint32_t idesc = umma_idesc_bf16(C::BM2, C::N);
            int it = 0, acc_it = 0;
            bool ok = true;
            for (int tile = pair; tile < num_tiles && ok; tile += npairs, ++acc_it) {
                const int b = acc_it & 1;
                const uint32_t aph = (uint32_t)(acc_it >> 1) & 1u;
                if (!mbar_wait(&acc_empty[b], aph ^ 1u))
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(b * ACC_STRIDE);
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = it % C::STAGES;
                    const uint32_t ph = (uint32_t)(it / C::STAGES) & 1u;
                    if ((NM > 0 && !mbar_wait(&built[s], ph)) || !mbar_wait(&xfull[s], ph)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(smem + s * C::STAGE);
                    const uint32_t b_addr = a_addr + C::A_BYTES;
#pragma unroll
                    for (int k16 = 0; k16 < BK / 16; ++k16)
                        umma_f16_ss_pair(d_tmem, sw128_kmajor_desc(a_addr + k16 * 32),
                                         sw128_kmajor_desc(b_addr + k16 * 32), idesc, (kb | k16) != 0 ? 1u : 0u);
                    umma_commit_pair(&empty[s], 3);
                }
                if (ok)
                    umma_commit_pair(&acc_full[b], 3);
            }
            umma_commit_pair(drain, 3);  // every MMA has completed, in both CTAs
        }
        if (lane == 0)
            mbar_wait(drain, 0);
        __syncwarp();
    } else if (warp < 2 + C::NBW) {
        // ---------------------------------------------------------- builders (both CTAs)
        if constexpr (NM > 0) {
        const int bt = threadIdx.x - 64;  // 0 .. 32 * NBW - 1
        constexpr int MAXI = (C::ITEMS + 32 * C::NBW - 1) / (32 * C::NBW);
        const uint32_t built0 = cluster_addr(built, 0);
        int it = 0;
        bool ok = true;
        for (int tile = pair; tile < num_tiles && ok; tile += npairs) {
            for (int kb = 0; kb < nkb; ++kb, ++it) {
                const int s = it % C::STAGES;
                const uint32_t ph = (uint32_t)(it / C::STAGES) & 1u;
                if (!mbar_wait_warp3(&wfull[s], &mfull[s], nullptr, ph)) {
                    ok = false;
                    break;
                }
                fence_proxy_async_smem();  // TMA-written tiles are read with ordinary loads below
                uint8_t *B = smem + s * C::STAGE + C::A_BYTES;
                const uint8_t *Mt = B + C::B_BYTES;
                const int moff = (kb * BK * NM / 8) % C::MB;  // nonzero only when NM = 1
#pragma unroll
                for (int q = 0; q < MAXI; ++q) {
                    const int item = bt + q * 32 * C::NBW;
                    if (item < C::ITEMS) {
                        const int r = item >> 3, c = item & 7;
                        const uint4 w = *reinterpret_cast<const uint4 *>(B + r * 128 + ((c ^ (r & 7)) << 4));
                        uint32_t lo, hi;
                        load_mask_bytes<NM>(Mt + r * C::MB + moff + c * NM, lo, hi);
                        build_variants_pair<NM, C::NJH, 0>(B, r, c, w, lo, hi);
                    }
                }
                fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core
                __syncwarp();
                if (lane == 0)
                    mbar_arrive_cluster(built0 + (uint32_t)(s * 8));
            }
        }
        }
    } else {
        // ---------------------------------------------------------- epilogue (both CTAs)
        const int q = warp & 3;  // TMEM lane quadrant this warp may access
        const uint32_t acc_empty0 = cluster_addr(acc_empty, 0);
        int acc_it = 0;
        for (int tile = pair; tile < num_tiles; tile += npairs, ++acc_it) {
            const int b = acc_it & 1;
            const uint32_t aph = (uint32_t)(acc_it >> 1) & 1u;
            if (!mbar_wait_warp(&acc_full[b], aph))
                break;
            tc_fence_after();
            const int m0 = (tile % num_m) * C::BM2 + (int)rank * BM;
            const int n0 = (tile / num_m) * C::NJ;
            const int tok = m0 + 32 * q + lane;
            const uint32_t tbase = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * ACC_STRIDE);
            if constexpr (GRAD) {
                // both halves of the tile: CTA 0's weight rows, then CTA 1's
                grad_epilogue<NM, C::NJH, C::NJH>(tbase, tok, T, rows, n0, act, dout, gout);
                grad_epilogue<NM, C::NJH, C::NJH>(tbase + (uint32_t)C::NHP, tok, T, rows, n0 + C::NJH, act, dout,
                                                  gout);
            } else if constexpr (NM == 0) {
                // the dense product: out = D
                __nv_bfloat16 *orow = out + (int64_t)tok * rows;
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
#pragma unroll 1
                    for (int jc = 0; jc < C::NJH; jc += C::EC) {
                        uint32_t dv[C::EC];
#pragma unroll
                        for (int h8 = 0; h8 < C::EC / 8; ++h8)
                            tmem_ld_x8(tbase + (uint32_t)(half * C::NHP + jc + 8 * h8),
                                       *reinterpret_cast<uint32_t(*)[8]>(&dv[8 * h8]));
                        tmem_wait_ld();
                        const int j = n0 + half * C::NJH + jc;
                        if (tok < T) {
#pragma unroll
                            for (int e = 0; e < C::EC; e += 8) {
                                float v8[8];
#pragma unroll
                                for (int z = 0; z < 8; ++z)
                                    v8[z] = __uint_as_float(dv[e + z]);
                                const int nv = rows - (j + e) < 8 ? (rows - (j + e) > 0 ? rows - (j + e) : 0) : 8;
                                if (nv > 0)
                                    store8_bf16(orow + j + e, v8, nv, (rows & 7) == 0);
                            }
                        }
                    }
                }
            } else {
            float wt[NM];
#pragma unroll
            for (int i = 0; i < NM; ++i)
                wt[i] = mw && tok < T ? mw[(int64_t)tok * NM + i] : 1.0f;
            __nv_bfloat16 *orow = out + (int64_t)tok * rows;
            const bool dense_gate = (act & GATE_DENSE) != 0;
            const int a = act & ACT_MASK;
            if constexpr (C::RAGGED) {
#pragma unroll 1
                for (int half = 0; half < 2; ++half) {
                    // all NHP columns of the half in one round of loads: a
                    // TMEM load waited for while the tensor core fills the
                    // other accumulator takes long, and one wait per variant
                    // block made this epilogue, not the MMA, set the pace
                    const uint32_t hbase = tbase + (uint32_t)(half * C::NHP);
                    uint32_t cols[C::NHP];
#pragma unroll
                    for (int c = 0; c < C::NHP / 8; ++c)
                        tmem_ld_x8(hbase + (uint32_t)(8 * c), *reinterpret_cast<uint32_t(*)[8]>(&cols[8 * c]));
                    tmem_wait_ld();
                    float o[C::NJH];
#pragma unroll
                    for (int e = 0; e < C::NJH; ++e) {
                        const float D = __uint_as_float(cols[e]);
                        float acc = 0.f;
#pragma unroll
                        for (int i = 0; i < NM; ++i) {
                            const float gi = __uint_as_float(cols[(1 + i) * C::NJH + e]);
                            acc += wt[i] * (act_fn(a, dense_gate ? D : gi) * (D - gi));
                        }
                        o[e] = acc;
                    }
                    const int j = n0 + half * C::NJH;  // even: NJ and NJH are
                    if (tok < T) {
                        if ((rows & 1) == 0 && j + C::NJH <= rows &&
                            (reinterpret_cast<uintptr_t>(orow) & 3) == 0) {
#pragma unroll
                            for (int e = 0; e < C::NJH; e += 2)
                                *reinterpret_cast<__nv_bfloat162 *>(orow + j + e) =
                                    __floats2bfloat162_rn(o[e], o[e + 1]);
                        } else {
#pragma unroll
                            for (int e = 0; e < C::NJH; ++e)
                                if (j + e < rows)
                                    orow[j + e] = __float2bfloat16_rn(o[e]);
                        }
                    }
                }
            } else {
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                const uint32_t hbase = tbase + (uint32_t)(half * C::NHP);
#pragma unroll 1
                for (int jc = 0; jc < C::NJH; jc += C::EC) {
                    float o[C::EC];
                    uint32_t dv[C::EC];
                    uint32_t gv[NM][C::EC];
#pragma unroll
                    for (int h8 = 0; h8 < C::EC / 8; ++h8)
                        tmem_ld_x8(hbase + jc + 8 * h8, *reinterpret_cast<uint32_t(*)[8]>(&dv[8 * h8]));
#pragma unroll
                    for (int i = 0; i < NM; ++i)
#pragma unroll
                        for (int h8 = 0; h8 < C::EC / 8; ++h8)
                            tmem_ld_x8(hbase + (1 + i) * C::NJH + jc + 8 * h8,
                                       *reinterpret_cast<uint32_t(*)[8]>(&gv[i][8 * h8]));
                    tmem_wait_ld();
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
                    const int j = n0 + half * C::NJH + jc;
                    if (tok < T) {
                        if ((rows & 7) == 0 && j + C::EC <= rows) {
#pragma unroll
                            for (int e = 0; e < C::EC; e += 8) {
                                float v8[8];
#pragma unroll
                                for (int z = 0; z < 8; ++z)
                                    v8[z] = o[e + z];
                                store8_bf16(orow + j + e, v8, 8, true);
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
            }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive_cluster(acc_empty0 + (uint32_t)(b * 8));
        }
    }

    __syncwarp();
    tc_fence_before();
    cluster_sync();  // no CTA leaves while the pair's MMAs or remote arrivals may touch it
    if (warp == 1) {
        __syncwarp();
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

}  // namespace pf
}  // namespace mglu
