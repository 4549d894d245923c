// prefill_wm.cuh -- the MGLU up-projection for 17 to 128 tokens with the
// weights on the MMA's M side and the tokens on N (the library runs it up
// to 128 tokens at n_m = 8, 96 at n_m = 4 and 32 at n_m <= 2).
//
// The token-major kernels (prefill.cuh, prefill_pair.cuh) multiply a whole
// 128- or 256-token tile whatever T is, so below a full tile their cost does
// not fall with T.  Here one tile is NJ weight rows: its stacked operand
// [W; M_1.W; ...; M_NM.W] (NJ rows per block, (NM+1) NJ <= 128, zero rows
// up to 128) is the MMA's A operand, built in shared memory exactly as in
// the other kernels, and the x tile of all T tokens (rounded up to NT, a
// multiple of 16) is B: one tcgen05.mma of 128 x NT per k16 step, so the
// tensor work follows T ("Masked Gated Linear Unit", "Approach": one shared
// W and n_m masks; D = x W, g_i = x (M_i . W), v_i = D - g_i).
//
// The accumulator holds stacked row r in TMEM lane r and token t in column
// t, so D and the g_i of one output sit in different lanes (different
// warps).  The epilogue stages 32 token columns of all 128 lanes at a time
// in shared memory (row stride 33 floats: conflict-free both ways), then
// each of its 128 threads forms outputs (token, j) from there.  Two
// mbarriers (count 4, one arrival per epilogue warp) hand the staging buffer
// between the TMEM-read and the combine step; every wait is bounded.
//
// Warp roles: warp 0 TMA producer, warp 1 TMEM allocation and the MMA
// thread, NBW builder warps, 4 epilogue warps.  Tiles (column blocks of NJ
// weight rows) are spread over a persistent grid; the accumulator is double
// buffered so a tile's MMAs overlap the previous tile's epilogue.
#pragma once
#include <cstdint>
#include <cuda_bf16.h>

#include "common.cuh"
#include "prefill.cuh"
#include "prefill_pair.cuh"
#include "ptx.cuh"

namespace mglu {
namespace pf {

constexpr int WM_MAX_T = 128;  // tokens (N) per MMA; more take the token-major kernels

template <int NM>
struct WmCfg {
    static_assert(NM > 0, "the masked product only");
    static constexpr int NJ = 128 / (NM + 1);       // weight rows per tile: 64 / 42 / 25 / 14
    static constexpr int MR = (NM + 1) * NJ;        // stacked rows in use (<= 128)
    // a stage spans KA 64-k swizzle atoms, so each load fetches KA
    // neighbouring 128-byte runs of every W row and the hand-offs per k halve
    static constexpr int KA = 2;
    static constexpr int BKS = KA * BK;             // k per stage
    static constexpr int ATOM = 128 * BK * 2;       // one atom of the stacked operand, 128 rows
    static constexpr int A_BYTES = KA * ATOM;
    static constexpr int MB = BKS * NM / 8 < 16 ? 16 : BKS * NM / 8;  // mask bytes per row per stage
    static constexpr int M_BYTES = NJ * MB;
    static constexpr int SROW = 33;                 // staging row stride (floats)
    static constexpr int S_BYTES = 128 * SROW * 4;  // 32 token columns of 128 lanes
    static constexpr int S_AL = (S_BYTES + 1023) / 1024 * 1024;
    static constexpr int BAR_OFF = S_AL;
    static constexpr int ST_OFF = BAR_OFF + 1024;   // stages, 1024-byte aligned
    static constexpr int SMEM = 227 * 1024;
    static constexpr int REGION = SMEM - 1024 - ST_OFF;  // bytes for stages (1024: alignment slack)
    static constexpr int MAXST = 12;
    // a stage holds the stacked operand, the x tile of NT tokens and the mask
    // tile; fewer tokens leave room for more stages, i.e. more of the weight
    // stream in flight
    static __host__ __device__ constexpr int stage_bytes(int NT)
    {
        return (A_BYTES + KA * NT * BK * 2 + M_BYTES + 1023) / 1024 * 1024;
    }
    static __host__ __device__ constexpr int stages(int NT)
    {
        return REGION / stage_bytes(NT) > MAXST ? MAXST : REGION / stage_bytes(NT);
    }
    static constexpr uint32_t W_TX = KA * NJ * BK * 2;
    static constexpr int ITEMS = KA * NJ * 8;       // 16-byte pieces of a stage's W tile
    // builder groups: where one item per thread takes at most 7 warps, two
    // groups of that many build alternate stages, so two stages are built at
    // once (a stage's build is a chain of waits, loads, stores and proxy
    // fences that one group cannot overlap with the next stage's)
    static constexpr int IW = (ITEMS + 31) / 32;
    static constexpr int BG = IW <= 4 ? 2 : 1;
    // warps per group: one piece per thread up to 10 warps, else two
    static constexpr int GW = BG == 2 ? IW : (IW <= 10 ? IW : ((IW + 1) / 2 > 8 ? (IW + 1) / 2 : 8));
    static constexpr int NBW = BG * GW;
    static constexpr int NTHREADS = (2 + NBW + 4) * 32;
    static_assert(stages(WM_MAX_T) >= 3, "ring too shallow");
    static_assert(5 * MAXST * 8 + 7 * 8 + 4 <= 1024, "barrier area");
    static_assert(ITEMS <= 2 * 32 * GW, "builder items");
};

// x: tensor map over [T][d] with boxes of NT rows; W, masks: boxes of NJ rows.
// mw: per-token mask weights [T][NM] (NULL: every weight 1).
template <int NM>
__global__ void __launch_bounds__(WmCfg<NM>::NTHREADS, 1)
    prefill_wm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                      const __grid_constant__ CUtensorMap tm_m, int T, int NT, int rows, int d, int act,
                      __nv_bfloat16 *__restrict__ out, const float *__restrict__ mw)
{
    using C = WmCfg<NM>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float *S = reinterpret_cast<float *>(smem);
    uint64_t *xfull = reinterpret_cast<uint64_t *>(smem + C::BAR_OFF);
    uint64_t *wfull = xfull + C::MAXST;
    uint64_t *mfull = wfull + C::MAXST;
    uint64_t *built = mfull + C::MAXST;
    uint64_t *empty = built + C::MAXST;
    uint64_t *acc_full = empty + C::MAXST;
    uint64_t *acc_empty = acc_full + 2;
    uint64_t *s_full = acc_empty + 2;  // the staging buffer holds a chunk
    uint64_t *s_free = s_full + 1;     // ... and has been read
    uint64_t *drain = s_free + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(drain + 1);

    pdl_launch_dependents();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_tiles = (rows + C::NJ - 1) / C::NJ;
    const int nkb = (d + C::BKS - 1) / C::BKS;
    const uint32_t x_tx = (uint32_t)NT * BK * 2;  // one atom of the x tile
    const int STG = C::stage_bytes(NT), NST = C::stages(NT);
    uint8_t *stages = smem + C::ST_OFF;

    if (threadIdx.x == 0) {
        for (int s = 0; s < NST; ++s) {
            mbar_init(&xfull[s], 1);
            mbar_init(&wfull[s], 1);
            mbar_init(&mfull[s], 1);
            mbar_init(&built[s], C::GW);
            mbar_init(&empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);
        }
        mbar_init(s_full, 4);
        mbar_init(s_free, 4);
        mbar_init(drain, 1);
        fence_mbar_init();
    }
    if constexpr (C::MR < 128) {
        // the stacked operand's pad rows are never loaded or built: zero them
        // once, for the tensor core (async proxy) to read
        constexpr int PIECES = (128 - C::MR) * 8;
        for (int i = threadIdx.x; i < NST * C::KA * PIECES; i += C::NTHREADS) {
            uint8_t *A = stages + (i / (C::KA * PIECES)) * STG + ((i / PIECES) % C::KA) * C::ATOM;
            *reinterpret_cast<uint4 *>(A + (C::MR + (i % PIECES) / 8) * 128 + (i % 8) * 16) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async_smem();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    pdl_wait();

    if (warp == 0) {
        // ---------------------------------------------------------- producer
        if (lane == 0) {
            prefetch_tensormap(&tm_x);
            prefetch_tensormap(&tm_w);
            prefetch_tensormap(&tm_m);
            int it = 0, s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
                const int n0 = tile * C::NJ;
                for (int kb = 0; kb < nkb; ++kb, ++it, s = s + 1 == NST ? 0 : s + 1, ph ^= s == 0 ? 1u : 0u) {
#ifdef MGLU_TEST_HOOKS
                    if (it >= 1 && *(volatile int *)&g_test_stall_producer) {
                        ok = false;  // stop issuing: the consumers' waits run out
                        break;
                    }
#endif
                    if (!mbar_wait(&empty[s], ph ^ 1u)) {
                        ok = false;
                        break;
                    }
                    uint8_t *st = stages + s * STG;
                    mbar_arrive_expect_tx(&wfull[s], C::W_TX);
#pragma unroll
                    for (int a = 0; a < C::KA; ++a)  // block 0 of each atom of the stacked operand
                        tma_load_2d(st + a * C::ATOM, &tm_w, &wfull[s], kb * C::BKS + a * BK, n0);
                    const int mc = (kb * C::BKS * NM / 8) / C::MB * C::MB;  // 16-byte aligned column
                    mbar_arrive_expect_tx(&mfull[s], C::M_BYTES);
                    tma_load_2d(st + C::A_BYTES + C::KA * x_tx, &tm_m, &mfull[s], mc, n0);
                    mbar_arrive_expect_tx(&xfull[s], C::KA * x_tx);
#pragma unroll
                    for (int a = 0; a < C::KA; ++a)
                        tma_load_2d(st + C::A_BYTES + a * x_tx, &tm_x, &xfull[s], kb * C::BKS + a * BK, 0);
                }
            }
            // every load issued has landed before the CTA may exit
            for (int j = it - NST < 0 ? 0 : it - NST; j < it; ++j) {
                const int s = j % NST;
                const uint32_t ph = (uint32_t)(j / NST) & 1u;
                mbar_wait(&xfull[s], ph);
                mbar_wait(&wfull[s], ph);
                mbar_wait(&mfull[s], ph);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------- MMA issuer
        if (lane == 0) {
            const uint32_t idesc = umma_idesc_bf16(128, NT);
            int acc_it = 0, s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++acc_it) {
                const int b = acc_it & 1;
                const uint32_t aph = (uint32_t)(acc_it >> 1) & 1u;
                if (!mbar_wait(&acc_empty[b], aph ^ 1u))
                    break;
                tc_fence_after();
                const uint32_t d_tmem = tmem_base + (uint32_t)(b * ACC_STRIDE);
                for (int kb = 0; kb < nkb; ++kb, s = s + 1 == NST ? 0 : s + 1, ph ^= s == 0 ? 1u : 0u) {
                    if (!mbar_wait(&built[s], ph) || !mbar_wait(&xfull[s], ph)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a_addr = smem_u32(stages + s * STG);
                    const uint32_t b_addr = a_addr + C::A_BYTES;
#pragma unroll
                    for (int a = 0; a < C::KA; ++a)
#pragma unroll
                        for (int k16 = 0; k16 < BK / 16; ++k16)
                            umma_f16_ss(d_tmem, sw128_kmajor_desc(a_addr + a * C::ATOM + k16 * 32),
                                        sw128_kmajor_desc(b_addr + a * x_tx + k16 * 32), idesc,
                                        (kb | a | k16) != 0 ? 1u : 0u);
                    umma_commit(&empty[s]);
                }
                if (ok)
                    umma_commit(&acc_full[b]);
            }
            umma_commit(drain);  // every MMA issued has completed before TMEM is released
            mbar_wait(drain, 0);
        }
    } else if (warp < 2 + C::NBW) {
        // ---------------------------------------------------------- builders
        const int grp = (warp - 2) / C::GW;                // builder group
        const int bt = threadIdx.x - 64 - grp * 32 * C::GW;  // 0 .. 32 * GW - 1
        constexpr int MAXI = (C::ITEMS + 32 * C::GW - 1) / (32 * C::GW);
        int it = 0, s = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
            for (int kb = 0; kb < nkb; ++kb, ++it, s = s + 1 == NST ? 0 : s + 1, ph ^= s == 0 ? 1u : 0u) {
                if (C::BG > 1 && (it & 1) != grp)
                    continue;  // the other group's stage
                if (!mbar_wait_warp3(&wfull[s], &mfull[s], nullptr, ph)) {
                    ok = false;
                    break;
                }
                fence_proxy_async_smem();  // TMA-written tiles are read with ordinary loads below
                uint8_t *A = stages + s * STG;
                const uint8_t *Mt = A + C::A_BYTES + C::KA * x_tx;
#pragma unroll
                for (int q = 0; q < MAXI; ++q) {
                    const int item = bt + q * 32 * C::GW;
                    if (item < C::ITEMS) {
                        const int a = item / (C::NJ * 8), rem = item % (C::NJ * 8);
                        const int r = rem >> 3, c = rem & 7;
                        uint8_t *Aa = A + a * C::ATOM;
                        const uint4 w = *reinterpret_cast<const uint4 *>(Aa + r * 128 + ((c ^ (r & 7)) << 4));
                        uint32_t lo, hi;
                        load_mask_bytes<NM>(Mt + r * C::MB + a * (BK * NM / 8) + c * NM, lo, hi);
                        build_variants_pair<NM, C::NJ, 0>(Aa, r, c, w, lo, hi);
                    }
                }
                fence_proxy_async_smem();  // generic-proxy writes -> visible to the tensor core
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&built[s]);
            }
        }
    } else {
        // ---------------------------------------------------------- epilogue
        const int q = warp & 3;                          // TMEM lane quadrant of this warp
        const int et = threadIdx.x - (2 + C::NBW) * 32;  // 0 .. 127
        const bool dense_gate = (act & GATE_DENSE) != 0;
        const int a = act & ACT_MASK;
        int acc_it = 0, chunk = 0;
        bool ok = true;
        for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++acc_it) {
            const int b = acc_it & 1;
            const uint32_t aph = (uint32_t)(acc_it >> 1) & 1u;
            if (!mbar_wait_warp(&acc_full[b], aph))
                break;
            tc_fence_after();
            const int n0 = tile * C::NJ;
            const uint32_t tbase = tmem_base + ((uint32_t)(32 * q) << 16) + (uint32_t)(b * ACC_STRIDE);
            for (int c0 = 0; c0 < NT; c0 += 32, ++chunk) {
                const uint32_t cph = (uint32_t)chunk & 1u;
                // 32 token columns of this warp's 32 lanes -> staging rows
                uint32_t v[32];
#pragma unroll
                for (int h8 = 0; h8 < 4; ++h8)
                    if (c0 + 8 * h8 < NT)
                        tmem_ld_x8(tbase + (uint32_t)(c0 + 8 * h8), *reinterpret_cast<uint32_t(*)[8]>(&v[8 * h8]));
                tmem_wait_ld();
                if (c0 + 32 >= NT) {
                    // the tile's last TMEM read: the MMA may refill this buffer
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0)
                        mbar_arrive(&acc_empty[b]);
                }
                // the previous chunk's combine has finished reading S
                if (chunk > 0 && !mbar_wait_warp(s_free, cph ^ 1u)) {
                    ok = false;
                    break;
                }
                float *Srow = S + (32 * q + lane) * C::SROW;
#pragma unroll
                for (int e = 0; e < 32; ++e)
                    Srow[e] = __uint_as_float(v[e]);
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(s_full);
                if (!mbar_wait_warp(s_full, cph)) {
                    ok = false;
                    break;
                }
                // combine: thread -> token c0 + lane, weight rows j = et/32 + 4k
                const int tok = c0 + lane;
                float wt[NM];
#pragma unroll
                for (int i = 0; i < NM; ++i)
                    wt[i] = mw && tok < T ? mw[(int64_t)tok * NM + i] : 1.0f;
                for (int j = et >> 5; j < C::NJ; j += 4) {
                    const float D = S[j * C::SROW + lane];
                    float acc = 0.f;
#pragma unroll
                    for (int i = 0; i < NM; ++i) {
                        const float gi = S[((1 + i) * C::NJ + j) * C::SROW + lane];
                        acc += wt[i] * (act_fn(a, dense_gate ? D : gi) * (D - gi));
                    }
                    if (tok < T && n0 + j < rows)
                        out[(int64_t)tok * rows + n0 + j] = __float2bfloat16_rn(acc);
                }
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(s_free);
            }
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
