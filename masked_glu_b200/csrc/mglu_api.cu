// mglu_api.cu -- the C ABI of libmglu.so (declared in include/mglu.h):
// argument checks, TMA descriptor encoding, kernel choice and launches.
// Everything is one translation unit so the device status word is shared.
#include <cublas_v2.h>
#include <cuda.h>
#include <cuda_runtime.h>
#include <dlfcn.h>

#include <cstdint>
#include <cstdio>
#include <atomic>
#include <cstring>
#include <mutex>

#include "mglu.h"
#include "common.cuh"
#include "decode.cuh"
#include "pack.cuh"
#include "prefill.cuh"
#include "prefill_pair.cuh"
#include "prefill_wm.cuh"
#include "ptx.cuh"
#include "route.cuh"
#include "simt.cuh"
#include "train.cuh"

namespace {

thread_local char g_last_cuda_error[256] = "";
std::atomic<int> g_decode_max_tokens{16};
constexpr int kMaxDevices = 64;

int cuda_fail(cudaError_t e, const char *what)
{
    snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "%s: %s", what, cudaGetErrorString(e));
    return MGLU_ERR_CUDA;
}

// Kernels this library has launched in this process (every launch ends in
// check_launch); read with mglu_kernel_launches().
std::atomic<uint64_t> g_kernel_launches{0};

int check_launch(const char *what)
{
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess)
        return cuda_fail(e, what);
    g_kernel_launches.fetch_add(1, std::memory_order_relaxed);
    return MGLU_OK;
}

bool aligned(const void *p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool nm_supported(int n_m) { return n_m == 1 || n_m == 2 || n_m == 4 || n_m == 8; }

int current_device(int *dev)
{
    const cudaError_t e = cudaGetDevice(dev);
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaGetDevice");
    if (*dev < 0 || *dev >= kMaxDevices)
        return MGLU_ERR_INVALID;
    return MGLU_OK;
}

// SM count per device, cached; concurrent first calls may both query, and
// both store the same value.
int sm_count(int dev)
{
    static std::atomic<int> cache[kMaxDevices];
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        n = n > 0 ? n : 148;
        cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

// cuTensorMapEncodeTiled through the runtime's driver entry point, so the
// library does not link libcuda directly.
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// Encoded maps are cached per thread, keyed by every encoding input, so a
// repeated call (same weights, same activation buffers) skips the encoding.
struct MapKey {
    const void *base;
    uint64_t dims[3], strides[2];
    uint32_t box[3];
    int rank, dt, sw;
    bool operator==(const MapKey &o) const { return memcmp(this, &o, sizeof(MapKey)) == 0; }
};
constexpr int kMapCache = 64;
struct MapCache {
    MapKey key[kMapCache];
    CUtensorMap map[kMapCache];
    int used = 0, next = 0;
};
thread_local MapCache g_maps;

// Tensor map of rank 2 or 3 (dims innermost first, strides in bytes for
// dims 1..rank-1, box in elements); out-of-range reads give zeros.
int make_map_n(CUtensorMap *m, CUtensorMapDataType dt, const void *base, int rank, const uint64_t *dims,
               const uint64_t *strides, const uint32_t *box, CUtensorMapSwizzle sw)
{
    MapKey key;
    memset(&key, 0, sizeof(key));
    key.base = base;
    key.rank = rank;
    key.dt = (int)dt;
    key.sw = (int)sw;
    for (int i = 0; i < rank; ++i) {
        key.dims[i] = dims[i];
        key.box[i] = box[i];
        if (i + 1 < rank)
            key.strides[i] = strides[i];
    }
    for (int i = 0; i < g_maps.used; ++i)
        if (g_maps.key[i] == key) {
            *m = g_maps.map[i];
            return MGLU_OK;
        }
    EncodeTiledFn fn = encode_fn();
    if (!fn) {
        snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "cuTensorMapEncodeTiled unavailable");
        return MGLU_ERR_CUDA;
    }
    cuuint64_t d[3], st[2];
    cuuint32_t bx[3], es[3] = {1, 1, 1};
    for (int i = 0; i < rank; ++i) {
        d[i] = dims[i];
        bx[i] = box[i];
        if (i + 1 < rank)
            st[i] = strides[i];
    }
    const CUresult r = fn(m, dt, (cuuint32_t)rank, const_cast<void *>(base), d, st, bx, es,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "cuTensorMapEncodeTiled failed (%d)", (int)r);
        return MGLU_ERR_CUDA;
    }
    const int slot = g_maps.used < kMapCache ? g_maps.used++ : (g_maps.next++ % kMapCache);
    g_maps.key[slot] = key;
    g_maps.map[slot] = *m;
    return MGLU_OK;
}

// 2-D tensor map: `outer` rows of `inner` elements, rows `row_bytes` apart.
int make_map(CUtensorMap *m, CUtensorMapDataType dt, const void *base, uint64_t inner, uint64_t outer,
             uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw)
{
    const uint64_t dims[2] = {inner, outer};
    const uint64_t strides[1] = {row_bytes};
    const uint32_t box[2] = {box_inner, box_outer};
    return make_map_n(m, dt, base, 2, dims, strides, box, sw);
}

std::mutex g_attr_mu;

// Raise the kernel's dynamic shared-memory limit once per device (one flag
// array per kernel instantiation; host threads making their first call at
// once serialize on a mutex).
template <auto Kernel>
int ensure_smem(int bytes, int dev)
{
    static std::atomic<bool> done[kMaxDevices];
    if (done[dev].load(std::memory_order_acquire))
        return MGLU_OK;
    std::lock_guard<std::mutex> lock(g_attr_mu);
    if (!done[dev].load(std::memory_order_relaxed)) {
        const cudaError_t e =
            cudaFuncSetAttribute(reinterpret_cast<const void *>(Kernel), cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (e != cudaSuccess)
            return cuda_fail(e, "cudaFuncSetAttribute");
        done[dev].store(true, std::memory_order_release);
    }
    return MGLU_OK;
}

// Launch with programmatic stream serialization, so a kernel's launch and
// prologue overlap the tail of the previous kernel on the stream; the kernels
// wait (griddepcontrol.wait) before they touch global memory.
template <typename... KArgs, typename... Args>
int launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, int smem, cudaStream_t s, const char *what,
               Args... args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
    if (e != cudaSuccess)
        return cuda_fail(e, what);
    return check_launch(what);
}

// ------------------------------------------------------------------ decode
template <int NM, int TT, bool ROUTED>
int launch_decode(const void *x, int64_t T, int64_t d, const void *W, int64_t rows, const uint8_t *packed, int act,
                  void *out, void *ws, cudaStream_t s, const float *mw, float *gv, mglu::dec::Router ro)
{
    using L = mglu::dec::Layout<NM, TT>;
    const int64_t rb = (rows + mglu::dec::ROWS - 1) / mglu::dec::ROWS;
    const int64_t units = rb * ((d + L::STEP - 1) / L::STEP);
    if (units >= ((int64_t)1 << 31))
        return MGLU_ERR_INVALID;  // the kernel's 32-bit unit numbering
    int dev = 0, rc = current_device(&dev);
    if (rc)
        return rc;
    if ((rc = ensure_smem<mglu::dec::decode_kernel<NM, TT, ROUTED>>(L::SMEM, dev)))
        return rc;
    int64_t grid = (int64_t)sm_count(dev);
    if (grid > mglu::dec::MAX_CTAS)
        grid = mglu::dec::MAX_CTAS;
    if (grid > units)
        grid = units;
    float *ws_part = reinterpret_cast<float *>(ws);
    __nv_bfloat16 *o = reinterpret_cast<__nv_bfloat16 *>(out);
    if ((rc = launch_pdl(mglu::dec::decode_kernel<NM, TT, ROUTED>, dim3((unsigned)grid), dim3(L::NTHREADS), L::SMEM, s,
                         "decode launch", reinterpret_cast<const __nv_bfloat16 *>(x),
                         reinterpret_cast<const __nv_bfloat16 *>(W), packed, (int)T, (int)rows, (int)d, act, ws_part, o,
                         mw, gv, ro)))
        return rc;
    // row blocks whose units several CTAs hold are finished by split_kernel
    mglu::dec::Plan pl;
    pl.init((int)rows, (int)d, L::STEP, (int)grid, L::NW);
    bool shared = false;
    for (int c = 0; c < (int)grid && !shared; ++c) {
        if (!pl.cta_has_units(c))
            continue;
        int cf, cl;
        pl.ctas_of(pl.last_rb(c), cf, cl);
        shared = cf != cl;
    }
    if (!shared)
        return MGLU_OK;
    // with routing in the kernel, CTA 0 has stored the weights for this kernel
    const float *mw_split = ro.Wr ? ro.weights : mw;
    return launch_pdl(mglu::dec::split_kernel<NM, TT, ROUTED>, dim3((unsigned)grid), dim3(32), 0, s, "split launch",
                      (int)rows, (int)d, L::STEP, (int)grid, L::NW, (int)T, act, (const float *)ws_part, o, mw_split,
                      gv);
}

// Token capacity by T: 2, 8 or 16 (the slots and the finisher's work follow
// the call's T; the capacity fixes the MMA column blocks and shared memory).
template <int NM, bool ROUTED>
int decode_tt(const void *x, int64_t T, int64_t d, const void *W, int64_t rows, const uint8_t *packed, int act,
              void *out, void *ws, cudaStream_t s, const float *mw, float *gv, mglu::dec::Router ro)
{
    if (T <= 2)
        return launch_decode<NM, 2, ROUTED>(x, T, d, W, rows, packed, act, out, ws, s, mw, gv, ro);
    if (T <= 8)
        return launch_decode<NM, 8, ROUTED>(x, T, d, W, rows, packed, act, out, ws, s, mw, gv, ro);
    return launch_decode<NM, 16, ROUTED>(x, T, d, W, rows, packed, act, out, ws, s, mw, gv, ro);
}

template <int NM>
int decode_nt(const void *x, int64_t T, int64_t d, const void *W, int64_t rows, const uint8_t *packed, int act,
              void *out, void *ws, cudaStream_t s, const float *mw, float *gv = nullptr,
              mglu::dec::Router ro = mglu::dec::Router{nullptr, 0, 0, 0, nullptr, nullptr})
{
    if constexpr (NM > 0) {
        if (mw || ro.Wr)
            return decode_tt<NM, true>(x, T, d, W, rows, packed, act, out, ws, s, mw, gv, ro);
    }
    return decode_tt<NM, false>(x, T, d, W, rows, packed, act, out, ws, s, nullptr, gv, ro);
}

// The routed forward on the decode kernel with the router inside it.
template <int NM>
int decode_routed(const void *x, int64_t T, int64_t d, const void *W, int64_t rows, const uint8_t *packed, int act,
                  void *out, void *ws, cudaStream_t s, mglu::dec::Router ro)
{
    return decode_nt<NM>(x, T, d, W, rows, packed, act, out, ws, s, nullptr, nullptr, ro);
}

// ------------------------------------------------------------------ prefill
// The forward on CTA pairs (clusters of two, one 256-token MMA per k16 step
// issued by the first CTA of each pair); the grid is as many pairs as fit at
// once, each looping over tiles.
template <int NM, bool GRAD>
int launch_prefill_pair(const void *x, int64_t T, int64_t d, const void *W, int64_t rows, const uint8_t *packed,
                        int act, void *out, cudaStream_t s, const float *mw, int dev, const void *dout, void *gout)
{
    using C = mglu::pf::PairCfg<NM, GRAD>;
    CUtensorMap tx, tw, tm;
    int rc;
    if ((rc = make_map(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, d, T, d * 2, mglu::pf::BK, mglu::pf::BM,
                       CU_TENSOR_MAP_SWIZZLE_128B)))
        return rc;
    if ((rc = make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W, d, rows, d * 2, mglu::pf::BK, C::NJH,
                       CU_TENSOR_MAP_SWIZZLE_128B)))
        return rc;
    if constexpr (NM > 0) {
        if ((rc = make_map(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, d * NM / 8, rows, d * NM / 8, C::MB, C::NJH,
                           CU_TENSOR_MAP_SWIZZLE_NONE)))
            return rc;
    } else {
        tm = tw;  // not read
    }
    if ((rc = ensure_smem<mglu::pf::prefill_pair_kernel<NM, GRAD>>(C::SMEM, dev)))
        return rc;
    static std::atomic<int> max_pairs[kMaxDevices];
    int pairs = max_pairs[dev].load(std::memory_order_relaxed);
    cudaLaunchConfig_t cfg = {};
    cfg.blockDim = dim3(C::NTHREADS);
    cfg.dynamicSmemBytes = (size_t)C::SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    if (pairs == 0) {
        cfg.gridDim = dim3((unsigned)(2 * sm_count(dev)));
        cfg.numAttrs = 1;
        const cudaError_t e = cudaOccupancyMaxActiveClusters(&pairs, mglu::pf::prefill_pair_kernel<NM, GRAD>, &cfg);
        if (e != cudaSuccess)
            return cuda_fail(e, "cudaOccupancyMaxActiveClusters");
        if (pairs < 1)
            return MGLU_ERR_UNSUPPORTED;
        max_pairs[dev].store(pairs, std::memory_order_relaxed);
    }
    const int64_t tiles = ((T + 2 * mglu::pf::BM - 1) / (2 * mglu::pf::BM)) * ((rows + C::NJ - 1) / C::NJ);
    const int64_t grid_pairs = tiles < pairs ? tiles : pairs;
    cfg.gridDim = dim3((unsigned)(2 * grid_pairs));
    cfg.numAttrs = 2;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, mglu::pf::prefill_pair_kernel<NM, GRAD>, tx, tw, tm, (int)T,
                                             (int)rows, (int)d, act, reinterpret_cast<__nv_bfloat16 *>(out), mw,
                                             reinterpret_cast<const __nv_bfloat16 *>(dout),
                                             reinterpret_cast<__nv_bfloat16 *>(gout));
    if (e != cudaSuccess)
        return cuda_fail(e, "prefill pair launch");
    return check_launch("prefill pair launch");
}

template <int NM>
int launch_prefill_wm(const void *x, int64_t T, int64_t d, const void *W, int64_t rows, const uint8_t *packed, int act,
                      void *out, cudaStream_t s, const float *mw, int dev)
{
    using C = mglu::pf::WmCfg<NM>;
    const int NT = (int)((T + 15) / 16 * 16);  // the MMA's N: tokens rounded up to 16
    CUtensorMap tx, tw, tm;
    int rc;
    if ((rc = make_map(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, d, T, d * 2, mglu::pf::BK, NT,
                       CU_TENSOR_MAP_SWIZZLE_128B)))
        return rc;
    if ((rc = make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W, d, rows, d * 2, mglu::pf::BK, C::NJ,
                       CU_TENSOR_MAP_SWIZZLE_128B)))
        return rc;
    if ((rc = make_map(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, d * NM / 8, rows, d * NM / 8, C::MB, C::NJ,
                       CU_TENSOR_MAP_SWIZZLE_NONE)))
        return rc;
    if ((rc = ensure_smem<mglu::pf::prefill_wm_kernel<NM>>(C::SMEM, dev)))
        return rc;
    const int64_t tiles = (rows + C::NJ - 1) / C::NJ;
    const int grid = (int)(tiles < sm_count(dev) ? tiles : sm_count(dev));
    return launch_pdl(mglu::pf::prefill_wm_kernel<NM>, dim3((unsigned)grid), dim3(C::NTHREADS), C::SMEM, s,
                      "prefill wm launch", tx, tw, tm, (int)T, NT, (int)rows, (int)d, act,
                      reinterpret_cast<__nv_bfloat16 *>(out), mw);
}

template <int NM, bool GRAD = false>
int launch_prefill(const void *x, int64_t T, int64_t d, const void *W, int64_t rows, const uint8_t *packed, int act,
                   void *out, void *, cudaStream_t s, const float *mw, const void *dout = nullptr,
                   void *gout = nullptr)
{
    using C = mglu::pf::Cfg<NM>;
    int dev = 0, rc = current_device(&dev);
    if (rc)
        return rc;
    CUtensorMap tx, tw, tm;
    if ((rc = make_map(&tx, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, d, T, d * 2, mglu::pf::BK, mglu::pf::BM,
                       CU_TENSOR_MAP_SWIZZLE_128B)))
        return rc;
    if ((rc = make_map(&tw, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, W, d, rows, d * 2, mglu::pf::BK, C::NJ,
                       CU_TENSOR_MAP_SWIZZLE_128B)))
        return rc;
    // a tensor map needs 16-byte row strides; other packed rows are read by
    // the builder warps directly
    const int mask_direct = NM > 0 && (d * NM / 8) % 16 != 0;
    // CTA pairs from two 128-token tiles on; the dense product (the
    // down-projection) at any T: its pair kernel was faster on B200 at
    // T = 24 and T = 128 as well (79 against 88 and 91 us at h = 14336,
    // d = 4096), with the same accumulation order per k16 step
    // up to 128 tokens at n_m = 8, 96 at n_m = 4 and 32 at n_m <= 2 the
    // forward puts the weight rows on the MMA's M side and the tokens on N.
    // On B200 at d=4096, h=14336: n_m = 8 143-200 us against 241 us
    // (T = 24..128); n_m = 4 89-121 us against 127-130 us (T = 17..96), about
    // equal at T = 128; n_m = 2 68-70 us against 88 us (T = 17..32), slower
    // from T = 96 (at d=2048, h=8192 already from T = 64)
    if constexpr (NM > 0 && !GRAD) {
        if (!mask_direct && T <= (NM == 8 ? mglu::pf::WM_MAX_T : NM == 4 ? 96 : 32))
            return launch_prefill_wm<NM>(x, T, d, W, rows, packed, act, out, s, mw, dev);
    }
    if constexpr (NM > 0 || !GRAD) {
        if (!mask_direct && (NM == 0 || T > mglu::pf::BM))
            return launch_prefill_pair<NM, GRAD>(x, T, d, W, rows, packed, act, out, s, mw, dev, dout, gout);
    }
    if (NM > 0 && !mask_direct) {
        if ((rc = make_map(&tm, CU_TENSOR_MAP_DATA_TYPE_UINT8, packed, d * NM / 8, rows, d * NM / 8, C::MB, C::NJ,
                           CU_TENSOR_MAP_SWIZZLE_NONE)))
            return rc;
    } else {
        tm = tw;  // not read
    }
    if ((rc = ensure_smem<mglu::pf::prefill_kernel<NM, GRAD>>(C::SMEM, dev)))
        return rc;
    const int64_t tiles = ((T + mglu::pf::BM - 1) / mglu::pf::BM) * ((rows + C::NJ - 1) / C::NJ);
    const int grid = (int)(tiles < sm_count(dev) ? tiles : sm_count(dev));
    return launch_pdl(mglu::pf::prefill_kernel<NM, GRAD>, dim3((unsigned)grid), dim3(mglu::pf::Cfg<NM>::NTHREADS),
                      C::SMEM, s, "prefill launch", tx, tw, tm, (int)T, (int)rows, (int)d, act,
                      reinterpret_cast<__nv_bfloat16 *>(out), packed, mask_direct, mw,
                      reinterpret_cast<const __nv_bfloat16 *>(dout), reinterpret_cast<__nv_bfloat16 *>(gout));
}

// ------------------------------------------------------------------ fp32
template <int NM>
int launch_simt(const void *x, int64_t T, int64_t d, const void *W, int64_t rows, const uint8_t *packed, int act,
                void *out, void *, cudaStream_t s, const float *mw)
{
    const dim3 grid((unsigned)((rows + 7) / 8), (unsigned)((T + mglu::kSimtTokens - 1) / mglu::kSimtTokens));
    if (grid.y > 65535u)
        return MGLU_ERR_INVALID;
    mglu::simt_f32_kernel<NM><<<grid, 256, 0, s>>>(reinterpret_cast<const float *>(x), T, d,
                                                     reinterpret_cast<const float *>(W), rows, packed, act,
                                                     reinterpret_cast<float *>(out), mw);
    return check_launch("fp32 launch");
}

// Dispatch on n_m at compile time.
template <template <int> class F, typename... A>
int by_nm(int n_m, A... a)
{
    switch (n_m) {
    case 0: return F<0>::run(a...);
    case 1: return F<1>::run(a...);
    case 2: return F<2>::run(a...);
    case 4: return F<4>::run(a...);
    case 8: return F<8>::run(a...);
    default: return MGLU_ERR_UNSUPPORTED;
    }
}

template <int NM>
struct DecodeF {
    template <typename... A>
    static int run(A... a) { return decode_nt<NM>(a...); }
};
template <int NM>
struct PrefillF {
    template <typename... A>
    static int run(A... a) { return launch_prefill<NM>(a...); }
};
template <int NM>
struct SimtF {
    template <typename... A>
    static int run(A... a) { return launch_simt<NM>(a...); }
};

int path_for(int64_t T, int dtype)
{
    if (dtype == MGLU_F32)
        return MGLU_PATH_F32;
    return T <= g_decode_max_tokens ? MGLU_PATH_DECODE : MGLU_PATH_PREFILL;
}

// One product of the library: out[T][rows] from x[T][d] and W[rows][d] with
// n_m masks (n_m = 0: dense).  Arguments already validated.
int run_product(const void *x, int64_t T, int64_t d, const void *W, int64_t rows, const uint8_t *packed, int n_m,
                int act, int dtype, void *out, void *ws, cudaStream_t s, const float *mw = nullptr)
{
    if (T == 0)
        return MGLU_OK;
    switch (path_for(T, dtype)) {
    case MGLU_PATH_F32: return by_nm<SimtF>(n_m, x, T, d, W, rows, packed, act, out, ws, s, mw);
    case MGLU_PATH_DECODE: return by_nm<DecodeF>(n_m, x, T, d, W, rows, packed, act, out, ws, s, mw);
    default: return by_nm<PrefillF>(n_m, x, T, d, W, rows, packed, act, out, ws, s, mw);
    }
}

size_t scratch_bytes(int64_t rows) { return rows > 0 ? (size_t)mglu::dec::workspace_bytes(rows) : 0; }

size_t round256(size_t n) { return (n + 255) / 256 * 256; }

size_t dtype_bytes(int dtype) { return dtype == MGLU_BF16 ? 2u : 4u; }

// The decode kernel needs its scratch; other paths ignore it.
int check_scratch(int64_t T, int dtype, int64_t rows, const void *ws, size_t ws_bytes)
{
    if (T == 0 || path_for(T, dtype) != MGLU_PATH_DECODE)
        return MGLU_OK;
    if (!ws || ws_bytes < scratch_bytes(rows))
        return MGLU_ERR_INVALID;
    if (!aligned(ws, 16))
        return MGLU_ERR_ALIGN;
    return MGLU_OK;
}

bool sizes_ok(int64_t T, int64_t d, int64_t h)
{
    const int64_t lim = (int64_t)1 << 31;
    if (T < 0 || d <= 0 || h <= 0 || T >= lim || d >= lim || h >= lim)
        return false;
    const int64_t mx = d > h ? d : h;
    return T == 0 || mx <= ((int64_t)1 << 62) / (T > 0 ? T : 1);
}

int check_forward(const void *x, int64_t T, int64_t d, const void *W, int64_t h, const uint8_t *packed, int n_m,
                  int act, int dtype, const void *out)
{
    if (!sizes_ok(T, d, h))
        return MGLU_ERR_INVALID;
    if ((act & ~MGLU_GATE_DENSE) < 0 || (act & ~MGLU_GATE_DENSE) > 2 || (dtype != MGLU_BF16 && dtype != MGLU_F32))
        return MGLU_ERR_INVALID;
    if (!nm_supported(n_m))
        return MGLU_ERR_UNSUPPORTED;
    if (!W || !packed || (T > 0 && (!x || !out)))
        return MGLU_ERR_INVALID;
    if (dtype == MGLU_BF16) {
        if (!aligned(W, 16) || !aligned(packed, 16) || (T > 0 && (!aligned(x, 16) || !aligned(out, 16))))
            return MGLU_ERR_ALIGN;
        if (d % 8 != 0)
            return MGLU_ERR_ALIGN;  // rows of W start on 16 bytes and a lane's 8 weights share their mask bytes
    } else {
        if (!aligned(W, 4) || (T > 0 && (!aligned(x, 4) || !aligned(out, 4))))
            return MGLU_ERR_ALIGN;
    }
    return MGLU_OK;
}

int check_down(const void *hid, int64_t T, int64_t h, const void *Wd, int64_t d, int dtype, const void *y)
{
    if (!sizes_ok(T, h, d))
        return MGLU_ERR_INVALID;
    if (dtype != MGLU_BF16 && dtype != MGLU_F32)
        return MGLU_ERR_INVALID;
    if (!Wd || (T > 0 && (!hid || !y)))
        return MGLU_ERR_INVALID;
    if (dtype == MGLU_BF16) {
        if (!aligned(Wd, 16) || (T > 0 && (!aligned(hid, 16) || !aligned(y, 16))))
            return MGLU_ERR_ALIGN;
        if (h % 8 != 0)
            return MGLU_ERR_ALIGN;  // rows of W_down start on 16 bytes
    } else {
        if (!aligned(Wd, 4) || (T > 0 && (!aligned(hid, 4) || !aligned(y, 4))))
            return MGLU_ERR_ALIGN;
    }
    return MGLU_OK;
}

template <int NM>
int pack_dispatch(const uint8_t *in, int64_t d, int64_t h, uint8_t *outp, bool unpack, cudaStream_t s)
{
    const int64_t hd = h * d;
    const int64_t nbytes = (hd * NM + 7) / 8;
    const int64_t chunks = (nbytes + 15) / 16;
    const int vec = (hd % 16 == 0) && aligned(unpack ? outp : in, 16);
    const int64_t blocks = (chunks + 255) / 256;
    if (blocks > 0x7FFFFFFF)
        return MGLU_ERR_INVALID;
    if (unpack)
        mglu::unpack_kernel<NM><<<(unsigned)blocks, 256, 0, s>>>(in, hd, nbytes, outp, vec);
    else
        mglu::pack_kernel<NM><<<(unsigned)blocks, 256, 0, s>>>(in, hd, nbytes, outp, vec);
    return check_launch(unpack ? "unpack launch" : "pack launch");
}

template <int NM>
int pack_logits_dispatch(const uint16_t *in, int64_t d, int64_t h, uint8_t *outp, cudaStream_t s)
{
    const int64_t hd = h * d;
    const int64_t nbytes = (hd * NM + 7) / 8;
    const int64_t chunks = (nbytes + 15) / 16;
    const int vec = (hd % 8 == 0) && aligned(in, 16);
    const int64_t blocks = (chunks + 255) / 256;
    if (blocks > 0x7FFFFFFF)
        return MGLU_ERR_INVALID;
    mglu::pack_logits_kernel<NM><<<(unsigned)blocks, 256, 0, s>>>(in, hd, nbytes, outp, vec);
    return check_launch("pack logits launch");
}

int pack_common(const uint8_t *in, int n_m, int64_t d, int64_t h, uint8_t *outp, bool unpack, void *stream)
{
    if (d <= 0 || h <= 0 || !in || !outp)
        return MGLU_ERR_INVALID;
    if (!nm_supported(n_m))
        return MGLU_ERR_UNSUPPORTED;
    if (!aligned(unpack ? in : outp, 16))
        return MGLU_ERR_ALIGN;
    if (h > ((int64_t)1 << 62) / d)
        return MGLU_ERR_INVALID;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    switch (n_m) {
    case 1: return pack_dispatch<1>(in, d, h, outp, unpack, s);
    case 2: return pack_dispatch<2>(in, d, h, outp, unpack, s);
    case 4: return pack_dispatch<4>(in, d, h, outp, unpack, s);
    default: return pack_dispatch<8>(in, d, h, outp, unpack, s);
    }
}

// ------------------------------------------------------------------ built-in scratch
// Decode scratch for mglu_forward_decode_static: the same layout as a caller
// buffer of mglu_scratch_bytes(MGLU_STATIC_SCRATCH_MAX_ROWS) bytes.  It lives
// in the library's device image, so no call has to allocate it: that entry
// point serves callers with no device allocator of their own (a plain-C host)
// or with a fixed memory budget that forbids allocating after start-up.
constexpr size_t kStaticScratchBytes = (size_t)mglu::dec::workspace_bytes(MGLU_STATIC_SCRATCH_MAX_ROWS);

std::mutex g_static_mu;
void *g_static_scratch_ptr[kMaxDevices] = {nullptr};

}  // namespace

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

namespace {

// Device address of the built-in scratch on `dev`, looked up (and the whole
// scratch cleared on `s`) the first time each device is used.
int static_scratch(int dev, cudaStream_t s, void **ptr)
{
    std::lock_guard<std::mutex> lock(g_static_mu);
    if (!g_static_scratch_ptr[dev]) {
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess)
            return cuda_fail(e, "cudaGetSymbolAddress(built-in decode scratch)");
        if ((e = cudaMemsetAsync(p, 0, kStaticScratchBytes, s)) != cudaSuccess)
            return cuda_fail(e, "clear built-in decode scratch");
        g_static_scratch_ptr[dev] = p;
    }
    *ptr = g_static_scratch_ptr[dev];
    return MGLU_OK;
}

// ------------------------------------------------------------------ training path
// cuBLAS is loaded on the first backward call (dlopen), so the forward
// library does not depend on it.  It serves the two plain GEMMs of the
// backward; the MGLU-specific steps are this library's kernels.
struct Cublas {
    using Create = cublasStatus_t (*)(cublasHandle_t *);
    using SetStream = cublasStatus_t (*)(cublasHandle_t, cudaStream_t);
    using GemmEx = cublasStatus_t (*)(cublasHandle_t, cublasOperation_t, cublasOperation_t, int, int, int,
                                      const void *, const void *, cudaDataType, int, const void *, cudaDataType, int,
                                      const void *, void *, cudaDataType, int, cublasComputeType_t, cublasGemmAlgo_t);
    using GemmBatched = cublasStatus_t (*)(cublasHandle_t, cublasOperation_t, cublasOperation_t, int, int, int,
                                           const void *, const void *, cudaDataType, int, long long, const void *,
                                           cudaDataType, int, long long, const void *, void *, cudaDataType, int,
                                           long long, int, cublasComputeType_t, cublasGemmAlgo_t);
    Create create = nullptr;
    SetStream set_stream = nullptr;
    GemmEx gemm = nullptr;
    GemmBatched gemm_batched = nullptr;
    cublasHandle_t handle[kMaxDevices] = {};
};

std::mutex g_cublas_mu;
Cublas g_cublas;

int cublas_for(int dev, cudaStream_t s, Cublas **out)
{
    std::lock_guard<std::mutex> lock(g_cublas_mu);
    Cublas &c = g_cublas;
    if (!c.create) {
        void *h = dlopen("libcublas.so.12", RTLD_NOW | RTLD_LOCAL);
        if (!h)
            h = dlopen("libcublas.so", RTLD_NOW | RTLD_LOCAL);
        if (!h) {
            snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "libcublas could not be loaded");
            return MGLU_ERR_CUDA;
        }
        c.set_stream = reinterpret_cast<Cublas::SetStream>(dlsym(h, "cublasSetStream_v2"));
        c.gemm = reinterpret_cast<Cublas::GemmEx>(dlsym(h, "cublasGemmEx"));
        c.gemm_batched = reinterpret_cast<Cublas::GemmBatched>(dlsym(h, "cublasGemmStridedBatchedEx"));
        Cublas::Create cr = reinterpret_cast<Cublas::Create>(dlsym(h, "cublasCreate_v2"));
        if (!cr || !c.set_stream || !c.gemm || !c.gemm_batched) {
            snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "libcublas lacks a needed entry point");
            return MGLU_ERR_CUDA;
        }
        c.create = cr;
    }
    if (!c.handle[dev] && c.create(&c.handle[dev]) != CUBLAS_STATUS_SUCCESS) {
        c.handle[dev] = nullptr;
        snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "cublasCreate failed");
        return MGLU_ERR_CUDA;
    }
    if (c.set_stream(c.handle[dev], s) != CUBLAS_STATUS_SUCCESS) {
        snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "cublasSetStream failed");
        return MGLU_ERR_CUDA;
    }
    *out = &c;
    return MGLU_OK;
}

struct BwdLayout {
    size_t g, b, e, total;  // byte offsets of G, B, E in the workspace and its size
};

BwdLayout bwd_layout(int64_t T, int64_t d, int64_t h, int n_m)
{
    BwdLayout L;
    const size_t np = (size_t)n_m + 1;
    L.g = 0;
    L.b = L.g + round256((size_t)T * np * (size_t)h * 2);
    L.e = L.b + round256(np * (size_t)h * (size_t)d * 2);
    L.total = L.e + round256(np * (size_t)h * (size_t)d * 4);
    return L;
}

template <int NM>
int backward_nm(const void *x, int64_t T, int64_t d, const void *W, int64_t h, const uint8_t *packed, int act,
                const void *dout, float *dx, float *dW, float *dM, uint8_t *ws, cudaStream_t s)
{
    const BwdLayout L = bwd_layout(T, d, h, NM);
    __nv_bfloat16 *G = reinterpret_cast<__nv_bfloat16 *>(ws + L.g);
    __nv_bfloat16 *B = reinterpret_cast<__nv_bfloat16 *>(ws + L.b);
    float *E = reinterpret_cast<float *>(ws + L.e);
    int rc;
    // 1. a_i - c_i and sum_i c_i from the recomputed products (tcgen05)
    if ((rc = launch_prefill<NM, true>(x, T, d, W, h, packed, act, nullptr, nullptr, s, nullptr, dout, G)))
        return rc;
    // 2. the masked operand [M_1.W; ...; M_n.W; W]
    const int64_t chunks = h * (d / 8);
    mglu::tr::masked_weights_kernel<NM><<<(unsigned)((chunks + 255) / 256), 256, 0, s>>>(
        reinterpret_cast<const __nv_bfloat16 *>(W), packed, h, d, B);
    if ((rc = check_launch("masked weights launch")))
        return rc;
    int dev = 0;
    if ((rc = current_device(&dev)))
        return rc;
    Cublas *cb = nullptr;
    if ((rc = cublas_for(dev, s, &cb)))
        return rc;
    const float one = 1.0f, zero = 0.0f;
    const int K = (int)((NM + 1) * h);
    // 3. dx [T][d] = G [T][K] B [K][d]   (column-major: dx^T = B^T-view * G-view)
    if (cb->gemm(cb->handle[dev], CUBLAS_OP_N, CUBLAS_OP_N, (int)d, (int)T, K, &one, B, CUDA_R_16BF, (int)d, G,
                 CUDA_R_16BF, K, &zero, dx, CUDA_R_32F, (int)d, CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT) !=
        CUBLAS_STATUS_SUCCESS) {
        snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "cublasGemmEx (dx) failed");
        return MGLU_ERR_CUDA;
    }
    // 4. E_i [h][d] = G_i^T x for the NM + 1 column blocks G_i of G
    if (cb->gemm_batched(cb->handle[dev], CUBLAS_OP_N, CUBLAS_OP_T, (int)d, (int)h, (int)T, &one, x, CUDA_R_16BF,
                         (int)d, 0, G, CUDA_R_16BF, K, (long long)h, &zero, E, CUDA_R_32F, (int)d,
                         (long long)(h * d), NM + 1, CUBLAS_COMPUTE_32F, CUBLAS_GEMM_DEFAULT) != CUBLAS_STATUS_SUCCESS) {
        snprintf(g_last_cuda_error, sizeof(g_last_cuda_error), "cublasGemmStridedBatchedEx (E) failed");
        return MGLU_ERR_CUDA;
    }
    // 5. dW = sum_i M_i . E_i + E_NM, dM_i = W . E_i
    const int64_t quads = h * d / 4;
    mglu::tr::combine_kernel<NM><<<(unsigned)((quads + 255) / 256), 256, 0, s>>>(
        E, reinterpret_cast<const __nv_bfloat16 *>(W), packed, h, d, dW, dM);
    return check_launch("combine launch");
}

}  // namespace

extern "C" {

size_t mglu_backward_workspace_bytes(int64_t T, int64_t d, int64_t h, int n_m)
{
    if (T <= 0 || d <= 0 || h <= 0 || !nm_supported(n_m))
        return 0;
    return bwd_layout(T, d, h, n_m).total;
}

int mglu_backward(const void *x, int64_t T, int64_t d, const void *W, int64_t h, const uint8_t *packed, int n_m,
                  int act, const void *dout, float *dx, float *dW, float *dlogits, void *workspace,
                  size_t workspace_bytes, void *stream)
{
    int rc = check_forward(x, T, d, W, h, packed, n_m, act, MGLU_BF16, dout);
    if (rc)
        return rc;
    if (act & MGLU_GATE_DENSE)
        return MGLU_ERR_UNSUPPORTED;  // the backward covers the method's own gate
    if (T == 0)
        return MGLU_OK;
    if (!dx || !dW || !workspace)
        return MGLU_ERR_INVALID;
    if (!aligned(dx, 16) || !aligned(dW, 16) || (dlogits && !aligned(dlogits, 16)) || !aligned(workspace, 256))
        return MGLU_ERR_ALIGN;
    if (workspace_bytes < mglu_backward_workspace_bytes(T, d, h, n_m))
        return MGLU_ERR_INVALID;
    if (T > INT32_MAX / 8 || (n_m + 1) * h >= INT32_MAX || d >= INT32_MAX)
        return MGLU_ERR_INVALID;  // cuBLAS takes int dimensions
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    uint8_t *ws = reinterpret_cast<uint8_t *>(workspace);
    switch (n_m) {
    case 1: return backward_nm<1>(x, T, d, W, h, packed, act, dout, dx, dW, dlogits, ws, s);
    case 2: return backward_nm<2>(x, T, d, W, h, packed, act, dout, dx, dW, dlogits, ws, s);
    case 4: return backward_nm<4>(x, T, d, W, h, packed, act, dout, dx, dW, dlogits, ws, s);
    default: return backward_nm<8>(x, T, d, W, h, packed, act, dout, dx, dW, dlogits, ws, s);
    }
}

size_t mglu_packed_bytes(int n_m, int64_t d, int64_t h)
{
    if (!nm_supported(n_m) || d <= 0 || h <= 0)
        return 0;
    return (size_t)((h * d * n_m + 7) / 8);
}

int mglu_pack_masks(const uint8_t *masks, int n_m, int64_t d, int64_t h, uint8_t *packed, void *stream)
{
    return pack_common(masks, n_m, d, h, packed, false, stream);
}

int mglu_pack_mask_logits(const void *logits, int n_m, int64_t d, int64_t h, uint8_t *packed, void *stream)
{
    if (d <= 0 || h <= 0 || !logits || !packed)
        return MGLU_ERR_INVALID;
    if (!nm_supported(n_m))
        return MGLU_ERR_UNSUPPORTED;
    if (!aligned(packed, 16) || !aligned(logits, 2))
        return MGLU_ERR_ALIGN;
    if (h > ((int64_t)1 << 62) / d)
        return MGLU_ERR_INVALID;
    const uint16_t *in = reinterpret_cast<const uint16_t *>(logits);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    switch (n_m) {
    case 1: return pack_logits_dispatch<1>(in, d, h, packed, s);
    case 2: return pack_logits_dispatch<2>(in, d, h, packed, s);
    case 4: return pack_logits_dispatch<4>(in, d, h, packed, s);
    default: return pack_logits_dispatch<8>(in, d, h, packed, s);
    }
}

int mglu_unpack_masks(const uint8_t *packed, int n_m, int64_t d, int64_t h, uint8_t *masks, void *stream)
{
    return pack_common(packed, n_m, d, h, masks, true, stream);
}

size_t mglu_scratch_bytes(int64_t rows) { return scratch_bytes(rows); }

int mglu_forward(const void *x, int64_t T, int64_t d, const void *W, int64_t h, const uint8_t *packed, int n_m,
                 int act, int dtype, void *out, void *scratch, size_t scratch_bytes_, void *stream)
{
    int rc = check_forward(x, T, d, W, h, packed, n_m, act, dtype, out);
    if (rc)
        return rc;
    if ((rc = check_scratch(T, dtype, h, scratch, scratch_bytes_)))
        return rc;
    return run_product(x, T, d, W, h, packed, n_m, act, dtype, out, scratch, reinterpret_cast<cudaStream_t>(stream));
}

int mglu_forward_partials(const void *x, int64_t T, int64_t d, const void *W, int64_t h, const uint8_t *packed,
                          int n_m, float *partials, void *scratch, size_t scratch_bytes_, void *stream)
{
    // n_m = 0 (the dense product alone) is allowed here; packed is then not read
    int rc = check_forward(x, T, d, W, h, packed, n_m == 0 ? 1 : n_m, MGLU_ACT_SWISH, MGLU_BF16, partials);
    if (rc)
        return rc;
    if (T > 16)
        return MGLU_ERR_UNSUPPORTED;
    if (T == 0)
        return MGLU_OK;
    if (!scratch || scratch_bytes_ < scratch_bytes(h))
        return MGLU_ERR_INVALID;
    if (!aligned(scratch, 16))
        return MGLU_ERR_ALIGN;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    switch (n_m) {
    case 0: return decode_nt<0>(x, T, d, W, h, packed, 0, nullptr, scratch, s, nullptr, partials);
    case 1: return decode_nt<1>(x, T, d, W, h, packed, 0, nullptr, scratch, s, nullptr, partials);
    case 2: return decode_nt<2>(x, T, d, W, h, packed, 0, nullptr, scratch, s, nullptr, partials);
    case 4: return decode_nt<4>(x, T, d, W, h, packed, 0, nullptr, scratch, s, nullptr, partials);
    case 8: return decode_nt<8>(x, T, d, W, h, packed, 0, nullptr, scratch, s, nullptr, partials);
    default: return MGLU_ERR_UNSUPPORTED;
    }
}

int mglu_forward_weighted(const void *x, int64_t T, int64_t d, const void *W, int64_t h, const uint8_t *packed,
                          int n_m, int act, int dtype, const float *mask_weights, void *out, void *scratch,
                          size_t scratch_bytes_, void *stream)
{
    int rc = check_forward(x, T, d, W, h, packed, n_m, act, dtype, out);
    if (rc)
        return rc;
    if (T > 0 && !mask_weights)
        return MGLU_ERR_INVALID;
    if (T > 0 && !aligned(mask_weights, 4))
        return MGLU_ERR_ALIGN;
    if ((rc = check_scratch(T, dtype, h, scratch, scratch_bytes_)))
        return rc;
    return run_product(x, T, d, W, h, packed, n_m, act, dtype, out, scratch, reinterpret_cast<cudaStream_t>(stream),
                       mask_weights);
}

int mglu_route_topk(const void *x, int64_t T, int64_t d, const void *W_r, int n_m, int k, int mode, int dtype,
                    float *weights, float *scores, void *stream)
{
    if (!sizes_ok(T, d, 1) || (dtype != MGLU_BF16 && dtype != MGLU_F32) || (mode != MGLU_ROUTE_HARD &&
                                                                             mode != MGLU_ROUTE_SOFTMAX))
        return MGLU_ERR_INVALID;
    if (!nm_supported(n_m))
        return MGLU_ERR_UNSUPPORTED;
    if (k < 0 || k > n_m)
        return MGLU_ERR_INVALID;
    if (T == 0)
        return MGLU_OK;
    if (!x || !W_r || !weights)
        return MGLU_ERR_INVALID;
    const uintptr_t es = dtype == MGLU_BF16 ? 2 : 4;
    if (!aligned(x, es) || !aligned(W_r, es) || !aligned(weights, 4) || (scores && !aligned(scores, 4)))
        return MGLU_ERR_ALIGN;
    if (T > 0x7FFFFFFF)
        return MGLU_ERR_INVALID;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const int vec = d % 8 == 0 && aligned(x, 16) && aligned(W_r, 16);
    if (dtype == MGLU_BF16)
        return launch_pdl(mglu::route_kernel<__nv_bfloat16>, dim3((unsigned)T), dim3(256), 0, s, "route launch",
                          reinterpret_cast<const __nv_bfloat16 *>(x), T, d,
                          reinterpret_cast<const __nv_bfloat16 *>(W_r), n_m, k, mode, vec, weights, scores);
    return launch_pdl(mglu::route_kernel<float>, dim3((unsigned)T), dim3(256), 0, s, "route launch",
                      reinterpret_cast<const float *>(x), T, d, reinterpret_cast<const float *>(W_r), n_m, k, mode,
                      0, weights, scores);
}

int mglu_forward_routed(const void *x, int64_t T, int64_t d, const void *W, int64_t h, const uint8_t *packed,
                        int n_m, const void *W_r, int k, int mode, int act, int dtype, float *weights, float *scores,
                        void *out, void *scratch, size_t scratch_bytes_, void *stream)
{
    int rc = check_forward(x, T, d, W, h, packed, n_m, act, dtype, out);
    if (rc)
        return rc;
    if (mode != MGLU_ROUTE_HARD && mode != MGLU_ROUTE_SOFTMAX)
        return MGLU_ERR_INVALID;
    if (k < 0 || k > n_m)
        return MGLU_ERR_INVALID;
    if (T == 0)
        return MGLU_OK;
    if (!W_r || !weights)
        return MGLU_ERR_INVALID;
    const uintptr_t es = dtype == MGLU_BF16 ? 2 : 4;
    if (!aligned(W_r, es) || !aligned(weights, 4) || (scores && !aligned(scores, 4)))
        return MGLU_ERR_ALIGN;
    if ((rc = check_scratch(T, dtype, h, scratch, scratch_bytes_)))
        return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (path_for(T, dtype) != MGLU_PATH_DECODE) {
        // the router, then the weighted forward
        if ((rc = mglu_route_topk(x, T, d, W_r, n_m, k, mode, dtype, weights, scores, stream)))
            return rc;
        return run_product(x, T, d, W, h, packed, n_m, act, dtype, out, scratch, s, weights);
    }
    const mglu::dec::Router ro{reinterpret_cast<const __nv_bfloat16 *>(W_r), k, mode,
                               d % 8 == 0 && aligned(x, 16) && aligned(W_r, 16) ? 1 : 0, weights, scores};
    switch (n_m) {
    case 1: return decode_routed<1>(x, T, d, W, h, packed, act, out, scratch, s, ro);
    case 2: return decode_routed<2>(x, T, d, W, h, packed, act, out, scratch, s, ro);
    case 4: return decode_routed<4>(x, T, d, W, h, packed, act, out, scratch, s, ro);
    case 8: return decode_routed<8>(x, T, d, W, h, packed, act, out, scratch, s, ro);
    default: return MGLU_ERR_UNSUPPORTED;
    }
}

int mglu_down_proj(const void *hid, int64_t T, int64_t h, const void *W_down, int64_t d, int dtype, void *y,
                   void *scratch, size_t scratch_bytes_, void *stream)
{
    int rc = check_down(hid, T, h, W_down, d, dtype, y);
    if (rc)
        return rc;
    if ((rc = check_scratch(T, dtype, d, scratch, scratch_bytes_)))
        return rc;
    return run_product(hid, T, h, W_down, d, nullptr, 0, 0, dtype, y, scratch, reinterpret_cast<cudaStream_t>(stream));
}

size_t mglu_workspace_bytes(int64_t T, int64_t d, int64_t h, int n_m, int dtype)
{
    (void)n_m;
    if (T < 0 || d <= 0 || h <= 0 || (dtype != MGLU_BF16 && dtype != MGLU_F32))
        return 0;
    return scratch_bytes(d > h ? d : h) + round256((size_t)T * (size_t)h * dtype_bytes(dtype));
}

int mglu_forward_down(const void *x, int64_t T, int64_t d, const void *W, int64_t h, const uint8_t *packed, int n_m,
                      int act, int dtype, const void *W_down, void *workspace, size_t workspace_bytes, void *y,
                      void *stream)
{
    if (T < 0 || d <= 0 || h <= 0 || (dtype != MGLU_BF16 && dtype != MGLU_F32))
        return MGLU_ERR_INVALID;
    if (T > 0 && (!workspace || workspace_bytes < mglu_workspace_bytes(T, d, h, n_m, dtype)))
        return MGLU_ERR_INVALID;
    // workspace: the decode scratch first (its place does not depend on T),
    // then the hidden activation
    uint8_t *scratch = reinterpret_cast<uint8_t *>(workspace);
    uint8_t *hid = scratch + scratch_bytes(d > h ? d : h);
    int rc = check_forward(x, T, d, W, h, packed, n_m, act, dtype, T > 0 ? hid : nullptr);
    if (rc)
        return rc;
    if ((rc = check_down(hid, T, h, W_down, d, dtype, y)))
        return rc;
    if (T == 0)
        return MGLU_OK;
    if (!aligned(workspace, 16))
        return MGLU_ERR_ALIGN;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if ((rc = run_product(x, T, d, W, h, packed, n_m, act, dtype, hid, scratch, s)))
        return rc;
    return run_product(hid, T, h, W_down, d, nullptr, 0, 0, dtype, y, scratch, s);
}

int mglu_forward_decode_static(const void *x, int64_t T, int64_t d, const void *W, int64_t h,
                               const uint8_t *packed, int n_m, int act, void *out, void *stream)
{
    int rc = check_forward(x, T, d, W, h, packed, n_m, act, MGLU_BF16, out);
    if (rc)
        return rc;
    if (T > 16)
        return MGLU_ERR_UNSUPPORTED;
    if (h > MGLU_STATIC_SCRATCH_MAX_ROWS) {
        snprintf(g_last_cuda_error, sizeof(g_last_cuda_error),
                 "mglu_forward_decode_static: h = %lld exceeds the built-in scratch limit of %d rows", (long long)h,
                 MGLU_STATIC_SCRATCH_MAX_ROWS);
        return MGLU_ERR_INVALID;
    }
    if (T == 0)
        return MGLU_OK;
    int dev = 0;
    if ((rc = current_device(&dev)))
        return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    void *ws = nullptr;
    if ((rc = static_scratch(dev, s, &ws)))
        return rc;
    return by_nm<DecodeF>(n_m, x, T, d, W, h, packed, act, out, ws, s, (const float *)nullptr);
}

size_t mglu_host_workspace_bytes(int64_t T, int64_t d, int64_t h, int n_m, int dtype, int with_down)
{
    (void)n_m;
    if (T < 0 || d <= 0 || h <= 0 || (dtype != MGLU_BF16 && dtype != MGLU_F32))
        return 0;
    const size_t es = dtype_bytes(dtype);
    const size_t xb = round256((size_t)T * (size_t)d * es);
    const size_t rb = round256((size_t)T * (size_t)(with_down ? d : h) * es);
    const size_t hb = with_down ? round256((size_t)T * (size_t)h * es) : 0;
    return scratch_bytes(d > h ? d : h) + xb + rb + hb;
}

int mglu_forward_host(const void *x_host, int64_t T, int64_t d, const void *W, int64_t h, const uint8_t *packed,
                      int n_m, int act, int dtype, const void *W_down, void *workspace, size_t workspace_bytes,
                      void *result_host, void *stream)
{
    if (T < 0 || d <= 0 || h <= 0 || (dtype != MGLU_BF16 && dtype != MGLU_F32))
        return MGLU_ERR_INVALID;
    if (T == 0)
        return MGLU_OK;
    if (!x_host || !result_host || !workspace)
        return MGLU_ERR_INVALID;
    const int with_down = W_down != nullptr;
    if (workspace_bytes < mglu_host_workspace_bytes(T, d, h, n_m, dtype, with_down))
        return MGLU_ERR_INVALID;
    if (!aligned(workspace, 256))
        return MGLU_ERR_ALIGN;
    const size_t es = dtype_bytes(dtype);
    const size_t xbytes = (size_t)T * (size_t)d * es;
    const size_t rbytes = (size_t)T * (size_t)(with_down ? d : h) * es;
    // workspace: the decode scratch (sized for max(d, h) rows whatever the
    // call, so its place never moves), the staged x, the result, the hidden
    uint8_t *scratch = reinterpret_cast<uint8_t *>(workspace);
    uint8_t *x_dev = scratch + scratch_bytes(d > h ? d : h);
    uint8_t *r_dev = x_dev + round256(xbytes);
    uint8_t *hid = r_dev + round256(rbytes);
    // every argument is checked before anything is queued
    int rc = check_forward(x_dev, T, d, W, h, packed, n_m, act, dtype, with_down ? (const void *)hid : r_dev);
    if (rc)
        return rc;
    if (with_down && (rc = check_down(hid, T, h, W_down, d, dtype, r_dev)))
        return rc;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemcpyAsync(x_dev, x_host, xbytes, cudaMemcpyHostToDevice, s);
    if (e != cudaSuccess)
        return cuda_fail(e, "copy x to the device");
    if ((rc = run_product(x_dev, T, d, W, h, packed, n_m, act, dtype, with_down ? hid : r_dev, scratch, s)))
        return rc;
    if (with_down && (rc = run_product(hid, T, h, W_down, d, nullptr, 0, 0, dtype, r_dev, scratch, s)))
        return rc;
    if ((e = cudaMemcpyAsync(result_host, r_dev, rbytes, cudaMemcpyDeviceToHost, s)) != cudaSuccess)
        return cuda_fail(e, "copy the result to the host");
    return MGLU_OK;
}

int mglu_forward_path(int64_t T, int dtype) { return path_for(T, dtype); }

int mglu_set_decode_max_tokens(int t)
{
    if (t < 0 || t > 16)
        return MGLU_ERR_INVALID;
    return g_decode_max_tokens.exchange(t);
}

int mglu_last_device_status(void *stream)
{
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess)
        return cuda_fail(e, "cudaStreamSynchronize");
    int v = 0;
    if ((e = cudaMemcpyFromSymbol(&v, mglu::g_status, sizeof(int))) != cudaSuccess)
        return cuda_fail(e, "read status");
    if (v != 0) {
        const int zero = 0;
        if ((e = cudaMemcpyToSymbol(mglu::g_status, &zero, sizeof(int))) != cudaSuccess)
            return cuda_fail(e, "clear status");
    }
    return v;
}

const char *mglu_last_cuda_error(void) { return g_last_cuda_error; }

uint64_t mglu_kernel_launches(void) { return g_kernel_launches.load(std::memory_order_relaxed); }

#ifdef MGLU_TEST_HOOKS
// Test-hook build only (not part of the product ABI): nonzero stops the
// tensor-core kernel's producer after its first stage on the current device.
int mglu_test_set_stall(int on)
{
    const int v = on ? 1 : 0;
    const cudaError_t e = cudaMemcpyToSymbol(mglu::g_test_stall_producer, &v, sizeof(int));
    return e == cudaSuccess ? MGLU_OK : cuda_fail(e, "set test stall");
}
#endif

const char *mglu_status_string(int status)
{
    switch (status) {
    case MGLU_OK: return "ok";
    case MGLU_ERR_INVALID: return "invalid argument";
    case MGLU_ERR_UNSUPPORTED: return "unsupported n_m, or too many tokens for the decode-only entry point";
    case MGLU_ERR_ALIGN: return "alignment requirement not met";
    case MGLU_ERR_CUDA: return "CUDA error";
    case MGLU_ERR_TIMEOUT: return "device wait timed out";
    default: return "unknown status";
    }
}

}  // extern "C"
