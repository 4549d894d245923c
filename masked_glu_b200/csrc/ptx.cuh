// ptx.cuh -- thin inline-PTX wrappers for sm_100a used by the MGLU kernels:
// mbarriers with bounded waits, TMA tile loads, cluster / DSMEM access,
// legacy mma.sync (bf16), and the tcgen05 (TMEM / UMMA) instructions.
#pragma once
#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

namespace mglu {

// ---------------------------------------------------------------- status word
// Device status of the library (per device).  Kernels whose bounded waits run
// out store MGLU_ERR_TIMEOUT (-5) here and leave; the host reads and clears it
// in mglu_last_device_status().
__device__ int g_status;

__device__ __forceinline__ void record_status(int s) { atomicCAS(&g_status, 0, s); }

// ---------------------------------------------------------------- addresses
__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete, for at most about
// one second of wall time (20 ms in the test-hook build, whose tests make a
// wait run out on purpose).  Returns false (and records MGLU_ERR_TIMEOUT) if
// the wait gave up.  Every mbarrier wait in this library goes through here.
#ifdef MGLU_TEST_HOOKS
constexpr uint64_t kWaitLimitNs = 20000000ull;
// Test hook: when nonzero, the tensor-core kernel's producer issues the
// loads of its first stage only, so every later wait of the CTA runs out.
__device__ int g_test_stall_producer;
#else
constexpr uint64_t kWaitLimitNs = 1000000000ull;
#endif

__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((it & 63u) == 0 && global_timer_ns() - t0 > kWaitLimitNs) {
            record_status(-5);
            return false;
        }
    }
}

// Wait for a phase as a whole warp (all 32 lanes call it together): lane 0
// polls the barrier, then the warp synchronizes and every lane takes lane 0's
// answer, so the lanes' later shared-memory reads are ordered after lane 0's
// acquire.  On B200, warps whose 32 lanes each polled a TMA barrier
// themselves occasionally read stale operands afterwards (about one read in
// ten thousand, only when the warp had to wait); with one polling lane per
// warp every read was correct.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t *bar, uint32_t parity)
{
    int ok = 1;
    if ((threadIdx.x & 31) == 0)
        ok = mbar_wait(bar, parity) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

// The same for the phase of up to three barriers (null ones are skipped):
// lane 0 waits for each in turn, then one broadcast and warp synchronization.
__device__ __forceinline__ bool mbar_wait_warp3(uint64_t *a, uint64_t *b, uint64_t *c, uint32_t parity)
{
    int ok = 1;
    if ((threadIdx.x & 31) == 0)
        ok = (mbar_wait(a, parity) && (!b || mbar_wait(b, parity)) && (!c || mbar_wait(c, parity))) ? 1 : 0;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    __syncwarp();
    return ok != 0;
}

// ---------------------------------------------------------------- cp.async
// Per-thread asynchronous copy global -> shared of cp bytes (4, 8 or 16), of
// which the first src bytes are read and the rest zero-filled (src = 0
// reads nothing).  .cg (16 bytes) bypasses L1, .ca caches in L1.  The copy's
// data is visible to the issuing thread once cp.async.wait_group says its
// group has completed.
__device__ __forceinline__ void cp_async_cg16(uint32_t dst, const void *src, uint32_t src_bytes)
{
    asm volatile("cp.async.cg.shared.global.L2::256B [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes)
                 : "memory");
}

template <int CP>
__device__ __forceinline__ void cp_async_ca(uint32_t dst, const void *src, uint32_t src_bytes)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], %2, %3;" ::"r"(dst), "l"(src), "n"(CP), "r"(src_bytes)
                 : "memory");
}

// The same copies with every byte read.
__device__ __forceinline__ void cp_async_cg16(uint32_t dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global.L2::256B [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

template <int CP>
__device__ __forceinline__ void cp_async_ca(uint32_t dst, const void *src)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], %2;" ::"r"(dst), "l"(src), "n"(CP) : "memory");
}

__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }

template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// ---------------------------------------------------------------- dependent launch
// Kernels are launched with programmatic stream serialization: the next
// kernel on the stream may be scheduled once every CTA of this one has
// signalled, and it waits in pdl_wait() until this grid has completed and its
// memory is visible, before touching global memory.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---------------------------------------------------------------- fences
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- TMA
// 2-D tiled load of one box into shared memory; completion is signalled on
// `bar` as transaction bytes.  c0 is the innermost (contiguous) coordinate in
// elements and must be a multiple of 16 bytes; c1 the row.
__device__ __forceinline__ void tma_load_2d(void *smem_dst, const CUtensorMap *map, uint64_t *bar, int c0,
                                            int c1)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::
            "r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
        : "memory");
}

// 3-D tiled load; c0 innermost (16-byte aligned in bytes), then c1, c2.
__device__ __forceinline__ void tma_load_3d(void *smem_dst, const CUtensorMap *map, uint64_t *bar, int c0, int c1,
                                            int c2)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::
            "r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
        : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------- cluster
__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Every thread of every CTA of the cluster arrives; returns once all have
// (release / acquire at cluster scope).  Not the .aligned form: callers may
// reach it from divergent code.
__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

// Address of the same shared-memory location in CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

// ---------------------------------------------------------------- bit tricks
// prmt in its default mode.  A selector nibble with bit 3 set replicates the
// most significant bit of the selected byte into the whole output byte.
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// ---------------------------------------------------------------- mma.sync
// D(16x8, f32) += A(16x16, bf16, row) * B(16x8, bf16, col).
__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
        "{%0, %1, %2, %3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------- tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// D[tmem] (+)= A[smem desc] * B[smem desc]; kind::f16 (bf16 inputs, f32 accumulate).
__device__ __forceinline__ void umma_f16_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                            uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on an mbarrier once all previously issued tcgen05.mma of this thread
// have completed.
__device__ __forceinline__ void umma_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 bit, 8 consecutive columns: thread t of the warp gets lane
// (warp quadrant base + t), columns [col, col + 8).
__device__ __forceinline__ void tmem_ld_x8(uint32_t taddr, uint32_t (&r)[8])
{
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
}

// Shared-memory matrix descriptor for a K-major bf16 tile stored with the
// 128-byte swizzle: rows of 64 elements (128 B), 8-row groups 1024 B apart.
// The tile base must be 1024-byte aligned.  Advancing along K by 16 elements
// adds 32 bytes (2 in the >>4 encoding) to the start address.
__device__ __forceinline__ uint64_t sw128_kmajor_desc(uint32_t smem_addr)
{
    uint64_t desc = 0;
    desc |= (uint64_t)((smem_addr >> 4) & 0x3FFF);  // start address
    desc |= (uint64_t)1 << 16;                        // leading byte offset (unused for this layout)
    desc |= (uint64_t)(1024 >> 4) << 32;              // stride byte offset: 8 rows x 128 B
    desc |= (uint64_t)1 << 46;                        // descriptor version (sm_100)
    desc |= (uint64_t)2 << 61;                        // layout: 128-byte swizzle
    return desc;
}

// ---------------------------------------------------------------- CTA pairs (cta_group::2)
// A pair of CTAs in a cluster of two: one MMA issued by the first (rank 0)
// computes a 256-row tile whose A rows and B columns are split between the two
// CTAs' shared memories and whose accumulator rows live in both CTAs' TMEM.

// The address of this CTA's shared-memory location `p` in CTA `rank` of the
// cluster (same offset), for remote mbarrier arrivals and TMA barriers.
__device__ __forceinline__ uint32_t cluster_addr(const void *p, uint32_t rank)
{
    return mapa_shared(smem_u32(p), rank);
}

// Arrive on an mbarrier of a CTA of the cluster (default semantics: release
// at CTA scope).  Used to hand over data the arriving thread wrote into its
// OWN CTA's shared memory (made visible to the async proxy by a proxy fence
// first) to the peer CTA's MMA issuer, whose tensor-core reads go to that
// same shared memory; and to return an accumulator after its tcgen05.ld's
// completed.  A release at cluster scope would add a memory barrier per
// arrival that waits for the SM's TMA traffic (the builders of the CTA-pair
// kernel stalled on it: 1.09 ms instead of 0.60 ms for 4096 tokens, d = 2048,
// h = 8192, n_m = 4 on B200).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_bar)
{
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}

// 2-D tile load into this CTA's shared memory that completes its bytes on
// `leader_bar` (a cluster address, normally the pair's first CTA's barrier).
__device__ __forceinline__ void tma_load_2d_pair(void *smem_dst, const CUtensorMap *map, uint32_t leader_bar,
                                                 int c0, int c1)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
        "%4}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(leader_bar), "r"(c0), "r"(c1)
        : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t *dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// The pair's MMA, issued by the first CTA: D (both CTAs' TMEM, their own A
// rows) (+)= A (each CTA's shared memory, same offset) * B (columns split
// between the two CTAs' shared memories, same offset).
__device__ __forceinline__ void umma_f16_ss_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                                 uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on the mbarrier at `bar`'s offset in every CTA of `cta_mask` once all
// previously issued pair MMAs of this thread have completed.
__device__ __forceinline__ void umma_commit_pair(uint64_t *bar, uint16_t cta_mask)
{
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
            smem_u32(bar)),
        "h"(cta_mask)
        : "memory");
}

// Instruction descriptor, kind::f16: bf16 A and B, f32 accumulator, both
// operands K-major, shape M x N.
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N)
{
    return (1u << 4)                      // D format f32
           | (1u << 7)                    // A format bf16
           | (1u << 10)                   // B format bf16
           | ((uint32_t)(N >> 3) << 17)   // N / 8
           | ((uint32_t)(M >> 4) << 24);  // M / 16
}

}  // namespace mglu
