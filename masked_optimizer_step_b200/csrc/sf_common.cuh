// sf_common.cuh -- device helpers shared by the sm_100a kernels of the sparse step.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/sf.h"

#define SF_DEVICE __device__ __forceinline__

namespace sf {

// --------------------------------------------------------------------------------------------
// Status word and bounded waits.
// --------------------------------------------------------------------------------------------

// Programmatic dependent launch. A grid launched with programmatic stream serialization may
// start once every CTA of the grid before it has executed launch_dependents (or exited);
// griddep_wait blocks until that earlier grid has completed and its memory is visible. Without
// such a predecessor both are no-ops.
SF_DEVICE void griddep_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
SF_DEVICE void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

SF_DEVICE void set_status(uint32_t *st, uint32_t bits)
{
    if (st) atomicOr(st, bits);
}

SF_DEVICE uint64_t globaltimer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Every spin in these kernels gives up after this long, sets SF_STATUS_WAIT_TIMEOUT and lets
// the kernel unwind. A healthy wait lasts microseconds.
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s

// --------------------------------------------------------------------------------------------
// Block-wide scans and reductions (blockDim.x a multiple of 32, at most 1024).
// --------------------------------------------------------------------------------------------

SF_DEVICE int warp_inclusive_scan(int v)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        int n = __shfl_up_sync(0xffffffffu, v, d);
        if (lane >= d) v += n;
    }
    return v;
}

// Exclusive prefix sum over the block in thread order; *total gets the block sum.
// `scratch` holds at least 33 ints of shared memory. Contains __syncthreads.
SF_DEVICE int block_exclusive_scan(int v, int *scratch, int *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwarps = (blockDim.x + 31) >> 5;
    int inc = warp_inclusive_scan(v);
    if (lane == 31) scratch[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        int s = lane < nwarps ? scratch[lane] : 0;
        int si = warp_inclusive_scan(s);
        if (lane < nwarps) scratch[lane] = si - s;
        if (lane == nwarps - 1) scratch[32] = si;
    }
    __syncthreads();
    int res = scratch[warp] + inc - v;
    *total = scratch[32];
    __syncthreads();
    return res;
}

SF_DEVICE uint32_t warp_max_u32(uint32_t v)
{
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, d));
    return v;
}

// Block max of non-negative values as unsigned bits. `scratch` >= 33 words. Contains syncs.
SF_DEVICE uint32_t block_max_u32(uint32_t v, uint32_t *scratch)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int nwarps = (blockDim.x + 31) >> 5;
    v = warp_max_u32(v);
    if (lane == 0) scratch[warp] = v;
    __syncthreads();
    if (warp == 0) {
        uint32_t s = lane < nwarps ? scratch[lane] : 0u;
        s = warp_max_u32(s);
        if (lane == 0) scratch[32] = s;
    }
    __syncthreads();
    uint32_t r = scratch[32];
    __syncthreads();
    return r;
}

// --------------------------------------------------------------------------------------------
// mbarrier, TMA and tcgen05 wrappers (inline PTX, sm_100a).
// --------------------------------------------------------------------------------------------

SF_DEVICE uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

SF_DEVICE void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

SF_DEVICE void fence_mbarrier_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

SF_DEVICE void mbar_arrive(uint64_t *bar)
{
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}"
                 ::"r"(smem_u32(bar)) : "memory");
}

SF_DEVICE void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}"
                 ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

SF_DEVICE bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
    return ok != 0;
}

// Bounded wait for phase `parity` of `bar`. Returns false on timeout or when *abort is raised
// by another warp of the block (the caller then unwinds).
SF_DEVICE bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            *abort = 1;
            return false;
        }
    }
}

// Read-only 2-byte load that bypasses L1 and asks L2 to fetch 64 bytes around p from DRAM (the
// L2::64B prefetch-size qualifier) instead of the 128-byte line plain loads bring in: for
// scattered single elements this halves the DRAM bytes moved per element.
SF_DEVICE uint16_t ld_nc_l2_64b_u16(const uint16_t *p)
{
    uint16_t v;
    asm volatile("ld.global.nc.L1::no_allocate.L2::64B.b16 %0, [%1];" : "=h"(v) : "l"(p));
    return v;
}

// Ask L2 to fetch the line holding p (no register result; the load that follows hits L2).
SF_DEVICE void prefetch_l2(const void *p) { asm volatile("prefetch.global.L2 [%0];" ::"l"(p)); }

// Element-wise max of eight bf16 values into p[0..7] (16-byte aligned), one reduction for all.
// The row magnitudes reduced this way are non-negative and finite, so bf16 order is the order of
// the bit patterns.
SF_DEVICE void red_max_bf16x8(uint16_t *p, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("red.global.v4.bf16x2.max.noftz [%0], {%1, %2, %3, %4};" ::"l"(p), "r"(a), "r"(b), "r"(c),
                 "r"(d) : "memory");
}

// The same for two bf16 values into p[0..1] (4-byte aligned).
SF_DEVICE void red_max_bf16x2(uint16_t *p, uint16_t a, uint16_t b)
{
    asm volatile("red.global.v2.bf16.max.noftz [%0], {%1, %2};" ::"l"(p), "h"(a), "h"(b) : "memory");
}

SF_DEVICE void prefetch_tmap(const CUtensorMap *m)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 2-D tiled TMA load of box {x, y} (x innermost, in elements) into shared memory, completing
// transaction bytes on `bar`. No multicast.
SF_DEVICE void tma_load_2d(void *dst, const CUtensorMap *m, uint64_t *bar, int x, int y)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y),
          "r"(smem_u32(bar))
        : "memory");
}

// 2-D tiled TMA load by either CTA of a pair into its own shared memory, completing its bytes on
// the mbarrier at `bar`'s offset in the even CTA (the one whose thread issues the pair's MMAs).
// No multicast.
SF_DEVICE void tma_load_2d_pair(void *dst, const CUtensorMap *m, uint64_t *bar, int x, int y)
{
    asm volatile(
        "{\n\t.reg .b32 rb;\n\t"
        "mapa.shared::cluster.u32 rb, %2, 0;\n\t"
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4}], [rb];\n\t}"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// 3-D tiled TMA load of box {x, y, z} into shared memory (box element order x fastest, then y,
// then z), completing transaction bytes on `bar`. No multicast.
SF_DEVICE void tma_load_3d(void *dst, const CUtensorMap *m, uint64_t *bar, int x, int y, int z)
{
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3, %4}], [%5];"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(m)), "r"(x), "r"(y), "r"(z),
          "r"(smem_u32(bar))
        : "memory");
}

// The CTA-pair form of tma_load_3d (completing on the even CTA's barrier). No multicast.
SF_DEVICE void tma_load_3d_pair(void *dst, const CUtensorMap *m, uint64_t *bar, int x, int y, int z)
{
    asm volatile(
        "{\n\t.reg .b32 rb;\n\t"
        "mapa.shared::cluster.u32 rb, %2, 0;\n\t"
        "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5}], [rb];\n\t}"
        ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(x), "r"(y), "r"(z)
        : "memory");
}

SF_DEVICE void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
SF_DEVICE void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// TMEM allocation: one warp, `ncols` a power of two >= 32. The address lands in *dst (smem).
SF_DEVICE void tmem_alloc(uint32_t *dst, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(dst)), "r"(ncols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

SF_DEVICE void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// D[tmem] (+)= A[smem] * B[smem], kind::f16 (bf16 inputs, fp32 accumulate), one thread.
SF_DEVICE void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                        uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on `bar` once every tcgen05 operation this thread issued so far has completed.
SF_DEVICE void mma_commit(uint64_t *bar)
{
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
        ::"r"(smem_u32(bar)) : "memory");
}

// 32 lanes x 32 columns of 32-bit accumulator: lane i of the warp gets row (lane base + i),
// columns col .. col+31.
SF_DEVICE void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}

SF_DEVICE void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// --------------------------------------------------------------------------------------------
// CTA pairs (a cluster of two CTAs sharing one tcgen05.mma with cta_group::2).
// --------------------------------------------------------------------------------------------

SF_DEVICE uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Arrive on the mbarrier at the same shared-memory offset in CTA `rank` of the cluster.
SF_DEVICE void mbar_arrive_remote(uint64_t *bar, uint32_t rank)
{
    asm volatile("{\n\t.reg .b32 ra;\n\t"
                 "mapa.shared::cluster.u32 ra, %0, %1;\n\t"
                 "mbarrier.arrive.release.cluster.shared::cluster.b64 _, [ra];\n\t}"
                 ::"r"(smem_u32(bar)), "r"(rank) : "memory");
}

// Every thread of every CTA of the cluster arrives, then waits for all of them.
SF_DEVICE void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// TMEM allocation for a CTA pair: issued by the same warp of both CTAs, same destination offset.
SF_DEVICE void tmem_alloc_pair(uint32_t *dst, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(dst)), "r"(ncols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

SF_DEVICE void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// D[tmem] (+)= A * B over the CTA pair (M = 256: 128 rows of A and N/2 columns of B in each
// CTA's shared memory, at the same offsets), issued by one thread of the even CTA.
SF_DEVICE void mma_bf16_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                             uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on the mbarrier at `bar`'s offset in every CTA of `mask` once the pair's tcgen05
// operations issued so far by this thread have completed.
SF_DEVICE void mma_commit_pair(uint64_t *bar, uint16_t mask)
{
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
        ::"r"(smem_u32(bar)), "h"(mask) : "memory");
}

}  // namespace sf
