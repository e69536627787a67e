// fp8fg_device.cuh -- device-side building blocks of libfp8fg (sm_100a only).
//
// Inline-PTX wrappers for the Blackwell pieces the kernels are built from:
// mbarriers, TMA tensor loads for CTA pairs (no cluster multicast
// anywhere), tcgen05 MMA / TMEM allocation / TMEM loads, packed FP32x2 FMA,
// and the library's status word.  Every wait on an mbarrier is bounded: after a time limit it records
// FP8_ERR_TIMEOUT in the status word and reports failure to the caller, who
// then unwinds (drains its own in-flight copies, frees TMEM, returns).
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/fp8fg.h"

namespace fp8fg {

// Status word of this kernel module.  Device code is compiled per source
// file, so every source file that includes this header gets its own word
// (internal linkage, module scope, never allocated); each such file exports
// a reader, and fp8_get_status reads and clears them all.
namespace {
__device__ int g_module_status = 0;

// Record `code` in this module's status word (first error wins).
__device__ __forceinline__ void report_error(int code) { atomicCAS(&g_module_status, 0, code); }

// Host: return and clear this module's status word (caller synchronised).
inline int read_and_clear_module_status()
{
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_module_status, sizeof(int)) != cudaSuccess) return FP8_ERR_DEVICE;
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_module_status, &zero, sizeof(int)) != cudaSuccess) return FP8_ERR_DEVICE;
    return v;
}
}  // namespace

__device__ __forceinline__ uint32_t smem_u32(const void* p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------- mbarrier

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Same test, but a thread whose phase is not complete is suspended in hardware
// (for at most `hint_ns`) until it completes, instead of returning at once:
// a waiting warp then leaves its scheduler's issue slots to the other warps.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t hint_ns)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

constexpr uint32_t kWaitSleepNs = 20000;   // per suspended try_wait (bounded loop below)

// Wait until the phase of `bar` with parity `parity` has completed.
// Gives up (returns false) when *abort is set by another role of the CTA or
// when `timeout_ns` has passed; in the latter case it records
// FP8_ERR_TIMEOUT and sets *abort so the other roles unwind too.  The
// iteration count is capped as well, independently of the clock.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          uint64_t timeout_ns)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1; it < (1u << 30); ++it) {
        if (mbar_try_wait_sleep(bar, parity, kWaitSleepNs)) return true;
        if (*abort) return false;
        if ((it & 7) == 0 && globaltimer_ns() - t0 > timeout_ns) break;
    }
    report_error(FP8_ERR_TIMEOUT);
    *abort = 1;
    return false;
}

// Non-blocking test of a phase (mbarrier.test_wait never suspends).
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}\n"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// mbar_wait for a thread whose latency matters more than its issue slots
// (an MMA issuer): spins on mbarrier.test_wait, with the same time limit,
// abort flag and error report as mbar_wait.
__device__ __forceinline__ bool mbar_wait_spin(uint64_t* bar, uint32_t parity, volatile int* abort,
                                               uint64_t timeout_ns)
{
    if (mbar_test(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1; it < (1u << 30); ++it) {
        if (mbar_test(bar, parity)) return true;
        if ((it & 63) == 0) {
            if (*abort) return false;
            if (globaltimer_ns() - t0 > timeout_ns) break;
        }
    }
    report_error(FP8_ERR_TIMEOUT);
    *abort = 1;
    return false;
}

// Bounded wait used while unwinding: ignores the abort flag (the awaited
// operation is already in flight and must land before the CTA exits).
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity, uint64_t timeout_ns)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    for (uint32_t it = 1; it < (1u << 30); ++it) {
        if (mbar_try_wait_sleep(bar, parity, kWaitSleepNs)) return true;
        if ((it & 7) == 0 && globaltimer_ns() - t0 > timeout_ns) break;
    }
    report_error(FP8_ERR_TIMEOUT);
    return false;
}

// ---------------------------------------------------------------- TMA

__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map)
{
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled tensor store shared -> global of the box at (x, y), tracked by
// this thread's bulk async-group (x innermost, in elements; the parts of the
// box outside the tensor are not written).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* smem_src, int32_t x,
                                             int32_t y)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
                     reinterpret_cast<uint64_t>(map)),
                 "r"(x), "r"(y), "r"(smem_u32(smem_src))
                 : "memory");
}

// The same box added element-wise into global memory (the tensor map's type
// must be one the TMA adds, e.g. FP32).
__device__ __forceinline__ void tma_reduce_add_2d(const CUtensorMap* map, const void* smem_src,
                                                  int32_t x, int32_t y)
{
    asm volatile(
        "cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
            reinterpret_cast<uint64_t>(map)),
        "r"(x), "r"(y), "r"(smem_u32(smem_src))
        : "memory");
}

__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }

// Wait until at most N of this thread's bulk groups still read shared memory.
template <int N>
__device__ __forceinline__ void bulk_wait_group_read()
{
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

// Wait until every bulk group of this thread has completed (writes done).
__device__ __forceinline__ void bulk_wait_group_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (TMA stores, tcgen05 reads) before another thread starts one.
__device__ __forceinline__ void fence_proxy_async_shared()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- tcgen05

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// ---------------------------------------------------------------- CTA pairs
// (2-CTA clusters: one tcgen05.mma.cta_group::2 spans the tensor cores of
// both SMs; each CTA holds half of A's rows and half of B's columns.)

__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Address, in the cluster's shared window, of the variable at shared::cta
// address `saddr` in the CTA of rank `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t saddr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}

// Arrive on an mbarrier given by its cluster-window address (either CTA of
// the pair).  Default semantics (release at CTA scope): an explicit
// .release.cluster arrive measured ~1000+ cycles per arrive here, which
// serialises a K-block pipeline.
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr)
{
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}

__device__ __forceinline__ void cluster_sync()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                     : "memory");
}

// TMA 2-D load into this CTA's shared memory whose completion (bytes) is
// counted on an mbarrier of either CTA of the pair (cluster-window address).
// No cluster multicast.
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map,
                                                 uint32_t bar_cluster_addr, int32_t x, int32_t y)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar_cluster_addr)
        : "memory");
}

// TMA 2-D gather of four whole rows (row indices r0..r3, columns from x on,
// one box of the tensor map per row; the map's box is one row high) into
// consecutive rows of this CTA's shared memory, with the same 128-byte
// swizzle a tiled load of those rows would give.  Bytes count on an mbarrier
// of either CTA of the pair.  No cluster multicast.
__device__ __forceinline__ void tma_gather4_pair(void* smem_dst, const CUtensorMap* map,
                                                 uint32_t bar_cluster_addr, int32_t x, int32_t r0,
                                                 int32_t r1, int32_t r2, int32_t r3)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile::gather4.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6, %7}], [%2];" ::"r"(smem_u32(smem_dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster_addr), "r"(x), "r"(r0), "r"(r1), "r"(r2),
        "r"(r3)
        : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* smem_dst, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(smem_dst)),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish_pair()
{
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

// D[tmem of both CTAs] (+)= A x B over the pair (M = 256: rows 0-127 in the
// issuing (even) CTA, 128-255 in its peer), issued by the even CTA only.
__device__ __forceinline__ void mma_f8f6f4_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                                uint32_t idesc, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive (once) on the mbarrier at this offset in every CTA of `cta_mask`
// when the pair's tcgen05 ops issued by this thread have completed.
__device__ __forceinline__ void mma_commit_pair(uint64_t* bar, uint16_t cta_mask)
{
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
        " [%0], %1;" ::"r"(smem_u32(bar)),
        "h"(cta_mask)
        : "memory");
}

// 32 consecutive FP32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32"
        " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15,"
        " %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31},"
        " [%32];\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr));
}

// 16 consecutive FP32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32"
        " {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15},"
        " [%16];\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}

// Wait for this thread's outstanding TMEM loads.  The registers of the load
// are in/out operands, so code that reads them cannot be scheduled above the
// wait.
__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[16])
{
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                   "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                   "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15])
                 :
                 : "memory");
}

__device__ __forceinline__ void tmem_ld_wait(uint32_t (&r)[32])
{
    asm volatile("tcgen05.wait::ld.sync.aligned;"
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                   "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                   "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                   "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                   "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                   "+r"(r[30]), "+r"(r[31])
                 :
                 : "memory");
}

// Shared-memory matrix descriptor for a 128-byte-swizzled operand tile.
//   K-major : rows of 128 bytes along K, 8-row atoms 1024 B apart (SBO);
//             LBO unused (1).
//   MN-major: 128-byte runs along M/N; LBO = bytes between 128-element MN
//             atoms, SBO = bytes between groups of 8 K-rows.
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr, uint32_t lbo_bytes,
                                                    uint32_t sbo_bytes)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;            // descriptor version (sm_100)
    d |= (uint64_t)2 << 61;            // layout: 128-byte swizzle
    return d;
}

// Instruction descriptor: E4M3 x E4M3 -> FP32, dense, M x N, A K-major.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(uint32_t M, uint32_t N, uint32_t b_mn_major)
{
    return (1u << 4)                 // D format: FP32
           | (0u << 7)               // A format: E4M3
           | (0u << 10)              // B format: E4M3
           | (0u << 15)              // A K-major
           | (b_mn_major << 16)      // B major
           | ((N >> 3) << 17)        // N / 8
           | ((M >> 4) << 24);       // M / 16
}

// ---------------------------------------------------------------- GEMM tiles

// Persistent-GEMM tile order: bands of `band` m-blocks; inside a band n-blocks
// outer, m-blocks inner, so the tiles resident at once share a few A
// row-blocks and B column-blocks in L2.
__device__ __forceinline__ void gemm_tile_coord(int64_t tile, int64_t nmb, int64_t nnb, int band,
                                                int64_t& mb, int64_t& nb)
{
    const int64_t band_tiles = (int64_t)band * nnb;
    const int64_t bi = tile / band_tiles;
    const int64_t r = tile - bi * band_tiles;
    const int64_t mb0 = bi * band;
    const int64_t rows = (nmb - mb0 < band) ? (nmb - mb0) : band;
    nb = r / rows;
    mb = mb0 + r % rows;
}

// Group holding block index `row0` of a non-decreasing offset table: the
// largest e with off[e] <= row0; -1 when row0 >= off[G].
__device__ __forceinline__ int find_group(const int32_t* off, int G, int64_t row0)
{
    int lo = 0, hi = G;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if ((int64_t)off[mid] <= row0)
            lo = mid;
        else
            hi = mid - 1;
    }
    return lo < G ? lo : -1;
}

// The 128 rows of A (and of D) one CTA of a pair works on in m-block mb.
//   dense    m0 = mb * 256 + rank * 128, rows below M valid.
//   grouped  mb counts 256-row blocks group by group (poff), so a pair never
//            mixes two groups' rows (it shares one B); in a group whose row
//            count is an odd multiple of 128 the last pair's odd CTA lies
//            past the group end and idles.  Blocks at or past poff[G] hold
//            no group (false).
struct TileRows {
    int g;           // group (0 when dense)
    int64_t m0;      // first row of this CTA's 128
    int64_t m_end;   // rows m0 .. m_end-1 belong to the tile's group
};

__device__ __forceinline__ bool tile_rows(const int32_t* group_offsets, const int32_t* off,
                                          const int32_t* poff, int G, int64_t M, int64_t mb,
                                          uint32_t rank, TileRows& t)
{
    if (!group_offsets) {
        t.g = 0;
        t.m0 = mb * 256 + rank * 128;
        t.m_end = M;
        return true;
    }
    const int g = find_group(poff, G, mb);
    if (g < 0) return false;
    t.g = g;
    t.m0 = off[g] + (mb - poff[g]) * 256 + rank * 128;
    t.m_end = off[g + 1];
    return true;
}

// One warp: poff[e] = number of 256-row blocks in groups 0 .. e-1 (row
// counts off[e+1] - off[e]), poff[G] their total.  Each lane sums a run of
// groups; a warp scan turns the sums into the runs' first blocks.
__device__ __forceinline__ void pair_block_offsets(const int32_t* off, int32_t* poff, int G, int lane)
{
    const int per = (G + 31) / 32;
    const int e0 = lane * per < G ? lane * per : G;
    const int e1 = e0 + per < G ? e0 + per : G;
    int sum = 0;
    for (int e = e0; e < e1; ++e) sum += (off[e + 1] - off[e] + 255) >> 8;
    int incl = sum;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d) incl += t;
    }
    int run = incl - sum;
    for (int e = e0; e < e1; ++e) {
        poff[e] = run;
        run += (off[e + 1] - off[e] + 255) >> 8;
    }
    if (lane == 31) poff[G] = incl;
}

// Host: 2-D uint8 tensor map [outer][inner], rows `row_bytes` apart, boxes of
// box_inner x box_outer bytes, 128-byte swizzle (or none, with swizzle128 =
// false), zero fill out of bounds (defined in gemm.cu; false when the
// driver's encoder is unavailable).
bool make_map(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, bool swizzle128 = true);

// Host: 2-D tensor map of `dtype` elements [outer][inner] (inner in
// elements), rows `row_bytes` apart, boxes of box_inner x box_outer elements,
// no swizzle (defined in gemm.cu).
bool make_map_typed(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner,
                    uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer);

// ---------------------------------------------------------------- registers

// Warpgroup-wide register budget changes (all 128 threads of a warpgroup
// execute the same one).  The increases a kernel makes must fit in what its
// decreases free from the block's launch allocation.
template <uint32_t N>
__device__ __forceinline__ void regs_dec()
{
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
__device__ __forceinline__ void regs_inc()
{
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}

// ---------------------------------------------------------------- FP32x2

// acc += p * s on two lanes at once (one packed FMA instruction on sm_100).
__device__ __forceinline__ void ffma2(float& acc0, float& acc1, float p0, float p1, float s0,
                                      float s1)
{
    uint64_t a, p, s;
    asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(acc0), "f"(acc1));
    asm("mov.b64 %0, {%1, %2};" : "=l"(p) : "f"(p0), "f"(p1));
    asm("mov.b64 %0, {%1, %2};" : "=l"(s) : "f"(s0), "f"(s1));
    asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(a) : "l"(p), "l"(s));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(acc0), "=f"(acc1) : "l"(a));
}

__device__ __forceinline__ void fmul2(float& d0, float& d1, float a0, float a1, float b0, float b1)
{
    uint64_t a, b, d;
    asm("mov.b64 %0, {%1, %2};" : "=l"(a) : "f"(a0), "f"(a1));
    asm("mov.b64 %0, {%1, %2};" : "=l"(b) : "f"(b0), "f"(b1));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(d0), "=f"(d1) : "l"(d));
}

}  // namespace fp8fg
