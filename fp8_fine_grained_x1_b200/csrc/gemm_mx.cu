// gemm_mx.cu -- block-scaled E4M3 x E4M3 GEMM for power-of-two scales, with
// the scaling done by the tensor cores (sm_100a:
// tcgen05.mma.kind::mxf8f6f4.block_scale, UE8M0 scale factors in TMEM).
//
// What it computes is the same sum as gemm.cu -- D = sum over 128-element
// K-blocks of scale_a * scale_b * (A_kb . B_kb) -- restricted to scales that
// are integral powers of two ("5 Ways You can get More Deepseek While
// Spending Less": power-of-2 scaling factors for some activations; the
// gnrental.net post: the authors ask for Tensor Cores that take group scales
// themselves and accumulate at higher precision, so partials need not leave
// them).  A power of two is exactly a UE8M0 scale factor, so the multiply by
// scale_a * scale_b happens inside the MMA: each tcgen05.mma of K = 32 reads
// one scale per row of A and one per column of B from TMEM and accumulates
// the scaled products into the FP32 accumulator.  No partial leaves the
// tensor core until the tile's last K-block: there is no promotion step.
//
// Roles per CTA (persistent, one CTA per SM, 512 threads):
//   warp 0      TMA producer: A / B tiles per K-block into a shared-memory
//               ring (128-byte swizzle, no cluster multicast)
//   warp 1      MMA issuer: 4 x block-scaled MMA (K = 32) per K-block into
//               one TMEM accumulator, tcgen05.commit frees the stage
//   warp 2      TMEM allocator
//   warps 4-7   scale writers: per K-block, read the FP32 scales, take
//               their biased exponents (UE8M0) and store them into the
//               stage's scale-factor area of shared memory; the MMA thread
//               copies them to TMEM (tcgen05.cp) in order with its MMAs
//   warps 8-15  epilogue: tcgen05.ld the accumulator (two warps per lane
//               quarter, 128 columns each), release it, convert and store
// TMEM (512 columns): accumulator 0-255; per stage s a 16-column slot at
// 256 + 16 s: SFA in its first 4 columns, SFB in columns 8-15.
// Scale-factor layout (the tensor core's for M = 128, one scale per 32 K):
// column c of the SFA slot holds, in lane 32 q + l, the scale of row
// 32 c + l; column c of the SFB slot the scale of column 32 c + l; every
// lane quarter q holds the same copy.  All four bytes of a column word are
// the same scale, because one 128-element group covers all four K = 32
// steps of a K-block, so whichever byte an MMA selects is the right one.
// In shared memory each 128 rows (or columns) form one 512-byte block of 32
// lines of 16 bytes: line l = the words of rows l, l + 32, l + 64, l + 96.
// tcgen05.cp .32x128b.warpx4 moves line l to TMEM lane l of every quarter,
// four columns wide -- exactly the layout above.  (Writing TMEM with
// tcgen05.st from the scale warps instead measured 24 % tensor-pipe
// activity: the stores and the MMAs contend for TMEM.)
//
// CTA pairs (2-CTA clusters), as in gemm.cu: the even CTA issues one
// tcgen05.mma.cta_group::2 of 256 x 256 x 32 over both SMs; each CTA loads
// its own 128 rows of A and 128 of B's columns.  Each SM multiplies its own
// 128 rows by all 256 columns, so each CTA's TMEM holds the scale factors
// of its own rows (SFA) and of all 256 columns (SFB): the scale writers of
// both CTAs fill their own shared memory, and the even CTA's
// tcgen05.cp.cta_group::2 moves each CTA's block into that CTA's TMEM.
// Both CTAs' loads and scale writers count on the even CTA's `full`
// barrier; its commits arrive on both CTAs' `empty` and `acc_full`.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "fp8fg_device.cuh"
#include "fp8fg_host.h"

namespace fp8fg {

namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;
constexpr uint32_t A_BYTES = BM * BK;
constexpr int NUM_THREADS = 512;
constexpr int FIRST_SF_WARP = 4;
constexpr int FIRST_EPI_WARP = 8;
constexpr int NUM_SF_WARPS = 4;
constexpr int NUM_EPI_WARPS = 8;
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t SF_COL0 = BN;
constexpr uint32_t SF_SLOT_COLS = 16;
constexpr uint32_t SFB_OFF = 8;
// Raster bands (m-blocks per band): 16 for dense GEMMs; 8 for grouped ones,
// whose bands otherwise span several experts' rows and weights at once.
constexpr int BAND_DENSE = 16;
constexpr int BAND_GROUPED = 8;
constexpr int SF_AHEAD = 4;                 // K-blocks of scales each writer loads ahead
constexpr uint32_t SFA_BYTES = 512;              // 128 rows x 4 bytes
constexpr uint32_t SFB_BYTES = 1024;             // 256 columns x 4 bytes
constexpr uint32_t SF_BYTES = SFA_BYTES + SFB_BYTES;
constexpr int NS = 6;                       // ring stages
constexpr int TILE_M = 256;                 // rows per pair tile
constexpr uint32_t B_BYTES = 128 * BK;      // this CTA's 128 of B's columns
constexpr uint32_t RING_BYTES = NS * (A_BYTES + B_BYTES + SF_BYTES);   // 201 KB
static_assert(SF_COL0 + NS * SF_SLOT_COLS <= TMEM_COLS, "scale slots exceed the allocation");
constexpr uint32_t DYN_SMEM = 1024 + RING_BYTES;

constexpr int MAX_GROUPS = 1024;

struct MxParams {
    const float* sA;     // [K/128][M]
    const float* sB;     // as for fp8_blockscaled_gemm / fp8_grouped_gemm
    void* D;
    const int32_t* group_offsets;   // nullptr: dense
    int64_t M, N, K, ldd;
    int G;
    int b_major, sb_gran, out_dtype;
    int withhold;        // self-test: the odd CTA stops loading after one K-block
    int band;            // m-blocks per raster band
    uint64_t timeout_ns;
};

struct __align__(8) MxShared {
    uint64_t full[NS];         // operands landed (TMA bytes) and scales stored (scale warps)
    uint64_t empty[NS];
    uint64_t acc_full;
    uint64_t acc_empty;
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int bad;
    int32_t off[MAX_GROUPS + 1];   // grouped: the group offsets, validated on the device
    int32_t poff[MAX_GROUPS + 1];  // grouped pairs: first 256-row block of each group
};

// -------------------------------------------------------------- PTX helpers

// Block-scaled MMA over a CTA pair: D[tmem] (+)= (A * SFA) x (B * SFB),
// E4M3 operands from shared memory, UE8M0 scale factors from TMEM (M = 256:
// rows 0-127 in the even CTA, which issues it; each CTA's scale factors from
// its own TMEM).
__device__ __forceinline__ void mma_mxf8_pair(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                              uint32_t idesc, uint32_t sfa_tmem, uint32_t sfb_tmem,
                                              uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}\n" ::
            "r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(sfa_tmem), "r"(sfb_tmem)
        : "memory");
}

// Instruction descriptor of the block-scaled kind: E4M3 x E4M3, UE8M0 scale
// factors (bit 23), scale-factor ids 0, K = 32, A K-major; FP32 accumulator.
__host__ __device__ constexpr uint32_t idesc_mx_e4m3(uint32_t M, uint32_t N, uint32_t b_mn_major)
{
    return (0u << 7)                 // A format: E4M3
           | (0u << 10)              // B format: E4M3
           | (b_mn_major << 16)      // B major
           | ((N >> 3) << 17)        // N / 8
           | (1u << 23)              // scale factors: UE8M0
           | ((M >> 4) << 24);       // M / 16
}

// Copy 32 lines of 16 bytes (a 512-byte block at `saddr`, no swizzle) from
// shared memory to TMEM, for both CTAs of a pair (issued by the even CTA:
// each CTA's block goes to that CTA's TMEM at `taddr`): line l -> lane l of
// every lane quarter, four 32-bit columns from `taddr`.  Executes in order
// with the tcgen05.mma instructions issued after it.
__device__ __forceinline__ void tmem_cp_32x128b_x4_pair(uint32_t taddr, uint32_t saddr)
{
    const uint64_t desc = (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)(16 >> 4) << 16) |
                          ((uint64_t)(128 >> 4) << 32) | ((uint64_t)1 << 46);
    asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(desc)
                 : "memory");
}

// Make this thread's shared-memory stores visible to the async proxy (TMA,
// tcgen05.cp, tcgen05.mma operand reads).
__device__ __forceinline__ void fence_proxy_async_smem()
{
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// UE8M0 code of a scale 2^e (-126 <= e <= 127): its biased exponent, copied
// into all four bytes.  Anything that is not a positive normal power of two
// sets `bad` and is replaced by 2^0.
__device__ __forceinline__ uint32_t ue8m0_x4(float s, bool& bad)
{
    const uint32_t b = __float_as_uint(s);
    const uint32_t e = b >> 23;                       // sign bit included: negative -> > 255
    const bool ok = (b & 0x007FFFFFu) == 0u && e >= 1u && e <= 254u;
    bad = bad || !ok;
    return (ok ? e : 127u) * 0x01010101u;
}

__device__ __forceinline__ uint32_t pack_bf16x2_rn(float lo, float hi)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// One lane waits (bounded); the whole warp learns the outcome, so the warp's
// .sync.aligned tcgen05 instructions are never reached by part of it.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          uint64_t timeout_ns, int lane)
{
    int ok = 1;
    if (lane == 0) ok = mbar_wait(bar, parity, abort, timeout_ns) ? 1 : 0;
    return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// ------------------------------------------------------------------ roles

__device__ __forceinline__ bool mx_tile_rows(const MxParams& p, const MxShared& sh, int64_t mb,
                                             uint32_t rank, TileRows& t)
{
    return tile_rows(p.group_offsets, sh.off, sh.poff, p.G, p.M, mb, rank, t);
}

// Tiles are dealt round-robin to pairs: pair c is CTAs 2c, 2c+1.
__device__ __forceinline__ void mx_unit_range(int64_t& first, int64_t& stride)
{
    first = (int64_t)(blockIdx.x >> 1);
    stride = (int64_t)(gridDim.x >> 1);
}

__device__ void mx_producer(const CUtensorMap* tmA, const CUtensorMap* tmB, const MxParams& p,
                            uint8_t* smem, MxShared& sh, int64_t nmb, int64_t nnb, int64_t nkb)
{
    volatile int* abort = &sh.abort;
    const uint32_t rank = cluster_ctarank();
    int64_t it = 0;
    bool ok = true;
    int64_t first, stride;
    mx_unit_range(first, stride);
    for (int64_t tile = first; ok && tile < nmb * nnb; tile += stride) {
        int64_t mb, nb;
        gemm_tile_coord(tile, nmb, nnb, p.band, mb, nb);
        TileRows tr;
        if (!mx_tile_rows(p, sh, mb, rank, tr)) continue;
        const int64_t m0 = tr.m0, n0 = nb * BN;   // an idle odd CTA still loads
        const int32_t brow = (int32_t)((int64_t)tr.g * p.N + n0 + rank * 128);
        for (int64_t kb = 0; kb < nkb; ++kb) {
            if (p.withhold && rank == 1 && it == 1) {   // self-test only
                ok = false;
                break;
            }
            const int s = (int)(it % NS);
            const uint32_t ph = (uint32_t)((it / NS) & 1);
            if (!mbar_wait(&sh.empty[s], ph ^ 1u, abort, p.timeout_ns)) {
                ok = false;
                break;
            }
            ++it;
            uint8_t* a_dst = smem + s * A_BYTES;
            uint8_t* b_dst = smem + NS * A_BYTES + s * B_BYTES;
            // both CTAs' bytes count on the even CTA's barrier
            const uint32_t bar = mapa_shared(smem_u32(&sh.full[s]), 0);
            if (rank == 0) mbar_arrive_expect_tx(&sh.full[s], 2 * (A_BYTES + B_BYTES));
            tma_load_2d_pair(a_dst, tmA, bar, (int32_t)(kb * BK), (int32_t)m0);
            if (p.b_major == FP8_B_KMAJOR)
                tma_load_2d_pair(b_dst, tmB, bar, (int32_t)(kb * BK), brow);
            else
                tma_load_2d_pair(b_dst, tmB, bar, (int32_t)(n0 + rank * 128), (int32_t)(kb * BK));
        }
    }
    // every copy issued lands before the CTA exits (a pair's all count on the
    // even CTA's barriers; the odd CTA stays until the closing cluster barrier)
    if (rank != 0) return;
#pragma unroll
    for (int s = 0; s < NS; ++s) {
        const int64_t count = it > s ? (it - s + NS - 1) / NS : 0;
        if (count) mbar_wait_drain(&sh.full[s], (uint32_t)((count - 1) & 1), p.timeout_ns);
    }
}

// The tensor core takes a new MMA only about when the previous one ends, so
// the issuing thread runs at most one MMA ahead, and every cycle it spends on
// anything else while the last queued MMA drains leaves the tensor core
// idle.  The loop therefore waits for the next stage before issuing the
// current stage's last MMA, so the barrier latency hides behind the MMAs
// still executing, and it spins rather than suspends on barriers.
__device__ void mx_mma(const MxParams& p, uint8_t* smem, MxShared& sh, int64_t nmb, int64_t nnb,
                       int64_t nkb)
{
    volatile int* abort = &sh.abort;
    const uint32_t a_base = smem_u32(smem);
    const uint32_t b_base = a_base + NS * A_BYTES;
    const uint32_t sf_base = b_base + NS * B_BYTES;
    const uint32_t tmem = sh.tmem_base;
    const int64_t ntiles = nmb * nnb;
    uint32_t it = 0;          // K-blocks consumed so far (stage it % NS, round it / NS)
    uint32_t tcount = 0;
    bool ok = true;
    int64_t first, stride;
    mx_unit_range(first, stride);
    for (int64_t tile = first; ok && tile < ntiles; tile += stride) {
        int64_t mb, nb;
        gemm_tile_coord(tile, nmb, nnb, p.band, mb, nb);
        const int64_t n0 = nb * BN;
        (void)n0;
        // a pair's MMA always spans 256 columns (a B tail is zero-filled)
        const uint32_t idesc = idesc_mx_e4m3((uint32_t)TILE_M, (uint32_t)BN, (uint32_t)p.b_major);
        // the epilogue has read the previous tile's accumulator
        ok = mbar_wait_spin(&sh.acc_empty, (tcount & 1u) ^ 1u, abort, p.timeout_ns) &&
             mbar_wait_spin(&sh.full[it % NS], (it / NS) & 1u, abort, p.timeout_ns);
        if (!ok) break;
        for (int64_t kb = 0; kb < nkb; ++kb, ++it) {
            const uint32_t s = it % NS;
            tc_fence_after();
            const uint32_t a_addr = a_base + s * A_BYTES;
            const uint32_t b_addr = b_base + s * B_BYTES;
            const uint32_t sf_addr = sf_base + s * SF_BYTES;
            const uint32_t sfa = tmem + SF_COL0 + s * SF_SLOT_COLS;
            tmem_cp_32x128b_x4_pair(sfa, sf_addr);                            // SFA, rows 0-127
            tmem_cp_32x128b_x4_pair(sfa + SFB_OFF, sf_addr + SFA_BYTES);      // SFB, columns 0-127
            tmem_cp_32x128b_x4_pair(sfa + SFB_OFF + 4, sf_addr + SFA_BYTES + 512);   // 128-255
#pragma unroll
            for (int k = 0; k < BK / 32; ++k) {
                if (k == BK / 32 - 1 && kb + 1 < nkb) {
                    // next stage of this tile: wait while this stage's MMAs run
                    const uint32_t nx = it + 1;
                    if (!mbar_wait_spin(&sh.full[nx % NS], (nx / NS) & 1u, abort, p.timeout_ns)) {
                        ok = false;
                        break;
                    }
                }
                const uint64_t adesc = smem_desc_sw128(a_addr + k * 32, 16, 1024);
                const uint64_t bdesc = (p.b_major == FP8_B_KMAJOR)
                                           ? smem_desc_sw128(b_addr + k * 32, 16, 1024)
                                           : smem_desc_sw128(b_addr + k * 32 * 128, 128 * BK, 1024);
                const uint32_t acc = (kb | k) ? 1u : 0u;
                mma_mxf8_pair(tmem, adesc, bdesc, idesc, sfa, sfa + SFB_OFF, acc);
            }
            // stage and scale slot free once these are done (in both CTAs)
            mma_commit_pair(&sh.empty[s], 3);
            if (!ok) break;
        }
        if (!ok) break;
        // the tile's sum is complete
        mma_commit_pair(&sh.acc_full, 3);
        ++tcount;
    }
    mma_commit_pair(&sh.drain, 1);
    mbar_wait_drain(&sh.drain, 0, p.timeout_ns);
}

// Scales of K-block kb handled by scale-writer thread t (0..127): row t of
// the CTA's A block and columns t, t + 128 of the tile's B block; 1 outside
// the matrix or the tile's group.
struct SfRegs {
    float a;
    float b[2];
};

__device__ __forceinline__ void load_sf(const MxParams& p, int g, int64_t m0, int64_t m_end,
                                        int64_t n0, int64_t kb, int64_t nkb, int t, SfRegs& r)
{
    const int64_t m = m0 + t;
    r.a = m < m_end ? __ldg(p.sA + kb * p.M + m) : 1.0f;
    const int64_t nnb128 = p.N / 128;
#pragma unroll
    for (int j = 0; j < 2; ++j) {
        const int64_t n = n0 + t + 128 * j;
        float v = 1.0f;
        if (n < p.N) {
            if (p.sb_gran == 1)
                v = __ldg(p.sB + kb * p.N + n);
            else if (p.b_major == FP8_B_KMAJOR)   // grouped: sB [G][N/128][K/128]
                v = __ldg(p.sB + ((int64_t)g * nnb128 + n / 128) * nkb + kb);
            else
                v = __ldg(p.sB + kb * nnb128 + n / 128);
        }
        r.b[j] = v;
    }
}

// Byte offset of row (or column) i of a 128-row block in its 512-byte block:
// line i % 32, word i / 32.
__device__ __forceinline__ uint32_t sf_offset(int i) { return 16u * (uint32_t)(i & 31) + 4u * (uint32_t)(i >> 5); }

__device__ void mx_scale_writer(const MxParams& p, uint8_t* smem, MxShared& sh, int64_t nmb,
                                int64_t nnb, int64_t nkb, int warp, int lane)
{
    volatile int* abort = &sh.abort;
    const uint32_t rank = cluster_ctarank();
    const int t = (warp - FIRST_SF_WARP) * 32 + lane;          // 0..127
    uint8_t* sf_base = smem + NS * (A_BYTES + B_BYTES);
    const uint32_t off_a = sf_offset(t);
    const uint32_t off_b0 = SFA_BYTES + sf_offset(t);
    const uint32_t off_b1 = SFA_BYTES + 512 + sf_offset(t);
    int64_t it = 0;
    bool ok = true, bad = false;
    int64_t first, stride;
    mx_unit_range(first, stride);
    for (int64_t tile = first; ok && tile < nmb * nnb; tile += stride) {
        int64_t mb, nb;
        gemm_tile_coord(tile, nmb, nnb, p.band, mb, nb);
        TileRows tr;
        if (!mx_tile_rows(p, sh, mb, rank, tr)) continue;
        const int64_t n0 = nb * BN;
        // SF_AHEAD K-blocks of scale loads in flight per thread
        SfRegs ring[SF_AHEAD];
#pragma unroll
        for (int u = 0; u < SF_AHEAD; ++u)
            if (u < nkb) load_sf(p, tr.g, tr.m0, tr.m_end, n0, u, nkb, t, ring[u]);
        for (int64_t kb0 = 0; ok && kb0 < nkb; kb0 += SF_AHEAD) {
#pragma unroll
            for (int u = 0; u < SF_AHEAD; ++u) {
                const int64_t kb = kb0 + u;
                if (ok && kb < nkb) {            // warp-uniform
                    const uint32_t wa = ue8m0_x4(ring[u].a, bad);
                    const uint32_t wb0 = ue8m0_x4(ring[u].b[0], bad);
                    const uint32_t wb1 = ue8m0_x4(ring[u].b[1], bad);
                    if (kb + SF_AHEAD < nkb)
                        load_sf(p, tr.g, tr.m0, tr.m_end, n0, kb + SF_AHEAD, nkb, t, ring[u]);
                    const int s = (int)(it % NS);
                    const uint32_t ph = (uint32_t)((it / NS) & 1);
                    // the copies and MMAs that last read this stage have completed
                    if (warp_wait(&sh.empty[s], ph ^ 1u, abort, p.timeout_ns, lane)) {
                        ++it;
                        uint8_t* sf = sf_base + s * SF_BYTES;
                        *reinterpret_cast<uint32_t*>(sf + off_a) = wa;
                        *reinterpret_cast<uint32_t*>(sf + off_b0) = wb0;
                        *reinterpret_cast<uint32_t*>(sf + off_b1) = wb1;
                        fence_proxy_async_smem();
                        __syncwarp();
                        // the even CTA's MMA thread copies both CTAs' blocks
                        if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&sh.full[s]), 0));
                    } else {
                        ok = false;
                    }
                }
            }
        }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) report_error(FP8_ERR_VALUE);
}

__device__ void mx_epilogue(const MxParams& p, MxShared& sh, int64_t nmb, int64_t nnb, int warp,
                            int lane)
{
    volatile int* abort = &sh.abort;
    const uint32_t rank = cluster_ctarank();
    const int ew = warp - FIRST_EPI_WARP;       // 0..7
    const int q = warp & 3;
    const int col0 = (ew >> 2) * 128;
    const int row = q * 32 + lane;
    const uint32_t taddr0 = sh.tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)col0;
    uint32_t tcount = 0;
    int64_t first, stride;
    mx_unit_range(first, stride);
    for (int64_t tile = first; tile < nmb * nnb; tile += stride) {
        int64_t mb, nb;
        gemm_tile_coord(tile, nmb, nnb, p.band, mb, nb);
        TileRows tr;
        if (!mx_tile_rows(p, sh, mb, rank, tr)) continue;
        const uint32_t tph = tcount++ & 1u;
        const int64_t m = tr.m0 + row;
        const int64_t n0 = nb * BN + col0;
        // warp-uniform: columns inside N and this CTA's rows inside the group
        const bool active = n0 < p.N && tr.m0 < tr.m_end;
        const bool row_ok = m < tr.m_end;
        if (!warp_wait(&sh.acc_full, tph, abort, p.timeout_ns, lane)) break;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            uint32_t r[32];
            if (active) {
                tmem_ld32(taddr0 + (uint32_t)(c * 32), r);
                tmem_ld_wait(r);
            }
            if (c == 3) {                        // accumulator no longer needed
                tc_fence_before();
                __syncwarp();
                // the even CTA's MMA waits for both CTAs' epilogues
                if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&sh.acc_empty), 0));
            }
            if (!(active && row_ok)) continue;
            if (p.out_dtype == FP8_OUT_BF16) {
                uint4* d = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.D) + m * p.ldd +
                                                    n0 + c * 32);
#pragma unroll
                for (int v = 0; v < 4; ++v) {
                    uint4 w;
                    w.x = pack_bf16x2_rn(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
                    w.y = pack_bf16x2_rn(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
                    w.z = pack_bf16x2_rn(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
                    w.w = pack_bf16x2_rn(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
                    d[v] = w;
                }
            } else {
                uint4* d = reinterpret_cast<uint4*>(static_cast<float*>(p.D) + m * p.ldd + n0 + c * 32);
#pragma unroll
                for (int v = 0; v < 8; ++v)
                    d[v] = make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]);
            }
        }
    }
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_fp8_gemm_mx(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                  const MxParams p)
{
    extern __shared__ uint8_t smem_raw[];
    __shared__ MxShared sh;
    // same 1024-byte-aligned offset in both CTAs of a pair
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t nnb = (p.N + BN - 1) / BN;
    const int64_t nkb = p.K / BK;
    const uint32_t rank = cluster_ctarank();

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            // the TMA bytes' arrive plus every scale warp (of both CTAs of a pair)
            mbar_init(&sh.full[s], 1 + 2 * NUM_SF_WARPS);
            mbar_init(&sh.empty[s], 1);
        }
        mbar_init(&sh.acc_full, 1);
        mbar_init(&sh.acc_empty, 2 * NUM_EPI_WARPS);
        mbar_init(&sh.drain, 1);
        sh.abort = 0;
        sh.bad = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
    }
    if (warp == 2) {
        tmem_alloc_pair(&sh.tmem_base, TMEM_COLS);
        tmem_relinquish_pair();
    }
    if (p.group_offsets)
        for (int i = threadIdx.x; i <= p.G; i += NUM_THREADS) sh.off[i] = p.group_offsets[i];
    // barrier inits and the TMEM address visible to the peer CTA before use
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    if (threadIdx.x == 0) {
        bool bad = false;
        if (p.group_offsets) {
            bad = sh.off[0] != 0 || (int64_t)sh.off[p.G] > p.M;
            for (int e = 0; e < p.G; ++e) bad = bad || sh.off[e + 1] < sh.off[e] || (sh.off[e + 1] & 127);
            if (bad && blockIdx.x == 0) report_error(FP8_ERR_SHAPE);
        }
        sh.bad = bad ? 1 : 0;
    }
    __syncthreads();
    if (p.group_offsets && !sh.bad && warp == 0)
        pair_block_offsets(sh.off, sh.poff, p.G, lane);
    __syncthreads();
    const int64_t nmb = p.group_offsets ? (int64_t)sh.poff[p.G] : (p.M + TILE_M - 1) / TILE_M;

    if (sh.bad) {
        // malformed offsets: nothing is loaded, multiplied or written
    } else if (warp == 0) {
        if (lane == 0) mx_producer(&tmA, &tmB, p, smem, sh, nmb, nnb, nkb);
        __syncwarp();
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) mx_mma(p, smem, sh, nmb, nnb, nkb);
        __syncwarp();
    } else if (warp >= FIRST_SF_WARP && warp < FIRST_SF_WARP + NUM_SF_WARPS) {
        mx_scale_writer(p, smem, sh, nmb, nnb, nkb, warp, lane);
    } else if (warp >= FIRST_EPI_WARP) {
        mx_epilogue(p, sh, nmb, nnb, warp, lane);
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    if (warp == 2) tmem_dealloc_pair(sh.tmem_base, TMEM_COLS);
}

cudaLaunchConfig_t mx_pair_config(unsigned clusters, cudaStream_t st, cudaLaunchAttribute* attr)
{
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * clusters, 1, 1);
    cfg.blockDim = dim3(NUM_THREADS, 1, 1);
    cfg.dynamicSmemBytes = DYN_SMEM;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cfg;
}

// Once per device: shared-memory opt-in and the number of CTA pairs that fit
// at once (the persistent grid).
struct MxDeviceSetup {
    bool ok = false;
    int pair_clusters = 0;
};

MxDeviceSetup mx_device_setup()
{
    static MxDeviceSetup done[64];
    static bool tried[64] = {};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return MxDeviceSetup{};
    std::lock_guard<std::mutex> lk(mu);
    if (!tried[dev]) {
        tried[dev] = true;
        MxDeviceSetup r;
        r.ok = cudaFuncSetAttribute(k_fp8_gemm_mx, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)DYN_SMEM) == cudaSuccess;
        if (r.ok) {
            cudaLaunchAttribute attr[1];
            const cudaLaunchConfig_t cfg = mx_pair_config((unsigned)device_sm_count(), nullptr, attr);
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, k_fp8_gemm_mx, &cfg) != cudaSuccess) {
                n = 0;
                (void)cudaGetLastError();
            }
            r.pair_clusters = n;
        } else {
            (void)cudaGetLastError();
        }
        done[dev] = r;
    }
    return done[dev];
}

int launch_mx(const uint8_t* A, const float* sA, const uint8_t* B, int b_major, const float* sB,
              int sb_gran, int64_t M, int64_t N, int64_t K, const int32_t* group_offsets, int G,
              void* D, int out_dtype, int64_t ldd, int withhold, cudaStream_t st)
{
    if (M == 0) return FP8_OK;
    const MxDeviceSetup setup = mx_device_setup();
    if (!setup.ok) return FP8_ERR_LAUNCH;
    if (setup.pair_clusters < 1) return FP8_ERR_DEVICE;   // needs co-scheduled 2-CTA clusters
    CUtensorMap tmA, tmB;
    if (!make_map(&tmA, A, (uint64_t)K, (uint64_t)M, (uint64_t)K, BK, BM)) return FP8_ERR_LAUNCH;
    bool okB;
    if (b_major == FP8_B_KMAJOR) {
        const uint64_t rows = (uint64_t)N * (uint64_t)(group_offsets ? G : 1);
        okB = make_map(&tmB, B, (uint64_t)K, rows, (uint64_t)K, BK, 128);
    } else {
        okB = make_map(&tmB, B, (uint64_t)N, (uint64_t)K, (uint64_t)N, 128, BK);
    }
    if (!okB) return FP8_ERR_LAUNCH;

    MxParams p;
    p.sA = sA;
    p.sB = sB;
    p.D = D;
    p.group_offsets = group_offsets;
    p.M = M;
    p.N = N;
    p.K = K;
    p.ldd = ldd;
    p.G = group_offsets ? G : 0;
    p.b_major = b_major;
    p.sb_gran = sb_gran;
    p.out_dtype = out_dtype;
    p.withhold = withhold;
    p.band = group_offsets ? BAND_GROUPED : BAND_DENSE;
    p.timeout_ns = wait_timeout_ns();

    const int64_t nnb = (N + BN - 1) / BN;
    // grouped: each group adds at most one partly idle 256-row block
    const int64_t tiles = ((M + 255) / 256 + (group_offsets ? G : 0)) * nnb;
    const int64_t clusters = tiles < setup.pair_clusters ? tiles : setup.pair_clusters;
    cudaLaunchAttribute attr[1];
    const cudaLaunchConfig_t cfg = mx_pair_config((unsigned)clusters, st, attr);
    return cudaLaunchKernelEx(&cfg, k_fp8_gemm_mx, tmA, tmB, p) == cudaSuccess ? FP8_OK
                                                                               : FP8_ERR_LAUNCH;
}

}  // namespace

int launch_blockscaled_gemm_mx(const uint8_t* A, const float* sA, const uint8_t* B, int b_major,
                               const float* sB, int sb_gran, int64_t M, int64_t N, int64_t K,
                               const int32_t* group_offsets, int G, void* D, int out_dtype,
                               int64_t ldd, cudaStream_t st)
{
    return launch_mx(A, sA, B, b_major, sB, sb_gran, M, N, K, group_offsets, G, D, out_dtype, ldd,
                     0, st);
}

int launch_blockscaled_gemm_mx_withheld(const uint8_t* A, const float* sA, const uint8_t* B,
                                        int b_major, const float* sB, int sb_gran, int64_t M,
                                        int64_t N, int64_t K, const int32_t* group_offsets, int G,
                                        void* D, int out_dtype, int64_t ldd, cudaStream_t st)
{
    return launch_mx(A, sA, B, b_major, sB, sb_gran, M, N, K, group_offsets, G, D, out_dtype, ldd,
                     1, st);
}

int read_and_clear_mx_status() { return read_and_clear_module_status(); }

}  // namespace fp8fg
