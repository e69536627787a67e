// gemm.cu -- block-scaled E4M3 x E4M3 GEMM with FP32 promotion every 128 K
// (sm_100a: TMA -> shared memory -> tcgen05.mma.kind::f8f6f4 -> TMEM).
//
// What it computes (DeepSeek-V3 FP8 recipe as reproduced on the pages "5 Ways
// You can get More Deepseek While Spending Less", the why-be.co.kr post and
// the gnrental.net post, passage on increasing accumulation precision): the
// scales vary along the inner dimension every 128 elements, so the tensor
// cores produce one partial product per 128-element K-block, and that partial
// is moved out, multiplied by scale_a * scale_b and accumulated in full FP32.
//
// The pages' H800 design keeps two WGMMA warpgroups in flight so one promotes
// while the other multiplies.  On sm_100 the same overlap comes from the
// accumulator living in TMEM: the MMA writes K-block kb's partial into one of
// two TMEM buffers while the promotion warps drain the other buffer into
// FP32 registers.  Roles per CTA (persistent, one CTA per SM):
//   warp 0      TMA producer: A / B tiles for each K-block into a shared-
//               memory ring (128-byte swizzle, no cluster multicast)
//   warp 1      TMEM allocator + MMA issuer: 4 x tcgen05.mma (K = 32 each)
//               per K-block into TMEM buffer kb & 1, then tcgen05.commit
//   warps 2-3   idle (they complete warpgroup 0, which hands its registers
//               to the promotion warpgroups)
//   warps 4-11  promotion + epilogue: tcgen05.ld the partial, FMA it (packed
//               FP32x2) with its scale into a register accumulator, release the
//               buffer; after the last K-block convert to BF16/FP32, stage 32
//               rows x 32 bytes at a time in shared memory and hand them to a
//               TMA store, then go on with the next tile at once.
// Each CTA promotes a 128 (M) x 256 (N) block; warps 4-7 own its columns
// 0-127, warps 8-11 columns 128-255, each warp the 32 TMEM lanes (rows) its
// id allows.
//
// Dense GEMMs run on CTA pairs (2-CTA clusters): one tcgen05.mma.cta_group::2
// issued by the even CTA computes a 256 x 256 x 32 product on the tensor
// cores of both SMs.  Each CTA loads its own 128 rows of A and 128 of B's 256
// columns, so a K-block brings 32 KB into each SM instead of 48 KB; with the
// bytes freed the ring holds 6 stages instead of 4.  Both CTAs' loads count
// on the even CTA's `full` barrier, the MMA's commits arrive on both CTAs'
// `empty` / `tfull` barriers, and every promotion warp of the pair releases a
// TMEM buffer on the even CTA's `tempty` barrier.  Grouped (MoE) GEMMs count
// their 256-row blocks group by group, so that both halves of a pair use the
// same expert's B; a group of an odd number of 128-row blocks leaves the odd
// CTA of its last pair idle.
//
// Work is dealt to the pairs tile by tile, in raster bands of M-blocks.  For
// FP32 outputs whose tile count leaves the last round poorly filled, the
// pairs instead take equal contiguous ranges of (tile, K-block) units
// (stream-K): a tile cut between two pairs gets two partial sums, which TMA
// reduce-adds into D after a small kernel has zeroed those tiles.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>
#include <mutex>

#include "fp8fg_device.cuh"
#include "fp8fg_host.h"

namespace fp8fg {

namespace {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 128;
constexpr int TILE_M = 256;                             // rows per pair tile
constexpr uint32_t A_BYTES = BM * BK;                   // 16 KB per stage
constexpr uint32_t B_BYTES = 128 * BK;                  // this CTA's 128 of B's columns
constexpr int NS = 6;                                   // ring stages of 32 KB
constexpr uint32_t RING_BYTES = NS * (A_BYTES + B_BYTES);   // 192 KB
constexpr int NUM_PROMO_WARPS = 8;
constexpr int FIRST_PROMO_WARP = 4;                     // warpgroups 1 and 2
constexpr int NUM_THREADS = 128 + 32 * NUM_PROMO_WARPS; // 384 = 3 warpgroups
// Register split: launch gives every thread LAUNCH_REGS (65536 / 384 rounded
// down to 8); warpgroup 0 (TMA, MMA, 2 idle warps) drops to CTRL_REGS and the
// two promotion warpgroups rise to PROMO_REGS, within the launch total.
constexpr uint32_t LAUNCH_REGS = 168;
constexpr uint32_t CTRL_REGS = 72;
constexpr uint32_t PROMO_REGS = 216;
static_assert(128 * CTRL_REGS + 256 * PROMO_REGS <= NUM_THREADS * LAUNCH_REGS,
              "register split exceeds the launch allocation");
constexpr int PROMO_CHUNK = 32;                        // TMEM columns per load round trip
constexpr uint32_t TMEM_COLS = 2 * BN;                  // two FP32 partial buffers
constexpr int MAX_GROUPS = 1024;
// Raster bands (m-blocks per band): 16 for dense GEMMs; 6 for grouped ones,
// whose bands otherwise span several experts' rows and weights at once.
constexpr int BAND_DENSE = 16;
constexpr int BAND_GROUPED = 6;
constexpr uint32_t DYN_SMEM = 1024 + RING_BYTES;

struct GemmParams {
    const float* sA;               // [K/128][M]
    const float* sB;               // see fp8_blockscaled_gemm / fp8_grouped_gemm
    void* D;
    const int32_t* group_offsets;  // nullptr: dense
    int64_t M, N, K, ldd;
    int G;
    int b_major, sb_gran, out_dtype;
    int band;                      // m-blocks per raster band
    int streamk;                   // 1: contiguous ranges of (tile, K-block) units per pair
    int withhold;                  // self-test: the odd CTA stops loading after one K-block
    const int32_t* row_map;        // grouped gather: A row of each output row (nullptr: A as is)
    int64_t a_rows;                // gather: rows of A (and of sA's K-block rows)
    uint64_t timeout_ns;
};


// Epilogue staging: each promotion warp writes its 32 rows x 32 bytes of
// output at a time into one of two 1 KB buffers, from which a TMA store
// copies them to D (boxes EPI_BYTES wide, EPI_ROWS rows).
constexpr int EPI_BYTES = 32;                           // bytes of a row per store
constexpr int EPI_ROWS = 32;

struct __align__(128) Shared {
    uint8_t epi[NUM_PROMO_WARPS][2][EPI_ROWS * EPI_BYTES];   // first: 128-byte aligned
    float sbw[NUM_PROMO_WARPS][2][128];   // per-warp column scales (sb_gran == 1),
                                          // read and written as float4: 16-B aligned
    uint64_t full[NS];
    uint64_t empty[NS];
    uint64_t tfull[2];
    uint64_t tempty[2];
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
    int bad;
    int32_t off[MAX_GROUPS + 1];    // grouped: row offsets of the groups
    int32_t poff[MAX_GROUPS + 1];   // grouped pairs: first 256-row block of each group
};
static_assert(offsetof(Shared, sbw) % 16 == 0, "float4 accesses need 16-byte alignment");
static_assert(offsetof(Shared, epi) % 128 == 0 && EPI_ROWS * EPI_BYTES % 128 == 0,
              "TMA store sources stay 128-byte aligned");
static_assert(sizeof(float) * 128 % 16 == 0, "per-warp scale rows stay 16-byte aligned");
static_assert(offsetof(Shared, full) % 8 == 0, "mbarriers need 8-byte alignment");

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&v);
}

// ------------------------------------------------------------------ roles

__device__ __forceinline__ bool tile_rows(const GemmParams& p, const Shared& sh, int64_t mb,
                                          uint32_t rank, TileRows& t)
{
    return tile_rows(p.group_offsets, sh.off, sh.poff, p.G, p.M, mb, rank, t);
}

// The work of pair c (CTAs 2c, 2c+1) as a sequence of segments: a tile and
// the range [kb0, kb1) of its K-blocks.  Normally tiles are dealt round-robin
// and every segment is a whole tile.  With stream-K the tiles' K-blocks are
// laid end to end (tile t owns units t*nkb .. t*nkb+nkb-1) and pair c takes
// the contiguous units [c*U/P, (c+1)*U/P): every pair gets the same work, and
// a tile cut between two pairs has exactly two contributors (each range is
// at least one tile long), which add their partial sums into D.
struct Segments {
    int64_t tile, kb0, kb1;   // current segment
    int64_t u, u_end;         // stream-K: next unit, end of this pair's range
    int64_t stride;           // round-robin: tiles between this pair's tiles
    int64_t ntiles, nkb;
    bool streamk;
};

__device__ __forceinline__ void seg_set(Segments& g)
{
    g.tile = g.u / g.nkb;
    g.kb0 = g.u - g.tile * g.nkb;
    const int64_t left = g.u_end - g.u;
    g.kb1 = g.kb0 + left < g.nkb ? g.kb0 + left : g.nkb;
}

__device__ __forceinline__ void seg_begin(Segments& g, const GemmParams& p, int64_t ntiles,
                                          int64_t nkb)
{
    const int64_t pair = (int64_t)(blockIdx.x >> 1), pairs = (int64_t)(gridDim.x >> 1);
    g.ntiles = ntiles;
    g.nkb = nkb;
    g.streamk = p.streamk != 0;
    if (g.streamk) {
        const int64_t units = ntiles * nkb;
        g.u = pair * units / pairs;
        g.u_end = (pair + 1) * units / pairs;
        if (g.u < g.u_end) seg_set(g);
        else g.tile = ntiles;
    } else {
        g.stride = pairs;
        g.tile = pair;
        g.kb0 = 0;
        g.kb1 = nkb;
    }
}

__device__ __forceinline__ bool seg_valid(const Segments& g) { return g.tile < g.ntiles; }

__device__ __forceinline__ void seg_next(Segments& g)
{
    if (g.streamk) {
        g.u += g.kb1 - g.kb0;
        if (g.u < g.u_end) seg_set(g);
        else g.tile = g.ntiles;
    } else {
        g.tile += g.stride;
    }
}

// Run by the whole of warp 0.  Lane 0 arms the stage barrier and issues the
// tiled loads; with gathered A each lane issues one 4-row gather (rows
// 4*lane .. 4*lane+3 of the CTA's 128), so a stage's 32 gathers leave in one
// warp instruction.  Every decision is warp-uniform.
__device__ void run_producer(const CUtensorMap* tmA, const CUtensorMap* tmB, const GemmParams& p,
                             uint8_t* smem, Shared& sh, int64_t nmb, int64_t nnb, int64_t nkb,
                             int lane)
{
    volatile int* abort = &sh.abort;
    const uint32_t rank = cluster_ctarank();
    int64_t it = 0;   // loads issued so far; stage it % NS, round it / NS
    bool ok = true;
    Segments sg;
    for (seg_begin(sg, p, nmb * nnb, nkb); ok && seg_valid(sg); seg_next(sg)) {
        int64_t mb, nb;
        gemm_tile_coord(sg.tile, nmb, nnb, p.band, mb, nb);
        TileRows tr;
        if (!tile_rows(p, sh, mb, rank, tr)) continue;
        // (an idle odd CTA still loads its rows: the pair's MMA counts them)
        const int64_t m0 = tr.m0;
        const int64_t n0 = nb * BN;
        const int g = tr.g;
        // A CTA of a pair loads B's columns rank*128 .. rank*128+127 of the
        // tile (a box counts in full, its out-of-range part zero-filled).
        const int32_t brow = (int32_t)((int64_t)g * p.N + n0 + rank * 128);
        // Gathered A: the A rows of this lane's 4 output rows.  Rows past
        // the group, padding rows (-1) and invalid indices read row 0; their
        // promotion multiplies by a zero scale.
        int32_t ar[4] = {0, 0, 0, 0};
        if (p.row_map) {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int64_t m = m0 + 4 * lane + i;
                const int32_t r = (m < tr.m_end && m < p.M) ? __ldg(p.row_map + m) : -1;
                ar[i] = (r >= 0 && r < p.a_rows) ? r : 0;
            }
        }
        for (int64_t kb = sg.kb0; kb < sg.kb1; ++kb) {
            if (p.withhold && rank == 1 && it == 1) {   // self-test only
                ok = false;
                break;
            }
            const int s = (int)(it % NS);
            const uint32_t ph = (uint32_t)((it / NS) & 1);
            // every lane sees the stage free (or the warp gives up together)
            if (!__all_sync(0xFFFFFFFFu, mbar_wait(&sh.empty[s], ph ^ 1u, abort, p.timeout_ns))) {
                ok = false;
                break;
            }
            ++it;
            uint8_t* a_dst = smem + s * A_BYTES;
            uint8_t* b_dst = smem + NS * A_BYTES + s * B_BYTES;
            // Both CTAs' loads complete on the even CTA's barrier, which
            // expects the pair's bytes; the odd CTA only issues its loads.
            const uint32_t bar = mapa_shared(smem_u32(&sh.full[s]), 0);
            if (lane == 0 && rank == 0) mbar_arrive_expect_tx(&sh.full[s], 2 * (A_BYTES + B_BYTES));
            __syncwarp();
            if (p.row_map) {
                // 32 gathers of 4 rows each fill the same swizzled 128-row tile
                tma_gather4_pair(a_dst + lane * 4 * BK, tmA, bar, (int32_t)(kb * BK), ar[0], ar[1],
                                 ar[2], ar[3]);
            } else if (lane == 0) {
                tma_load_2d_pair(a_dst, tmA, bar, (int32_t)(kb * BK), (int32_t)m0);
            }
            if (lane == 0) {
                if (p.b_major == FP8_B_KMAJOR)
                    tma_load_2d_pair(b_dst, tmB, bar, (int32_t)(kb * BK), brow);
                else
                    tma_load_2d_pair(b_dst, tmB, bar, (int32_t)(n0 + rank * 128), (int32_t)(kb * BK));
            }
        }
    }
    // Every copy issued must land before the CTA may exit: stage s received
    // ceil((it - s) / NS) loads, the last one completing phase (count-1)&1.
    // A pair's loads all count on the even CTA's barriers, so it drains for
    // both (the odd CTA stays resident until the closing cluster barrier).
    if (rank != 0 || lane != 0) return;
#pragma unroll
    for (int s = 0; s < NS; ++s) {
        const int64_t count = it > s ? (it - s + NS - 1) / NS : 0;
        if (count) mbar_wait_drain(&sh.full[s], (uint32_t)((count - 1) & 1), p.timeout_ns);
    }
}

__device__ void run_mma(const GemmParams& p, uint8_t* smem, Shared& sh, int64_t nmb, int64_t nnb,
                        int64_t nkb)
{
    volatile int* abort = &sh.abort;
    const uint32_t a_base = smem_u32(smem);
    const uint32_t b_base = a_base + NS * A_BYTES;
    const uint32_t tmem = sh.tmem_base;
    int64_t it = 0, kbg = 0;
    bool ok = true;
    Segments sg;
    for (seg_begin(sg, p, nmb * nnb, nkb); ok && seg_valid(sg); seg_next(sg)) {
        // A pair's MMA always spans 256 columns (a B tail is zero-filled).
        const uint32_t idesc = idesc_e4m3_f32((uint32_t)TILE_M, (uint32_t)BN, (uint32_t)p.b_major);
        for (int64_t kb = sg.kb0; kb < sg.kb1; ++kb, ++it, ++kbg) {
            const int s = (int)(it % NS);
            const uint32_t ph = (uint32_t)((it / NS) & 1);
            const uint32_t buf = (uint32_t)(kbg & 1);
            const uint32_t tph = (uint32_t)((kbg >> 1) & 1);
            if (!mbar_wait(&sh.tempty[buf], tph ^ 1u, abort, p.timeout_ns) ||
                !mbar_wait(&sh.full[s], ph, abort, p.timeout_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t d = tmem + buf * BN;
            const uint32_t a_addr = a_base + s * A_BYTES;
            const uint32_t b_addr = b_base + s * B_BYTES;
#pragma unroll
            for (int k = 0; k < BK / 32; ++k) {
                const uint64_t adesc = smem_desc_sw128(a_addr + k * 32, 16, 1024);
                const uint64_t bdesc = (p.b_major == FP8_B_KMAJOR)
                                           ? smem_desc_sw128(b_addr + k * 32, 16, 1024)
                                           : smem_desc_sw128(b_addr + k * 32 * 128, 128 * BK, 1024);
                mma_f8f6f4_pair(d, adesc, bdesc, idesc, k > 0 ? 1u : 0u);
            }
            // stage free and partial ready in both CTAs of the pair
            mma_commit_pair(&sh.empty[s], 3);
            mma_commit_pair(&sh.tfull[buf], 3);
        }
    }
    // Wait for every MMA this thread issued before TMEM is released.
    mma_commit_pair(&sh.drain, 1);
    mbar_wait_drain(&sh.drain, 0, p.timeout_ns);
}

// GRAN is the weight-scale granularity along N (p.sb_gran): 128 (one scale
// per 128x128 block) or 1 (one per column); each gets its own instance.
template <int GRAN>
__device__ void run_promotion(const CUtensorMap* tmD, const GemmParams& p, Shared& sh, int nmb,
                              int nnb, int nkb, int warp, int lane)
{
    volatile int* abort = &sh.abort;
    const int rank = (int)cluster_ctarank();
    const int ew = warp - FIRST_PROMO_WARP;   // 0..7
    const int quad = warp & 3;            // TMEM lanes this warp may access
    const int half = ew >> 2;             // column half of the tile
    const int row = quad * 32 + lane;     // tile row == TMEM lane
    const int col0 = half * 128;
    const uint32_t tmem_lane = sh.tmem_base + ((uint32_t)(quad * 32) << 16);
    const int nnb128 = (int)(p.N / 128);
    uint32_t kbg = 0;

    Segments sg;
    for (seg_begin(sg, p, (int64_t)nmb * nnb, nkb); seg_valid(sg); seg_next(sg)) {
        int64_t mb64, nb64;
        gemm_tile_coord(sg.tile, nmb, nnb, p.band, mb64, nb64);
        const int kb0 = (int)sg.kb0, kb1 = (int)sg.kb1;
        // the whole K range of the tile (a plain store), or a stream-K part
        // of it (the two parts are added into D, which starts at zero)
        const bool whole = kb0 == 0 && kb1 == nkb;
        TileRows tr;
        if (!tile_rows(p, sh, mb64, (uint32_t)rank, tr)) continue;
        const int nb = (int)nb64;
        const int m0 = (int)tr.m0, n0 = nb * BN;
        const int g = tr.g;
        const int m = m0 + row;
        const bool row_ok = m < tr.m_end;
        // a warp whose columns lie past N, or whose CTA idles in this tile,
        // only keeps the K-block handshakes going
        const bool active = (n0 + col0) < p.N && tr.m0 < tr.m_end;
        const int cb = (n0 + col0) / 128;   // 128-column block of B

        // Scales of K-block kb for this thread, prefetched one K-block ahead:
        //   sa   its row's activation scale, sA[kb][m]
        //   sb   its 128-column block's weight scale (sb_gran 128), or
        //   sb4  4 of its half's 128 column scales (sb_gran 1), staged in this
        //        warp's shared buffer so every lane can read all 128.
        // the row's activation scales: sA[kb][m], or with gathered A the
        // scales of its A row (none for padding rows: scale 0, output 0)
        int64_t sa_row = m, sa_ld = p.M;
        bool sa_ok = row_ok;
        if (p.row_map) {
            const int32_t r = row_ok ? __ldg(p.row_map + m) : -1;
            if (r < -1 || r >= p.a_rows) report_error(FP8_ERR_SHAPE);
            sa_ok = r >= 0 && r < p.a_rows;
            sa_row = r;
            sa_ld = p.a_rows;
        }
        const float* sa_ptr = p.sA + (sa_ok ? sa_row + (int64_t)kb0 * sa_ld : 0);
        const int64_t sa_step = sa_ok ? sa_ld : 0;
        const bool use_sb = active && GRAN == 128;
        const float* sb_ptr = p.sB;
        int64_t sb_step = 0;
        if (GRAN == 128) {
            if (p.b_major == FP8_B_KMAJOR) {
                sb_ptr = p.sB + ((int64_t)g * nnb128 + cb) * nkb + kb0;
                sb_step = 1;
            } else {
                sb_ptr = p.sB + cb + (int64_t)kb0 * nnb128;
                sb_step = nnb128;
            }
        }
        const bool use_sb4 = active && GRAN == 1;
        const float4* sb4_ptr =
            reinterpret_cast<const float4*>(p.sB + (int64_t)kb0 * p.N + n0 + col0) + lane;
        const int64_t sb4_step = p.N / 4;

        float acc[128];
#pragma unroll
        for (int i = 0; i < 128; ++i) acc[i] = 0.0f;

        float sa_next = sa_ok ? __ldg(sa_ptr) : 0.0f;
        float sb_next = use_sb ? __ldg(sb_ptr) : 0.0f;
        if (GRAN == 1) {
            *reinterpret_cast<float4*>(&sh.sbw[ew][kb0 & 1][lane * 4]) =
                use_sb4 ? __ldg(sb4_ptr) : make_float4(0.f, 0.f, 0.f, 0.f);
            __syncwarp();
        }
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb, ++kbg) {
            const float sa = sa_next, sb = sb_next;
            float4 sb4_next = make_float4(0.f, 0.f, 0.f, 0.f);
            if (kb + 1 < kb1) {
                sa_ptr += sa_step;
                sb_ptr += sb_step;
                sb4_ptr += sb4_step;
                if (sa_ok) sa_next = __ldg(sa_ptr);
                if (use_sb) sb_next = __ldg(sb_ptr);
                if (use_sb4) sb4_next = __ldg(sb4_ptr);
            }
            const uint32_t buf = kbg & 1;
            const uint32_t tph = (kbg >> 1) & 1;
            if (!mbar_wait(&sh.tfull[buf], tph, abort, p.timeout_ns)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (active) {
                const uint32_t taddr = tmem_lane + buf * BN + col0;
                // PROMO_CHUNK columns per TMEM round trip: their 16-column
                // loads are all in flight before the first wait.
                constexpr int NL = PROMO_CHUNK / 16;
                if (GRAN == 128) {
                    // the next chunk's loads are in flight while this chunk's
                    // FMAs run (two register sets, used in turn)
                    const float sc = sa * sb;
                    constexpr int NC = 128 / PROMO_CHUNK;
                    uint32_t ra[NL][16], rb[NL][16];
#pragma unroll
                    for (int l = 0; l < NL; ++l) tmem_ld16(taddr + l * 16, ra[l]);
#pragma unroll
                    for (int l = 0; l < NL; ++l) tmem_ld_wait(ra[l]);
#pragma unroll
                    for (int c = 0; c < NC; ++c) {
                        uint32_t (&cur)[NL][16] = (c & 1) ? rb : ra;
                        uint32_t (&nxt)[NL][16] = (c & 1) ? ra : rb;
                        if (c + 1 < NC) {
#pragma unroll
                            for (int l = 0; l < NL; ++l)
                                tmem_ld16(taddr + (c + 1) * PROMO_CHUNK + l * 16, nxt[l]);
                        }
#pragma unroll
                        for (int l = 0; l < NL; ++l)
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const int j = c * PROMO_CHUNK + l * 16 + 2 * i;
                                ffma2(acc[j], acc[j + 1], __uint_as_float(cur[l][2 * i]),
                                      __uint_as_float(cur[l][2 * i + 1]), sc, sc);
                            }
                        if (c + 1 < NC) {
#pragma unroll
                            for (int l = 0; l < NL; ++l) tmem_ld_wait(nxt[l]);
                        }
                    }
                } else {
                    // The chunk's products sa * sb[col] only need shared memory
                    // and registers, so they are formed while its TMEM loads
                    // are in flight; after the wait only the FMAs remain.
                    const float* sbv = sh.sbw[ew][kb & 1];
#pragma unroll
                    for (int c = 0; c < 128 / PROMO_CHUNK; ++c) {
                        uint32_t r[NL][16];
#pragma unroll
                        for (int l = 0; l < NL; ++l) tmem_ld16(taddr + c * PROMO_CHUNK + l * 16, r[l]);
                        float t[PROMO_CHUNK];
#pragma unroll
                        for (int i = 0; i < PROMO_CHUNK / 4; ++i) {
                            const float4 b = *reinterpret_cast<const float4*>(sbv + c * PROMO_CHUNK + 4 * i);
                            fmul2(t[4 * i], t[4 * i + 1], b.x, b.y, sa, sa);
                            fmul2(t[4 * i + 2], t[4 * i + 3], b.z, b.w, sa, sa);
                        }
#pragma unroll
                        for (int l = 0; l < NL; ++l) tmem_ld_wait(r[l]);
#pragma unroll
                        for (int l = 0; l < NL; ++l)
#pragma unroll
                            for (int i = 0; i < 8; ++i) {
                                const int j = c * PROMO_CHUNK + l * 16 + 2 * i;
                                ffma2(acc[j], acc[j + 1], __uint_as_float(r[l][2 * i]),
                                      __uint_as_float(r[l][2 * i + 1]), t[l * 16 + 2 * i],
                                      t[l * 16 + 2 * i + 1]);
                            }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            // the even CTA's MMA waits for both CTAs' warps
            if (lane == 0) mbar_arrive_cluster(mapa_shared(smem_u32(&sh.tempty[buf]), 0));
            if (GRAN == 1) {
                *reinterpret_cast<float4*>(&sh.sbw[ew][(kb + 1) & 1][lane * 4]) = sb4_next;
                __syncwarp();
            }
        }
        if (!ok) break;

        // Epilogue: round the FP32 sums to the output type and store them.
        // Each lane writes its row's next 32 bytes into this warp's staging
        // buffer; one lane hands the 32 x 32-byte box to a TMA store (or, for
        // a stream-K part of a tile, a TMA reduce-add), which drops the rows
        // beyond M and the columns beyond N.  Two buffers alternate, so a
        // store's read of one overlaps the writes of the other.
        if (active) {
            const int esz = p.out_dtype == FP8_OUT_BF16 ? 2 : 4;
            const int nch = 128 * esz / EPI_BYTES;                 // 8 (BF16) or 16 (FP32)
            const int32_t y = m0 + quad * 32;
            const int32_t x0 = n0 + col0;                          // elements
            const int xstep = EPI_BYTES / esz;
#pragma unroll
            for (int ch = 0; ch < 16; ++ch) {
                if (ch >= nch) break;
                uint8_t* buf = sh.epi[ew][ch & 1];
                if (lane == 0) bulk_wait_group_read<1>();   // the store that read `buf` is done
                __syncwarp();
                uint4 w0, w1;
                if (esz == 2) {
                    const int j = 16 * ch;
                    w0 = make_uint4(pack_bf16x2(acc[j + 0], acc[j + 1]), pack_bf16x2(acc[j + 2], acc[j + 3]),
                                    pack_bf16x2(acc[j + 4], acc[j + 5]), pack_bf16x2(acc[j + 6], acc[j + 7]));
                    w1 = make_uint4(pack_bf16x2(acc[j + 8], acc[j + 9]), pack_bf16x2(acc[j + 10], acc[j + 11]),
                                    pack_bf16x2(acc[j + 12], acc[j + 13]), pack_bf16x2(acc[j + 14], acc[j + 15]));
                } else {
                    const int j = 8 * ch;
                    w0 = make_uint4(__float_as_uint(acc[j + 0]), __float_as_uint(acc[j + 1]),
                                    __float_as_uint(acc[j + 2]), __float_as_uint(acc[j + 3]));
                    w1 = make_uint4(__float_as_uint(acc[j + 4]), __float_as_uint(acc[j + 5]),
                                    __float_as_uint(acc[j + 6]), __float_as_uint(acc[j + 7]));
                }
                *reinterpret_cast<uint4*>(buf + lane * EPI_BYTES) = w0;
                *reinterpret_cast<uint4*>(buf + lane * EPI_BYTES + 16) = w1;
                fence_proxy_async_shared();
                __syncwarp();
                if (lane == 0) {
                    if (whole)
                        tma_store_2d(tmD, buf, x0 + ch * xstep, y);
                    else   // stream-K part of an FP32 tile: add into D
                        tma_reduce_add_2d(tmD, buf, x0 + ch * xstep, y);
                    bulk_commit_group();
                }
            }
        }
    }
    // every store has written D before the CTA exits
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    k_fp8_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmD, const GemmParams p)
{
    extern __shared__ uint8_t smem_raw[];
    __shared__ Shared sh;
    // Operand tiles need 1024-byte alignment (128-byte swizzle atoms).  The
    // offset is the same in both CTAs of a pair, as the pair MMA requires.
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* smem = smem_raw + (((raw + 1023u) & ~1023u) - raw);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int64_t nnb = (p.N + BN - 1) / BN;
    const int64_t nkb = p.K / BK;
    const uint32_t rank = cluster_ctarank();

    if (threadIdx.x == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(&sh.full[s], 1);
            mbar_init(&sh.empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&sh.tfull[b], 1);
            // a TMEM buffer is released by the promotion warps of both CTAs
            mbar_init(&sh.tempty[b], 2 * NUM_PROMO_WARPS);
        }
        mbar_init(&sh.drain, 1);
        sh.abort = 0;
        sh.bad = 0;
        fence_barrier_init();
        tma_prefetch_desc(&tmA);
        tma_prefetch_desc(&tmB);
        tma_prefetch_desc(&tmD);
    }
    if (warp == 1) {
        tmem_alloc_pair(&sh.tmem_base, TMEM_COLS);
        tmem_relinquish_pair();
    }
    if (p.group_offsets)
        for (int i = threadIdx.x; i <= p.G; i += NUM_THREADS) sh.off[i] = p.group_offsets[i];
    // Barrier inits and the TMEM address must be visible to the peer CTA
    // before any of its loads, commits or arrives target them.
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    if (p.group_offsets && threadIdx.x == 0) {
        bool bad = sh.off[0] != 0 || (int64_t)sh.off[p.G] > p.M;
        for (int e = 0; e < p.G; ++e)
            bad = bad || sh.off[e + 1] < sh.off[e] || (sh.off[e + 1] & 127);
        if (bad) {
            sh.bad = 1;
            if (blockIdx.x == 0) report_error(FP8_ERR_SHAPE);
        }
    }
    __syncthreads();
    if (p.group_offsets && !sh.bad && warp == 0) pair_block_offsets(sh.off, sh.poff, p.G, lane);
    __syncthreads();
    const int64_t nmb = p.group_offsets ? (int64_t)sh.poff[p.G] : (p.M + TILE_M - 1) / TILE_M;

    if (warp < FIRST_PROMO_WARP) {
        regs_dec<CTRL_REGS>();
        if (!sh.bad) {
            if (warp == 0) {
                run_producer(&tmA, &tmB, p, smem, sh, nmb, nnb, nkb, lane);
                __syncwarp();
            } else if (warp == 1 && rank == 0) {   // a pair's MMAs issue from the even CTA
                if (lane == 0) run_mma(p, smem, sh, nmb, nnb, nkb);
                __syncwarp();
            }
        }
    } else {
        regs_inc<PROMO_REGS>();
        if (!sh.bad) {
            if (p.sb_gran == 128)
                run_promotion<128>(&tmD, p, sh, (int)nmb, (int)nnb, (int)nkb, warp, lane);
            else
                run_promotion<1>(&tmD, p, sh, (int)nmb, (int)nnb, (int)nkb, warp, lane);
        }
    }
    tc_fence_before();
    cluster_sync();
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(sh.tmem_base, TMEM_COLS);
}

__global__ void k_selftest_wait(uint64_t timeout_ns)
{
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    // Nothing ever arrives on `bar`: the wait runs into its time limit.
    if (threadIdx.x == 0) mbar_wait(&bar, 0, &abort_flag, timeout_ns);
}

// ------------------------------------------------------------------ host side

cudaLaunchConfig_t pair_launch_config(unsigned clusters, cudaStream_t st, cudaLaunchAttribute* attr)
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

// Once per device: opt the kernel into the large dynamic shared memory and
// ask how many CTA pairs fit at once (the persistent grid).
struct GemmDeviceSetup {
    bool ok = false;
    int pair_clusters = 0;
};

GemmDeviceSetup gemm_device_setup()
{
    static GemmDeviceSetup done[64];
    static bool tried[64] = {};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return GemmDeviceSetup{};
    std::lock_guard<std::mutex> lk(mu);
    if (!tried[dev]) {
        tried[dev] = true;
        GemmDeviceSetup r;
        r.ok = cudaFuncSetAttribute(k_fp8_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    (int)DYN_SMEM) == cudaSuccess;
        if (r.ok) {
            cudaLaunchAttribute attr[1];
            const cudaLaunchConfig_t cfg =
                pair_launch_config((unsigned)device_sm_count(), nullptr, attr);
            int n = 0;
            if (cudaOccupancyMaxActiveClusters(&n, k_fp8_gemm, &cfg) != cudaSuccess) {
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

}  // namespace

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(f);
    });
    return fn;
}

// 2-D uint8 tensor [outer][inner] with rows `row_bytes` apart; boxes of
// box_inner x box_outer bytes, 128-byte swizzle (or none), zero fill out of
// bounds.
bool make_map(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer,
              uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, bool swizzle128)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              swizzle128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_typed(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, uint64_t inner,
                    uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn) return false;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

// Zero the tiles that stream-K splits between two pairs (the tile holding
// the first unit of each pair's range, when that unit is not a tile's
// first): their two parts are added into D.  CTA c handles pair c's tile,
// 256 threads over its 256 rows x 256 FP32 columns (clipped to M and N).
__global__ void __launch_bounds__(256) k_zero_split_tiles(float* __restrict__ D, int64_t ldd,
                                                          int64_t M, int64_t N, int64_t nmb,
                                                          int64_t nnb, int64_t nkb, int64_t pairs,
                                                          int band)
{
    const int64_t units = nmb * nnb * nkb;
    const int64_t u = (int64_t)blockIdx.x * units / pairs;
    if (blockIdx.x == 0 || u % nkb == 0) return;
    int64_t mb, nb;
    gemm_tile_coord(u / nkb, nmb, nnb, band, mb, nb);
    const int64_t r0 = mb * TILE_M, c0 = nb * BN;
    const int64_t rows = M - r0 < TILE_M ? M - r0 : TILE_M;
    const int64_t cols = N - c0 < BN ? N - c0 : BN;
    for (int64_t i = threadIdx.x; i < rows * (cols / 4); i += blockDim.x) {
        const int64_t r = i / (cols / 4), c = (i % (cols / 4)) * 4;
        *reinterpret_cast<float4*>(D + (r0 + r) * ldd + c0 + c) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
}

// row_map != nullptr: gathered A (grouped GEMMs), A [a_rows][K] read row by
// row through row_map[M]; sA [K/128][a_rows].
int launch_gemm(const uint8_t* A, const float* sA, const uint8_t* B, int b_major, const float* sB,
                int sb_gran, int64_t M, int64_t N, int64_t K, const int32_t* group_offsets, int G,
                void* D, int out_dtype, int64_t ldd, int withhold, const int32_t* row_map,
                int64_t a_rows, cudaStream_t st)
{
    if (M == 0) return FP8_OK;
    const GemmDeviceSetup setup = gemm_device_setup();
    if (!setup.ok) return FP8_ERR_LAUNCH;
    if (setup.pair_clusters < 1) return FP8_ERR_DEVICE;   // needs co-scheduled 2-CTA clusters
    CUtensorMap tmA, tmB;
    // gathered A: boxes one row high, four rows per gather
    if (!(row_map ? make_map(&tmA, A, (uint64_t)K, (uint64_t)a_rows, (uint64_t)K, BK, 1)
                  : make_map(&tmA, A, (uint64_t)K, (uint64_t)M, (uint64_t)K, BK, BM)))
        return FP8_ERR_LAUNCH;
    bool okB;
    if (b_major == FP8_B_KMAJOR) {
        const uint64_t rows = (uint64_t)N * (uint64_t)(group_offsets ? G : 1);
        okB = make_map(&tmB, B, (uint64_t)K, rows, (uint64_t)K, BK, 128);
    } else {
        okB = make_map(&tmB, B, (uint64_t)N, (uint64_t)K, (uint64_t)N, 128, BK);
    }
    if (!okB) return FP8_ERR_LAUNCH;
    // D in its element type, rows `ldd` elements apart; the epilogue stores
    // boxes of 32 bytes x 32 rows
    CUtensorMap tmD;
    const bool bf16 = out_dtype == FP8_OUT_BF16;
    const uint32_t esz = bf16 ? 2 : 4;
    if (!make_map_typed(&tmD, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32,
                        D, (uint64_t)N, (uint64_t)M, (uint64_t)ldd * esz, EPI_BYTES / esz, EPI_ROWS))
        return FP8_ERR_LAUNCH;
    GemmParams p;
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
    p.row_map = row_map;
    p.a_rows = row_map ? a_rows : M;
    p.band = group_offsets ? BAND_GROUPED : BAND_DENSE;
    p.timeout_ns = wait_timeout_ns();
    // grouped: each group adds at most one partly idle 256-row block
    const int64_t nnb = (N + BN - 1) / BN, nkb = K / BK;
    const int64_t tiles = ((M + 255) / 256 + (group_offsets ? G : 0)) * nnb;
    const int64_t clusters = tiles < setup.pair_clusters ? tiles : setup.pair_clusters;
    // Stream-K for dense FP32 outputs whose tiles fill the last round of the
    // pairs badly (the parts of a split tile are added exactly: two FP32
    // sums onto zero, in either order, give the same result).  Each pair's
    // range must hold at least a whole tile, so that no tile has more than
    // two contributors.
    const int64_t rounds = (tiles + clusters - 1) / clusters;
    p.streamk = !bf16 && !group_offsets && tiles > clusters && tiles % clusters != 0 &&
                (double)rounds * clusters / (double)tiles > 1.05 && tiles * nkb / clusters >= nkb;
    if (p.streamk) {
        const int64_t nmb = (M + TILE_M - 1) / TILE_M;
        k_zero_split_tiles<<<(unsigned)clusters, 256, 0, st>>>(static_cast<float*>(D), ldd, M, N,
                                                              nmb, nnb, nkb, clusters, p.band);
        if (cudaGetLastError() != cudaSuccess) return FP8_ERR_LAUNCH;
    }
    cudaLaunchAttribute attr[1];
    const cudaLaunchConfig_t cfg = pair_launch_config((unsigned)clusters, st, attr);
    return cudaLaunchKernelEx(&cfg, k_fp8_gemm, tmA, tmB, tmD, p) == cudaSuccess ? FP8_OK
                                                                                  : FP8_ERR_LAUNCH;
}

}  // namespace

int launch_blockscaled_gemm(const uint8_t* A, const float* sA, const uint8_t* B, int b_major,
                            const float* sB, int sb_gran, int64_t M, int64_t N, int64_t K,
                            const int32_t* group_offsets, int G, void* D, int out_dtype,
                            int64_t ldd, cudaStream_t st)
{
    return launch_gemm(A, sA, B, b_major, sB, sb_gran, M, N, K, group_offsets, G, D, out_dtype,
                       ldd, 0, nullptr, 0, st);
}

int launch_grouped_gemm_gather(const uint8_t* A, const float* sA, int64_t a_rows,
                               const int32_t* row_map, const uint8_t* B, const float* sB,
                               const int32_t* group_offsets, int G, int64_t M, int64_t N, int64_t K,
                               void* D, int out_dtype, cudaStream_t st)
{
    return launch_gemm(A, sA, B, FP8_B_KMAJOR, sB, 128, M, N, K, group_offsets, G, D, out_dtype, N,
                       0, row_map, a_rows, st);
}

int launch_blockscaled_gemm_withheld(const uint8_t* A, const float* sA, const uint8_t* B,
                                     int b_major, const float* sB, int sb_gran, int64_t M,
                                     int64_t N, int64_t K, const int32_t* group_offsets, int G,
                                     void* D, int out_dtype, int64_t ldd, cudaStream_t st)
{
    return launch_gemm(A, sA, B, b_major, sB, sb_gran, M, N, K, group_offsets, G, D, out_dtype,
                       ldd, 1, nullptr, 0, st);
}

cudaError_t launch_selftest_wait(cudaStream_t st)
{
    k_selftest_wait<<<1, 32, 0, st>>>(wait_timeout_ns());
    return cudaGetLastError();
}

// Synchronise, then read and clear this module's status word on the current
// device.
int read_and_clear_status(cudaStream_t st)
{
    if (cudaStreamSynchronize(st) != cudaSuccess) return FP8_ERR_DEVICE;
    return read_and_clear_module_status();
}

}  // namespace fp8fg
