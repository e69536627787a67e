// quant.cu -- online E4M3 quantizers of the fine-grained FP8 Linear (sm_100a).
//
// Three HBM-bound kernels, one per grouping of the DeepSeek-V3 FP8 recipe
// (pages: why-be.co.kr post, cameseeing.com post and "Three Fast Methods To
// Study Deepseek", Figure 7 (a); "5 Ways You can get More Deepseek While
// Spending Less", max-abs -> FP8 maximum and power-of-2 scales):
//   k_quant_1x128    one scale per token per 128 channels
//   k_quant_128x1    one scale per channel per 128 tokens, written transposed
//   k_quant_w128     one scale per 128x128 weight block
//   k_requant_128x1  cached 1x128 codes -> dequantize -> 128x1 groups (Wgrad)
// Each reads its input once with 16-byte vector loads, reduces the group's
// max-abs with warp shuffles (plus shared memory for the wider groups),
// derives the scale with correctly rounded FP32 division, and writes packed
// E4M3 codes (cvt.rn.satfinite.e4m3x2) with 8- or 16-byte stores.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "fp8fg_device.cuh"
#include "fp8fg_host.h"

namespace fp8fg {

namespace {

// ------------------------------------------------------------ group scale

struct GroupScale {
    float s;    // stored scale (dequantisation multiplier)
    float inv;  // factor applied before the E4M3 cast
};

// Scale of a group with max-abs `amax` (amax >= 0, finite).
//   FP32 mode: s = amax/448, inv = 448/amax, both correctly rounded; a zero
//              group gets s = inv = 1; when amax/448 would fall below the
//              smallest normal FP32 the scale saturates at 2^-126.
//   POW2 mode: s = 2^e, e least with amax <= 448*2^e, e >= -126; inv = 2^-e.
__device__ __forceinline__ GroupScale group_scale(float amax, int mode)
{
    GroupScale g;
    if (amax == 0.0f) {
        g.s = 1.0f;
        g.inv = 1.0f;
        return g;
    }
    if (mode == FP8_SCALE_POW2) {
        const uint32_t b = __float_as_uint(amax);
        const int ex = (int)((b >> 23) & 0xFF);
        int e = -126;
        if (ex != 0) {
            // amax = m * 2^(ex-127), m in [1,2).  448 = 1.75 * 2^8, so the
            // least e is ex-127-8 when m <= 1.75 and one more otherwise.
            e = ex - 127 - 8 + (((b & 0x7FFFFFu) > 0x600000u) ? 1 : 0);
            if (e < -126) e = -126;
        }
        g.s = __uint_as_float((uint32_t)(e + 127) << 23);
        g.inv = __uint_as_float((uint32_t)(127 - e) << 23);
        return g;
    }
    if (amax < __uint_as_float(0x04E00000u)) {        // 1.75 * 2^-118
        g.s = __uint_as_float(0x00800000u);            // 2^-126
        g.inv = __uint_as_float(0x7E800000u);          // 2^126
        return g;
    }
    g.inv = __fdiv_rn(448.0f, amax);
    g.s = __fdiv_rn(amax, 448.0f);
    return g;
}

// Four scaled values -> four E4M3 codes packed little-endian in a uint32:
// byte i = E4M3(fl32(x_i * inv)), round to nearest even, saturating to
// +-448.  The products are two packed FP32x2 multiplies (each lane rounded
// to nearest like a scalar multiply); each cvt packs two codes, its first
// source going to the upper byte.
__device__ __forceinline__ uint32_t encode4(float a, float b, float c, float d, float inv)
{
    float a2, b2, c2, d2;
    fmul2(a2, b2, a, b, inv, inv);
    fmul2(c2, d2, c, d, inv, inv);
    uint32_t r;
    asm("{\n\t.reg .b16 lo, hi;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 lo, %2, %1;\n\t"
        "cvt.rn.satfinite.e4m3x2.f32 hi, %4, %3;\n\t"
        "mov.b32 %0, {lo, hi};\n\t}"
        : "=r"(r)
        : "f"(a2), "f"(b2), "f"(c2), "f"(d2));
    return r;
}

// ------------------------------------------------------------ vector loads

__device__ __forceinline__ uint4 ld_stream16(const void* p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Eight consecutive input elements held as raw bits (16 B of BF16 or 32 B of
// FP32) until they are needed as floats.
template <typename Tin>
struct Chunk8;

template <>
struct Chunk8<__nv_bfloat16> {
    uint4 r;
    __device__ __forceinline__ void load(const __nv_bfloat16* p) { r = ld_stream16(p); }
    __device__ __forceinline__ void zero() { r = make_uint4(0, 0, 0, 0); }
    __device__ __forceinline__ void get(float (&v)[8]) const
    {
        v[0] = bf16_lo(r.x); v[1] = bf16_hi(r.x); v[2] = bf16_lo(r.y); v[3] = bf16_hi(r.y);
        v[4] = bf16_lo(r.z); v[5] = bf16_hi(r.z); v[6] = bf16_lo(r.w); v[7] = bf16_hi(r.w);
    }
};

template <>
struct Chunk8<float> {
    uint4 a, b;
    __device__ __forceinline__ void load(const float* p)
    {
        a = ld_stream16(p);
        b = ld_stream16(p + 4);
    }
    __device__ __forceinline__ void zero() { a = b = make_uint4(0, 0, 0, 0); }
    __device__ __forceinline__ void get(float (&v)[8]) const
    {
        v[0] = __uint_as_float(a.x); v[1] = __uint_as_float(a.y);
        v[2] = __uint_as_float(a.z); v[3] = __uint_as_float(a.w);
        v[4] = __uint_as_float(b.x); v[5] = __uint_as_float(b.y);
        v[6] = __uint_as_float(b.z); v[7] = __uint_as_float(b.w);
    }
};

__device__ __forceinline__ float absmax8(const float (&v)[8])
{
    float a = fabsf(v[0]);
#pragma unroll
    for (int i = 1; i < 8; ++i) a = fmaxf(a, fabsf(v[i]));
    return a;
}

// ------------------------------------------------------------ 1x128

constexpr int kGroupsPerThread1x128 = 8;
constexpr int kRowsPerCta1x128 = 16 * kGroupsPerThread1x128;   // 128

// CTA = 256 threads = 16 half-warps; a half-warp owns one 1x128 group at a
// time (16 lanes x 8 elements); each thread keeps 8 groups' loads (128 B) in
// flight before reducing any of them.
// Grid: x = K/128 K-blocks (adjacent CTAs read adjacent 256-byte segments of
// the same rows), y = ceil(M/128) row blocks.
template <typename Tin>
__global__ void __launch_bounds__(256) k_quant_1x128(const Tin* __restrict__ x, int64_t M,
                                                     int64_t ldx, uint8_t* __restrict__ q,
                                                     int64_t ldq, float* __restrict__ sA, int mode)
{
    const int h = threadIdx.x >> 4;
    const int l = threadIdx.x & 15;
    const int64_t kb = blockIdx.x;
    const int64_t m0 = (int64_t)blockIdx.y * kRowsPerCta1x128;

    Chunk8<Tin> c[kGroupsPerThread1x128];
#pragma unroll
    for (int u = 0; u < kGroupsPerThread1x128; ++u) {
        const int64_t m = m0 + u * 16 + h;
        if (m < M)
            c[u].load(x + m * ldx + kb * 128 + l * 8);
        else
            c[u].zero();
    }
#pragma unroll
    for (int u = 0; u < kGroupsPerThread1x128; ++u) {
        const int64_t m = m0 + u * 16 + h;
        float v[8];
        c[u].get(v);
        float a = absmax8(v);
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 8));
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 4));
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
        const GroupScale g = group_scale(a, mode);
        if (m < M) {
            uint2 out;
            out.x = encode4(v[0], v[1], v[2], v[3], g.inv);
            out.y = encode4(v[4], v[5], v[6], v[7], g.inv);
            *reinterpret_cast<uint2*>(q + m * ldq + kb * 128 + l * 8) = out;
            if (l == 0) sA[kb * M + m] = g.s;
        }
    }
}

// 1x128 quantization straight into the MoE dispatch layout: the same groups,
// scales and codes as k_quant_1x128, but each token's codes and scales are
// written to every destination row its routing gave it (token_row[t][j],
// j < k; -1 means the pair was dropped) instead of to the token's own row.
// The token's codes never round-trip through HBM before the dispatch.
//
// A half-warp owns one token and two adjacent K-blocks (256 elements): lane l
// holds elements 16l .. 16l+15, so lanes 0-7 form the first 1x128 group and
// lanes 8-15 the second (max-abs over 8 lanes each), and every destination
// row gets one 16-byte store per lane, 256 contiguous bytes per half-warp.
// Lanes 0..k-1 fetch the token's destinations; full-warp shuffles (both
// half-warps walk the same j) hand them to all lanes, and the stores are
// predicated on the row being valid, so the walk never diverges.
// CTA = 256 threads = 16 half-warps x 4 tokens each (64 tokens).
// Grid: x = ceil(K/256) K-block pairs, y = ceil(T/64).
constexpr int kTokPerHalfWarpDispatch = 4;
constexpr int kTokPerCtaDispatch = 16 * kTokPerHalfWarpDispatch;   // 64

template <typename Tin>
__global__ void __launch_bounds__(256) k_quant_1x128_dispatch(
    const Tin* __restrict__ x, int64_t T, int64_t ldx, const int32_t* __restrict__ token_row,
    int k, int64_t M_cap, uint8_t* __restrict__ q_out, int64_t K, float* __restrict__ sA_out,
    int mode)
{
    const int h = threadIdx.x >> 4;
    const int l = threadIdx.x & 15;
    const int half = threadIdx.x & 16;              // lane offset of this half-warp
    const int64_t kb = (int64_t)blockIdx.x * 2 + (l >> 3);   // this lane's K-block
    const bool kb_ok = kb < K / 128;                 // an odd K/128 leaves the last pair half empty
    const int64_t col = kb * 128 + (l & 7) * 16;     // this lane's first element / code byte
    const int64_t t0 = (int64_t)blockIdx.y * kTokPerCtaDispatch;
    uint8_t* const q_col = q_out + col;
    float* const s_col = sA_out + kb * M_cap;

    Chunk8<Tin> c[kTokPerHalfWarpDispatch][2];
#pragma unroll
    for (int u = 0; u < kTokPerHalfWarpDispatch; ++u) {
        const int64_t t = t0 + u * 16 + h;
        if (t < T && kb_ok) {
            c[u][0].load(x + t * ldx + col);
            c[u][1].load(x + t * ldx + col + 8);
        } else {
            c[u][0].zero();
            c[u][1].zero();
        }
    }
#pragma unroll
    for (int u = 0; u < kTokPerHalfWarpDispatch; ++u) {
        const int64_t t = t0 + u * 16 + h;
        float v0[8], v1[8];
        c[u][0].get(v0);
        c[u][1].get(v1);
        float a = fmaxf(absmax8(v0), absmax8(v1));
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 4));
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 2));
        a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
        const GroupScale g = group_scale(a, mode);
        uint4 out;
        out.x = encode4(v0[0], v0[1], v0[2], v0[3], g.inv);
        out.y = encode4(v0[4], v0[5], v0[6], v0[7], g.inv);
        out.z = encode4(v1[0], v1[1], v1[2], v1[3], g.inv);
        out.w = encode4(v1[4], v1[5], v1[6], v1[7], g.inv);
        const bool live = t < T;
        for (int j0 = 0; j0 < k; j0 += 16) {
            const int32_t mine = (live && j0 + l < k) ? __ldg(token_row + t * k + j0 + l) : -1;
            const int nj = k - j0 < 16 ? k - j0 : 16;
            for (int j = 0; j < nj; ++j) {
                const int32_t r = __shfl_sync(0xffffffffu, mine, half + j);
                if (r >= 0 && r < M_cap && kb_ok) {
                    *reinterpret_cast<uint4*>(q_col + (int64_t)r * K) = out;
                    if ((l & 7) == 0) s_col[r] = g.s;
                }
            }
        }
    }
}

// ------------------------------------------------------------ 128x128

// CTA = 256 threads per 128x128 block: thread (r0 = tid/16, c = tid%16) loads
// rows r0 + 16 i (i < 8), elements c*8 .. c*8+7 of the block's row segment.
// Grid: x = K/128, y = N/128.
template <typename Tin>
__global__ void __launch_bounds__(256) k_quant_w128(const Tin* __restrict__ w, int64_t ldw,
                                                    uint8_t* __restrict__ q, int64_t ldq,
                                                    float* __restrict__ sW, int64_t nkb, int mode)
{
    __shared__ float red[8];
    const int c = threadIdx.x & 15;
    const int r0 = threadIdx.x >> 4;
    const int64_t kb = blockIdx.x;
    const int64_t nb = blockIdx.y;
    const Tin* base = w + (nb * 128 + r0) * ldw + kb * 128 + c * 8;

    Chunk8<Tin> ch[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) ch[i].load(base + (int64_t)(16 * i) * ldw);

    float a = 0.0f;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float v[8];
        ch[i].get(v);
        a = fmaxf(a, absmax8(v));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = a;
    __syncthreads();
    a = red[0];
#pragma unroll
    for (int i = 1; i < 8; ++i) a = fmaxf(a, red[i]);
    const GroupScale g = group_scale(a, mode);

    uint8_t* qb = q + (nb * 128 + r0) * ldq + kb * 128 + c * 8;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        float v[8];
        ch[i].get(v);
        uint2 out;
        out.x = encode4(v[0], v[1], v[2], v[3], g.inv);
        out.y = encode4(v[4], v[5], v[6], v[7], g.inv);
        *reinterpret_cast<uint2*>(qb + (int64_t)(16 * i) * ldq) = out;
    }
    if (threadIdx.x == 0) sW[nb * nkb + kb] = g.s;
}

// ------------------------------------------------------------ 128x1

constexpr int kTok = 128;        // tokens per tile (one group along tokens)
constexpr int kThr128x1 = 256;
constexpr int kTiles128x1 = 4;   // token blocks per CTA, double-buffered
// Tile geometry per input type: 128-byte row segments (64 BF16 or 32 FP32
// channels), threads own channel pairs x (kTok / kGroups) tokens.  (256-byte
// segments with 512 threads measured slower.)
template <typename Tin>
struct Geo128x1 {
    static constexpr int kCh = 128 / (int)sizeof(Tin);
    static constexpr int kPairs = kCh / 2;
    static constexpr int kGroups = kThr128x1 / kPairs;   // 8 (BF16) or 16 (FP32)
    static constexpr int kTokPerThr = kTok / kGroups;    // 16 (BF16) or 8 (FP32)
    static_assert(kTokPerThr == 16 || kTokPerThr == 8, "16- or 8-byte code stores");
};

// CTA = 256 threads per tile of 128 tokens x 128 bytes of channels (64 BF16
// or 32 FP32 channels).  The tile is staged
// in shared memory with register-free 16-byte cp.async copies (coalesced row
// segments), so registers do not limit how many tiles are in flight per SM.
// Thread (p = tid % kPairs, g = tid / kPairs) then owns channels 2p, 2p+1 and
// kTokPerThr tokens starting at g * kTokPerThr, read as two-channel words (a
// warp reads 128 or 256 contiguous bytes of one row per load, conflict-free):
// a first pass takes the max-abs, the token groups combine theirs through
// shared memory, and a second pass encodes the thread's tokens of each
// channel into one 16- or 8-byte store per channel of the transposed output.
// Each CTA walks kTiles128x1 consecutive token blocks of its channel
// slice, loading the next block (cp.async, double buffered) while it
// processes the current one.
// Grid: x = ceil(C / kCh), y = ceil(T/128 / kTiles128x1).
template <typename Tin>
struct Pair;
template <>
struct Pair<__nv_bfloat16> {
    // two adjacent bf16 channels of one token as one 32-bit word
    static __device__ __forceinline__ float2 get(const __nv_bfloat16* p)
    {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(p);
        return make_float2(bf16_lo(w), bf16_hi(w));
    }
};
template <>
struct Pair<float> {
    static __device__ __forceinline__ float2 get(const float* p) { return *reinterpret_cast<const float2*>(p); }
};

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc)
                 : "memory");
}
__device__ __forceinline__ void cp_async4(void* smem_dst, const void* gsrc)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem_dst)), "l"(gsrc)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_group()
{
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}


template <typename Tin>
__global__ void __launch_bounds__(kThr128x1, 5) k_quant_128x1(const Tin* __restrict__ x, int64_t ntb,
                                                              int64_t C, int64_t ldx,
                                                              uint8_t* __restrict__ qT, int64_t ldqT,
                                                              float* __restrict__ s, int mode)
{
    using G = Geo128x1<Tin>;
    constexpr int kElemsPerChunk = 16 / (int)sizeof(Tin);
    constexpr int kChunksPerRow = G::kCh / kElemsPerChunk;           // 8
    constexpr int kChunksPerThread = kTok * kChunksPerRow / kThr128x1;   // 4
    __shared__ __align__(16) Tin tile[2][kTok][G::kCh];
    __shared__ float2 part[G::kGroups][G::kPairs];
    // transposed codes of one token block: kCh rows of 128 bytes, 16-byte
    // chunks XOR-swizzled by row so both the scattered writes and the row
    // reads are conflict-free
    __shared__ __align__(16) uint8_t outT[G::kCh][kTok];

    const int64_t c0 = (int64_t)blockIdx.x * G::kCh;
    const int64_t tb0 = (int64_t)blockIdx.y * kTiles128x1;
    const int64_t tb_end = ntb < tb0 + kTiles128x1 ? ntb : tb0 + kTiles128x1;

    // stage token block tb into buffer buf (channels beyond C are zero; C % 8 == 0)
    auto stage = [&](int64_t tb, int buf) {
#pragma unroll
        for (int i = 0; i < kChunksPerThread; ++i) {
            const int id = threadIdx.x + kThr128x1 * i;
            const int r = id / kChunksPerRow;
            const int j = id % kChunksPerRow;
            const int64_t ch = c0 + j * kElemsPerChunk;
            if (ch < C)
                cp_async16(&tile[buf][r][j * kElemsPerChunk], x + (tb * kTok + r) * ldx + ch);
            else
                *reinterpret_cast<uint4*>(&tile[buf][r][j * kElemsPerChunk]) = make_uint4(0, 0, 0, 0);
        }
    };

    const int pch = threadIdx.x % G::kPairs;
    const int g = threadIdx.x / G::kPairs;
    const int t0 = g * G::kTokPerThr;
    const int64_t ch = c0 + 2 * pch;

    stage(tb0, 0);
    cp_async_commit();
    for (int jt = 0; jt < kTiles128x1; ++jt) {
        const int64_t tb = tb0 + jt;
        if (tb >= tb_end) break;                       // block-uniform
        const int buf = jt & 1;
        if (tb + 1 < tb_end) stage(tb + 1, buf ^ 1);   // its buffer was freed by tile jt - 1
        cp_async_commit();
        cp_async_wait_group<1>();                      // tile jt has landed
        __syncthreads();

        // max-abs of channels 2p, 2p+1 over this thread's tokens, then over groups
        float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
        for (int t = 0; t < G::kTokPerThr; ++t) {
            const float2 v = Pair<Tin>::get(&tile[buf][t0 + t][2 * pch]);
            a0 = fmaxf(a0, fabsf(v.x));
            a1 = fmaxf(a1, fabsf(v.y));
        }
        part[g][pch] = make_float2(a0, a1);
        __syncthreads();
#pragma unroll
        for (int i = 0; i < G::kGroups; ++i) {
            const float2 q = part[i][pch];
            a0 = fmaxf(a0, q.x);
            a1 = fmaxf(a1, q.y);
        }
        const GroupScale g0 = group_scale(a0, mode);
        const GroupScale g1 = group_scale(a1, mode);

        // encode this thread's tokens of channels 2p, 2p+1 into the transposed
        // tile (byte offset t0 of rows 2p and 2p+1, chunk-swizzled)
        {
            uint32_t w0[G::kTokPerThr / 4], w1[G::kTokPerThr / 4];
#pragma unroll
            for (int q4 = 0; q4 < G::kTokPerThr / 4; ++q4) {
                float2 v[4];
#pragma unroll
                for (int t = 0; t < 4; ++t) v[t] = Pair<Tin>::get(&tile[buf][t0 + q4 * 4 + t][2 * pch]);
                w0[q4] = encode4(v[0].x, v[1].x, v[2].x, v[3].x, g0.inv);
                w1[q4] = encode4(v[0].y, v[1].y, v[2].y, v[3].y, g1.inv);
            }
            const int r0 = 2 * pch, r1 = 2 * pch + 1;
            const int off0 = (t0 ^ ((r0 & 7) << 4)), off1 = (t0 ^ ((r1 & 7) << 4));
            if constexpr (G::kTokPerThr == 16) {
                *reinterpret_cast<uint4*>(&outT[r0][off0]) = make_uint4(w0[0], w0[1], w0[2], w0[3]);
                *reinterpret_cast<uint4*>(&outT[r1][off1]) = make_uint4(w1[0], w1[1], w1[2], w1[3]);
            } else {
                *reinterpret_cast<uint2*>(&outT[r0][off0]) = make_uint2(w0[0], w0[1]);
                *reinterpret_cast<uint2*>(&outT[r1][off1]) = make_uint2(w1[0], w1[1]);
            }
            if (g == 0 && ch < C) {   // s is only guaranteed 4-byte aligned: two scalar stores
                s[tb * C + ch] = g0.s;
                s[tb * C + ch + 1] = g1.s;
            }
        }
        __syncthreads();
        // whole 128-byte rows of qT: 8 threads per row, 16 bytes each
        for (int id = threadIdx.x; id < G::kCh * 8; id += kThr128x1) {
            const int r = id >> 3, c16 = id & 7;
            const int64_t chr = c0 + r;
            if (chr < C) {
                const uint4 v = *reinterpret_cast<const uint4*>(&outT[r][(c16 << 4) ^ ((r & 7) << 4)]);
                *reinterpret_cast<uint4*>(qT + chr * ldqT + tb * kTok + (c16 << 4)) = v;
            }
        }
        __syncthreads();   // the buffers may be rewritten by the next tile
    }
    cp_async_wait_group<0>();
}

// ------------------------------------------------------------ requantize 1x128 -> 128x1

// Activations cached as 1x128 E4M3 tiles (the forward pass's quantized X)
// regrouped for the Wgrad GEMM: every code is dequantized to
// fl32(decode(q) * sA) -- E4M3 -> FP16 -> FP32 is exact, so one FP32
// multiply gives that single rounding -- and the FP32 values are quantized in 128x1 groups
// along tokens, exactly as k_quant_128x1 quantizes an FP32 input.
//
// CTA = 256 threads over kReqTiles consecutive tiles of 128 tokens x 128
// channels (one channel block, hence one cached scale per token), with the
// next tile's 16 KB of codes and 128 scales loading (cp.async, double
// buffered) while the current one is processed.  Per tile, warp w owns
// tokens 16w .. 16w+15 and lane l channels 4l .. 4l+3, read as one 32-bit
// word per token (a warp reads a whole 128-byte row, conflict-free).
// Pass 1: dequantize once (the 64 products stay in registers) and take the
// max-abs, combined over the 8 warps through shared memory, where thread c
// (c < 128) derives channel c's scale once for the CTA.  Pass 2: each
// thread encodes its 16 tokens of each of its 4 channels into one 16-byte
// word.  The transposed codes go into their own buffer (16-byte chunks
// XOR-swizzled by (channel / 4) % 8, conflict-free) and leave as coalesced
// 128-byte rows of qT; with the staged codes in separate buffers, a tile
// needs four block barriers, none at its end.
// Grid: x = C/128, y = ceil(T/128 / kReqTiles).
constexpr int kReqTok = 128;
constexpr int kReqCh = 128;
constexpr int kReqTiles = 4;

// Four E4M3 codes (little-endian in w) -> their exact values: each pair of
// codes widens to FP16x2 (exact: E4M3 is a subset of FP16), each FP16 to FP32.
__device__ __forceinline__ void decode4_e4m3(uint32_t w, float (&f)[4])
{
    asm("{\n\t.reg .b16 q0, q1, h0, h1, h2, h3;\n\t.reg .b32 p0, p1;\n\t"
        "mov.b32 {q0, q1}, %4;\n\t"
        "cvt.rn.f16x2.e4m3x2 p0, q0;\n\t"
        "cvt.rn.f16x2.e4m3x2 p1, q1;\n\t"
        "mov.b32 {h0, h1}, p0;\n\t"
        "mov.b32 {h2, h3}, p1;\n\t"
        "cvt.f32.f16 %0, h0;\n\t"
        "cvt.f32.f16 %1, h1;\n\t"
        "cvt.f32.f16 %2, h2;\n\t"
        "cvt.f32.f16 %3, h3;\n\t}"
        : "=f"(f[0]), "=f"(f[1]), "=f"(f[2]), "=f"(f[3])
        : "r"(w));
}

struct __align__(16) ReqShared {
    uint8_t tile[2][kReqTok * kReqCh];   // staged codes, double-buffered
    uint8_t outT[kReqCh * kReqTok];      // the current tile's transposed codes
    float part[8][kReqCh];               // per-warp max-abs of each channel
    float inv_s[kReqCh];                 // per-channel encode factors of the tile
    float scl[2][kReqTok];               // staged 1x128 scales of the tile's tokens
};
constexpr uint32_t kReqSmemBytes = (uint32_t)sizeof(ReqShared);

__global__ void __launch_bounds__(256, 3) k_requant_128x1(const uint8_t* __restrict__ q, int64_t ldq,
                                                       const float* __restrict__ sA, int64_t T,
                                                       int64_t C, uint8_t* __restrict__ qT,
                                                       int64_t ldqT, float* __restrict__ s, int mode)
{
    extern __shared__ __align__(16) uint8_t req_raw[];
    ReqShared& sh = *reinterpret_cast<ReqShared*>(req_raw);
    auto& tile = sh.tile;
    auto& part = sh.part;
    auto& inv_s = sh.inv_s;
    auto& scl = sh.scl;

    const int64_t cb = blockIdx.x;
    const int64_t c0 = cb * kReqCh;
    const int64_t ntb = T / kReqTok;
    const int64_t tb0 = (int64_t)blockIdx.y * kReqTiles;
    const int w = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    auto stage = [&](int64_t tb, int buf) {
        const int64_t t0 = tb * kReqTok;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int id = threadIdx.x + 256 * i;
            const int r = id >> 3, j = id & 7;
            cp_async16(&tile[buf][r * kReqCh + j * 16], q + (t0 + r) * ldq + c0 + j * 16);
        }
        if (threadIdx.x < kReqTok) cp_async4(&scl[buf][threadIdx.x], sA + cb * T + t0 + threadIdx.x);
    };

    stage(tb0, 0);
    cp_async_commit();
    for (int j = 0; j < kReqTiles; ++j) {
        const int64_t tb = tb0 + j;
        if (tb >= ntb) break;                          // block-uniform
        const int buf = j & 1;
        const bool more = j + 1 < kReqTiles && tb + 1 < ntb;
        if (more) stage(tb + 1, buf ^ 1);              // its buffer was freed by tile j - 1
        cp_async_commit();
        cp_async_wait_group<1>();                      // tile j's group has landed
        __syncthreads();

        // pass 1: dequantize this thread's 16 tokens x 4 channels once (kept in
        // registers for pass 2) and take their max-abs per channel
        const uint32_t* tw = reinterpret_cast<const uint32_t*>(tile[buf]);
        const float* sc_t = scl[buf];
        float v[16][4];
        float a[4] = {0.f, 0.f, 0.f, 0.f};
        // tokens are taken in pairs (i, i+1): one packed multiply scales the
        // same channel of both, the pairing the encode below uses as well
#pragma unroll
        for (int i = 0; i < 16; i += 2) {
            const int t = w * 16 + i;
            float f0[4], f1[4];
            decode4_e4m3(tw[t * (kReqCh / 4) + lane], f0);
            decode4_e4m3(tw[(t + 1) * (kReqCh / 4) + lane], f1);
            const float2 sc = *reinterpret_cast<const float2*>(&sc_t[t]);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                fmul2(v[i][k], v[i + 1][k], f0[k], f1[k], sc.x, sc.y);
                a[k] = fmaxf(a[k], fmaxf(fabsf(v[i][k]), fabsf(v[i + 1][k])));
            }
        }
        *reinterpret_cast<float4*>(&part[w][4 * lane]) = make_float4(a[0], a[1], a[2], a[3]);
        __syncthreads();
        if (threadIdx.x < kReqCh) {   // channel c = threadIdx.x: combine the warps, derive its scale
            const int c = threadIdx.x;
            float am = part[0][c];
#pragma unroll
            for (int k = 1; k < 8; ++k) am = fmaxf(am, part[k][c]);
            const GroupScale gs = group_scale(am, mode);
            inv_s[c] = gs.inv;
            s[tb * C + c0 + c] = gs.s;
        }
        __syncthreads();   // inv_s is ready
        const float4 inv4 = *reinterpret_cast<const float4*>(&inv_s[4 * lane]);
        const float inv[4] = {inv4.x, inv4.y, inv4.z, inv4.w};

        // pass 2: encode 16 tokens x 4 channels into four 16-byte words
        uint32_t out[4][4];
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
#pragma unroll
            for (int k = 0; k < 4; ++k)
                out[k][q4] = encode4(v[4 * q4][k], v[4 * q4 + 1][k], v[4 * q4 + 2][k], v[4 * q4 + 3][k],
                                     inv[k]);
        }
        uint8_t* tl = sh.outT;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int c = 4 * lane + k;
            const int chunk = w ^ (lane & 7);
            *reinterpret_cast<uint4*>(&tl[c * kReqTok + chunk * 16]) =
                make_uint4(out[k][0], out[k][1], out[k][2], out[k][3]);
        }
        __syncthreads();
        const int64_t t0 = tb * kReqTok;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int id = threadIdx.x + 256 * i;
            const int c = id >> 3, chunk = id & 7;
            const uint4 v = *reinterpret_cast<const uint4*>(&tl[c * kReqTok + ((chunk ^ ((c >> 2) & 7)) * 16)]);
            *reinterpret_cast<uint4*>(qT + (c0 + c) * ldqT + t0 + chunk * 16) = v;
        }
        // No barrier here.  The next tile's prefetch into this tile's staging
        // buffer comes after this tile's second barrier, which follows every
        // thread's reads of the staged codes and scales; the next tile's
        // writes of part, inv_s and outT come after the next tile's first
        // barrier, which every thread passes only after finishing this tile.
    }
    cp_async_wait_group<0>();
}

}  // namespace

// ------------------------------------------------------------ launchers

cudaError_t launch_quant_act_1x128(const void* x, int in_dtype, int64_t M, int64_t K, int64_t ldx,
                                   uint8_t* q, int64_t ldq, float* sA, int mode, cudaStream_t st)
{
    const dim3 grid((unsigned)(K / 128), (unsigned)((M + kRowsPerCta1x128 - 1) / kRowsPerCta1x128));
    if (in_dtype == FP8_IN_BF16)
        k_quant_1x128<__nv_bfloat16><<<grid, 256, 0, st>>>(
            static_cast<const __nv_bfloat16*>(x), M, ldx, q, ldq, sA, mode);
    else
        k_quant_1x128<float><<<grid, 256, 0, st>>>(static_cast<const float*>(x), M, ldx, q, ldq,
                                                   sA, mode);
    return cudaGetLastError();
}

cudaError_t launch_quant_act_1x128_dispatch(const void* x, int in_dtype, int64_t T, int64_t K,
                                            int64_t ldx, const int32_t* token_row, int k,
                                            int64_t M_cap, uint8_t* q_out, float* sA_out, int mode,
                                            cudaStream_t st)
{
    if (T == 0) return cudaSuccess;
    const dim3 grid((unsigned)((K / 128 + 1) / 2),
                    (unsigned)((T + kTokPerCtaDispatch - 1) / kTokPerCtaDispatch));
    if (in_dtype == FP8_IN_BF16)
        k_quant_1x128_dispatch<__nv_bfloat16><<<grid, 256, 0, st>>>(
            static_cast<const __nv_bfloat16*>(x), T, ldx, token_row, k, M_cap, q_out, K, sA_out,
            mode);
    else
        k_quant_1x128_dispatch<float><<<grid, 256, 0, st>>>(static_cast<const float*>(x), T, ldx,
                                                            token_row, k, M_cap, q_out, K, sA_out,
                                                            mode);
    return cudaGetLastError();
}

cudaError_t launch_quant_act_128x1(const void* x, int in_dtype, int64_t T, int64_t C, int64_t ldx,
                                   uint8_t* qT, int64_t ldqT, float* s, int mode, cudaStream_t st)
{
    const int ch_tile = in_dtype == FP8_IN_BF16 ? Geo128x1<__nv_bfloat16>::kCh : Geo128x1<float>::kCh;
    const int64_t ntb = T / kTok;
    const dim3 grid((unsigned)((C + ch_tile - 1) / ch_tile),
                    (unsigned)((ntb + kTiles128x1 - 1) / kTiles128x1));
    if (in_dtype == FP8_IN_BF16)
        k_quant_128x1<__nv_bfloat16><<<grid, kThr128x1, 0, st>>>(
            static_cast<const __nv_bfloat16*>(x), ntb, C, ldx, qT, ldqT, s, mode);
    else
        k_quant_128x1<float><<<grid, kThr128x1, 0, st>>>(static_cast<const float*>(x), ntb, C, ldx,
                                                         qT, ldqT, s, mode);
    return cudaGetLastError();
}

cudaError_t launch_requant_128x1(const uint8_t* q, int64_t ldq, const float* sA, int64_t T,
                                 int64_t C, uint8_t* qT, int64_t ldqT, float* s, int mode,
                                 cudaStream_t st)
{
    static bool ready[64] = {};
    static std::mutex mu;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (!ready[dev]) {   // above the 48 KB default for dynamic shared memory
            const cudaError_t e = cudaFuncSetAttribute(
                k_requant_128x1, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kReqSmemBytes);
            if (e != cudaSuccess) return e;
            ready[dev] = true;
        }
    }
    const int64_t ntb = T / kReqTok;
    const dim3 grid((unsigned)(C / kReqCh), (unsigned)((ntb + kReqTiles - 1) / kReqTiles));
    k_requant_128x1<<<grid, 256, kReqSmemBytes, st>>>(q, ldq, sA, T, C, qT, ldqT, s, mode);
    return cudaGetLastError();
}

cudaError_t launch_quant_w_128x128(const void* w, int in_dtype, int64_t N, int64_t K, int64_t ldw,
                                   uint8_t* q, int64_t ldq, float* sW, int mode, cudaStream_t st)
{
    const dim3 grid((unsigned)(K / 128), (unsigned)(N / 128));
    if (in_dtype == FP8_IN_BF16)
        k_quant_w128<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(w),
                                                          ldw, q, ldq, sW, K / 128, mode);
    else
        k_quant_w128<float><<<grid, 256, 0, st>>>(static_cast<const float*>(w), ldw, q, ldq, sW,
                                                  K / 128, mode);
    return cudaGetLastError();
}

}  // namespace fp8fg
