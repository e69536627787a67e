// moe.cu -- FP8 dispatch of MoE activations into expert-contiguous groups and
// the weighted combine of the expert outputs (sm_100a).
//
// The recipe caches and dispatches MoE activations in FP8 ("5 Ways You can
// get More Deepseek While Spending Less" and the cameseeing.com post: cache
// and dispatch activations in FP8; "Three Fast Methods To Study Deepseek":
// 8 routed experts per token; gnrental.net post: the MoE part loads the
// parameters of one expert per group).  Tokens are quantized once (1x128,
// row-local), and their E4M3 rows and scales -- not BF16 rows -- are moved to
// the layout the grouped GEMM reads.
//
// Dispatch is a stable counting sort of the (token, slot) pairs by expert:
//   k_moe_count   per chunk of 1024 pairs: expert histogram -> workspace
//   k_moe_scan    per expert: exclusive prefix over chunks; padded group
//                 offsets (multiples of 128) -> workspace bases, offsets[]
//   k_moe_rank    per chunk, one warp in pair order: stable rank of each pair
//                 among equal experts (__match_any_sync) -> token_row[],
//                 row_token[]
//   k_moe_rows    per destination row: copy the token's codes (or zeros for
//                 padding) and its 1x128 scales (or 1 for padding)
// Padding rows get codes 0 and scale 1: exactly what quantizing a zero row
// gives, so the result equals quantizing the gathered BF16 rows.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "fp8fg_device.cuh"
#include "fp8fg_host.h"

namespace fp8fg {

namespace {

constexpr int kPairsPerChunk = 1024;


// Fixed dispatch scratch for the non-allocating entry point (one per device,
// in every context the module is loaded in).  Every entry a dispatch reads is
// written earlier in the same dispatch, so it never needs clearing.
__device__ __align__(256) int32_t g_moe_static_ws[kMoeStaticWsInts];

__global__ void __launch_bounds__(256) k_moe_count(const int32_t* __restrict__ topk, int64_t P,
                                                   int G, int32_t* __restrict__ ws)
{
    extern __shared__ int32_t hist[];
    for (int e = threadIdx.x; e < G; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    const int64_t i0 = (int64_t)blockIdx.x * kPairsPerChunk;
    for (int i = threadIdx.x; i < kPairsPerChunk; i += blockDim.x) {
        const int64_t idx = i0 + i;
        if (idx >= P) break;
        const int32_t e = topk[idx];
        if (e >= 0 && e < G) atomicAdd(&hist[e], 1);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < G; e += blockDim.x) ws[(int64_t)blockIdx.x * G + e] = hist[e];
}

// One CTA of 1024 threads.  Each expert e gets `tpe` consecutive threads
// (the largest power of two with tpe * G <= 1024); thread `sub` of the group
// sums a run of chunks of expert e, the group scans those sums in shared
// memory, and each thread then rewrites its chunks with running bases.  In
// the end ws[c][e] is the first destination row of expert e's pairs in chunk
// c: the expert's padded group offset plus the pairs of earlier chunks.
__global__ void __launch_bounds__(1024) k_moe_scan(int32_t* __restrict__ ws, int nchunks, int G,
                                                   int64_t M_cap, int32_t* __restrict__ offsets)
{
    __shared__ int32_t part[1024];
    __shared__ int32_t padded[1024];
    __shared__ int32_t base[1025];
    int tpe = 1;
    while (tpe * 2 * G <= 1024) tpe *= 2;
    const int e = threadIdx.x / tpe;
    const int sub = threadIdx.x % tpe;
    const bool mine = e < G;
    const int per = (nchunks + tpe - 1) / tpe;
    const int c0 = sub * per < nchunks ? sub * per : nchunks;
    const int c1 = c0 + per < nchunks ? c0 + per : nchunks;
    int32_t sum = 0;
    if (mine)
        for (int c = c0; c < c1; ++c) sum += ws[(int64_t)c * G + e];
    part[threadIdx.x] = sum;
    __syncthreads();
    // inclusive scan inside each group of tpe threads (Hillis-Steele)
    for (int d = 1; d < tpe; d <<= 1) {
        const int32_t add = (sub >= d) ? part[threadIdx.x - d] : 0;
        __syncthreads();
        part[threadIdx.x] += add;
        __syncthreads();
    }
    if (mine && sub == tpe - 1) padded[e] = (part[threadIdx.x] + 127) / 128 * 128;
    __syncthreads();
    if (threadIdx.x == 0) {
        int64_t acc = 0;
        for (int j = 0; j < G; ++j) {
            base[j] = (int32_t)acc;
            acc += padded[j];
        }
        base[G] = (int32_t)(acc < 0x7FFFFFFF ? acc : 0x7FFFFFFF);
        if (acc > M_cap) report_error(FP8_ERR_SHAPE);
    }
    __syncthreads();
    for (int j = threadIdx.x; j <= G; j += blockDim.x) offsets[j] = base[j];
    if (mine) {
        int32_t run = base[e] + part[threadIdx.x] - sum;   // pairs of expert e before chunk c0
        for (int c = c0; c < c1; ++c) {
            const int32_t v = ws[(int64_t)c * G + e];
            ws[(int64_t)c * G + e] = run;
            run += v;
        }
    }
}

// One warp per chunk walks its pairs in order, 32 at a time.  The chunk's
// expert ids are all loaded before the walk, so the walk itself waits on
// shared memory only.
__global__ void __launch_bounds__(32) k_moe_rank(const int32_t* __restrict__ topk, int64_t P, int k,
                                                 int G, const int32_t* __restrict__ ws,
                                                 int64_t M_cap, int32_t* __restrict__ token_row,
                                                 int32_t* __restrict__ row_token)
{
    extern __shared__ int32_t cursor[];
    constexpr int kSteps = kPairsPerChunk / 32;
    const int lane = threadIdx.x;
    const int64_t i0 = (int64_t)blockIdx.x * kPairsPerChunk;
    int32_t ids[kSteps];
#pragma unroll
    for (int j = 0; j < kSteps; ++j) {
        const int64_t idx = i0 + j * 32 + lane;
        ids[j] = idx < P ? __ldg(topk + idx) : -1;
    }
    for (int e = lane; e < G; e += 32) cursor[e] = ws[(int64_t)blockIdx.x * G + e];
    __syncwarp();
#pragma unroll
    for (int j = 0; j < kSteps; ++j) {
        const int64_t idx = i0 + j * 32 + lane;
        const bool live = idx < P;
        int32_t e = ids[j];
        const bool ok = live && e >= 0 && e < G;
        if (live && !ok) report_error(FP8_ERR_SHAPE);
        if (!ok) e = -1 - lane;                 // unique key: never matches another lane
        const unsigned same = __match_any_sync(0xffffffffu, e);
        const unsigned below = same & ((1u << lane) - 1u);
        int32_t pos = -1;
        if (ok) pos = cursor[e] + __popc(below);
        __syncwarp();
        if (ok && below == 0) cursor[e] += __popc(same);   // lowest lane of the group advances
        __syncwarp();
        if (live) {
            const bool fits = ok && pos >= 0 && pos < M_cap;
            if (ok && !fits) report_error(FP8_ERR_SHAPE);
            token_row[idx] = fits ? pos : -1;
            if (fits) row_token[pos] = (int32_t)(idx / k);
        }
    }
}

// A padding row: K zero codes (16-byte stores by the warp's lanes) and K/128
// scales of 1, what quantizing a zero row gives.
__device__ __forceinline__ void fill_pad_row(int64_t r, int64_t K, int64_t M_cap, int lane,
                                             uint8_t* __restrict__ q_out, float* __restrict__ sA_out)
{
    uint4* dst = reinterpret_cast<uint4*>(q_out + r * K);
    for (int64_t v = lane; v < K / 16; v += 32) dst[v] = make_uint4(0, 0, 0, 0);
    for (int64_t kb = lane; kb < K / 128; kb += 32) sA_out[kb * M_cap + r] = 1.0f;
}

// CTA = 8 warps, one destination row per warp: the row's K code bytes in
// 16-byte vectors, then its K/128 scales.
__global__ void __launch_bounds__(256) k_moe_rows(const uint8_t* __restrict__ q,
                                                  const float* __restrict__ sA, int64_t T, int64_t K,
                                                  const int32_t* __restrict__ row_token,
                                                  int64_t M_cap, uint8_t* __restrict__ q_out,
                                                  float* __restrict__ sA_out)
{
    const int lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (r >= M_cap) return;
    const int32_t t = row_token[r];
    if (t >= 0 && t < T) {
        uint4* dst = reinterpret_cast<uint4*>(q_out + r * K);
        const uint4* src = reinterpret_cast<const uint4*>(q + (int64_t)t * K);
        for (int64_t v = lane; v < K / 16; v += 32) dst[v] = __ldg(src + v);
        for (int64_t kb = lane; kb < K / 128; kb += 32) sA_out[kb * M_cap + r] = __ldg(sA + kb * T + t);
    } else {
        fill_pad_row(r, K, M_cap, lane, q_out, sA_out);
    }
}

// The padding rows only, for the fused quantize-and-dispatch (whose quantizer
// has written every claimed row).  A group's claimed rows come first, so its
// padding lies in its last 127 rows; rows from offsets[G] to M_cap are
// unclaimed.  Warps walk the slots: G x 128 candidate rows (row_token < 0
// marks padding), then the tail rows; every row written is inside [0, M_cap).
__global__ void __launch_bounds__(256) k_moe_pad_rows(const int32_t* __restrict__ offsets, int G,
                                                      int64_t K, const int32_t* __restrict__ row_token,
                                                      int64_t M_cap, uint8_t* __restrict__ q_out,
                                                      float* __restrict__ sA_out)
{
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * 8;
    int64_t end = offsets[G];
    end = end < 0 ? 0 : (end > M_cap ? M_cap : end);
    const int64_t slots = (int64_t)G * 128 + (M_cap - end);
    for (int64_t sl = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); sl < slots; sl += warps) {
        int64_t r;
        if (sl < (int64_t)G * 128) {
            const int e = (int)(sl >> 7);
            const int64_t lo = offsets[e], hi = offsets[e + 1];
            r = hi - 128 + (sl & 127);
            if (r < lo || r < 0 || r >= M_cap || row_token[r] >= 0) continue;
        } else {
            r = end + (sl - (int64_t)G * 128);
        }
        fill_pad_row(r, K, M_cap, lane, q_out, sA_out);
    }
}

// out[t][:] = sum_j w[t][j] * D[token_row[t][j]][:], FP32 sums, BF16 out.
// CTA = 256 threads per token row of N columns (8 columns per thread step).
// Entries of token_row outside [0, M_cap) are skipped like dropped pairs.
template <typename Tin>
__global__ void __launch_bounds__(256) k_moe_combine(const Tin* __restrict__ D, int64_t M_cap,
                                                     int64_t N,
                                                     const int32_t* __restrict__ token_row,
                                                     const float* __restrict__ w, int k,
                                                     __nv_bfloat16* __restrict__ out)
{
    const int64_t t = blockIdx.x;
    for (int64_t c = (int64_t)threadIdx.x * 8; c < N; c += 256 * 8) {
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int j = 0; j < k; ++j) {
            const int32_t r = token_row[t * k + j];
            if (r < 0 || r >= M_cap) continue;
            const float wj = w[t * k + j];
            if constexpr (sizeof(Tin) == 2) {
                const uint4 v = __ldg(reinterpret_cast<const uint4*>(D + (int64_t)r * N + c));
                const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    acc[2 * i] = fmaf(wj, __uint_as_float(u[i] << 16), acc[2 * i]);
                    acc[2 * i + 1] = fmaf(wj, __uint_as_float(u[i] & 0xFFFF0000u), acc[2 * i + 1]);
                }
            } else {
                const float4 a = __ldg(reinterpret_cast<const float4*>(D + (int64_t)r * N + c));
                const float4 b = __ldg(reinterpret_cast<const float4*>(D + (int64_t)r * N + c) + 1);
                const float f[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
                for (int i = 0; i < 8; ++i) acc[i] = fmaf(wj, f[i], acc[i]);
            }
        }
        uint4 o;
        __nv_bfloat162 h0 = __floats2bfloat162_rn(acc[0], acc[1]);
        __nv_bfloat162 h1 = __floats2bfloat162_rn(acc[2], acc[3]);
        __nv_bfloat162 h2 = __floats2bfloat162_rn(acc[4], acc[5]);
        __nv_bfloat162 h3 = __floats2bfloat162_rn(acc[6], acc[7]);
        o.x = *reinterpret_cast<uint32_t*>(&h0);
        o.y = *reinterpret_cast<uint32_t*>(&h1);
        o.z = *reinterpret_cast<uint32_t*>(&h2);
        o.w = *reinterpret_cast<uint32_t*>(&h3);
        *reinterpret_cast<uint4*>(out + t * N + c) = o;
    }
}

}  // namespace

int64_t moe_dispatch_workspace_ints(int64_t P, int G)
{
    return ((P + kPairsPerChunk - 1) / kPairsPerChunk) * (int64_t)G;
}

// Routing half of the dispatch: group offsets, token_row and row_token.
cudaError_t launch_moe_route(const int32_t* topk, int64_t T, int k, int G, int64_t M_cap,
                             int32_t* offsets, int32_t* token_row, int32_t* row_token, int32_t* ws,
                             cudaStream_t st)
{
    const int64_t P = T * k;
    const int nchunks = (int)((P + kPairsPerChunk - 1) / kPairsPerChunk);
    // rows beyond the real ones are padding until the rank pass claims them
    cudaError_t err = cudaMemsetAsync(row_token, 0xFF, (size_t)M_cap * sizeof(int32_t), st);
    if (err != cudaSuccess) return err;
    if (nchunks > 0) {
        k_moe_count<<<nchunks, 256, G * sizeof(int32_t), st>>>(topk, P, G, ws);
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }
    k_moe_scan<<<1, 1024, 0, st>>>(ws, nchunks, G, M_cap, offsets);
    if ((err = cudaGetLastError()) != cudaSuccess) return err;
    if (nchunks > 0) {
        k_moe_rank<<<nchunks, 32, G * sizeof(int32_t), st>>>(topk, P, k, G, ws, M_cap, token_row,
                                                            row_token);
        if ((err = cudaGetLastError()) != cudaSuccess) return err;
    }
    return cudaSuccess;
}

// Row half: copy each claimed row's codes and scales from the token's, and
// fill the padding rows.
cudaError_t launch_moe_rows(const uint8_t* q, const float* sA, int64_t T, int64_t K,
                            const int32_t* row_token, int64_t M_cap, uint8_t* q_out,
                            float* sA_out, cudaStream_t st)
{
    if (M_cap > 0)
        k_moe_rows<<<(unsigned)((M_cap + 7) / 8), 256, 0, st>>>(q, sA, T, K, row_token, M_cap,
                                                              q_out, sA_out);
    return cudaGetLastError();
}

cudaError_t launch_moe_pad_rows(const int32_t* offsets, int G, int64_t K, const int32_t* row_token,
                                int64_t M_cap, uint8_t* q_out, float* sA_out, cudaStream_t st)
{
    if (M_cap <= 0) return cudaSuccess;
    const int64_t slot_ctas = ((int64_t)G * 128 + M_cap + 7) / 8;
    const int64_t cap = 4 * (int64_t)device_sm_count();
    k_moe_pad_rows<<<(unsigned)(slot_ctas < cap ? slot_ctas : cap), 256, 0, st>>>(
        offsets, G, K, row_token, M_cap, q_out, sA_out);
    return cudaGetLastError();
}

cudaError_t launch_moe_dispatch(const uint8_t* q, const float* sA, int64_t T, int64_t K,
                                const int32_t* topk, int k, int G, uint8_t* q_out, float* sA_out,
                                int64_t M_cap, int32_t* offsets, int32_t* token_row,
                                int32_t* row_token, int32_t* ws, cudaStream_t st)
{
    cudaError_t err = launch_moe_route(topk, T, k, G, M_cap, offsets, token_row, row_token, ws, st);
    if (err != cudaSuccess) return err;
    return launch_moe_rows(q, sA, T, K, row_token, M_cap, q_out, sA_out, st);
}

cudaError_t launch_moe_combine(const void* D, int d_dtype, int64_t M_cap, int64_t N,
                               const int32_t* token_row, const float* w, int64_t T, int k, void* out,
                               cudaStream_t st)
{
    if (T == 0) return cudaSuccess;
    if (d_dtype == FP8_OUT_BF16)
        k_moe_combine<__nv_bfloat16><<<(unsigned)T, 256, 0, st>>>(
            static_cast<const __nv_bfloat16*>(D), M_cap, N, token_row, w, k,
            static_cast<__nv_bfloat16*>(out));
    else
        k_moe_combine<float><<<(unsigned)T, 256, 0, st>>>(static_cast<const float*>(D), M_cap, N,
                                                          token_row, w, k,
                                                          static_cast<__nv_bfloat16*>(out));
    return cudaGetLastError();
}

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);

// The driver's cuCtxGetCurrent, looked up once (the runtime is linked
// statically; the driver is reached through its entry-point table).
CtxGetCurrentFn ctx_get_current()
{
    static CtxGetCurrentFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<CtxGetCurrentFn>(f);
    });
    return fn;
}

// Device address of g_moe_static_ws in the current context.  A __device__
// array has one address per context the module is loaded in, so the address
// is cached per device together with the context it was looked up in, and
// looked up again when the caller's current context is another one.
cudaError_t moe_static_workspace(int32_t** ws)
{
    constexpr int kMaxDevices = 64;
    static std::mutex mu;
    static int32_t* addr[kMaxDevices] = {};
    static CUcontext ctx_of[kMaxDevices] = {};
    int dev = 0;
    cudaError_t err = cudaGetDevice(&dev);
    if (err != cudaSuccess) return err;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    const CtxGetCurrentFn get_ctx = ctx_get_current();
    CUcontext ctx = nullptr;
    if (get_ctx && get_ctx(&ctx) != CUDA_SUCCESS) ctx = nullptr;
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev] || ctx_of[dev] != ctx) {
        void* p = nullptr;
        err = cudaGetSymbolAddress(&p, g_moe_static_ws);     // with this device current
        if (err != cudaSuccess) return err;
        addr[dev] = static_cast<int32_t*>(p);
        // the lookup makes the device's primary context current if no
        // context was: remember the one current now
        if (get_ctx && get_ctx(&ctx) != CUDA_SUCCESS) ctx = nullptr;
        ctx_of[dev] = ctx;
    }
    *ws = addr[dev];
    return cudaSuccess;
}

// Malformed routing entries and capacity overflows are recorded in this
// module's status word.
int read_and_clear_moe_status() { return read_and_clear_module_status(); }

}  // namespace fp8fg
