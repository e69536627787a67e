// api.cu -- the extern "C" entry points of libfp8fg (declared in
// include/fp8fg.h).  Each validates its arguments on the host, in the order
// dtype/enum -> shape -> (empty: return) -> null -> alignment -> device, and
// launches nothing when a check fails.  No entry point allocates memory.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <mutex>

#include "../../include/fp8fg.h"
#include "fp8fg_host.h"

#define FP8FG_API extern "C" __attribute__((visibility("default")))

namespace fp8fg {

namespace {
constexpr uint64_t kDefaultTimeoutNs = 4000000000ull;
std::atomic<uint64_t> g_timeout_ns{kDefaultTimeoutNs};
constexpr int64_t kMaxDim = 0x7FFFFFFF;   // sizes and coordinates fit in int32
// MoE pairs T*k: their padded rows (at most T*k + 1024*127) also fit in int32
constexpr int64_t kMaxPairs = kMaxDim - 1024 * 128;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }
bool is_mode(int m) { return m == FP8_SCALE_FP32 || m == FP8_SCALE_POW2; }
bool is_in(int d) { return d == FP8_IN_BF16 || d == FP8_IN_FP32; }
bool is_out(int d) { return d == FP8_OUT_BF16 || d == FP8_OUT_FP32; }
int in_size(int d) { return d == FP8_IN_BF16 ? 2 : 4; }
}  // namespace

uint64_t wait_timeout_ns() { return g_timeout_ns.load(std::memory_order_relaxed); }
void set_wait_timeout_ns(uint64_t ns)
{
    g_timeout_ns.store(ns ? ns : kDefaultTimeoutNs, std::memory_order_relaxed);
}

int device_sm_count()
{
    static int cache[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return 0;
    if (dev >= 0 && dev < 64 && cache[dev]) return cache[dev];
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    if (dev >= 0 && dev < 64) cache[dev] = n;
    return n;
}

bool device_is_sm100()
{
    int dev = 0, major = 0, minor = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
        return false;
    return major == 10 && minor == 0;
}

}  // namespace fp8fg

using namespace fp8fg;

FP8FG_API int fp8_quant_act_1x128(const void* x, int in_dtype, int64_t M, int64_t K, int64_t ldx,
                                  uint8_t* q, int64_t ldq, float* sA, int scale_mode, void* stream)
{
    if (!is_in(in_dtype) || !is_mode(scale_mode)) return FP8_ERR_DTYPE;
    if (M < 0 || M > kMaxDim || (M + 127) / 128 > 65535 || K <= 0 || K > kMaxDim || K % 128 || ldx < K ||
        ldq < K || ldx > kMaxDim || ldq > kMaxDim)
        return FP8_ERR_SHAPE;
    if (M == 0) return FP8_OK;
    if (!x || !q || !sA) return FP8_ERR_NULL;
    if (!aligned(x, 16) || !aligned(q, 16) || !aligned(sA, 4) || (ldx * in_size(in_dtype)) % 16 ||
        ldq % 16)
        return FP8_ERR_ALIGN;
    if (!device_is_sm100()) return FP8_ERR_DEVICE;
    return launch_quant_act_1x128(x, in_dtype, M, K, ldx, q, ldq, sA, scale_mode,
                                  static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? FP8_OK
               : FP8_ERR_LAUNCH;
}

FP8FG_API int fp8_quant_act_128x1(const void* x, int in_dtype, int64_t T, int64_t C, int64_t ldx,
                                  uint8_t* qT, int64_t ldqT, float* s, int scale_mode, void* stream)
{
    if (!is_in(in_dtype) || !is_mode(scale_mode)) return FP8_ERR_DTYPE;
    if (T <= 0 || T > kMaxDim || T % 128 || T / 128 > 65535 || C < 0 || C > kMaxDim || C % 8 ||
        ldx < C || ldqT < T || ldx > kMaxDim || ldqT > kMaxDim)
        return FP8_ERR_SHAPE;
    if (C == 0) return FP8_OK;
    if (!x || !qT || !s) return FP8_ERR_NULL;
    if (!aligned(x, 16) || !aligned(qT, 16) || !aligned(s, 4) || (ldx * in_size(in_dtype)) % 16 ||
        ldqT % 16)
        return FP8_ERR_ALIGN;
    if (!device_is_sm100()) return FP8_ERR_DEVICE;
    return launch_quant_act_128x1(x, in_dtype, T, C, ldx, qT, ldqT, s, scale_mode,
                                  static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? FP8_OK
               : FP8_ERR_LAUNCH;
}

FP8FG_API int fp8_requant_1x128_to_128x1(const uint8_t* q, int64_t ldq, const float* sA,
                                         int64_t T, int64_t C, uint8_t* qT, int64_t ldqT,
                                         float* s, int scale_mode, void* stream)
{
    if (!is_mode(scale_mode)) return FP8_ERR_DTYPE;
    if (T <= 0 || T > kMaxDim || T % 128 || T / 128 > 65535 || C < 0 || C > kMaxDim || C % 128 ||
        ldq < C || ldqT < T || ldq > kMaxDim || ldqT > kMaxDim)
        return FP8_ERR_SHAPE;
    if (C == 0) return FP8_OK;
    if (!q || !sA || !qT || !s) return FP8_ERR_NULL;
    if (!aligned(q, 16) || !aligned(qT, 16) || !aligned(sA, 4) || !aligned(s, 4) || ldq % 16 ||
        ldqT % 16)
        return FP8_ERR_ALIGN;
    if (!device_is_sm100()) return FP8_ERR_DEVICE;
    return launch_requant_128x1(q, ldq, sA, T, C, qT, ldqT, s, scale_mode,
                                static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? FP8_OK
               : FP8_ERR_LAUNCH;
}

FP8FG_API int fp8_quant_w_128x128(const void* w, int in_dtype, int64_t N, int64_t K, int64_t ldw,
                                  uint8_t* q, int64_t ldq, float* sW, int scale_mode, void* stream)
{
    if (!is_in(in_dtype) || !is_mode(scale_mode)) return FP8_ERR_DTYPE;
    if (N < 0 || N > kMaxDim || N % 128 || N / 128 > 65535 || K <= 0 || K > kMaxDim || K % 128 ||
        ldw < K || ldq < K || ldw > kMaxDim || ldq > kMaxDim)
        return FP8_ERR_SHAPE;
    if (N == 0) return FP8_OK;
    if (!w || !q || !sW) return FP8_ERR_NULL;
    if (!aligned(w, 16) || !aligned(q, 16) || !aligned(sW, 4) || (ldw * in_size(in_dtype)) % 16 ||
        ldq % 16)
        return FP8_ERR_ALIGN;
    if (!device_is_sm100()) return FP8_ERR_DEVICE;
    return launch_quant_w_128x128(w, in_dtype, N, K, ldw, q, ldq, sW, scale_mode,
                                  static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? FP8_OK
               : FP8_ERR_LAUNCH;
}

FP8FG_API int fp8_blockscaled_gemm(const uint8_t* A, const float* sA, const uint8_t* B, int b_major,
                                   const float* sB, int sb_gran, int64_t M, int64_t N, int64_t K,
                                   void* D, int out_dtype, int64_t ldd, void* stream)
{
    if (!is_out(out_dtype) || (b_major != FP8_B_KMAJOR && b_major != FP8_B_MNMAJOR) ||
        (sb_gran != 128 && sb_gran != 1) || (sb_gran == 1 && b_major != FP8_B_KMAJOR))
        return FP8_ERR_DTYPE;
    if (M < 0 || M > kMaxDim || N <= 0 || N > kMaxDim || N % 128 || K <= 0 || K > kMaxDim ||
        K % 128 || ldd < N || ldd > kMaxDim)
        return FP8_ERR_SHAPE;
    if (M == 0) return FP8_OK;
    if (!A || !sA || !B || !sB || !D) return FP8_ERR_NULL;
    const int osz = out_dtype == FP8_OUT_BF16 ? 2 : 4;
    if (!aligned(A, 16) || !aligned(B, 16) || !aligned(D, 16) || !aligned(sA, 4) ||
        !aligned(sB, sb_gran == 1 ? 16 : 4) || (ldd * osz) % 16)
        return FP8_ERR_ALIGN;
    if (!device_is_sm100()) return FP8_ERR_DEVICE;
    return launch_blockscaled_gemm(A, sA, B, b_major, sB, sb_gran, M, N, K, nullptr, 0, D,
                                   out_dtype, ldd, static_cast<cudaStream_t>(stream));
}

FP8FG_API int fp8_blockscaled_gemm_pow2(const uint8_t* A, const float* sA, const uint8_t* B,
                                        int b_major, const float* sB, int sb_gran, int64_t M,
                                        int64_t N, int64_t K, void* D, int out_dtype, int64_t ldd,
                                        void* stream)
{
    if (!is_out(out_dtype) || (b_major != FP8_B_KMAJOR && b_major != FP8_B_MNMAJOR) ||
        (sb_gran != 128 && sb_gran != 1) || (sb_gran == 1 && b_major != FP8_B_KMAJOR))
        return FP8_ERR_DTYPE;
    if (M < 0 || M > kMaxDim || N <= 0 || N > kMaxDim || N % 128 || K <= 0 || K > kMaxDim ||
        K % 128 || ldd < N || ldd > kMaxDim)
        return FP8_ERR_SHAPE;
    if (M == 0) return FP8_OK;
    if (!A || !sA || !B || !sB || !D) return FP8_ERR_NULL;
    const int osz = out_dtype == FP8_OUT_BF16 ? 2 : 4;
    if (!aligned(A, 16) || !aligned(B, 16) || !aligned(D, 16) || !aligned(sA, 4) ||
        !aligned(sB, 4) || (ldd * osz) % 16)
        return FP8_ERR_ALIGN;
    if (!device_is_sm100()) return FP8_ERR_DEVICE;
    return launch_blockscaled_gemm_mx(A, sA, B, b_major, sB, sb_gran, M, N, K, nullptr, 0, D,
                                      out_dtype, ldd, static_cast<cudaStream_t>(stream));
}

FP8FG_API int fp8_grouped_gemm_pow2(const uint8_t* A, const float* sA, const uint8_t* B,
                                    const float* sB, const int32_t* group_offsets, int G,
                                    int64_t M_total, int64_t N, int64_t K, void* D, int out_dtype,
                                    void* stream)
{
    if (!is_out(out_dtype)) return FP8_ERR_DTYPE;
    if (G < 1 || G > 1024 || M_total < 0 || M_total > kMaxDim || M_total % 128 || N <= 0 ||
        N > kMaxDim || N % 128 || K <= 0 || K > kMaxDim || K % 128 || (int64_t)G * N > kMaxDim)
        return FP8_ERR_SHAPE;
    if (M_total == 0) return FP8_OK;
    if (!A || !sA || !B || !sB || !group_offsets || !D) return FP8_ERR_NULL;
    const int osz = out_dtype == FP8_OUT_BF16 ? 2 : 4;
    if (!aligned(A, 16) || !aligned(B, 16) || !aligned(D, 16) || !aligned(sA, 4) ||
        !aligned(sB, 4) || !aligned(group_offsets, 4) || (N * osz) % 16)
        return FP8_ERR_ALIGN;
    if (!device_is_sm100()) return FP8_ERR_DEVICE;
    return launch_blockscaled_gemm_mx(A, sA, B, FP8_B_KMAJOR, sB, 128, M_total, N, K, group_offsets,
                                      G, D, out_dtype, N, static_cast<cudaStream_t>(stream));
}

FP8FG_API int fp8_grouped_gemm(const uint8_t* A, const float* sA, const uint8_t* B, const float* sB,
                               const int32_t* group_offsets, int G, int64_t M_total, int64_t N,
                               int64_t K, void* D, int out_dtype, void* stream)
{
    if (!is_out(out_dtype)) return FP8_ERR_DTYPE;
    if (G < 1 || G > 1024 || M_total < 0 || M_total > kMaxDim || M_total % 128 || N <= 0 ||
        N > kMaxDim || N % 128 || K <= 0 || K > kMaxDim || K % 128 || (int64_t)G * N > kMaxDim)
        return FP8_ERR_SHAPE;
    if (M_total == 0) return FP8_OK;
    if (!A || !sA || !B || !sB || !group_offsets || !D) return FP8_ERR_NULL;
    const int osz = out_dtype == FP8_OUT_BF16 ? 2 : 4;
    if (!aligned(A, 16) || !aligned(B, 16) || !aligned(D, 16) || !aligned(sA, 4) ||
        !aligned(sB, 4) || !aligned(group_offsets, 4) || (N * osz) % 16)
        return FP8_ERR_ALIGN;
    if (!device_is_sm100()) return FP8_ERR_DEVICE;
    return launch_blockscaled_gemm(A, sA, B, FP8_B_KMAJOR, sB, 128, M_total, N, K, group_offsets, G,
                                   D, out_dtype, N, static_cast<cudaStream_t>(stream));
}

FP8FG_API int fp8_grouped_gemm_gather(const uint8_t* A, const float* sA, int64_t T,
                                      const int32_t* row_token, const uint8_t* B, const float* sB,
                                      const int32_t* group_offsets, int G, int64_t M_total,
                                      int64_t N, int64_t K, void* D, int out_dtype, void* stream)
{
    if (!is_out(out_dtype)) return FP8_ERR_DTYPE;
    if (G < 1 || G > 1024 || M_total < 0 || M_total > kMaxDim || M_total % 128 || N <= 0 ||
        N > kMaxDim || N % 128 || K <= 0 || K > kMaxDim || K % 128 || (int64_t)G * N > kMaxDim ||
        T < 0 || T > kMaxDim)
        return FP8_ERR_SHAPE;
    if (M_total == 0) return FP8_OK;
    if (T < 1) return FP8_ERR_SHAPE;   // every row of D would be padding
    if (!A || !sA || !row_token || !B || !sB || !group_offsets || !D) return FP8_ERR_NULL;
    const int osz = out_dtype == FP8_OUT_BF16 ? 2 : 4;
    if (!aligned(A, 16) || !aligned(B, 16) || !aligned(D, 16) || !aligned(sA, 4) ||
        !aligned(sB, 4) || !aligned(group_offsets, 4) || !aligned(row_token, 4) || (N * osz) % 16)
        return FP8_ERR_ALIGN;
    if (!device_is_sm100()) return FP8_ERR_DEVICE;
    return launch_grouped_gemm_gather(A, sA, T, row_token, B, sB, group_offsets, G, M_total, N, K, D,
                                      out_dtype, static_cast<cudaStream_t>(stream));
}

FP8FG_API int fp8_moe_route(const int32_t* topk, int64_t T, int k, int G, int64_t M_cap,
                            int32_t* group_offsets, int32_t* token_row, int32_t* row_token,
                            void* workspace, int64_t workspace_bytes, void* stream)
{
    if (T < 0 || k < 1 || G < 1 || G > 1024 || M_cap < 0 || M_cap % 128 || M_cap > kMaxDim ||
        T > kMaxPairs / k)
        return FP8_ERR_SHAPE;
    if (workspace_bytes < fp8_moe_dispatch_workspace_bytes(T, k, G)) return FP8_ERR_SHAPE;
    if (!group_offsets || (T > 0 && (!topk || !token_row || !workspace)) || (M_cap > 0 && !row_token))
        return FP8_ERR_NULL;
    if (!aligned(topk, 4) || !aligned(group_offsets, 4) || !aligned(token_row, 4) ||
        !aligned(row_token, 4) || !aligned(workspace, 4))
        return FP8_ERR_ALIGN;
    if (!device_is_sm100()) return FP8_ERR_DEVICE;
    return launch_moe_route(topk, T, k, G, M_cap, group_offsets, token_row, row_token,
                            static_cast<int32_t*>(workspace), static_cast<cudaStream_t>(stream)) ==
                   cudaSuccess
               ? FP8_OK
               : FP8_ERR_LAUNCH;
}

FP8FG_API int64_t fp8_moe_dispatch_workspace_bytes(int64_t T, int k, int G)
{
    if (T < 0 || k < 1 || G < 1 || G > 1024 || T > kMaxPairs / k) return 0;
    return moe_dispatch_workspace_ints(T * k, G) * (int64_t)sizeof(int32_t);
}

FP8FG_API int fp8_moe_dispatch(const uint8_t* q, const float* sA, int64_t T, int64_t K,
                               const int32_t* topk, int k, int G, uint8_t* q_out, float* sA_out,
                               int64_t M_cap, int32_t* group_offsets, int32_t* token_row,
                               int32_t* row_token, void* workspace, int64_t workspace_bytes,
                               void* stream)
{
    if (T < 0 || K <= 0 || K % 128 || K > kMaxDim || k < 1 || G < 1 || G > 1024 || M_cap < 0 ||
        M_cap % 128 || M_cap > kMaxDim || T > kMaxPairs / k)
        return FP8_ERR_SHAPE;
    if (workspace_bytes < fp8_moe_dispatch_workspace_bytes(T, k, G)) return FP8_ERR_SHAPE;
    if (!group_offsets || (T > 0 && (!q || !sA || !topk || !token_row || !workspace)) ||
        (M_cap > 0 && (!q_out || !sA_out || !row_token)))
        return FP8_ERR_NULL;
    if (!aligned(q, 16) || !aligned(q_out, 16) || !aligned(sA, 4) || !aligned(sA_out, 4) ||
        !aligned(topk, 4) || !aligned(group_offsets, 4) || !aligned(token_row, 4) ||
        !aligned(row_token, 4) || !aligned(workspace, 4))
        return FP8_ERR_ALIGN;
    if (!device_is_sm100()) return FP8_ERR_DEVICE;
    return launch_moe_dispatch(q, sA, T, K, topk, k, G, q_out, sA_out, M_cap, group_offsets,
                               token_row, row_token, static_cast<int32_t*>(workspace),
                               static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? FP8_OK
               : FP8_ERR_LAUNCH;
}

FP8FG_API int fp8_moe_quant_dispatch(const void* x, int in_dtype, int64_t T, int64_t K,
                                     int64_t ldx, const int32_t* topk, int k, int G,
                                     uint8_t* q_out, float* sA_out, int64_t M_cap,
                                     int32_t* group_offsets, int32_t* token_row,
                                     int32_t* row_token, void* workspace, int64_t workspace_bytes,
                                     int scale_mode, void* stream)
{
    if (!is_in(in_dtype) || !is_mode(scale_mode)) return FP8_ERR_DTYPE;
    if (T < 0 || K <= 0 || K % 128 || K > kMaxDim || k < 1 || G < 1 || G > 1024 || M_cap < 0 ||
        M_cap % 128 || M_cap > kMaxDim || T > kMaxPairs / k || (T + 127) / 128 > 65535 ||
        ldx < K || ldx > kMaxDim)
        return FP8_ERR_SHAPE;
    if (workspace_bytes < fp8_moe_dispatch_workspace_bytes(T, k, G)) return FP8_ERR_SHAPE;
    if (!group_offsets || (T > 0 && (!x || !topk || !token_row || !workspace)) ||
        (M_cap > 0 && (!q_out || !sA_out || !row_token)))
        return FP8_ERR_NULL;
    if (!aligned(x, 16) || (ldx * in_size(in_dtype)) % 16 || !aligned(q_out, 16) ||
        !aligned(sA_out, 4) || !aligned(topk, 4) || !aligned(group_offsets, 4) ||
        !aligned(token_row, 4) || !aligned(row_token, 4) || !aligned(workspace, 4))
        return FP8_ERR_ALIGN;
    if (!device_is_sm100()) return FP8_ERR_DEVICE;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    int32_t* ws = static_cast<int32_t*>(workspace);
    if (launch_moe_route(topk, T, k, G, M_cap, group_offsets, token_row, row_token, ws, st) !=
            cudaSuccess ||
        launch_quant_act_1x128_dispatch(x, in_dtype, T, K, ldx, token_row, k, M_cap, q_out,
                                        sA_out, scale_mode, st) != cudaSuccess ||
        launch_moe_pad_rows(group_offsets, G, K, row_token, M_cap, q_out, sA_out, st) !=
            cudaSuccess)
        return FP8_ERR_LAUNCH;
    return FP8_OK;
}

static_assert(kMoeStaticWsInts * (int64_t)sizeof(int32_t) == FP8_MOE_NOALLOC_WS_BYTES,
              "static dispatch scratch and its advertised size disagree");
static int32_t g_no_device_ws = 0;

FP8FG_API int fp8_moe_dispatch_noalloc(const uint8_t* q, const float* sA, int64_t T, int64_t K,
                                       const int32_t* topk, int k, int G, uint8_t* q_out,
                                       float* sA_out, int64_t M_cap, int32_t* group_offsets,
                                       int32_t* token_row, int32_t* row_token, void* stream)
{
    const int64_t need = fp8_moe_dispatch_workspace_bytes(T, k, G);
    if (need > FP8_MOE_NOALLOC_WS_BYTES) return FP8_ERR_SHAPE;
    int32_t* ws = &g_no_device_ws;   // never dereferenced: without a device the call
                                     // below validates the rest, then returns FP8_ERR_DEVICE
    if (device_is_sm100() && moe_static_workspace(&ws) != cudaSuccess) return FP8_ERR_DEVICE;
    return fp8_moe_dispatch(q, sA, T, K, topk, k, G, q_out, sA_out, M_cap, group_offsets,
                            token_row, row_token, ws, FP8_MOE_NOALLOC_WS_BYTES, stream);
}

FP8FG_API int fp8_moe_combine(const void* D, int d_dtype, int64_t M_cap, int64_t N,
                              const int32_t* token_row, const float* weights, int64_t T, int k,
                              void* out, void* stream)
{
    if (!is_out(d_dtype)) return FP8_ERR_DTYPE;
    if (T < 0 || T > 0x7FFFFFFF || k < 1 || N <= 0 || N % 8 || N > kMaxDim || M_cap < 0)
        return FP8_ERR_SHAPE;
    if (T == 0) return FP8_OK;
    if (!D || !token_row || !weights || !out) return FP8_ERR_NULL;
    if (!aligned(D, 16) || !aligned(out, 16) || !aligned(token_row, 4) || !aligned(weights, 4))
        return FP8_ERR_ALIGN;
    if (!device_is_sm100()) return FP8_ERR_DEVICE;
    return launch_moe_combine(D, d_dtype, M_cap, N, token_row, weights, T, k, out,
                              static_cast<cudaStream_t>(stream)) == cudaSuccess
               ? FP8_OK
               : FP8_ERR_LAUNCH;
}

FP8FG_API int fp8_get_status(void* stream)
{
    const int a = read_and_clear_status(static_cast<cudaStream_t>(stream));
    const int b = read_and_clear_moe_status();
    const int c = read_and_clear_mx_status();
    return a != FP8_OK ? a : (b != FP8_OK ? b : c);
}

FP8FG_API const char* fp8_status_string(int code)
{
    switch (code) {
        case FP8_OK: return "FP8_OK";
        case FP8_ERR_NULL: return "FP8_ERR_NULL: a required pointer is NULL";
        case FP8_ERR_SHAPE: return "FP8_ERR_SHAPE: unsupported or inconsistent sizes";
        case FP8_ERR_ALIGN: return "FP8_ERR_ALIGN: pointer or leading dimension misaligned";
        case FP8_ERR_DTYPE: return "FP8_ERR_DTYPE: unknown dtype, mode, layout or granularity";
        case FP8_ERR_LAUNCH: return "FP8_ERR_LAUNCH: CUDA launch failed";
        case FP8_ERR_TIMEOUT: return "FP8_ERR_TIMEOUT: a device-side wait ran out of time";
        case FP8_ERR_DEVICE: return "FP8_ERR_DEVICE: no supported (sm_100) CUDA device";
        case FP8_ERR_VALUE: return "FP8_ERR_VALUE: a scale is not a positive normal power of two";
        default: return "unknown fp8fg status";
    }
}

FP8FG_API void fp8_set_wait_timeout_ns(uint64_t ns) { set_wait_timeout_ns(ns); }

FP8FG_API int fp8_selftest_wait_timeout(void* stream)
{
    if (!device_is_sm100()) return FP8_ERR_DEVICE;
    return launch_selftest_wait(static_cast<cudaStream_t>(stream)) == cudaSuccess ? FP8_OK
                                                                                 : FP8_ERR_LAUNCH;
}

FP8FG_API int fp8_selftest_gemm_unwind(int kernel, const uint8_t* A, const float* sA,
                                       const uint8_t* B, const float* sB,
                                       const int32_t* group_offsets, int G, int64_t M, int64_t N,
                                       int64_t K, void* D, int out_dtype, void* stream)
{
    if ((kernel != 0 && kernel != 1) || !is_out(out_dtype)) return FP8_ERR_DTYPE;
    if (M <= 0 || M > kMaxDim || M % 128 || N <= 0 || N > kMaxDim || N % 128 || K < 256 ||
        K > kMaxDim || K % 128 || (group_offsets && (G < 1 || G > 1024 || (int64_t)G * N > kMaxDim)))
        return FP8_ERR_SHAPE;
    if (!A || !sA || !B || !sB || !D) return FP8_ERR_NULL;
    const int osz = out_dtype == FP8_OUT_BF16 ? 2 : 4;
    if (!aligned(A, 16) || !aligned(B, 16) || !aligned(D, 16) || !aligned(sA, 4) ||
        !aligned(sB, 4) || !aligned(group_offsets, 4) || (N * osz) % 16)
        return FP8_ERR_ALIGN;
    if (!device_is_sm100()) return FP8_ERR_DEVICE;
    const int g = group_offsets ? G : 0;
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    return kernel == 0 ? launch_blockscaled_gemm_withheld(A, sA, B, FP8_B_KMAJOR, sB, 128, M, N, K,
                                                          group_offsets, g, D, out_dtype, N, st)
                       : launch_blockscaled_gemm_mx_withheld(A, sA, B, FP8_B_KMAJOR, sB, 128, M,
                                                             N, K, group_offsets, g, D, out_dtype,
                                                             N, st);
}

FP8FG_API int fp8_device_supported(void) { return device_is_sm100() ? 1 : 0; }
