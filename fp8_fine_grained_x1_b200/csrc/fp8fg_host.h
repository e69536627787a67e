// fp8fg_host.h -- internal host-side interface between the C ABI (api.cu) and
// the kernel launchers (quant.cu, gemm.cu).  Arguments reaching these
// functions have already been validated by api.cu.
#pragma once

#include <cuda_runtime.h>

#include <cstdint>

namespace fp8fg {

cudaError_t launch_quant_act_1x128(const void* x, int in_dtype, int64_t M, int64_t K, int64_t ldx,
                                   uint8_t* q, int64_t ldq, float* sA, int mode, cudaStream_t st);
cudaError_t launch_quant_act_128x1(const void* x, int in_dtype, int64_t T, int64_t C, int64_t ldx,
                                   uint8_t* qT, int64_t ldqT, float* s, int mode, cudaStream_t st);
cudaError_t launch_requant_128x1(const uint8_t* q, int64_t ldq, const float* sA, int64_t T,
                                 int64_t C, uint8_t* qT, int64_t ldqT, float* s, int mode,
                                 cudaStream_t st);
cudaError_t launch_quant_w_128x128(const void* w, int in_dtype, int64_t N, int64_t K, int64_t ldw,
                                   uint8_t* q, int64_t ldq, float* sW, int mode, cudaStream_t st);

// Dense (G == 0, group_offsets == nullptr) or grouped block-scaled GEMM.
// For the grouped form B is [G][N][K] K-major and sB [G][N/128][K/128].
// Returns cudaSuccess or the launch / tensor-map error; *status_out gets the
// fp8_status code to report.
int launch_blockscaled_gemm(const uint8_t* A, const float* sA, const uint8_t* B, int b_major,
                            const float* sB, int sb_gran, int64_t M, int64_t N, int64_t K,
                            const int32_t* group_offsets, int G, void* D, int out_dtype,
                            int64_t ldd, cudaStream_t st);
// Grouped GEMM whose A rows are gathered: output row m reads A row row_map[m]
// of A [a_rows][K] (sA [K/128][a_rows]); -1 marks a padding row (output 0).
int launch_grouped_gemm_gather(const uint8_t* A, const float* sA, int64_t a_rows,
                               const int32_t* row_map, const uint8_t* B, const float* sB,
                               const int32_t* group_offsets, int G, int64_t M, int64_t N, int64_t K,
                               void* D, int out_dtype, cudaStream_t st);

// Self-test forms of the two GEMMs: the odd CTA of every pair withholds its
// operand loads after its first K-block, so the pair's waits run out.
int launch_blockscaled_gemm_withheld(const uint8_t* A, const float* sA, const uint8_t* B,
                                     int b_major, const float* sB, int sb_gran, int64_t M,
                                     int64_t N, int64_t K, const int32_t* group_offsets, int G,
                                     void* D, int out_dtype, int64_t ldd, cudaStream_t st);
int launch_blockscaled_gemm_mx_withheld(const uint8_t* A, const float* sA, const uint8_t* B,
                                        int b_major, const float* sB, int sb_gran, int64_t M,
                                        int64_t N, int64_t K, const int32_t* group_offsets, int G,
                                        void* D, int out_dtype, int64_t ldd, cudaStream_t st);

cudaError_t launch_selftest_wait(cudaStream_t st);

// MoE dispatch / combine (moe.cu).
int64_t moe_dispatch_workspace_ints(int64_t P, int G);
cudaError_t launch_moe_dispatch(const uint8_t* q, const float* sA, int64_t T, int64_t K,
                                const int32_t* topk, int k, int G, uint8_t* q_out, float* sA_out,
                                int64_t M_cap, int32_t* offsets, int32_t* token_row,
                                int32_t* row_token, int32_t* ws, cudaStream_t st);
// The dispatch in two halves: routing (group offsets, token_row, row_token)
// and the row copy; for the fused quantize-and-dispatch, the padding rows
// alone (every row no pair claimed).
cudaError_t launch_moe_route(const int32_t* topk, int64_t T, int k, int G, int64_t M_cap,
                             int32_t* offsets, int32_t* token_row, int32_t* row_token, int32_t* ws,
                             cudaStream_t st);
cudaError_t launch_moe_rows(const uint8_t* q, const float* sA, int64_t T, int64_t K,
                            const int32_t* row_token, int64_t M_cap, uint8_t* q_out,
                            float* sA_out, cudaStream_t st);
cudaError_t launch_moe_pad_rows(const int32_t* offsets, int G, int64_t K, const int32_t* row_token,
                                int64_t M_cap, uint8_t* q_out, float* sA_out, cudaStream_t st);
// 1x128 quantization written straight to the rows token_row gives each token.
cudaError_t launch_quant_act_1x128_dispatch(const void* x, int in_dtype, int64_t T, int64_t K,
                                            int64_t ldx, const int32_t* token_row, int k,
                                            int64_t M_cap, uint8_t* q_out, float* sA_out, int mode,
                                            cudaStream_t st);
cudaError_t launch_moe_combine(const void* D, int d_dtype, int64_t M_cap, int64_t N,
                               const int32_t* token_row, const float* w, int64_t T, int k, void* out,
                               cudaStream_t st);
// Capacity of the fixed device scratch used by fp8_moe_dispatch_noalloc.
constexpr int64_t kMoeStaticWsInts = 65536;
// Address of that scratch on the current device (looked up once per device).
cudaError_t moe_static_workspace(int32_t** ws);
// Read and clear the dispatch kernels' error word (caller synchronised).
int read_and_clear_moe_status();

// Power-of-two-scale GEMM on the tensor cores' UE8M0 block scaling
// (gemm_mx.cu); same arguments as fp8_blockscaled_gemm.
// fp8_grouped_gemm's layout when group_offsets is not null.
int launch_blockscaled_gemm_mx(const uint8_t* A, const float* sA, const uint8_t* B, int b_major,
                               const float* sB, int sb_gran, int64_t M, int64_t N, int64_t K,
                               const int32_t* group_offsets, int G, void* D, int out_dtype,
                               int64_t ldd, cudaStream_t st);
// Read and clear that module's status word (caller synchronised).
int read_and_clear_mx_status();

// Synchronise `st`, then read and clear the current device's status word.
int read_and_clear_status(cudaStream_t st);

// Process-wide settings / device facts.
uint64_t wait_timeout_ns();
void set_wait_timeout_ns(uint64_t ns);
int device_sm_count();          // of the current device (cached per device)
bool device_is_sm100();         // current device is compute capability 10.x

}  // namespace fp8fg
