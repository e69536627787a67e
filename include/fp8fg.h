/*
 * fp8fg.h -- C ABI of libfp8fg: the fine-grained FP8 Linear operator on B200
 * (sm_100a).  Online E4M3 quantization (1x128 activation tiles, 128x1
 * token-axis tiles for Wgrad, 128x128 weight blocks) and the block-scaled
 * E4M3 x E4M3 GEMM with FP32 promotion of every 128-element K partial, for
 * Fprop, Dgrad, Wgrad and MoE grouped Fprop.
 *
 * Sources (web pages reproducing the DeepSeek-V3 report's FP8 training
 * section; cited by page title, or by host where the page has no title, and
 * by the figure or passage):
 *   [P1] "5 Ways You can get More Deepseek While Spending Less"
 *        (xn--jj0bz6z98ct0a29q.com) -- power-of-2 scaling factors; max-abs
 *        mapped to the FP8 maximum; per-group scaling along the GEMM inner
 *        dimension; promotion every 128 elements (four WGMMAs) to FP32 on
 *        CUDA cores; Figure 6 (Fprop, Dgrad, Wgrad in FP8); 1x128 FP8 tiles
 *        cached for backward; K = 4096 limited-accumulation error.
 *   [P2] why-be.co.kr board post -- Figure 7 (a): 1x128 activation tiles and
 *        128x128 weight blocks; promotion to FP32 registers.
 *   [P3] cameseeing.com community post -- Figure 7 (a); max-abs computed
 *        online per 1x128 tile / 128x128 block, scale derived, cast online.
 *   [P4] "Three Fast Methods To Study Deepseek" -- E4M3 on all tensors;
 *        Figure 7 (a); MoE layer shapes (expert hidden size 2048, top-8).
 *   [P5] gnrental.net free-board post -- GEMMs take FP8 inputs and give BF16
 *        or FP32 outputs; two WGMMAs in flight so promotion overlaps MMA;
 *        128 BF16 activations read from HBM, FP8 written back, read again.
 *
 * Conventions shared by every entry point
 *   - Every tensor pointer is caller-owned DEVICE memory on the current CUDA
 *     device (e.g. PyTorch-allocated).  The library allocates nothing and
 *     keeps no per-call state; its only global state is two status words per
 *     device (__device__ variables: one for the GEMM, one for the MoE
 *     dispatch) and a host-side wait time limit.
 *   - Per-device set-up (kernel attributes, device addresses of the
 *     library's __device__ arrays) happens at the first call on a device and
 *     is kept for the process; it does not survive cudaDeviceReset().
 *   - All calls are asynchronous on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream).  None synchronises except fp8_get_status().
 *   - Arguments are validated on the host before anything is launched; on a
 *     validation error the call returns its code, launches nothing and
 *     writes nothing.  Launch failures return FP8_ERR_LAUNCH.
 *   - Errors found on the device (a bounded wait that ran out, malformed
 *     group offsets) are recorded in the status word; read and clear it with
 *     fp8_get_status().
 *   - Outputs must not alias inputs.  Pointers must be 16-byte aligned and
 *     leading dimensions multiples of 16 bytes.
 *   - Entry points are reentrant; concurrent calls on different streams are
 *     safe as long as their outputs do not overlap.
 *   - E4M3 is OCP E4M3FN: 1 sign, 4 exponent (bias 7), 3 mantissa bits; max
 *     finite 448; codes are stored one per byte.
 */
#ifndef FP8FG_H
#define FP8FG_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes. */
enum fp8_status {
    FP8_OK = 0,
    FP8_ERR_NULL = 1,     /* a required pointer is NULL                          */
    FP8_ERR_SHAPE = 2,    /* size <= 0 where not allowed, not a multiple of 128,
                             overflow, ld too small, bad group offsets (device)  */
    FP8_ERR_ALIGN = 3,    /* pointer or leading dimension not 16-byte aligned    */
    FP8_ERR_DTYPE = 4,    /* unknown dtype / mode / major / granularity enum     */
    FP8_ERR_LAUNCH = 5,   /* the CUDA launch failed (cudaGetLastError)           */
    FP8_ERR_TIMEOUT = 6,  /* a bounded device-side wait gave up (status word)    */
    FP8_ERR_DEVICE = 7,   /* no CUDA device, or not an sm_100 (B200-class) GPU   */
    FP8_ERR_VALUE = 8     /* a scale given to fp8_blockscaled_gemm_pow2 is not a
                             positive normal power of two (status word)          */
};

enum { FP8_IN_BF16 = 0, FP8_IN_FP32 = 1 };          /* quantizer input dtype   */
enum { FP8_OUT_BF16 = 0, FP8_OUT_FP32 = 1 };        /* GEMM output dtype       */
enum { FP8_SCALE_FP32 = 0, FP8_SCALE_POW2 = 1 };    /* scale mode              */
enum { FP8_B_KMAJOR = 0, FP8_B_MNMAJOR = 1 };       /* layout of GEMM operand B */

/*
 * Group scale (all three quantizers), per group of 128 or 128x128 elements
 * with max-abs `amax` ([P1] max-abs -> FP8 max; [P3] online max-abs):
 *   FP8_SCALE_FP32: s = fl32(amax / 448); codes E(fl32(x * fl32(448 / amax))).
 *                   amax == 0 gives s = 1 (codes +-0); amax < 1.75*2^-118
 *                   (amax/448 below FLT_MIN) gives s = 2^-126, codes E(x*2^126).
 *   FP8_SCALE_POW2: s = 2^e, e the least integer with amax <= 448 * 2^e,
 *                   clamped to e >= -126 ([P1] integral power-of-2 scales);
 *                   codes E(x * 2^-e), exact scaling.  amax == 0 gives s = 1.
 * E() rounds to nearest even and saturates to +-448.  Dequantisation is
 * code * s.
 */

/*
 * 1x128 activation tiles: one scale per token (row) per 128 consecutive
 * channels ([P2]/[P3]/[P4] Figure 7 (a); [P1] FP8 tiles cached for backward).
 *   x    [M][ldx] input, row-major, dtype in_dtype (BF16 or FP32)
 *   q    [M][ldq] E4M3 codes (uint8), same positions as x
 *   sA   [K/128][M] FP32 scales, sA[kb*M + m] for x[m][kb*128 .. +127]
 *        ("K-block-major": the M scales of one K-block are contiguous)
 * Sizes: M >= 0 (M == 0 launches nothing), K > 0 and K % 128 == 0,
 * ldx >= K, ldq >= K.
 */
int fp8_quant_act_1x128(const void* x, int in_dtype, int64_t M, int64_t K, int64_t ldx,
                        uint8_t* q, int64_t ldq, float* sA, int scale_mode, void* stream);

/*
 * 128x1 tiles along tokens for the Wgrad operands: one scale per channel
 * per 128 consecutive tokens, so that the groups run along the Wgrad GEMM's
 * inner dimension (tokens) as [P1] asks of every FP8 GEMM operand.  The
 * output is written transposed so the token axis is contiguous (K-major
 * operand of fp8_blockscaled_gemm).
 *   x    [T][ldx] input (token-major), BF16 or FP32
 *   qT   [C][ldqT] E4M3 codes, qT[c][t] is the code of x[t][c]
 *   s    [T/128][C] FP32 scales, s[tb*C + c] for x[tb*128 .. +127][c]
 * Sizes: T > 0 and T % 128 == 0; C >= 0 and C % 8 == 0 (C == 0 launches
 * nothing); ldx >= C, ldqT >= T.
 */
int fp8_quant_act_128x1(const void* x, int in_dtype, int64_t T, int64_t C, int64_t ldx,
                        uint8_t* qT, int64_t ldqT, float* s, int scale_mode, void* stream);

/*
 * Requantization of activations cached in FP8 for the backward pass ([P5]:
 * the FP8 Wgrad GEMM lets activations be stored in FP8 for backward; [P2]/
 * [P3]: activations cached and dispatched in FP8 with the fine-grained
 * grouping).  The cache holds 1x128 tiles (fp8_quant_act_1x128's output);
 * Wgrad needs 128x1 groups along tokens.  Each code is dequantized to
 * fl32(decode(q) * sA) -- one FP32 rounding -- and those values are
 * quantized exactly as fp8_quant_act_128x1 quantizes an FP32 input.
 *   q    [T][ldq] E4M3 codes, sA [C/128][T] FP32 scales (sA[cb*T + t])
 *   qT   [C][ldqT] E4M3 codes, s [T/128][C] FP32 scales (as fp8_quant_act_128x1)
 * Sizes: T > 0, T % 128 == 0, T/128 <= 65535; C >= 0, C % 128 == 0 (C == 0
 * launches nothing); ldq >= C and ldqT >= T, both multiples of 16; q and qT
 * 16-byte aligned, sA and s 4-byte aligned.  All buffers are caller-owned
 * device memory; argument errors return before any launch.  One kernel.
 */
int fp8_requant_1x128_to_128x1(const uint8_t* q, int64_t ldq, const float* sA, int64_t T,
                               int64_t C, uint8_t* qT, int64_t ldqT, float* s, int scale_mode,
                               void* stream);

/*
 * 128x128 weight blocks: one scale per 128 output x 128 input channels
 * ([P2]/[P3]/[P4] Figure 7 (a)).
 *   w    [N][ldw] input, row-major, BF16 or FP32
 *   q    [N][ldq] E4M3 codes
 *   sW   [N/128][K/128] FP32 scales, sW[nb*(K/128) + kb]
 * Sizes: N >= 0, N % 128 == 0; K > 0, K % 128 == 0; ldw >= K, ldq >= K.
 */
int fp8_quant_w_128x128(const void* w, int in_dtype, int64_t N, int64_t K, int64_t ldw,
                        uint8_t* q, int64_t ldq, float* sW, int scale_mode, void* stream);

/*
 * Block-scaled FP8 GEMM  D[m][n] = sum_kb sA[kb][m] * sB(n, kb) * P(m, n, kb)
 * with P the E4M3 x E4M3 dot product over K-block kb (128 elements) computed
 * on the tensor cores and promoted to an FP32 running sum every 128 K
 * ([P1]/[P2]/[P5] increased-precision accumulation, N_C = 128; [P1]
 * per-group scales along the inner dimension; [P5] FP8 in, BF16/FP32 out;
 * [P1] Figure 6: used for Fprop, Dgrad and Wgrad).
 *   A    [M][K] E4M3, row-major (K contiguous)
 *   sA   [K/128][M] FP32 (as written by fp8_quant_act_1x128 / _128x1)
 *   B    b_major == FP8_B_KMAJOR : [N][K] E4M3 (K contiguous), e.g. the
 *                                   quantized weight W[N][K] in Fprop or a
 *                                   128x1-quantized qT in Wgrad;
 *        b_major == FP8_B_MNMAJOR: [K][N] E4M3 (N contiguous), e.g. the
 *                                   forward weight W[K][N] read transposed
 *                                   in Dgrad ([P5] transposed operand reads)
 *   sB   sb_gran == 128: 128x128 block scales of the stored B:
 *                        K-major [N/128][K/128], MN-major [K/128][N/128];
 *        sb_gran == 1  : per-column scales [K/128][N] (K-major B only)
 *   D    [M][ldd] row-major, BF16 (round to nearest even) or FP32
 * Sizes: M >= 0 (0 launches nothing); N > 0, N % 128 == 0; K > 0,
 * K % 128 == 0; ldd >= N.
 */
int fp8_blockscaled_gemm(const uint8_t* A, const float* sA, const uint8_t* B, int b_major,
                         const float* sB, int sb_gran, int64_t M, int64_t N, int64_t K, void* D,
                         int out_dtype, int64_t ldd, void* stream);

/*
 * fp8_blockscaled_gemm for power-of-two scales (FP8_SCALE_POW2 quantizers;
 * [P1]: integral power-of-2 scaling factors), with the scaling done inside
 * the tensor cores: each scale 2^e becomes the UE8M0 block-scale factor of
 * a tcgen05.mma.kind::mxf8f6f4.block_scale, so the per-128-K partials are
 * accumulated in the MMA's FP32 accumulator with their scales applied
 * ([P5]: the hardware ask for Tensor Cores that take group scales and keep
 * full-precision accumulation), and no partial is promoted by software.
 * The result is the same sum as fp8_blockscaled_gemm's (up to rounding
 * order).  Arguments, layouts, sizes and errors as fp8_blockscaled_gemm;
 * additionally every sA / sB value must be 2^e with -126 <= e <= 127: any
 * other value is used as 1 and reported as FP8_ERR_VALUE through the status
 * word.
 */
int fp8_blockscaled_gemm_pow2(const uint8_t* A, const float* sA, const uint8_t* B, int b_major,
                              const float* sB, int sb_gran, int64_t M, int64_t N, int64_t K,
                              void* D, int out_dtype, int64_t ldd, void* stream);

/*
 * fp8_grouped_gemm for power-of-two scales, scaled inside the tensor cores
 * as fp8_blockscaled_gemm_pow2 does ([P1] power-of-2 scales; [P5] the MoE
 * part reads one expert's weights per group).  Arguments, layouts, sizes and
 * errors as fp8_grouped_gemm; every sA / sB value must be 2^e with
 * -126 <= e <= 127, else FP8_ERR_VALUE through the status word.
 */
int fp8_grouped_gemm_pow2(const uint8_t* A, const float* sA, const uint8_t* B, const float* sB,
                          const int32_t* group_offsets, int G, int64_t M_total, int64_t N, int64_t K,
                          void* D, int out_dtype, void* stream);

/*
 * Grouped (MoE expert) block-scaled GEMM: rows [off[e], off[e+1]) of A are
 * multiplied by expert e's weight ([P4] MoE layer; [P5] each group only
 * loads the parameters of one expert).
 *   A        [M_total][K] E4M3, rows grouped by expert, zero rows as padding
 *   sA       [K/128][M_total] FP32
 *   B        [G][N][K] E4M3 (K-major per expert)
 *   sB       [G][N/128][K/128] FP32
 *   group_offsets  [G+1] int32 in DEVICE memory: off[0] == 0, non-decreasing,
 *            every entry a multiple of 128, off[G] <= M_total.  Empty groups
 *            are allowed.  Checked on the device: malformed offsets record
 *            FP8_ERR_SHAPE in the status word and nothing is written.
 *   D        [M_total][N] (row stride N), BF16 or FP32; rows at or beyond
 *            off[G] are left untouched.
 * Sizes: G >= 1; M_total >= 0 and M_total % 128 == 0; N > 0, N % 128 == 0;
 * K > 0, K % 128 == 0.
 */
int fp8_grouped_gemm(const uint8_t* A, const float* sA, const uint8_t* B, const float* sB,
                     const int32_t* group_offsets, int G, int64_t M_total, int64_t N, int64_t K,
                     void* D, int out_dtype, void* stream);

/*
 * fp8_grouped_gemm with A gathered from per-token rows instead of read from
 * an expert-ordered copy ([P1]/[P3] MoE activations move in FP8; [P5] each
 * group loads one expert's weights): output row m of D is the product of A
 * row row_token[m] with its expert's weight, so the dispatched rows are never
 * written to memory.  The tensor cores read the rows through TMA gathers.
 * It saves the k-fold copy of the token rows in HBM (and the traffic of
 * writing it) but not time: a K-block's 128 rows take 32 four-row gathers
 * where a tiled load takes one TMA operation, and on the MoE workload (16384
 * tokens, top-8, 32 experts, N = 2048, K = 7168) this GEMM ran 2.3x as long
 * as fp8_grouped_gemm on the dispatched rows.
 *   A        [T][K] E4M3 codes of the tokens (1x128 groups), row-major
 *   sA       [K/128][T] FP32, their scales
 *   row_token [M_total] int32 in DEVICE memory: the A row of each output row,
 *            -1 for padding rows, whose output is 0 (fp8_moe_route's
 *            row_token has this layout).  An entry below -1 or at or beyond T
 *            is treated as padding and records FP8_ERR_SHAPE.
 *   B, sB, group_offsets, G, M_total, N, K, D, out_dtype as fp8_grouped_gemm.
 * Sizes: as fp8_grouped_gemm, plus 1 <= T <= 2^31 - 1 when M_total > 0.
 * row_token 4-byte aligned.  One kernel launch.
 */
int fp8_grouped_gemm_gather(const uint8_t* A, const float* sA, int64_t T, const int32_t* row_token,
                            const uint8_t* B, const float* sB, const int32_t* group_offsets, int G,
                            int64_t M_total, int64_t N, int64_t K, void* D, int out_dtype,
                            void* stream);

/*
 * FP8 dispatch of MoE activations ([P1]/[P3] cache and dispatch activations
 * in FP8; [P4] top-8 routing): rows of 1x128-quantized tokens, with their
 * scales, are gathered into expert-contiguous groups, each padded with zero
 * rows to a multiple of 128 -- the A operand of fp8_grouped_gemm.  Pairs
 * (token t, slot j) are ordered by expert, then by t, then by j (a stable
 * counting sort), so the layout is deterministic.
 *   q          [T][K] E4M3 codes of the tokens, sA [K/128][T] FP32 scales
 *              (as written by fp8_quant_act_1x128)
 *   topk       [T][k] int32 expert ids in [0, G), device memory
 *   q_out      [M_cap][K] E4M3, sA_out [K/128][M_cap] FP32: expert-ordered
 *              rows; padding rows and rows at or beyond group_offsets[G]
 *              get codes 0 and scale 1 (exactly a quantized zero row)
 *   group_offsets [G+1] int32: first row of each group, group_offsets[G] =
 *              padded total (device memory, written)
 *   token_row  [T][k] int32: destination row of each pair (for the combine)
 *   row_token  [M_cap] int32: source token of each row, -1 for padding
 *   workspace  caller-owned device scratch of fp8_moe_dispatch_workspace_bytes
 *              bytes (per-chunk expert counts); contents on entry ignored
 * Sizes: T >= 0; K > 0, K % 128 == 0; 1 <= k; 1 <= G <= 1024; T*k <=
 * 2^31 - 1 - 1024*128 (so every padded row index fits in int32); M_cap >= 0
 * and M_cap % 128 == 0; q and q_out 16-byte aligned, the rest 4-byte
 * aligned.  Argument errors return FP8_ERR_SHAPE / NULL / ALIGN before any
 * launch.  A padded total above M_cap, or an expert id outside
 * [0, G), is reported as FP8_ERR_SHAPE through the status word; such pairs get
 * token_row -1 and are not copied.  Launches four kernels and one memset.
 */
int64_t fp8_moe_dispatch_workspace_bytes(int64_t T, int k, int G);
int fp8_moe_dispatch(const uint8_t* q, const float* sA, int64_t T, int64_t K, const int32_t* topk,
                     int k, int G, uint8_t* q_out, float* sA_out, int64_t M_cap,
                     int32_t* group_offsets, int32_t* token_row, int32_t* row_token,
                     void* workspace, int64_t workspace_bytes, void* stream);

/*
 * The routing half of fp8_moe_dispatch alone: group_offsets, token_row and
 * row_token exactly as fp8_moe_dispatch writes them, and no rows moved (for
 * fp8_grouped_gemm_gather, which reads the token rows through row_token).
 * Arguments, sizes, workspace and errors as fp8_moe_dispatch without q, sA,
 * K, q_out and sA_out.  Launches three kernels and one memset.
 */
int fp8_moe_route(const int32_t* topk, int64_t T, int k, int G, int64_t M_cap,
                  int32_t* group_offsets, int32_t* token_row, int32_t* row_token, void* workspace,
                  int64_t workspace_bytes, void* stream);

/*
 * 1x128 quantization of the tokens fused with their FP8 dispatch ([P5]
 * hardware passage: 128 BF16 activations are read from HBM, quantized, the
 * FP8 values written back and read again -- here the codes go straight to
 * the expert-ordered rows; [P1]/[P3] dispatch in FP8; [P4] top-8 routing).
 * Writes exactly what fp8_quant_act_1x128 followed by fp8_moe_dispatch
 * writes into q_out, sA_out, group_offsets, token_row and row_token (the
 * per-token codes q / sA are not produced).
 *   x          [T][ldx] BF16 or FP32 tokens (in_dtype FP8_IN_*), row-major
 *   scale_mode FP8_SCALE_FP32 or FP8_SCALE_POW2, as fp8_quant_act_1x128
 *   the other arguments as fp8_moe_dispatch (same workspace size)
 * Sizes: as fp8_moe_dispatch, plus ldx >= K and ldx * element size a
 * multiple of 16 bytes; x 16-byte aligned.  Errors as fp8_moe_dispatch.
 * Launches five kernels and one memset: three routing passes, the fused
 * quantizer, and a pass that fills the padding rows.
 */
int fp8_moe_quant_dispatch(const void* x, int in_dtype, int64_t T, int64_t K, int64_t ldx,
                           const int32_t* topk, int k, int G, uint8_t* q_out, float* sA_out,
                           int64_t M_cap, int32_t* group_offsets, int32_t* token_row,
                           int32_t* row_token, void* workspace, int64_t workspace_bytes,
                           int scale_mode, void* stream);

/*
 * fp8_moe_dispatch without a caller workspace: the same dispatch, writing
 * the same outputs, with its scratch in a fixed device array of
 * FP8_MOE_NOALLOC_WS_BYTES inside the library (one per device, held by every
 * device that loads the library until the process exits).  The pages have
 * no counterpart.  It is for callers that cannot allocate device memory:
 * code whose device memory is all handed out by a framework's own pool and
 * that has no allocator to ask for scratch, and code that must not call
 * cudaMalloc because cudaMalloc can synchronise the device in the middle of
 * its queued work.  The call allocates nothing (no cudaMalloc, no library
 * routine that allocates); the caller still passes inputs and outputs.
 *   Limit: fp8_moe_dispatch_workspace_bytes(T, k, G) <= FP8_MOE_NOALLOC_WS_BYTES
 *          (e.g. T*k <= 2^21 pairs at G = 32), else FP8_ERR_SHAPE.
 *   Set-up: the first call in a CUDA context looks the array's device
 *   address up (cudaGetSymbolAddress with the device current); a call from
 *   another context looks it up again.
 *   Calls that overlap on one device (other streams, other threads) share
 *   the array and race: serialise them.  Every scratch entry a call reads is
 *   written earlier in the same call, so nothing needs clearing between
 *   calls.  Other arguments, errors and launches as fp8_moe_dispatch.
 */
#define FP8_MOE_NOALLOC_WS_BYTES 262144
int fp8_moe_dispatch_noalloc(const uint8_t* q, const float* sA, int64_t T, int64_t K,
                             const int32_t* topk, int k, int G, uint8_t* q_out, float* sA_out,
                             int64_t M_cap, int32_t* group_offsets, int32_t* token_row,
                             int32_t* row_token, void* stream);

/*
 * Weighted combine of the expert outputs back to token order:
 *   out[t][n] = BF16( sum_j w[t][j] * D[token_row[t][j]][n] )  (FP32 sums in
 * slot order; pairs whose token_row is outside [0, M_cap), e.g. -1, are
 * skipped).
 *   D          [M_cap][N] BF16 or FP32 (d_dtype FP8_OUT_*), the grouped GEMM
 *              output; token_row [T][k] int32 from fp8_moe_dispatch;
 *   weights    [T][k] FP32 gate weights; out [T][N] BF16
 * Sizes: T >= 0, k >= 1, N > 0 and N % 8 == 0; D and out 16-byte aligned.
 * All buffers are caller-owned device memory.  One kernel launch.
 */
int fp8_moe_combine(const void* D, int d_dtype, int64_t M_cap, int64_t N, const int32_t* token_row,
                    const float* weights, int64_t T, int k, void* out, void* stream);

/*
 * Synchronise `stream`, then return and clear the current device's status
 * word (FP8_OK if no kernel reported an error since the last call).  Returns
 * FP8_ERR_DEVICE if the status cannot be read.
 */
int fp8_get_status(void* stream);

/* Human-readable name of a return code (static string, never NULL). */
const char* fp8_status_string(int code);

/*
 * Time limit, in nanoseconds, of every device-side wait of kernels launched
 * after this call (default 4e9).  0 restores the default.  Not thread-safe
 * with respect to concurrent launches; meant for tests and debugging.
 */
void fp8_set_wait_timeout_ns(uint64_t ns);

/*
 * Self-test of the bounded-wait machinery: launches one CTA that waits on an
 * mbarrier nothing ever arrives at, with the current time limit.  The kernel
 * gives up after the limit, records FP8_ERR_TIMEOUT and returns normally, so
 * fp8_get_status() afterwards reports FP8_ERR_TIMEOUT and the context stays
 * usable.  Returns FP8_OK if the launch succeeded.
 */
int fp8_selftest_wait_timeout(void* stream);

/*
 * Self-test of the GEMMs' unwinding after a wait runs out (no counterpart in
 * the pages; it exercises the failure path of the kernels that do the work).
 * Launches the promotion GEMM (kernel 0, fp8_blockscaled_gemm /
 * fp8_grouped_gemm) or the tensor-core-scaled one (kernel 1,
 * fp8_blockscaled_gemm_pow2 / fp8_grouped_gemm_pow2) -- grouped when
 * group_offsets is not NULL -- with the odd CTA of every CTA pair holding
 * back its operand loads after its first K-block.  The pair's MMA then waits
 * for bytes that never come: the wait runs into its time limit
 * (fp8_set_wait_timeout_ns), FP8_ERR_TIMEOUT is recorded in the status word,
 * and every role of both CTAs unwinds (copies in flight drained, TMEM
 * freed) and returns, leaving the context usable.  D is left partly written.
 * Arguments as fp8_blockscaled_gemm with B K-major and per-block scales
 * (ldd = N) or as fp8_grouped_gemm; K >= 256, so that a second K-block
 * exists.  Returns FP8_OK if the launch succeeded.
 */
int fp8_selftest_gemm_unwind(int kernel, const uint8_t* A, const float* sA, const uint8_t* B,
                             const float* sB, const int32_t* group_offsets, int G, int64_t M,
                             int64_t N, int64_t K, void* D, int out_dtype, void* stream);

/* 1 if the current device is an sm_100 GPU the library runs on, else 0. */
int fp8_device_supported(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8FG_H */
