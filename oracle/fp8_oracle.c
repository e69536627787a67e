/*
 * fp8_oracle.c -- plain, slow CPU oracle for the fine-grained FP8 Linear.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py may load this code.  It shares no
 * code, header, table or constant generator with the CUDA library under
 * fp8_fine_grained_x1_b200/csrc, and it imports nothing from it.
 *
 * Source: "DeepSeek-V3 technical report, FP8 training" as reproduced on five
 * web pages (the pages paste the report's Section 3.3 "FP8 Training"):
 *   - "Fine-grained quantization" (Figure 7 (a)): activations are grouped
 *     and scaled per 1x128 tile (one token, 128 channels); weights per
 *     128x128 block (128 input x 128 output channels).
 *   - "Online quantization": the max-abs of each tile/block is computed
 *     online, a scaling factor is derived from it and the tensor is cast to
 *     FP8 online.
 *   - Standard practice cited there (Narang et al., 2017): the max-abs value
 *     of a group is scaled to the largest representable FP8 value.
 *   - "E4M3 on all tensors" (Mixed precision framework, Figure 6): Fprop,
 *     Dgrad and Wgrad all take E4M3 inputs; GEMM outputs are BF16 or FP32.
 *   - "Increasing accumulation precision": per-group scales along the GEMM
 *     inner dimension; partial results are promoted to FP32 every N_C = 128
 *     elements of K (four WGMMAs) where they are scaled and accumulated.
 *   - Integral power-of-2 scaling factors are used for some activations
 *     (Linear after attention; activation gradient before MoE down-proj).
 *
 * Readings where the pages are silent:
 *   R1  stored scale s is the dequantisation multiplier amax/448; values are
 *       encoded as E(fl32(x * fl32(448/amax))).  All scale arithmetic is
 *       correctly rounded FP32 (the precision of the stored scale).
 *   R2  FP8 cast rounds to nearest, ties to even, saturating to +-448.
 *   R3  amax == 0: s = 1 and every code is +-0.
 *   R3b amax/448 below the smallest normal FP32 (amax < 1.75 * 2^-118):
 *       s = 2^-126 and inv = 2^126 (the scale saturates at FLT_MIN instead of
 *       overflowing 448/amax).
 *   R4  power-of-2 mode: s = 2^e with e the least integer such that
 *       amax <= 448 * 2^e, clamped to e >= -126; codes E(x * 2^-e) exactly.
 *   R5  GEMM reference: sum over K-blocks of sA * sB * P in FP64, with P the
 *       exact FP64 dot product of the decoded E4M3 values inside the block.
 *   R13 requantizing cached 1x128 FP8 activations for Wgrad: each element is
 *       dequantized to fl32(decode(q) * sA) (the exact product rounded once
 *       to FP32), and those FP32 values are quantized in 128x1 groups
 *       exactly as an FP32 input would be.
 *
 * Every routine is single-purpose and written straight from the definition;
 * OpenMP only splits independent outputs across threads.
 */
#include <math.h>
#include <stdint.h>
#include <stddef.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_API __attribute__((visibility("default")))

/* ------------------------------------------------------------------ */
/* E4M3 (OCP "E4M3FN") scalar format: 1 sign, 4 exponent (bias 7), 3     */
/* mantissa bits; no infinities; S.1111.111 is NaN; max finite 448.      */
/* ------------------------------------------------------------------ */

/* Value of one E4M3 byte, straight from the bit fields. NaN for 0x7F/0xFF. */
ORACLE_API double oracle_e4m3_decode(uint8_t b)
{
    int sign = (b >> 7) & 1;
    int ex = (b >> 3) & 0xF;
    int man = b & 7;
    double mag;
    if (ex == 15 && man == 7) return NAN;
    if (ex == 0)
        mag = ldexp((double)man / 8.0, -6);          /* subnormal: m/8 * 2^-6 */
    else
        mag = ldexp(1.0 + (double)man / 8.0, ex - 7); /* normal */
    return sign ? -mag : mag;
}

/* Round a non-negative real r to the nearest integer, ties to the even one. */
static double round_half_even(double r)
{
    double f = floor(r);
    double frac = r - f;          /* exact for the r used here */
    if (frac > 0.5) return f + 1.0;
    if (frac < 0.5) return f;
    return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;
}

/*
 * Encode a real value v to the nearest E4M3 value (ties to even mantissa),
 * saturating magnitudes above 448 to 448, keeping the sign of zero (and of
 * a negative value that rounds to zero).  NaN encodes to 0x7F.
 */
ORACLE_API uint8_t oracle_e4m3_encode(double v)
{
    uint8_t sign;
    double a, code;
    int e;
    if (isnan(v)) return 0x7F;
    sign = signbit(v) ? 0x80 : 0x00;
    a = fabs(v);
    if (a >= 448.0) return (uint8_t)(sign | 0x7E);    /* satfinite */
    if (a < ldexp(1.0, -6)) {
        /* subnormal spacing 2^-9: code = round(a / 2^-9); code 8 is 2^-6,
         * the first normal, whose byte is also 8 (exponent 1, mantissa 0). */
        code = round_half_even(ldexp(a, 9));
        return (uint8_t)(sign | (uint8_t)code);
    }
    /* normal: a = m * 2^e with m in [1, 2), e in [-6, 8] */
    (void)frexp(a, &e);
    e -= 1;
    code = round_half_even((ldexp(a, -e) - 1.0) * 8.0); /* mantissa 0..8 */
    if (code == 8.0) { code = 0.0; e += 1; }
    return (uint8_t)(sign | (uint8_t)(((e + 7) << 3) | (int)code));
}

/* Encode an array of FP32 values one by one with oracle_e4m3_encode(). */
ORACLE_API void oracle_e4m3_encode_array(const float* v, int64_t n, uint8_t* out)
{
    int64_t i;
#pragma omp parallel for schedule(static)
    for (i = 0; i < n; i++) out[i] = oracle_e4m3_encode((double)v[i]);
}

/* ------------------------------------------------------------------ */
/* Group scale (reading R1-R4).                                        */
/* ------------------------------------------------------------------ */

enum { ORACLE_SCALE_FP32 = 0, ORACLE_SCALE_POW2 = 1 };

/*
 * From a group's max-abs (an FP32 value) derive
 *   *s     the stored FP32 scale (dequantisation multiplier), and
 *   *inv   the FP32 factor the group's elements are multiplied by before
 *          the E4M3 cast (FP32 mode), or
 *   *e_out the exponent e with s = 2^e (POW2 mode).
 */
static void group_scale(float amax, int mode, float* s, float* inv, int* e_out)
{
    const float fp8_max = 448.0f;
    if (mode == ORACLE_SCALE_POW2) {
        int e;
        if (amax == 0.0f) { *s = 1.0f; *inv = 1.0f; *e_out = 0; return; }
        /* least integer e with amax <= 448 * 2^e; comparisons are exact in
         * double because 448 * 2^e and amax are both representable. */
        e = 0;
        while (448.0 * ldexp(1.0, e) < (double)amax) e++;
        while (448.0 * ldexp(1.0, e - 1) >= (double)amax) e--;
        if (e < -126) e = -126;
        *s = (float)ldexp(1.0, e);
        *inv = (float)ldexp(1.0, -e);
        *e_out = e;
        return;
    }
    if (amax == 0.0f) { *s = 1.0f; *inv = 1.0f; *e_out = 0; return; }
    if ((double)amax < 1.75 * ldexp(1.0, -118)) {   /* amax/448 < FLT_MIN */
        *s = (float)ldexp(1.0, -126);
        *inv = (float)ldexp(1.0, 126);
        *e_out = 0;
        return;
    }
    /* FP32 divisions, correctly rounded (SSE arithmetic, no contraction) */
    {
        volatile float a = amax;
        *inv = fp8_max / a;
        *s = a / fp8_max;
    }
    *e_out = 0;
}

/* Encode one element of a group whose scale was set by group_scale(). */
static uint8_t encode_scaled(float x, int mode, float inv, int e)
{
    if (mode == ORACLE_SCALE_POW2)
        return oracle_e4m3_encode(ldexp((double)x, -e));   /* exact scaling */
    {
        volatile float y = x * inv;                         /* fl32 product  */
        return oracle_e4m3_encode((double)y);
    }
}

/* Input element readers: BF16 is the upper half of an FP32 bit pattern. */
enum { ORACLE_IN_BF16 = 0, ORACLE_IN_FP32 = 1 };

static float load_elem(const void* base, int dtype, int64_t idx)
{
    if (dtype == ORACLE_IN_FP32) return ((const float*)base)[idx];
    {
        uint32_t bits = (uint32_t)((const uint16_t*)base)[idx] << 16;
        float f;
        memcpy(&f, &bits, 4);
        return f;
    }
}

/* Quantise the elements idx[0..n) of one group: amax, scale, codes. */
static float quantize_group(const void* x, int dtype, const int64_t* in_idx,
                            uint8_t* q, const int64_t* out_idx, int n, int mode)
{
    float amax = 0.0f, s, inv;
    int i, e;
    for (i = 0; i < n; i++) {
        float a = fabsf(load_elem(x, dtype, in_idx[i]));
        if (a > amax) amax = a;
    }
    group_scale(amax, mode, &s, &inv, &e);
    for (i = 0; i < n; i++)
        q[out_idx[i]] = encode_scaled(load_elem(x, dtype, in_idx[i]), mode, inv, e);
    return s;
}

/*
 * 1x128 activation tiles (one token, 128 consecutive channels).
 *   x   [M][ldx] elements, row-major; groups x[m][kb*128 .. kb*128+127]
 *   q   [M][ldq] bytes, same positions
 *   sA  [K/128][M] floats ("kb-major": sA[kb*M + m])
 */
ORACLE_API void oracle_quant_act_1x128(const void* x, int dtype, int64_t M, int64_t K,
                                       int64_t ldx, uint8_t* q, int64_t ldq, float* sA,
                                       int mode)
{
    int64_t nkb = K / 128, g;
#pragma omp parallel for schedule(static)
    for (g = 0; g < M * nkb; g++) {
        int64_t m = g / nkb, kb = g % nkb, in_idx[128], out_idx[128];
        int i;
        for (i = 0; i < 128; i++) {
            in_idx[i] = m * ldx + kb * 128 + i;
            out_idx[i] = m * ldq + kb * 128 + i;
        }
        sA[kb * M + m] = quantize_group(x, dtype, in_idx, q, out_idx, 128, mode);
    }
}

/*
 * 128x1 tiles along tokens, for the Wgrad operands (inner dimension = tokens).
 *   x   [T][ldx] elements, row-major (token-major)
 *   qT  [C][ldqT] bytes: qT[c][t] = code of x[t][c]   (tokens contiguous)
 *   s   [T/128][C] floats: s[tb*C + c] scales x[tb*128 .. tb*128+127][c]
 */
ORACLE_API void oracle_quant_act_128x1(const void* x, int dtype, int64_t T, int64_t C,
                                       int64_t ldx, uint8_t* qT, int64_t ldqT, float* s,
                                       int mode)
{
    int64_t ntb = T / 128, g;
#pragma omp parallel for schedule(static)
    for (g = 0; g < ntb * C; g++) {
        int64_t tb = g / C, c = g % C, in_idx[128], out_idx[128];
        int i;
        for (i = 0; i < 128; i++) {
            in_idx[i] = (tb * 128 + i) * ldx + c;
            out_idx[i] = c * ldqT + tb * 128 + i;
        }
        s[tb * C + c] = quantize_group(x, dtype, in_idx, qT, out_idx, 128, mode);
    }
}

/*
 * Backward-pass requantization of activations cached in FP8 (gnrental.net
 * post, mixed precision framework: the FP8 Wgrad GEMM lets activations be
 * stored in FP8 for the backward pass; why-be.co.kr and cameseeing.com
 * posts: activations are cached in FP8 with the fine-grained grouping).
 * The cached form is 1x128 (per token, 128 channels); Wgrad wants 128x1
 * groups along tokens.  Reading R13: dequantize, then group again.
 *   q   [T][ldq] E4M3 codes of the 1x128 tiles; sA [C/128][T] floats
 *       (sA[cb*T + t]); codes 0x7F/0xFF (NaN) are outside the domain
 *   qT  [C][ldqT] bytes, s [T/128][C] floats: as oracle_quant_act_128x1
 */
ORACLE_API void oracle_requant_1x128_to_128x1(const uint8_t* q, int64_t ldq, const float* sA,
                                              int64_t T, int64_t C, uint8_t* qT, int64_t ldqT,
                                              float* s, int mode)
{
    int64_t ntb = T / 128, g;
#pragma omp parallel for schedule(static)
    for (g = 0; g < ntb * C; g++) {
        int64_t tb = g / C, c = g % C, in_idx[128], out_idx[128];
        float xs[128];
        int i;
        for (i = 0; i < 128; i++) {
            int64_t t = tb * 128 + i;
            /* decode(q) has 4 significant bits, sA 24: the FP64 product is
             * exact, so the cast is the single FP32 rounding of R13 */
            xs[i] = (float)(oracle_e4m3_decode(q[t * ldq + c]) * (double)sA[(c / 128) * T + t]);
            in_idx[i] = i;
            out_idx[i] = c * ldqT + t;
        }
        s[tb * C + c] = quantize_group(xs, ORACLE_IN_FP32, in_idx, qT, out_idx, 128, mode);
    }
}

/*
 * 128x128 weight blocks.
 *   w   [N][ldw] elements, row-major
 *   q   [N][ldq] bytes
 *   sW  [N/128][K/128] floats: sW[nb*(K/128) + kb]
 */
ORACLE_API void oracle_quant_w_128x128(const void* w, int dtype, int64_t N, int64_t K,
                                       int64_t ldw, uint8_t* q, int64_t ldq, float* sW,
                                       int mode)
{
    int64_t nkb = K / 128, nnb = N / 128, g;
#pragma omp parallel for schedule(static)
    for (g = 0; g < nnb * nkb; g++) {
        int64_t nb = g / nkb, kb = g % nkb;
        static __thread int64_t in_idx[128 * 128], out_idx[128 * 128];
        int r, c;
        for (r = 0; r < 128; r++)
            for (c = 0; c < 128; c++) {
                in_idx[r * 128 + c] = (nb * 128 + r) * ldw + kb * 128 + c;
                out_idx[r * 128 + c] = (nb * 128 + r) * ldq + kb * 128 + c;
            }
        sW[nb * nkb + kb] = quantize_group(w, dtype, in_idx, q, out_idx, 128 * 128, mode);
    }
}

/* ------------------------------------------------------------------ */
/* Block-scaled GEMM reference (reading R5).                           */
/* ------------------------------------------------------------------ */

enum { ORACLE_B_KMAJOR = 0, ORACLE_B_MNMAJOR = 1 };

typedef struct {
    const uint8_t* A; int64_t lda; const float* sA; int64_t M;   /* A[m][k], sA[kb][m] */
    const uint8_t* B; int64_t ldb; int b_major;                   /* B(n,k)             */
    const float* sB; int sb_gran;                                 /* see b_scale()      */
    int64_t N, K;
} gemm_args;

static uint8_t a_code(const gemm_args* g, int64_t m, int64_t k) { return g->A[m * g->lda + k]; }

/* B(n, k): K-major stores B[n][k]; MN-major stores B[k][n] (a weight W[K][N]). */
static uint8_t b_code(const gemm_args* g, int64_t n, int64_t k)
{
    return g->b_major == ORACLE_B_KMAJOR ? g->B[n * g->ldb + k] : g->B[k * g->ldb + n];
}

/*
 * Scale of B for output column n in K-block kb.
 *   sb_gran == 128, K-major : sB[N/128][K/128]  (128x128 blocks of B[N][K])
 *   sb_gran == 128, MN-major: sB[K/128][N/128]  (128x128 blocks of W[K][N])
 *   sb_gran == 1            : sB[K/128][N]      (128x1 groups, per column)
 */
static double b_scale(const gemm_args* g, int64_t n, int64_t kb)
{
    int64_t nkb = g->K / 128;
    if (g->sb_gran == 1) return g->sB[kb * g->N + n];
    if (g->b_major == ORACLE_B_KMAJOR) return g->sB[(n / 128) * nkb + kb];
    return g->sB[kb * ((g->N + 127) / 128) + n / 128];   /* ceil: tiny N < 128 too */
}

/* ref = sum_kb sA*sB*P_kb, P_kb exact in FP64; tol_scale = sum_k |a_k * b_k|
 * with a_k, b_k the dequantised operands (sA*dec(qa), sB*dec(qb)).         */
static void gemm_point(const gemm_args* g, int64_t m, int64_t n, double* ref, double* tol)
{
    double acc = 0.0, t = 0.0;
    int64_t kb, nkb = g->K / 128;
    for (kb = 0; kb < nkb; kb++) {
        double p = 0.0, pabs = 0.0, scale;
        int64_t k;
        for (k = kb * 128; k < kb * 128 + 128; k++) {
            double prod = oracle_e4m3_decode(a_code(g, m, k)) * oracle_e4m3_decode(b_code(g, n, k));
            p += prod;                 /* exact: <= 8 significant bits per term */
            pabs += fabs(prod);
        }
        scale = (double)g->sA[kb * g->M + m] * b_scale(g, n, kb);
        acc += scale * p;
        t += fabs(scale) * pabs;
    }
    *ref = acc;
    *tol = t;
}

/*
 * Reference outputs at npts points (pts[2i], pts[2i+1]) = (m, n).
 * ref[i] is the FP64 reference, tol[i] = sum_k |a_k b_k| (the tolerance scale).
 */
ORACLE_API void oracle_gemm_points(const uint8_t* A, int64_t lda, const float* sA, int64_t M,
                                   const uint8_t* B, int64_t ldb, int b_major,
                                   const float* sB, int sb_gran, int64_t N, int64_t K,
                                   const int64_t* pts, int64_t npts, double* ref, double* tol)
{
    gemm_args g = {A, lda, sA, M, B, ldb, b_major, sB, sb_gran, N, K};
    int64_t i;
#pragma omp parallel for schedule(dynamic, 64)
    for (i = 0; i < npts; i++)
        gemm_point(&g, pts[2 * i], pts[2 * i + 1], &ref[i], &tol[i]);
}

/* Full M x N reference (small problems only). */
ORACLE_API void oracle_gemm_full(const uint8_t* A, int64_t lda, const float* sA, int64_t M,
                                 const uint8_t* B, int64_t ldb, int b_major,
                                 const float* sB, int sb_gran, int64_t N, int64_t K,
                                 double* ref, double* tol)
{
    gemm_args g = {A, lda, sA, M, B, ldb, b_major, sB, sb_gran, N, K};
    int64_t i;
#pragma omp parallel for schedule(dynamic, 16)
    for (i = 0; i < M * N; i++)
        gemm_point(&g, i / N, i % N, &ref[i], &tol[i]);
}

/*
 * Grouped (MoE) GEMM reference at sampled points.  Rows [off[e], off[e+1])
 * of A belong to expert e and are multiplied by B_e = B + e*N*K (K-major,
 * [N][K]) with scales sB_e = sB + e*(N/128)*(K/128).  Rows outside every
 * group get ref = tol = 0 and group id -1.
 */
ORACLE_API void oracle_grouped_gemm_points(const uint8_t* A, int64_t lda, const float* sA,
                                           int64_t M_total, const uint8_t* B, const float* sB,
                                           const int32_t* off, int G, int64_t N, int64_t K,
                                           const int64_t* pts, int64_t npts, double* ref,
                                           double* tol, int32_t* group_of_point)
{
    int64_t i;
#pragma omp parallel for schedule(dynamic, 64)
    for (i = 0; i < npts; i++) {
        int64_t m = pts[2 * i], n = pts[2 * i + 1];
        int e, found = -1;
        for (e = 0; e < G; e++)
            if (m >= off[e] && m < off[e + 1]) { found = e; break; }
        group_of_point[i] = found;
        if (found < 0) { ref[i] = 0.0; tol[i] = 0.0; continue; }
        {
            gemm_args g = {A, lda, sA, M_total,
                           B + (int64_t)found * N * K, K, ORACLE_B_KMAJOR,
                           sB + (int64_t)found * ((N + 127) / 128) * (K / 128), 128, N, K};
            gemm_point(&g, m, n, &ref[i], &tol[i]);
        }
    }
}

/* ------------------------------------------------------------------ */
/* Limited-precision accumulation emulation ("Increasing accumulation  */
/* precision": a K = 4096 GEMM with Tensor-Core accumulation of limited */
/* width reaches about 2% max relative error).                          */
/* ------------------------------------------------------------------ */

/* Keep the top `bits` significant bits of v (round toward zero). */
static double truncate_mantissa(double v, int bits)
{
    int e;
    double f;
    if (v == 0.0 || bits >= 53) return v;
    f = frexp(v, &e);                      /* v = f * 2^e, |f| in [0.5, 1) */
    f = trunc(ldexp(f, bits));             /* keep `bits` bits            */
    return ldexp(f, e - bits);
}

/*
 * Dot product of two E4M3 code rows of length K (scales 1), accumulated the
 * way a limited-precision MMA unit would: each K=32 MMA step's 32 products
 * are summed exactly and added to the accumulator, which is then truncated
 * to `bits` mantissa bits.
 *   promote_every == 0 : one accumulator over all of K (no promotion)
 *   promote_every  > 0 : every `promote_every` elements the limited
 *                        accumulator is added to an FP32 running sum and
 *                        restarted from zero (promotion, N_C = promote_every)
 */
ORACLE_API double oracle_limited_dot(const uint8_t* a, const uint8_t* b, int64_t K, int bits,
                                     int promote_every)
{
    double acc = 0.0;
    float sum32 = 0.0f;
    int64_t k0, k;
    for (k0 = 0; k0 < K; k0 += 32) {
        double step = 0.0;
        for (k = k0; k < k0 + 32 && k < K; k++)
            step += oracle_e4m3_decode(a[k]) * oracle_e4m3_decode(b[k]);
        acc = truncate_mantissa(acc + step, bits);
        if (promote_every > 0 && (k0 + 32) % promote_every == 0) {
            sum32 = sum32 + (float)acc;
            acc = 0.0;
        }
    }
    if (promote_every > 0) return (double)(sum32 + (float)acc);
    return acc;
}

ORACLE_API int oracle_num_threads(void)
{
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
