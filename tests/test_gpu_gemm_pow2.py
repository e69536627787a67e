"""GPU parity of fp8_blockscaled_gemm_pow2 (power-of-two scales applied by the
tensor cores' UE8M0 block scaling) against the CPU oracle's FP64 block-scaled
sum, within the same bound as the software-promoted GEMM: FP32 out
|gpu - ref| <= 1e-4 * sum_k |s_a s_b a_k b_k|, BF16 out plus half a BF16 ulp.
Operands are quantized by the oracle in power-of-two mode.
"""
import numpy as np
import pytest
import torch

import fp8_fine_grained_x1_b200 as fg
import oracle
from fp8_fine_grained_x1_b200 import synth

from gpu_util import assert_gemm_close, d2h, dev, to_dev

pytestmark = pytest.mark.gpu
P2 = oracle.SCALE_POW2


def _operands(M, N, K, seed, b_major=oracle.B_KMAJOR):
    x = synth.activations(M, K, seed=seed, outlier_seed=seed + 1).float().numpy()
    w = synth.normal((N, K), 0.02, seed + 2).float().numpy()
    qa, sa = oracle.quant_act_1x128(x, P2)
    qw, sw = oracle.quant_w_128x128(w, P2)
    if b_major == oracle.B_MNMAJOR:
        # a weight stored [K][N] (the Dgrad orientation): quantize W^T in
        # 128x128 blocks; its scales are then [K/128][N/128]
        qw, sw = oracle.quant_w_128x128(np.ascontiguousarray(w.T), P2)
    return qa, sa, qw, sw


def _run(qa, sa, qb, sb, N, b_major=fg.B_KMAJOR, gran=128, out=torch.float32):
    M = qa.shape[0]
    D = torch.full((M, N), float("nan"), dtype=out, device=dev())
    fg.fp8_blockscaled_gemm_pow2(to_dev(qa), to_dev(sa), to_dev(qb), to_dev(sb), D, b_major, gran)
    torch.cuda.synchronize()
    assert fg.fp8_get_status() == fg.FP8_OK
    return d2h(D)


@pytest.mark.parametrize("out", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("M,N,K", [(128, 256, 512), (200, 384, 640), (384, 512, 1024)])
def test_pow2_gemm_kmajor_full_output(M, N, K, out):
    qa, sa, qw, sw = _operands(M, N, K, seed=M + N)
    got = _run(qa, sa, qw, sw, N, out=out)
    ref, tol = oracle.gemm_full(qa, sa, qw, sw)
    assert_gemm_close(got, ref, tol, out == torch.bfloat16, f"pow2 {M}x{N}x{K}")


def test_pow2_gemm_mnmajor_weight():
    M, N, K = 256, 384, 512
    qa, sa, qw, sw = _operands(M, N, K, seed=5, b_major=oracle.B_MNMAJOR)
    got = _run(qa, sa, qw, sw, N, b_major=fg.B_MNMAJOR, out=torch.bfloat16)
    ref, tol = oracle.gemm_full(qa, sa, qw, sw, b_major=oracle.B_MNMAJOR)
    assert_gemm_close(got, ref, tol, True, "pow2 MN-major")


def test_pow2_gemm_per_column_scales():
    """Wgrad form: both operands 128x1 along the inner (token) axis."""
    T, C_out, C_in = 512, 256, 384
    x = synth.activations(T, C_in, seed=7, outlier_seed=8).float().numpy()
    dy = synth.normal((T, C_out), 1e-3, 9).float().numpy()
    qx, sx = oracle.quant_act_128x1(x, P2)
    qdy, sdy = oracle.quant_act_128x1(dy, P2)
    got = _run(qdy, sdy, qx, sx, C_in, gran=1)
    ref, tol = oracle.gemm_full(qdy, sdy, qx, sx, sb_gran=1)
    assert_gemm_close(got, ref, tol, False, "pow2 per-column")


def test_pow2_gemm_long_k_against_software_promotion():
    """K = 8192 (the Wgrad reduction length) with wide scale spread."""
    M, N, K = 128, 256, 8192
    qa, sa, qw, sw = _operands(M, N, K, seed=11)
    got = _run(qa, sa, qw, sw, N)
    ref, tol = oracle.gemm_full(qa, sa, qw, sw)
    err = assert_gemm_close(got, ref, tol, False, "pow2 K=8192")
    assert err < 1.0


def test_pow2_gemm_reports_non_power_of_two_scale():
    M, N, K = 128, 256, 256
    qa, sa, qw, sw = _operands(M, N, K, seed=13)
    sa = sa.copy()
    sa[1, 5] = np.float32(0.75)
    D = torch.empty((M, N), dtype=torch.float32, device=dev())
    fg.fp8_blockscaled_gemm_pow2(to_dev(qa), to_dev(sa), to_dev(qw), to_dev(sw), D)
    assert fg.fp8_get_status() == fg.FP8_ERR_VALUE
    assert fg.fp8_get_status() == fg.FP8_OK


@pytest.mark.parametrize("row", [5, 200])
def test_pow2_gemm_reports_bad_scale_in_either_half_of_a_pair_tile(row):
    """Rows 0-127 and 128-255 of a 256-row tile are scaled by different CTAs;
    a non-power-of-two scale in either is reported."""
    M, N, K = 256, 256, 256
    qa, sa, qw, sw = _operands(M, N, K, seed=17)
    sa = sa.copy()
    sa[1, row] = np.float32(3.0)
    D = torch.empty((M, N), dtype=torch.float32, device=dev())
    fg.fp8_blockscaled_gemm_pow2(to_dev(qa), to_dev(sa), to_dev(qw), to_dev(sw), D)
    assert fg.fp8_get_status() == fg.FP8_ERR_VALUE
    assert fg.fp8_get_status() == fg.FP8_OK


def _pow2(s):
    """Nearest power of two of each positive scale (test input construction)."""
    return np.exp2(np.round(np.log2(s))).astype(np.float32)


def _grouped_pow2_operands(counts, N, K, seed):
    G = len(counts)
    off = np.zeros(G + 1, np.int32)
    off[1:] = np.cumsum([(c + 127) // 128 * 128 for c in counts])
    A = np.zeros((int(off[-1]), K), np.uint8)
    for e, c in enumerate(counts):
        A[off[e]:off[e] + c] = synth.random_e4m3_codes((c, K), seed + e)
    sA = _pow2(synth.random_scales((K // 128, A.shape[0]), seed + 100))
    B = synth.random_e4m3_codes((G, N, K), seed + 200)
    sB = _pow2(synth.random_scales((G, N // 128, K // 128), seed + 300))
    return A, sA, B, sB, off


@pytest.mark.parametrize("out", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("counts,N,K", [([130, 0, 5, 256], 256, 512), ([1, 300, 0, 0, 77], 384, 256)])
def test_pow2_grouped_matches_oracle(counts, N, K, out):
    A, sA, B, sB, off = _grouped_pow2_operands(counts, N, K, seed=len(counts) * 17 + N)
    M_total = A.shape[0] + 128                                # one block beyond off[G]
    A = np.concatenate([A, synth.random_e4m3_codes((128, K), 71)])
    sA = np.ascontiguousarray(np.concatenate([sA, np.ones((K // 128, 128), np.float32)], axis=1))
    D = torch.full((M_total, N), -3.0, dtype=out, device=dev())
    fg.fp8_grouped_gemm_pow2(to_dev(A), to_dev(sA), to_dev(B), to_dev(sB), to_dev(off), D)
    assert fg.fp8_get_status() == fg.FP8_OK
    got = d2h(D)
    pts = np.array([(m, n) for m in range(M_total) for n in range(N)], np.int64)
    ref, tol, grp = oracle.grouped_gemm_points(A, sA, B, sB, off, pts)
    inside = grp >= 0
    assert_gemm_close(got.reshape(-1)[inside], ref[inside], tol[inside], out == torch.bfloat16,
                      "pow2 grouped")
    assert np.all(got.reshape(-1)[~inside] == -3.0)           # rows beyond off[G] untouched


def test_pow2_grouped_bad_offsets_report_shape_error_and_write_nothing():
    A, sA, B, sB, off = _grouped_pow2_operands([128, 128], 256, 256, seed=5)
    bad = off.copy()
    bad[1] = 100                                              # not a multiple of 128
    D = torch.full((A.shape[0], 256), 5.0, dtype=torch.float32, device=dev())
    fg.fp8_grouped_gemm_pow2(to_dev(A), to_dev(sA), to_dev(B), to_dev(sB), to_dev(bad), D)
    assert fg.fp8_get_status() == fg.FP8_ERR_SHAPE
    assert torch.all(D == 5.0)
