"""GPU parity of the block-scaled GEMM and grouped GEMM against the CPU oracle
(every output element compared), plus the device-side status word.

Tolerance (elementwise): FP32 out |gpu - ref| <= 1e-4 * T, BF16 out
<= 1e-4 * T + half a BF16 ulp, with T = sum_k |a_k b_k| of the dequantised
operands.  Operands are uniformly random finite E4M3 codes (all magnitudes
2^-9 .. 448, both signs) with log-uniform FP32 scales, so every product
range the hardware sees is exercised.
"""
import numpy as np
import pytest
import torch

import fp8_fine_grained_x1_b200 as fg
import oracle
from fp8_fine_grained_x1_b200 import synth

from gpu_util import assert_gemm_close, d2h, dev, to_dev

pytestmark = pytest.mark.gpu


def _operands(M, N, K, b_major, sb_gran, seed):
    A = synth.random_e4m3_codes((M, K), seed)
    sA = synth.random_scales((K // 128, M), seed + 1)
    if b_major == fg.B_KMAJOR:
        B = synth.random_e4m3_codes((N, K), seed + 2)
        sB = (synth.random_scales((N // 128, K // 128), seed + 3) if sb_gran == 128
              else synth.random_scales((K // 128, N), seed + 3))
    else:
        B = synth.random_e4m3_codes((K, N), seed + 2)
        sB = synth.random_scales((K // 128, N // 128), seed + 3)
    return A, sA, B, sB


def _run(A, sA, B, sB, b_major, sb_gran, out_dtype):
    D = fg.gemm(to_dev(A), to_dev(sA), to_dev(B), to_dev(sB), out_dtype=out_dtype,
                b_major=b_major, sb_gran=sb_gran)
    torch.cuda.synchronize()
    assert fg.fp8_get_status() == fg.FP8_OK
    return d2h(D)


CASES = [
    # M, N, K, b_major, sb_gran
    (128, 256, 512, fg.B_KMAJOR, 128),
    (1, 128, 128, fg.B_KMAJOR, 128),          # one row, one tile, one K-block
    (200, 384, 256, fg.B_KMAJOR, 128),        # ragged M, 128-wide tail n-tile
    (129, 512, 1024, fg.B_KMAJOR, 128),
    (256, 256, 4096, fg.B_KMAJOR, 128),       # long K: 32 promotions
    (128, 256, 256, fg.B_MNMAJOR, 128),       # Dgrad layout (B stored [K][N])
    (200, 384, 512, fg.B_MNMAJOR, 128),
    (128, 256, 512, fg.B_KMAJOR, 1),          # Wgrad layout (per-column B scales)
    (256, 384, 1024, fg.B_KMAJOR, 1),
    # 256-row tiles of CTA pairs: the odd CTA's 128 rows wholly beyond M, and
    # a last n-tile whose second 128 columns lie beyond N
    (384, 640, 384, fg.B_KMAJOR, 1),
    (384, 640, 256, fg.B_MNMAJOR, 128),
    (300, 640, 256, fg.B_KMAJOR, 128),
    # per-column B scales: N = 896 leaves the last 256-wide tile half empty
    (256, 896, 512, fg.B_KMAJOR, 1),
    (300, 1792, 640, fg.B_KMAJOR, 1),
]


@pytest.mark.parametrize("out", ["bf16", "fp32"])
@pytest.mark.parametrize("M,N,K,b_major,sb_gran", CASES)
def test_gemm_matches_oracle_everywhere(M, N, K, b_major, sb_gran, out):
    A, sA, B, sB = _operands(M, N, K, b_major, sb_gran, seed=M * 7 + N * 3 + K)
    ref, tol = oracle.gemm_full(A, sA, B, sB, b_major=b_major, sb_gran=sb_gran)
    dt = torch.bfloat16 if out == "bf16" else torch.float32
    got = _run(A, sA, B, sB, b_major, sb_gran, dt)
    assert_gemm_close(got, ref, tol, out == "bf16", f"{M}x{N}x{K} major={b_major} gran={sb_gran}")


def test_gemm_many_tiles_persistent_loop():
    """More tiles than SMs: every CTA walks several tiles (M=1280, N=4096)."""
    M, N, K = 1280, 4096, 256
    A, sA, B, sB = _operands(M, N, K, fg.B_KMAJOR, 128, seed=99)
    got = _run(A, sA, B, sB, fg.B_KMAJOR, 128, torch.float32)
    rng = np.random.default_rng(0)
    pts = np.stack([rng.integers(0, M, 20000), rng.integers(0, N, 20000)], 1)
    ref, tol = oracle.gemm_points(A, sA, B, sB, pts)
    assert_gemm_close(got[pts[:, 0], pts[:, 1]], ref, tol, False, "persistent")


def test_gemm_zero_operands_give_exact_zeros():
    M, N, K = 128, 256, 256
    A = np.zeros((M, K), np.uint8)
    A[:, ::2] = 0x80                                          # -0 codes too
    B = synth.random_e4m3_codes((N, K), 5)
    got = _run(A, synth.random_scales((K // 128, M), 1), B,
               synth.random_scales((N // 128, K // 128), 2), fg.B_KMAJOR, 128, torch.float32)
    assert np.all(got == 0.0)


def test_gemm_output_leading_dimension_and_guards():
    M, N, K, ldd = 130, 256, 256, 384
    A, sA, B, sB = _operands(M, N, K, fg.B_KMAJOR, 128, seed=11)
    Dbuf = torch.full((M, ldd), 7.0, dtype=torch.float32, device=dev())
    fg.fp8_blockscaled_gemm(to_dev(A), to_dev(sA), to_dev(B), to_dev(sB), Dbuf[:, :N])
    torch.cuda.synchronize()
    d = Dbuf.cpu().numpy()
    ref, tol = oracle.gemm_full(A, sA, B, sB)
    assert_gemm_close(d[:, :N], ref, tol, False, "ldd")
    assert np.all(d[:, N:] == 7.0)


# ------------------------------------------------------------ grouped

def _grouped_operands(counts, N, K, seed):
    """Expert-contiguous A with each group padded to 128 by zero rows."""
    G = len(counts)
    padded = [(c + 127) // 128 * 128 for c in counts]
    off = np.zeros(G + 1, np.int32)
    off[1:] = np.cumsum(padded)
    A = np.zeros((int(off[-1]), K), np.uint8)
    for e, c in enumerate(counts):
        A[off[e]:off[e] + c] = synth.random_e4m3_codes((c, K), seed + e)
    sA = synth.random_scales((K // 128, A.shape[0]), seed + 100)
    B = synth.random_e4m3_codes((G, N, K), seed + 200)
    sB = synth.random_scales((G, N // 128, K // 128), seed + 300)
    return A, sA, B, sB, off


@pytest.mark.parametrize("out", ["bf16", "fp32"])
@pytest.mark.parametrize("counts,N,K", [([130, 0, 5, 256], 256, 512),
                                        ([1, 300, 0, 0, 77], 384, 256),
                                        ([128], 128, 128)])
def test_grouped_matches_oracle(counts, N, K, out):
    A, sA, B, sB, off = _grouped_operands(counts, N, K, seed=len(counts) * 31 + N)
    M_total = A.shape[0] + 128                                # one block beyond off[G]
    A = np.concatenate([A, synth.random_e4m3_codes((128, K), 77)])
    sA = np.concatenate([sA, synth.random_scales((K // 128, 128), 78)], axis=1)
    dt = torch.bfloat16 if out == "bf16" else torch.float32
    D = torch.full((M_total, N), -3.0, dtype=dt, device=dev())
    fg.fp8_grouped_gemm(to_dev(A), to_dev(np.ascontiguousarray(sA)), to_dev(B), to_dev(sB),
                        to_dev(off), D)
    assert fg.fp8_get_status() == fg.FP8_OK
    got = d2h(D)
    pts = np.array([(m, n) for m in range(M_total) for n in range(N)], np.int64)
    ref, tol, grp = oracle.grouped_gemm_points(A, np.ascontiguousarray(sA), B, sB, off, pts)
    inside = grp >= 0
    assert_gemm_close(got.reshape(-1)[inside], ref[inside], tol[inside], out == "bf16", "grouped")
    assert np.all(got.reshape(-1)[~inside] == -3.0)           # rows beyond off[G] untouched
    pad = np.zeros(M_total, bool)                             # zero padding rows -> exact 0
    for e, c in enumerate(counts):
        pad[off[e] + c:off[e + 1]] = True
    assert np.all(got[pad] == 0.0)


@pytest.mark.parametrize("out", ["bf16", "fp32"])
def test_grouped_many_groups_across_raster_bands(out):
    """40 experts of 0..700 rows (odd and even 128-row block counts, empty
    ones): the 256-row pair blocks span several raster bands and N-blocks,
    so band boundaries fall inside and between groups.  Full output."""
    rng = np.random.default_rng(91)
    counts = [int(c) for c in rng.integers(0, 700, 40)]
    counts[3] = counts[17] = 0
    N, K = 512, 256
    A, sA, B, sB, off = _grouped_operands(counts, N, K, seed=900)
    dt = torch.bfloat16 if out == "bf16" else torch.float32
    D = torch.full((A.shape[0], N), -3.0, dtype=dt, device=dev())
    fg.fp8_grouped_gemm(to_dev(A), to_dev(sA), to_dev(B), to_dev(sB), to_dev(off), D)
    assert fg.fp8_get_status() == fg.FP8_OK
    got = d2h(D)
    mm, nn = np.meshgrid(np.arange(A.shape[0]), np.arange(N), indexing="ij")
    pts = np.stack([mm.reshape(-1), nn.reshape(-1)], axis=1).astype(np.int64)
    ref, tol, grp = oracle.grouped_gemm_points(A, sA, B, sB, off, pts)
    assert np.all(grp >= 0)
    assert_gemm_close(got.reshape(-1), ref, tol, out == "bf16", "grouped, many groups")


def test_grouped_bad_offsets_report_shape_error_and_write_nothing():
    N, K = 256, 256
    A, sA, B, sB, off = _grouped_operands([128, 128], N, K, seed=5)
    bad = off.copy()
    bad[1] = 100                                              # not a multiple of 128
    D = torch.full((A.shape[0], N), 5.0, dtype=torch.float32, device=dev())
    fg.fp8_grouped_gemm(to_dev(A), to_dev(sA), to_dev(B), to_dev(sB), to_dev(bad), D)
    assert fg.fp8_get_status() == fg.FP8_ERR_SHAPE
    assert torch.all(D == 5.0)
    assert fg.fp8_get_status() == fg.FP8_OK                   # cleared by the read


# ------------------------------------------------------------ status word

def test_bounded_wait_times_out_and_context_survives():
    fg.fp8_set_wait_timeout_ns(20_000_000)                    # 20 ms
    try:
        fg.fp8_selftest_wait_timeout()
        assert fg.fp8_get_status() == fg.FP8_ERR_TIMEOUT
        assert fg.fp8_get_status() == fg.FP8_OK
    finally:
        fg.fp8_set_wait_timeout_ns(0)                         # back to the default
    # the context is still usable
    A, sA, B, sB = _operands(128, 256, 256, fg.B_KMAJOR, 128, seed=3)
    got = _run(A, sA, B, sB, fg.B_KMAJOR, 128, torch.float32)
    ref, tol = oracle.gemm_full(A, sA, B, sB)
    assert_gemm_close(got, ref, tol, False, "after timeout")


def test_device_supported():
    assert fg.fp8_device_supported()


@pytest.mark.parametrize("sb_gran", [128, 1])
def test_stream_k_fp32_output_matches_oracle_and_is_deterministic(sb_gran):
    # 10 x 8 = 80 pair tiles on 74 pairs: the FP32 GEMM splits its K-blocks
    # evenly over the pairs, so tiles cut between two pairs get their two
    # parts added into D.  The sum of two FP32 parts onto zero does not depend
    # on their order: two runs give identical bits.
    M, N, K = 2560, 2048, 512
    A, sA, B, sB = _operands(M, N, K, fg.B_KMAJOR, sb_gran, seed=77)
    got = _run(A, sA, B, sB, fg.B_KMAJOR, sb_gran, torch.float32)
    again = _run(A, sA, B, sB, fg.B_KMAJOR, sb_gran, torch.float32)
    assert np.array_equal(got.view(np.uint64), again.view(np.uint64))
    ref, tol = oracle.gemm_full(A, sA, B, sB, sb_gran=sb_gran)
    assert_gemm_close(got, ref, tol, False, f"stream-K sb_gran={sb_gran}")
