"""Pins of the oracle's block-scaled GEMM, grouped GEMM and the
limited-accumulation emulation.

What the pages fix ("Increasing accumulation precision"): per-group scaling
factors along the GEMM inner dimension; every N_C = 128 elements of K the
partial result is moved out of the Tensor Cores, multiplied by its scaling
factors and accumulated in FP32; outputs BF16 or FP32.  The oracle computes
the same sum in FP64.  Independent references here:
  * exact rational arithmetic (fractions.Fraction) on tiny problems;
  * integer-valued E4M3 codes with unit scales == an int64 matmul, exactly;
  * dequantise -> torch.matmul in float64 (a library GEMM);
  * for the emulation: the exact dot product, and the pages' qualitative
    statement that without promotion K = 4096 reaches percent-level error.
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

TAB = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn) \
    .to(torch.float64).numpy()
FINITE = np.array([c for c in range(256) if not np.isnan(TAB[c])], np.uint8)


def rand_codes(rng, shape):
    return FINITE[rng.integers(0, len(FINITE), shape)]


def rand_scales(rng, shape):
    return np.exp2(rng.uniform(-12, 4, shape)).astype(np.float32)


def exact_gemm(A, sA, Bnk, sB_of):
    """Exact rational sum_k (sA*qa) * (sB*qb) and sum_k |...| over all k.
    Bnk[n][k] codes; sB_of(n, kb) the scale of B in block kb for column n."""
    M, K = A.shape
    N = Bnk.shape[0]
    ref = [[Fraction(0)] * N for _ in range(M)]
    tol = [[Fraction(0)] * N for _ in range(M)]
    for m in range(M):
        for n in range(N):
            acc = Fraction(0)
            t = Fraction(0)
            for k in range(K):
                a = Fraction(float(sA[k // 128, m])) * Fraction(TAB[A[m, k]])
                b = Fraction(float(sB_of(n, k // 128))) * Fraction(TAB[Bnk[n, k]])
                acc += a * b
                t += abs(a * b)
            ref[m][n] = acc
            tol[m][n] = t
    return ref, tol


def _check_exact(ref, tol, eref, etol):
    M, N = ref.shape
    for m in range(M):
        for n in range(N):
            t = float(etol[m][n])
            assert abs(Fraction(ref[m, n]) - eref[m][n]) <= Fraction(2.0 ** -48) * etol[m][n]
            assert abs(Fraction(tol[m, n]) - etol[m][n]) <= Fraction(2.0 ** -48) * etol[m][n]
            assert t >= 0


@pytest.mark.parametrize("K", [128, 256])
def test_kmajor_gran128_equals_exact_rationals(K):
    rng = np.random.default_rng(K)
    M, N = 3, 4
    A = rand_codes(rng, (M, K))
    B = rand_codes(rng, (N, K))
    sA = rand_scales(rng, (K // 128, M))
    sB = rand_scales(rng, (1, K // 128))                     # N < 128: one row of blocks
    ref, tol = oracle.gemm_full(A, sA, B, sB)
    eref, etol = exact_gemm(A, sA, B, lambda n, kb: sB[n // 128, kb])
    _check_exact(ref, tol, eref, etol)


def test_mnmajor_gran128_equals_exact_rationals():
    rng = np.random.default_rng(3)
    M, N, K = 2, 3, 256
    A = rand_codes(rng, (M, K))
    W = rand_codes(rng, (K, N))                               # stored [K][N]
    sW = rand_scales(rng, (K // 128, 1))                      # [K/128][N/128]
    ref, tol = oracle.gemm_full(A, sA := rand_scales(rng, (K // 128, M)), W, sW,
                                b_major=oracle.B_MNMAJOR)
    eref, etol = exact_gemm(A, sA, np.ascontiguousarray(W.T), lambda n, kb: sW[kb, n // 128])
    _check_exact(ref, tol, eref, etol)


def test_gran1_per_column_scales_equal_exact_rationals():
    rng = np.random.default_rng(4)
    M, N, K = 3, 5, 256
    A = rand_codes(rng, (M, K))
    B = rand_codes(rng, (N, K))
    sA = rand_scales(rng, (K // 128, M))
    sB = rand_scales(rng, (K // 128, N))                      # [K/128][N]
    ref, tol = oracle.gemm_full(A, sA, B, sB, sb_gran=1)
    eref, etol = exact_gemm(A, sA, B, lambda n, kb: sB[kb, n])
    _check_exact(ref, tol, eref, etol)


def test_integer_codes_with_unit_scales_equal_int64_matmul():
    rng = np.random.default_rng(5)
    ints = {int(TAB[c]): c for c in FINITE if TAB[c] == np.round(TAB[c]) and abs(TAB[c]) <= 16}
    vals = np.array(sorted(ints))
    M, N, K = 16, 24, 512
    Av = vals[rng.integers(0, len(vals), (M, K))]
    Bv = vals[rng.integers(0, len(vals), (N, K))]
    A = np.vectorize(ints.get)(Av).astype(np.uint8)
    B = np.vectorize(ints.get)(Bv).astype(np.uint8)
    ref, tol = oracle.gemm_full(A, np.ones((K // 128, M), np.float32), B,
                                np.ones((1, K // 128), np.float32))
    exact = Av.astype(np.int64) @ Bv.astype(np.int64).T
    assert np.array_equal(ref, exact.astype(np.float64))
    assert np.array_equal(tol, (np.abs(Av) @ np.abs(Bv).T).astype(np.float64))


def test_matches_library_float64_matmul_of_dequantised_operands():
    rng = np.random.default_rng(6)
    M, N, K = 64, 256, 1024
    A = rand_codes(rng, (M, K))
    B = rand_codes(rng, (N, K))
    sA = rand_scales(rng, (K // 128, M))
    sB = rand_scales(rng, (N // 128, K // 128))
    ref, tol = oracle.gemm_full(A, sA, B, sB)
    a = torch.from_numpy(TAB[A] * np.repeat(sA.T.astype(np.float64), 128, axis=1))
    b = torch.from_numpy(TAB[B] * np.kron(sB.astype(np.float64), np.ones((128, 128))))
    lib = (a @ b.T).numpy()
    lib_t = (a.abs() @ b.abs().T).numpy()
    assert np.all(np.abs(ref - lib) <= 1e-12 * tol)
    assert np.allclose(tol, lib_t, rtol=1e-12, atol=0)


def test_points_equal_full_and_orientations_agree():
    rng = np.random.default_rng(7)
    M, N, K = 128, 256, 512
    A = rand_codes(rng, (M, K))
    B = rand_codes(rng, (N, K))
    sA = rand_scales(rng, (K // 128, M))
    sB = rand_scales(rng, (N // 128, K // 128))
    ref, tol = oracle.gemm_full(A, sA, B, sB)
    # MN-major storage of the same operand with its block scales transposed
    ref2, tol2 = oracle.gemm_full(A, sA, np.ascontiguousarray(B.T), np.ascontiguousarray(sB.T),
                                  b_major=oracle.B_MNMAJOR)
    assert np.array_equal(ref, ref2) and np.array_equal(tol, tol2)
    # per-column scales replicated from the block scales
    sB1 = np.repeat(sB.T, 128, axis=1)                        # [K/128][N]
    ref3, _ = oracle.gemm_full(A, sA, B, np.ascontiguousarray(sB1), sb_gran=1)
    assert np.array_equal(ref, ref3)
    pts = np.stack([rng.integers(0, M, 300), rng.integers(0, N, 300)], 1)
    r, t = oracle.gemm_points(A, sA, B, sB, pts)
    assert np.array_equal(r, ref[pts[:, 0], pts[:, 1]]) and np.array_equal(t, tol[pts[:, 0], pts[:, 1]])


def test_grouped_equals_per_group_dense_and_skips_rows_outside_groups():
    rng = np.random.default_rng(8)
    G, N, K = 3, 256, 256
    off = np.array([0, 128, 128, 384], np.int32)              # expert 1 is empty
    M_total = 512                                             # rows 384.. are in no group
    A = rand_codes(rng, (M_total, K))
    sA = rand_scales(rng, (K // 128, M_total))
    B = rand_codes(rng, (G, N, K))
    sB = rand_scales(rng, (G, N // 128, K // 128))
    pts = np.array([(m, n) for m in range(0, M_total, 7) for n in range(0, N, 37)], np.int64)
    ref, tol, grp = oracle.grouped_gemm_points(A, sA, B, sB, off, pts)
    for e in range(G):
        lo, hi = off[e], off[e + 1]
        sel = (pts[:, 0] >= lo) & (pts[:, 0] < hi)
        assert np.all(grp[sel] == e)
        if hi > lo:
            dref, dtol = oracle.gemm_full(A[lo:hi], np.ascontiguousarray(sA[:, lo:hi]), B[e], sB[e])
            p = pts[sel]
            assert np.array_equal(ref[sel], dref[p[:, 0] - lo, p[:, 1]])
            assert np.array_equal(tol[sel], dtol[p[:, 0] - lo, p[:, 1]])
    out = pts[:, 0] >= off[-1]
    assert np.all(grp[out] == -1) and np.all(ref[out] == 0) and np.all(tol[out] == 0)


def test_grouped_tiny_equals_exact_rationals():
    rng = np.random.default_rng(9)
    G, N, K = 2, 2, 128
    off = np.array([0, 2, 3], np.int32)
    A = rand_codes(rng, (3, K))
    sA = rand_scales(rng, (1, 3))
    B = rand_codes(rng, (G, N, K))
    sB = rand_scales(rng, (G, 1, 1))
    pts = np.array([(m, n) for m in range(3) for n in range(N)], np.int64)
    ref, tol, grp = oracle.grouped_gemm_points(A, sA, B, sB, off, pts)
    for i, (m, n) in enumerate(pts):
        e = 0 if m < 2 else 1
        eref, etol = exact_gemm(A[m:m + 1], sA[:, m:m + 1], B[e][n:n + 1],
                                lambda nn, kb: sB[e, 0, kb])
        assert grp[i] == e
        assert abs(Fraction(ref[i]) - eref[0][0]) <= Fraction(2.0 ** -48) * etol[0][0]


# ---------------------------------------------------------------- limited accumulation

def test_limited_dot_with_full_width_is_exact():
    rng = np.random.default_rng(10)
    a = rand_codes(rng, 4096)
    b = rand_codes(rng, 4096)
    exact = sum(Fraction(TAB[x]) * Fraction(TAB[y]) for x, y in zip(a, b))
    assert Fraction(oracle.limited_dot(a, b, 53, 0)) == exact


def _positive_codes(rng, n):
    """E4M3 codes of U(0,1) values scaled so the max maps near 448."""
    v = rng.uniform(0, 1, n).astype(np.float32) * np.float32(448.0)
    return oracle.e4m3_encode_array(v)


def test_limited_accumulation_degrades_without_promotion_at_k4096():
    """The pages: K = 4096 with limited Tensor-Core accumulation precision
    gives a max relative error near 2%; promotion every 128 elements to FP32
    removes most of it.  Reproduced qualitatively with a 13-bit truncating
    accumulator (the width is not on the pages)."""
    rng = np.random.default_rng(11)
    K, rows = 4096, 64
    err_plain, err_prom = [], []
    for _ in range(rows):
        a = _positive_codes(rng, K)
        b = _positive_codes(rng, K)
        exact = float(sum(Fraction(TAB[x]) * Fraction(TAB[y]) for x, y in zip(a, b)))
        err_plain.append(abs(oracle.limited_dot(a, b, 13, 0) - exact) / exact)
        err_prom.append(abs(oracle.limited_dot(a, b, 13, 128) - exact) / exact)
    assert 5e-3 < max(err_plain) < 5e-2           # percent level, as on the pages
    assert max(err_prom) < max(err_plain) / 10    # promotion every 128 fixes most of it
    # more bits -> smaller error, monotonically (a sanity pin on the truncation)
    a = _positive_codes(rng, K)
    b = _positive_codes(rng, K)
    exact = float(sum(Fraction(TAB[x]) * Fraction(TAB[y]) for x, y in zip(a, b)))
    errs = [abs(oracle.limited_dot(a, b, m, 0) - exact) / exact for m in range(10, 17)]
    assert all(e1 >= e2 for e1, e2 in zip(errs, errs[1:]))
