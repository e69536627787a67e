"""The GEMM kernels' failure path on the GPU, without a fault: a self-test
launch makes the odd CTA of every CTA pair hold back its operand loads, so
the pair's MMA waits for bytes that never come.  With a short wait limit the
wait runs out, the kernel records FP8_ERR_TIMEOUT, every role of both CTAs
unwinds (copies in flight drained, TMEM freed) and the kernel returns.  The
context must stay usable: the same GEMM, launched normally right after,
must match the oracle.

Both GEMM kernels (software promotion; power-of-two scales in the tensor
cores), dense and grouped."""
import numpy as np
import pytest
import torch

import fp8_fine_grained_x1_b200 as fg
import oracle
from fp8_fine_grained_x1_b200 import synth

from gpu_util import assert_gemm_close, d2h, dev, to_dev

pytestmark = pytest.mark.gpu


def _pow2(s):
    return np.exp2(np.round(np.log2(s))).astype(np.float32)


def _case(kernel, grouped, seed):
    K, N = 512, 384
    if grouped:
        counts = [128, 384, 0, 256]                      # an empty group, an odd 128-row count
        off = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
        G, M = len(counts), int(off[-1])
        B = synth.random_e4m3_codes((G, N, K), seed + 2)
        sB = synth.random_scales((G, N // 128, K // 128), seed + 3)
    else:
        off, G, M = None, 0, 512
        B = synth.random_e4m3_codes((N, K), seed + 2)
        sB = synth.random_scales((N // 128, K // 128), seed + 3)
    A = synth.random_e4m3_codes((M, K), seed)
    sA = synth.random_scales((K // 128, M), seed + 1)
    if kernel == 1:
        sA, sB = _pow2(sA), _pow2(sB)
    return A, sA, B, sB, off


def _normal_run(kernel, A, sA, B, sB, off):
    D = torch.zeros((A.shape[0], B.shape[-2]), dtype=torch.float32, device=dev())
    if off is None:
        f = fg.fp8_blockscaled_gemm if kernel == 0 else fg.fp8_blockscaled_gemm_pow2
        f(to_dev(A), to_dev(sA), to_dev(B), to_dev(sB), D)
    else:
        f = fg.fp8_grouped_gemm if kernel == 0 else fg.fp8_grouped_gemm_pow2
        f(to_dev(A), to_dev(sA), to_dev(B), to_dev(sB), to_dev(off), D)
    torch.cuda.synchronize()
    return D


@pytest.mark.parametrize("grouped", [False, True])
@pytest.mark.parametrize("kernel", [0, 1])
def test_gemm_wait_runs_out_unwinds_and_context_survives(kernel, grouped):
    A, sA, B, sB, off = _case(kernel, grouped, seed=60 + 2 * kernel + grouped)
    D = torch.zeros((A.shape[0], B.shape[-2]), dtype=torch.float32, device=dev())
    assert fg.fp8_get_status() == fg.FP8_OK
    fg.fp8_set_wait_timeout_ns(20_000_000)                   # 20 ms
    try:
        fg.fp8_selftest_gemm_unwind(kernel, to_dev(A), to_dev(sA), to_dev(B), to_dev(sB), D,
                                    None if off is None else to_dev(off))
        assert fg.fp8_get_status() == fg.FP8_ERR_TIMEOUT
        assert fg.fp8_get_status() == fg.FP8_OK
    finally:
        fg.fp8_set_wait_timeout_ns(0)                         # back to the default
    got = d2h(_normal_run(kernel, A, sA, B, sB, off))
    assert fg.fp8_get_status() == fg.FP8_OK
    if off is None:
        ref, tol = oracle.gemm_full(A, sA, B, sB)
    else:
        M, N = got.shape
        pts = np.array([(m, n) for m in range(M) for n in range(N)], np.int64)
        ref, tol, _ = oracle.grouped_gemm_points(A, sA, B, sB, off, pts)
        ref, tol = ref.reshape(M, N), tol.reshape(M, N)
    assert_gemm_close(got, ref, tol, False, f"kernel {kernel} after the unwind")


def test_unwind_self_test_rejects_bad_arguments():
    A, sA, B, sB, _ = _case(0, False, seed=70)
    D = torch.zeros((A.shape[0], B.shape[0]), dtype=torch.float32, device=dev())
    lib = fg.load_library()
    # kernel id outside {0, 1}
    rc = lib.fp8_selftest_gemm_unwind(2, to_dev(A).data_ptr(), to_dev(sA).data_ptr(),
                                      to_dev(B).data_ptr(), to_dev(sB).data_ptr(), None, 0,
                                      A.shape[0], B.shape[0], 512, D.data_ptr(), fg.OUT_FP32, None)
    assert rc == fg.FP8_ERR_DTYPE
    # a single K-block has no second load to hold back
    rc = lib.fp8_selftest_gemm_unwind(0, to_dev(A).data_ptr(), to_dev(sA).data_ptr(),
                                      to_dev(B).data_ptr(), to_dev(sB).data_ptr(), None, 0,
                                      A.shape[0], B.shape[0], 128, D.data_ptr(), fg.OUT_FP32, None)
    assert rc == fg.FP8_ERR_SHAPE
