"""Helpers shared by the GPU parity tests (not collected by pytest)."""
import numpy as np
import torch

REL_TOL = 1e-4     # |gpu - ref| <= 1e-4 * sum_k |a_k b_k|   (+ half a BF16 ulp)


def dev():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    return torch.device("cuda", 0)


def to_dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev())


def bits_to_bf16_dev(bits):
    """uint16 BF16 bit patterns -> device bfloat16 tensor."""
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev())


def half_ulp_bf16(x):
    """Half the BF16 spacing at |x| (8 significant bits; subnormals included)."""
    a = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -133)))
    return np.exp2(np.maximum(e, -126.0) - 8.0)


def gemm_bound(ref, tol, gpu, out_bf16):
    b = REL_TOL * tol
    if out_bf16:
        b = b + half_ulp_bf16(np.maximum(np.abs(ref), np.abs(gpu)))
    return b


def assert_gemm_close(gpu, ref, tol, out_bf16, what=""):
    gpu = np.asarray(gpu, np.float64)
    err = np.abs(gpu - ref)
    bound = gemm_bound(ref, tol, gpu, out_bf16)
    bad = np.flatnonzero(~(err <= bound))
    if bad.size:
        i = bad[:6]
        raise AssertionError(
            f"{what}: {bad.size}/{gpu.size} outside the bound; first: gpu={gpu.flat[i]}, "
            f"ref={np.asarray(ref).flat[i]}, tol={np.asarray(tol).flat[i]}")
    nz = tol > 0
    return float((err[nz] / tol[nz]).max()) if nz.any() else 0.0


def d2h(t):
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy()
