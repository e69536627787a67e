"""fp8_fine_grained_x1_b200 -- the fine-grained FP8 Linear operator on B200.

A thin Python binding over the C-ABI library ``libfp8fg.so`` (declared in
``include/fp8fg.h``).  Every function here only marshals arguments -- torch
tensors become device pointers, sizes and the current CUDA stream -- and
checks the return code; all arithmetic runs in the library's CUDA kernels.
There is no CPU fallback: if the library is missing or the device is not an
sm_100 GPU, the calls raise.

Entry points (same names as the C ABI):
  fp8_quant_act_1x128(x, q, sA, scale_mode=SCALE_FP32)
  fp8_quant_act_128x1(x, qT, s, scale_mode=SCALE_FP32)
  fp8_quant_w_128x128(w, q, sW, scale_mode=SCALE_FP32)
  fp8_blockscaled_gemm(A, sA, B, sB, D, b_major=B_KMAJOR, sb_gran=128)
  fp8_grouped_gemm(A, sA, B, sB, group_offsets, D)
  fp8_get_status(), fp8_set_wait_timeout_ns(ns), fp8_selftest_wait_timeout()
plus allocating conveniences quant_act_1x128 / quant_act_128x1 / quant_w_128x128
/ gemm / grouped_gemm that create the output tensors with torch first.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libfp8fg.so")

FP8_OK = 0
FP8_ERR_NULL = 1
FP8_ERR_SHAPE = 2
FP8_ERR_ALIGN = 3
FP8_ERR_DTYPE = 4
FP8_ERR_LAUNCH = 5
FP8_ERR_TIMEOUT = 6
FP8_ERR_DEVICE = 7
FP8_ERR_VALUE = 8

IN_BF16, IN_FP32 = 0, 1
OUT_BF16, OUT_FP32 = 0, 1
SCALE_FP32, SCALE_POW2 = 0, 1
B_KMAJOR, B_MNMAJOR = 0, 1

EXPORTED = (
    "fp8_quant_act_1x128", "fp8_quant_act_128x1", "fp8_quant_w_128x128",
    "fp8_blockscaled_gemm", "fp8_grouped_gemm", "fp8_get_status", "fp8_status_string",
    "fp8_set_wait_timeout_ns", "fp8_selftest_wait_timeout", "fp8_device_supported",
    "fp8_moe_dispatch_workspace_bytes", "fp8_moe_dispatch", "fp8_moe_combine",
    "fp8_moe_dispatch_noalloc", "fp8_requant_1x128_to_128x1", "fp8_blockscaled_gemm_pow2",
    "fp8_grouped_gemm_pow2", "fp8_moe_quant_dispatch", "fp8_selftest_gemm_unwind",
    "fp8_grouped_gemm_gather", "fp8_moe_route",
)


class Fp8Error(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_string(code)} (code {code})")


_lib = None
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libfp8fg.so (build it with ``python -m fp8_fine_grained_x1_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libfp8fg.so not found at {path}; build it with "
                           "`python -m fp8_fine_grained_x1_b200.build` (there is no fallback)")
    lib = ctypes.CDLL(path)
    q = [_P, _I, _I64, _I64, _I64, _P, _I64, _P, _I, _P]
    for name in ("fp8_quant_act_1x128", "fp8_quant_act_128x1", "fp8_quant_w_128x128"):
        getattr(lib, name).argtypes = q
        getattr(lib, name).restype = _I
    lib.fp8_blockscaled_gemm.argtypes = [_P, _P, _P, _I, _P, _I, _I64, _I64, _I64, _P, _I, _I64, _P]
    lib.fp8_blockscaled_gemm.restype = _I
    lib.fp8_blockscaled_gemm_pow2.argtypes = [_P, _P, _P, _I, _P, _I, _I64, _I64, _I64, _P, _I,
                                              _I64, _P]
    lib.fp8_blockscaled_gemm_pow2.restype = _I
    lib.fp8_grouped_gemm_pow2.argtypes = [_P, _P, _P, _P, _P, _I, _I64, _I64, _I64, _P, _I, _P]
    lib.fp8_grouped_gemm_pow2.restype = _I
    lib.fp8_grouped_gemm.argtypes = [_P, _P, _P, _P, _P, _I, _I64, _I64, _I64, _P, _I, _P]
    lib.fp8_grouped_gemm.restype = _I
    lib.fp8_grouped_gemm_gather.argtypes = [_P, _P, _I64, _P, _P, _P, _P, _I, _I64, _I64, _I64, _P,
                                            _I, _P]
    lib.fp8_grouped_gemm_gather.restype = _I
    lib.fp8_moe_route.argtypes = [_P, _I64, _I, _I, _I64, _P, _P, _P, _P, _I64, _P]
    lib.fp8_moe_route.restype = _I
    lib.fp8_get_status.argtypes = [_P]
    lib.fp8_get_status.restype = _I
    lib.fp8_status_string.argtypes = [_I]
    lib.fp8_status_string.restype = ctypes.c_char_p
    lib.fp8_set_wait_timeout_ns.argtypes = [ctypes.c_uint64]
    lib.fp8_set_wait_timeout_ns.restype = None
    lib.fp8_selftest_wait_timeout.argtypes = [_P]
    lib.fp8_selftest_wait_timeout.restype = _I
    lib.fp8_selftest_gemm_unwind.argtypes = [_I, _P, _P, _P, _P, _P, _I, _I64, _I64, _I64, _P,
                                             _I, _P]
    lib.fp8_selftest_gemm_unwind.restype = _I
    lib.fp8_device_supported.argtypes = []
    lib.fp8_device_supported.restype = _I
    lib.fp8_moe_dispatch_workspace_bytes.argtypes = [_I64, _I, _I]
    lib.fp8_moe_dispatch_workspace_bytes.restype = _I64
    lib.fp8_moe_dispatch.argtypes = [_P, _P, _I64, _I64, _P, _I, _I, _P, _P, _I64, _P, _P, _P,
                                     _P, _I64, _P]
    lib.fp8_moe_dispatch.restype = _I
    lib.fp8_moe_combine.argtypes = [_P, _I, _I64, _I64, _P, _P, _I64, _I, _P, _P]
    lib.fp8_moe_combine.restype = _I
    lib.fp8_moe_quant_dispatch.argtypes = [_P, _I, _I64, _I64, _I64, _P, _I, _I, _P, _P, _I64,
                                           _P, _P, _P, _P, _I64, _I, _P]
    lib.fp8_moe_quant_dispatch.restype = _I
    lib.fp8_moe_dispatch_noalloc.argtypes = [_P, _P, _I64, _I64, _P, _I, _I, _P, _P, _I64, _P,
                                             _P, _P, _P]
    lib.fp8_moe_dispatch_noalloc.restype = _I
    lib.fp8_requant_1x128_to_128x1.argtypes = [_P, _I64, _P, _I64, _I64, _P, _I64, _P, _I, _P]
    lib.fp8_requant_1x128_to_128x1.restype = _I
    _lib = lib
    return lib


def status_string(code: int) -> str:
    return load_library().fp8_status_string(int(code)).decode()


def _check(code: int, where: str) -> None:
    if code != FP8_OK:
        raise Fp8Error(code, where)


def _stream(stream):
    """cudaStream_t of `stream` (a torch.cuda.Stream), else torch's current stream."""
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t) -> int:
    return t.data_ptr() if t is not None and t.numel() > 0 else 0


def _in_dtype(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return IN_BF16
    if t.dtype == torch.float32:
        return IN_FP32
    raise TypeError(f"quantizer input must be bfloat16 or float32, got {t.dtype}")


def _out_dtype(t) -> int:
    import torch
    if t.dtype == torch.bfloat16:
        return OUT_BF16
    if t.dtype == torch.float32:
        return OUT_FP32
    raise TypeError(f"GEMM output must be bfloat16 or float32, got {t.dtype}")


def _row_stride(t) -> int:
    assert t.dim() == 2 and t.stride(1) == 1, "2-D tensors with unit column stride"
    return t.stride(0)


# ---------------------------------------------------------------- C-ABI calls

def fp8_quant_act_1x128(x, q, sA, scale_mode: int = SCALE_FP32, stream=None) -> None:
    """x [M, K] bf16/fp32 -> q [M, K] uint8 (E4M3 codes), sA [K/128, M] fp32."""
    M, K = x.shape
    _check(load_library().fp8_quant_act_1x128(
        _ptr(x), _in_dtype(x), M, K, _row_stride(x), _ptr(q), _row_stride(q), _ptr(sA),
        scale_mode, _stream(stream)), "fp8_quant_act_1x128")


def fp8_quant_act_128x1(x, qT, s, scale_mode: int = SCALE_FP32, stream=None) -> None:
    """x [T, C] -> qT [C, T] uint8 (token axis contiguous), s [T/128, C] fp32."""
    T, C = x.shape
    _check(load_library().fp8_quant_act_128x1(
        _ptr(x), _in_dtype(x), T, C, _row_stride(x), _ptr(qT), _row_stride(qT), _ptr(s),
        scale_mode, _stream(stream)), "fp8_quant_act_128x1")


def fp8_requant_1x128_to_128x1(q, sA, qT, s, scale_mode: int = SCALE_FP32, stream=None) -> None:
    """Cached 1x128 codes q [T, C] with sA [C/128, T] -> dequantize -> qT [C, T],
    s [T/128, C] in 128x1 groups along tokens."""
    T, C = q.shape
    _check(load_library().fp8_requant_1x128_to_128x1(
        _ptr(q), _row_stride(q), _ptr(sA), T, C, _ptr(qT), _row_stride(qT), _ptr(s),
        scale_mode, _stream(stream)), "fp8_requant_1x128_to_128x1")


def fp8_quant_w_128x128(w, q, sW, scale_mode: int = SCALE_FP32, stream=None) -> None:
    """w [N, K] -> q [N, K] uint8, sW [N/128, K/128] fp32."""
    N, K = w.shape
    _check(load_library().fp8_quant_w_128x128(
        _ptr(w), _in_dtype(w), N, K, _row_stride(w), _ptr(q), _row_stride(q), _ptr(sW),
        scale_mode, _stream(stream)), "fp8_quant_w_128x128")


def fp8_blockscaled_gemm(A, sA, B, sB, D, b_major: int = B_KMAJOR, sb_gran: int = 128,
                         stream=None) -> None:
    """D [M, N] = block-scaled A [M, K] x B (K-major [N, K] or MN-major [K, N])."""
    M, K = A.shape
    N = B.shape[0] if b_major == B_KMAJOR else B.shape[1]
    _check(load_library().fp8_blockscaled_gemm(
        _ptr(A), _ptr(sA), _ptr(B), b_major, _ptr(sB), sb_gran, M, N, K, _ptr(D),
        _out_dtype(D), _row_stride(D), _stream(stream)), "fp8_blockscaled_gemm")


def fp8_blockscaled_gemm_pow2(A, sA, B, sB, D, b_major: int = B_KMAJOR, sb_gran: int = 128,
                              stream=None) -> None:
    """fp8_blockscaled_gemm for power-of-two scales, scaled inside the tensor
    cores (UE8M0 block scaling); a scale that is not 2^e reports FP8_ERR_VALUE."""
    M, K = A.shape
    N = B.shape[0] if b_major == B_KMAJOR else B.shape[1]
    _check(load_library().fp8_blockscaled_gemm_pow2(
        _ptr(A), _ptr(sA), _ptr(B), b_major, _ptr(sB), sb_gran, M, N, K, _ptr(D),
        _out_dtype(D), _row_stride(D), _stream(stream)), "fp8_blockscaled_gemm_pow2")


def fp8_grouped_gemm_pow2(A, sA, B, sB, group_offsets, D, stream=None) -> None:
    """fp8_grouped_gemm for power-of-two scales, scaled inside the tensor cores."""
    M_total, K = A.shape
    G, N, _ = B.shape
    _check(load_library().fp8_grouped_gemm_pow2(
        _ptr(A), _ptr(sA), _ptr(B), _ptr(sB), _ptr(group_offsets), G, M_total, N, K, _ptr(D),
        _out_dtype(D), _stream(stream)), "fp8_grouped_gemm_pow2")


def fp8_grouped_gemm(A, sA, B, sB, group_offsets, D, stream=None) -> None:
    """Rows [off[e], off[e+1]) of A [M_total, K] times expert e of B [G, N, K]."""
    M_total, K = A.shape
    G, N, _ = B.shape
    _check(load_library().fp8_grouped_gemm(
        _ptr(A), _ptr(sA), _ptr(B), _ptr(sB), _ptr(group_offsets), G, M_total, N, K, _ptr(D),
        _out_dtype(D), _stream(stream)), "fp8_grouped_gemm")


def fp8_grouped_gemm_gather(A, sA, row_token, B, sB, group_offsets, D, stream=None) -> None:
    """Output row m of D [M_total, N] = token row row_token[m] of A [T, K]
    (sA [K/128, T]) times its expert's weight (B [G, N, K]); -1 rows give 0."""
    T, K = A.shape
    G, N, _ = B.shape
    M_total = D.shape[0]
    _check(load_library().fp8_grouped_gemm_gather(
        _ptr(A), _ptr(sA), T, _ptr(row_token), _ptr(B), _ptr(sB), _ptr(group_offsets), G, M_total,
        N, K, _ptr(D), _out_dtype(D), _stream(stream)), "fp8_grouped_gemm_gather")


def fp8_moe_route(topk, G, group_offsets, token_row, row_token, workspace, stream=None) -> None:
    """The routing of fp8_moe_dispatch alone (offsets, token_row, row_token)."""
    T, k = topk.shape
    M_cap = row_token.shape[0]
    _check(load_library().fp8_moe_route(
        _ptr(topk), T, k, G, M_cap, _ptr(group_offsets), _ptr(token_row), _ptr(row_token),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)),
        "fp8_moe_route")


def fp8_moe_dispatch_workspace_bytes(T: int, k: int, G: int) -> int:
    return int(load_library().fp8_moe_dispatch_workspace_bytes(T, k, G))


def fp8_moe_dispatch(q, sA, topk, G, q_out, sA_out, group_offsets, token_row, row_token,
                     workspace, stream=None) -> None:
    """FP8 rows of the tokens (q [T,K], sA [K/128,T]) to expert-contiguous,
    128-padded groups (q_out [M_cap,K], sA_out [K/128,M_cap]); topk [T,k] int32."""
    T, K = q.shape
    k = topk.shape[1]
    M_cap = q_out.shape[0]
    _check(load_library().fp8_moe_dispatch(
        _ptr(q), _ptr(sA), T, K, _ptr(topk), k, G, _ptr(q_out), _ptr(sA_out), M_cap,
        _ptr(group_offsets), _ptr(token_row), _ptr(row_token), _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)), "fp8_moe_dispatch")


def fp8_moe_quant_dispatch(x, topk, G, q_out, sA_out, group_offsets, token_row, row_token,
                           workspace, scale_mode: int = SCALE_FP32, stream=None) -> None:
    """Tokens x [T,K] (BF16 or FP32) quantized 1x128 straight into the
    expert-contiguous, 128-padded rows q_out [M_cap,K], sA_out [K/128,M_cap];
    topk [T,k] int32."""
    T, K = x.shape
    k = topk.shape[1]
    M_cap = q_out.shape[0]
    _check(load_library().fp8_moe_quant_dispatch(
        _ptr(x), _in_dtype(x), T, K, _row_stride(x), _ptr(topk), k, G, _ptr(q_out),
        _ptr(sA_out), M_cap, _ptr(group_offsets), _ptr(token_row), _ptr(row_token),
        _ptr(workspace), workspace.numel() * workspace.element_size(), scale_mode,
        _stream(stream)), "fp8_moe_quant_dispatch")


def fp8_moe_dispatch_noalloc(q, sA, topk, G, q_out, sA_out, group_offsets, token_row, row_token,
                             stream=None) -> None:
    """fp8_moe_dispatch with the library's fixed device scratch (no workspace
    argument; nothing allocated).  Overlapping calls on one device race."""
    T, K = q.shape
    k = topk.shape[1]
    M_cap = q_out.shape[0]
    _check(load_library().fp8_moe_dispatch_noalloc(
        _ptr(q), _ptr(sA), T, K, _ptr(topk), k, G, _ptr(q_out), _ptr(sA_out), M_cap,
        _ptr(group_offsets), _ptr(token_row), _ptr(row_token), _stream(stream)),
        "fp8_moe_dispatch_noalloc")


def fp8_moe_combine(D, token_row, weights, out, stream=None) -> None:
    """out[t] = BF16(sum_j weights[t,j] * D[token_row[t,j]]), FP32 sums."""
    M_cap, N = D.shape
    T, k = weights.shape
    _check(load_library().fp8_moe_combine(
        _ptr(D), _out_dtype(D), M_cap, N, _ptr(token_row), _ptr(weights), T, k, _ptr(out),
        _stream(stream)), "fp8_moe_combine")


def fp8_get_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device status word."""
    return load_library().fp8_get_status(_stream(stream))


def fp8_set_wait_timeout_ns(ns: int) -> None:
    load_library().fp8_set_wait_timeout_ns(int(ns))


def fp8_selftest_wait_timeout(stream=None) -> None:
    _check(load_library().fp8_selftest_wait_timeout(_stream(stream)), "fp8_selftest_wait_timeout")


def fp8_selftest_gemm_unwind(kernel: int, A, sA, B, sB, D, group_offsets=None,
                             stream=None) -> None:
    """Launch GEMM `kernel` (0: software promotion, 1: tensor-core scaling) with
    the odd CTA of every pair withholding its loads, so that its waits run out
    (B [N,K] dense or [G,N,K] grouped)."""
    M, K = A.shape
    N = B.shape[-2]
    G = B.shape[0] if group_offsets is not None else 0
    _check(load_library().fp8_selftest_gemm_unwind(
        kernel, _ptr(A), _ptr(sA), _ptr(B), _ptr(sB), _ptr(group_offsets), G, M, N, K, _ptr(D),
        _out_dtype(D), _stream(stream)), "fp8_selftest_gemm_unwind")


def fp8_device_supported() -> bool:
    return bool(load_library().fp8_device_supported())


# ---------------------------------------------------------------- allocating helpers

def quant_act_1x128(x, scale_mode: int = SCALE_FP32, stream=None):
    import torch
    M, K = x.shape
    q = torch.empty((M, K), dtype=torch.uint8, device=x.device)
    s = torch.empty((K // 128, M), dtype=torch.float32, device=x.device)
    fp8_quant_act_1x128(x, q, s, scale_mode, stream)
    return q, s


def quant_act_128x1(x, scale_mode: int = SCALE_FP32, stream=None):
    import torch
    T, C = x.shape
    q = torch.empty((C, T), dtype=torch.uint8, device=x.device)
    s = torch.empty((T // 128, C), dtype=torch.float32, device=x.device)
    fp8_quant_act_128x1(x, q, s, scale_mode, stream)
    return q, s


def requant_1x128_to_128x1(q, sA, scale_mode: int = SCALE_FP32, stream=None):
    import torch
    T, C = q.shape
    qT = torch.empty((C, T), dtype=torch.uint8, device=q.device)
    s = torch.empty((T // 128, C), dtype=torch.float32, device=q.device)
    fp8_requant_1x128_to_128x1(q, sA, qT, s, scale_mode, stream)
    return qT, s


def quant_w_128x128(w, scale_mode: int = SCALE_FP32, stream=None):
    import torch
    N, K = w.shape
    q = torch.empty((N, K), dtype=torch.uint8, device=w.device)
    s = torch.empty((N // 128, K // 128), dtype=torch.float32, device=w.device)
    fp8_quant_w_128x128(w, q, s, scale_mode, stream)
    return q, s


def gemm(A, sA, B, sB, out_dtype=None, b_major: int = B_KMAJOR, sb_gran: int = 128,
         stream=None):
    import torch
    M, K = A.shape
    N = B.shape[0] if b_major == B_KMAJOR else B.shape[1]
    D = torch.empty((M, N), dtype=out_dtype or torch.bfloat16, device=A.device)
    fp8_blockscaled_gemm(A, sA, B, sB, D, b_major, sb_gran, stream)
    return D


def moe_capacity(T: int, k: int, G: int) -> int:
    """Rows that always hold the padded groups: T*k + G*127, rounded up to 128."""
    return (T * k + G * 127 + 127) // 128 * 128


def moe_dispatch(q, sA, topk, G: int, M_cap: int = None, stream=None):
    """Allocating form of fp8_moe_dispatch; returns a dict of the outputs."""
    import torch
    T, K = q.shape
    k = topk.shape[1]
    M_cap = moe_capacity(T, k, G) if M_cap is None else M_cap
    d = q.device
    out = dict(q=torch.empty((M_cap, K), dtype=torch.uint8, device=d),
               sA=torch.empty((K // 128, M_cap), dtype=torch.float32, device=d),
               offsets=torch.empty(G + 1, dtype=torch.int32, device=d),
               token_row=torch.empty((T, k), dtype=torch.int32, device=d),
               row_token=torch.empty(M_cap, dtype=torch.int32, device=d))
    ws = torch.empty(max(1, fp8_moe_dispatch_workspace_bytes(T, k, G) // 4), dtype=torch.int32,
                     device=d)
    fp8_moe_dispatch(q, sA, topk, G, out["q"], out["sA"], out["offsets"], out["token_row"],
                     out["row_token"], ws, stream)
    return out


def grouped_gemm(A, sA, B, sB, group_offsets, out_dtype=None, stream=None):
    import torch
    D = torch.empty((A.shape[0], B.shape[1]), dtype=out_dtype or torch.bfloat16, device=A.device)
    fp8_grouped_gemm(A, sA, B, sB, group_offsets, D, stream)
    return D
