"""CPU oracle for the fine-grained FP8 Linear -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product path (``fp8_fine_grained_x1_b200``) never imports it, and it never
imports the product path: the two share no code.

The arithmetic lives in ``fp8_oracle.c`` (plain C, FP64 GEMM reference,
FP32 scale arithmetic); this module only builds it with gcc and marshals
numpy arrays through ctypes.  Each function cites the passage of the
DeepSeek-V3 report ("FP8 Training" section, as reproduced on the pages) that
it follows; see the header of ``fp8_oracle.c``.

Parity pins: every public function here is checked in ``tests/`` against
something other than itself (library casts, brute force, exact rational
arithmetic, closed forms and invariants).  None is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fp8_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

SCALE_FP32 = 0
SCALE_POW2 = 1
IN_BF16 = 0
IN_FP32 = 1
B_KMAJOR = 0
B_MNMAJOR = 1


def build(force: bool = False) -> str:
    """Compile fp8_oracle.c into liboracle.so (gcc, OpenMP, no fast-math)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
           "-fno-fast-math", "-ffp-contract=off", "-fvisibility=hidden",
           _SRC, "-o", _LIB_PATH + ".tmp", "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(_LIB_PATH + ".tmp", _LIB_PATH)
    return _LIB_PATH


_lib = None

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_I = ctypes.c_int


def _load():
    global _lib
    if _lib is not None:
        return _lib
    lib = ctypes.CDLL(build())
    lib.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    lib.oracle_e4m3_decode.restype = ctypes.c_double
    lib.oracle_e4m3_encode.argtypes = [ctypes.c_double]
    lib.oracle_e4m3_encode.restype = ctypes.c_uint8
    for name in ("oracle_quant_act_1x128", "oracle_quant_act_128x1", "oracle_quant_w_128x128"):
        f = getattr(lib, name)
        f.argtypes = [_P, _I, _I64, _I64, _I64, _P, _I64, _P, _I]
        f.restype = None
    lib.oracle_gemm_points.argtypes = [_P, _I64, _P, _I64, _P, _I64, _I, _P, _I, _I64, _I64,
                                       _P, _I64, _P, _P]
    lib.oracle_gemm_points.restype = None
    lib.oracle_gemm_full.argtypes = [_P, _I64, _P, _I64, _P, _I64, _I, _P, _I, _I64, _I64,
                                     _P, _P]
    lib.oracle_gemm_full.restype = None
    lib.oracle_grouped_gemm_points.argtypes = [_P, _I64, _P, _I64, _P, _P, _P, _I, _I64, _I64,
                                               _P, _I64, _P, _P, _P]
    lib.oracle_grouped_gemm_points.restype = None
    lib.oracle_limited_dot.argtypes = [_P, _P, _I64, _I, _I]
    lib.oracle_limited_dot.restype = ctypes.c_double
    lib.oracle_e4m3_encode_array.argtypes = [_P, _I64, _P]
    lib.oracle_e4m3_encode_array.restype = None
    lib.oracle_requant_1x128_to_128x1.argtypes = [_P, _I64, _P, _I64, _I64, _P, _I64, _P, _I]
    lib.oracle_requant_1x128_to_128x1.restype = None
    lib.oracle_num_threads.argtypes = []
    lib.oracle_num_threads.restype = _I
    _lib = lib
    return lib


def _ptr(a: np.ndarray) -> int:
    assert a.flags["C_CONTIGUOUS"], "oracle takes C-contiguous arrays"
    return a.ctypes.data


def _as_input(x: np.ndarray):
    """BF16 inputs travel as uint16 bit patterns; FP32 as float32."""
    if x.dtype == np.uint16:
        return np.ascontiguousarray(x), IN_BF16
    if x.dtype == np.float32:
        return np.ascontiguousarray(x), IN_FP32
    raise TypeError("oracle inputs are bf16 bit patterns (uint16) or float32")


def num_threads() -> int:
    return _load().oracle_num_threads()


def e4m3_decode(b: int) -> float:
    """Value of one E4M3FN byte from its bit fields (E4M3 on all tensors)."""
    return _load().oracle_e4m3_decode(int(b))


def e4m3_encode(v: float) -> int:
    """Nearest E4M3 code, ties to even, saturating at +-448 (reading R2)."""
    return int(_load().oracle_e4m3_encode(float(v)))


def e4m3_encode_array(v: np.ndarray) -> np.ndarray:
    """e4m3_encode applied to every element of a float32 array."""
    v = np.ascontiguousarray(v, np.float32)
    out = np.empty(v.shape, np.uint8)
    _load().oracle_e4m3_encode_array(_ptr(v), v.size, _ptr(out))
    return out


def e4m3_decode_table() -> np.ndarray:
    """All 256 byte values decoded (NaN at 0x7F and 0xFF)."""
    return np.array([e4m3_decode(b) for b in range(256)], dtype=np.float64)


def quant_act_1x128(x: np.ndarray, mode: int = SCALE_FP32):
    """1x128 activation tiles (Fine-grained quantization, Figure 7 (a)).

    x: [M, K] bf16 bits (uint16) or float32.  Returns (q [M, K] uint8,
    sA [K/128, M] float32)."""
    x, dt = _as_input(x)
    M, K = x.shape
    q = np.empty((M, K), np.uint8)
    s = np.empty((K // 128, M), np.float32)
    _load().oracle_quant_act_1x128(_ptr(x), dt, M, K, K, _ptr(q), K, _ptr(s), mode)
    return q, s


def quant_act_128x1(x: np.ndarray, mode: int = SCALE_FP32):
    """128x1 tiles along tokens for Wgrad operands (groups along the GEMM
    inner dimension, which for Wgrad is the token axis).

    x: [T, C].  Returns (qT [C, T] uint8, s [T/128, C] float32)."""
    x, dt = _as_input(x)
    T, C = x.shape
    q = np.empty((C, T), np.uint8)
    s = np.empty((T // 128, C), np.float32)
    _load().oracle_quant_act_128x1(_ptr(x), dt, T, C, C, _ptr(q), T, _ptr(s), mode)
    return q, s


def requant_1x128_to_128x1(q: np.ndarray, sA: np.ndarray, mode: int = SCALE_FP32):
    """Activations cached as 1x128 FP8 (q [T, C] codes, sA [C/128, T]) regrouped
    for Wgrad: dequantize to FP32, then 128x1 groups along tokens (reading R13).
    Returns (qT [C, T] uint8, s [T/128, C] float32)."""
    q = np.ascontiguousarray(q, np.uint8)
    sA = np.ascontiguousarray(sA, np.float32)
    T, C = q.shape
    assert sA.shape == (C // 128, T) and T % 128 == 0 and C % 128 == 0
    qT = np.empty((C, T), np.uint8)
    s = np.empty((T // 128, C), np.float32)
    _load().oracle_requant_1x128_to_128x1(_ptr(q), C, _ptr(sA), T, C, _ptr(qT), T, _ptr(s), mode)
    return qT, s


def quant_w_128x128(w: np.ndarray, mode: int = SCALE_FP32):
    """128x128 weight blocks (Fine-grained quantization, Figure 7 (a)).

    w: [N, K].  Returns (q [N, K] uint8, sW [N/128, K/128] float32)."""
    w, dt = _as_input(w)
    N, K = w.shape
    q = np.empty((N, K), np.uint8)
    s = np.empty((N // 128, K // 128), np.float32)
    _load().oracle_quant_w_128x128(_ptr(w), dt, N, K, K, _ptr(q), K, _ptr(s), mode)
    return q, s


def _b_dims(B, b_major, K):
    if b_major == B_KMAJOR:
        N, Kb = B.shape
    else:
        Kb, N = B.shape
    assert Kb == K
    return N, B.shape[1]


def gemm_full(A, sA, B, sB, b_major=B_KMAJOR, sb_gran=128):
    """FP64 reference of the block-scaled GEMM (Increasing accumulation
    precision: per-128-K partials scaled by sA*sB and summed).

    Returns (ref [M, N] float64, tol [M, N] float64 = sum_k |a_k b_k|)."""
    A = np.ascontiguousarray(A, np.uint8)
    B = np.ascontiguousarray(B, np.uint8)
    sA = np.ascontiguousarray(sA, np.float32)
    sB = np.ascontiguousarray(sB, np.float32)
    M, K = A.shape
    N, ldb = _b_dims(B, b_major, K)
    ref = np.empty((M, N), np.float64)
    tol = np.empty((M, N), np.float64)
    _load().oracle_gemm_full(_ptr(A), K, _ptr(sA), M, _ptr(B), ldb, b_major, _ptr(sB),
                             sb_gran, N, K, _ptr(ref), _ptr(tol))
    return ref, tol


def gemm_points(A, sA, B, sB, pts, b_major=B_KMAJOR, sb_gran=128):
    """Reference at sampled output points pts [P, 2] = (m, n)."""
    A = np.ascontiguousarray(A, np.uint8)
    B = np.ascontiguousarray(B, np.uint8)
    sA = np.ascontiguousarray(sA, np.float32)
    sB = np.ascontiguousarray(sB, np.float32)
    pts = np.ascontiguousarray(pts, np.int64)
    M, K = A.shape
    N, ldb = _b_dims(B, b_major, K)
    ref = np.empty(len(pts), np.float64)
    tol = np.empty(len(pts), np.float64)
    _load().oracle_gemm_points(_ptr(A), K, _ptr(sA), M, _ptr(B), ldb, b_major, _ptr(sB),
                               sb_gran, N, K, _ptr(pts), len(pts), _ptr(ref), _ptr(tol))
    return ref, tol


def grouped_gemm_points(A, sA, B, sB, offsets, pts):
    """Grouped (MoE expert) reference: rows [off[e], off[e+1]) use expert e.

    A [M_total, K], sA [K/128, M_total], B [G, N, K], sB [G, N/128, K/128],
    offsets [G+1] int32.  Returns (ref, tol, group) at pts [P, 2]."""
    A = np.ascontiguousarray(A, np.uint8)
    B = np.ascontiguousarray(B, np.uint8)
    sA = np.ascontiguousarray(sA, np.float32)
    sB = np.ascontiguousarray(sB, np.float32)
    off = np.ascontiguousarray(offsets, np.int32)
    pts = np.ascontiguousarray(pts, np.int64)
    M_total, K = A.shape
    G, N, _ = B.shape
    ref = np.empty(len(pts), np.float64)
    tol = np.empty(len(pts), np.float64)
    grp = np.empty(len(pts), np.int32)
    _load().oracle_grouped_gemm_points(_ptr(A), K, _ptr(sA), M_total, _ptr(B), _ptr(sB),
                                       _ptr(off), G, N, K, _ptr(pts), len(pts), _ptr(ref),
                                       _ptr(tol), _ptr(grp))
    return ref, tol, grp


def limited_dot(a_codes, b_codes, bits: int, promote_every: int) -> float:
    """Dot product with a `bits`-bit truncating accumulator per K=32 MMA step,
    optionally promoted to FP32 every `promote_every` elements."""
    a = np.ascontiguousarray(a_codes, np.uint8)
    b = np.ascontiguousarray(b_codes, np.uint8)
    assert a.shape == b.shape and a.ndim == 1
    return _load().oracle_limited_dot(_ptr(a), _ptr(b), len(a), bits, promote_every)
