"""The C-ABI library, checked on the host (no GPU needed, no kernel launched).

  * libfp8fg.so builds, loads and exports every function include/fp8fg.h
    declares (and nothing else);
  * argument validation returns the documented codes, in the documented
    order, before any device call -- fake non-null pointers are safe here
    because a failing check launches nothing;
  * with no supported device, well-formed calls report FP8_ERR_DEVICE;
  * the library never links the oracle and the oracle never links it.
"""
import ctypes
import os
import re

import pytest

import fp8_fine_grained_x1_b200 as fg
from fp8_fine_grained_x1_b200 import build as fgbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fp8fg.h")

FAKE = 0x10000     # 64 KiB-aligned fake device address: never dereferenced
FAKE2 = 0x20000
FAKE3 = 0x30000
FAKE4 = 0x40000
FAKE5 = 0x50000


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:int64_t|int|void|const char\*)\s+(fp8_\w+)\s*\(", text, re.M)))


@pytest.fixture(scope="module")
def lib():
    fgbuild.build()
    return fg.load_library()


def test_library_exports_exactly_the_header(lib):
    declared = _declared_functions()
    assert set(declared) == set(fg.EXPORTED)
    for name in declared:
        assert hasattr(lib, name), name
    out = os.popen(f"nm -D --defined-only {fg.LIB_PATH}").read()
    exported = sorted(set(re.findall(r" T (\w+)$", out, re.M)))
    assert exported == declared


def test_status_strings(lib):
    for code in range(9):
        assert fg.status_string(code).startswith("FP8_")
    assert "unknown" in fg.status_string(99)


def q1(lib, *, x=FAKE, dt=fg.IN_BF16, M=128, K=512, ldx=None, q=FAKE2, ldq=None, s=FAKE3,
       mode=fg.SCALE_FP32):
    return lib.fp8_quant_act_1x128(x, dt, M, K, K if ldx is None else ldx, q,
                                   K if ldq is None else ldq, s, mode, None)


def test_quant_1x128_validation(lib):
    assert q1(lib, dt=7) == fg.FP8_ERR_DTYPE
    assert q1(lib, mode=3) == fg.FP8_ERR_DTYPE
    assert q1(lib, K=100) == fg.FP8_ERR_SHAPE
    assert q1(lib, K=0) == fg.FP8_ERR_SHAPE
    assert q1(lib, M=-1) == fg.FP8_ERR_SHAPE
    assert q1(lib, ldx=256) == fg.FP8_ERR_SHAPE
    assert q1(lib, M=0, x=0, q=0, s=0) == fg.FP8_OK            # empty: nothing to do
    assert q1(lib, x=0) == fg.FP8_ERR_NULL
    assert q1(lib, s=0) == fg.FP8_ERR_NULL
    assert q1(lib, x=FAKE + 8) == fg.FP8_ERR_ALIGN
    assert q1(lib, q=FAKE2 + 4) == fg.FP8_ERR_ALIGN
    assert q1(lib, ldx=516) == fg.FP8_ERR_ALIGN                 # 1032-B bf16 rows
    assert q1(lib, ldq=520) == fg.FP8_ERR_ALIGN                 # 520-B code rows
    assert q1(lib) in (fg.FP8_ERR_DEVICE, fg.FP8_OK)


def test_quant_1x128_fp32_rows_alignment(lib):
    # 516 fp32 = 2064 B (16-B multiple): alignment passes, fails later on device
    assert q1(lib, dt=fg.IN_FP32, ldx=516) not in (fg.FP8_ERR_ALIGN, fg.FP8_ERR_SHAPE)
    # 514 bf16 = 1028 B: not a 16-B multiple
    assert q1(lib, ldx=514) == fg.FP8_ERR_ALIGN


def test_quant_128x1_and_w_validation(lib):
    f = lib.fp8_quant_act_128x1
    assert f(FAKE, 0, 100, 64, 64, FAKE2, 100, FAKE3, 0, None) == fg.FP8_ERR_SHAPE   # T % 128
    assert f(FAKE, 0, 128, 60, 64, FAKE2, 128, FAKE3, 0, None) == fg.FP8_ERR_SHAPE   # C % 8
    assert f(FAKE, 0, 128, 64, 64, FAKE2, 64, FAKE3, 0, None) == fg.FP8_ERR_SHAPE    # ldqT < T
    assert f(0, 0, 128, 0, 0, 0, 128, 0, 0, None) == fg.FP8_OK                       # C == 0
    assert f(FAKE, 0, 128, 64, 64, 0, 128, FAKE3, 0, None) == fg.FP8_ERR_NULL
    assert f(FAKE, 2, 128, 64, 64, FAKE2, 128, FAKE3, 0, None) == fg.FP8_ERR_DTYPE
    w = lib.fp8_quant_w_128x128
    assert w(FAKE, 0, 200, 128, 128, FAKE2, 128, FAKE3, 0, None) == fg.FP8_ERR_SHAPE  # N % 128
    assert w(FAKE, 0, 128, 128, 128, FAKE2, 128, 0, 0, None) == fg.FP8_ERR_NULL
    assert w(FAKE + 1, 0, 128, 128, 128, FAKE2, 128, FAKE3, 0, None) == fg.FP8_ERR_ALIGN
    assert w(FAKE, 0, 0, 128, 128, 0, 128, 0, 0, None) == fg.FP8_OK


def g(lib, *, A=FAKE, sA=FAKE2, B=FAKE3, bm=0, sB=FAKE4, gran=128, M=256, N=256, K=512,
      D=FAKE5, od=0, ldd=None, fn=None):
    fn = lib.fp8_blockscaled_gemm if fn is None else fn
    return fn(A, sA, B, bm, sB, gran, M, N, K, D, od, N if ldd is None else ldd, None)


def test_gemm_validation(lib):
    assert g(lib, od=5) == fg.FP8_ERR_DTYPE
    assert g(lib, bm=2) == fg.FP8_ERR_DTYPE
    assert g(lib, gran=64) == fg.FP8_ERR_DTYPE
    assert g(lib, gran=1, bm=fg.B_MNMAJOR) == fg.FP8_ERR_DTYPE   # per-column scales: K-major only
    assert g(lib, N=200) == fg.FP8_ERR_SHAPE
    assert g(lib, K=130) == fg.FP8_ERR_SHAPE
    assert g(lib, N=0) == fg.FP8_ERR_SHAPE
    assert g(lib, ldd=128) == fg.FP8_ERR_SHAPE
    assert g(lib, M=0, A=0, sA=0, B=0, sB=0, D=0) == fg.FP8_OK
    assert g(lib, D=0) == fg.FP8_ERR_NULL
    assert g(lib, sB=0) == fg.FP8_ERR_NULL
    assert g(lib, A=FAKE + 16 + 8) == fg.FP8_ERR_ALIGN
    assert g(lib, gran=1, sB=FAKE4 + 4) == fg.FP8_ERR_ALIGN      # float4 column-scale loads
    assert g(lib, gran=128, sB=FAKE4 + 4) not in (fg.FP8_ERR_ALIGN,)
    assert g(lib, od=fg.OUT_BF16, ldd=260) == fg.FP8_ERR_ALIGN   # 520-B rows
    assert g(lib) in (fg.FP8_ERR_DEVICE, fg.FP8_OK)


def test_gemm_pow2_validation(lib):
    def gp(**kw):
        return g(lib, fn=lib.fp8_blockscaled_gemm_pow2, **kw)
    assert gp(od=5) == fg.FP8_ERR_DTYPE
    assert gp(gran=1, bm=fg.B_MNMAJOR) == fg.FP8_ERR_DTYPE
    assert gp(N=200) == fg.FP8_ERR_SHAPE
    assert gp(K=130) == fg.FP8_ERR_SHAPE
    assert gp(M=0, A=0, sA=0, B=0, sB=0, D=0) == fg.FP8_OK
    assert gp(D=0) == fg.FP8_ERR_NULL
    assert gp(A=FAKE + 16 + 8) == fg.FP8_ERR_ALIGN
    assert gp(gran=1, sB=FAKE4 + 4) in (fg.FP8_ERR_DEVICE, fg.FP8_OK)   # scalar scale loads
    assert gp() in (fg.FP8_ERR_DEVICE, fg.FP8_OK)


def test_requant_validation(lib):
    def rq(q=FAKE, ldq=256, sA=FAKE3, T=256, C=256, qT=FAKE2, ldqT=256, s=FAKE4, mode=fg.SCALE_FP32):
        return lib.fp8_requant_1x128_to_128x1(q, ldq, sA, T, C, qT, ldqT, s, mode, None)
    assert rq(mode=7) == fg.FP8_ERR_DTYPE
    assert rq(T=200) == fg.FP8_ERR_SHAPE
    assert rq(C=200, ldq=256) == fg.FP8_ERR_SHAPE                # channels in 128-blocks
    assert rq(ldq=128) == fg.FP8_ERR_SHAPE
    assert rq(ldqT=128) == fg.FP8_ERR_SHAPE
    assert rq(C=0) == fg.FP8_OK
    assert rq(sA=0) == fg.FP8_ERR_NULL
    assert rq(ldq=264) == fg.FP8_ERR_ALIGN
    assert rq(q=FAKE + 8) == fg.FP8_ERR_ALIGN
    assert rq() in (fg.FP8_ERR_DEVICE, fg.FP8_OK)


@pytest.mark.parametrize("name", ["fp8_grouped_gemm", "fp8_grouped_gemm_pow2"])
def test_grouped_validation(lib, name):
    f = getattr(lib, name)
    args = dict(A=FAKE, sA=FAKE2, B=FAKE3, sB=FAKE4, off=FAKE5, G=4, M=512, N=256, K=256,
                D=0x60000, od=0)

    def call(**kw):
        a = dict(args, **kw)
        return f(a["A"], a["sA"], a["B"], a["sB"], a["off"], a["G"], a["M"], a["N"], a["K"],
                 a["D"], a["od"], None)
    assert call(od=9) == fg.FP8_ERR_DTYPE
    assert call(G=0) == fg.FP8_ERR_SHAPE
    assert call(G=2000) == fg.FP8_ERR_SHAPE
    assert call(M=500) == fg.FP8_ERR_SHAPE
    assert call(M=0, A=0, sA=0, B=0, sB=0, off=0, D=0) == fg.FP8_OK
    assert call(off=0) == fg.FP8_ERR_NULL
    assert call(off=FAKE5 + 2) == fg.FP8_ERR_ALIGN
    assert call() in (fg.FP8_ERR_DEVICE, fg.FP8_OK)


def test_product_and_oracle_share_no_code():
    """Neither side imports or links the other (checked on the sources)."""
    pkg = os.path.join(ROOT, "fp8_fine_grained_x1_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".c")):
                src = open(os.path.join(dirpath, f)).read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", src, re.M), f
                assert "oracle/" not in src and "liboracle" not in src, f
    osrc = open(os.path.join(ROOT, "oracle", "fp8_oracle.c")).read()
    assert "#include \"" not in osrc            # system headers only
    opy = open(os.path.join(ROOT, "oracle", "__init__.py")).read()
    assert "fp8_fine_grained_x1_b200" not in opy.replace("``fp8_fine_grained_x1_b200``", "")
