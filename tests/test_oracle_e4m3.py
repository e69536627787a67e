"""Pins of the oracle's E4M3 codec against things other than itself.

The pages fix E4M3 "on all tensors" (4 exponent bits, 3 mantissa bits) for
Fprop, Dgrad and Wgrad (Mixed precision framework, Figure 6); the pages do
not state the rounding, so the oracle rounds to nearest-even and saturates at
+-448 (reading R2 in the header of oracle/fp8_oracle.c).

Independent references used here:
  * torch's own float8_e4m3fn type (a library implementation of OCP E4M3FN):
    its 256-value decode table, and its FP32 -> E4M3 cast for |v| <= 448;
  * a brute-force nearest-value search over the 254 finite values of that
    library table (ties to the even code), which also covers saturation.
"""
import numpy as np
import pytest
import torch

import oracle


def _torch_table():
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    return codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()


def test_decode_table_matches_library():
    ours = oracle.e4m3_decode_table()
    lib = _torch_table()
    nan_ours = np.isnan(ours)
    assert np.array_equal(nan_ours, np.isnan(lib))
    assert sorted(np.flatnonzero(nan_ours).tolist()) == [0x7F, 0xFF]
    assert np.array_equal(ours[~nan_ours], lib[~nan_ours])
    # sign of zero kept: 0x80 is -0
    assert np.signbit(ours[0x80]) and not np.signbit(ours[0x00])


def test_decode_named_values():
    # max finite, smallest normal, smallest subnormal of E4M3FN
    assert oracle.e4m3_decode(0x7E) == 448.0
    assert oracle.e4m3_decode(0xFE) == -448.0
    assert oracle.e4m3_decode(0x08) == 2.0 ** -6
    assert oracle.e4m3_decode(0x01) == 2.0 ** -9
    assert oracle.e4m3_decode(0x38) == 1.0


def _boundary_values():
    """Every finite E4M3 value, every midpoint between neighbours, and the
    float32 values 1..64 ulps either side of each midpoint."""
    tab = _torch_table()
    pos = np.unique(tab[(tab >= 0) & ~np.isnan(tab)])
    mids = (pos[:-1] + pos[1:]) / 2.0
    vals = [pos, mids]
    mids32 = mids.astype(np.float32)
    assert np.array_equal(mids32.astype(np.float64), mids)   # midpoints are exact in fp32
    bits = mids32.view(np.uint32).astype(np.int64)
    for d in range(1, 65):
        vals.append((bits + d).astype(np.uint32).view(np.float32).astype(np.float64))
        vals.append((bits - d).astype(np.uint32).view(np.float32).astype(np.float64))
    v = np.concatenate(vals).astype(np.float32)
    return np.concatenate([v, -v])


def _strided_fp32(lo_bits=0, hi=464.0, stride=97):
    hi_bits = int(np.float32(hi).view(np.uint32))
    b = np.arange(lo_bits, hi_bits + 1, stride, dtype=np.uint32)
    v = b.view(np.float32)
    return np.concatenate([v, -v])


def test_encode_matches_library_cast_in_range():
    v = np.concatenate([_boundary_values(), _strided_fp32(hi=448.0, stride=61)])
    v = v[np.abs(v) <= 448.0]
    ours = oracle.e4m3_encode_array(v)
    lib = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    bad = np.flatnonzero(ours != lib)
    assert bad.size == 0, (v[bad[:8]], ours[bad[:8]], lib[bad[:8]])


def _brute_nearest(v):
    """Nearest finite E4M3 value by exhaustive search; ties -> even code;
    |v| > 448 saturates to +-448; the sign of v is kept for zero results."""
    tab = _torch_table()
    finite = np.flatnonzero(~np.isnan(tab) & (np.arange(256) < 0x80))   # 0x00..0x7E
    mags = tab[finite]
    a = np.abs(v.astype(np.float64))
    out = np.empty(v.shape, np.uint8)
    chunk = 1 << 16
    for s in range(0, len(a), chunk):
        aa = a[s:s + chunk, None]
        d = np.abs(aa - mags[None, :])
        dmin = d.min(axis=1, keepdims=True)
        cand = (d == dmin)
        # among tied candidates prefer the one with an even code (mantissa LSB 0)
        even = cand & ((finite[None, :] & 1) == 0)
        pick = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
        code = finite[pick]
        code = np.where(a[s:s + chunk] > 448.0, 0x7E, code)
        out[s:s + chunk] = code
    sign = np.signbit(v).astype(np.uint8) << 7
    return out | sign


def test_encode_matches_brute_force_nearest_including_saturation():
    v = np.concatenate([_boundary_values(), _strided_fp32(hi=600.0, stride=4099),
                        np.array([449.0, 464.0, 465.0, 1e6, 3.0e38, -1e6, 0.0, -0.0],
                                 np.float32)])
    ours = oracle.e4m3_encode_array(v)
    ref = _brute_nearest(v)
    bad = np.flatnonzero(ours != ref)
    assert bad.size == 0, (v[bad[:8]], ours[bad[:8]], ref[bad[:8]])


def test_encode_zero_and_underflow_keep_sign():
    assert oracle.e4m3_encode(0.0) == 0x00
    assert oracle.e4m3_encode(-0.0) == 0x80
    assert oracle.e4m3_encode(-1e-30) == 0x80
    assert oracle.e4m3_encode(2.0 ** -10) == 0x00          # tie between 0 and 2^-9 -> even (0)
    assert oracle.e4m3_encode(1.5 * 2.0 ** -10) == 0x01
    assert oracle.e4m3_encode(float("nan")) == 0x7F


@pytest.mark.slow
def test_encode_exhaustive_against_library():
    """Every FP32 bit pattern of [0, 448] (about 1.14e9 values), in chunks,
    against the library cast; the negative patterns follow by the sign bit
    (checked on a strided sample here and in the tests above)."""
    hi_bits = int(np.float32(448.0).view(np.uint32))
    for start in range(0, hi_bits + 1, 1 << 26):
        b = np.arange(start, min(start + (1 << 26), hi_bits + 1), dtype=np.uint32)
        v = b.view(np.float32)
        ours = oracle.e4m3_encode_array(v)
        lib = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        assert np.array_equal(ours, lib), start
    neg = -np.arange(0, hi_bits + 1, 9973, dtype=np.uint32).view(np.float32)
    assert np.array_equal(oracle.e4m3_encode_array(neg),
                          torch.from_numpy(neg).to(torch.float8_e4m3fn).view(torch.uint8).numpy())
