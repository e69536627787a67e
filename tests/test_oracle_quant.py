"""Pins of the oracle's quantizers (1x128, 128x1, 128x128; FP32 and POW2).

What the pages fix: groups of 1x128 (per token per 128 channels) for
activations and 128x128 (per 128 input x 128 output channels) for weights
(Fine-grained quantization, Figure 7 (a)); the max-abs of each group is
computed online and mapped to the largest FP8 value (Online quantization;
the max-abs -> FP8-max practice cited to Narang et al.); some scales are
integral powers of 2.  The checks below are closed forms, invariants,
planted-layout cases and exact special cases -- none re-types the oracle's
scale formula.
"""
import bisect
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from fp8_fine_grained_x1_b200 import synth

TAB = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn) \
    .to(torch.float64).numpy()


def dec(q):
    return TAB[q]


def _bits(x32):
    """float32 array -> bf16 bit patterns (RNE), via torch."""
    return synth.bf16_bits(torch.from_numpy(np.ascontiguousarray(x32)).to(torch.bfloat16))


def _from_bits(b):
    return (b.astype(np.uint32) << 16).view(np.float32)


# ---------------------------------------------------------------- exact arithmetic
# Correct rounding written out on rationals: no float operation decides a
# result, so these checks pin the oracle's FP32 arithmetic itself.

def fl32(fr: Fraction) -> Fraction:
    """The FP32 value nearest to the positive rational fr, ties to the even
    significand (normal FP32 range)."""
    assert fr > 0
    e = fr.numerator.bit_length() - fr.denominator.bit_length()   # 2^e <= fr < 2^(e+2)
    if Fraction(2) ** e > fr:
        e -= 1
    elif Fraction(2) ** (e + 1) <= fr:
        e += 1
    assert -126 <= e <= 127
    ulp = Fraction(2) ** (e - 23)
    n = math.floor(fr / ulp)                  # 2^23 <= n < 2^24
    rem = fr / ulp - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return n * ulp


def fl32_signed(fr: Fraction) -> Fraction:
    return fl32(fr) if fr > 0 else -fl32(-fr)


# non-negative finite E4M3 values in code order (torch's float8_e4m3fn table)
_POS = [Fraction(float(TAB[c])) for c in range(0x7F)]


def e4m3_nearest(y: Fraction, negative: bool) -> int:
    """Code of the E4M3 value nearest to y (ties to the even code, |y| >= 448
    saturating to 448), with the sign bit of the input."""
    a = abs(y)
    sign = 0x80 if negative else 0
    if a >= 448:
        return sign | 0x7E
    hi = bisect.bisect_left(_POS, a)
    if _POS[hi] == a:
        return sign | hi
    lo = hi - 1
    dlo, dhi = a - _POS[lo], _POS[hi] - a
    if dlo < dhi or (dlo == dhi and lo % 2 == 0):
        return sign | lo
    return sign | hi


# ---------------------------------------------------------------- layout pins

def test_1x128_planted_group_maxima_fix_scale_layout():
    M, K = 6, 512
    rng = np.random.default_rng(10)
    x = rng.uniform(-0.9, 0.9, (M, K)).astype(np.float32)
    want = np.empty((K // 128, M), np.float32)
    for m in range(M):
        for kb in range(K // 128):
            c = (m * 7 + kb * 3) % 17 - 8                  # distinct exponents per group
            j = (m * 31 + kb * 53) % 128                    # position of the max
            x[m, kb * 128 + j] = (1 if (m + kb) % 2 else -1) * 448.0 * 2.0 ** c
            want[kb, m] = 2.0 ** c
            x[m, kb * 128:(kb + 1) * 128] *= 1.0            # keep others |x| < 448*2^c
            small = np.abs(x[m, kb * 128:(kb + 1) * 128]) < 448.0 * 2.0 ** c
            x[m, kb * 128:(kb + 1) * 128][small] *= 2.0 ** c
    q, s = oracle.quant_act_1x128(x)
    assert s.shape == (K // 128, M)
    assert np.array_equal(s, want)
    # the planted max is exactly 448 * s -> code +-0x7E
    for m in range(M):
        for kb in range(K // 128):
            j = (m * 31 + kb * 53) % 128
            assert q[m, kb * 128 + j] & 0x7F == 0x7E


def test_128x1_planted_group_maxima_fix_scale_layout():
    T, C = 384, 5
    rng = np.random.default_rng(11)
    x = rng.uniform(-0.5, 0.5, (T, C)).astype(np.float32)
    want = np.empty((T // 128, C), np.float32)
    for tb in range(T // 128):
        for c in range(C):
            e = (tb * 5 + c * 3) % 13 - 6
            x[tb * 128:(tb + 1) * 128, c] *= 2.0 ** e
            t = (tb * 17 + c * 29) % 128
            x[tb * 128 + t, c] = 448.0 * 2.0 ** e
            want[tb, c] = 2.0 ** e
    qT, s = oracle.quant_act_128x1(x)
    assert qT.shape == (C, T) and s.shape == (T // 128, C)
    assert np.array_equal(s, want)
    for tb in range(T // 128):
        for c in range(C):
            t = (tb * 17 + c * 29) % 128
            assert qT[c, tb * 128 + t] == 0x7E


def test_128x128_planted_block_maxima_fix_scale_layout():
    N, K = 256, 384
    rng = np.random.default_rng(12)
    w = rng.uniform(-0.5, 0.5, (N, K)).astype(np.float32)
    want = np.empty((N // 128, K // 128), np.float32)
    for nb in range(N // 128):
        for kb in range(K // 128):
            e = nb * 4 - kb * 3 + 1
            blk = w[nb * 128:(nb + 1) * 128, kb * 128:(kb + 1) * 128]
            blk *= 2.0 ** e
            blk[(nb * 37 + kb * 11) % 128, (nb * 5 + kb * 71) % 128] = -448.0 * 2.0 ** e
            want[nb, kb] = 2.0 ** e
    q, s = oracle.quant_w_128x128(w)
    assert np.array_equal(s, want)
    for nb in range(N // 128):
        for kb in range(K // 128):
            assert q[nb * 128 + (nb * 37 + kb * 11) % 128, kb * 128 + (nb * 5 + kb * 71) % 128] == 0xFE


# ---------------------------------------------------------------- exact scale and codes
# Reading R1: s = fl32(amax/448) is stored and the codes are
# E(fl32(x * fl32(448/amax))).  Written out on rationals; the groups hold
# max-abs values that are not powers of two (where 1/448 and 448/amax are
# inexact) and elements planted within a few FP32 ulps of a midpoint between
# two E4M3 values, so that a product formed any other way -- x/s, or
# x * fl32(1/s) -- rounds to the neighbouring code.

def _ulp32(v: Fraction) -> Fraction:
    e = v.numerator.bit_length() - v.denominator.bit_length()
    if Fraction(2) ** e > v:
        e -= 1
    elif Fraction(2) ** (e + 1) <= v:
        e += 1
    return Fraction(2) ** (e - 23)


def _f32(v: Fraction):
    """v as an np.float32 if it is an FP32 value, else None."""
    f = np.float32(float(v))
    return f if Fraction(float(f)) == v else None


def _non_pow2_amax(rng):
    while True:
        a = np.float32(rng.uniform(1.0, 2.0) * 2.0 ** int(rng.integers(-20, 21)))
        if math.frexp(float(a))[0] != 0.5:
            return a


def _planted_values(rng, amax, n, n_planted):
    """n values below amax in magnitude: random ones, and n_planted placed at
    E4M3 rounding midpoints of the scaled space, alternately chosen where
    fl32(x/s) and where fl32(x*fl32(1/s)) round to another code than
    fl32(x*inv)."""
    A = Fraction(float(amax))
    inv, s = fl32(448 / A), fl32(A / 448)
    r = fl32(1 / s)
    out = (rng.uniform(2.0 ** -12, 1.0, n) * float(amax)).astype(np.float32)
    for i in range(n_planted):
        c = int(rng.integers(8, 0x7D))                    # normal codes c, c+1
        mid = (_POS[c] + _POS[c + 1]) / 2
        x0 = fl32(mid / inv)
        pick = _f32(x0)
        for k in (0, 1, -1, 2, -2, 3, -3, 4, -4):
            x = _f32(x0 + k * _ulp32(x0))
            if x is None:
                continue
            X = Fraction(float(x))
            good = e4m3_nearest(fl32(X * inv), False)
            other = fl32(X / s) if i % 2 == 0 else fl32(X * r)
            if e4m3_nearest(other, False) != good:
                pick = x
                break
        out[i] = pick
    out *= np.where(rng.integers(0, 2, n) == 1, -1, 1).astype(np.float32)
    return out


def _expected_group(vals):
    """(scale, codes) of one group from the definition, on rationals."""
    A = max(abs(Fraction(float(v))) for v in vals)
    inv = fl32(448 / A)
    codes = [e4m3_nearest(fl32_signed(Fraction(float(v)) * inv), bool(np.signbit(v)))
             for v in vals]
    return fl32(A / 448), np.array(codes, np.uint8)


def _planted_group(rng, n=128, n_planted=48):
    amax = _non_pow2_amax(rng)
    g = _planted_values(rng, amax, n, n_planted)
    g[int(rng.integers(n_planted, n))] = amax * (1 if rng.integers(0, 2) else -1)
    return g


def test_fp32_scale_and_codes_are_the_correctly_rounded_definition_1x128():
    rng = np.random.default_rng(21)
    M, K = 8, 512
    x = np.stack([np.concatenate([_planted_group(rng) for _ in range(K // 128)])
                  for _ in range(M)]).astype(np.float32)
    q, s = oracle.quant_act_1x128(x)
    for m in range(M):
        for kb in range(K // 128):
            want_s, want_q = _expected_group(x[m, kb * 128:(kb + 1) * 128])
            assert Fraction(float(s[kb, m])) == want_s, (m, kb)
            assert np.array_equal(q[m, kb * 128:(kb + 1) * 128], want_q), (m, kb)


def test_fp32_scale_and_codes_are_the_correctly_rounded_definition_128x1():
    rng = np.random.default_rng(22)
    T, C = 256, 16
    x = np.stack([np.concatenate([_planted_group(rng) for _ in range(T // 128)])
                  for _ in range(C)], axis=1).astype(np.float32)      # [T, C]
    qT, s = oracle.quant_act_128x1(x)
    for tb in range(T // 128):
        for c in range(C):
            want_s, want_q = _expected_group(x[tb * 128:(tb + 1) * 128, c])
            assert Fraction(float(s[tb, c])) == want_s, (tb, c)
            assert np.array_equal(qT[c, tb * 128:(tb + 1) * 128], want_q), (tb, c)


def test_fp32_scale_and_codes_are_the_correctly_rounded_definition_128x128():
    rng = np.random.default_rng(23)
    N, K = 128, 256
    w = np.empty((N, K), np.float32)
    for kb in range(K // 128):
        amax = _non_pow2_amax(rng)
        blk = _planted_values(rng, amax, 128 * 128, 160)
        blk[int(rng.integers(160, 128 * 128))] = -amax
        w[:, kb * 128:(kb + 1) * 128] = rng.permutation(blk).reshape(128, 128)
    q, s = oracle.quant_w_128x128(w)
    for kb in range(K // 128):
        blk = w[:, kb * 128:(kb + 1) * 128]
        want_s, want_q = _expected_group(blk.reshape(-1))
        assert Fraction(float(s[0, kb])) == want_s, kb
        assert np.array_equal(q[:, kb * 128:(kb + 1) * 128].reshape(-1), want_q), kb


# ---------------------------------------------------------------- invariants

def _groups_1x128(a):
    M, K = a.shape
    return a.reshape(M, K // 128, 128)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_every_nonzero_group_has_a_448_code_and_bounded_round_trip(dtype):
    x32 = synth.activations(64, 1024, seed=5, outlier_seed=6).float().numpy()
    x32[3, 128:256] = 0.0                                       # an all-zero group
    x_in = _bits(x32) if dtype == "bf16" else x32
    x_val = _from_bits(x_in) if dtype == "bf16" else x32
    q, s = oracle.quant_act_1x128(x_in)
    g = _groups_1x128(q)
    xv = _groups_1x128(x_val.astype(np.float64))
    amax = np.abs(xv).max(axis=2)
    has448 = ((g & 0x7F) == 0x7E).any(axis=2)
    assert np.array_equal(has448, amax > 0)
    # zero group: scale 1, codes +-0
    assert s[1, 3] == 1.0 and np.all((g[3, 1] & 0x7F) == 0)
    # the stored scale is amax/448 correctly rounded to FP32 (exact rationals)
    nz = amax > 0
    sv = s.T.astype(np.float64)
    want = [fl32(Fraction(float(a)) / 448) for a in amax[nz]]
    assert [Fraction(float(v)) for v in sv[nz]] == want
    # round trip: relative error <= 2^-4 (3 mantissa bits, RNE) in the normal range
    deq = dec(g) * sv[:, :, None]
    r = np.abs(xv) / sv[:, :, None]
    normal = (r >= 2.0 ** -6) & nz[:, :, None]
    err = np.abs(deq - xv)
    assert np.all(err[normal] <= np.abs(xv[normal]) * (2.0 ** -4 + 2.0 ** -20))
    sub = (r < 2.0 ** -6) & nz[:, :, None]
    bound_sub = (2.0 ** -10 + 2.0 ** -20) * np.broadcast_to(sv[:, :, None], xv.shape)
    assert np.all(err[sub] <= bound_sub[sub])
    # sign bit follows the input's sign (zeros keep theirs)
    assert np.array_equal((g >> 7).astype(bool), np.signbit(xv))
    # codes are monotone in x inside a group
    for m in range(0, 64, 9):
        for kb in range(8):
            o = np.argsort(xv[m, kb], kind="stable")
            d = dec(g[m, kb][o])
            assert np.all(np.diff(d) >= 0)


def test_pow2_mode_scales_are_least_powers_of_two_and_exact():
    rng = np.random.default_rng(7)
    x32 = (rng.standard_normal((16, 512)) * np.exp(rng.uniform(-20, 20, (16, 1)))).astype(np.float32)
    q, s = oracle.quant_act_1x128(x32, oracle.SCALE_POW2)
    xv = _groups_1x128(x32.astype(np.float64))
    amax = np.abs(xv).max(axis=2)
    sv = s.T.astype(np.float64)
    m, e = np.frexp(sv)
    assert np.all(m == 0.5)                                     # powers of two
    assert np.all(amax <= 448.0 * sv) and np.all(amax > 224.0 * sv)   # least such power
    # scaling is exact: codes equal the nearest-E4M3 of x/s, no saturation
    g = _groups_1x128(q)
    assert np.all(np.abs(dec(g)) <= 448.0)
    ref = oracle.e4m3_encode_array((xv / sv[:, :, None]).astype(np.float32))
    assert np.array_equal(ref, g)      # x/s is exact in fp32 (power-of-two scaling)


def test_pow2_round_trip_is_exact_for_values_already_on_the_grid():
    rng = np.random.default_rng(8)
    codes = rng.integers(0, 0x7E, (4, 256)).astype(np.uint8) | (rng.integers(0, 2, (4, 256)) << 7).astype(np.uint8)
    codes[:, 5] = 0x7E                     # first groups: max 448, on the grid
    # second groups: magnitudes below 240 (code 0x77), then one -240 (0xF7) as
    # the max, which lies in (224, 448] so the least power-of-two scale is 2^e0
    mag = rng.integers(0, 0x77, (4, 128)).astype(np.uint8)
    codes[:, 128:256] = mag | (codes[:, 128:256] & 0x80)
    codes[:, 128 + 9] = 0xF7
    e0 = np.array([[-3, 5], [0, -12], [7, 1], [-20, 20]])
    x = dec(codes).reshape(4, 2, 128) * (2.0 ** e0)[:, :, None]
    q, s = oracle.quant_act_1x128(x.reshape(4, 256).astype(np.float32), oracle.SCALE_POW2)
    assert np.array_equal(q, codes)
    assert np.array_equal(s.T, (2.0 ** e0).astype(np.float32))


def test_tiny_group_scale_saturates_at_flt_min():
    x = np.zeros((1, 256), np.float32)
    x[0, :128] = np.float32(1e-37) * np.linspace(-1, 1, 128, dtype=np.float32)
    x[0, 128:] = np.float32(2.0 ** -117)                     # just above the threshold
    q, s = oracle.quant_act_1x128(x)
    assert s[0, 0] == np.float32(2.0 ** -126)
    assert np.array_equal(q[0, :128], oracle.e4m3_encode_array(x[0, :128] * np.float32(2.0 ** 126)))
    assert s[1, 0] != np.float32(2.0 ** -126) and np.all(q[0, 128:] == 0x7E)


# ---------------------------------------------------------------- cross-orientation relations

def test_128x1_equals_1x128_of_the_transpose():
    x = synth.activations(256, 384, seed=13, outlier_seed=14)
    xb = synth.bf16_bits(x)
    qT, s = oracle.quant_act_128x1(xb)
    q2, s2 = oracle.quant_act_1x128(np.ascontiguousarray(xb.T))
    assert np.array_equal(qT, q2) and np.array_equal(s, s2)


def test_128x128_scale_is_the_max_of_its_rows_1x128_scales():
    w = synth.normal((384, 256), 0.02, 15)
    wb = synth.bf16_bits(w)
    q, s = oracle.quant_w_128x128(wb)
    _, s_rows = oracle.quant_act_1x128(wb)                     # [K/128, N]
    blockmax = s_rows.reshape(256 // 128, 384 // 128, 128).max(axis=2).T
    assert np.array_equal(s, blockmax)
    # and every 128x128 block has its +-448 code
    blk = q.reshape(3, 128, 2, 128).transpose(0, 2, 1, 3).reshape(3, 2, -1)
    assert np.all(((blk & 0x7F) == 0x7E).any(axis=2))
