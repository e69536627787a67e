"""Pins of the oracle's requantization of cached 1x128 FP8 activations into
the 128x1 groups Wgrad reads (reading R13: dequantize each element to
fl32(decode(q) * sA), then group along tokens as for an FP32 input).

What fixes it: the pages cache activations in FP8 with the fine-grained
(1x128) grouping and run Wgrad in FP8 on them, which needs groups along the
token axis.  The checks are special cases with closed forms, a planted
single element (catches any transposed or shifted index), the round-trip
bound of E4M3, the max-abs -> +-448 invariant, and agreement with the
separately pinned 128x1 quantizer applied to independently dequantized
values.
"""
import numpy as np
import pytest
import torch

import oracle
from fp8_fine_grained_x1_b200 import synth

TAB = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn) \
    .to(torch.float64).numpy()
MODES = [oracle.SCALE_FP32, oracle.SCALE_POW2]


def _dequant(q, sA):
    """Independent dequantization: the FP64 product is exact, one cast to FP32."""
    T, C = q.shape
    s_full = np.repeat(sA.astype(np.float64).T, 128, axis=1)          # [T, C]
    return (TAB[q] * s_full).astype(np.float32)


@pytest.mark.parametrize("mode", MODES)
def test_unit_scales_with_a_448_in_every_column_give_the_transpose(mode):
    T, C = 256, 256
    q = synth.random_e4m3_codes((T, C), 1)
    q[q == 0x7E] = 0x7D
    q[q == 0xFE] = 0xFD
    rng = np.random.default_rng(2)
    for tb in range(T // 128):
        rows = tb * 128 + rng.integers(0, 128, C)
        q[rows, np.arange(C)] = np.where(rng.random(C) < 0.5, 0x7E, 0xFE)   # +-448
    sA = np.ones((C // 128, T), np.float32)
    qT, s = oracle.requant_1x128_to_128x1(q, sA, mode)
    assert np.array_equal(qT, q.T)
    assert np.all(s == 1.0)


@pytest.mark.parametrize("mode", MODES)
def test_single_planted_element_lands_transposed(mode):
    T, C = 384, 256
    t, c = 200, 131
    q = np.zeros((T, C), np.uint8)
    q[t, c] = 0x4B                                       # 1.375 * 2^2 = 5.5
    sA = synth.random_scales((C // 128, T), 3)
    qT, s = oracle.requant_1x128_to_128x1(q, sA, mode)
    x = np.float32(5.5 * np.float64(sA[c // 128, t]))
    expect = np.zeros((C, T), np.uint8)
    if mode == oracle.SCALE_FP32:
        expect[c, t] = 0x7E                              # its own group's max -> 448
        assert s[t // 128, c] == np.float32(np.float64(x) / 448.0)
    else:
        e = int(np.ceil(np.log2(np.float64(x) / 448.0)))
        assert s[t // 128, c] == np.float32(2.0 ** e)
        expect[c, t] = oracle.e4m3_encode_array(np.array([np.float64(x) * 2.0 ** -e],
                                                         np.float32))[0]
    assert np.array_equal(qT, expect)
    others = np.ones_like(s, bool)
    others[t // 128, c] = False
    assert np.all(s[others] == 1.0)                      # empty groups: s = 1


@pytest.mark.parametrize("mode", MODES)
def test_equals_pinned_128x1_of_independently_dequantized_values(mode):
    T, C = 512, 384
    q = synth.random_e4m3_codes((T, C), 5)
    sA = synth.random_scales((C // 128, T), 6)
    qT, s = oracle.requant_1x128_to_128x1(q, sA, mode)
    qT2, s2 = oracle.quant_act_128x1(_dequant(q, sA), mode)
    assert np.array_equal(qT, qT2) and np.array_equal(s, s2)


@pytest.mark.parametrize("mode", MODES)
def test_round_trip_and_max_abs_invariant(mode):
    T, C = 256, 256
    q = synth.random_e4m3_codes((T, C), 7)
    sA = synth.random_scales((C // 128, T), 8)
    qT, s = oracle.requant_1x128_to_128x1(q, sA, mode)
    x = _dequant(q, sA).astype(np.float64)                # [T, C]
    s_full = np.repeat(s.astype(np.float64), 128, axis=0)  # [T, C]
    back = TAB[qT.T] * s_full
    # E4M3 normals: half an ulp is 2^-4 relative; subnormals: 2^-10 absolute
    bound = np.maximum(2.0 ** -4 * np.abs(x), 2.0 ** -10 * s_full) * (1 + 1e-12)
    assert np.all(np.abs(back - x) <= bound)
    if mode == oracle.SCALE_FP32:
        for tb in range(T // 128):
            grp = np.abs(x[tb * 128:(tb + 1) * 128])
            arg = grp.argmax(axis=0)
            codes = qT[np.arange(C), tb * 128 + arg]
            assert np.all((codes & 0x7F) == 0x7E)
