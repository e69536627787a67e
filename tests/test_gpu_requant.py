"""GPU parity of fp8_requant_1x128_to_128x1 (cached 1x128 FP8 activations ->
dequantize -> 128x1 groups along tokens) against the CPU oracle: codes and
scales bit-exact, both scale modes, padded leading dimensions, degenerate
groups, the quantize -> requantize chain, and the full Wgrad activation.
"""
import numpy as np
import pytest
import torch

import fp8_fine_grained_x1_b200 as fg
import oracle
from fp8_fine_grained_x1_b200 import synth

from gpu_util import dev, to_dev

pytestmark = pytest.mark.gpu
MODES = [fg.SCALE_FP32, fg.SCALE_POW2]


def _check(q, sA, mode, pad_q=0, pad_qT=0):
    T, C = q.shape
    qd = torch.zeros((T, C + pad_q), dtype=torch.uint8, device=dev())[:, :C]
    qd.copy_(to_dev(q))
    qT = torch.full((C, T + pad_qT), 0xA5, dtype=torch.uint8, device=dev())
    s = torch.empty((T // 128, C), dtype=torch.float32, device=dev())
    fg.fp8_requant_1x128_to_128x1(qd, to_dev(sA), qT[:, :T], s, mode)
    torch.cuda.synchronize()
    qT_ref, s_ref = oracle.requant_1x128_to_128x1(q, sA, mode)
    got = qT.cpu().numpy()
    assert np.array_equal(got[:, :T], qT_ref)
    assert np.all(got[:, T:] == 0xA5)                          # padding untouched
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("T,C", [(128, 128), (256, 384), (640, 1024), (1152, 256)])
def test_requant_bitexact(mode, T, C):
    q = synth.random_e4m3_codes((T, C), T + C)
    sA = synth.random_scales((C // 128, T), T + C + 1)
    _check(q, sA, mode)


@pytest.mark.parametrize("mode", MODES)
def test_requant_padded_strides(mode):
    q = synth.random_e4m3_codes((384, 256), 3)
    sA = synth.random_scales((2, 384), 4)
    _check(q, sA, mode, pad_q=48, pad_qT=32)


@pytest.mark.parametrize("mode", MODES)
def test_requant_degenerate_groups(mode):
    T, C = 384, 512
    q = synth.random_e4m3_codes((T, C), 5)
    sA = synth.random_scales((C // 128, T), 6)
    q[:128, :128] = 0                                          # all-zero groups
    q[128:256, 128:256] = np.where(np.arange(128) % 2, 0x80, 0x00)[None, :]   # signed zeros
    q[:, 256:384] &= 0x87                                      # E4M3 subnormals only
    sA[2, :] = np.float32(2.0 ** -126)                         # ... at the smallest scale
    sA[3, :128] = np.float32(2.0 ** 100)                       # huge scales
    q[256:, 384:] = np.where(np.random.default_rng(7).random((128, 128)) < 0.5, 0x7E, 0xFE)
    _check(q, sA, mode)


@pytest.mark.parametrize("mode", MODES)
def test_quantize_then_requantize_chain(mode):
    T, C = 512, 768
    x = synth.activations(T, C, seed=11, outlier_seed=12)
    q, sA = fg.quant_act_1x128(x.to(dev()), mode)
    qT, s = fg.requant_1x128_to_128x1(q, sA, mode)
    torch.cuda.synchronize()
    oq, osA = oracle.quant_act_1x128(synth.bf16_bits(x), mode)
    oqT, os_ = oracle.requant_1x128_to_128x1(oq, osA, mode)
    assert np.array_equal(qT.cpu().numpy(), oqT)
    assert np.array_equal(s.cpu().numpy(), os_)


def test_requant_full_size_wgrad_activation():
    """X of the Wgrad workload (8192 tokens x 7168 channels), cached as 1x128."""
    x = synth.wgrad()["x"]
    oq, osA = oracle.quant_act_1x128(synth.bf16_bits(x))
    _check(oq, osA, fg.SCALE_FP32)
