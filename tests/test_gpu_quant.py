"""GPU parity of the three quantizers against the CPU oracle: E4M3 bytes and
FP32 scales must be bit-exact (integer/byte work), on ragged small shapes,
special groups (all-zero, signed zeros, subnormal-range, tiny amax,
saturation edges, max in the last lane), both scale modes, both input
dtypes, padded leading dimensions, and the full-size workload tensors.
"""
import numpy as np
import pytest
import torch

import fp8_fine_grained_x1_b200 as fg
import oracle
from fp8_fine_grained_x1_b200 import synth

from gpu_util import bits_to_bf16_dev, dev, to_dev

pytestmark = pytest.mark.gpu


def _host_input(x32, dtype):
    """(oracle input array, device tensor) of the same values."""
    if dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(x32)).to(torch.bfloat16)
        return synth.bf16_bits(t), t.to(dev())
    return np.ascontiguousarray(x32, np.float32), to_dev(np.ascontiguousarray(x32, np.float32))


def _special_rows(K, seed):
    """Rows whose 1x128 groups hit the method's degenerate cases."""
    rng = np.random.default_rng(seed)
    nkb = K // 128
    rows = []
    r = rng.standard_normal((8, K)).astype(np.float32)
    r[0] = 0.0                                               # all-zero groups
    r[1] = np.where(rng.random(K) < 0.5, -0.0, 0.0)          # signed zeros only
    r[2] *= np.float32(1e-3)
    r[2, ::128] = np.float32(448.0)                          # max in first lane, others tiny
    r[3, 127::128] = -np.float32(1e4)                        # max in the last lane
    r[4] = rng.uniform(-1, 1, K).astype(np.float32) * np.float32(2.0 ** -120)  # tiny amax
    r[5] = np.float32(448.0) * np.sign(rng.standard_normal(K)).astype(np.float32)  # saturation
    r[6] = rng.uniform(-1, 1, K).astype(np.float32) * np.float32(3.0e38)            # huge
    r[7, :] = np.float32(2.0 ** -133)                        # bf16 subnormal-range values
    rows.append(r)
    del nkb
    return np.concatenate(rows)


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("mode", [fg.SCALE_FP32, fg.SCALE_POW2])
@pytest.mark.parametrize("M,K", [(1, 128), (3, 256), (129, 384), (200, 1024)])
def test_quant_1x128_bitexact(dtype, mode, M, K):
    x32 = synth.activations(M, K, seed=M + K, outlier_seed=7).float().numpy()
    if M >= 8:
        x32[:8] = _special_rows(K, seed=M)
    xh, xd = _host_input(x32, dtype)
    q_ref, s_ref = oracle.quant_act_1x128(xh, mode)
    q, s = fg.quant_act_1x128(xd, mode)
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("mode", [fg.SCALE_FP32, fg.SCALE_POW2])
@pytest.mark.parametrize("T,C", [(128, 8), (256, 72), (384, 200), (128, 1024)])
def test_quant_128x1_bitexact(dtype, mode, T, C):
    x32 = synth.activations(T, C, seed=T + C, outlier_seed=8).float().numpy()
    if C >= 8:
        x32[:, :8] = _special_rows(T, seed=C).T
    xh, xd = _host_input(x32, dtype)
    q_ref, s_ref = oracle.quant_act_128x1(xh, mode)
    q, s = fg.quant_act_128x1(xd, mode)
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("mode", [fg.SCALE_FP32, fg.SCALE_POW2])
@pytest.mark.parametrize("N,K", [(128, 128), (256, 384), (384, 1280)])
def test_quant_w_128x128_bitexact(dtype, mode, N, K):
    w32 = synth.normal((N, K), 0.02, N * K).float().numpy()
    w32[:128, :128] = 0.0                                     # an all-zero block
    if K >= 256:
        w32[:8, 128:256] = _special_rows(128, seed=N)[:, :128]
    xh, xd = _host_input(w32, dtype)
    q_ref, s_ref = oracle.quant_w_128x128(xh, mode)
    q, s = fg.quant_w_128x128(xd, mode)
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


def test_padded_leading_dimensions_and_guard_bytes():
    """Strided inputs/outputs: only the logical region is written."""
    M, K, ldx, ldq = 130, 256, 384, 272
    x32 = synth.activations(M, ldx, seed=3, outlier_seed=4).float().numpy()
    xb = torch.from_numpy(x32).to(torch.bfloat16)
    xd = xb.to(dev())[:, :K]
    qbuf = torch.full((M, ldq), 0xA5, dtype=torch.uint8, device=dev())
    s = torch.empty((K // 128, M), dtype=torch.float32, device=dev())
    fg.fp8_quant_act_1x128(xd, qbuf[:, :K], s)
    torch.cuda.synchronize()
    q_ref, s_ref = oracle.quant_act_1x128(np.ascontiguousarray(synth.bf16_bits(xb)[:, :K]))
    qh = qbuf.cpu().numpy()
    assert np.array_equal(qh[:, :K], q_ref)
    assert np.all(qh[:, K:] == 0xA5)
    assert np.array_equal(s.cpu().numpy(), s_ref)


# ------------------------------------------------------------ full-size tensors

@pytest.mark.parametrize("name", ["fprop_x", "fprop_w", "dgrad_dy", "dgrad_w"])
def test_full_size_bitexact(name):
    if name == "fprop_x":
        t, kind = synth.activations(4096, 7168, seed=0, outlier_seed=2), "1x128"
    elif name == "fprop_w":
        t, kind = synth.normal((18432, 7168), 0.006, 1), "w"
    elif name == "dgrad_dy":
        t, kind = synth.normal((4096, 7168), 1e-3, 4), "1x128"
    else:
        t, kind = synth.normal((7168, 2048), 0.02, 1), "w"
    bits = synth.bf16_bits(t)
    xd = t.to(dev())
    if kind == "1x128":
        q_ref, s_ref = oracle.quant_act_1x128(bits)
        q, s = fg.quant_act_1x128(xd)
    else:
        q_ref, s_ref = oracle.quant_w_128x128(bits)
        q, s = fg.quant_w_128x128(xd)
    torch.cuda.synchronize()
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy(), s_ref)


@pytest.mark.parametrize("mode", [fg.SCALE_FP32, fg.SCALE_POW2])
def test_full_size_wgrad_operands_bitexact(mode):
    wl = synth.wgrad()
    for t in (wl["x"], wl["dy"]):
        q_ref, s_ref = oracle.quant_act_128x1(synth.bf16_bits(t), mode)
        q, s = fg.quant_act_128x1(t.to(dev()), mode)
        torch.cuda.synchronize()
        assert np.array_equal(q.cpu().numpy(), q_ref)
        assert np.array_equal(s.cpu().numpy(), s_ref)


def test_gpu_encode_of_every_fp32_pattern_in_range():
    """The GPU's E4M3 encode on every FP32 bit pattern of [0, 448]: each 1x128
    group holds 448 in its first lane, so its scale is amax/448 = 1 and its
    encode factor 448/amax = 1, and every other lane's code is E(x) of its
    own value.  Compared with the oracle's encoder (itself pinned to the
    library cast on the same patterns); negatives on a strided sample."""
    hi_bits = int(np.float32(448.0).view(np.uint32))
    per = 127 << 19                                     # values per launch, 127 per group
    for start in range(0, hi_bits + 1, per):
        b = np.arange(start, min(start + per, hi_bits + 1), dtype=np.uint32)
        _encode_groups_match(b.view(np.float32))
    neg = -np.arange(0, hi_bits + 1, 9973, dtype=np.uint32).view(np.float32)
    _encode_groups_match(neg)


def _encode_groups_match(vals):
    n = vals.size
    G = (n + 126) // 127
    body = np.zeros(G * 127, np.float32)
    body[:n] = vals
    x = np.empty((G, 128), np.float32)
    x[:, 0] = 448.0
    x[:, 1:] = body.reshape(G, 127)
    q, s = fg.quant_act_1x128(to_dev(x))
    assert fg.fp8_get_status() == fg.FP8_OK
    assert torch.all(s == 1.0).item()
    got = q[:, 1:].reshape(-1)[:n].cpu().numpy()
    ref = oracle.e4m3_encode_array(vals)
    bad = np.flatnonzero(got != ref)
    assert bad.size == 0, (vals[bad[:8]], got[bad[:8]], ref[bad[:8]])


@pytest.mark.parametrize("mode", [fg.SCALE_FP32, fg.SCALE_POW2])
def test_gpu_group_scale_across_the_fp32_range(mode):
    """Group scales for maxima spread over every binade of FP32 (every 4096th
    bit pattern from the smallest subnormal to the largest finite value, and
    their negatives): one nonzero element per 1x128 group, scale and codes
    bit-exact against the oracle."""
    top = int(np.float32(np.finfo(np.float32).max).view(np.uint32))
    v = np.arange(1, top + 1, 4096, dtype=np.uint32).view(np.float32)
    v = np.concatenate([v, -v[::7]])
    x = np.zeros((v.size, 128), np.float32)
    lanes = np.arange(v.size) % 128                      # the nonzero element visits every lane
    x[np.arange(v.size), lanes] = v
    q, s = fg.quant_act_1x128(to_dev(x), mode)
    assert fg.fp8_get_status() == fg.FP8_OK
    oq, os_ = oracle.quant_act_1x128(x, mode)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), os_.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), oq)
