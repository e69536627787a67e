"""Full-size parity of the five workloads (plus Wgrad from cached FP8 X), run exactly as bench.py runs them
(the step objects of fp8_fine_grained_x1_b200.linear, one GPU, persistent
GEMM grid), against the CPU oracle on the same seeded inputs.

Quantized operands are compared in full (bit-exact); GEMM outputs at
sampled points the oracle computes one by one: 4096 random (m, n), whole
rows and columns at the first/last tile edges, and for the MoE layer the
first, last-real and last-padding row of every expert group.
"""
import numpy as np
import pytest
import torch

import fp8_fine_grained_x1_b200 as fg
import oracle
from fp8_fine_grained_x1_b200 import linear, synth
from oracle import moe as omoe

from gpu_util import assert_gemm_close, d2h, dev

pytestmark = pytest.mark.gpu


def _points(M, N, seed, n_random=4096, rows=(), cols=()):
    rng = np.random.default_rng(seed)
    pts = [np.stack([rng.integers(0, M, n_random), rng.integers(0, N, n_random)], 1)]
    for m in rows:
        pts.append(np.stack([np.full(N, m), np.arange(N)], 1))
    for n in cols:
        pts.append(np.stack([np.arange(M), np.full(M, n)], 1))
    return np.concatenate(pts).astype(np.int64)


def _edges(n, tile):
    return sorted({0, min(tile - 1, n - 1), min(tile, n - 1), n - 1})


def _bits(t):
    return synth.bf16_bits(t) if t.dtype == torch.bfloat16 else t.numpy()


def test_pr1_tiny_fprop_full_output():
    wl = synth.pr1()
    step = linear.FpropStep(wl["x"].to(dev()), wl["w"].to(dev()), out_dtype=torch.float32)
    y = d2h(step())
    assert fg.fp8_get_status() == fg.FP8_OK
    qx, sx = oracle.quant_act_1x128(wl["x"].numpy())
    qw, sw = oracle.quant_w_128x128(wl["w"].numpy())
    assert np.array_equal(step.qx.cpu().numpy(), qx) and np.array_equal(step.sx.cpu().numpy(), sx)
    assert np.array_equal(step.qw.cpu().numpy(), qw) and np.array_equal(step.sw.cpu().numpy(), sw)
    ref, tol = oracle.gemm_full(qx, sx, qw, sw)
    assert_gemm_close(y, ref, tol, False, "pr1")


def test_fprop_dense_mlp():
    wl = synth.fprop()
    step = linear.FpropStep(wl["x"].to(dev()), wl["w"].to(dev()))
    y = step()
    torch.cuda.synchronize()
    assert fg.fp8_get_status() == fg.FP8_OK
    qx, sx = oracle.quant_act_1x128(_bits(wl["x"]))
    qw, sw = oracle.quant_w_128x128(_bits(wl["w"]))
    assert np.array_equal(step.qx.cpu().numpy(), qx) and np.array_equal(step.sx.cpu().numpy(), sx)
    assert np.array_equal(step.qw.cpu().numpy(), qw) and np.array_equal(step.sw.cpu().numpy(), sw)
    M, N = y.shape
    pts = _points(M, N, 1, rows=_edges(M, 128), cols=_edges(N, 256))
    ref, tol = oracle.gemm_points(qx, sx, qw, sw, pts)
    got = d2h(y)[pts[:, 0], pts[:, 1]]
    assert_gemm_close(got, ref, tol, True, "fprop")


def test_dgrad_reads_weight_transposed():
    wl = synth.dgrad()
    step = linear.DgradStep(wl["dy"].to(dev()), wl["w"].to(dev()))
    dx = step()
    torch.cuda.synchronize()
    assert fg.fp8_get_status() == fg.FP8_OK
    qdy, sdy = oracle.quant_act_1x128(_bits(wl["dy"]))
    qw, sw = oracle.quant_w_128x128(_bits(wl["w"]))               # stored [N_out][K_in]
    assert np.array_equal(step.qdy.cpu().numpy(), qdy) and np.array_equal(step.qw.cpu().numpy(), qw)
    assert np.array_equal(step.sdy.cpu().numpy(), sdy) and np.array_equal(step.sw.cpu().numpy(), sw)
    M, N = dx.shape
    pts = _points(M, N, 2, rows=_edges(M, 128), cols=_edges(N, 256))
    ref, tol = oracle.gemm_points(qdy, sdy, qw, sw, pts, b_major=oracle.B_MNMAJOR)
    assert_gemm_close(d2h(dx)[pts[:, 0], pts[:, 1]], ref, tol, True, "dgrad")


@pytest.mark.parametrize("mode", [fg.SCALE_FP32, fg.SCALE_POW2])
def test_wgrad_token_axis_groups(mode):
    wl = synth.wgrad()
    step = linear.WgradStep(wl["x"].to(dev()), wl["dy"].to(dev()), scale_mode=mode)
    dw = step()
    torch.cuda.synchronize()
    assert fg.fp8_get_status() == fg.FP8_OK
    qxT, sx = oracle.quant_act_128x1(_bits(wl["x"]), mode)
    qdyT, sdy = oracle.quant_act_128x1(_bits(wl["dy"]), mode)
    assert np.array_equal(step.qxT.cpu().numpy(), qxT) and np.array_equal(step.sx.cpu().numpy(), sx)
    assert np.array_equal(step.qdyT.cpu().numpy(), qdyT) and np.array_equal(step.sdy.cpu().numpy(), sdy)
    M, N = dw.shape
    pts = _points(M, N, 3, rows=_edges(M, 128), cols=_edges(N, 256))
    ref, tol = oracle.gemm_points(qdyT, sdy, qxT, sx, pts, sb_gran=1)
    assert_gemm_close(d2h(dw)[pts[:, 0], pts[:, 1]], ref, tol, False, f"wgrad mode={mode}")


def test_wgrad_pow2_scaled_in_tensor_cores():
    wl = synth.wgrad()
    step = linear.WgradStep(wl["x"].to(dev()), wl["dy"].to(dev()), scale_mode=fg.SCALE_POW2,
                            tensor_core_scaling=True)
    dw = step()
    torch.cuda.synchronize()
    assert fg.fp8_get_status() == fg.FP8_OK
    qxT, sx = oracle.quant_act_128x1(_bits(wl["x"]), fg.SCALE_POW2)
    qdyT, sdy = oracle.quant_act_128x1(_bits(wl["dy"]), fg.SCALE_POW2)
    assert np.array_equal(step.qxT.cpu().numpy(), qxT) and np.array_equal(step.sx.cpu().numpy(), sx)
    M, N = dw.shape
    pts = _points(M, N, 6, rows=_edges(M, 128), cols=_edges(N, 256))
    ref, tol = oracle.gemm_points(qdyT, sdy, qxT, sx, pts, sb_gran=1)
    assert_gemm_close(d2h(dw)[pts[:, 0], pts[:, 1]], ref, tol, False, "wgrad pow2 tensor-core")


def test_fprop_pow2_scaled_in_tensor_cores():
    wl = synth.fprop()
    step = linear.FpropStep(wl["x"].to(dev()), wl["w"].to(dev()), scale_mode=fg.SCALE_POW2,
                            tensor_core_scaling=True)
    y = step()
    torch.cuda.synchronize()
    assert fg.fp8_get_status() == fg.FP8_OK
    qx, sx = oracle.quant_act_1x128(_bits(wl["x"]), fg.SCALE_POW2)
    qw, sw = oracle.quant_w_128x128(_bits(wl["w"]), fg.SCALE_POW2)
    assert np.array_equal(step.qx.cpu().numpy(), qx) and np.array_equal(step.qw.cpu().numpy(), qw)
    M, N = y.shape
    pts = _points(M, N, 7, rows=_edges(M, 128), cols=_edges(N, 256))
    ref, tol = oracle.gemm_points(qx, sx, qw, sw, pts)
    assert_gemm_close(d2h(y)[pts[:, 0], pts[:, 1]], ref, tol, True, "fprop pow2 tensor-core")


def test_wgrad_from_cached_fp8_activations():
    """Wgrad with X taken from its cached 1x128 FP8 form (the forward's cache
    is made by the oracle here), requantized to 128x1 on the GPU."""
    wl = synth.wgrad()
    cq, cs = oracle.quant_act_1x128(_bits(wl["x"]))
    step = linear.WgradCachedStep(torch.from_numpy(cq).to(dev()), torch.from_numpy(cs).to(dev()),
                                  wl["dy"].to(dev()))
    dw = step()
    torch.cuda.synchronize()
    assert fg.fp8_get_status() == fg.FP8_OK
    qxT, sx = oracle.requant_1x128_to_128x1(cq, cs)
    qdyT, sdy = oracle.quant_act_128x1(_bits(wl["dy"]))
    assert np.array_equal(step.qxT.cpu().numpy(), qxT) and np.array_equal(step.sxT.cpu().numpy(), sx)
    assert np.array_equal(step.qdyT.cpu().numpy(), qdyT) and np.array_equal(step.sdy.cpu().numpy(), sdy)
    M, N = dw.shape
    pts = _points(M, N, 5, rows=_edges(M, 128), cols=_edges(N, 256))
    ref, tol = oracle.gemm_points(qdyT, sdy, qxT, sx, pts, sb_gran=1)
    assert_gemm_close(d2h(dw)[pts[:, 0], pts[:, 1]], ref, tol, False, "wgrad from cache")


@pytest.mark.parametrize("pow2_tc", [False, True], ids=["fp32_scales", "pow2_tensor_cores"])
def test_moe_grouped_fprop(pow2_tc):
    wl = synth.moe()
    lay = wl["layout"]
    G, N, K = wl["w"].shape
    mode = fg.SCALE_POW2 if pow2_tc else fg.SCALE_FP32
    topk = lay.topk.to(torch.int32)
    step = linear.MoeStep(wl["x"].to(dev()), topk.to(dev()), wl["w"].to(dev()), scale_mode=mode,
                          tensor_core_scaling=pow2_tc)
    y = step()
    torch.cuda.synchronize()
    assert fg.fp8_get_status() == fg.FP8_OK
    # layout: identical to the generator's independent expert ordering
    off = step.offsets.cpu().numpy()
    assert np.array_equal(off, lay.offsets.numpy())
    assert np.array_equal(step.row_token.cpu().numpy()[:lay.m_total], lay.row_token.numpy())

    # weights quantized by the oracle, bit-exact; the tokens' codes exist
    # only in their dispatched rows (checked below)
    qx, sx = oracle.quant_act_1x128(_bits(wl["x"]), mode)
    qw, sw = oracle.quant_w_128x128(_bits(wl["w"].view(G * N, K)), mode)
    assert np.array_equal(step.qw.cpu().numpy().reshape(G * N, K), qw)
    assert np.array_equal(step.sw.cpu().numpy().reshape(G * N // 128, K // 128), sw)
    qw = qw.reshape(G, N, K)
    sw = sw.reshape(G, N // 128, K // 128)

    # the oracle's dispatch of the oracle's codes: the rows the GEMM must see;
    # the step holds them dispatched (tensor-core scaling) or reads them
    # through row_token from the tokens' own codes (gather), bit-exact either way
    od = omoe.moe_dispatch(qx, sx, topk.numpy(), G, step.M_cap)
    if step.gather:
        assert np.array_equal(step.qx.cpu().numpy(), qx)
        assert np.array_equal(step.sx.cpu().numpy(), sx)
        assert np.array_equal(step.row_token.cpu().numpy(), od["row_token"])
    else:
        assert np.array_equal(step.qa.cpu().numpy(), od["q"])
        assert np.array_equal(step.sa.cpu().numpy(), od["sA"])

    # GEMM at the first, last-real and last-padding row of every expert + random rows
    rng = np.random.default_rng(4)
    rows = set(rng.integers(0, lay.m_total, 64).tolist())
    for e in range(G):
        if off[e + 1] > off[e]:
            rows |= {int(off[e]), int(off[e] + lay.counts[e] - 1), int(off[e + 1] - 1)}
    rows = np.array(sorted(rows))
    yh = d2h(y)
    for e in range(G):
        sel = rows[(rows >= off[e]) & (rows < off[e + 1])]
        if sel.size == 0:
            continue
        pts = np.array([(i, n) for i in sel for n in range(N)], np.int64)
        ref, tol = oracle.gemm_points(od["q"], od["sA"], qw[e], sw[e], pts)
        assert_gemm_close(yh[pts[:, 0], pts[:, 1]], ref, tol, True, f"moe expert {e}")
    pad = step.row_token.cpu().numpy()[:lay.m_total] < 0
    assert np.all(yh[:lay.m_total][pad] == 0.0)
