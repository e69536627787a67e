"""GPU parity of the FP8 MoE dispatch and combine against the CPU oracle.

Dispatch is byte and index work: codes, scales, group offsets, token_row and
row_token must equal the oracle's bit for bit.  The combine is compared
within 2^-20 * sum_j |w D| + half a BF16 ulp.
"""
import numpy as np
import pytest
import torch

import fp8_fine_grained_x1_b200 as fg
import oracle
from fp8_fine_grained_x1_b200 import synth
from oracle import moe as omoe

from gpu_util import assert_gemm_close, d2h, dev, half_ulp_bf16, to_dev

pytestmark = pytest.mark.gpu


def _dispatch_case(T, K, k, G, seed, topk=None):
    q = synth.random_e4m3_codes((T, K), seed)
    sA = synth.random_scales((K // 128, T), seed + 1)
    if topk is None:
        topk = synth.zipf_topk_routing(T, G, k, seed=seed + 2).numpy().astype(np.int32)
    return q, sA, topk


def _check_dispatch(q, sA, topk, G, M_cap=None):
    T, K = q.shape
    k = topk.shape[1]
    M_cap = fg.moe_capacity(T, k, G) if M_cap is None else M_cap
    got = fg.moe_dispatch(to_dev(q), to_dev(sA), to_dev(topk), G, M_cap)
    assert fg.fp8_get_status() == fg.FP8_OK
    ref = omoe.moe_dispatch(q, sA, topk, G, M_cap)
    for key in ("offsets", "token_row", "row_token", "q"):
        assert np.array_equal(got[key].cpu().numpy(), ref[key]), key
    assert np.array_equal(got["sA"].cpu().numpy().view(np.uint32), ref["sA"].view(np.uint32))
    return got, ref


@pytest.mark.parametrize("T,K,k,G", [(1, 128, 1, 1), (300, 256, 4, 6), (3000, 512, 8, 32)])
def test_dispatch_bitexact(T, K, k, G):
    q, sA, topk = _dispatch_case(T, K, k, G, seed=T + G)
    if G > 1:
        topk[topk == G - 1] = 0                       # one expert receives nothing
    _check_dispatch(q, sA, topk, G)


def test_dispatch_repeated_expert_in_a_token():
    topk = np.zeros((200, 4), np.int32)
    topk[:, 1] = 2                                    # slots 0, 2, 3 all pick expert 0
    q, sA, topk = _dispatch_case(200, 256, 4, 3, seed=9, topk=topk)
    _check_dispatch(q, sA, topk, 3)


def test_dispatch_full_size_moe_routing():
    wl_topk = synth.zipf_topk_routing(16384, 32, 8, seed=3).numpy().astype(np.int32)
    q = synth.random_e4m3_codes((16384, 7168), 5)
    sA = synth.random_scales((56, 16384), 6)
    got, ref = _check_dispatch(q, sA, wl_topk, 32)
    lay = synth.moe_layout(torch.from_numpy(wl_topk.astype(np.int64)), 32)
    assert np.array_equal(got["offsets"].cpu().numpy(), lay.offsets.numpy())


def test_dispatch_reports_bad_expert_ids_and_overflow():
    q, sA, topk = _dispatch_case(256, 128, 2, 4, seed=11)
    bad = topk.copy()
    bad[5, 1] = 4                                     # outside [0, G)
    got = fg.moe_dispatch(to_dev(q), to_dev(sA), to_dev(bad), 4)
    assert fg.fp8_get_status() == fg.FP8_ERR_SHAPE
    assert got["token_row"][5, 1].item() == -1
    fg.moe_dispatch(to_dev(q), to_dev(sA), to_dev(topk), 4, M_cap=128)   # too small
    assert fg.fp8_get_status() == fg.FP8_ERR_SHAPE
    assert fg.fp8_get_status() == fg.FP8_OK


def _quant_dispatch(x, topk, G, mode, M_cap=None):
    T, K = x.shape
    k = topk.shape[1]
    M_cap = fg.moe_capacity(T, k, G) if M_cap is None else M_cap
    d = dev()
    # outputs filled with junk, so that anything left unwritten shows
    out = dict(q=torch.full((M_cap, K), 0x5A, dtype=torch.uint8, device=d),
               sA=torch.full((K // 128, M_cap), -7.0, dtype=torch.float32, device=d),
               offsets=torch.full((G + 1,), -9, dtype=torch.int32, device=d),
               token_row=torch.full((T, k), -9, dtype=torch.int32, device=d),
               row_token=torch.full((M_cap,), -9, dtype=torch.int32, device=d))
    ws = torch.empty(max(1, fg.fp8_moe_dispatch_workspace_bytes(T, k, G) // 4), dtype=torch.int32,
                     device=d)
    fg.fp8_moe_quant_dispatch(x, to_dev(topk), G, out["q"], out["sA"], out["offsets"],
                              out["token_row"], out["row_token"], ws, mode)
    return out


@pytest.mark.parametrize("T,K,k,G,dtype,mode", [
    (1, 128, 1, 1, "bf16", fg.SCALE_POW2),
    (300, 256, 4, 6, "bf16", fg.SCALE_FP32),       # ragged token count, an empty expert
    (1000, 512, 8, 32, "fp32", fg.SCALE_POW2),
    (129, 384, 20, 32, "bf16", fg.SCALE_FP32),     # more than 16 destinations per token
])
def test_quant_dispatch_equals_oracle_quantizer_then_dispatch(T, K, k, G, dtype, mode):
    x = synth.activations(T, K, seed=T + k, outlier_seed=T + k + 1)
    topk = synth.zipf_topk_routing(T, G, k, seed=T + G).numpy().astype(np.int32)
    if G > 2:
        topk[topk == G - 1] = 0                       # one expert receives nothing
    xin = x if dtype == "bf16" else x.float()
    got = _quant_dispatch(xin.to(dev()), topk, G, mode)
    assert fg.fp8_get_status() == fg.FP8_OK
    oq, os_ = oracle.quant_act_1x128(synth.bf16_bits(x) if dtype == "bf16" else xin.numpy(), mode)
    ref = omoe.moe_dispatch(oq, os_, topk, G, got["q"].shape[0])
    for key in ("offsets", "token_row", "row_token", "q"):
        assert np.array_equal(got[key].cpu().numpy(), ref[key]), key
    assert np.array_equal(got["sA"].cpu().numpy().view(np.uint32), ref["sA"].view(np.uint32))


def test_quant_dispatch_reports_bad_expert_ids_like_the_dispatch():
    T, K, k, G = 256, 256, 2, 4
    x = synth.activations(T, K, seed=31, outlier_seed=32).to(dev())
    topk = synth.zipf_topk_routing(T, G, k, seed=33).numpy().astype(np.int32)
    topk[5, 1] = 4                                    # outside [0, G)
    got = _quant_dispatch(x, topk, G, fg.SCALE_FP32)
    assert fg.fp8_get_status() == fg.FP8_ERR_SHAPE
    assert got["token_row"][5, 1].item() == -1
    qx, sx = fg.quant_act_1x128(x)
    ref = fg.moe_dispatch(qx, sx, to_dev(topk), G)
    assert fg.fp8_get_status() == fg.FP8_ERR_SHAPE
    for key in ("offsets", "token_row", "row_token", "q"):
        assert torch.equal(got[key], ref[key]), key
    assert torch.equal(got["sA"].view(torch.int32), ref["sA"].view(torch.int32))


@pytest.mark.parametrize("M_cap", [384, 640])
def test_quant_dispatch_over_capacity_matches_the_dispatch(M_cap):
    """A capacity below the padded total: both paths report it, drop the same
    pairs, and write the same rows (the padding kernel of the fused path only
    visits each group's last 127 rows and the unclaimed tail)."""
    T, K, k, G = 200, 256, 3, 5
    x = synth.activations(T, K, seed=41, outlier_seed=42).to(dev())
    topk = synth.zipf_topk_routing(T, G, k, seed=43).numpy().astype(np.int32)
    got = _quant_dispatch(x, topk, G, fg.SCALE_FP32, M_cap=M_cap)
    assert fg.fp8_get_status() == fg.FP8_ERR_SHAPE
    qx, sx = fg.quant_act_1x128(x)
    ref = fg.moe_dispatch(qx, sx, to_dev(topk), G, M_cap=M_cap)
    assert fg.fp8_get_status() == fg.FP8_ERR_SHAPE
    for key in ("offsets", "token_row", "row_token", "q"):
        assert torch.equal(got[key], ref[key]), key
    assert torch.equal(got["sA"].view(torch.int32), ref["sA"].view(torch.int32))
    assert fg.fp8_get_status() == fg.FP8_OK


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_combine_matches_oracle(dtype):
    rng = np.random.default_rng(3)
    M_cap, N, T, k = 2048, 256, 300, 4
    D32 = rng.standard_normal((M_cap, N)).astype(np.float32)
    Dt = torch.from_numpy(D32).to(torch.bfloat16 if dtype == "bf16" else torch.float32)
    token_row = rng.permutation(M_cap)[:T * k].reshape(T, k).astype(np.int32)
    token_row[7, 2] = -1                              # a dropped pair
    w = rng.uniform(0, 1, (T, k)).astype(np.float32)
    out = torch.empty((T, N), dtype=torch.bfloat16, device=dev())
    fg.fp8_moe_combine(Dt.to(dev()), to_dev(token_row), to_dev(w), out)
    torch.cuda.synchronize()
    ref, mag = omoe.moe_combine(Dt.float().numpy(), token_row, w)
    got = d2h(out)
    bound = 2.0 ** -20 * mag + half_ulp_bf16(np.maximum(np.abs(ref), np.abs(got)))
    assert np.all(np.abs(got - ref) <= bound)


def test_moe_layer_quantize_dispatch_grouped_gemm_combine():
    """Tokens -> 1x128 -> FP8 dispatch -> grouped GEMM -> weighted combine."""
    T, K, N, G, k = 640, 512, 256, 8, 4
    x = synth.activations(T, K, seed=21, outlier_seed=22)
    w = synth.normal((G, N, K), 0.02, 23)
    topk = synth.zipf_topk_routing(T, G, k, seed=24).numpy().astype(np.int32)
    gate = np.random.default_rng(25).uniform(0, 1, (T, k)).astype(np.float32)

    qx, sx = fg.quant_act_1x128(x.to(dev()))
    disp = fg.moe_dispatch(qx, sx, to_dev(topk), G)
    qw, sw = fg.quant_w_128x128(w.to(dev()).view(G * N, K))
    y = fg.grouped_gemm(disp["q"], disp["sA"], qw.view(G, N, K), sw.view(G, N // 128, K // 128),
                        disp["offsets"])
    out = torch.empty((T, N), dtype=torch.bfloat16, device=dev())
    fg.fp8_moe_combine(y, disp["token_row"], to_dev(gate), out)
    torch.cuda.synchronize()
    assert fg.fp8_get_status() == fg.FP8_OK

    oq, os_ = oracle.quant_act_1x128(synth.bf16_bits(x))
    ow, osw = oracle.quant_w_128x128(synth.bf16_bits(w.view(G * N, K)))
    od = omoe.moe_dispatch(oq, os_, topk, G, disp["q"].shape[0])
    assert np.array_equal(disp["q"].cpu().numpy(), od["q"])
    # reference chain entirely from the oracle: FP64 GEMM of every real row,
    # then the FP64 combine of those rows
    rows = int(od["offsets"][-1])
    pts = np.array([(m, n) for m in range(rows) for n in range(N)], np.int64)
    ref, tol, _ = oracle.grouped_gemm_points(od["q"], od["sA"], ow.reshape(G, N, K),
                                             osw.reshape(G, N // 128, K // 128), od["offsets"], pts)
    ref_y = np.zeros((disp["q"].shape[0], N))
    tol_y = np.zeros_like(ref_y)
    ref_y[:rows] = ref.reshape(rows, N)
    tol_y[:rows] = tol.reshape(rows, N)
    assert_gemm_close(d2h(y)[:rows], ref_y[:rows], tol_y[:rows], True, "moe layer gemm")
    cref, mag = omoe.moe_combine(ref_y, od["token_row"], gate)
    # each gathered row may differ from its FP64 value by the GEMM bound plus
    # its BF16 rounding; the combine adds FP32 sums and one BF16 rounding
    y_err = 1e-4 * tol_y + half_ulp_bf16(np.abs(ref_y) + 1e-4 * tol_y)
    err_in, _ = omoe.moe_combine(y_err, od["token_row"], np.abs(gate))
    got = d2h(out)
    bound = err_in + 2.0 ** -20 * (mag + err_in) + half_ulp_bf16(np.abs(cref) + err_in)
    assert np.all(np.abs(got - cref) <= bound)
