"""The grouped GEMM with gathered A rows (fp8_grouped_gemm_gather) and the
routing-only entry point (fp8_moe_route): against the oracle on explicitly
dispatched rows, and bit for bit against the materialized dispatch path."""
import numpy as np
import pytest
import torch

import fp8_fine_grained_x1_b200 as fg
import oracle
from fp8_fine_grained_x1_b200 import synth

from gpu_util import assert_gemm_close, d2h, dev, to_dev

pytestmark = pytest.mark.gpu


def _route(topk, G, M_cap):
    T, k = topk.shape
    d = dev()
    out = dict(offsets=torch.full((G + 1,), -9, dtype=torch.int32, device=d),
               token_row=torch.full((T, k), -9, dtype=torch.int32, device=d),
               row_token=torch.full((M_cap,), -9, dtype=torch.int32, device=d))
    ws = torch.empty(max(1, fg.fp8_moe_dispatch_workspace_bytes(T, k, G) // 4), dtype=torch.int32,
                     device=d)
    fg.fp8_moe_route(to_dev(topk), G, out["offsets"], out["token_row"], out["row_token"], ws)
    return out


@pytest.mark.parametrize("T,k,G,N,K,out", [(300, 4, 6, 256, 512, "bf16"),
                                            (1000, 8, 32, 384, 256, "fp32"),
                                            (77, 2, 3, 128, 128, "bf16")])
def test_gather_gemm_matches_oracle_on_dispatched_rows(T, k, G, N, K, out):
    topk = synth.zipf_topk_routing(T, G, k, seed=T + G).numpy().astype(np.int32)
    if G > 2:
        topk[topk == G - 1] = 0                                   # an empty expert
    A = synth.random_e4m3_codes((T, K), 501)
    sA = synth.random_scales((K // 128, T), 502)
    B = synth.random_e4m3_codes((G, N, K), 503)
    sB = synth.random_scales((G, N // 128, K // 128), 504)
    M_cap = fg.moe_capacity(T, k, G)
    r = _route(topk, G, M_cap)
    assert fg.fp8_get_status() == fg.FP8_OK
    dt = torch.bfloat16 if out == "bf16" else torch.float32
    D = torch.full((M_cap, N), -3.0, dtype=dt, device=dev())
    fg.fp8_grouped_gemm_gather(to_dev(A), to_dev(sA), r["row_token"], to_dev(B), to_dev(sB),
                               r["offsets"], D)
    assert fg.fp8_get_status() == fg.FP8_OK
    got = d2h(D)
    off = r["offsets"].cpu().numpy()
    rt = r["row_token"].cpu().numpy()
    # the dispatched operand, built on the host from the routing
    A_d = np.zeros((M_cap, K), np.uint8)
    sA_d = np.ones((K // 128, M_cap), np.float32)
    real = rt >= 0
    A_d[real] = A[rt[real]]
    sA_d[:, real] = sA[:, rt[real]]
    mm, nn = np.meshgrid(np.arange(M_cap), np.arange(N), indexing="ij")
    pts = np.stack([mm.reshape(-1), nn.reshape(-1)], axis=1).astype(np.int64)
    ref, tol, grp = oracle.grouped_gemm_points(A_d, sA_d, B, sB, off, pts)
    inside = grp >= 0
    assert_gemm_close(got.reshape(-1)[inside], ref[inside], tol[inside], out == "bf16", "gather")
    assert np.all(got.reshape(-1)[~inside] == -3.0)               # rows beyond off[G] untouched
    inside_rows = np.zeros(M_cap, bool)
    inside_rows[:off[-1]] = True
    assert np.all(got[inside_rows & ~real] == 0.0)                # padding rows exactly 0


def test_route_equals_the_dispatch_routing():
    T, k, G = 2000, 8, 32
    topk = synth.zipf_topk_routing(T, G, k, seed=7).numpy().astype(np.int32)
    M_cap = fg.moe_capacity(T, k, G)
    r = _route(topk, G, M_cap)
    q = to_dev(synth.random_e4m3_codes((T, 256), 8))
    sA = to_dev(synth.random_scales((2, T), 9))
    ref = fg.moe_dispatch(q, sA, to_dev(topk), G, M_cap=M_cap)
    assert fg.fp8_get_status() == fg.FP8_OK
    for key in ("offsets", "token_row", "row_token"):
        assert torch.equal(r[key], ref[key]), key


@pytest.mark.parametrize("out", ["bf16", "fp32"])
def test_gather_equals_the_materialized_dispatch_bit_for_bit(out):
    """Quantize the tokens, then either gather their rows in the GEMM or
    dispatch them first: the same rows and scales meet the same promotion,
    so the outputs agree bit for bit."""
    T, k, G, N, K = 2048, 8, 32, 512, 1024
    x = synth.activations(T, K, seed=11, outlier_seed=12).to(dev())
    topk = synth.zipf_topk_routing(T, G, k, seed=13).numpy().astype(np.int32)
    B = to_dev(synth.random_e4m3_codes((G, N, K), 14))
    sB = to_dev(synth.random_scales((G, N // 128, K // 128), 15))
    M_cap = fg.moe_capacity(T, k, G)
    dt = torch.bfloat16 if out == "bf16" else torch.float32
    # gathered
    r = _route(topk, G, M_cap)
    qx, sx = fg.quant_act_1x128(x)
    Dg = torch.zeros((M_cap, N), dtype=dt, device=dev())
    fg.fp8_grouped_gemm_gather(qx, sx, r["row_token"], B, sB, r["offsets"], Dg)
    # materialized
    qa = torch.empty((M_cap, K), dtype=torch.uint8, device=dev())
    sa = torch.empty((K // 128, M_cap), dtype=torch.float32, device=dev())
    off = torch.empty((G + 1,), dtype=torch.int32, device=dev())
    tr = torch.empty((T, k), dtype=torch.int32, device=dev())
    rt = torch.empty((M_cap,), dtype=torch.int32, device=dev())
    ws = torch.empty(max(1, fg.fp8_moe_dispatch_workspace_bytes(T, k, G) // 4), dtype=torch.int32,
                     device=dev())
    fg.fp8_moe_quant_dispatch(x, to_dev(topk), G, qa, sa, off, tr, rt, ws)
    Dm = torch.zeros((M_cap, N), dtype=dt, device=dev())
    fg.fp8_grouped_gemm(qa, sa, B, sB, off, Dm)
    assert fg.fp8_get_status() == fg.FP8_OK
    assert torch.equal(r["offsets"], off) and torch.equal(r["row_token"], rt)
    assert torch.equal(Dg.view(torch.int16 if out == "bf16" else torch.int32),
                       Dm.view(torch.int16 if out == "bf16" else torch.int32))


def test_gather_row_index_out_of_range_is_reported_and_gives_zero():
    T, k, G, N, K = 256, 2, 4, 128, 256
    topk = synth.zipf_topk_routing(T, G, k, seed=21).numpy().astype(np.int32)
    M_cap = fg.moe_capacity(T, k, G)
    r = _route(topk, G, M_cap)
    A = to_dev(synth.random_e4m3_codes((T, K), 22))
    sA = to_dev(synth.random_scales((K // 128, T), 23))
    B = to_dev(synth.random_e4m3_codes((G, N, K), 24))
    sB = to_dev(synth.random_scales((G, N // 128, K // 128), 25))
    rt = r["row_token"].clone()
    first = int(torch.nonzero(rt >= 0)[0].item())
    rt[first] = T + 5                                             # beyond the token rows
    D = torch.zeros((M_cap, N), dtype=torch.float32, device=dev())
    fg.fp8_grouped_gemm_gather(A, sA, rt, B, sB, r["offsets"], D)
    assert fg.fp8_get_status() == fg.FP8_ERR_SHAPE
    assert torch.all(D[first] == 0).item()
    assert fg.fp8_get_status() == fg.FP8_OK


def test_gather_rejects_bad_arguments():
    d = dev()
    A = torch.zeros((4, 128), dtype=torch.uint8, device=d)
    sA = torch.ones((1, 4), dtype=torch.float32, device=d)
    B = torch.zeros((1, 128, 128), dtype=torch.uint8, device=d)
    sB = torch.ones((1, 1, 1), dtype=torch.float32, device=d)
    off = torch.tensor([0, 128], dtype=torch.int32, device=d)
    rt = torch.full((128,), -1, dtype=torch.int32, device=d)
    D = torch.zeros((128, 128), dtype=torch.float32, device=d)
    lib = fg.load_library()
    P = lambda t: t.data_ptr()
    assert lib.fp8_grouped_gemm_gather(P(A), P(sA), 0, P(rt), P(B), P(sB), P(off), 1, 128, 128,
                                       128, P(D), 1, None) == fg.FP8_ERR_SHAPE
    assert lib.fp8_grouped_gemm_gather(P(A), P(sA), 4, None, P(B), P(sB), P(off), 1, 128, 128,
                                       128, P(D), 1, None) == fg.FP8_ERR_NULL
    assert lib.fp8_grouped_gemm_gather(P(A) + 1, P(sA), 4, P(rt), P(B), P(sB), P(off), 1, 128,
                                       128, 128, P(D), 1, None) == fg.FP8_ERR_ALIGN
    # all padding: a valid call whose output is all zero
    D.fill_(5.0)
    assert lib.fp8_grouped_gemm_gather(P(A), P(sA), 4, P(rt), P(B), P(sB), P(off), 1, 128, 128,
                                       128, P(D), 1, None) == fg.FP8_OK
    assert fg.fp8_get_status() == fg.FP8_OK
    assert torch.all(D == 0).item()


def test_moe_step_with_gather_equals_the_default_step():
    """MoeStep(gather=True) (route, quantize tokens once, gathered GEMM) and
    the default step (fused quantize-and-dispatch, grouped GEMM) give the
    same output bit for bit, and the same routing."""
    from fp8_fine_grained_x1_b200 import linear
    T, k, G, N, K = 1024, 8, 16, 256, 512
    x = synth.activations(T, K, seed=31, outlier_seed=32).to(dev())
    topk = to_dev(synth.zipf_topk_routing(T, G, k, seed=33).numpy().astype(np.int32))
    w = synth.normal((G, N, K), 0.006, 34).to(dev())
    a = linear.MoeStep(x, topk, w)
    b = linear.MoeStep(x, topk, w, gather=True)
    ya, yb = a(), b()
    torch.cuda.synchronize()
    assert fg.fp8_get_status() == fg.FP8_OK
    assert b.kernel_calls == 6 and a.kernel_calls == 7
    assert torch.equal(a.offsets, b.offsets) and torch.equal(a.row_token, b.row_token)
    assert torch.equal(a.token_row, b.token_row)
    used = int(a.offsets[-1].item())                              # rows past off[G] are not written
    assert torch.equal(ya[:used].view(torch.int16), yb[:used].view(torch.int16))
