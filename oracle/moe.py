"""CPU oracle of the FP8 MoE dispatch and combine -- TEST INFRASTRUCTURE ONLY
(imported by tests/ only; shares no code with the CUDA path).

The recipe caches and dispatches MoE activations in FP8 ("5 Ways You can get
More Deepseek While Spending Less", cameseeing.com post) with 8 routed
experts per token ("Three Fast Methods To Study Deepseek").  Readings:
  - every (token t, slot j) pair goes to expert topk[t, j]; the rows of an
    expert are its pairs in (t, j) order -- a stable sort by expert;
  - each expert's group is padded with zero rows to a multiple of 128, and a
    zero row's 1x128 quantization is codes 0 with scale 1;
  - the combine is out[t] = sum_j w[t, j] * D[row of (t, j)], rounded to BF16
    once from the exact sum (here computed in FP64).
"""
from __future__ import annotations

import numpy as np


def moe_dispatch(q, sA, topk, G: int, M_cap: int):
    """Returns dict(q, sA, offsets, token_row, row_token) like fp8_moe_dispatch."""
    q = np.asarray(q, np.uint8)
    sA = np.asarray(sA, np.float32)
    topk = np.asarray(topk, np.int64)
    T, K = q.shape
    k = topk.shape[1]
    flat = topk.reshape(-1)
    assert np.all((flat >= 0) & (flat < G))
    counts = np.bincount(flat, minlength=G)
    padded = (counts + 127) // 128 * 128
    offsets = np.zeros(G + 1, np.int64)
    offsets[1:] = np.cumsum(padded)
    assert offsets[-1] <= M_cap
    order = np.argsort(flat, kind="stable")              # by expert, then pair order
    starts = np.zeros(G + 1, np.int64)
    starts[1:] = np.cumsum(counts)
    rank = np.arange(len(order)) - starts[flat[order]]
    token_row = np.full(T * k, -1, np.int64)
    token_row[order] = offsets[flat[order]] + rank
    row_token = np.full(M_cap, -1, np.int64)
    row_token[token_row] = np.arange(T * k) // k
    q_out = np.zeros((M_cap, K), np.uint8)
    sA_out = np.ones((K // 128, M_cap), np.float32)
    real = row_token >= 0
    q_out[real] = q[row_token[real]]
    sA_out[:, real] = sA[:, row_token[real]]
    return dict(q=q_out, sA=sA_out, offsets=offsets.astype(np.int32),
                token_row=token_row.reshape(T, k).astype(np.int32),
                row_token=row_token.astype(np.int32))


def moe_combine(D, token_row, w):
    """FP64 reference of out[t] = sum_j w[t, j] * D[token_row[t, j]] and the
    tolerance scale sum_j |w[t, j] * D[token_row[t, j]]|."""
    D = np.asarray(D, np.float64)
    token_row = np.asarray(token_row, np.int64)
    w = np.asarray(w, np.float64)
    T, k = token_row.shape
    out = np.zeros((T, D.shape[1]))
    mag = np.zeros((T, D.shape[1]))
    for j in range(k):
        r = token_row[:, j]
        ok = r >= 0
        term = w[ok, j, None] * D[r[ok]]
        out[ok] += term
        mag[ok] += np.abs(term)
    return out, mag
