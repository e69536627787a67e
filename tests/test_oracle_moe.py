"""Pins of the MoE dispatch / combine oracle against brute-force loops and
against the input generator's independently built expert layout."""
import numpy as np
import torch

from fp8_fine_grained_x1_b200 import synth
from oracle import moe as omoe


def _brute_dispatch(q, sA, topk, G, M_cap):
    T, K = q.shape
    k = topk.shape[1]
    rows = {e: [] for e in range(G)}
    for t in range(T):
        for j in range(k):
            rows[int(topk[t, j])].append((t, j))
    offsets = [0]
    for e in range(G):
        offsets.append(offsets[-1] + (len(rows[e]) + 127) // 128 * 128)
    token_row = -np.ones((T, k), np.int64)
    q_out = np.zeros((M_cap, K), np.uint8)
    s_out = np.ones((K // 128, M_cap), np.float32)
    for e in range(G):
        for i, (t, j) in enumerate(rows[e]):
            r = offsets[e] + i
            token_row[t, j] = r
            q_out[r] = q[t]
            s_out[:, r] = sA[:, t]
    return offsets, token_row, q_out, s_out


def test_dispatch_equals_brute_force_loops():
    rng = np.random.default_rng(0)
    T, K, k, G = 37, 256, 3, 5
    q = rng.integers(0, 256, (T, K)).astype(np.uint8)
    sA = rng.uniform(0.1, 2, (K // 128, T)).astype(np.float32)
    topk = rng.integers(0, G - 1, (T, k)).astype(np.int32)     # expert G-1 stays empty
    M_cap = 1024
    got = omoe.moe_dispatch(q, sA, topk, G, M_cap)
    offsets, token_row, q_out, s_out = _brute_dispatch(q, sA, topk, G, M_cap)
    assert got["offsets"].tolist() == offsets
    assert np.array_equal(got["token_row"], token_row)
    assert np.array_equal(got["q"], q_out) and np.array_equal(got["sA"], s_out)
    rt = got["row_token"]
    for t in range(T):
        for j in range(k):
            assert rt[token_row[t, j]] == t


def test_dispatch_layout_matches_input_generator():
    topk = synth.zipf_topk_routing(2000, 32, 8, seed=3)
    lay = synth.moe_layout(topk, 32)
    T = 2000
    q = np.zeros((T, 128), np.uint8)
    sA = np.ones((1, T), np.float32)
    got = omoe.moe_dispatch(q, sA, topk.numpy().astype(np.int32), 32, lay.m_total + 128)
    assert np.array_equal(got["offsets"], lay.offsets.numpy())
    assert np.array_equal(got["row_token"][:lay.m_total], lay.row_token.numpy())
    assert np.all(got["row_token"][lay.m_total:] == -1)


def test_combine_reduces_to_a_gather_and_is_linear():
    rng = np.random.default_rng(1)
    D = rng.standard_normal((64, 16))
    rows = rng.permutation(64)[:40].reshape(20, 2)
    out, mag = omoe.moe_combine(D, rows[:, :1], np.ones((20, 1)))
    assert np.array_equal(out, D[rows[:, 0]]) and np.array_equal(mag, np.abs(D[rows[:, 0]]))
    w = rng.uniform(-1, 1, (20, 2))
    out2, _ = omoe.moe_combine(D, rows, w)
    assert np.allclose(out2, w[:, :1] * D[rows[:, 0]] + w[:, 1:] * D[rows[:, 1]], rtol=0, atol=1e-15)
    rows_m = rows.copy()
    rows_m[3, 1] = -1                                   # a dropped pair contributes nothing
    out3, _ = omoe.moe_combine(D, rows_m, w)
    assert np.allclose(out3[3], w[3, 0] * D[rows[3, 0]], rtol=0, atol=1e-15)
