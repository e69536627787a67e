"""fp8_moe_dispatch_noalloc (the dispatch with the library's fixed device
scratch) against fp8_moe_dispatch with a caller workspace.

Collected last on purpose: it must pass both alone and after every other
test has used the library on the same device.
"""
import ctypes

import numpy as np
import pytest
import torch

import fp8_fine_grained_x1_b200 as fg
from fp8_fine_grained_x1_b200 import synth

from gpu_util import dev, to_dev


def _case(T, K, k, G, seed):
    q = synth.random_e4m3_codes((T, K), seed)
    sA = synth.random_scales((K // 128, T), seed + 1)
    topk = synth.zipf_topk_routing(T, G, k, seed=seed + 2).numpy().astype(np.int32)
    return to_dev(q), to_dev(sA), to_dev(topk)


def _outputs(T, K, k, G):
    M_cap = fg.moe_capacity(T, k, G)
    d = dev()
    # filled with junk so that anything left unwritten shows
    return dict(q=torch.full((M_cap, K), 0x5A, dtype=torch.uint8, device=d),
                sA=torch.full((K // 128, M_cap), -7.0, dtype=torch.float32, device=d),
                offsets=torch.full((G + 1,), -9, dtype=torch.int32, device=d),
                token_row=torch.full((T, k), -9, dtype=torch.int32, device=d),
                row_token=torch.full((M_cap,), -9, dtype=torch.int32, device=d))


@pytest.mark.gpu
def test_noalloc_dispatch_equals_workspace_dispatch_twice_in_a_row():
    # the second case has a different expert count and chunk count, so scratch
    # left over from the first call would change its result; the third fills
    # the fixed scratch exactly (64 chunks of 1024 pairs x 1024 experts)
    cases = [(3000, 512, 8, 32, 41), (1000, 256, 4, 6, 43), (8192, 128, 8, 1024, 47)]
    assert fg.fp8_moe_dispatch_workspace_bytes(8192, 8, 1024) == 262144
    for (T, K, k, G, seed) in cases:
        q, sA, topk = _case(T, K, k, G, seed)
        ref = _outputs(T, K, k, G)
        ws = torch.empty(max(1, fg.fp8_moe_dispatch_workspace_bytes(T, k, G) // 4),
                         dtype=torch.int32, device=dev())
        fg.fp8_moe_dispatch(q, sA, topk, G, ref["q"], ref["sA"], ref["offsets"],
                            ref["token_row"], ref["row_token"], ws)
        assert fg.fp8_get_status() == fg.FP8_OK
        got = _outputs(T, K, k, G)
        fg.fp8_moe_dispatch_noalloc(q, sA, topk, G, got["q"], got["sA"], got["offsets"],
                                    got["token_row"], got["row_token"])
        assert fg.fp8_get_status() == fg.FP8_OK
        for key in ref:
            assert torch.equal(got[key].view(torch.int32) if key == "sA" else got[key],
                               ref[key].view(torch.int32) if key == "sA" else ref[key]), key


def test_noalloc_dispatch_rejects_sizes_beyond_its_scratch():
    lib = fg.load_library()
    limit = 262144
    # G = 1024 experts: 64 chunks of 1024 pairs fit, 65 do not
    assert fg.fp8_moe_dispatch_workspace_bytes(8192, 8, 1024) == limit
    assert fg.fp8_moe_dispatch_workspace_bytes(8193, 8, 1024) > limit
    nul = ctypes.c_void_p(0)
    rc = lib.fp8_moe_dispatch_noalloc(nul, nul, 8193, 128, nul, 8, 1024, nul, nul, 0,
                                      nul, nul, nul, nul)
    assert rc == fg.FP8_ERR_SHAPE
