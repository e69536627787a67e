"""Seeded synthetic inputs shaped like the workloads of the fine-grained FP8
Linear (dense-MLP Fprop, Dgrad, Wgrad and an MoE expert layer).

This module only draws random numbers and arranges rows: it holds none of the
method's arithmetic (no max-abs, no scaling, no FP8 cast, no GEMM).  Both the
CUDA path and the CPU oracle consume what it returns, so it is the single
shared dependency of the two.

All draws are made on the CPU with ``torch.Generator().manual_seed(seed)`` in
FP32 and then cast (round to nearest even) to BF16 where the workload says
BF16.  Shapes follow the workloads the pages describe: hidden size 7168,
MoE expert intermediate size 2048 ("each MoE layer consists of 1 shared
expert and 256 routed experts ... intermediate hidden dimension of each
expert is 2048"; "8 experts activated for each token").
"""
from __future__ import annotations

import dataclasses

import torch

HIDDEN = 7168
EXPERT_HIDDEN = 2048


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def normal(shape, std: float, seed: int, dtype=torch.bfloat16) -> torch.Tensor:
    """N(0, std^2) draws (std is the standard deviation), cast to `dtype`."""
    x = torch.randn(*shape, generator=_gen(seed), dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def outlier_channels(n_channels: int, seed: int, frac: float = 0.01) -> torch.Tensor:
    """round(frac * n_channels) distinct channel indices (72 of 7168)."""
    k = int(round(frac * n_channels))
    return torch.randperm(n_channels, generator=_gen(seed))[:k].sort().values


def activations(tokens: int, channels: int = HIDDEN, seed: int = 0, outlier_seed: int = 2,
                outlier_gain: float = 50.0, dtype=torch.bfloat16) -> torch.Tensor:
    """X ~ N(0, 1) with 1% of the channels multiplied by `outlier_gain`."""
    x = torch.randn(tokens, channels, generator=_gen(seed), dtype=torch.float32)
    if outlier_gain != 1.0:
        ch = outlier_channels(channels, outlier_seed)
        x[:, ch] *= outlier_gain
    return x.to(dtype)


def bf16_bits(x: torch.Tensor):
    """BF16 tensor -> numpy uint16 bit patterns (the oracle's input format)."""
    assert x.dtype == torch.bfloat16
    return x.contiguous().view(torch.int16).numpy().view("uint16")


# --------------------------------------------------------------------------
# MoE routing and expert-contiguous row layout
# --------------------------------------------------------------------------

@dataclasses.dataclass
class MoeLayout:
    """Rows of the grouped GEMM operand, expert by expert.

    row_token[r] is the token whose activation row sits at row r, or -1 for a
    zero padding row; offsets[e] .. offsets[e+1] are expert e's rows (each
    group padded with zero rows to a multiple of 128)."""
    row_token: torch.Tensor      # int64 [M_total]
    offsets: torch.Tensor        # int32 [G + 1]
    counts: torch.Tensor         # int64 [G], real rows per expert
    topk: torch.Tensor           # int64 [tokens, k], the experts of each token

    @property
    def m_total(self) -> int:
        return int(self.offsets[-1])


def zipf_topk_routing(tokens: int, experts: int = 32, k: int = 8, s: float = 1.1,
                      seed: int = 3) -> torch.Tensor:
    """k distinct experts per token from a truncated Zipf(s) law p_e ~ (e+1)^-s,
    drawn without replacement by Gumbel-top-k.  Returns int64 [tokens, k]."""
    logp = -s * torch.log(torch.arange(1, experts + 1, dtype=torch.float64))
    u = torch.rand(tokens, experts, generator=_gen(seed), dtype=torch.float64)
    u = u.clamp_(min=1e-300)
    gumbel = -torch.log(-torch.log(u))
    return torch.topk(logp.unsqueeze(0) + gumbel, k, dim=1).indices


def moe_layout(topk: torch.Tensor, experts: int, pad_to: int = 128) -> MoeLayout:
    """Expert-contiguous order of (token, expert) pairs, tokens ascending within
    an expert, each expert's group padded with -1 rows to a multiple of pad_to."""
    tokens, k = topk.shape
    flat_e = topk.reshape(-1)
    flat_t = torch.arange(tokens).repeat_interleave(k)
    counts = torch.bincount(flat_e, minlength=experts)
    padded = (counts + pad_to - 1) // pad_to * pad_to
    offsets = torch.zeros(experts + 1, dtype=torch.int64)
    offsets[1:] = torch.cumsum(padded, 0)
    order = torch.argsort(flat_e * tokens + flat_t)        # by expert, then token
    row_token = torch.full((int(offsets[-1]),), -1, dtype=torch.int64)
    sorted_e = flat_e[order]
    starts = torch.zeros(experts + 1, dtype=torch.int64)
    starts[1:] = torch.cumsum(counts, 0)
    rank_in_e = torch.arange(len(order)) - starts[sorted_e]
    row_token[offsets[sorted_e] + rank_in_e] = flat_t[order]
    return MoeLayout(row_token=row_token, offsets=offsets.to(torch.int32), counts=counts,
                     topk=topk)


def gather_rows(x: torch.Tensor, row_token: torch.Tensor) -> torch.Tensor:
    """Rows x[row_token[r]] (zero rows where row_token[r] < 0), on x's device."""
    idx = row_token.to(x.device)
    out = x.index_select(0, idx.clamp(min=0))
    out[idx < 0] = 0
    return out


# --------------------------------------------------------------------------
# The workloads
# --------------------------------------------------------------------------

WORKLOADS = ("pr1", "fprop", "dgrad", "wgrad", "moe")


def pr1():
    """Tiny Fprop: X[128,512] fp32 N(0,1) seed 0, W[256,512] fp32 N(0,0.02) seed 1."""
    return dict(x=normal((128, 512), 1.0, 0, torch.float32),
                w=normal((256, 512), 0.02, 1, torch.float32))


def fprop(M: int = 4096, N: int = 18432, K: int = HIDDEN):
    """Dense-MLP Fprop: X[M,K] N(0,1) with 1% outlier channels x50, W[N,K] N(0,0.006)."""
    return dict(x=activations(M, K, seed=0, outlier_seed=2), w=normal((N, K), 0.006, 1))


def dgrad(M: int = 4096, N_out: int = HIDDEN, K_in: int = EXPERT_HIDDEN):
    """Dgrad: dY[M,N_out] N(0,1e-3) seed 4; W[N_out,K_in] N(0,0.02) seed 1
    (the forward weight, read transposed by dX = dY . W)."""
    return dict(dy=normal((M, N_out), 1e-3, 4), w=normal((N_out, K_in), 0.02, 1))


def wgrad(T: int = 8192, C_in: int = HIDDEN, C_out: int = EXPERT_HIDDEN):
    """Wgrad: X[T,C_in] as in Fprop, dY[T,C_out] N(0,1e-3) seed 4;
    dW[C_out, C_in] = dY^T . X reduces over the T tokens."""
    return dict(x=activations(T, C_in, seed=0, outlier_seed=2),
                dy=normal((T, C_out), 1e-3, 4))


def moe(tokens: int = 16384, experts: int = 32, k: int = 8, N: int = EXPERT_HIDDEN,
        K: int = HIDDEN):
    """MoE grouped Fprop: X[tokens,K] (+outliers), top-k Zipf(1.1) routing,
    W_e[experts, N, K] N(0,0.006) seed 1."""
    x = activations(tokens, K, seed=0, outlier_seed=2)
    layout = moe_layout(zipf_topk_routing(tokens, experts, k, seed=3), experts)
    w = normal((experts, N, K), 0.006, 1)
    return dict(x=x, w=w, layout=layout)


# --------------------------------------------------------------------------
# Raw operands for GEMM-only cases
# --------------------------------------------------------------------------

def random_e4m3_codes(shape, seed: int):
    """Uniformly drawn finite E4M3FN byte codes (every byte except 0x7F, 0xFF)."""
    import numpy as np
    rng = np.random.default_rng(seed)
    finite = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    return finite[rng.integers(0, len(finite), shape)]


def random_scales(shape, seed: int, lo: float = -12.0, hi: float = 4.0):
    """FP32 values 2^u with u ~ U(lo, hi)."""
    import numpy as np
    rng = np.random.default_rng(seed)
    return np.exp2(rng.uniform(lo, hi, shape)).astype(np.float32)
