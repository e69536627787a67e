"""The fine-grained FP8 Linear's three GEMM passes and the MoE expert pass, as
ready-to-run steps over device-resident inputs.

Each step owns its output buffers (allocated once with torch) and, when
called, issues only library calls: on the caller's stream (torch's current
one by default), and for one of its two quantizers on a side stream forked
from it and joined back before the GEMM:

  FpropStep    X[M,K] --1x128--> (qX, sX);  W[N,K] --128x128--> (qW, sW);
               Y[M,N] = qX . qW^T                      (BF16 or FP32 out)
  DgradStep    dY[M,N_out] --1x128--> ;  W[N_out,K_in] --128x128--> (stored
               orientation); dX[M,K_in] = dY . W, W read MN-major
  WgradStep    X[T,C_in], dY[T,C_out] --128x1--> token-contiguous codes with
               per-channel scales; dW[C_out,C_in] = dY^T . X, FP32 out
  WgradCachedStep  as WgradStep, with X taken from its cached 1x128 FP8
               form and requantized into 128x1 groups
  MoeStep      tokens X[T,K] --1x128, written straight to their expert-
               contiguous, 128-padded FP8 rows-->; W[G,N,K] --128x128-->;
               grouped GEMM (or, gather=True, quantized once and gathered by
               the GEMM)

("5 Ways You can get More Deepseek While Spending Less", Figure 6: Fprop,
Dgrad and Wgrad all run in FP8; why-be.co.kr / cameseeing.com posts and
"Three Fast Methods To Study Deepseek", Figure 7 (a): 1x128 / 128x128
grouping; gnrental.net post: BF16 or FP32 GEMM outputs.)

`kernel_calls` on each step counts the kernels one call launches.

With scale_mode=SCALE_POW2 the dense steps accept tensor_core_scaling=True:
the GEMM then applies the power-of-two scales inside the tensor cores
(fp8_blockscaled_gemm_pow2, UE8M0 block scaling) instead of promoting every
128-K partial in software.
"""
from __future__ import annotations

import torch

from . import (B_KMAJOR, B_MNMAJOR, SCALE_FP32, SCALE_POW2, fp8_blockscaled_gemm,
               fp8_blockscaled_gemm_pow2, fp8_grouped_gemm, fp8_grouped_gemm_gather,
               fp8_grouped_gemm_pow2,
               fp8_moe_combine, fp8_moe_dispatch_workspace_bytes, fp8_moe_quant_dispatch,
               fp8_moe_route, fp8_quant_act_128x1, fp8_quant_act_1x128, fp8_quant_w_128x128,
               fp8_requant_1x128_to_128x1, moe_capacity)


def _empty(shape, dtype, device):
    return torch.empty(shape, dtype=dtype, device=device)


class _Fork:
    """Each step's two quantizers share no input, so one of them runs on a
    side stream forked from the caller's stream and joined back before the
    GEMM: the tail of one overlaps the other, and short launches overlap
    each other's start-up."""

    def __init__(self, device):
        self.side = torch.cuda.Stream(device=device)
        self.fork, self.join = torch.cuda.Event(), torch.cuda.Event()
        self.device = device

    def begin(self, stream):
        cur = stream if stream is not None else torch.cuda.current_stream(self.device)
        self.fork.record(cur)
        self.side.wait_event(self.fork)
        return cur, self.side

    def end(self, cur):
        self.join.record(self.side)
        cur.wait_event(self.join)


def _gemm_fn(scale_mode, tensor_core_scaling):
    if not tensor_core_scaling:
        return fp8_blockscaled_gemm
    if scale_mode != SCALE_POW2:
        raise ValueError("tensor-core scaling needs power-of-two scales (SCALE_POW2)")
    return fp8_blockscaled_gemm_pow2


class FpropStep:
    kernel_calls = 3

    def __init__(self, x, w, out_dtype=torch.bfloat16, scale_mode=SCALE_FP32,
                 tensor_core_scaling=False):
        M, K = x.shape
        N = w.shape[0]
        d = x.device
        self.x, self.w, self.mode = x, w, scale_mode
        self._gemm = _gemm_fn(scale_mode, tensor_core_scaling)
        self.qx, self.sx = _empty((M, K), torch.uint8, d), _empty((K // 128, M), torch.float32, d)
        self.qw, self.sw = _empty((N, K), torch.uint8, d), _empty((N // 128, K // 128), torch.float32, d)
        self.y = _empty((M, N), out_dtype, d)
        self.flops = 2 * M * N * K
        self.inputs, self.output = [x, w], self.y
        self._fork = _Fork(d)

    def quantize(self, stream=None):
        cur, side = self._fork.begin(stream)
        fp8_quant_w_128x128(self.w, self.qw, self.sw, self.mode, side)
        fp8_quant_act_1x128(self.x, self.qx, self.sx, self.mode, cur)
        self._fork.end(cur)

    def gemm(self, stream=None):
        self._gemm(self.qx, self.sx, self.qw, self.sw, self.y, B_KMAJOR, 128, stream)

    def __call__(self, stream=None):
        self.quantize(stream)
        self.gemm(stream)
        return self.y


class DgradStep:
    kernel_calls = 3

    def __init__(self, dy, w, out_dtype=torch.bfloat16, scale_mode=SCALE_FP32,
                 tensor_core_scaling=False):
        M, N_out = dy.shape
        N_out2, K_in = w.shape
        assert N_out == N_out2
        d = dy.device
        self.dy, self.w, self.mode = dy, w, scale_mode
        self._gemm = _gemm_fn(scale_mode, tensor_core_scaling)
        self.qdy = _empty((M, N_out), torch.uint8, d)
        self.sdy = _empty((N_out // 128, M), torch.float32, d)
        self.qw = _empty((N_out, K_in), torch.uint8, d)
        self.sw = _empty((N_out // 128, K_in // 128), torch.float32, d)
        self.dx = _empty((M, K_in), out_dtype, d)
        self.flops = 2 * M * K_in * N_out
        self.inputs, self.output = [dy, w], self.dx
        self._fork = _Fork(d)

    def quantize(self, stream=None):
        cur, side = self._fork.begin(stream)
        fp8_quant_w_128x128(self.w, self.qw, self.sw, self.mode, side)
        fp8_quant_act_1x128(self.dy, self.qdy, self.sdy, self.mode, cur)
        self._fork.end(cur)

    def gemm(self, stream=None):
        # B = W stored [K = N_out][N = K_in]: MN-major; its block scales
        # sW[N_out/128][K_in/128] are [K/128][N/128] in GEMM terms.
        self._gemm(self.qdy, self.sdy, self.qw, self.sw, self.dx, B_MNMAJOR, 128, stream)

    def __call__(self, stream=None):
        self.quantize(stream)
        self.gemm(stream)
        return self.dx


class WgradStep:
    kernel_calls = 3

    def __init__(self, x, dy, scale_mode=SCALE_FP32, tensor_core_scaling=False):
        T, C_in = x.shape
        T2, C_out = dy.shape
        assert T == T2
        d = x.device
        self.x, self.dy, self.mode = x, dy, scale_mode
        self._gemm = _gemm_fn(scale_mode, tensor_core_scaling)
        self.qxT = _empty((C_in, T), torch.uint8, d)
        self.sx = _empty((T // 128, C_in), torch.float32, d)
        self.qdyT = _empty((C_out, T), torch.uint8, d)
        self.sdy = _empty((T // 128, C_out), torch.float32, d)
        self.dw = _empty((C_out, C_in), torch.float32, d)
        self.flops = 2 * C_out * C_in * T
        self.inputs, self.output = [x, dy], self.dw
        self._fork = _Fork(d)

    def quantize(self, stream=None):
        cur, side = self._fork.begin(stream)
        fp8_quant_act_128x1(self.dy, self.qdyT, self.sdy, self.mode, side)
        fp8_quant_act_128x1(self.x, self.qxT, self.sx, self.mode, cur)
        self._fork.end(cur)

    def gemm(self, stream=None):
        self._gemm(self.qdyT, self.sdy, self.qxT, self.sx, self.dw, B_KMAJOR, 1, stream)

    def __call__(self, stream=None):
        self.quantize(stream)
        self.gemm(stream)
        return self.dw


class WgradCachedStep:
    """Wgrad with X kept from the forward pass as 1x128 FP8 (codes qx [T, C_in],
    scales sx [C_in/128, T]): the cache is requantized into 128x1 groups along
    tokens instead of quantizing a BF16 copy of X; dY is quantized 128x1."""
    kernel_calls = 3

    def __init__(self, qx, sx, dy, scale_mode=SCALE_FP32):
        T, C_in = qx.shape
        T2, C_out = dy.shape
        assert T == T2
        d = qx.device
        self.qx, self.sx, self.dy, self.mode = qx, sx, dy, scale_mode
        self.qxT = _empty((C_in, T), torch.uint8, d)
        self.sxT = _empty((T // 128, C_in), torch.float32, d)
        self.qdyT = _empty((C_out, T), torch.uint8, d)
        self.sdy = _empty((T // 128, C_out), torch.float32, d)
        self.dw = _empty((C_out, C_in), torch.float32, d)
        self.flops = 2 * C_out * C_in * T
        self.inputs, self.output = [qx, sx, dy], self.dw
        self._fork = _Fork(d)

    def quantize(self, stream=None):
        cur, side = self._fork.begin(stream)
        fp8_quant_act_128x1(self.dy, self.qdyT, self.sdy, self.mode, side)
        fp8_requant_1x128_to_128x1(self.qx, self.sx, self.qxT, self.sxT, self.mode, cur)
        self._fork.end(cur)

    def gemm(self, stream=None):
        fp8_blockscaled_gemm(self.qdyT, self.sdy, self.qxT, self.sxT, self.dw, B_KMAJOR, 1, stream)

    def __call__(self, stream=None):
        self.quantize(stream)
        self.gemm(stream)
        return self.dw


class MoeStep:
    """MoE expert layer forward.  Tokens X[T,K] are quantized 1x128 straight
    into their expert-contiguous, 128-padded rows (fp8_moe_quant_dispatch),
    W[G,N,K] is quantized 128x128, and the grouped GEMM reads A in place.
    With gather=True the tokens are instead quantized once in token order,
    routed without moving rows (fp8_moe_route), and the grouped GEMM reads
    each row's token codes through TMA gathers (fp8_grouped_gemm_gather): the
    dispatched copy (k rows per token) is never written, at the price of a
    slower GEMM (the gathers issue 32 TMA operations per K-block where a
    tiled load issues one).  `combine(weights)` adds the weighted return to
    token order."""

    def __init__(self, x, topk, w, out_dtype=torch.bfloat16, scale_mode=SCALE_FP32,
                 tensor_core_scaling=False, gather=False):
        T, K = x.shape
        G, N, K2 = w.shape
        assert K == K2
        if tensor_core_scaling and scale_mode != SCALE_POW2:
            raise ValueError("tensor-core scaling needs power-of-two scales (SCALE_POW2)")
        if tensor_core_scaling and gather:
            raise ValueError("the tensor-core-scaled grouped GEMM reads dispatched rows only")
        self.gather = gather
        self._gemm = fp8_grouped_gemm_pow2 if tensor_core_scaling else fp8_grouped_gemm
        # gather: routing (count, scan, rank), token quantizer, weight quantizer
        # (side stream), gathered grouped GEMM; else routing, fused quantizer,
        # padding rows, weight quantizer, grouped GEMM (+1 memset either way)
        self.kernel_calls = 6 if self.gather else 7
        k = topk.shape[1]
        d = x.device
        self.x, self.topk, self.w, self.mode, self.G = x, topk, w, scale_mode, G
        self.M_cap = moe_capacity(T, k, G)
        if self.gather:
            self.qx = _empty((T, K), torch.uint8, d)
            self.sx = _empty((K // 128, T), torch.float32, d)
        else:
            self.qa = _empty((self.M_cap, K), torch.uint8, d)
            self.sa = _empty((K // 128, self.M_cap), torch.float32, d)
        self.offsets = _empty((G + 1,), torch.int32, d)
        self.token_row = _empty((T, k), torch.int32, d)
        self.row_token = _empty((self.M_cap,), torch.int32, d)
        self.ws = _empty((max(1, fp8_moe_dispatch_workspace_bytes(T, k, G) // 4),), torch.int32, d)
        self.qw = _empty((G, N, K), torch.uint8, d)
        self.sw = _empty((G, N // 128, K // 128), torch.float32, d)
        self.y = _empty((self.M_cap, N), out_dtype, d)
        self.out = None
        self.inputs, self.output = [x, w, topk], self.y
        # the weight quantizer on the side stream: the short routing kernels
        # and the token path overlap it
        self._fork = _Fork(d)

    def quantize(self, stream=None):
        cur, side = self._fork.begin(stream)
        G, N, K = self.w.shape
        fp8_quant_w_128x128(self.w.view(G * N, K), self.qw.view(G * N, K),
                            self.sw.view(G * N // 128, K // 128), self.mode, side)
        if self.gather:
            fp8_moe_route(self.topk, self.G, self.offsets, self.token_row, self.row_token, self.ws,
                          cur)
            fp8_quant_act_1x128(self.x, self.qx, self.sx, self.mode, cur)
        else:
            fp8_moe_quant_dispatch(self.x, self.topk, self.G, self.qa, self.sa, self.offsets,
                                   self.token_row, self.row_token, self.ws, self.mode, cur)
        self._fork.end(cur)

    def gemm(self, stream=None):
        if self.gather:
            fp8_grouped_gemm_gather(self.qx, self.sx, self.row_token, self.qw, self.sw,
                                    self.offsets, self.y, stream)
        else:
            self._gemm(self.qa, self.sa, self.qw, self.sw, self.offsets, self.y, stream)

    def combine(self, weights, stream=None):
        T = self.x.shape[0]
        if self.out is None:
            self.out = _empty((T, self.y.shape[1]), torch.bfloat16, self.x.device)
        fp8_moe_combine(self.y, self.token_row, weights, self.out, stream)
        return self.out

    def __call__(self, stream=None):
        self.quantize(stream)
        self.gemm(stream)
        return self.y
