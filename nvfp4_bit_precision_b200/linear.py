"""NVFP4 linear layer as a PyTorch autograd op: y = x W^T with both operands in NVFP4.

The training recipe it sequences (iitak.ru, "Thinking Machines uskorila obuchenie
Inkling 2 Small 4-bitnymi chislami", sections "Details" and "How it works";
asector.ru, "Nvidia dobivaetsya uspekha s 4-bitnym formatom NVFP4", section "NVFP4
and Blackwell"):

  forward   x is quantised in 16-element blocks along the hidden dimension (RNE);
            the weight gets 16x16 2D block scales, which a transpose leaves unchanged,
            so its columnwise copy serves the backward pass; y = x_hat W_hat^T on the
            tensor cores.  The same staged pass over x also writes x's columnwise
            copy with the random Hadamard transform, kept for the weight gradient.
  backward  dY is quantised rowwise with stochastic rounding (the dgrad operand) and
            columnwise with the Hadamard transform and stochastic rounding (the wgrad
            operand); dX = dY_hat W_hat and dW = dY_hat^T x_hat.

The Hadamard signs depend on the seed alone, so the transform applied to dY and to x
along the token dimension cancels in dW.  Stochastic rounding draws fresh Philox
counters on every step through a per-layer offset.  The master weight stays in bf16;
y, dX and dW are bf16.  Every step runs in libnvfp4's kernels: this module only
sequences the calls and keeps the quantised operands between the two passes.
"""
from __future__ import annotations

import torch

from . import (NVFP4_2D16x16, NVFP4_OUT_BF16, NVFP4_SF_MMA, NVFP4_SR, gemm, quantize)

# K of every GEMM of the layer (hidden, out_features, tokens) is a whole number of
# 256-element pipeline stages.
_ALIGN = 256


def _check(x: torch.Tensor, weight: torch.Tensor) -> None:
    if not (x.is_cuda and weight.is_cuda):
        raise ValueError("nvfp4 linear: x and weight must be CUDA tensors")
    if x.dtype != torch.bfloat16 or weight.dtype != torch.bfloat16:
        raise ValueError("nvfp4 linear: x and weight must be bfloat16")
    if x.dim() != 2 or weight.dim() != 2 or x.shape[1] != weight.shape[1]:
        raise ValueError("nvfp4 linear: x [tokens, in] and weight [out, in] expected")
    t, h = x.shape
    f = weight.shape[0]
    if t % _ALIGN or h % _ALIGN or f % _ALIGN:
        raise ValueError(f"nvfp4 linear: tokens, in and out features must be multiples of "
                         f"{_ALIGN} (got {t}, {h}, {f})")


class NVFP4LinearFunction(torch.autograd.Function):
    """y = x W^T in NVFP4; see the module docstring for the recipe."""

    @staticmethod
    def forward(ctx, x, weight, seed: int, offset: int):
        _check(x, weight)
        x = x.contiguous()
        weight = weight.contiguous()
        xq = quantize(x, rowwise=True, colwise=True, rht=True, seed=seed, offset=offset,
                      sf_layout=NVFP4_SF_MMA)
        wq = quantize(weight, rowwise=True, colwise=True, scaling=NVFP4_2D16x16, seed=seed,
                      offset=offset, sf_layout=NVFP4_SF_MMA)
        y = gemm(xq["row"], wq["row"], NVFP4_OUT_BF16)
        ctx.x_col, ctx.w_col = xq["col"], wq["col"]
        ctx.seed, ctx.offset = seed, offset
        return y

    @staticmethod
    def backward(ctx, dy):
        dy = dy.to(torch.bfloat16).contiguous()
        dq = quantize(dy, rowwise=True, colwise=True, rounding=NVFP4_SR, rht=True,
                      seed=ctx.seed, offset=ctx.offset, sf_layout=NVFP4_SF_MMA)
        dx = gemm(dq["row"], ctx.w_col, NVFP4_OUT_BF16) if ctx.needs_input_grad[0] else None
        dw = gemm(dq["col"], ctx.x_col, NVFP4_OUT_BF16) if ctx.needs_input_grad[1] else None
        ctx.x_col = ctx.w_col = None
        return dx, dw, None, None


def nvfp4_linear(x: torch.Tensor, weight: torch.Tensor, seed: int = 0,
                 offset: int = 0) -> torch.Tensor:
    """y = x W^T with NVFP4 operands; x [..., in] bf16, weight [out, in] bf16."""
    lead = x.shape[:-1]
    y = NVFP4LinearFunction.apply(x.reshape(-1, x.shape[-1]), weight, seed, offset)
    return y.reshape(*lead, weight.shape[0])


class NVFP4Linear(torch.nn.Module):
    """Linear layer (no bias) whose forward and backward GEMMs run in NVFP4 with a bf16
    master weight.  Each forward call advances the stochastic-rounding offset."""

    def __init__(self, in_features: int, out_features: int, device=None, seed: int = 0,
                 init_std: float = 0.02):
        super().__init__()
        self.in_features, self.out_features = in_features, out_features
        self.weight = torch.nn.Parameter(
            torch.empty((out_features, in_features), dtype=torch.bfloat16, device=device))
        with torch.no_grad():
            self.weight.normal_(0.0, init_std)
        self.seed = seed
        self.offset = 0

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        y = nvfp4_linear(x, self.weight, self.seed, self.offset)
        self.offset += 1
        return y
