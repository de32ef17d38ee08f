"""Autograd form of the layer for training.

The Sparse-BitNet Guide's module ("End-to-End Implementation: Building a
Sparse-BitLinear Layer") keeps fp32 latent weights, rebuilds the N:M mask and
the ternary weights from them on every forward, and trains them through the
straight-through estimator ("Training Stability & The Straight-Through
Estimator").  Here every step of that runs in the library's kernels:

    forward   sbl_prepare_weights (mask, scale, ternarise, pack; every call,
              so the mask follows the latent weights), sbl_quant_act (the
              int8 activations kept for the backward) and sbl_linear_q on
              those (sbl_linear, which quantises x itself, when K % 64 != 0);
    backward  sbl_linear_backward (dX = dY . (scale * W_t) to the activations,
              dW = dY^T . (x_q / s_t) to every latent weight).

The guide's module normalises x with an RMSNorm first; that normalisation and
its gradient belong to the caller here (x is the layer's input as quantised).
Argument marshalling only: no arithmetic of the layer runs in PyTorch.
"""
from __future__ import annotations

import math

import torch

from . import _lib, api


class SparseBitLinearFunction(torch.autograd.Function):
    """y = dequant(int8(x) . ternary_NM(W)^T) with straight-through gradients.

    x: bf16 [T, K] (contiguous), weight: fp32 [O, K] latent weights; returns fp32 [T, O]."""

    @staticmethod
    def forward(ctx, x, weight, n, m, dw_ternary, check_finite=True):
        w = api.sbl_prepare_weights(weight.detach(), n, m)
        xq, s = api.sbl_quant_act(x)
        # contract the x_q kept for the backward (x is quantised once); the
        # contraction on quantised activations needs K % 64 == 0
        y = api.sbl_linear_q(xq, s, w) if weight.shape[1] % 64 == 0 else api.sbl_linear(x, w)
        if check_finite:
            # The kernels do not pass NaN or Inf through: a non-finite latent
            # weight or activation only sets the device status word while the
            # outputs stay finite, so a diverging run would keep training on
            # garbage.  Read the word (this waits for the stream) and stop.
            status = api.sbl_device_status()
            if status == _lib.SBL_ERR_NONFINITE:
                raise FloatingPointError("SparseBitLinear: non-finite latent weights or activations")
            if status != _lib.SBL_OK:
                raise _lib.SblError(status, "SparseBitLinear forward")
        ctx.save_for_backward(xq, s, w.packed, w.row_scale)
        ctx.layer = (n, m, weight.shape[1], x.dtype, bool(dw_ternary))
        return y

    @staticmethod
    def backward(ctx, dy):
        xq, s, packed, row_scale = ctx.saved_tensors
        n, m, K, x_dtype, dw_ternary = ctx.layer
        need_dx, need_dw = ctx.needs_input_grad[0], ctx.needs_input_grad[1]
        if not (need_dx or need_dw):
            return None, None, None, None, None, None
        w = api.PreparedWeights(packed, row_scale, n, m, K)
        dX, dW = api.sbl_linear_backward(dy.float().contiguous(), xq, s, w, need_dx=need_dx, need_dw=need_dw,
                                         dw_ternary=dw_ternary)
        return (dX.to(x_dtype) if need_dx else None), dW, None, None, None, None


class SparseBitLinear(torch.nn.Module):
    """The guide's Sparse-BitLinear layer without its RMSNorm: fp32 latent
    weights [out_features, in_features], N:M-sparse ternary in the forward.

    ``dw_ternary`` selects the guide module's weight gradient (taken at the
    ternary matrix, i.e. scaled by the row scale) instead of the
    straight-through gradient of the dequantised weight.  Inputs of any
    leading shape with last dimension in_features are cast to bf16 (the
    library's activation type); the output is fp32.

    With ``check_finite`` (the default) every forward reads the library's
    device status word and raises FloatingPointError when a latent weight or
    an activation was NaN or Inf (the kernels flag such values rather than
    propagate them).  Reading it waits for the stream; ``check_finite=False``
    skips the wait and the check."""

    def __init__(self, in_features: int, out_features: int, n: int = 2, m: int = 4, dw_ternary: bool = False,
                 device=None, check_finite: bool = True):
        super().__init__()
        self.in_features, self.out_features = in_features, out_features
        self.n, self.m, self.dw_ternary, self.check_finite = n, m, dw_ternary, check_finite
        self.weight = torch.nn.Parameter(torch.empty((out_features, in_features), dtype=torch.float32,
                                                     device=device))
        self.reset_parameters()

    def reset_parameters(self) -> None:
        # the same initialisation as the guide's module (torch's Linear default)
        torch.nn.init.kaiming_uniform_(self.weight, a=math.sqrt(5))

    def forward(self, x: torch.Tensor) -> torch.Tensor:
        lead = x.shape[:-1]
        x2 = x.reshape(-1, self.in_features).to(torch.bfloat16).contiguous()
        y = SparseBitLinearFunction.apply(x2, self.weight, self.n, self.m, self.dw_ternary, self.check_finite)
        return y.reshape(*lead, self.out_features)

    def extra_repr(self) -> str:
        return f"in_features={self.in_features}, out_features={self.out_features}, {self.n}:{self.m}"
