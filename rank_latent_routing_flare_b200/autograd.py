"""torch.autograd wrappers of the FLARE / FLARE++ mixer.

Argument marshalling only: the forward calls ``flarepp_mixer_fwd`` /
``flare_mixer_fwd`` and the backward ``flarepp_mixer_bwd`` /
``flare_mixer_bwd`` of the CUDA library (which recompute the forward's
statistics from the saved inputs, so only the inputs are kept for the
backward).  Gradients come back in the dtype of their inputs (the library's
weight and seed gradients are fp32 and are rounded to the parameters' dtype
here).

With the shared-projection variant (the same tensors passed as W~_K, W~_V and
W_K, W_V) the library returns the whole gradient of the shared weights; it is
handed to autograd once, through W_K and W_V, so that autograd's own
accumulation over the two uses does not count it twice.
"""
from __future__ import annotations

import torch

from . import _binding as b


def _same(a, c) -> bool:
    return a.data_ptr() == c.data_ptr() and a.shape == c.shape and a.dtype == c.dtype


class FlareppMixer(torch.autograd.Function):
    """Y [B, H, N, D] = FLARE++ mixer of X [B, N, C] (section "FLARE++: dynamic
    token routing", eq. 7-11); differentiable in X, the four weights and Q0."""

    @staticmethod
    def forward(ctx, X, Wk, Wv, Wk_syn, Wv_syn, Q0, lengths=None, scale: float = 0.0):
        Y = b.flarepp_mixer_fwd(X, Wk, Wv, Wk_syn, Wv_syn, Q0, lengths=lengths, scale=scale)
        ctx.save_for_backward(X, Wk, Wv, Wk_syn, Wv_syn, Q0)
        ctx.lengths = lengths
        ctx.scale = scale
        return Y

    @staticmethod
    def backward(ctx, dY):
        X, Wk, Wv, Wk_syn, Wv_syn, Q0 = ctx.saved_tensors
        dY = dY.to(torch.bfloat16).contiguous()
        g = b.flarepp_mixer_bwd(X, Wk, Wv, Wk_syn, Wv_syn, Q0, dY, lengths=ctx.lengths, scale=ctx.scale)
        shared = _same(Wk, Wk_syn) and _same(Wv, Wv_syn)
        dX = g["dX"].to(X.dtype)
        dWk, dWv = g["dWk"].to(Wk.dtype), g["dWv"].to(Wv.dtype)
        dWk_syn = None if shared else g["dWk_syn"].to(Wk_syn.dtype)
        dWv_syn = None if shared else g["dWv_syn"].to(Wv_syn.dtype)
        return dX, dWk, dWv, dWk_syn, dWv_syn, g["dQ0"].to(Q0.dtype), None, None


class FlareMixer(torch.autograd.Function):
    """Y [B, H, N, D] = FLARE mixer of K, V [B, H, N, D] with learned queries
    Q [H, M, D] (section "FLARE: fixed-query latent routing", eq. 5-6);
    differentiable in K, V and Q."""

    @staticmethod
    def forward(ctx, K, V, Q, lengths=None, scale: float = 0.0):
        Y = b.flare_mixer_fwd(K, V, Q, lengths=lengths, scale=scale)
        ctx.save_for_backward(K, V, Q)
        ctx.lengths = lengths
        ctx.scale = scale
        return Y

    @staticmethod
    def backward(ctx, dY):
        K, V, Q = ctx.saved_tensors
        dY = dY.to(torch.bfloat16).contiguous()
        dK, dV, dQ = b.flare_mixer_bwd(K, V, Q, dY, lengths=ctx.lengths, scale=ctx.scale)
        return dK.to(K.dtype), dV.to(V.dtype), dQ.to(Q.dtype), None, None


def flarepp_mixer(X, Wk, Wv, Wk_syn, Wv_syn, Q0, lengths=None, scale: float = 0.0):
    """Differentiable FLARE++ mixer (see FlareppMixer)."""
    return FlareppMixer.apply(X, Wk, Wv, Wk_syn, Wv_syn, Q0, lengths, scale)


def flare_mixer(K, V, Q, lengths=None, scale: float = 0.0):
    """Differentiable FLARE mixer (see FlareMixer)."""
    return FlareMixer.apply(K, V, Q, lengths, scale)
