"""torch.autograd wrappers of the FLARE / FLARE++ mixer.

Argument marshalling only: the forward calls ``flarepp_mixer_fwd`` /
``flare_mixer_fwd`` and the backward ``flarepp_mixer_bwd`` /
``flare_mixer_bwd`` of the CUDA library (which recompute the forward's
statistics from the saved inputs, so only the inputs are kept for the
backward).  With ``save_state=True`` the training pair runs instead
(``*_fwd_train`` / ``*_bwd_train``): the forward keeps its projections,
latents and encoder normalisers in the backward's workspace, which autograd
holds until the backward, and the backward skips their recomputation --
less time, more memory held between the passes.  Gradients come back in the
dtype of their inputs (the library's weight and seed gradients are fp32 and
are rounded to the parameters' dtype here).

With the shared-projection variant (the same tensors passed as W~_K, W~_V and
W_K, W_V) the library returns the whole gradient of the shared weights; it is
handed to autograd once, through W_K and W_V, so that autograd's own
accumulation over the two uses does not count it twice.
"""
from __future__ import annotations

import torch

from . import _binding as b


def _take_state(ctx):
    """The training forward's workspace, handed out once: the backward that
    uses it consumes the state, so a second backward through the same graph
    (retain_graph) cannot reuse it."""
    if ctx.state is None:
        raise RuntimeError("the forward's saved state was already used by a backward; run the forward again "
                           "(or use save_state=False to backward twice through one graph)")
    return ctx.state, None


def _same(a, c) -> bool:
    return a.data_ptr() == c.data_ptr() and a.shape == c.shape and a.dtype == c.dtype


class FlareppMixer(torch.autograd.Function):
    """Y [B, H, N, D] = FLARE++ mixer of X [B, N, C] (section "FLARE++: dynamic
    token routing", eq. 7-11); differentiable in X, the four weights and Q0."""

    @staticmethod
    def forward(ctx, X, Wk, Wv, Wk_syn, Wv_syn, Q0, lengths=None, scale: float = 0.0, save_state: bool = False):
        ctx.state = None
        if save_state:
            Y, ctx.state = b.flarepp_mixer_fwd_train(X, Wk, Wv, Wk_syn, Wv_syn, Q0, lengths=lengths, scale=scale)
        else:
            Y = b.flarepp_mixer_fwd(X, Wk, Wv, Wk_syn, Wv_syn, Q0, lengths=lengths, scale=scale)
        ctx.save_state = save_state
        ctx.save_for_backward(X, Wk, Wv, Wk_syn, Wv_syn, Q0)
        ctx.lengths = lengths
        ctx.scale = scale
        return Y

    @staticmethod
    def backward(ctx, dY):
        X, Wk, Wv, Wk_syn, Wv_syn, Q0 = ctx.saved_tensors
        dY = dY.to(torch.bfloat16).contiguous()
        if ctx.save_state:
            ws, ctx.state = _take_state(ctx)
            g = b.flarepp_mixer_bwd_train(X, Wk, Wv, Wk_syn, Wv_syn, Q0, dY, ws, lengths=ctx.lengths,
                                          scale=ctx.scale)
        else:
            g = b.flarepp_mixer_bwd(X, Wk, Wv, Wk_syn, Wv_syn, Q0, dY, lengths=ctx.lengths, scale=ctx.scale)
        shared = _same(Wk, Wk_syn) and _same(Wv, Wv_syn)
        dX = g["dX"].to(X.dtype)
        dWk, dWv = g["dWk"].to(Wk.dtype), g["dWv"].to(Wv.dtype)
        dWk_syn = None if shared else g["dWk_syn"].to(Wk_syn.dtype)
        dWv_syn = None if shared else g["dWv_syn"].to(Wv_syn.dtype)
        return dX, dWk, dWv, dWk_syn, dWv_syn, g["dQ0"].to(Q0.dtype), None, None, None


class FlareMixer(torch.autograd.Function):
    """Y [B, H, N, D] = FLARE mixer of K, V [B, H, N, D] with learned queries
    Q [H, M, D] (section "FLARE: fixed-query latent routing", eq. 5-6);
    differentiable in K, V and Q."""

    @staticmethod
    def forward(ctx, K, V, Q, lengths=None, scale: float = 0.0, save_state: bool = False):
        ctx.state = None
        if save_state:
            Y, ctx.state = b.flare_mixer_fwd_train(K, V, Q, lengths=lengths, scale=scale)
        else:
            Y = b.flare_mixer_fwd(K, V, Q, lengths=lengths, scale=scale)
        ctx.save_state = save_state
        ctx.save_for_backward(K, V, Q)
        ctx.lengths = lengths
        ctx.scale = scale
        return Y

    @staticmethod
    def backward(ctx, dY):
        K, V, Q = ctx.saved_tensors
        dY = dY.to(torch.bfloat16).contiguous()
        if ctx.save_state:
            ws, ctx.state = _take_state(ctx)
            dK, dV, dQ = b.flare_mixer_bwd_train(K, V, Q, dY, ws, lengths=ctx.lengths, scale=ctx.scale)
        else:
            dK, dV, dQ = b.flare_mixer_bwd(K, V, Q, dY, lengths=ctx.lengths, scale=ctx.scale)
        return dK.to(K.dtype), dV.to(V.dtype), dQ.to(Q.dtype), None, None, None


def flarepp_mixer(X, Wk, Wv, Wk_syn, Wv_syn, Q0, lengths=None, scale: float = 0.0, save_state: bool = False):
    """Differentiable FLARE++ mixer (see FlareppMixer)."""
    return FlareppMixer.apply(X, Wk, Wv, Wk_syn, Wv_syn, Q0, lengths, scale, save_state)


def flare_mixer(K, V, Q, lengths=None, scale: float = 0.0, save_state: bool = False):
    """Differentiable FLARE mixer (see FlareMixer)."""
    return FlareMixer.apply(K, V, Q, lengths, scale, save_state)
