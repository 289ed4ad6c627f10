"""Pins of the fp64 backward oracle (gradients of the FLARE / FLARE++ mixer)
against facts fixed independently of its code.

The pages name the paper's backward equations (eq. 13-40) without printing
them; every step of the mixer is one SDPA call (FLARE++ paper, arXiv
2608.11519, section "FLARE++: dynamic token routing", eq. 8, 10, 11), so the
gradients are pinned by:
  - central finite differences of the forward oracle (directional
    derivatives of the scalar loss <dY, Y> in random directions);
  - torch float64 autograd through a chain of
    ``scaled_dot_product_attention`` calls (a library routine);
  - shift invariances of the softmax: adding one vector to every key leaves
    each encoder row unchanged (so the encoder's key gradients sum to zero),
    adding one vector to every latent query leaves each decoder row unchanged
    (so the decoder's query gradients sum to zero);
  - sum rules of row-stochastic maps (sum_n dV_n = sum_m dZ_m and
    sum_m dZ_m = sum over valid n of dY_n), a single latent (M = 1), and
    masked tokens (no gradient; the rest equals the truncated problem).
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F


def rel(a, b):
    a, b = np.asarray(a), np.asarray(b)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def rand_problem(rng, B=2, N=41, C=32, H=2, M=5, wscale=2.0):
    D = C // H
    X = rng.standard_normal((B, N, C))
    Ws = [rng.standard_normal((C, C)) * wscale / math.sqrt(C) for _ in range(4)]
    Q0 = rng.standard_normal((H, M, D))
    dY = rng.standard_normal((B, H, N, D))
    return X, Ws, Q0, dY


# --------------------------------------------------------------------------
# library routine: torch float64 autograd through the SDPA chain
# --------------------------------------------------------------------------

def torch_flarepp_grads(X, Ws, Q0, dY, H, lengths, scale):
    B, N, C = X.shape
    D = C // H
    Xt = torch.tensor(X, requires_grad=True)
    Wt = [torch.tensor(W, requires_grad=True) for W in Ws]
    Q0t = torch.tensor(Q0, requires_grad=True)

    def heads(W):
        return (Xt @ W).view(B, N, H, D).transpose(1, 2)

    Wk, Wv, Wks, Wvs = Wt
    if lengths is None:
        mask, valid = None, torch.ones(B, N, dtype=torch.bool)
    else:
        valid = torch.arange(N)[None, :] < torch.as_tensor(lengths)[:, None]
        mask = valid[:, None, None, :]
    Qx = F.scaled_dot_product_attention(Q0t[None].expand(B, -1, -1, -1), heads(Wks), heads(Wvs),
                                        attn_mask=mask, scale=scale)
    K, V = heads(Wk), heads(Wv)
    Z = F.scaled_dot_product_attention(Qx, K, V, attn_mask=mask, scale=scale)
    Y = F.scaled_dot_product_attention(K, Qx, Z, scale=scale) * valid[:, None, :, None]
    (Y * torch.from_numpy(dY)).sum().backward()
    return {"dX": Xt.grad.numpy(), "dWk": Wk.grad.numpy(), "dWv": Wv.grad.numpy(),
            "dWk_syn": Wks.grad.numpy(), "dWv_syn": Wvs.grad.numpy(), "dQ0": Q0t.grad.numpy()}


@pytest.mark.parametrize("masked", [False, True])
def test_flarepp_grads_match_torch_autograd(oracle_mod, masked):
    rng = np.random.default_rng(21)
    B, N, C, H, M = 3, 57, 48, 3, 6
    X, Ws, Q0, dY = rand_problem(rng, B, N, C, H, M, wscale=3.0)
    lengths = np.array([57, 20, 1], dtype=np.int32) if masked else None
    s = 1.0 / math.sqrt(C // H)
    got = oracle_mod.flarepp_backward(X, *Ws, Q0, dY, H, lengths, s)
    ref = torch_flarepp_grads(X, Ws, Q0, dY, H, lengths, s)
    for k, v in ref.items():
        assert rel(got[k], v) < 1e-11, k


def test_flare_grads_match_torch_autograd(oracle_mod):
    rng = np.random.default_rng(22)
    B, H, N, M, D = 2, 3, 70, 7, 16
    K, V = rng.standard_normal((B, H, N, D)), rng.standard_normal((B, H, N, D))
    Q = rng.standard_normal((H, M, D)) * 2.0
    dY = rng.standard_normal((B, H, N, D))
    s = 0.3
    got = oracle_mod.flare_backward(K, V, Q, dY, None, s)
    Kt, Vt, Qt = (torch.tensor(a, requires_grad=True) for a in (K, V, Q))
    Qb = Qt[None].expand(B, -1, -1, -1)
    Z = F.scaled_dot_product_attention(Qb, Kt, Vt, scale=s)
    Y = F.scaled_dot_product_attention(Kt, Qb, Z, scale=s)
    (Y * torch.from_numpy(dY)).sum().backward()
    assert rel(got["dK"], Kt.grad.numpy()) < 1e-11
    assert rel(got["dV"], Vt.grad.numpy()) < 1e-11
    assert rel(got["dQ"], Qt.grad.numpy()) < 1e-11


# --------------------------------------------------------------------------
# central finite differences of the forward oracle
# --------------------------------------------------------------------------

def test_flarepp_directional_derivatives(oracle_mod):
    rng = np.random.default_rng(23)
    B, N, C, H, M = 2, 33, 32, 2, 4
    X, Ws, Q0, dY = rand_problem(rng, B, N, C, H, M, wscale=2.5)
    lengths = np.array([33, 17], dtype=np.int32)
    s = 1.0 / math.sqrt(C // H)
    g = oracle_mod.flarepp_backward(X, *Ws, Q0, dY, H, lengths, s)
    args = {"X": X, "Wk": Ws[0], "Wv": Ws[1], "Wk_syn": Ws[2], "Wv_syn": Ws[3], "Q0": Q0}

    def loss(a):
        Y = oracle_mod.flarepp_forward(a["X"], a["Wk"], a["Wv"], a["Wk_syn"], a["Wv_syn"], a["Q0"],
                                       H, lengths, s)["Y"]
        return float((Y * dY).sum())

    eps = 1e-5
    for name in args:
        u = rng.standard_normal(args[name].shape)
        hi, lo = dict(args), dict(args)
        hi[name] = args[name] + eps * u
        lo[name] = args[name] - eps * u
        fd = (loss(hi) - loss(lo)) / (2 * eps)
        an = float((g["d" + name] * u).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


def test_flare_directional_derivatives_masked(oracle_mod):
    rng = np.random.default_rng(24)
    B, H, N, M, D = 2, 2, 29, 6, 16
    K, V = rng.standard_normal((B, H, N, D)), rng.standard_normal((B, H, N, D))
    Q = rng.standard_normal((H, M, D))
    dY = rng.standard_normal((B, H, N, D))
    lengths = np.array([12, 29], dtype=np.int32)
    g = oracle_mod.flare_backward(K, V, Q, dY, lengths, 0.4)
    args = {"K": K, "V": V, "Q": Q}

    def loss(a):
        return float((oracle_mod.flare_forward(a["K"], a["V"], a["Q"], lengths, 0.4)["Y"] * dY).sum())

    eps = 1e-5
    for name in args:
        u = rng.standard_normal(args[name].shape)
        hi, lo = dict(args), dict(args)
        hi[name] = args[name] + eps * u
        lo[name] = args[name] - eps * u
        fd = (loss(hi) - loss(lo)) / (2 * eps)
        an = float((g["d" + name] * u).sum())
        assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (name, fd, an)


# --------------------------------------------------------------------------
# invariances and sum rules
# --------------------------------------------------------------------------

def _enc_problem(rng, B=2, H=2, N=37, M=6, D=16, per_batch=True):
    Q = rng.standard_normal((B, H, M, D) if per_batch else (H, M, D)) * 1.5
    K, V = rng.standard_normal((B, H, N, D)), rng.standard_normal((B, H, N, D))
    dZ = rng.standard_normal((B, H, M, D))
    return Q, K, V, dZ


def test_encoder_key_gradients_sum_to_zero(oracle_mod):
    """Adding one vector to every key shifts each encoder row's scores by a
    constant, so the softmax and Z do not change: sum_n dK_n = 0."""
    rng = np.random.default_rng(25)
    Q, K, V, dZ = _enc_problem(rng)
    lengths = np.array([37, 11], dtype=np.int32)
    dQ, dK, dV = oracle_mod.encode_bwd(Q, K, V, dZ, lengths, 0.35)
    tot = dK.sum(axis=2)
    assert np.abs(tot).max() < 1e-12 * np.abs(dK).max() * dK.shape[2]
    assert np.abs(dK).max() > 1e-3


def test_decoder_query_gradients_sum_to_zero(oracle_mod):
    """Adding one vector to every latent query shifts each decoder row's
    scores by a constant: sum_m dQ_m = 0 (per sample and shared)."""
    rng = np.random.default_rng(26)
    B, H, N, M, D = 2, 2, 31, 7, 16
    K = rng.standard_normal((B, H, N, D))
    Z = rng.standard_normal((B, H, M, D))
    dY = rng.standard_normal((B, H, N, D))
    for Q in (rng.standard_normal((B, H, M, D)), rng.standard_normal((H, M, D))):
        dK, dQ, dZ = oracle_mod.decode_bwd(K, Q, Z, dY, None, 0.5)
        tot = dQ.sum(axis=-2)
        assert np.abs(tot).max() < 1e-12 * np.abs(dQ).max() * M
        assert np.abs(dQ).max() > 1e-3


def test_row_stochastic_sum_rules(oracle_mod):
    """Every encoder row and every decoder row is a convex combination:
    sum_n dV_n = sum_m dZ_m (encoder) and sum_m dZ_m = sum_{n<L} dY_n (decoder)."""
    rng = np.random.default_rng(27)
    Q, K, V, dZ = _enc_problem(rng, per_batch=False)
    lengths = np.array([20, 37], dtype=np.int32)
    _, _, dV = oracle_mod.encode_bwd(Q, K, V, dZ, lengths, 0.25)
    assert np.allclose(dV.sum(axis=2), dZ.sum(axis=2), rtol=0, atol=1e-11)
    Z = rng.standard_normal(dZ.shape)
    dY = rng.standard_normal(K.shape)
    _, _, dZd = oracle_mod.decode_bwd(K, Q, Z, dY, lengths, 0.25)
    for b, L in enumerate(lengths):
        assert np.allclose(dZd[b].sum(axis=1), dY[b, :, :L].sum(axis=1), rtol=0, atol=1e-11)


def test_single_latent(oracle_mod):
    """M = 1: the decoder's softmax is 1 for every token, so Y_n = Z_0; the
    decoder passes dZ_0 = sum_n dY_n and gives K and Q no gradient."""
    rng = np.random.default_rng(28)
    B, H, N, D = 2, 3, 25, 16
    K = rng.standard_normal((B, H, N, D))
    Q = rng.standard_normal((B, H, 1, D))
    Z = rng.standard_normal((B, H, 1, D))
    dY = rng.standard_normal((B, H, N, D))
    dK, dQ, dZ = oracle_mod.decode_bwd(K, Q, Z, dY, None, 0.25)
    assert np.abs(dK).max() < 1e-14 and np.abs(dQ).max() < 1e-14
    assert np.allclose(dZ[:, :, 0], dY.sum(axis=2), rtol=0, atol=1e-12)


def test_masked_tokens_get_no_gradient_and_match_truncation(oracle_mod):
    rng = np.random.default_rng(29)
    B, N, C, H, M = 2, 40, 32, 2, 5
    X, Ws, Q0, dY = rand_problem(rng, B, N, C, H, M)
    lengths = np.array([40, 13], dtype=np.int32)
    g = oracle_mod.flarepp_backward(X, *Ws, Q0, dY, H, lengths)
    assert np.all(g["dX"][1, 13:] == 0)
    t = oracle_mod.flarepp_backward(X[1:, :13], *Ws, Q0, dY[1:, :, :13], H)
    assert rel(g["dX"][1, :13], t["dX"][0]) < 1e-12
    # the weight and seed gradients are sums over samples: sample 1 alone
    # (truncated) plus sample 0 alone (full) give the masked batch's values
    f = oracle_mod.flarepp_backward(X[:1], *Ws, Q0, dY[:1], H)
    for k in ("dWk", "dWv", "dWk_syn", "dWv_syn", "dQ0"):
        assert rel(g[k], f[k] + t[k]) < 1e-12, k
