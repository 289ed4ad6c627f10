"""Pins of the fp64 oracle against facts the FLARE/FLARE++ pages and the
mathematics fix, independent of the oracle's own code.

Passages (FLARE++ paper, arXiv 2608.11519, section "Method"):
  - SDPA definition, scale 1/sqrt(D), head split into width D = C/H
    ("Full self-attention")
  - FLARE encoder/decoder Z = SDPA(Q, K, V), Y = SDPA(K, Q, Z), Y = W_dec W_enc V,
    rank <= M ("FLARE: fixed-query latent routing", eq. 5-6)
  - FLARE++ query synthesis Q(X) = SDPA(Q~, K~, V~) and the encode/decode with
    Q(X), rank <= M ("FLARE++: dynamic token routing", eq. 7-11)
  - exact shard combine L = logsumexp_r L_r, Z = sum_r exp(L_r - L) O_r
    ("Multi-GPU context parallelism", eq. 13-14)
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from workloads import bf16_bits_to_f64, make_workload, to_bf16_bits


def rel(a, b):
    a, b = np.asarray(a), np.asarray(b)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def rand_flarepp(rng, B=2, N=97, C=32, H=2, M=6, wscale=1.0):
    D = C // H
    X = rng.standard_normal((B, N, C))
    Ws = [rng.standard_normal((C, C)) * wscale / math.sqrt(C) for _ in range(4)]
    Q0 = rng.standard_normal((H, M, D))
    return X, Ws, Q0


# --------------------------------------------------------------------------
# library routine: torch float64 scaled_dot_product_attention chain
# --------------------------------------------------------------------------

def torch_heads(X, W, H):
    B, N, C = X.shape
    D = C // H
    return (torch.from_numpy(X) @ torch.from_numpy(W)).view(B, N, H, D).transpose(1, 2)


def torch_flarepp(X, Ws, Q0, H, lengths, scale):
    Wk, Wv, Wks, Wvs = Ws
    B, N, C = X.shape
    Kt, Vt = torch_heads(X, Wks, H), torch_heads(X, Wvs, H)
    K, V = torch_heads(X, Wk, H), torch_heads(X, Wv, H)
    if lengths is None:
        mask = None
        valid = torch.ones(B, N, dtype=torch.bool)
    else:
        valid = torch.arange(N)[None, :] < torch.as_tensor(lengths)[:, None]
        mask = valid[:, None, None, :]
    Q0t = torch.from_numpy(Q0)[None].expand(B, -1, -1, -1)
    Qx = F.scaled_dot_product_attention(Q0t, Kt, Vt, attn_mask=mask, scale=scale)
    Z = F.scaled_dot_product_attention(Qx, K, V, attn_mask=mask, scale=scale)
    Y = F.scaled_dot_product_attention(K, Qx, Z, scale=scale)
    Y = Y * valid[:, None, :, None]
    return Qx.numpy(), Z.numpy(), Y.numpy()


@pytest.mark.parametrize("masked", [False, True])
def test_flarepp_matches_torch_sdpa_chain(oracle_mod, masked):
    rng = np.random.default_rng(11)
    B, N, C, H, M = 3, 131, 48, 3, 7
    X, Ws, Q0 = rand_flarepp(rng, B, N, C, H, M, wscale=3.0)
    lengths = np.array([131, 40, 1], dtype=np.int32) if masked else None
    s = 1.0 / math.sqrt(C // H)
    out = oracle_mod.flarepp_forward(X, *Ws, Q0, H, lengths, s)
    Qx, Z, Y = torch_flarepp(X, Ws, Q0, H, lengths, s)
    assert rel(out["Qx"], Qx) < 1e-12
    assert rel(out["Z"], Z) < 1e-12
    assert rel(out["Y"], Y) < 1e-12
    if masked:
        assert np.all(out["Y"][1, :, 40:] == 0) and np.all(out["Y"][2, :, 1:] == 0)


def test_flare_matches_torch_sdpa_chain(oracle_mod):
    rng = np.random.default_rng(12)
    B, H, N, M, D = 2, 3, 200, 9, 16
    K = rng.standard_normal((B, H, N, D))
    V = rng.standard_normal((B, H, N, D))
    Q = rng.standard_normal((H, M, D)) * 2.0
    s = 0.3
    out = oracle_mod.flare_forward(K, V, Q, None, s)
    Kt, Vt = torch.from_numpy(K), torch.from_numpy(V)
    Qt = torch.from_numpy(Q)[None].expand(B, -1, -1, -1)
    Z = F.scaled_dot_product_attention(Qt, Kt, Vt, scale=s)
    Y = F.scaled_dot_product_attention(Kt, Qt, Z, scale=s)
    assert rel(out["Z"], Z.numpy()) < 1e-12
    assert rel(out["Y"], Y.numpy()) < 1e-12


def test_project_matches_matmul(oracle_mod):
    rng = np.random.default_rng(1)
    X = rng.standard_normal((2, 33, 64))
    W = rng.standard_normal((64, 64))
    P = oracle_mod.project(X, W, 4)
    ref = np.einsum("bnc,cj->bnj", X, W).reshape(2, 33, 4, 16).transpose(0, 2, 1, 3)
    assert rel(P, ref) < 1e-13


# --------------------------------------------------------------------------
# brute force: the materialised N x N mixing matrix (tiny N)
# --------------------------------------------------------------------------

def softmax_rows(A):
    A = A - A.max(axis=1, keepdims=True)
    E = np.exp(A)
    return E / E.sum(axis=1, keepdims=True)


@pytest.mark.parametrize("variant", ["flare", "flarepp"])
def test_materialised_mixing_matrix(oracle_mod, variant):
    """Y_h = W_dec W_enc V_h with W_enc row-stochastic over tokens (M x N) and
    W_dec row-stochastic over latents (N x M); the product has rank <= M."""
    rng = np.random.default_rng(5)
    N, C, H, M = 64, 16, 2, 5
    D = C // H
    s = 1.0 / math.sqrt(D)
    if variant == "flare":
        K = rng.standard_normal((1, H, N, D)) * 1.5
        V = rng.standard_normal((1, H, N, D))
        Q = rng.standard_normal((H, M, D)) * 1.5
        out = oracle_mod.flare_forward(K, V, Q, None, s)
        Qh = Q
    else:
        X, Ws, Q0 = rand_flarepp(rng, 1, N, C, H, M, wscale=4.0)
        out = oracle_mod.flarepp_forward(X, *Ws, Q0, H, None, s)
        K = np.einsum("bnc,cj->bnj", X, Ws[0]).reshape(1, N, H, D).transpose(0, 2, 1, 3)
        V = np.einsum("bnc,cj->bnj", X, Ws[1]).reshape(1, N, H, D).transpose(0, 2, 1, 3)
        Qh = out["Qx"][0]
    for h in range(H):
        S = s * Qh[h] @ K[0, h].T                      # M x N
        W_enc = softmax_rows(S)                        # softmax over tokens
        W_dec = softmax_rows(S.T)                      # softmax over latents
        A = W_dec @ W_enc                              # N x N
        assert np.all(A >= 0)
        assert np.max(np.abs(A.sum(axis=1) - 1.0)) < 1e-12
        sv = np.linalg.svd(A, compute_uv=False)
        assert sv[M] / sv[0] < 1e-10                   # rank <= M
        assert rel(out["Y"][0, h], A @ V[0, h]) < 1e-12


# --------------------------------------------------------------------------
# closed forms and special cases
# --------------------------------------------------------------------------

def test_two_tokens_one_latent_closed_form(oracle_mod):
    """Softmax over two scores is the logistic function of their difference."""
    q, k1, k2, v1, v2, s = 0.7, 1.3, -0.4, 2.5, -1.25, 0.9
    K = np.array([k1, k2]).reshape(1, 1, 2, 1)
    V = np.array([v1, v2]).reshape(1, 1, 2, 1)
    Q = np.array([q]).reshape(1, 1, 1)
    Z = oracle_mod.encode(Q, K, V, None, s)
    sig = 1.0 / (1.0 + math.exp(-s * q * (k1 - k2)))
    assert abs(Z[0, 0, 0, 0] - (sig * v1 + (1 - sig) * v2)) < 1e-15
    # one latent: the decoder softmax over a single latent is 1 for every token
    Y = oracle_mod.decode(K, Q, Z, None, s)
    assert np.all(Y[0, 0, :, 0] == Z[0, 0, 0, 0])


def test_identical_keys_give_token_mean(oracle_mod):
    rng = np.random.default_rng(2)
    B, H, N, M, D = 1, 2, 50, 4, 16
    K = np.broadcast_to(rng.standard_normal((1, H, 1, D)), (B, H, N, D)).copy()
    V = rng.standard_normal((B, H, N, D))
    Q = rng.standard_normal((H, M, D))
    Z = oracle_mod.encode(Q, K, V)
    assert np.max(np.abs(Z - V.mean(axis=2, keepdims=True))) < 1e-13


def test_zero_queries_give_uniform_routing(oracle_mod):
    rng = np.random.default_rng(3)
    B, H, N, M, D = 2, 2, 77, 3, 16
    K = rng.standard_normal((B, H, N, D))
    V = rng.standard_normal((B, H, N, D))
    Q = np.zeros((H, M, D))
    out = oracle_mod.flare_forward(K, V, Q)
    mean = V.mean(axis=2, keepdims=True)
    assert np.max(np.abs(out["Z"] - mean)) < 1e-13
    assert np.max(np.abs(out["Y"] - mean)) < 1e-13


def test_zero_seeds_give_mean_synthesis_values(oracle_mod):
    """Q~ = 0: the synthesis softmax is uniform, so Q(X) = mean_n X W~_V."""
    rng = np.random.default_rng(4)
    B, N, C, H, M = 2, 60, 32, 2, 4
    X, Ws, _ = rand_flarepp(rng, B, N, C, H, M)
    Q0 = np.zeros((H, M, C // H))
    out = oracle_mod.flarepp_forward(X, *Ws, Q0, H)
    xbar = X.mean(axis=1)                                # B x C
    want = (xbar @ Ws[3]).reshape(B, H, 1, C // H)
    assert np.max(np.abs(out["Qx"] - want)) < 1e-13


def test_single_latent_broadcasts_z(oracle_mod):
    rng = np.random.default_rng(6)
    X, Ws, Q0 = rand_flarepp(rng, 2, 40, 32, 2, 1)
    out = oracle_mod.flarepp_forward(X, *Ws, Q0, 2)
    assert np.max(np.abs(out["Y"] - out["Z"][:, :, 0:1, :])) < 1e-14


def test_hard_max_limit(oracle_mod):
    """Scores of order 1e3: the softmax is one-hot at the arg-max; no overflow."""
    H, N, M, D = 1, 8, 3, 16
    rng = np.random.default_rng(7)
    K = rng.standard_normal((1, H, N, D)) * 300
    V = rng.standard_normal((1, H, N, D))
    Q = rng.standard_normal((H, M, D)) * 300
    Z = oracle_mod.encode(Q, K, V)
    for m in range(M):
        n_star = int(np.argmax(K[0, 0] @ Q[0, m]))
        assert np.allclose(Z[0, 0, m], V[0, 0, n_star], atol=1e-12)
    assert np.all(np.isfinite(Z))
    # decoder: every token takes the latent value of its arg-max latent
    Y = oracle_mod.decode(K, Q, Z)
    for n in range(N):
        m_star = int(np.argmax(Q[0] @ K[0, 0, n]))
        assert np.allclose(Y[0, 0, n], Z[0, 0, m_star], atol=1e-12)


# --------------------------------------------------------------------------
# invariants
# --------------------------------------------------------------------------

def test_token_permutation_equivariance(oracle_mod):
    rng = np.random.default_rng(8)
    X, Ws, Q0 = rand_flarepp(rng, 1, 90, 32, 2, 5, wscale=3.0)
    perm = rng.permutation(90)
    a = oracle_mod.flarepp_forward(X, *Ws, Q0, 2)
    b = oracle_mod.flarepp_forward(X[:, perm], *Ws, Q0, 2)
    assert rel(b["Qx"], a["Qx"]) < 1e-13
    assert rel(b["Z"], a["Z"]) < 1e-13
    assert rel(b["Y"], a["Y"][:, :, perm]) < 1e-13


def test_mask_equals_truncation(oracle_mod):
    """With key padding, sample b equals the unmasked forward on X[b, :L_b];
    padded rows of Y are exactly zero."""
    rng = np.random.default_rng(9)
    B, N, C, H, M = 3, 64, 32, 2, 4
    X, Ws, Q0 = rand_flarepp(rng, B, N, C, H, M, wscale=2.0)
    L = np.array([64, 17, 1], dtype=np.int32)
    out = oracle_mod.flarepp_forward(X, *Ws, Q0, H, L)
    for b in range(B):
        sub = oracle_mod.flarepp_forward(X[b:b + 1, :L[b]], *Ws, Q0, H)
        assert rel(out["Qx"][b], sub["Qx"][0]) < 1e-13
        assert rel(out["Z"][b], sub["Z"][0]) < 1e-13
        assert rel(out["Y"][b, :, :L[b]], sub["Y"][0]) < 1e-13
        assert np.all(out["Y"][b, :, L[b]:] == 0)


@pytest.mark.parametrize("cuts", [(1,), (37, 38), (5, 50, 99)])
def test_shard_combine_identity(oracle_mod, cuts):
    """eq. 14: encoding token shards separately and combining their outputs with
    L = logsumexp_r L_r, Z = sum_r exp(L_r - L) O_r equals encoding all tokens."""
    rng = np.random.default_rng(10)
    B, H, N, M, D = 2, 2, 128, 6, 16
    K = rng.standard_normal((B, H, N, D)) * 2
    V = rng.standard_normal((B, H, N, D))
    Q = rng.standard_normal((H, M, D)) * 2
    Z, lse = oracle_mod.encode(Q, K, V, return_lse=True)
    bounds = [0, *cuts, N]
    parts = [oracle_mod.encode(Q, K[:, :, a:b], V[:, :, a:b], return_lse=True)
             for a, b in zip(bounds[:-1], bounds[1:])]
    Ls = np.stack([p[1] for p in parts])           # R x B x H x M
    L = np.logaddexp.reduce(Ls, axis=0)
    Zc = sum(np.exp(Lr - L)[..., None] * Or for Or, Lr in parts)
    assert rel(L, lse) < 1e-14
    assert rel(Zc, Z) < 1e-13


def test_scale_argument(oracle_mod):
    rng = np.random.default_rng(13)
    K = rng.standard_normal((1, 2, 30, 16))
    V = rng.standard_normal((1, 2, 30, 16))
    Q = rng.standard_normal((2, 4, 16))
    a = oracle_mod.flare_forward(K, V, Q, scale=0.7)
    b = oracle_mod.flare_forward(K, V, Q * (0.7 * 4.0), scale=0.25)
    c = oracle_mod.flare_forward(K, V, Q * (0.7 * 4.0))        # default 1/sqrt(D)
    assert rel(a["Z"], b["Z"]) < 1e-13
    assert rel(b["Y"], c["Y"]) < 1e-15


def test_decode_row_sampling_is_exact(oracle_mod):
    rng = np.random.default_rng(14)
    X, Ws, Q0 = rand_flarepp(rng, 2, 50, 32, 2, 3)
    full = oracle_mod.flarepp_forward(X, *Ws, Q0, 2, np.array([50, 20], np.int32))
    rows = np.array([0, 7, 19, 20, 49])
    part = oracle_mod.flarepp_forward(X, *Ws, Q0, 2, np.array([50, 20], np.int32), rows=rows)
    assert np.array_equal(part["Y"], full["Y"][:, :, rows])


# --------------------------------------------------------------------------
# input generator
# --------------------------------------------------------------------------

def test_bf16_rounding():
    vals = np.array([1.0, -2.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9,
                     3.0e38, 1e-40], dtype=np.float32)
    bits = to_bf16_bits(vals)
    # 1+2^-8 is a tie between 1 and 1+2^-7: round to even (1.0)
    assert list(bits[:5]) == [0x3F80, 0xC000, 0x3F80, 0x3F82, 0x3F80]
    back = bf16_bits_to_f64(bits)
    assert back[0] == 1.0 and back[1] == -2.0


def test_workloads_are_deterministic():
    a = make_workload("flarepp_n1k")
    b = make_workload("flarepp_n1k")
    c = make_workload("flarepp_n1k", seed=99)
    assert np.array_equal(a.X, b.X) and np.array_equal(a.Q0, b.Q0)
    assert not np.array_equal(a.X, c.X)
    m = make_workload("flarepp_masked_n4k", N=512, B=4)
    assert m.lengths.dtype == np.int32 and m.lengths.min() >= 128 and m.lengths.max() <= 512


# --------------------------------------------------------------------------
# head concatenation and output projection ("Full self-attention": the heads'
# outputs side by side, times W_O; row-vector convention Out = Ycat @ W_O)
# --------------------------------------------------------------------------

def test_output_projection_closed_form(oracle_mod):
    a, b = 0.75, -2.5
    Y = np.array([[[[a]], [[b]]]])                  # B=1, H=2, N=1, D=1
    Wo = np.array([[1.0, 2.0], [3.0, 4.0]])
    out = oracle_mod.output_projection(Y, Wo)
    assert out.shape == (1, 1, 2)
    assert np.array_equal(out[0, 0], [a * 1.0 + b * 3.0, a * 2.0 + b * 4.0])


def test_output_projection_identity_concatenates_heads_in_order(oracle_mod):
    rng = np.random.default_rng(21)
    B, H, N, D = 2, 3, 5, 4
    Y = rng.standard_normal((B, H, N, D))
    out = oracle_mod.output_projection(Y, np.eye(H * D))
    for h in range(H):
        assert np.array_equal(out[:, :, h * D:(h + 1) * D], Y[:, h])


def test_output_projection_matches_torch_linear(oracle_mod):
    rng = np.random.default_rng(22)
    X, Ws, Q0 = rand_flarepp(rng, 2, 57, 32, 2, 5)
    Wo = rng.standard_normal((32, 32)) / math.sqrt(32)
    s = 1.0 / math.sqrt(16)
    out = oracle_mod.flarepp_forward(X, *Ws, Q0, 2, None, s)
    _, _, Y = torch_flarepp(X, Ws, Q0, 2, None, s)
    Ycat = torch.from_numpy(Y).transpose(1, 2).reshape(2, 57, 32)
    ref = F.linear(Ycat, torch.from_numpy(Wo).t()).numpy()
    assert rel(oracle_mod.output_projection(out["Y"], Wo), ref) < 1e-12
