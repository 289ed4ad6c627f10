"""Host-side checks of the torch.autograd wrappers (no GPU): the library
calls are replaced by recording stand-ins, so what is checked is the
plumbing -- which saved tensors reach the backward, the dtypes of the
returned gradients, and that the shared-projection variant hands the shared
weights' gradient to autograd once."""
import torch

import rank_latent_routing_flare_b200 as fl
from rank_latent_routing_flare_b200 import _binding, autograd


def _fake_pp(monkeypatch, calls):
    def fwd(X, Wk, Wv, Wk_syn, Wv_syn, Q0, lengths=None, scale=0.0):
        B, N, C = X.shape
        H, M, D = Q0.shape
        calls.append(("fwd", scale))
        return torch.zeros((B, H, N, D), dtype=torch.bfloat16)

    def bwd(X, Wk, Wv, Wk_syn, Wv_syn, Q0, dY, lengths=None, scale=0.0):
        calls.append(("bwd", dY.dtype, dY.is_contiguous(), Wk_syn is Wk))
        C = X.shape[2]
        full = lambda v: torch.full((C, C), v, dtype=torch.float32)  # noqa: E731
        return {"dX": torch.ones_like(X), "dWk": full(1.0), "dWv": full(2.0), "dWk_syn": full(1.0),
                "dWv_syn": full(2.0), "dQ0": torch.full(Q0.shape, 3.0, dtype=torch.float32)}

    monkeypatch.setattr(_binding, "flarepp_mixer_fwd", fwd)
    monkeypatch.setattr(_binding, "flarepp_mixer_bwd", bwd)


def _inputs(shared):
    B, N, C, H, M = 1, 8, 64, 4, 16
    X = torch.zeros((B, N, C), dtype=torch.bfloat16, requires_grad=True)
    Wk = torch.zeros((C, C), dtype=torch.bfloat16, requires_grad=True)
    Wv = torch.zeros((C, C), dtype=torch.bfloat16, requires_grad=True)
    Wks = Wk if shared else torch.zeros((C, C), dtype=torch.bfloat16, requires_grad=True)
    Wvs = Wv if shared else torch.zeros((C, C), dtype=torch.bfloat16, requires_grad=True)
    Q0 = torch.zeros((H, M, C // H), dtype=torch.bfloat16, requires_grad=True)
    return X, Wk, Wv, Wks, Wvs, Q0


def test_flarepp_wrapper_plumbing(monkeypatch):
    calls = []
    _fake_pp(monkeypatch, calls)
    X, Wk, Wv, Wks, Wvs, Q0 = _inputs(shared=False)
    Y = fl.flarepp_mixer(X, Wk, Wv, Wks, Wvs, Q0, scale=0.5)
    (Y.float() * 2.0).sum().backward()
    assert calls[0] == ("fwd", 0.5)
    assert calls[1][:3] == ("bwd", torch.bfloat16, True)
    assert X.grad.dtype == torch.bfloat16 and torch.all(X.grad == 1)
    assert Wk.grad.dtype == torch.bfloat16 and torch.all(Wk.grad == 1) and torch.all(Wks.grad == 1)
    assert torch.all(Wv.grad == 2) and torch.all(Wvs.grad == 2)
    assert Q0.grad.dtype == torch.bfloat16 and torch.all(Q0.grad == 3)


def test_flarepp_wrapper_shared_weights_counted_once(monkeypatch):
    calls = []
    _fake_pp(monkeypatch, calls)
    X, Wk, Wv, Wks, Wvs, Q0 = _inputs(shared=True)
    Y = autograd.flarepp_mixer(X, Wk, Wv, Wks, Wvs, Q0)
    Y.float().sum().backward()
    assert calls[1][3] is True
    # the library's dWk already holds both uses; autograd must not add dWk_syn on top
    assert torch.all(Wk.grad == 1) and torch.all(Wv.grad == 2)


def test_flare_wrapper_plumbing(monkeypatch):
    def fwd(K, V, Q, lengths=None, scale=0.0):
        return torch.zeros_like(K)

    def bwd(K, V, Q, dY, lengths=None, scale=0.0):
        return torch.ones_like(K), torch.full_like(V, 2.0), torch.full(Q.shape, 3.0, dtype=torch.float32)

    monkeypatch.setattr(_binding, "flare_mixer_fwd", fwd)
    monkeypatch.setattr(_binding, "flare_mixer_bwd", bwd)
    K = torch.zeros((1, 2, 8, 16), dtype=torch.bfloat16, requires_grad=True)
    V = torch.zeros_like(K, requires_grad=True)
    Q = torch.zeros((2, 16, 16), dtype=torch.bfloat16, requires_grad=True)
    fl.flare_mixer(K, V, Q).float().sum().backward()
    assert torch.all(K.grad == 1) and torch.all(V.grad == 2)
    assert Q.grad.dtype == torch.bfloat16 and torch.all(Q.grad == 3)
