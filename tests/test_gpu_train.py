"""GPU parity of the training pair (flarepp_mixer_fwd_train / _bwd_train and
the FLARE ones) against the fp64 oracle and against the stand-alone calls.

At D = 32 the training forward writes the same Y as flarepp_mixer_fwd (bit
for bit: the same kernels, the normalisers also stored).  At D = 16 its
decoder runs the value product on fp16 Z and weights (so that the fp32 Y it
keeps for the backward sees Z to 2^-12): Y is then held to the forward's own
parity criteria against the oracle (``tests/parity.py``) and is at least as
close to it as the plain forward's.  The backward reuses the forward's state instead
of recomputing it; its gradients are held to the backward's tolerance
against the oracle: rel-L2 <= 5e-3 and max |error| <= 3e-2 * max |reference|
per tensor.  The self-contained backward calls (flarepp_mixer_bwd,
flare_mixer_bwd) run the training forward's launches themselves and then the
same backward launches, so their gradients equal the pair's bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import rank_latent_routing_flare_b200 as fl
from tests.gpu_util import compare, dev_bf16, host_f64, rel_l2
from tests.test_gpu_backward import check, flare_case, lengths_dev, run_flare_bwd, run_flarepp_bwd
from workloads import make_upstream_grad, make_workload

pytestmark = pytest.mark.gpu


def flarepp_inputs(w, shared=False):
    X = dev_bf16(w.X)
    Wk, Wv = dev_bf16(w.Wk), dev_bf16(w.Wv)
    Wks, Wvs = (Wk, Wv) if shared else (dev_bf16(w.Wk_syn), dev_bf16(w.Wv_syn))
    return X, Wk, Wv, Wks, Wvs, dev_bf16(w.Q0)


def run_flarepp_train(w, dY, shared=False):
    args = flarepp_inputs(w, shared)
    L = lengths_dev(w)
    Y, ws = fl.flarepp_mixer_fwd_train(*args, lengths=L)
    g = fl.flarepp_mixer_bwd_train(*args, dev_bf16(dY), ws, lengths=L, device_check=True)
    torch.cuda.synchronize()
    return Y, {k: host_f64(v) for k, v in g.items()}, ws


def run_flare_train(w, dY):
    K, V, Q = dev_bf16(w.K), dev_bf16(w.V), dev_bf16(w.Q)
    L = lengths_dev(w)
    Y, ws = fl.flare_mixer_fwd_train(K, V, Q, lengths=L)
    dK, dV, dQ = fl.flare_mixer_bwd_train(K, V, Q, dev_bf16(dY), ws, lengths=L, device_check=True)
    torch.cuda.synchronize()
    return Y, {"dK": host_f64(dK), "dV": host_f64(dV), "dQ": host_f64(dQ)}, ws


PP_KEYS = ("dX", "dWk", "dWv", "dWk_syn", "dWv_syn", "dQ0")


def check_train_y(w, Y, Y_plain, label):
    """The training forward's Y: bitwise the plain forward's at D = 32; at
    D = 16 (the decoder's value product in fp16) within the forward's parity
    criteria and no further from the oracle than the plain forward's Y."""
    if w.D != 16:
        assert torch.equal(Y.view(torch.int16), Y_plain.view(torch.int16)), label
        return
    ref = oracle.forward_workload(w)
    got, plain = host_f64(Y), host_f64(Y_plain)
    compare({"Y": got}, ref, label=label, lengths=w.lengths)
    e_train, e_plain = rel_l2(got, ref["Y"]), rel_l2(plain, ref["Y"])
    print(f"{label}: Y rel-L2 training forward {e_train:.3e}, plain forward {e_plain:.3e}")
    assert e_train <= e_plain * 1.02 + 1e-6, (label, e_train, e_plain)


@pytest.mark.parametrize("name,N,B", [
    ("flarepp_n1k", None, None),
    ("flarepp_n8k_mesh2d", 1500, 2),
    ("flarepp_masked_n4k", 640, 3),
    ("flarepp_n1m_mesh3d", 3000, None),
])
def test_flarepp_training_pair_matches_oracle(name, N, B):
    w = make_workload(name, N=N, B=B)
    dY = make_upstream_grad(w)
    Y, got, _ = run_flarepp_train(w, dY)
    Y_ref = fl.flarepp_mixer_fwd(*flarepp_inputs(w), lengths=lengths_dev(w))
    check_train_y(w, Y, Y_ref, f"train {name} forward")
    ref = oracle.backward_workload(w, dY)
    plain = run_flarepp_bwd(w, dY)
    for k in PP_KEYS:
        check(got[k], ref[k], f"train {name} N{w.N} B{w.B} {k}")
        assert np.array_equal(got[k], plain[k]), (name, k, rel_l2(got[k], plain[k]))
    if w.lengths is not None:
        for b, L in enumerate(w.lengths):
            assert np.all(got["dX"][b, L:] == 0)


@pytest.mark.parametrize("B,H,N,M,D,lengths", [
    (2, 2, 777, 64, 16, None),
    (2, 2, 777, 64, 16, [777, 300]),
    (1, 3, 1000, 48, 32, None),
    (3, 2, 200, 16, 16, [1, 200, 129]),
    (1, 2, 500, 112, 16, [433]),
])
def test_flare_training_pair_matches_oracle(B, H, N, M, D, lengths):
    w = flare_case(B, H, N, M, D, lengths)
    dY = make_upstream_grad(w)
    Y, got, _ = run_flare_train(w, dY)
    Y_ref = fl.flare_mixer_fwd(dev_bf16(w.K), dev_bf16(w.V), dev_bf16(w.Q), lengths=lengths_dev(w))
    check_train_y(w, Y, Y_ref, f"train FLARE forward D{D}")
    ref = oracle.backward_workload(w, dY)
    plain = run_flare_bwd(w, dY)
    for k in ("dK", "dV", "dQ"):
        check(got[k], ref[k], f"train FLARE {k} B{B} H{H} N{N} M{M} D{D} L{lengths}")
        assert np.array_equal(got[k], plain[k]), (k, rel_l2(got[k], plain[k]))
    if lengths is not None:
        for b, L in enumerate(lengths):
            assert np.all(got["dK"][b, :, L:] == 0) and np.all(got["dV"][b, :, L:] == 0)


def test_training_pair_shared_projections():
    w = make_workload("flarepp_n1k", N=700)
    w.Wk_syn, w.Wv_syn = w.Wk.copy(), w.Wv.copy()
    dY = make_upstream_grad(w)
    _, got, _ = run_flarepp_train(w, dY, shared=True)
    ref = oracle.backward_workload(w, dY)
    check(got["dWk"], ref["dWk"] + ref["dWk_syn"], "train shared dWk")
    check(got["dWv"], ref["dWv"] + ref["dWv_syn"], "train shared dWv")
    check(got["dX"], ref["dX"], "train shared dX")
    check(got["dQ0"], ref["dQ0"], "train shared dQ0")


def test_training_pair_is_deterministic():
    w = make_workload("flarepp_n8k_mesh2d", N=2048, B=2)
    dY = make_upstream_grad(w)
    _, a, _ = run_flarepp_train(w, dY)
    _, b, _ = run_flarepp_train(w, dY)
    for k in a:
        assert np.array_equal(a[k], b[k]), k


def test_training_backward_without_forward_state_is_reported():
    """One forward serves one backward: a second backward, or a backward after
    another call in the same workspace, finds no mark and reports
    ERR_NO_FORWARD (it still runs to its end on the stale workspace)."""
    w = make_workload("flarepp_n1k", N=384)
    dY = dev_bf16(make_upstream_grad(w))
    args = flarepp_inputs(w)
    Y, ws = fl.flarepp_mixer_fwd_train(*args)
    fl.flarepp_mixer_bwd_train(*args, dY, ws)
    assert fl.flare_last_device_status(ws) == fl.Status.OK
    fl.flarepp_mixer_bwd_train(*args, dY, ws)
    assert fl.flare_last_device_status(ws) == fl.Status.ERR_NO_FORWARD
    # a training forward, then a plain forward in the same workspace: no state
    fl.flarepp_mixer_fwd_train(*args, workspace=ws)
    fl.flarepp_mixer_fwd(*args, workspace=ws)
    fl.flarepp_mixer_bwd_train(*args, dY, ws)
    assert fl.flare_last_device_status(ws) == fl.Status.ERR_NO_FORWARD
    with pytest.raises(fl.FlareError):
        fl.flarepp_mixer_bwd_train(*args, dY, ws, device_check=True)
    # FLARE: a fresh (zeroed) workspace has no mark
    wf = flare_case(1, 2, 300, 32, 16)
    K, V, Q = dev_bf16(wf.K), dev_bf16(wf.V), dev_bf16(wf.Q)
    nb = fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLARE_BWD, 1, 2, 300, 32, 16)
    wsf = torch.zeros(nb, dtype=torch.uint8, device="cuda")
    fl.flare_mixer_bwd_train(K, V, Q, dev_bf16(make_upstream_grad(wf)), wsf)
    assert fl.flare_last_device_status(wsf) == fl.Status.ERR_NO_FORWARD


def test_autograd_save_state_matches_the_training_calls():
    """fl.flarepp_mixer(..., save_state=True) gives the bits of the training
    pair called directly; a second backward through the graph raises."""
    w = make_workload("flarepp_n1k", N=512)
    X = dev_bf16(w.X).requires_grad_()
    Ws = [dev_bf16(a).requires_grad_() for a in (w.Wk, w.Wv, w.Wk_syn, w.Wv_syn)]
    Q0 = dev_bf16(w.Q0).requires_grad_()
    dY = dev_bf16(make_upstream_grad(w))
    Y = fl.flarepp_mixer(X, *Ws, Q0, save_state=True)
    loss = (Y.float() * dY.float()).sum()
    loss.backward(retain_graph=True)
    det = [X.detach(), *[a.detach() for a in Ws], Q0.detach()]
    Y_direct, ws = fl.flarepp_mixer_fwd_train(*det)
    g = fl.flarepp_mixer_bwd_train(*det, dY, ws)
    torch.cuda.synchronize()
    assert torch.equal(Y.detach().view(torch.int16), Y_direct.view(torch.int16))
    assert torch.equal(X.grad.view(torch.int16), g["dX"].view(torch.int16))
    for W, k in zip(Ws, ("dWk", "dWv", "dWk_syn", "dWv_syn")):
        assert torch.equal(W.grad.view(torch.int16), g[k].to(torch.bfloat16).view(torch.int16)), k
    assert torch.equal(Q0.grad.view(torch.int16), g["dQ0"].to(torch.bfloat16).view(torch.int16))
    with pytest.raises(RuntimeError, match="already used"):
        loss.backward()
    # FLARE
    wf = flare_case(2, 2, 400, 32, 16, [400, 250])
    K, V, Q = (dev_bf16(a).requires_grad_() for a in (wf.K, wf.V, wf.Q))
    L = lengths_dev(wf)
    dYf = dev_bf16(make_upstream_grad(wf))
    (fl.flare_mixer(K, V, Q, L, save_state=True).float() * dYf.float()).sum().backward()
    _, wsf = fl.flare_mixer_fwd_train(K.detach(), V.detach(), Q.detach(), lengths=L)
    dK, dV, dQ = fl.flare_mixer_bwd_train(K.detach(), V.detach(), Q.detach(), dYf, wsf, lengths=L)
    torch.cuda.synchronize()
    assert torch.equal(K.grad.view(torch.int16), dK.view(torch.int16))
    assert torch.equal(V.grad.view(torch.int16), dV.view(torch.int16))
    assert torch.equal(Q.grad.view(torch.int16), dQ.to(torch.bfloat16).view(torch.int16))


def test_training_pair_cuda_graph_replays_the_same_bits():
    """Both training calls only enqueue work on their stream: one graph of
    forward + backward replays the eager bits (the mark is set and cleared
    inside the graph)."""
    w = make_workload("flarepp_n8k_mesh2d", N=1024, B=2)
    dY = dev_bf16(make_upstream_grad(w))
    args = flarepp_inputs(w)
    nbytes = fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLAREPP_BWD, w.B, w.H, w.N, w.M, w.D, w.C)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        Y, _ = fl.flarepp_mixer_fwd_train(*args, workspace=ws, stream=s)
        g = fl.flarepp_mixer_bwd_train(*args, dY, ws, stream=s)
        torch.cuda.synchronize()
        eager = {k: v.clone() for k, v in g.items()}
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            fl.flarepp_mixer_fwd_train(*args, workspace=ws, stream=s, Y=Y, check=False)
            fl.flarepp_mixer_bwd_train(*args, dY, ws, stream=s, grads=g, check=False)
    for v in g.values():
        v.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert fl.flare_last_device_status(ws) == fl.Status.OK
    for k in g:
        a = g[k].view(torch.int16) if g[k].dtype == torch.bfloat16 else g[k]
        b = eager[k].view(torch.int16) if eager[k].dtype == torch.bfloat16 else eager[k]
        assert torch.equal(a, b), k
    del graph
