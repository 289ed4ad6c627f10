"""GPU parity of the backward (gradients) against the fp64 oracle.

The CUDA path (flare_mixer_bwd / flarepp_mixer_bwd through the C ABI) and
the oracle (oracle.flare_backward / flarepp_backward) get the same bf16
inputs and the same upstream gradient dY.  Tolerance per gradient tensor:
rel-L2 <= 5e-3 and max |error| <= 3e-2 * max |reference| (the forward's
bounds, the absolute one taken relative to the tensor's scale because
gradients of different tensors differ by orders of magnitude).
"""
import numpy as np
import pytest
import torch

import oracle
import rank_latent_routing_flare_b200 as fl
from tests.gpu_util import dev_bf16, host_f64, rel_l2
from workloads import make_upstream_grad, make_workload

pytestmark = pytest.mark.gpu

REL_L2 = 5e-3
MAX_REL = 3e-2


def check(got, ref, label, rel_bound=REL_L2, max_bound=MAX_REL):
    r = rel_l2(got, ref)
    m = float(np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-30))
    print(f"{label}: rel_l2={r:.3e} max_err/max_ref={m:.3e}")
    assert r <= rel_bound and m <= max_bound, (label, r, m)


def lengths_dev(w):
    return None if w.lengths is None else torch.from_numpy(w.lengths).cuda()


def run_flare_bwd(w, dY):
    dK, dV, dQ = fl.flare_mixer_bwd(dev_bf16(w.K), dev_bf16(w.V), dev_bf16(w.Q), dev_bf16(dY),
                                    lengths=lengths_dev(w))
    torch.cuda.synchronize()
    return {"dK": host_f64(dK), "dV": host_f64(dV), "dQ": host_f64(dQ)}


def run_flarepp_bwd(w, dY, shared=False):
    X = dev_bf16(w.X)
    Wk, Wv = dev_bf16(w.Wk), dev_bf16(w.Wv)
    Wks, Wvs = (Wk, Wv) if shared else (dev_bf16(w.Wk_syn), dev_bf16(w.Wv_syn))
    g = fl.flarepp_mixer_bwd(X, Wk, Wv, Wks, Wvs, dev_bf16(w.Q0), dev_bf16(dY), lengths=lengths_dev(w))
    torch.cuda.synchronize()
    return {k: host_f64(v) for k, v in g.items()}


def flare_case(B, H, N, M, D, lengths=None, seed=5):
    rng = np.random.default_rng(seed)
    from workloads import to_bf16_bits
    w = make_workload("flare_n64k", N=N, B=B, M=M, seed=seed)
    if D != w.D or H != w.H:
        w.H, w.D, w.C = H, D, H * D
        w.K = to_bf16_bits(rng.standard_normal((B, H, N, D), dtype=np.float32))
        w.V = to_bf16_bits(rng.standard_normal((B, H, N, D), dtype=np.float32))
        w.Q = to_bf16_bits(rng.standard_normal((H, M, D), dtype=np.float32))
    if lengths is not None:
        w.lengths = np.asarray(lengths, dtype=np.int32)
    return w


@pytest.mark.parametrize("B,H,N,M,D,lengths", [
    (2, 2, 777, 64, 16, None),
    (2, 2, 777, 64, 16, [777, 300]),
    (1, 3, 1000, 48, 32, None),
    (3, 2, 200, 16, 16, [1, 200, 129]),
    (2, 2, 2000, 256, 32, [2000, 1537]),
    (1, 2, 700, 80, 16, None),        # M = 80: 96 latent rows per CTA, the last 16 idle
    (1, 2, 500, 112, 16, [433]),      # M = 112
])
def test_flare_backward_matches_oracle(B, H, N, M, D, lengths):
    w = flare_case(B, H, N, M, D, lengths)
    dY = make_upstream_grad(w)
    got = run_flare_bwd(w, dY)
    ref = oracle.backward_workload(w, dY)
    for k in ("dK", "dV", "dQ"):
        check(got[k], ref[k], f"FLARE {k} B{B} H{H} N{N} M{M} D{D} L{lengths}")
    if lengths is not None:
        for b, L in enumerate(lengths):
            assert np.all(got["dK"][b, :, L:] == 0) and np.all(got["dV"][b, :, L:] == 0)


@pytest.mark.parametrize("name,N,B", [
    ("flarepp_n1k", None, None),
    ("flarepp_n8k_mesh2d", 1500, 2),
    ("flarepp_masked_n4k", 640, 3),
    ("flarepp_n1m_mesh3d", 3000, None),   # the million-token shape's M = 512: 8 chunks, 4 latent blocks
])
def test_flarepp_backward_matches_oracle(name, N, B):
    w = make_workload(name, N=N, B=B)
    dY = make_upstream_grad(w)
    got = run_flarepp_bwd(w, dY)
    ref = oracle.backward_workload(w, dY)
    for k in ("dX", "dWk", "dWv", "dWk_syn", "dWv_syn", "dQ0"):
        check(got[k], ref[k], f"{name} N{w.N} B{w.B} {k}")
    if w.lengths is not None:
        for b, L in enumerate(w.lengths):
            assert np.all(got["dX"][b, L:] == 0)


def storage_model_bwd(w, dY, p_round=False):
    """The oracle's FLARE++ backward in fp64 on the bf16 tensors that the
    forward stores and the backward reuses: the projections K~, V~, K, V and
    the synthesised queries Q(X), which the encode and the decode scores take
    in bf16 (eq. 10-11 on the forward's stored Q(X); its gradient passes
    through the rounding unchanged).  Everything else is kept in fp32 on the
    GPU and in fp64 here.  With ``p_round`` Q(X) and Z come from the forward
    storage model that also rounds the softmax weights of the value products
    to bf16 (as the forward's kernels read them)."""
    from tests.parity import storage_model
    from workloads import bf16_bits_to_f64 as f64, to_bf16_bits
    r = lambda a: f64(to_bf16_bits(a.astype(np.float32)))
    X, Q0, dy = f64(w.X), f64(w.Q0), f64(dY)
    Wk, Wv, Wks, Wvs = (f64(a) for a in (w.Wk, w.Wv, w.Wk_syn, w.Wv_syn))
    Kt, Vt = r(oracle.project(X, Wks, w.H)), r(oracle.project(X, Wvs, w.H))
    K, V = r(oracle.project(X, Wk, w.H)), r(oracle.project(X, Wv, w.H))
    if p_round:
        fwd = storage_model(w, oracle, p_round=True)
        Qx, Z = r(fwd["Qx"]), fwd["Z"]
    else:
        Qx = r(oracle.encode(Q0, Kt, Vt, w.lengths))
        Z = oracle.encode(Qx, K, V, w.lengths)
    dK, dQx, dZ = oracle.decode_bwd(K, Qx, Z, dy, w.lengths)
    dQx_e, dK_e, dV = oracle.encode_bwd(Qx, K, V, dZ, w.lengths)
    dQ0, dKt, dVt = oracle.encode_bwd(Q0, Kt, Vt, dQx + dQx_e, w.lengths)
    out = {"dQ0": dQ0, "dX": np.zeros_like(X)}
    for nm, W, d in (("dWk", Wk, dK + dK_e), ("dWv", Wv, dV), ("dWk_syn", Wks, dKt), ("dWv_syn", Wvs, dVt)):
        dXi, out[nm] = oracle.project_bwd(X, W, d)
        out["dX"] += dXi
    return out


def test_flarepp_backward_sharp_matches_bf16_storage_model():
    """Diagnostic with all weights ~ N(0, 16/C) (not a graded workload): the
    sharp softmaxes make the gradients sensitive to the bf16 storage of the
    projections and of Q(X), which alone moves them by 2-11 % from the exact
    fp64 values (Q(X) in bf16 accounts for up to 3 % of it).  The forward
    also rounds its softmax weights to bf16 for the value products that give
    Q(X) and Z; that rounding is random (its pattern depends on the shift,
    which differs between the kernels and any model), so it is bounded by its
    size in the model: r_P = rel-L2 between the storage model with and
    without it (1-2 % here).  Checked: the GPU within 1e-2 + 1.5 r_P (rel-L2)
    of the storage model, and no further from the exact gradients than the
    storage model plus 1e-2; the distances are printed."""
    w = make_workload("flarepp_n8k_sharp", N=1200, B=2)
    dY = make_upstream_grad(w)
    got = run_flarepp_bwd(w, dY)
    model = storage_model_bwd(w, dY)
    model_p = storage_model_bwd(w, dY, p_round=True)
    exact = oracle.backward_workload(w, dY)
    for k in ("dX", "dWk", "dWv", "dWk_syn", "dWv_syn", "dQ0"):
        r_p = rel_l2(model_p[k], model[k])
        print(f"sharp {k}: storage model vs exact {rel_l2(model[k], exact[k]):.3e}, "
              f"gpu vs exact {rel_l2(got[k], exact[k]):.3e}, weight rounding r_P {r_p:.3e}")
        check(got[k], model[k], f"sharp {k} vs storage model", rel_bound=1e-2 + 1.5 * r_p, max_bound=5e-2)
        assert rel_l2(got[k], exact[k]) <= rel_l2(model[k], exact[k]) + 1e-2


def test_flarepp_backward_shared_projections():
    """Wk_syn is Wk and Wv_syn is Wv: the shared weights get the sum of both
    uses; the oracle with two identical copies gives the reference."""
    w = make_workload("flarepp_n1k", N=700)
    w.Wk_syn, w.Wv_syn = w.Wk.copy(), w.Wv.copy()
    dY = make_upstream_grad(w)
    got = run_flarepp_bwd(w, dY, shared=True)
    ref = oracle.backward_workload(w, dY)
    check(got["dWk"], ref["dWk"] + ref["dWk_syn"], "shared dWk")
    check(got["dWv"], ref["dWv"] + ref["dWv_syn"], "shared dWv")
    assert np.array_equal(got["dWk"], got["dWk_syn"]) and np.array_equal(got["dWv"], got["dWv_syn"])
    check(got["dX"], ref["dX"], "shared dX")
    check(got["dQ0"], ref["dQ0"], "shared dQ0")


def test_backward_is_deterministic():
    w = make_workload("flarepp_n8k_mesh2d", N=2048, B=2)
    dY = make_upstream_grad(w)
    a = run_flarepp_bwd(w, dY)
    b = run_flarepp_bwd(w, dY)
    for k in a:
        assert np.array_equal(a[k], b[k]), k


def test_backward_reports_bad_lengths():
    w = make_workload("flarepp_n1k", N=256)
    w.lengths = np.array([300], dtype=np.int32)     # > N: clamped, reported
    dY = make_upstream_grad(w)
    ws = torch.empty(fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLAREPP_BWD, w.B, w.H, w.N, w.M, w.D, w.C),
                     dtype=torch.uint8, device="cuda")
    fl.flarepp_mixer_bwd(dev_bf16(w.X), dev_bf16(w.Wk), dev_bf16(w.Wv), dev_bf16(w.Wk_syn), dev_bf16(w.Wv_syn),
                         dev_bf16(w.Q0), dev_bf16(dY), lengths=lengths_dev(w), workspace=ws)
    assert fl.flare_last_device_status(ws) == fl.Status.ERR_SHAPE


def test_backward_cuda_graph_replays_the_same_bits():
    """The backward call only enqueues kernels, memsets and a device-to-device
    copy on its stream, so it can be captured into a CUDA graph; a replay
    gives the eager bits."""
    w = make_workload("flarepp_n8k_mesh2d", N=1024, B=2)
    dY = dev_bf16(make_upstream_grad(w))
    X, Q0 = dev_bf16(w.X), dev_bf16(w.Q0)
    Ws = [dev_bf16(a) for a in (w.Wk, w.Wv, w.Wk_syn, w.Wv_syn)]
    nbytes = fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLAREPP_BWD, w.B, w.H, w.N, w.M, w.D, w.C)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        g = fl.flarepp_mixer_bwd(X, *Ws, Q0, dY, workspace=ws, stream=s)
        torch.cuda.synchronize()
        eager = {k: v.clone() for k, v in g.items()}
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=s):
            fl.flarepp_mixer_bwd(X, *Ws, Q0, dY, workspace=ws, stream=s, grads=g, check=False)
    for v in g.values():
        v.zero_()
    graph.replay()
    torch.cuda.synchronize()
    for k in g:
        assert torch.equal(g[k].view(torch.int16) if g[k].dtype == torch.bfloat16 else g[k],
                           eager[k].view(torch.int16) if eager[k].dtype == torch.bfloat16 else eager[k]), k
    del graph


@pytest.mark.slow
@pytest.mark.parametrize("name", ["flare_n64k", "flarepp_n64k"])
def test_backward_full_size(name):
    """The 64K-token configurations at full size (B=4, N=65536, M=256): every
    gradient against the fp64 oracle (15-60 s of host time)."""
    w = make_workload(name)
    dY = make_upstream_grad(w)
    got = run_flare_bwd(w, dY) if w.variant == "flare" else run_flarepp_bwd(w, dY)
    ref = oracle.backward_workload(w, dY)
    keys = ("dK", "dV", "dQ") if w.variant == "flare" else ("dX", "dWk", "dWv", "dWk_syn", "dWv_syn", "dQ0")
    for k in keys:
        check(got[k], ref[k], f"{name} full {k}")


def test_autograd_wrapper_matches_the_direct_calls():
    """fl.flarepp_mixer (torch.autograd) gives the bits of flarepp_mixer_fwd and
    flarepp_mixer_bwd called directly (weight and seed gradients rounded to
    the parameters' bf16)."""
    w = make_workload("flarepp_n1k", N=512)
    X = dev_bf16(w.X).requires_grad_()
    Ws = [dev_bf16(a).requires_grad_() for a in (w.Wk, w.Wv, w.Wk_syn, w.Wv_syn)]
    Q0 = dev_bf16(w.Q0).requires_grad_()
    dY = dev_bf16(make_upstream_grad(w))
    Y = fl.flarepp_mixer(X, *Ws, Q0)
    (Y.float() * dY.float()).sum().backward()
    Y_direct = fl.flarepp_mixer_fwd(X.detach(), *[a.detach() for a in Ws], Q0.detach())
    g = fl.flarepp_mixer_bwd(X.detach(), *[a.detach() for a in Ws], Q0.detach(), dY)
    torch.cuda.synchronize()
    assert torch.equal(Y.detach().view(torch.int16), Y_direct.view(torch.int16))
    assert torch.equal(X.grad.view(torch.int16), g["dX"].view(torch.int16))
    for W, k in zip(Ws, ("dWk", "dWv", "dWk_syn", "dWv_syn")):
        assert torch.equal(W.grad.view(torch.int16), g[k].to(torch.bfloat16).view(torch.int16)), k
    assert torch.equal(Q0.grad.view(torch.int16), g["dQ0"].to(torch.bfloat16).view(torch.int16))
