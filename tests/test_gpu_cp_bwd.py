"""GPU parity of the context-parallel FLARE++ backward (FLARE++ paper,
section "Multi-GPU context parallelism", eq. 13-14: the token-sharded encoder
and its backward).

One GPU plays R ranks: each rank runs the seven phases of
flarepp_cp_bwd_phase through the C ABI on its own token shard and workspace,
and the all-gather between two phases is a concatenation in rank order.
Checked: with one rank the phases match the fp64 oracle and flarepp_mixer_bwd
(which takes the forward's state from the forward kernels, so the two agree
to rounding, not bit for bit); with several ranks every rank holds bitwise the same weight and seed
gradients, and the gradients (dX from the shards' rows) match the fp64
oracle on the whole sequences, including a rank whose shard has no valid
token of a sample.
"""
import numpy as np
import pytest
import torch

import oracle
import rank_latent_routing_flare_b200 as fl
from workloads import make_upstream_grad, make_workload

from .gpu_util import dev_bf16, host_f64, rel_l2

pytestmark = pytest.mark.gpu

PHASES = 7
KEYS = ("dX", "dWk", "dWv", "dWk_syn", "dWv_syn", "dQ0")


def check(got, ref, label, bound=5e-3):
    r = rel_l2(got, ref)
    m = float(np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-30))
    print(f"{label}: rel_l2={r:.3e} max_err/max_ref={m:.3e}")
    assert r <= bound and m <= 3e-2, (label, r, m)


def emulate(w, dY, R):
    lib = fl.load_library()
    B, N, C, H, M, D = w.B, w.N // R, w.C, w.H, w.M, w.D
    X, dYd = dev_bf16(w.X), dev_bf16(dY)
    Ws = [dev_bf16(a) for a in (w.Wk, w.Wv, w.Wk_syn, w.Wv_syn)]
    Q0 = dev_bf16(w.Q0)
    lengths = None if w.lengths is None else torch.from_numpy(w.lengths).cuda()
    lp = None if lengths is None else lengths.data_ptr()
    nbytes = fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLAREPP_BWD, B, H, N, M, D, C)
    st = torch.cuda.current_stream().cuda_stream
    Xs = [X[:, r * N:(r + 1) * N].contiguous() for r in range(R)]
    dYs = [dYd[:, :, r * N:(r + 1) * N].contiguous() for r in range(R)]
    wss = [torch.empty(nbytes, dtype=torch.uint8, device="cuda") for _ in range(R)]
    outs = [{"dX": torch.empty((B, N, C), dtype=torch.bfloat16, device="cuda"),
             **{k: torch.empty((C, C), dtype=torch.float32, device="cuda") for k in KEYS[1:5]},
             "dQ0": torch.empty((H, M, D), dtype=torch.float32, device="cuda")} for _ in range(R)]
    gathered = None
    for phase in range(PHASES):
        exch = [None] * R
        if phase < PHASES - 1:
            nb = lib.flarepp_cp_bwd_exchange_bytes(phase, B, N, C, H, M, D)
            assert nb > 0
            exch = [torch.empty(nb // 4, dtype=torch.float32, device="cuda") for _ in range(R)]
        for r in range(R):
            rc = lib.flarepp_cp_bwd_phase(
                phase, Xs[r].data_ptr(), *[a.data_ptr() for a in Ws], Q0.data_ptr(), dYs[r].data_ptr(),
                None if gathered is None else gathered.data_ptr(), None if exch[r] is None else exch[r].data_ptr(),
                *[outs[r][k].data_ptr() for k in KEYS], B, N, C, H, M, D, lp, r, R, 0.0, wss[r].data_ptr(), nbytes,
                st)
            assert rc == 0, (phase, r, rc)
        if phase < PHASES - 1:
            gathered = torch.cat(exch)
    torch.cuda.synchronize()
    for r in range(R):
        assert fl.flare_last_device_status(wss[r]) == fl.Status.OK
    return outs


def test_one_rank_matches_the_single_gpu_backward():
    w = make_workload("flarepp_n1k", N=900)
    dY = make_upstream_grad(w)
    outs = emulate(w, dY, 1)[0]
    g = fl.flarepp_mixer_bwd(dev_bf16(w.X), dev_bf16(w.Wk), dev_bf16(w.Wv), dev_bf16(w.Wk_syn),
                             dev_bf16(w.Wv_syn), dev_bf16(w.Q0), dev_bf16(dY))
    torch.cuda.synchronize()
    ref = oracle.backward_workload(w, dY)
    for k in KEYS:
        check(host_f64(outs[k]), ref[k], f"one rank {k} vs oracle")
        check(host_f64(outs[k]), host_f64(g[k]), f"one rank {k} vs flarepp_mixer_bwd")


@pytest.mark.parametrize("name,N,B,R,lengths", [
    ("flarepp_n1k", 1024, 1, 2, None),
    ("flarepp_n8k_mesh2d", 1536, 2, 3, [1536, 700]),      # rank 2 holds no valid token of sample 1
    ("flarepp_masked_n4k", 512, 2, 4, [512, 77]),         # D = 32; ranks 1-3 empty for sample 1
])
def test_sharded_backward_matches_oracle(name, N, B, R, lengths):
    w = make_workload(name, N=N, B=B, lengths=None if lengths is None else np.array(lengths, dtype=np.int32))
    dY = make_upstream_grad(w)
    outs = emulate(w, dY, R)
    for r in range(1, R):
        for k in KEYS[1:]:
            assert torch.equal(outs[r][k], outs[0][k]), (r, k)
    got = {k: host_f64(outs[0][k]) for k in KEYS[1:]}
    got["dX"] = np.concatenate([host_f64(outs[r]["dX"]) for r in range(R)], axis=1)
    ref = oracle.backward_workload(w, dY)
    for k in KEYS:
        check(got[k], ref[k], f"{name} R={R} {k}")
    if lengths is not None:
        for b, L in enumerate(lengths):
            assert np.all(got["dX"][b, L:] == 0)


# ---------------------------------------------------------------------------
# FLARE (fixed queries): four phases of flare_cp_bwd_phase
# ---------------------------------------------------------------------------

FL_PHASES = 4


def flare_case(B, H, N, M, D, seed, lengths=None):
    from workloads import Workload, to_bf16_bits
    rng = np.random.default_rng(seed)
    w = Workload(name="flare_cp_bwd", variant="flare", B=B, H=H, N=N, C=H * D, D=D, M=M, seed=seed)
    w.K = to_bf16_bits(rng.standard_normal((B, H, N, D)))
    w.V = to_bf16_bits(rng.standard_normal((B, H, N, D)))
    w.Q = to_bf16_bits(rng.standard_normal((H, M, D)))
    w.lengths = None if lengths is None else np.asarray(lengths, np.int32)
    return w


def emulate_flare(w, dY, R):
    lib = fl.load_library()
    B, H, N, M, D = w.B, w.H, w.N // R, w.M, w.D
    K, V, Q, dYd = dev_bf16(w.K), dev_bf16(w.V), dev_bf16(w.Q), dev_bf16(dY)
    lengths = None if w.lengths is None else torch.from_numpy(w.lengths).cuda()
    lp = None if lengths is None else lengths.data_ptr()
    nbytes = fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLARE_BWD, B, H, N, M, D)
    st = torch.cuda.current_stream().cuda_stream
    shard = lambda t, r: t[:, :, r * N:(r + 1) * N].contiguous()  # noqa: E731
    Ks, Vs, dYs = [shard(K, r) for r in range(R)], [shard(V, r) for r in range(R)], [shard(dYd, r) for r in range(R)]
    wss = [torch.empty(nbytes, dtype=torch.uint8, device="cuda") for _ in range(R)]
    outs = [{"dK": torch.empty_like(Ks[r]), "dV": torch.empty_like(Ks[r]),
             "dQ": torch.empty((H, M, D), dtype=torch.float32, device="cuda")} for r in range(R)]
    gathered = None
    for phase in range(FL_PHASES):
        exch = [None] * R
        if phase < FL_PHASES - 1:
            nb = lib.flare_cp_bwd_exchange_bytes(phase, B, H, N, M, D)
            assert nb > 0
            exch = [torch.empty(nb // 4, dtype=torch.float32, device="cuda") for _ in range(R)]
        for r in range(R):
            rc = lib.flare_cp_bwd_phase(
                phase, Ks[r].data_ptr(), Vs[r].data_ptr(), Q.data_ptr(), dYs[r].data_ptr(),
                None if gathered is None else gathered.data_ptr(), None if exch[r] is None else exch[r].data_ptr(),
                outs[r]["dK"].data_ptr(), outs[r]["dV"].data_ptr(), outs[r]["dQ"].data_ptr(), B, H, N, M, D, lp, r, R,
                0.0, wss[r].data_ptr(), nbytes, st)
            assert rc == 0, (phase, r, rc)
        if phase < FL_PHASES - 1:
            gathered = torch.cat(exch)
    torch.cuda.synchronize()
    for r in range(R):
        assert fl.flare_last_device_status(wss[r]) == fl.Status.OK
    return outs


def test_flare_one_rank_matches_the_single_gpu_backward():
    w = flare_case(2, 2, 1000, 64, 16, seed=5, lengths=[1000, 613])
    dY = make_upstream_grad(w)
    outs = emulate_flare(w, dY, 1)[0]
    lengths = torch.from_numpy(w.lengths).cuda()
    dK, dV, dQ = fl.flare_mixer_bwd(dev_bf16(w.K), dev_bf16(w.V), dev_bf16(w.Q), dev_bf16(dY), lengths=lengths)
    torch.cuda.synchronize()
    ref = oracle.backward_workload(w, dY)
    for k, single in (("dK", dK), ("dV", dV), ("dQ", dQ)):
        check(host_f64(outs[k]), ref[k], f"flare one rank {k} vs oracle")
        check(host_f64(outs[k]), host_f64(single), f"flare one rank {k} vs flare_mixer_bwd")
    for b, L in enumerate(w.lengths):
        assert torch.all(outs["dK"][b, :, L:] == 0) and torch.all(dK[b, :, L:] == 0)


@pytest.mark.parametrize("B,H,N,M,D,R,lengths", [
    (2, 2, 2048, 64, 16, 2, None),
    (2, 3, 1536, 128, 16, 3, [1536, 500]),      # ranks 1 and 2 hold no valid token of sample 1
    (1, 2, 1024, 96, 32, 4, None),              # D = 32
])
def test_flare_sharded_backward_matches_oracle(B, H, N, M, D, R, lengths):
    w = flare_case(B, H, N, M, D, seed=N + R, lengths=lengths)
    dY = make_upstream_grad(w)
    outs = emulate_flare(w, dY, R)
    for r in range(1, R):
        assert torch.equal(outs[r]["dQ"], outs[0]["dQ"]), r
    got = {"dK": np.concatenate([host_f64(outs[r]["dK"]) for r in range(R)], axis=2),
           "dV": np.concatenate([host_f64(outs[r]["dV"]) for r in range(R)], axis=2),
           "dQ": host_f64(outs[0]["dQ"])}
    ref = oracle.backward_workload(w, dY)
    for k in ("dK", "dV", "dQ"):
        check(got[k], ref[k], f"flare {B}x{H}x{N} M={M} D={D} R={R} {k}")
    if lengths is not None:
        for b, L in enumerate(lengths):
            assert np.all(got["dK"][b, :, L:] == 0) and np.all(got["dV"][b, :, L:] == 0)
