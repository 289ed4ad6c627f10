"""GPU parity of the context-parallel forward (FLARE++ paper, section
"Multi-GPU context parallelism", eq. 13-14).

One GPU plays R ranks: each rank's phases run through the C ABI on its own
token shard and workspace, and every all-gather (the partials, then the exact
partials of rows whose fast-path sums underflowed) is a concatenation in rank
order.  Every rank must hold bitwise the same Q(X) and
Z, and the shards of Y together must match the fp64 oracle on the whole
sequences.  With one rank, the Python layer must reproduce flarepp_mixer_fwd
bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
import rank_latent_routing_flare_b200 as fl
from rank_latent_routing_flare_b200 import cp
from workloads import bf16_bits_to_f64, make_workload, to_bf16_bits

from .gpu_util import MAX_ABS, REL_L2, compare, dev_bf16, host_f64, max_abs, rel_l2, run_gpu
from .parity import storage_model

pytestmark = pytest.mark.gpu


def check(got, want, label):
    e_rel, e_abs = rel_l2(got, want), max_abs(got, want)
    print(label, f"rel_l2={e_rel:.3e} max_abs={e_abs:.3e}")
    assert np.all(np.isfinite(got)), label
    assert e_rel <= REL_L2 and e_abs <= MAX_ABS, (label, e_rel, e_abs)


def emulate_flarepp(w, R, exact_step=True):
    """FLARE++ over R emulated ranks: (Y, each rank's Q(X), each rank's Z);
    without the exact step, also the ranks' device statuses."""
    lib = fl.load_library()
    B, N, C, H, M, D = w.B, w.N // R, w.C, w.H, w.M, w.D
    X = dev_bf16(w.X)
    Ws = [dev_bf16(a) for a in (w.Wk, w.Wv, w.Wk_syn, w.Wv_syn)]
    Q0 = dev_bf16(w.Q0)
    lengths = None if w.lengths is None else torch.from_numpy(w.lengths).cuda()
    nbytes = fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLAREPP, B, H, N, M, D, C)
    npart = cp.partials_numel(B, H, N, M, D)
    st = torch.cuda.current_stream().cuda_stream
    Xs = [X[:, r * N:(r + 1) * N].contiguous() for r in range(R)]
    wss = [torch.empty(nbytes, dtype=torch.uint8, device="cuda") for _ in range(R)]
    parts = [torch.empty(npart, dtype=torch.float32, device="cuda") for _ in range(R)]
    lp = None if lengths is None else lengths.data_ptr()

    def common(r):
        return (B, N, C, H, M, D, lp, r, R, 0.0, wss[r].data_ptr(), nbytes, st)

    wp = [a.data_ptr() for a in Ws] + [Q0.data_ptr()]
    exact = [torch.empty(cp.exact_numel(B, H, M, D), dtype=torch.float32, device="cuda") for _ in range(R)]

    def exact_gather(pass_, gathered):
        if not exact_step:
            return None
        for r in range(R):
            assert lib.flarepp_cp_exact(pass_, gathered.data_ptr(), *wp, *common(r), exact[r].data_ptr()) == 0
        return torch.cat(exact)

    def ptr(t):
        return None if t is None else t.data_ptr()

    for r in range(R):
        assert lib.flarepp_cp_begin(Xs[r].data_ptr(), *wp, *common(r), parts[r].data_ptr()) == 0
    gathered = torch.cat(parts)
    gathered_exact = exact_gather(0, gathered)
    qxs = [torch.empty((B, H, M, D), dtype=torch.float32, device="cuda") for _ in range(R)]
    parts2 = [torch.empty_like(p) for p in parts]
    for r in range(R):
        assert lib.flarepp_cp_middle(gathered.data_ptr(), ptr(gathered_exact), *common(r), parts2[r].data_ptr(),
                                     qxs[r].data_ptr()) == 0
    gathered2 = torch.cat(parts2)
    gathered_exact2 = exact_gather(1, gathered2)
    Ys = [torch.empty((B, H, N, D), dtype=torch.bfloat16, device="cuda") for _ in range(R)]
    zs = [torch.empty((B, H, M, D), dtype=torch.float32, device="cuda") for _ in range(R)]
    for r in range(R):
        assert lib.flarepp_cp_end(gathered2.data_ptr(), ptr(gathered_exact2), Ys[r].data_ptr(), *common(r),
                                  zs[r].data_ptr()) == 0
    torch.cuda.synchronize()
    status = [fl.flare_last_device_status(wss[r]) for r in range(R)]
    if not exact_step:
        return torch.cat(Ys, dim=2), qxs, zs, status
    assert all(st_ == fl.Status.OK for st_ in status), status
    return torch.cat(Ys, dim=2), qxs, zs


CASES = [
    ("flarepp_n8k_mesh2d", {"N": 2048, "B": 2}, 2),
    ("flarepp_n1m_mesh3d", {"N": 12288}, 3),
    ("flarepp_masked_n4k", {"N": 1024, "B": 8}, 4),   # some shards hold no valid token of a sequence
]


@pytest.mark.parametrize("name,kw,R", CASES, ids=[c[0] for c in CASES])
def test_emulated_ranks_match_oracle_and_agree(name, kw, R):
    w = make_workload(name, **kw)
    Y, qxs, zs = emulate_flarepp(w, R)
    for r in range(1, R):
        assert torch.equal(qxs[r], qxs[0]) and torch.equal(zs[r], zs[0]), r
    ref = oracle.forward_workload(w)
    compare({"Y": host_f64(Y)}, {"Y": ref["Y"]}, lengths=w.lengths, label=f"cp Y {name} R={R}")
    check(host_f64(qxs[0]), ref["Qx"], f"cp Qx {name}")
    check(host_f64(zs[0]), ref["Z"], f"cp Z {name}")


def test_single_rank_equals_the_one_gpu_call():
    w = make_workload("flarepp_n8k_mesh2d", N=2048, B=2)
    X = dev_bf16(w.X)
    Ws = [dev_bf16(a) for a in (w.Wk, w.Wv, w.Wk_syn, w.Wv_syn)]
    Q0 = dev_bf16(w.Q0)
    Y1 = fl.flarepp_mixer_fwd(X, *Ws, Q0)
    Y2 = cp.flarepp_mixer_cp_fwd(X, *Ws, Q0)
    torch.cuda.synchronize()
    assert torch.equal(Y1.view(torch.int16), Y2.view(torch.int16))


def emulate_flare(w, R, exact_step=True):
    """FLARE over R emulated ranks; returns (Y of the whole sequences, the
    ranks' device statuses)."""
    lib = fl.load_library()
    B, H, N, M, D = w.B, w.H, w.N // R, w.M, w.D
    K, V, Q = dev_bf16(w.K), dev_bf16(w.V), dev_bf16(w.Q)
    Ks = [K[:, :, r * N:(r + 1) * N].contiguous() for r in range(R)]
    Vs = [V[:, :, r * N:(r + 1) * N].contiguous() for r in range(R)]
    lengths = None if w.lengths is None else torch.from_numpy(w.lengths).cuda()
    lp = None if lengths is None else lengths.data_ptr()
    nbytes = fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLARE, B, H, N, M, D)
    wss = [torch.empty(nbytes, dtype=torch.uint8, device="cuda") for _ in range(R)]
    parts = [torch.empty(cp.partials_numel(B, H, N, M, D), dtype=torch.float32, device="cuda") for _ in range(R)]
    exact = [torch.empty(cp.exact_numel(B, H, M, D), dtype=torch.float32, device="cuda") for _ in range(R)]
    st = torch.cuda.current_stream().cuda_stream
    for r in range(R):
        assert lib.flare_cp_begin(Ks[r].data_ptr(), Vs[r].data_ptr(), Q.data_ptr(), B, H, N, M, D, lp, r, R, 0.0,
                                  wss[r].data_ptr(), nbytes, st, parts[r].data_ptr()) == 0
    gathered = torch.cat(parts)
    gathered_exact = None
    if exact_step:
        for r in range(R):
            assert lib.flare_cp_exact(gathered.data_ptr(), Ks[r].data_ptr(), Vs[r].data_ptr(), Q.data_ptr(), B, H, N,
                                      M, D, lp, r, R, 0.0, wss[r].data_ptr(), nbytes, st, exact[r].data_ptr()) == 0
        gathered_exact = torch.cat(exact)
    Ys = [torch.empty_like(Ks[r]) for r in range(R)]
    for r in range(R):
        assert lib.flare_cp_end(gathered.data_ptr(), None if gathered_exact is None else gathered_exact.data_ptr(),
                                Ks[r].data_ptr(), Q.data_ptr(), Ys[r].data_ptr(), B, H, N, M, D, lp, r, R, 0.0,
                                wss[r].data_ptr(), nbytes, st, None) == 0
    torch.cuda.synchronize()
    return torch.cat(Ys, dim=2), [fl.flare_last_device_status(wss[r]) for r in range(R)]


def test_flare_emulated_ranks():
    w = make_workload("flare_n64k", N=8192, B=1)
    Y, status = emulate_flare(w, 2)
    assert all(s == fl.Status.OK for s in status)
    compare({"Y": host_f64(Y)}, {"Y": oracle.forward_workload(w)["Y"]}, lengths=w.lengths, label="cp flare")


def huge_key_case(R, seed=7):
    """FLARE with one key of huge norm in shard 0 and one in the last shard:
    the norm bound of their splits is far above the other rows' scores, so
    the fast-path sums of those splits underflow (the case the merge must
    recompute exactly, here across shards)."""
    from .test_gpu_parity import flare_case
    N = 2048 * R
    w = flare_case(2, 2, N, 32, 16, seed=seed, lengths=[N, N - 700])
    K = bf16_bits_to_f64(w.K)
    u = np.random.default_rng(1).standard_normal(16)
    K[0, 0, 5] = 2000.0 * u / np.linalg.norm(u)
    K[1, 1, N - 800] = -3000.0 * u / np.linalg.norm(u)
    w.K = to_bf16_bits(K)
    return w


@pytest.mark.parametrize("R", [2, 3])
def test_underflowing_rows_are_exact_across_shards(R):
    w = huge_key_case(R)
    Y, status = emulate_flare(w, R)
    assert all(s == fl.Status.OK for s in status), status
    compare({"Y": host_f64(Y)}, {"Y": oracle.forward_workload(w)["Y"]}, lengths=w.lengths,
            label=f"cp flare underflow R={R}")


def test_without_the_exact_step_underflow_is_reported():
    w = huge_key_case(2)
    _, status = emulate_flare(w, 2, exact_step=False)
    assert fl.Status.ERR_UNDERFLOW in status


def test_flarepp_underflowing_rows_are_exact_across_shards():
    """FLARE++ with one token of huge features in the second shard: its key
    norm inflates the shift bound of its splits, so some rows' fast-path sums
    underflow (without the exact step that is reported).  With it, every
    rank agrees and the result matches the one-GPU call, whose merge
    recomputes those rows from all keys; the one-GPU call in turn matches the
    oracle evaluated on its bf16-stored projections (the scores of the huge
    token spread over hundreds of units, so the bf16 storage alone moves the
    exact result beyond the standard tolerance)."""
    w = make_workload("flarepp_n8k_mesh2d", N=2048, B=2)
    X = bf16_bits_to_f64(w.X)
    X[1, 1500] *= 400.0
    w.X = to_bf16_bits(X)
    *_, status = emulate_flarepp(w, 2, exact_step=False)
    assert fl.Status.ERR_UNDERFLOW in status, status
    Y, qxs, zs = emulate_flarepp(w, 2)
    assert torch.equal(qxs[0], qxs[1]) and torch.equal(zs[0], zs[1])
    one = run_gpu(w)
    for name, got, want in (("Qx", host_f64(qxs[0]), one["Qx"]), ("Z", host_f64(zs[0]), one["Z"]),
                            ("Y", host_f64(Y), one["Y"])):
        e = rel_l2(got, want)
        print(f"cp flare++ underflow, 2 ranks vs one GPU: {name} rel_l2={e:.3e}")
        assert np.all(np.isfinite(got)) and e <= 1e-3, name
    model = storage_model(w, oracle)
    for name in ("Qx", "Z", "Y"):
        e = rel_l2(one[name], model[name])
        print(f"cp flare++ underflow, one GPU vs bf16 storage model: {name} rel_l2={e:.3e}")
        assert e <= REL_L2, name
