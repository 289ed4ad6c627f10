"""GPU parity of the context-parallel forward (FLARE++ paper, section
"Multi-GPU context parallelism", eq. 13-14).

One GPU plays R ranks: each rank's phases run through the C ABI on its own
token shard and workspace, and the all-gather of the partials is a
concatenation in rank order.  Every rank must hold bitwise the same Q(X) and
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
from workloads import make_workload

from .gpu_util import MAX_ABS, REL_L2, compare, dev_bf16, host_f64, max_abs, rel_l2

pytestmark = pytest.mark.gpu


def check(got, want, label):
    e_rel, e_abs = rel_l2(got, want), max_abs(got, want)
    print(label, f"rel_l2={e_rel:.3e} max_abs={e_abs:.3e}")
    assert np.all(np.isfinite(got)), label
    assert e_rel <= REL_L2 and e_abs <= MAX_ABS, (label, e_rel, e_abs)


def emulate_flarepp(w, R):
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

    for r in range(R):
        assert lib.flarepp_cp_begin(Xs[r].data_ptr(), *[a.data_ptr() for a in Ws], Q0.data_ptr(), *common(r),
                                    parts[r].data_ptr()) == 0
    gathered = torch.cat(parts)
    qxs = [torch.empty((B, H, M, D), dtype=torch.float32, device="cuda") for _ in range(R)]
    parts2 = [torch.empty_like(p) for p in parts]
    for r in range(R):
        assert lib.flarepp_cp_middle(gathered.data_ptr(), *common(r), parts2[r].data_ptr(), qxs[r].data_ptr()) == 0
    gathered2 = torch.cat(parts2)
    Ys = [torch.empty((B, H, N, D), dtype=torch.bfloat16, device="cuda") for _ in range(R)]
    zs = [torch.empty((B, H, M, D), dtype=torch.float32, device="cuda") for _ in range(R)]
    for r in range(R):
        assert lib.flarepp_cp_end(gathered2.data_ptr(), Ys[r].data_ptr(), *common(r), zs[r].data_ptr()) == 0
    torch.cuda.synchronize()
    for r in range(R):
        assert fl.flare_last_device_status(wss[r]) == fl.Status.OK
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


def test_flare_emulated_ranks():
    w = make_workload("flare_n64k", N=8192, B=1)
    R = 2
    lib = fl.load_library()
    B, H, N, M, D = w.B, w.H, w.N // R, w.M, w.D
    K, V, Q = dev_bf16(w.K), dev_bf16(w.V), dev_bf16(w.Q)
    Ks = [K[:, :, r * N:(r + 1) * N].contiguous() for r in range(R)]
    Vs = [V[:, :, r * N:(r + 1) * N].contiguous() for r in range(R)]
    nbytes = fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLARE, B, H, N, M, D)
    wss = [torch.empty(nbytes, dtype=torch.uint8, device="cuda") for _ in range(R)]
    parts = [torch.empty(cp.partials_numel(B, H, N, M, D), dtype=torch.float32, device="cuda") for _ in range(R)]
    st = torch.cuda.current_stream().cuda_stream
    for r in range(R):
        assert lib.flare_cp_begin(Ks[r].data_ptr(), Vs[r].data_ptr(), Q.data_ptr(), B, H, N, M, D, None, r, R, 0.0,
                                  wss[r].data_ptr(), nbytes, st, parts[r].data_ptr()) == 0
    gathered = torch.cat(parts)
    Ys = [torch.empty_like(Ks[r]) for r in range(R)]
    for r in range(R):
        assert lib.flare_cp_end(gathered.data_ptr(), Ks[r].data_ptr(), Q.data_ptr(), Ys[r].data_ptr(), B, H, N, M, D,
                                None, r, R, 0.0, wss[r].data_ptr(), nbytes, st, None) == 0
    torch.cuda.synchronize()
    compare({"Y": host_f64(torch.cat(Ys, dim=2))}, {"Y": oracle.forward_workload(w)["Y"]}, lengths=w.lengths,
            label="cp flare")
