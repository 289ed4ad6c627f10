"""Parity of the CUDA path (through the C ABI) with the fp64 oracle.

Tolerance on Y (bf16 output, fp32 accumulation): relative L2 <= 5e-3 and
max-abs <= 3e-2; the fp32 diagnostics Q(X) and Z are held to the same relative
L2.  Cases span several tiles and ragged tails, every named workload (reduced
and at full size, the 1M-token one on sampled rows), key padding, the
degenerate cases (one token, one latent block, M = 16, M = 512), the exact
fallback for underflowing rows, determinism and the device error paths.
"""
import numpy as np
import pytest
import torch

import oracle
import rank_latent_routing_flare_b200 as fl
from rank_latent_routing_flare_b200 import Status
from workloads import Workload, bf16_bits_to_f64, make_workload, to_bf16_bits

from .gpu_util import compare, dev_bf16, host_f64, run_gpu
from .parity import storage_model

pytestmark = pytest.mark.gpu


def flare_case(B, H, N, M, D, seed=0, qscale=1.0, lengths=None):
    rng = np.random.default_rng(seed)
    w = Workload(name="flare_case", variant="flare", B=B, H=H, N=N, C=H * D, D=D, M=M, seed=seed)
    w.K = to_bf16_bits(rng.standard_normal((B, H, N, D)))
    w.V = to_bf16_bits(rng.standard_normal((B, H, N, D)))
    w.Q = to_bf16_bits(rng.standard_normal((H, M, D)) * qscale)
    w.lengths = None if lengths is None else np.asarray(lengths, np.int32)
    return w


# ---------------------------------------------------------------------------
# device error paths
# ---------------------------------------------------------------------------

def test_bounded_wait_expires_and_reports_timeout():
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    fl.flare_selftest_wait_timeout(ws, 200_000)          # 0.2 ms
    assert fl.flare_last_device_status(ws) == Status.ERR_TIMEOUT
    # the context is still usable afterwards
    w = flare_case(1, 1, 300, 32, 16)
    compare(run_gpu(w), oracle.forward_workload(w), label="after-timeout")


def test_invalid_length_is_reported():
    w = flare_case(2, 1, 256, 32, 16, lengths=[0, 256])
    K, V, Q = dev_bf16(w.K), dev_bf16(w.V), dev_bf16(w.Q)
    lengths = torch.tensor([0, 256], dtype=torch.int32, device="cuda")
    ws = torch.empty(fl.flare_workspace_bytes(0, 2, 1, 256, 32, 16), dtype=torch.uint8, device="cuda")
    Y = fl.flare_mixer_fwd(K, V, Q, lengths=lengths, workspace=ws)
    assert fl.flare_last_device_status(ws) == Status.ERR_SHAPE
    ref = oracle.forward_workload(w)
    assert np.all(host_f64(Y)[0] == 0)                  # clamped to length 0: all padding
    compare({"Y": host_f64(Y)[1:]}, {"Y": ref["Y"][1:]}, label="valid-sample")


# ---------------------------------------------------------------------------
# special values: isolate the score MMA from the value MMA
# ---------------------------------------------------------------------------

def test_unit_values_give_unit_outputs():
    """V = 1: each split's value column equals its sum column, so Z = 1 and Y = 1
    whatever the scores are."""
    w = flare_case(2, 2, 1000, 64, 16)
    w.V = to_bf16_bits(np.ones((2, 2, 1000, 16)))
    g = run_gpu(w)
    assert np.max(np.abs(g["Z"] - 1.0)) < 1e-6
    assert np.max(np.abs(g["Y"] - 1.0)) == 0.0


@pytest.mark.parametrize("D", [16, 32])
def test_zero_queries_give_token_means(D):
    w = flare_case(1, 2, 777, 32, D)
    w.Q = to_bf16_bits(np.zeros((2, 32, D)))
    g = run_gpu(w)
    mean = bf16_bits_to_f64(w.V).mean(axis=2, keepdims=True)
    assert np.max(np.abs(g["Z"] - mean)) < 1e-5
    assert np.max(np.abs(g["Y"] - mean)) < 1e-2


# ---------------------------------------------------------------------------
# FLARE (keys, values and queries given)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("B,H,N,M,D", [
    (2, 2, 1000, 32, 16),      # ragged tail, M below one latent block
    (1, 3, 777, 64, 16),
    (1, 2, 4096, 256, 16),     # two latent blocks
    (2, 1, 3000, 512, 16),     # four latent blocks, eight decode chunks
    (1, 2, 1500, 128, 32),     # D = 32
    (3, 2, 200, 144, 32),      # a 16-row partial latent block and decode chunk
    (1, 1, 1, 16, 16),         # one token, smallest M
    (1, 1, 65, 48, 16),        # one full tile + 1 token; 48-latent chunk
    (1, 2, 777, 512, 32),      # D = 32 with the largest M: eight 64-latent decoder chunks
    (2, 3, 130, 80, 32),       # D = 32, a short last decoder chunk (16 latents)
])
def test_flare_parity(B, H, N, M, D):
    w = flare_case(B, H, N, M, D, seed=B * 1000 + N)
    compare(run_gpu(w), oracle.forward_workload(w), label=f"flare {B}x{H}x{N} M={M} D={D}")


def test_flare_masked_edges():
    N = 700
    w = flare_case(5, 2, N, 64, 16, lengths=[1, N, N - 1, 64, 65])
    compare(run_gpu(w), oracle.forward_workload(w), label="flare masked")


def test_underflow_rows_use_exact_fallback():
    """One key with a huge norm makes the Cauchy-Schwarz shift of its split (and
    of its own decode row) far too loose; those rows must fall back to the exact
    two-pass softmax and still match the oracle."""
    w = flare_case(1, 2, 2000, 32, 16, seed=7)
    K = bf16_bits_to_f64(w.K)
    u = np.random.default_rng(1).standard_normal(16)
    K[0, 0, 5] = 2000.0 * u / np.linalg.norm(u)
    K[0, 1, 1999] = -3000.0 * u / np.linalg.norm(u)
    w.K = to_bf16_bits(K)
    compare(run_gpu(w), oracle.forward_workload(w), label="fallback")


# ---------------------------------------------------------------------------
# FLARE++ named workloads
# ---------------------------------------------------------------------------

REDUCED = [
    ("flarepp_n1k", {}),
    ("flarepp_n8k_mesh2d", {"N": 2048, "B": 2}),
    ("flarepp_n64k", {"N": 8192, "B": 1}),
    ("flare_n64k", {"N": 8192, "B": 1}),
    ("flarepp_n1m_mesh3d", {"N": 16384}),
    ("flarepp_masked_n4k", {"N": 1024, "B": 8}),
]


@pytest.mark.parametrize("name,kw", REDUCED, ids=[r[0] for r in REDUCED])
def test_workload_reduced(name, kw):
    w = make_workload(name, **kw)
    compare(run_gpu(w), oracle.forward_workload(w), label=f"{name} {kw}")


def test_sharp_scores_match_bf16_storage_model():
    """Diagnostic with all weights ~ N(0, 16/C): encode/decode scores spread
    over tens of units and many tokens sit near ties between latents with very
    different values, so the result is ill-conditioned at bf16 precision.  The
    bf16 storage of the projected keys and values alone moves the exact result
    by ~2e-2 (relative L2), and any re-rounding of Q(X) or Z flips the near
    ties either way.  Checked: the synthesised queries (before any
    amplification) match the storage model to the standard tolerance, and the
    output is no further from the exact oracle than 1.5x the storage model's
    own distance plus the standard tolerance."""
    from .gpu_util import REL_L2, rel_l2
    w = make_workload("flarepp_n8k_sharp", N=2048, B=2)
    g = run_gpu(w)
    model = storage_model(w, oracle)
    exact = oracle.forward_workload(w)
    assert rel_l2(g["Qx"], model["Qx"]) <= REL_L2
    storage_err = rel_l2(model["Y"], exact["Y"])
    gpu_err = rel_l2(g["Y"], exact["Y"])
    print("sharp: storage model vs exact %.3e, gpu vs exact %.3e" % (storage_err, gpu_err))
    assert np.all(np.isfinite(g["Y"]))
    assert gpu_err <= 1.5 * storage_err + REL_L2


FULL = ["flarepp_n1k", "flarepp_n8k_mesh2d", "flare_n64k", "flarepp_n64k", "flarepp_masked_n4k"]


@pytest.mark.parametrize("name", FULL)
def test_workload_full_size(name):
    w = make_workload(name)
    compare(run_gpu(w), oracle.forward_workload(w), label=f"{name} full")


def test_million_token_workload_sampled_rows():
    """N = 1,048,576: the oracle computes Q(X) and Z over every token and Y on
    4096 sampled tokens (plus the first and last ones)."""
    w = make_workload("flarepp_n1m_mesh3d")
    rng = np.random.default_rng(0)
    rows = np.unique(np.concatenate([[0, 1, w.N - 1], rng.choice(w.N, 4096, replace=False)]))
    g = run_gpu(w)
    ref = oracle.forward_workload(w, rows=rows)
    compare(g, ref, rows=rows, label="n1m sampled")


def test_deterministic_bits():
    w = make_workload("flarepp_n64k", N=4096, B=2)
    a = run_gpu(w)
    b = run_gpu(w)
    assert np.array_equal(a["Y"], b["Y"])
    assert np.array_equal(a["Qx"], b["Qx"]) and np.array_equal(a["Z"], b["Z"])


def test_cuda_graph_capture_replays_the_same_bits():
    """A whole FLARE++ call can be captured into a CUDA graph (it only enqueues
    kernels and a memset on the given stream) and replayed with new inputs."""
    w = make_workload("flarepp_n8k_mesh2d", N=2048, B=2)
    X = dev_bf16(w.X)
    Ws = [dev_bf16(a) for a in (w.Wk, w.Wv, w.Wk_syn, w.Wv_syn)]
    Q0 = dev_bf16(w.Q0)
    nbytes = fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLAREPP, w.B, w.H, w.N, w.M, w.D, w.C)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    Y = torch.empty((w.B, w.H, w.N, w.D), dtype=torch.bfloat16, device="cuda")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        fl.flarepp_mixer_fwd(X, *Ws, Q0, Y=Y, workspace=ws)   # first call outside the capture
        torch.cuda.synchronize()
        eager = Y.clone()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            fl.flarepp_mixer_fwd(X, *Ws, Q0, Y=Y, workspace=ws, check=False)
    Y.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(Y.view(torch.int16), eager.view(torch.int16))
    # new inputs in the same buffers
    w2 = make_workload("flarepp_n8k_mesh2d", N=2048, B=2, seed=77)
    w2.Wk, w2.Wv, w2.Wk_syn, w2.Wv_syn, w2.Q0 = w.Wk, w.Wv, w.Wk_syn, w.Wv_syn, w.Q0   # only X changes
    X.copy_(dev_bf16(w2.X))
    g.replay()
    torch.cuda.synchronize()
    compare({"Y": host_f64(Y)}, oracle.forward_workload(w2), label="graph replay")
    del g
