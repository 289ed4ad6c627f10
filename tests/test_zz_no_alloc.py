"""The entry point for callers that cannot allocate device memory.

Some callers are not allowed to call cudaMalloc themselves: code that runs
where device allocation is forbidden, or that must keep its footprint fixed.
flare_mixer_fwd_static serves them: it takes the same arguments as
flare_mixer_fwd minus the workspace and uses the library's fixed device
scratch instead.  These tests call it through the C ABI and check that it
gives what the workspace entry point gives, and what the fp64 oracle gives,
on two calls in a row (the scratch keeps the previous call's contents, so the
second call checks that every word that must start at zero is cleared), and
that a length outside [1, N] is reported through the static scratch's error
word (flare_static_last_device_status) and cleared by the next call.  This file is collected last
so that a run stopping at the first failure has run every other test first.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import rank_latent_routing_flare_b200 as fl
from workloads import Workload, to_bf16_bits

from .gpu_util import MAX_ABS, REL_L2, compare, host_f64, max_abs, rel_l2

pytestmark = pytest.mark.gpu


def _case(B=2, H=3, N=3000, M=128, D=16, seed=3):
    rng = np.random.default_rng(seed)
    w = Workload(name="no_alloc", variant="flare", B=B, H=H, N=N, C=H * D, D=D, M=M, seed=seed)
    w.K = to_bf16_bits(rng.standard_normal((B, H, N, D)))
    w.V = to_bf16_bits(rng.standard_normal((B, H, N, D)))
    w.Q = to_bf16_bits(rng.standard_normal((H, M, D)))
    w.lengths = np.array([N, N - 517][:B], dtype=np.int32)
    dev = lambda a: torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).cuda()  # noqa: E731
    lengths = torch.from_numpy(w.lengths).cuda()
    return w, dev(w.K), dev(w.V), dev(w.Q), lengths


def _static_call(lib, K, V, Q, Y, Z, w, lengths):
    stream = torch.cuda.current_stream()
    return lib.flare_mixer_fwd_static(K.data_ptr(), V.data_ptr(), Q.data_ptr(), Y.data_ptr(), w.B, w.H, w.N,
                                      w.M, w.D, lengths.data_ptr(), ctypes.c_float(0.0),
                                      ctypes.c_void_p(stream.cuda_stream), None if Z is None else Z.data_ptr())


def test_static_scratch_matches_workspace_entry_point_twice():
    w, K, V, Q, lengths = _case()
    assert fl.flare_workspace_bytes(0, w.B, w.H, w.N, w.M, w.D) <= fl._binding.FLARE_STATIC_SCRATCH_BYTES
    ref = host_f64(fl.flare_mixer_fwd(K, V, Q, lengths=lengths))
    exact = oracle.forward_workload(w)
    lib = fl.load_library()
    for call in range(2):
        Y = torch.full_like(K, float("nan"))
        Z = torch.full((w.B, w.H, w.M, w.D), float("nan"), dtype=torch.float32, device="cuda")
        st = _static_call(lib, K, V, Q, Y, Z, w, lengths)
        assert st == 0, fl.flare_status_string(st)
        assert fl.flare_static_last_device_status() == fl.Status.OK
        y = host_f64(Y)
        assert np.all(np.isfinite(y)) and np.all(np.isfinite(host_f64(Z))), f"call {call}"
        assert rel_l2(y, ref) <= REL_L2 and max_abs(y, ref) <= MAX_ABS, f"call {call}"
        compare({"Y": y, "Z": host_f64(Z)}, exact, lengths=w.lengths, label=f"static call {call} vs oracle")


def test_static_scratch_reports_a_bad_length_and_clears_it():
    w, K, V, Q, lengths = _case(B=2, H=1, N=700, M=64)
    lib = fl.load_library()
    bad = torch.tensor([0, w.N], dtype=torch.int32, device="cuda")
    Y = torch.empty_like(K)
    assert _static_call(lib, K, V, Q, Y, None, w, bad) == 0
    assert fl.flare_static_last_device_status() == fl.Status.ERR_SHAPE
    y = host_f64(Y)
    assert np.all(y[0] == 0)  # clamped to length 0: all padding
    w.lengths = np.array([w.N, w.N], dtype=np.int32)
    ref = oracle.forward_workload(w)
    compare({"Y": y[1:]}, {"Y": ref["Y"][1:]}, label="static, valid sample next to a bad one")
    # the next call clears the word
    assert _static_call(lib, K, V, Q, Y, None, w, lengths) == 0
    assert fl.flare_static_last_device_status() == fl.Status.OK


def test_static_scratch_refuses_sizes_beyond_its_limit():
    K = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    lib = fl.load_library()
    st = lib.flare_mixer_fwd_static(K.data_ptr(), K.data_ptr(), K.data_ptr(), K.data_ptr(), 64, 8, 1 << 20, 512,
                                    16, None, ctypes.c_float(0.0), None, None)
    assert st == fl.Status.ERR_WORKSPACE
