"""The entry point for callers that cannot allocate device memory.

Some callers are not allowed to call cudaMalloc themselves: code that runs
where device allocation is forbidden, or that must keep its footprint fixed.
flare_mixer_fwd_static serves them: it takes the same arguments as
flare_mixer_fwd minus the workspace and uses the library's fixed device
scratch instead.  These tests call it through the C ABI and check that it
gives what the workspace entry point gives, on two calls in a row (the
scratch keeps the previous call's contents, so the second call checks that
every word that must start at zero is cleared).  This file is collected last
so that a run stopping at the first failure has run every other test first.
"""
import ctypes

import numpy as np
import pytest
import torch

import rank_latent_routing_flare_b200 as fl
from workloads import Workload, to_bf16_bits

from .gpu_util import MAX_ABS, REL_L2, host_f64, max_abs, rel_l2

pytestmark = pytest.mark.gpu


def _case(B=2, H=3, N=3000, M=128, D=16, seed=3):
    rng = np.random.default_rng(seed)
    w = Workload(name="no_alloc", variant="flare", B=B, H=H, N=N, C=H * D, D=D, M=M, seed=seed)
    dev = lambda a: torch.from_numpy(to_bf16_bits(a).view(np.int16)).view(torch.bfloat16).cuda()  # noqa: E731
    K = dev(rng.standard_normal((B, H, N, D)))
    V = dev(rng.standard_normal((B, H, N, D)))
    Q = dev(rng.standard_normal((H, M, D)))
    lengths = torch.tensor([N, N - 517][:B], dtype=torch.int32, device="cuda")
    return w, K, V, Q, lengths


def test_static_scratch_matches_workspace_entry_point_twice():
    w, K, V, Q, lengths = _case()
    assert fl.flare_workspace_bytes(0, w.B, w.H, w.N, w.M, w.D) <= fl._binding.FLARE_STATIC_SCRATCH_BYTES
    ref = host_f64(fl.flare_mixer_fwd(K, V, Q, lengths=lengths))
    lib = fl.load_library()
    stream = torch.cuda.current_stream()
    for call in range(2):
        Y = torch.full_like(K, float("nan"))
        Z = torch.full((w.B, w.H, w.M, w.D), float("nan"), dtype=torch.float32, device="cuda")
        st = lib.flare_mixer_fwd_static(K.data_ptr(), V.data_ptr(), Q.data_ptr(), Y.data_ptr(), w.B, w.H, w.N,
                                        w.M, w.D, lengths.data_ptr(), ctypes.c_float(0.0),
                                        ctypes.c_void_p(stream.cuda_stream), Z.data_ptr())
        assert st == 0, fl.flare_status_string(st)
        torch.cuda.synchronize()
        y = host_f64(Y)
        assert np.all(np.isfinite(y)) and np.all(np.isfinite(host_f64(Z))), f"call {call}"
        assert rel_l2(y, ref) <= REL_L2 and max_abs(y, ref) <= MAX_ABS, f"call {call}"


def test_static_scratch_refuses_sizes_beyond_its_limit():
    K = torch.empty(16, dtype=torch.bfloat16, device="cuda")
    lib = fl.load_library()
    st = lib.flare_mixer_fwd_static(K.data_ptr(), K.data_ptr(), K.data_ptr(), K.data_ptr(), 64, 8, 1 << 20, 512,
                                    16, None, ctypes.c_float(0.0), None, None)
    assert st == fl.Status.ERR_WORKSPACE
