"""Host-only checks of the C ABI (no GPU needed, no kernel is launched).

The library must load on a machine without a GPU, export every function that
include/flare.h declares, size workspaces from the shapes alone and reject
invalid arguments on the host, before anything is enqueued.
"""
import ctypes
import os
import re

import pytest

import rank_latent_routing_flare_b200 as fl
from rank_latent_routing_flare_b200 import Status

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "flare.h")

# fake, 256-byte aligned "device" addresses: never dereferenced, because every
# call below fails validation before it touches CUDA
A = 0x10000
W = 0x20000


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"FLARE_API\s+[\w\s\*]+?\b(flare\w*)\s*\(", text)))


def test_header_declares_the_abi():
    names = declared_functions()
    assert names == sorted(["flare_workspace_bytes", "flare_mixer_fwd", "flarepp_mixer_fwd", "flarepp_mixer_out_fwd",
                            "flare_mixer_fwd_profiled", "flarepp_mixer_fwd_profiled", "flare_mixer_fwd_static",
                            "flare_last_device_status", "flare_status_string",
                            "flare_selftest_wait_timeout", "flare_cp_partials_bytes", "flarepp_cp_begin",
                            "flarepp_cp_middle", "flarepp_cp_end", "flare_cp_begin", "flare_cp_end",
                            "flare_cp_exact_bytes", "flarepp_cp_exact", "flare_cp_exact",
                            "flare_cp_bwd_exchange_bytes", "flare_cp_bwd_phase",
                            "flare_mixer_bwd", "flarepp_mixer_bwd", "flarepp_cp_bwd_exchange_bytes",
                            "flarepp_cp_bwd_phase", "flare_mixer_fwd_inspect", "flarepp_mixer_fwd_inspect",
                            "flare_static_last_device_status", "flare_probe_scratch_bytes",
                            "flare_probe_pipe_rates", "flarepp_mixer_fwd_train", "flarepp_mixer_bwd_train",
                            "flare_mixer_fwd_train", "flare_mixer_bwd_train"])


def test_library_loads_and_exports_every_declared_symbol():
    lib = fl.load_library()
    for name in declared_functions():
        assert hasattr(lib, name), name
    out = os.popen(f"nm -D --defined-only {fl.library_path()}").read()
    exported = set(re.findall(r"\bT (\w+)", out))
    assert set(declared_functions()) <= exported
    # nothing else leaks out of the library except the C ABI
    assert all(e.startswith("flare") or e.startswith("_") for e in exported), exported


def test_library_needs_no_libcuda_at_load_time():
    out = os.popen(f"ldd {fl.library_path()}").read()
    assert "libcuda.so" not in out and "libcudart" not in out


def test_status_strings():
    for s in Status:
        txt = fl.flare_status_string(int(s))
        assert txt.startswith("FLARE_" if s else "FLARE_OK")
    assert "unknown" in fl.flare_status_string(99)


@pytest.mark.parametrize("cfg", [
    (1, 4, 1024, 32, 16, 64, 1),
    (1, 8, 8192, 64, 16, 128, 8),
    (0, 8, 65536, 256, 16, 128, 4),
    (1, 8, 65536, 256, 16, 128, 4),
    (1, 8, 1048576, 512, 16, 128, 1),
    (1, 8, 4096, 128, 32, 256, 32),
])
def test_workspace_sizes(cfg):
    variant, H, N, M, D, C, B = cfg
    n = fl.flare_workspace_bytes(variant, B, H, N, M, D, C)
    proj = B * H * N * D * 2
    lat = B * H * M * D * 4
    assert n > 0 and n % 256 == 0
    if variant == 1:
        assert n >= 4 * proj + 2 * lat      # K~, V~, K, V and the fp32 Q(X), Z
    else:
        assert n >= lat
    # shape-only: the same question always gets the same answer
    assert n == fl.flare_workspace_bytes(variant, B, H, N, M, D, C)


def test_workspace_unsupported_sizes_return_zero():
    assert fl.flare_workspace_bytes(0, 1, 1, 64, 32, 8, 0) == 0        # D not in {16, 32}
    assert fl.flare_workspace_bytes(0, 1, 1, 64, 24, 16, 0) == 0       # M not a multiple of 16
    assert fl.flare_workspace_bytes(0, 1, 1, 64, 528, 16, 0) == 0      # M > 512
    assert fl.flare_workspace_bytes(1, 1, 2, 64, 32, 16, 48) == 0      # C != H*D
    assert fl.flare_workspace_bytes(1, 1, 3, 64, 32, 16, 48) == 0      # C not a multiple of 64
    assert fl.flare_workspace_bytes(5, 1, 1, 64, 32, 16, 64) == 0      # bad variant
    assert fl.flare_workspace_bytes(-1, 1, 1, 64, 32, 16, 64) == 0     # bad variant
    assert fl.flare_workspace_bytes(2, 1, 3, 64, 32, 16, 48) == 0      # C not a multiple of 64
    assert fl.flare_workspace_bytes(0, 0, 1, 64, 32, 16, 0) == 0       # B = 0


def test_output_projection_workspace_adds_the_concatenated_heads():
    for B, H, N, M, D, C in [(1, 4, 1024, 32, 16, 64), (32, 8, 4096, 128, 32, 256), (1, 8, 1 << 20, 512, 16, 128)]:
        base = fl.flare_workspace_bytes(1, B, H, N, M, D, C)
        out = fl.flare_workspace_bytes(2, B, H, N, M, D, C)
        assert out >= base + B * N * C * 2 and out % 256 == 0


def flare_call(K=A, V=A, Q=A, Y=A, B=1, H=2, N=100, M=32, D=16, lengths=None, ws=W, ws_bytes=1 << 40,
               Z=None):
    lib = fl.load_library()
    return lib.flare_mixer_fwd(K, V, Q, Y, B, H, N, M, D, lengths, 0.0, ws, ws_bytes, None, Z)


def flarepp_call(X=A, Wk=A, Wv=A, Wks=A, Wvs=A, Q0=A, Y=A, B=1, N=100, C=64, H=4, M=32, D=16,
                 lengths=None, ws=W, ws_bytes=1 << 40, Qx=None, Z=None):
    lib = fl.load_library()
    return lib.flarepp_mixer_fwd(X, Wk, Wv, Wks, Wvs, Q0, Y, B, N, C, H, M, D, lengths, 0.0, ws, ws_bytes,
                                 None, Qx, Z)


def flarepp_out_call(X=A, Wk=A, Wv=A, Wks=A, Wvs=A, Q0=A, Wo=A, Out=A, B=1, N=100, C=64, H=4, M=32, D=16,
                     lengths=None, ws=W, ws_bytes=1 << 40):
    lib = fl.load_library()
    return lib.flarepp_mixer_out_fwd(X, Wk, Wv, Wks, Wvs, Q0, Wo, Out, B, N, C, H, M, D, lengths, 0.0, ws, ws_bytes,
                                     None)


def test_flare_argument_errors():
    assert flare_call(K=None) == Status.ERR_NULL
    assert flare_call(Y=None) == Status.ERR_NULL
    assert flare_call(ws=None) == Status.ERR_NULL
    assert flare_call(N=0) == Status.ERR_SHAPE
    assert flare_call(B=-1) == Status.ERR_SHAPE
    assert flare_call(D=64) == Status.ERR_UNSUPPORTED
    assert flare_call(M=40) == Status.ERR_UNSUPPORTED
    assert flare_call(K=A + 8) == Status.ERR_ALIGN
    assert flare_call(lengths=A + 4) == Status.ERR_ALIGN
    assert flare_call(Z=A + 2) == Status.ERR_ALIGN
    assert flare_call(ws=W + 16) == Status.ERR_ALIGN
    need = fl.flare_workspace_bytes(0, 1, 2, 100, 32, 16)
    assert flare_call(ws_bytes=need - 1) == Status.ERR_WORKSPACE


def test_flarepp_argument_errors():
    assert flarepp_call(Wvs=None) == Status.ERR_NULL
    assert flarepp_call(Q0=None) == Status.ERR_NULL
    assert flarepp_call(C=128) == Status.ERR_SHAPE                  # C != H*D
    assert flarepp_call(C=48, H=3) == Status.ERR_UNSUPPORTED        # C % 64 != 0
    assert flarepp_call(C=512, H=16, D=32) == Status.ERR_UNSUPPORTED
    assert flarepp_call(X=A + 2) == Status.ERR_ALIGN
    assert flarepp_call(Qx=A + 4) == Status.ERR_ALIGN
    need = fl.flare_workspace_bytes(1, 1, 4, 100, 32, 16, 64)
    assert flarepp_call(ws_bytes=need - 256) == Status.ERR_WORKSPACE


def test_flarepp_out_argument_errors():
    assert flarepp_out_call(Wo=None) == Status.ERR_NULL
    assert flarepp_out_call(Out=None) == Status.ERR_NULL
    assert flarepp_out_call(C=128) == Status.ERR_SHAPE
    assert flarepp_out_call(Wo=A + 2) == Status.ERR_ALIGN
    assert flarepp_out_call(Out=A + 8) == Status.ERR_ALIGN
    need = fl.flare_workspace_bytes(2, 1, 4, 100, 32, 16, 64)
    assert need > fl.flare_workspace_bytes(1, 1, 4, 100, 32, 16, 64)
    assert flarepp_out_call(ws_bytes=need - 256) == Status.ERR_WORKSPACE


def test_valid_call_without_gpu_reports_launch_error():
    """With valid arguments the library reaches CUDA; on a machine without a
    GPU that fails cleanly with ERR_LAUNCH instead of crashing."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert flare_call() == Status.ERR_LAUNCH
    assert flarepp_call() == Status.ERR_LAUNCH
    assert flarepp_out_call() == Status.ERR_LAUNCH
    lib = fl.load_library()
    assert lib.flare_selftest_wait_timeout(W, None, 1000) == Status.ERR_LAUNCH
    assert lib.flare_last_device_status(None, None) == Status.ERR_NULL


def test_static_scratch_entry_point_rejects_oversized_problems():
    """Sizes whose workspace exceeds the fixed scratch are refused on the host."""
    lib = fl.load_library()
    assert fl.flare_workspace_bytes(0, 64, 8, 1 << 20, 512, 16) > fl._binding.FLARE_STATIC_SCRATCH_BYTES
    st = lib.flare_mixer_fwd_static(A, A, A, A, 64, 8, 1 << 20, 512, 16, None, 0.0, None, None)
    assert st == Status.ERR_WORKSPACE
    assert lib.flare_mixer_fwd_static(None, A, A, A, 1, 1, 64, 16, 16, None, 0.0, None, None) == Status.ERR_NULL
    assert lib.flare_mixer_fwd_static(A, A, A, A + 2, 1, 1, 64, 16, 16, None, 0.0, None, None) == Status.ERR_ALIGN


def test_context_parallel_argument_errors():
    lib = fl.load_library()
    assert lib.flare_cp_partials_bytes(1, 2, 100, 32, 16) > 0
    assert lib.flare_cp_partials_bytes(1, 2, 100, 40, 16) == 0                 # M not a multiple of 16
    args = (1, 100, 64, 4, 32, 16, None)
    ws = fl.flare_workspace_bytes(1, 1, 4, 100, 32, 16, 64)
    # rank outside [0, world), missing partials, unaligned partials
    assert lib.flarepp_cp_begin(A, A, A, A, A, A, *args, 2, 2, 0.0, W, ws, None, A) == Status.ERR_SHAPE
    assert lib.flarepp_cp_begin(A, A, A, A, A, A, *args, 0, 1, 0.0, W, ws, None, None) == Status.ERR_NULL
    assert lib.flarepp_cp_begin(A, A, A, A, A, A, *args, 0, 1, 0.0, W, ws, None, A + 4) == Status.ERR_ALIGN
    assert lib.flarepp_cp_begin(A, A, A, A, A, A, *args, 0, 1, 0.0, W, ws - 256, None, A) == Status.ERR_WORKSPACE
    assert lib.flarepp_cp_middle(A, A, *args, 0, 0, 0.0, W, ws, None, A, None) == Status.ERR_SHAPE   # world 0
    assert lib.flarepp_cp_middle(A, A + 4, *args, 0, 1, 0.0, W, ws, None, A, None) == Status.ERR_ALIGN
    assert lib.flarepp_cp_end(None, A, A, *args, 0, 1, 0.0, W, ws, None, None) == Status.ERR_NULL
    # the exact step: pass 0 or 1 only, every pointer, alignment, workspace
    assert lib.flare_cp_exact_bytes(1, 4, 32, 16) == 4 * 32 * 18 * 4
    assert lib.flare_cp_exact_bytes(1, 4, 40, 16) == 0
    assert lib.flarepp_cp_exact(2, A, A, A, A, A, A, *args, 0, 1, 0.0, W, ws, None, A) == Status.ERR_SHAPE
    assert lib.flarepp_cp_exact(0, A, A, A, A, A, A, *args, 0, 1, 0.0, W, ws, None, None) == Status.ERR_NULL
    assert lib.flarepp_cp_exact(1, A, A, A, A, A, A, *args, 0, 1, 0.0, W, ws, None, A + 4) == Status.ERR_ALIGN
    assert lib.flarepp_cp_exact(1, A, A, A, A, A, A, *args, 0, 1, 0.0, W, ws - 256, None, A) == Status.ERR_WORKSPACE
    fargs = (1, 2, 100, 32, 16, None)
    fws = fl.flare_workspace_bytes(0, 1, 2, 100, 32, 16)
    assert lib.flare_cp_begin(A, A, A, *fargs, -1, 2, 0.0, W, fws, None, A) == Status.ERR_SHAPE
    assert lib.flare_cp_end(A, None, A, A, None, *fargs, 0, 2, 0.0, W, fws, None, None) == Status.ERR_NULL
    assert lib.flare_cp_exact(A, A, None, A, *fargs, 0, 2, 0.0, W, fws, None, A) == Status.ERR_NULL
    assert lib.flare_cp_exact(A, A, A, A, *fargs, 2, 2, 0.0, W, fws, None, A) == Status.ERR_SHAPE
    assert fl.flare_status_string(8).startswith("FLARE_ERR_UNDERFLOW")


# ---------------------------------------------------------------------------
# backward entry points
# ---------------------------------------------------------------------------

def flare_bwd_call(K=A, V=A, Q=A, dY=A, dK=A, dV=A, dQ=A, B=1, H=2, N=100, M=32, D=16, lengths=None,
                   ws=W, ws_bytes=None):
    lib = fl.load_library()
    if ws_bytes is None:
        ws_bytes = fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLARE_BWD, B, H, N, M, D) or (1 << 40)
    return lib.flare_mixer_bwd(K, V, Q, dY, dK, dV, dQ, B, H, N, M, D, lengths, 0.0, ws, ws_bytes, None)


def flarepp_bwd_call(X=A, Wk=A, Wv=A, Wks=A + 0x100, Wvs=A + 0x200, Q0=A, dY=A, dX=A, dWk=A, dWv=A, dWks=A,
                     dWvs=A, dQ0=A, B=1, N=100, C=64, H=4, M=32, D=16, lengths=None, ws=W, ws_bytes=None):
    lib = fl.load_library()
    if ws_bytes is None:
        ws_bytes = fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLAREPP_BWD, B, H, N, M, D, C) or (1 << 40)
    return lib.flarepp_mixer_bwd(X, Wk, Wv, Wks, Wvs, Q0, dY, dX, dWk, dWv, dWks, dWvs, dQ0, B, N, C, H, M, D,
                                 lengths, 0.0, ws, ws_bytes, None)


def test_backward_workspace_sizes():
    f_fwd = fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLARE, 2, 4, 5000, 64, 16)
    f_bwd = fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLARE_BWD, 2, 4, 5000, 64, 16)
    assert f_bwd > f_fwd > 0 and f_bwd % 256 == 0
    p_fwd = fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLAREPP, 2, 4, 5000, 64, 16, 64)
    p_bwd = fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLAREPP_BWD, 2, 4, 5000, 64, 16, 64)
    # the FLARE++ backward holds fp32 gradient rows of the four projections
    assert p_bwd > p_fwd + 2 * 5000 * 4 * 64 * 4
    assert fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLAREPP_BWD, 2, 4, 5000, 64, 16, 128) == 0   # C != H*D
    assert fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLARE_BWD, 65536, 1, 64, 16, 16) == 0      # B*H > 65535
    assert fl.flare_workspace_bytes(5, 1, 4, 100, 32, 16, 64) == 0


def test_flare_backward_argument_errors():
    assert flare_bwd_call(dY=None) == Status.ERR_NULL
    assert flare_bwd_call(dQ=None) == Status.ERR_NULL
    assert flare_bwd_call(ws=None) == Status.ERR_NULL
    assert flare_bwd_call(N=0) == Status.ERR_SHAPE
    assert flare_bwd_call(D=64) == Status.ERR_UNSUPPORTED
    assert flare_bwd_call(B=70000, H=1) == Status.ERR_UNSUPPORTED
    assert flare_bwd_call(dK=A + 8) == Status.ERR_ALIGN
    assert flare_bwd_call(dQ=A + 4) == Status.ERR_ALIGN
    need = fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLARE_BWD, 1, 2, 100, 32, 16)
    assert flare_bwd_call(ws_bytes=need - 256) == Status.ERR_WORKSPACE


def test_flarepp_backward_argument_errors():
    assert flarepp_bwd_call(dX=None) == Status.ERR_NULL
    assert flarepp_bwd_call(dQ0=None) == Status.ERR_NULL
    assert flarepp_bwd_call(dWks=None) == Status.ERR_NULL           # separate synthesis weights need it
    assert flarepp_bwd_call(C=128) == Status.ERR_SHAPE
    assert flarepp_bwd_call(dWv=A + 4) == Status.ERR_ALIGN
    assert flarepp_bwd_call(dY=A + 2) == Status.ERR_ALIGN
    need = fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLAREPP_BWD, 1, 4, 100, 32, 16, 64)
    assert flarepp_bwd_call(ws_bytes=need - 256) == Status.ERR_WORKSPACE


def test_backward_valid_calls_without_gpu_report_launch_error():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert flare_bwd_call() == Status.ERR_LAUNCH
    assert flarepp_bwd_call() == Status.ERR_LAUNCH
    # shared projections: the synthesis weight gradients may be NULL
    assert flarepp_bwd_call(Wks=A, Wvs=A, dWks=None, dWvs=None) == Status.ERR_LAUNCH


def test_training_pair_argument_errors():
    """The training pair takes the backward's workspace for both calls and
    the backward's argument checks."""
    lib = fl.load_library()
    need_f = fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLARE_BWD, 1, 2, 100, 32, 16)
    need_p = fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLAREPP_BWD, 1, 4, 100, 32, 16, 64)
    fwd_f = lambda Y=A, ws=W, nb=need_f, D=16: lib.flare_mixer_fwd_train(A, A, A, Y, 1, 2, 100, 32, D, None, 0.0,
                                                                         ws, nb, None)
    fwd_p = lambda Y=A, ws=W, nb=need_p, C=64: lib.flarepp_mixer_fwd_train(A, A, A, A + 0x100, A + 0x200, A, Y, 1,
                                                                           100, C, 4, 32, 16, None, 0.0, ws, nb,
                                                                           None)
    assert fwd_f(Y=None) == Status.ERR_NULL and fwd_p(Y=None) == Status.ERR_NULL
    assert fwd_f(ws=None) == Status.ERR_NULL and fwd_p(ws=None) == Status.ERR_NULL
    assert fwd_f(D=64) == Status.ERR_UNSUPPORTED
    assert fwd_p(C=128) == Status.ERR_SHAPE
    # the forward's own workspace is too small: the state lives in the backward's
    small_f = fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLARE, 1, 2, 100, 32, 16)
    small_p = fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLAREPP, 1, 4, 100, 32, 16, 64)
    assert fwd_f(nb=small_f) == Status.ERR_WORKSPACE and fwd_p(nb=small_p) == Status.ERR_WORKSPACE
    assert fwd_f(nb=need_f - 256) == Status.ERR_WORKSPACE and fwd_p(nb=need_p - 256) == Status.ERR_WORKSPACE
    bwd_f = lambda dQ=A, nb=need_f: lib.flare_mixer_bwd_train(A, A, A, A, A, A, dQ, 1, 2, 100, 32, 16, None, 0.0, W,
                                                             nb, None)
    bwd_p = lambda dX=A, nb=need_p: lib.flarepp_mixer_bwd_train(A, A, A, A + 0x100, A + 0x200, A, A, dX, A, A, A,
                                                               A, A, 1, 100, 64, 4, 32, 16, None, 0.0, W, nb,
                                                               None)
    assert bwd_f(dQ=None) == Status.ERR_NULL and bwd_p(dX=None) == Status.ERR_NULL
    assert bwd_f(dQ=A + 4) == Status.ERR_ALIGN
    assert bwd_f(nb=need_f - 256) == Status.ERR_WORKSPACE and bwd_p(nb=need_p - 256) == Status.ERR_WORKSPACE
    import torch
    if not torch.cuda.is_available():
        assert fwd_f() == Status.ERR_LAUNCH and fwd_p() == Status.ERR_LAUNCH
        assert bwd_f() == Status.ERR_LAUNCH and bwd_p() == Status.ERR_LAUNCH


def cp_bwd_call(phase=0, gathered=None, exchange=A, rank=0, world=2, B=1, N=100, C=64, H=4, M=32, D=16, ws=W,
                ws_bytes=None, dX=A):
    lib = fl.load_library()
    if ws_bytes is None:
        ws_bytes = fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLAREPP_BWD, B, H, N, M, D, C) or (1 << 40)
    return lib.flarepp_cp_bwd_phase(phase, A, A, A, A + 0x100, A + 0x200, A, A, gathered, exchange, dX, A, A, A, A,
                                    A, B, N, C, H, M, D, None, rank, world, 0.0, ws, ws_bytes, None)


def test_cp_backward_exchange_sizes():
    lib = fl.load_library()
    sizes = [lib.flarepp_cp_bwd_exchange_bytes(p, 1, 1000, 64, 4, 32, 16) for p in range(8)]
    assert all(x > 0 and x % 16 == 0 for x in sizes[:6]) and sizes[6] == 0 and sizes[7] == 0
    assert sizes[0] == sizes[1] and sizes[3] == sizes[4]
    assert sizes[2] == 2 * sizes[3]                       # [dZ | dQ] partials
    assert lib.flarepp_cp_bwd_exchange_bytes(0, 1, 1000, 128, 4, 32, 16) == 0   # C != H*D
    assert lib.flarepp_cp_bwd_exchange_bytes(-1, 1, 1000, 64, 4, 32, 16) == 0


def test_cp_backward_argument_errors():
    assert cp_bwd_call(phase=7) == Status.ERR_SHAPE
    assert cp_bwd_call(phase=-1) == Status.ERR_SHAPE
    assert cp_bwd_call(rank=2, world=2) == Status.ERR_SHAPE
    assert cp_bwd_call(phase=1, gathered=None) == Status.ERR_NULL   # phases after the first read the gather
    assert cp_bwd_call(phase=0, exchange=None) == Status.ERR_NULL
    assert cp_bwd_call(phase=6, gathered=A, exchange=None, dX=None) == Status.ERR_NULL
    assert cp_bwd_call(phase=2, gathered=A + 4) == Status.ERR_ALIGN
    need = fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLAREPP_BWD, 1, 4, 100, 32, 16, 64)
    assert cp_bwd_call(ws_bytes=need - 256) == Status.ERR_WORKSPACE


def test_cp_backward_valid_call_without_gpu_reports_launch_error():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert cp_bwd_call() == Status.ERR_LAUNCH
    assert cp_bwd_call(phase=6, gathered=A, exchange=None) == Status.ERR_LAUNCH


def fl_cp_bwd_call(phase=0, gathered=None, exchange=A, rank=0, world=2, B=1, H=2, N=100, M=32, D=16, ws=W,
                   ws_bytes=None, dK=A):
    lib = fl.load_library()
    if ws_bytes is None:
        ws_bytes = fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLARE_BWD, B, H, N, M, D) or (1 << 40)
    return lib.flare_cp_bwd_phase(phase, A, A, A, A, gathered, exchange, dK, A, A, B, H, N, M, D, None, rank, world,
                                  0.0, ws, ws_bytes, None)


def test_flare_cp_backward_exchange_sizes():
    lib = fl.load_library()
    sizes = [lib.flare_cp_bwd_exchange_bytes(p, 1, 2, 1000, 32, 16) for p in range(5)]
    assert all(x > 0 and x % 16 == 0 for x in sizes[:3]) and sizes[3] == 0 and sizes[4] == 0
    assert sizes[1] == 2 * sizes[2]                       # [dZ | dQ] partials
    assert sizes[0] * 16 == sizes[2] * 18                 # recompute partials carry D + 2 floats per row
    assert lib.flare_cp_bwd_exchange_bytes(0, 1, 2, 1000, 40, 16) == 0      # M not a multiple of 16
    assert lib.flare_cp_bwd_exchange_bytes(-1, 1, 2, 1000, 32, 16) == 0


def test_flare_cp_backward_argument_errors():
    assert fl_cp_bwd_call(phase=4) == Status.ERR_SHAPE
    assert fl_cp_bwd_call(phase=-1) == Status.ERR_SHAPE
    assert fl_cp_bwd_call(rank=2, world=2) == Status.ERR_SHAPE
    assert fl_cp_bwd_call(phase=1, gathered=None) == Status.ERR_NULL
    assert fl_cp_bwd_call(phase=0, exchange=None) == Status.ERR_NULL
    assert fl_cp_bwd_call(phase=3, gathered=A, exchange=None, dK=None) == Status.ERR_NULL
    assert fl_cp_bwd_call(phase=2, gathered=A + 4) == Status.ERR_ALIGN
    need = fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLARE_BWD, 1, 2, 100, 32, 16)
    assert fl_cp_bwd_call(ws_bytes=need - 256) == Status.ERR_WORKSPACE
