"""ctypes binding of include/flare.h (argument marshalling only)."""
from __future__ import annotations

import ctypes
import enum
import os
import threading
from typing import Optional

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG, "libflare.so")
_lock = threading.Lock()
_lib = None

FLARE_VARIANT_FLARE = 0
FLARE_VARIANT_FLAREPP = 1
FLARE_VARIANT_FLAREPP_OUT = 2
FLARE_VARIANT_FLARE_BWD = 3
FLARE_VARIANT_FLAREPP_BWD = 4


class Status(enum.IntEnum):
    OK = 0
    ERR_NULL = 1
    ERR_SHAPE = 2
    ERR_UNSUPPORTED = 3
    ERR_ALIGN = 4
    ERR_WORKSPACE = 5
    ERR_LAUNCH = 6
    ERR_TIMEOUT = 7
    ERR_UNDERFLOW = 8
    ERR_NO_FORWARD = 9


class FlareError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = Status(status)
        super().__init__(f"{where}: {flare_status_string(status)}")


def library_path() -> str:
    return _LIB_PATH


def load_library(build_if_missing: bool = True):
    """Load libflare.so, compiling it with nvcc first if it is missing or stale."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        from . import build as _build
        if build_if_missing and not _build.up_to_date():
            _build.build()
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"FLARE CUDA library not found at {_LIB_PATH}")
        lib = ctypes.CDLL(_LIB_PATH)
        vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        lib.flare_workspace_bytes.argtypes = [i, i, i, i, i, i, i]
        lib.flare_workspace_bytes.restype = sz
        lib.flare_mixer_fwd.argtypes = [vp, vp, vp, vp, i, i, i, i, i, vp, f, vp, sz, vp, vp]
        lib.flare_mixer_fwd.restype = i
        lib.flarepp_mixer_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, vp, f, vp, sz, vp, vp, vp]
        lib.flarepp_mixer_fwd.restype = i
        lib.flare_mixer_fwd_profiled.argtypes = lib.flare_mixer_fwd.argtypes + [vp]
        lib.flare_mixer_fwd_profiled.restype = i
        lib.flarepp_mixer_fwd_profiled.argtypes = lib.flarepp_mixer_fwd.argtypes + [vp]
        lib.flare_mixer_fwd_inspect.argtypes = lib.flare_mixer_fwd.argtypes + [vp]
        lib.flare_mixer_fwd_inspect.restype = i
        lib.flarepp_mixer_fwd_inspect.argtypes = lib.flarepp_mixer_fwd.argtypes + [vp]
        lib.flarepp_mixer_fwd_inspect.restype = i
        lib.flare_probe_scratch_bytes.argtypes = []
        lib.flare_probe_scratch_bytes.restype = sz
        lib.flare_probe_pipe_rates.argtypes = [vp, sz, vp, ctypes.POINTER(ctypes.c_double),
                                               ctypes.POINTER(ctypes.c_double)]
        lib.flare_probe_pipe_rates.restype = i
        lib.flare_static_last_device_status.argtypes = [vp]
        lib.flare_static_last_device_status.restype = i
        lib.flare_cp_partials_bytes.restype = sz
        lib.flare_cp_partials_bytes.argtypes = [i, i, i, i, i]
        lib.flare_cp_exact_bytes.restype = sz
        lib.flare_cp_exact_bytes.argtypes = [i, i, i, i]
        for name, args in (
                ("flarepp_cp_begin", [vp] * 6 + [i] * 6 + [vp, i, i, f, vp, sz, vp, vp]),
                ("flarepp_cp_exact", [i] + [vp] * 6 + [i] * 6 + [vp, i, i, f, vp, sz, vp, vp]),
                ("flarepp_cp_middle", [vp, vp] + [i] * 6 + [vp, i, i, f, vp, sz, vp, vp, vp]),
                ("flarepp_cp_end", [vp, vp, vp] + [i] * 6 + [vp, i, i, f, vp, sz, vp, vp]),
                ("flare_cp_begin", [vp] * 3 + [i] * 5 + [vp, i, i, f, vp, sz, vp, vp]),
                ("flare_cp_exact", [vp] * 4 + [i] * 5 + [vp, i, i, f, vp, sz, vp, vp]),
                ("flare_cp_end", [vp] * 5 + [i] * 5 + [vp, i, i, f, vp, sz, vp, vp])):
            fn = getattr(lib, name)
            fn.restype = i
            fn.argtypes = args
        lib.flarepp_mixer_out_fwd.restype = i
        lib.flare_mixer_bwd.restype = i
        lib.flare_mixer_bwd.argtypes = [vp] * 7 + [i] * 5 + [vp, f, vp, sz, vp]
        lib.flarepp_mixer_bwd.restype = i
        lib.flarepp_mixer_bwd.argtypes = [vp] * 13 + [i] * 6 + [vp, f, vp, sz, vp]
        lib.flarepp_mixer_fwd_train.restype = i
        lib.flarepp_mixer_fwd_train.argtypes = [vp] * 7 + [i] * 6 + [vp, f, vp, sz, vp]
        lib.flarepp_mixer_bwd_train.restype = i
        lib.flarepp_mixer_bwd_train.argtypes = lib.flarepp_mixer_bwd.argtypes
        lib.flare_mixer_fwd_train.restype = i
        lib.flare_mixer_fwd_train.argtypes = [vp] * 4 + [i] * 5 + [vp, f, vp, sz, vp]
        lib.flare_mixer_bwd_train.restype = i
        lib.flare_mixer_bwd_train.argtypes = lib.flare_mixer_bwd.argtypes
        lib.flarepp_cp_bwd_exchange_bytes.restype = sz
        lib.flarepp_cp_bwd_exchange_bytes.argtypes = [i] * 7
        lib.flare_cp_bwd_exchange_bytes.restype = sz
        lib.flare_cp_bwd_exchange_bytes.argtypes = [i] * 6
        lib.flare_cp_bwd_phase.restype = i
        lib.flare_cp_bwd_phase.argtypes = [i] + [vp] * 9 + [i] * 5 + [vp, i, i, f, vp, sz, vp]
        lib.flarepp_cp_bwd_phase.restype = i
        lib.flarepp_cp_bwd_phase.argtypes = [i] + [vp] * 15 + [i] * 6 + [vp, i, i, f, vp, sz, vp]
        lib.flarepp_mixer_out_fwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, vp, f, vp, sz, vp]
        lib.flarepp_mixer_fwd_profiled.restype = i
        lib.flare_mixer_fwd_static.argtypes = [vp, vp, vp, vp, i, i, i, i, i, vp, f, vp, vp]
        lib.flare_mixer_fwd_static.restype = i
        lib.flare_last_device_status.argtypes = [vp, vp]
        lib.flare_last_device_status.restype = i
        lib.flare_status_string.argtypes = [i]
        lib.flare_status_string.restype = ctypes.c_char_p
        lib.flare_selftest_wait_timeout.argtypes = [vp, vp, ctypes.c_ulonglong]
        lib.flare_selftest_wait_timeout.restype = i
        _lib = lib
        return lib


def flare_status_string(status: int) -> str:
    return load_library().flare_status_string(int(status)).decode()


def flare_workspace_bytes(variant: int, B: int, H: int, N: int, M: int, D: int, C: int = 0) -> int:
    return int(load_library().flare_workspace_bytes(variant, B, H, N, M, D, C))


# ----------------------------------------------------------------------------
# torch helpers (plumbing only)
# ----------------------------------------------------------------------------

def _torch():
    import torch
    return torch


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _check_dev(name, t, dtype, shape=None):
    torch = _torch()
    if t is None:
        return
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _stream_ptr(stream, device) -> int:
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return int(stream.cuda_stream)


def _workspace(workspace, nbytes, device):
    torch = _torch()
    if workspace is None:
        return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
    _check_dev("workspace", workspace, torch.uint8)
    if workspace.numel() < nbytes:
        raise ValueError(f"workspace has {workspace.numel()} bytes, needs {nbytes}")
    return workspace


def _device_check(device_check, workspace_given: bool, workspace, stream, where: str) -> None:
    """Read the device error word (an expired bounded wait, a length outside
    [1, N], an underflowed context-parallel merge) after the call's work and
    raise FlareError if it is set.  ``device_check`` None means: check when the
    workspace was allocated here, since the caller then has no workspace to
    query.  Checking synchronises the stream."""
    if device_check is None:
        device_check = not workspace_given
    if not device_check:
        return
    st = load_library().flare_last_device_status(_ptr(workspace), _stream_ptr(stream, workspace.device))
    if st != 0:
        raise FlareError(st, where + " (device status)")


def _event_array(events):
    """cudaEvent_t handles of torch.cuda.Event objects (each recorded once so
    that its handle exists) as a ctypes void* array."""
    if events is None:
        return None
    handles = []
    for e in events:
        if e.cuda_event == 0:
            e.record()
        handles.append(e.cuda_event)
    return (ctypes.c_void_p * len(handles))(*handles)


def flare_mixer_fwd(K, V, Q, lengths=None, scale: float = 0.0, Y=None, workspace=None, stream=None,
                    Z_out=None, check: bool = True, stage_events=None, Y_f32_out=None, device_check=None):
    """FLARE forward (eq. 5-6).  K, V: [B,H,N,D] bf16; Q: [H,M,D] bf16 -> Y [B,H,N,D] bf16.
    ``Y_f32_out`` ([B,H,N,D] float32) selects flare_mixer_fwd_inspect: it also
    receives the fp32 values Y is rounded from.  ``device_check``: see
    ``_device_check`` (default: only when no workspace is passed)."""
    torch = _torch()
    B, H, N, D = K.shape
    M = Q.shape[1]
    if check:
        _check_dev("K", K, torch.bfloat16)
        _check_dev("V", V, torch.bfloat16, K.shape)
        _check_dev("Q", Q, torch.bfloat16, (H, M, D))
        _check_dev("lengths", lengths, torch.int32, (B,))
        _check_dev("Z_out", Z_out, torch.float32, (B, H, M, D))
        _check_dev("Y_f32_out", Y_f32_out, torch.float32, (B, H, N, D))
    if Y is None:
        Y = torch.empty_like(K)
    nbytes = flare_workspace_bytes(FLARE_VARIANT_FLARE, B, H, N, M, D)
    given = workspace is not None
    workspace = _workspace(workspace, nbytes, K.device)
    args = (_ptr(K), _ptr(V), _ptr(Q), _ptr(Y), B, H, N, M, D, _ptr(lengths), float(scale), _ptr(workspace),
            workspace.numel(), _stream_ptr(stream, K.device), _ptr(Z_out))
    if Y_f32_out is not None:
        assert stage_events is None, "stage events and Y_f32_out are not combined"
        st = load_library().flare_mixer_fwd_inspect(*args, _ptr(Y_f32_out))
    elif stage_events is None:
        st = load_library().flare_mixer_fwd(*args)
    else:
        assert len(stage_events) == 5
        st = load_library().flare_mixer_fwd_profiled(*args, _event_array(stage_events))
    if st != 0:
        raise FlareError(st, "flare_mixer_fwd")
    _device_check(device_check, given, workspace, stream, "flare_mixer_fwd")
    return Y


def flarepp_mixer_fwd(X, Wk, Wv, Wk_syn, Wv_syn, Q0, lengths=None, scale: float = 0.0, Y=None,
                      workspace=None, stream=None, Qx_out=None, Z_out=None, check: bool = True,
                      stage_events=None, Y_f32_out=None, device_check=None):
    """FLARE++ forward (eq. 7-11).  X: [B,N,C] bf16; W*: [C,C] bf16; Q0: [H,M,D] bf16
    -> Y [B,H,N,D] bf16.  ``Y_f32_out`` ([B,H,N,D] float32) selects
    flarepp_mixer_fwd_inspect: it also receives the fp32 values Y is rounded from."""
    torch = _torch()
    B, N, C = X.shape
    H, M, D = Q0.shape
    if check:
        _check_dev("X", X, torch.bfloat16)
        for nm, w in (("Wk", Wk), ("Wv", Wv), ("Wk_syn", Wk_syn), ("Wv_syn", Wv_syn)):
            _check_dev(nm, w, torch.bfloat16, (C, C))
        _check_dev("Q0", Q0, torch.bfloat16)
        _check_dev("lengths", lengths, torch.int32, (B,))
        _check_dev("Qx_out", Qx_out, torch.float32, (B, H, M, D))
        _check_dev("Z_out", Z_out, torch.float32, (B, H, M, D))
        _check_dev("Y_f32_out", Y_f32_out, torch.float32, (B, H, N, D))
    if Y is None:
        Y = torch.empty((B, H, N, D), dtype=torch.bfloat16, device=X.device)
    nbytes = flare_workspace_bytes(FLARE_VARIANT_FLAREPP, B, H, N, M, D, C)
    given = workspace is not None
    workspace = _workspace(workspace, nbytes, X.device)
    args = (_ptr(X), _ptr(Wk), _ptr(Wv), _ptr(Wk_syn), _ptr(Wv_syn), _ptr(Q0), _ptr(Y), B, N, C, H, M, D,
            _ptr(lengths), float(scale), _ptr(workspace), workspace.numel(), _stream_ptr(stream, X.device),
            _ptr(Qx_out), _ptr(Z_out))
    if Y_f32_out is not None:
        assert stage_events is None, "stage events and Y_f32_out are not combined"
        st = load_library().flarepp_mixer_fwd_inspect(*args, _ptr(Y_f32_out))
    elif stage_events is None:
        st = load_library().flarepp_mixer_fwd(*args)
    else:
        assert len(stage_events) == 7
        st = load_library().flarepp_mixer_fwd_profiled(*args, _event_array(stage_events))
    if st != 0:
        raise FlareError(st, "flarepp_mixer_fwd")
    _device_check(device_check, given, workspace, stream, "flarepp_mixer_fwd")
    return Y


def flarepp_mixer_out_fwd(X, Wk, Wv, Wk_syn, Wv_syn, Q0, Wo, lengths=None, scale: float = 0.0, Out=None,
                          workspace=None, stream=None, check: bool = True, device_check=None):
    """FLARE++ forward with the head concatenation and output projection:
    Out [B,N,C] bf16 = (Y_1 | ... | Y_H) @ Wo.  Passing the same tensors as
    Wk_syn/Wv_syn and Wk/Wv selects the shared-projection variant."""
    torch = _torch()
    B, N, C = X.shape
    H, M, D = Q0.shape
    if check:
        _check_dev("X", X, torch.bfloat16)
        for nm, w in (("Wk", Wk), ("Wv", Wv), ("Wk_syn", Wk_syn), ("Wv_syn", Wv_syn), ("Wo", Wo)):
            _check_dev(nm, w, torch.bfloat16, (C, C))
        _check_dev("Q0", Q0, torch.bfloat16)
        _check_dev("lengths", lengths, torch.int32, (B,))
    if Out is None:
        Out = torch.empty((B, N, C), dtype=torch.bfloat16, device=X.device)
    nbytes = flare_workspace_bytes(FLARE_VARIANT_FLAREPP_OUT, B, H, N, M, D, C)
    given = workspace is not None
    workspace = _workspace(workspace, nbytes, X.device)
    st = load_library().flarepp_mixer_out_fwd(
        _ptr(X), _ptr(Wk), _ptr(Wv), _ptr(Wk_syn), _ptr(Wv_syn), _ptr(Q0), _ptr(Wo), _ptr(Out), B, N, C, H, M, D,
        _ptr(lengths), float(scale), _ptr(workspace), workspace.numel(), _stream_ptr(stream, X.device))
    if st != 0:
        raise FlareError(st, "flarepp_mixer_out_fwd")
    _device_check(device_check, given, workspace, stream, "flarepp_mixer_out_fwd")
    return Out


FLARE_STATIC_SCRATCH_BYTES = 64 << 20


def flare_mixer_fwd_static(K, V, Q, lengths=None, scale: float = 0.0, Y=None, stream=None, Z_out=None,
                           device_check: bool = True):
    """FLARE forward without a caller-provided workspace (the library's fixed
    device scratch of FLARE_STATIC_SCRATCH_BYTES is used; nothing is
    allocated by the library).  Calls must not overlap on the GPU.  With
    ``device_check`` the static scratch's error word is read after the call
    (synchronises the stream) and a set word raises FlareError."""
    torch = _torch()
    B, H, N, D = K.shape
    M = Q.shape[1]
    _check_dev("K", K, torch.bfloat16)
    _check_dev("V", V, torch.bfloat16, K.shape)
    _check_dev("Q", Q, torch.bfloat16, (H, M, D))
    _check_dev("lengths", lengths, torch.int32, (B,))
    _check_dev("Z_out", Z_out, torch.float32, (B, H, M, D))
    if Y is None:
        Y = torch.empty_like(K)
    st = load_library().flare_mixer_fwd_static(_ptr(K), _ptr(V), _ptr(Q), _ptr(Y), B, H, N, M, D, _ptr(lengths),
                                               float(scale), _stream_ptr(stream, K.device), _ptr(Z_out))
    if st != 0:
        raise FlareError(st, "flare_mixer_fwd_static")
    if device_check:
        st = load_library().flare_static_last_device_status(_stream_ptr(stream, K.device))
        if st != 0:
            raise FlareError(st, "flare_mixer_fwd_static (device status)")
    return Y


def flare_mixer_fwd_train(K, V, Q, lengths=None, scale: float = 0.0, Y=None, workspace=None, stream=None,
                          check: bool = True, device_check=None):
    """FLARE forward that keeps its state for ``flare_mixer_bwd_train``:
    returns (Y, workspace), the workspace (FLARE_VARIANT_FLARE_BWD bytes)
    holding that state.  Y is the same as flare_mixer_fwd's."""
    torch = _torch()
    B, H, N, D = K.shape
    M = Q.shape[1]
    if check:
        _check_dev("K", K, torch.bfloat16)
        _check_dev("V", V, torch.bfloat16, K.shape)
        _check_dev("Q", Q, torch.bfloat16, (H, M, D))
        _check_dev("lengths", lengths, torch.int32, (B,))
        _check_dev("Y", Y, torch.bfloat16, K.shape)
    if Y is None:
        Y = torch.empty_like(K)
    given = workspace is not None
    workspace = _workspace(workspace, flare_workspace_bytes(FLARE_VARIANT_FLARE_BWD, B, H, N, M, D), K.device)
    st = load_library().flare_mixer_fwd_train(_ptr(K), _ptr(V), _ptr(Q), _ptr(Y), B, H, N, M, D, _ptr(lengths),
                                              float(scale), _ptr(workspace), workspace.numel(),
                                              _stream_ptr(stream, K.device))
    if st != 0:
        raise FlareError(st, "flare_mixer_fwd_train")
    _device_check(device_check, given, workspace, stream, "flare_mixer_fwd_train")
    return Y, workspace


def flare_mixer_bwd_train(K, V, Q, dY, workspace, lengths=None, scale: float = 0.0, stream=None,
                          dK=None, dV=None, dQ=None, check: bool = True, device_check: bool = False):
    """FLARE backward from the state that ``flare_mixer_fwd_train`` left in
    ``workspace`` (same inputs, lengths and scale).  Returns (dK, dV, dQ) as
    flare_mixer_bwd.  With ``device_check`` the device status is read after
    the call (synchronises), which also reports a workspace without a
    training forward's state (Status.ERR_NO_FORWARD)."""
    return flare_mixer_bwd(K, V, Q, dY, lengths=lengths, scale=scale, workspace=workspace, stream=stream, dK=dK,
                           dV=dV, dQ=dQ, check=check, device_check=device_check, _train=True)


def flare_mixer_bwd(K, V, Q, dY, lengths=None, scale: float = 0.0, workspace=None, stream=None,
                    dK=None, dV=None, dQ=None, check: bool = True, device_check=None, _train: bool = False):
    """FLARE backward (gradients of eq. 5-6 given dY).  K, V, dY: [B,H,N,D] bf16;
    Q: [H,M,D] bf16 -> (dK, dV) [B,H,N,D] bf16 and dQ [H,M,D] float32."""
    torch = _torch()
    B, H, N, D = K.shape
    M = Q.shape[1]
    if check:
        _check_dev("K", K, torch.bfloat16)
        for nm, t in (("V", V), ("dY", dY), ("dK", dK), ("dV", dV)):
            _check_dev(nm, t, torch.bfloat16, K.shape)
        _check_dev("Q", Q, torch.bfloat16, (H, M, D))
        _check_dev("dQ", dQ, torch.float32, (H, M, D))
        _check_dev("lengths", lengths, torch.int32, (B,))
    dK = torch.empty_like(K) if dK is None else dK
    dV = torch.empty_like(K) if dV is None else dV
    dQ = torch.empty((H, M, D), dtype=torch.float32, device=K.device) if dQ is None else dQ
    nbytes = flare_workspace_bytes(FLARE_VARIANT_FLARE_BWD, B, H, N, M, D)
    given = workspace is not None
    workspace = _workspace(workspace, nbytes, K.device)
    fn = load_library().flare_mixer_bwd_train if _train else load_library().flare_mixer_bwd
    where = "flare_mixer_bwd_train" if _train else "flare_mixer_bwd"
    st = fn(_ptr(K), _ptr(V), _ptr(Q), _ptr(dY), _ptr(dK), _ptr(dV), _ptr(dQ), B, H, N, M, D, _ptr(lengths),
            float(scale), _ptr(workspace), workspace.numel(), _stream_ptr(stream, K.device))
    if st != 0:
        raise FlareError(st, where)
    _device_check(device_check, given, workspace, stream, where)
    return dK, dV, dQ


def flarepp_mixer_fwd_train(X, Wk, Wv, Wk_syn, Wv_syn, Q0, lengths=None, scale: float = 0.0, Y=None,
                            workspace=None, stream=None, check: bool = True, device_check=None):
    """FLARE++ forward that keeps its state (projections, Q(X), Z and the
    synthesis and encode log-normalisers) for ``flarepp_mixer_bwd_train``:
    returns (Y, workspace), the workspace (FLARE_VARIANT_FLAREPP_BWD bytes)
    holding that state.  Y is the same as flarepp_mixer_fwd's."""
    torch = _torch()
    B, N, C = X.shape
    H, M, D = Q0.shape
    if check:
        _check_dev("X", X, torch.bfloat16)
        for nm, w in (("Wk", Wk), ("Wv", Wv), ("Wk_syn", Wk_syn), ("Wv_syn", Wv_syn)):
            _check_dev(nm, w, torch.bfloat16, (C, C))
        _check_dev("Q0", Q0, torch.bfloat16)
        _check_dev("lengths", lengths, torch.int32, (B,))
        _check_dev("Y", Y, torch.bfloat16, (B, H, N, D))
    if Y is None:
        Y = torch.empty((B, H, N, D), dtype=torch.bfloat16, device=X.device)
    given = workspace is not None
    workspace = _workspace(workspace, flare_workspace_bytes(FLARE_VARIANT_FLAREPP_BWD, B, H, N, M, D, C), X.device)
    st = load_library().flarepp_mixer_fwd_train(
        _ptr(X), _ptr(Wk), _ptr(Wv), _ptr(Wk_syn), _ptr(Wv_syn), _ptr(Q0), _ptr(Y), B, N, C, H, M, D,
        _ptr(lengths), float(scale), _ptr(workspace), workspace.numel(), _stream_ptr(stream, X.device))
    if st != 0:
        raise FlareError(st, "flarepp_mixer_fwd_train")
    _device_check(device_check, given, workspace, stream, "flarepp_mixer_fwd_train")
    return Y, workspace


def flarepp_mixer_bwd_train(X, Wk, Wv, Wk_syn, Wv_syn, Q0, dY, workspace, lengths=None, scale: float = 0.0,
                            stream=None, grads=None, check: bool = True, device_check: bool = False):
    """FLARE++ backward from the state that ``flarepp_mixer_fwd_train`` left
    in ``workspace`` (same inputs, lengths and scale).  Returns the gradients
    as flarepp_mixer_bwd.  With ``device_check`` the device status is read
    after the call (synchronises), which also reports a workspace without a
    training forward's state (Status.ERR_NO_FORWARD)."""
    return flarepp_mixer_bwd(X, Wk, Wv, Wk_syn, Wv_syn, Q0, dY, lengths=lengths, scale=scale, workspace=workspace,
                             stream=stream, grads=grads, check=check, device_check=device_check, _train=True)


def flarepp_mixer_bwd(X, Wk, Wv, Wk_syn, Wv_syn, Q0, dY, lengths=None, scale: float = 0.0, workspace=None,
                      stream=None, grads=None, check: bool = True, device_check=None, _train: bool = False):
    """FLARE++ backward (gradients of eq. 7-11 given dY [B,H,N,D] bf16).
    Returns a dict: dX [B,N,C] bf16; dWk, dWv, dWk_syn, dWv_syn [C,C] float32;
    dQ0 [H,M,D] float32.  ``grads`` may hold preallocated outputs by name."""
    torch = _torch()
    B, N, C = X.shape
    H, M, D = Q0.shape
    if check:
        _check_dev("X", X, torch.bfloat16)
        for nm, w in (("Wk", Wk), ("Wv", Wv), ("Wk_syn", Wk_syn), ("Wv_syn", Wv_syn)):
            _check_dev(nm, w, torch.bfloat16, (C, C))
        _check_dev("Q0", Q0, torch.bfloat16)
        _check_dev("dY", dY, torch.bfloat16, (B, H, N, D))
        _check_dev("lengths", lengths, torch.int32, (B,))
    g = dict(grads or {})
    dev = X.device
    if g.get("dX") is None:
        g["dX"] = torch.empty((B, N, C), dtype=torch.bfloat16, device=dev)
    for nm in ("dWk", "dWv", "dWk_syn", "dWv_syn"):
        if g.get(nm) is None:
            g[nm] = torch.empty((C, C), dtype=torch.float32, device=dev)
    if g.get("dQ0") is None:
        g["dQ0"] = torch.empty((H, M, D), dtype=torch.float32, device=dev)
    if check:
        _check_dev("dX", g["dX"], torch.bfloat16, (B, N, C))
        for nm in ("dWk", "dWv", "dWk_syn", "dWv_syn"):
            _check_dev(nm, g[nm], torch.float32, (C, C))
        _check_dev("dQ0", g["dQ0"], torch.float32, (H, M, D))
    nbytes = flare_workspace_bytes(FLARE_VARIANT_FLAREPP_BWD, B, H, N, M, D, C)
    given = workspace is not None
    workspace = _workspace(workspace, nbytes, dev)
    lib = load_library()
    fn, where = (lib.flarepp_mixer_bwd_train, "flarepp_mixer_bwd_train") if _train else \
        (lib.flarepp_mixer_bwd, "flarepp_mixer_bwd")
    st = fn(_ptr(X), _ptr(Wk), _ptr(Wv), _ptr(Wk_syn), _ptr(Wv_syn), _ptr(Q0), _ptr(dY), _ptr(g["dX"]),
            _ptr(g["dWk"]), _ptr(g["dWv"]), _ptr(g["dWk_syn"]), _ptr(g["dWv_syn"]), _ptr(g["dQ0"]),
            B, N, C, H, M, D, _ptr(lengths), float(scale), _ptr(workspace), workspace.numel(),
            _stream_ptr(stream, dev))
    if st != 0:
        raise FlareError(st, where)
    _device_check(device_check, given, workspace, stream, where)
    return g


def flare_last_device_status(workspace, stream=None) -> Status:
    return Status(load_library().flare_last_device_status(_ptr(workspace), _stream_ptr(stream, workspace.device)))


def flare_static_last_device_status(stream=None) -> Status:
    """Device error word of the last flare_mixer_fwd_static call (syncs the stream)."""
    torch = _torch()
    return Status(load_library().flare_static_last_device_status(_stream_ptr(stream, torch.device("cuda"))))


def flare_probe_pipe_rates(device=None, stream=None) -> dict:
    """Measured results per SM clock of ex2.approx.f32 (special-function unit)
    and fp32 fma (FMA pipe) on this device: {"ex2": ..., "ffma": ...}."""
    torch = _torch()
    device = torch.device("cuda") if device is None else torch.device(device)
    lib = load_library()
    scratch = torch.empty(int(lib.flare_probe_scratch_bytes()), dtype=torch.uint8, device=device)
    e, f = ctypes.c_double(0.0), ctypes.c_double(0.0)
    st = lib.flare_probe_pipe_rates(_ptr(scratch), scratch.numel(), _stream_ptr(stream, device), ctypes.byref(e),
                                    ctypes.byref(f))
    if st != 0:
        raise FlareError(st, "flare_probe_pipe_rates")
    return {"ex2": e.value, "ffma": f.value}


def flare_selftest_wait_timeout(workspace, timeout_ns: int, stream=None) -> None:
    st = load_library().flare_selftest_wait_timeout(_ptr(workspace), _stream_ptr(stream, workspace.device),
                                                    int(timeout_ns))
    if st != 0:
        raise FlareError(st, "flare_selftest_wait_timeout")
