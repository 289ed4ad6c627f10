"""Plain fp64 CPU oracle for the FLARE / FLARE++ mixer, forward and backward.

TEST INFRASTRUCTURE ONLY: the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` are the only code
allowed to import this package.  The CUDA library never calls it and shares no
code with it.

The arithmetic lives in ``flare_oracle.c`` (forward) and
``flare_oracle_bwd.c`` (gradients: the SDPA backward of every call, written
out per call) -- plain loops, fp64, two-pass softmax in ascending index
order, OpenMP over independent rows; this module only marshals numpy arrays.
Every function cites the passage of the FLARE++ paper (arXiv 2608.11519,
section "Method") it follows:

  project   eq. 7 / eq. 9   K_h = X W_{K,h}, heads = column blocks of width D
  encode    eq. 5 / 8 / 10  Z_h = softmax_n(Q_h K_h^T / sqrt(D)) V_h
  decode    eq. 6 / 11      Y_h = softmax_m(K_h Q_h^T / sqrt(D)) Z_h
  *_bwd     the gradients of the three above (the pages name the paper's
            backward equations, eq. 13-40, without printing them)

Pins (tests/test_oracle_pins.py): torch float64 SDPA chain, the materialised
rank-M mixing matrix, closed forms (two tokens, identical keys, zero queries,
one latent), token-permutation equivariance, the masked/unmasked identity and
the shard-combine identity of section "Multi-GPU context parallelism" (eq. 14).
Gradient pins (tests/test_oracle_bwd_pins.py): central finite differences of
the forward oracle, torch float64 autograd through the SDPA chain, the
shift invariances of the softmax and the sum rules of row-stochastic maps.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "flare_oracle.c")
_SRC_BWD = os.path.join(_HERE, "flare_oracle_bwd.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libflare_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (OpenMP, IEEE semantics, no FMA contraction)."""
    if not force and os.path.exists(_LIB_PATH) and \
            os.path.getmtime(_LIB_PATH) >= max(os.path.getmtime(_SRC), os.path.getmtime(_SRC_BWD)):
        return _LIB_PATH
    os.makedirs(_BUILD, exist_ok=True)
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fPIC",
           "-shared", "-o", tmp, _SRC, _SRC_BWD, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int32)
        lp = ctypes.POINTER(ctypes.c_int64)
        L = ctypes.c_long
        lib.flare_oracle_project.argtypes = [dp, dp, dp, L, L, L, L, L]
        lib.flare_oracle_project.restype = None
        lib.flare_oracle_encode.argtypes = [dp, ctypes.c_int, dp, dp, ip, ctypes.c_double,
                                            L, L, L, L, L, dp, dp]
        lib.flare_oracle_encode.restype = None
        lib.flare_oracle_decode.argtypes = [dp, dp, ctypes.c_int, dp, ip, ctypes.c_double,
                                            L, L, L, L, L, lp, L, dp]
        lib.flare_oracle_decode.restype = None
        lib.flare_oracle_encode_bwd.argtypes = [dp, ctypes.c_int, dp, dp, ip, ctypes.c_double,
                                                L, L, L, L, L, dp, dp, dp, dp]
        lib.flare_oracle_encode_bwd.restype = None
        lib.flare_oracle_decode_bwd.argtypes = [dp, dp, ctypes.c_int, dp, ip, ctypes.c_double,
                                                L, L, L, L, L, dp, dp, dp, dp]
        lib.flare_oracle_decode_bwd.restype = None
        lib.flare_oracle_project_bwd.argtypes = [dp, dp, dp, L, L, L, L, L, dp, dp]
        lib.flare_oracle_project_bwd.restype = None
        lib.flare_oracle_num_threads.argtypes = []
        lib.flare_oracle_num_threads.restype = ctypes.c_int
        _lib = lib
        return lib


def num_threads() -> int:
    return int(_load().flare_oracle_num_threads())


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.float64)


def _dptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _lens(lengths, B):
    if lengths is None:
        return None, None
    arr = np.ascontiguousarray(lengths, dtype=np.int32)
    assert arr.shape == (B,)
    return arr, arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def project(X, W, H: int) -> np.ndarray:
    """eq. 7 / eq. 9: X [B][N][C] @ W [C][C], split into H heads -> [B][H][N][D]."""
    X, W = _f64(X), _f64(W)
    B, N, C = X.shape
    assert W.shape == (C, C) and C % H == 0
    D = C // H
    out = np.empty((B, H, N, D), dtype=np.float64)
    _load().flare_oracle_project(_dptr(X), _dptr(W), _dptr(out), B, N, C, H, D)
    return out


def encode(Q, K, V, lengths=None, scale: Optional[float] = None,
           return_lse: bool = False):
    """eq. 5 (FLARE encoder), eq. 8 (query synthesis), eq. 10 (encode with Q(X)).

    Q: [H][M][D] (shared over the batch) or [B][H][M][D] (one set per sample).
    K, V: [B][H][N][D].  Returns Z [B][H][M][D] (and the row log-normaliser
    lse [B][H][M] = max + log(sum exp) when ``return_lse``)."""
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    B, H, N, D = K.shape
    assert V.shape == K.shape
    if Q.ndim == 3:
        per_batch, M = 0, Q.shape[1]
        assert Q.shape == (H, M, D)
    else:
        per_batch, M = 1, Q.shape[2]
        assert Q.shape == (B, H, M, D)
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    lens, lp = _lens(lengths, B)
    Z = np.empty((B, H, M, D), dtype=np.float64)
    lse = np.empty((B, H, M), dtype=np.float64) if return_lse else None
    _load().flare_oracle_encode(_dptr(Q), per_batch, _dptr(K), _dptr(V), lp, float(scale),
                                B, H, N, M, D, _dptr(Z), _dptr(lse))
    return (Z, lse) if return_lse else Z


def decode(K, Q, Z, lengths=None, scale: Optional[float] = None, rows=None) -> np.ndarray:
    """eq. 6 (FLARE decoder) / eq. 11 (decode with Q(X)).

    K [B][H][N][D]; Q [H][M][D] or [B][H][M][D]; Z [B][H][M][D].
    ``rows``: optional token indices (same for every head); the output is then
    [B][H][len(rows)][D].  Masked tokens (n >= lengths[b]) give zero rows."""
    K, Q, Z = _f64(K), _f64(Q), _f64(Z)
    B, H, N, D = K.shape
    if Q.ndim == 3:
        per_batch, M = 0, Q.shape[1]
    else:
        per_batch, M = 1, Q.shape[2]
    assert Z.shape == (B, H, M, D)
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    lens, lp = _lens(lengths, B)
    if rows is None:
        rp, nrows = None, N
    else:
        rows = np.ascontiguousarray(rows, dtype=np.int64)
        assert rows.ndim == 1 and (rows.size == 0 or (rows.min() >= 0 and rows.max() < N))
        rp, nrows = rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), rows.size
    Y = np.empty((B, H, nrows, D), dtype=np.float64)
    _load().flare_oracle_decode(_dptr(K), _dptr(Q), per_batch, _dptr(Z), lp, float(scale),
                                B, H, N, M, D, rp, nrows, _dptr(Y))
    return Y


def flare_forward(K, V, Q, lengths=None, scale=None, rows=None) -> dict:
    """FLARE mixer (section "FLARE: fixed-query latent routing", eq. 5-6)."""
    Z = encode(Q, K, V, lengths, scale)
    Y = decode(K, Q, Z, lengths, scale, rows)
    return {"Z": Z, "Y": Y}


def flarepp_forward(X, Wk, Wv, Wk_syn, Wv_syn, Q0, H: int, lengths=None, scale=None,
                    rows=None, keep_projections: bool = False) -> dict:
    """FLARE++ mixer (section "FLARE++: dynamic token routing", eq. 7-11):
    K~ = X W~_K, V~ = X W~_V, Q(X) = SDPA(Q~, K~, V~); K = X W_K, V = X W_V,
    Z = SDPA(Q(X), K, V), Y = SDPA(K, Q(X), Z)."""
    Kt = project(X, Wk_syn, H)
    Vt = project(X, Wv_syn, H)
    Qx = encode(Q0, Kt, Vt, lengths, scale)
    if not keep_projections:
        del Kt, Vt
    K = project(X, Wk, H)
    V = project(X, Wv, H)
    Z = encode(Qx, K, V, lengths, scale)
    Y = decode(K, Qx, Z, lengths, scale, rows)
    out = {"Qx": Qx, "Z": Z, "Y": Y}
    if keep_projections:
        out.update(Kt=Kt, Vt=Vt, K=K, V=V)
    return out


def output_projection(Y, Wo):
    """Head concatenation and output projection (section "Full self-attention":
    the heads' outputs side by side, times W_O): Out[b, n, :] =
    (Y[b, 0, n, :], ..., Y[b, H-1, n, :]) @ Wo, in float64."""
    Y = np.asarray(Y, dtype=np.float64)
    B, H, N, D = Y.shape
    Ycat = np.ascontiguousarray(np.transpose(Y, (0, 2, 1, 3))).reshape(B, N, H * D)
    return Ycat @ np.asarray(Wo, dtype=np.float64)


def forward_workload(w, rows=None, keep_projections: bool = False) -> dict:
    """Run the oracle on a ``workloads.Workload`` (bf16 bits widened to fp64)."""
    from workloads import bf16_bits_to_f64 as f64
    if w.variant == "flare":
        return flare_forward(f64(w.K), f64(w.V), f64(w.Q), w.lengths, w.scale, rows)
    out = flarepp_forward(f64(w.X), f64(w.Wk), f64(w.Wv), f64(w.Wk_syn), f64(w.Wv_syn),
                          f64(w.Q0), w.H, w.lengths, w.scale, rows, keep_projections)
    if w.Wo is not None and rows is None:
        out["Out"] = output_projection(out["Y"], f64(w.Wo))
    return out


# ---------------------------------------------------------------------------
# backward (gradients of a scalar loss given dY = dLoss/dY)
# ---------------------------------------------------------------------------

def _qinfo(Q, B, H, D):
    if Q.ndim == 3:
        assert Q.shape[0] == H and Q.shape[2] == D
        return 0, Q.shape[1]
    assert Q.shape[:2] == (B, H) and Q.shape[3] == D
    return 1, Q.shape[2]


def encode_bwd(Q, K, V, dZ, lengths=None, scale: Optional[float] = None):
    """Gradients of the encoder (eq. 5 / 8 / 10) given dZ [B][H][M][D]:
    returns (dQ shaped like Q, dK, dV [B][H][N][D]).  A query set shared over
    the batch ([H][M][D]) gets the sum of its per-sample gradients."""
    Q, K, V, dZ = _f64(Q), _f64(K), _f64(V), _f64(dZ)
    B, H, N, D = K.shape
    per_batch, M = _qinfo(Q, B, H, D)
    assert V.shape == K.shape and dZ.shape == (B, H, M, D)
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    lens, lp = _lens(lengths, B)
    dQ, dK, dV = np.zeros_like(Q), np.zeros_like(K), np.zeros_like(V)
    _load().flare_oracle_encode_bwd(_dptr(Q), per_batch, _dptr(K), _dptr(V), lp, float(scale),
                                    B, H, N, M, D, _dptr(dZ), _dptr(dQ), _dptr(dK), _dptr(dV))
    return dQ, dK, dV


def decode_bwd(K, Q, Z, dY, lengths=None, scale: Optional[float] = None):
    """Gradients of the decoder (eq. 6 / 11) given dY [B][H][N][D] (rows of
    masked tokens are ignored: their outputs are constant zeros): returns
    (dK [B][H][N][D], dQ shaped like Q, dZ [B][H][M][D])."""
    K, Q, Z, dY = _f64(K), _f64(Q), _f64(Z), _f64(dY)
    B, H, N, D = K.shape
    per_batch, M = _qinfo(Q, B, H, D)
    assert Z.shape == (B, H, M, D) and dY.shape == K.shape
    if scale is None:
        scale = 1.0 / np.sqrt(D)
    lens, lp = _lens(lengths, B)
    dK, dQ, dZ = np.zeros_like(K), np.zeros_like(Q), np.zeros_like(Z)
    _load().flare_oracle_decode_bwd(_dptr(K), _dptr(Q), per_batch, _dptr(Z), lp, float(scale),
                                    B, H, N, M, D, _dptr(dY), _dptr(dK), _dptr(dQ), _dptr(dZ))
    return dK, dQ, dZ


def project_bwd(X, W, dOut):
    """Gradients of the per-head projection (eq. 7 / 9) given dOut
    [B][H][N][D]: returns (dX [B][N][C], dW [C][C])."""
    X, W, dOut = _f64(X), _f64(W), _f64(dOut)
    B, N, C = X.shape
    _, H, _, D = dOut.shape
    assert W.shape == (C, C) and dOut.shape == (B, H, N, D) and H * D == C
    dX, dW = np.zeros_like(X), np.zeros_like(W)
    _load().flare_oracle_project_bwd(_dptr(X), _dptr(W), _dptr(dOut), B, N, C, H, D,
                                     _dptr(dX), _dptr(dW))
    return dX, dW


def flare_backward(K, V, Q, dY, lengths=None, scale=None) -> dict:
    """Gradients of the FLARE mixer Y = SDPA(K, Q, SDPA(Q, K, V)) (eq. 5-6):
    K gets the sum of its decoder and encoder gradients, Q (shared over the
    batch) the sum over the batch of both."""
    Z = encode(Q, K, V, lengths, scale)
    dK, dQ, dZ = decode_bwd(K, Q, Z, dY, lengths, scale)
    dQe, dKe, dV = encode_bwd(Q, K, V, dZ, lengths, scale)
    return {"dK": dK + dKe, "dV": dV, "dQ": dQ + dQe, "dZ": dZ}


def flarepp_backward(X, Wk, Wv, Wk_syn, Wv_syn, Q0, dY, H: int, lengths=None,
                     scale=None) -> dict:
    """Gradients of the FLARE++ mixer (eq. 7-11) with respect to X, the four
    projection weights and the seeds Q0, given dY [B][H][N][D].  The chain:
    decode -> (dK, dQ(X), dZ); encode with Q(X) -> (dQ(X), dK, dV); synthesis
    with Q0 -> (dQ0, dK~, dV~); projections -> dX and the weight gradients.
    The intermediate dQ(X) and dZ are returned as well."""
    Kt, Vt = project(X, Wk_syn, H), project(X, Wv_syn, H)
    Qx = encode(Q0, Kt, Vt, lengths, scale)
    K, V = project(X, Wk, H), project(X, Wv, H)
    Z = encode(Qx, K, V, lengths, scale)
    dK, dQx, dZ = decode_bwd(K, Qx, Z, dY, lengths, scale)
    dQx_e, dK_e, dV = encode_bwd(Qx, K, V, dZ, lengths, scale)
    dK = dK + dK_e
    dQx = dQx + dQx_e
    dQ0, dKt, dVt = encode_bwd(Q0, Kt, Vt, dQx, lengths, scale)
    dX = np.zeros_like(_f64(X))
    grads = {}
    for name, W, dOut in (("dWk", Wk, dK), ("dWv", Wv, dV), ("dWk_syn", Wk_syn, dKt),
                          ("dWv_syn", Wv_syn, dVt)):
        dXi, dWi = project_bwd(X, W, dOut)
        dX += dXi
        grads[name] = dWi
    grads.update(dX=dX, dQ0=dQ0, dQx=dQx, dZ=dZ)
    return grads


def backward_workload(w, dY) -> dict:
    """Run the backward oracle on a ``workloads.Workload`` and an upstream
    gradient dY [B][H][N][D] (both bf16 bits, widened to fp64)."""
    from workloads import bf16_bits_to_f64 as f64
    if w.variant == "flare":
        return flare_backward(f64(w.K), f64(w.V), f64(w.Q), f64(dY), w.lengths, w.scale)
    return flarepp_backward(f64(w.X), f64(w.Wk), f64(w.Wv), f64(w.Wk_syn), f64(w.Wv_syn),
                            f64(w.Q0), f64(dY), w.H, w.lengths, w.scale)
