"""Seeded synthetic inputs for the FLARE / FLARE++ mixer (forward inputs, and
the upstream gradient dY of the backward).

This module only draws random numbers and rounds them to bfloat16.  It holds
none of the mixer's arithmetic, so the fp64 oracle (``oracle/``) and the CUDA
path (``rank_latent_routing_flare_b200``) can both consume its output without
sharing any computation.

Every array is produced as bf16 *bit patterns* (``numpy.uint16``); the same
bytes are copied to the GPU and widened to float64 for the oracle.

Draw order for one workload (one ``numpy.random.Generator(PCG64(seed))``):
  FLARE++ : X (coordinates P, lift A, noise E for the mesh kinds), W_K, W_V,
            W~_K, W~_V, Q0, lengths, W_O
  FLARE   : K, V, Q, lengths

Rounding: every value is drawn in float32, then rounded to bf16 with
round-to-nearest-even on the float32 bit pattern.

The named workloads follow the shapes of the mixer forward that the FLARE++
paper (arXiv 2608.11519, section "Method") describes: X in R^{N x C}, H heads
of width D = C/H, M latent routes per head.  The value distributions and the
point-cloud structure of X ("mesh2d"/"mesh3d": uniform coordinates in the unit
square/cube lifted by a random linear map plus N(0,1) noise) stand in for the
PDE meshes of the paper's experiments; no dataset item is reproduced.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

__all__ = [
    "WORKLOADS",
    "Workload",
    "make_workload",
    "make_upstream_grad",
    "to_bf16_bits",
    "bf16_bits_to_f64",
    "bf16_bits_to_f32",
]


# name -> spec.  "x" is the distribution of the token features X.
WORKLOADS = {
    # FLARE++ B=1, N=1024, C=64, H=4, D=16, M=32; X ~ N(0,1); seed 0
    "flarepp_n1k": dict(variant="flarepp", B=1, N=1024, C=64, H=4, D=16, M=32,
                        x="normal", seed=0),
    # FLARE++ B=8, N=8192, C=128, H=8, D=16, M=64; 2-D point cloud; seed 1
    "flarepp_n8k_mesh2d": dict(variant="flarepp", B=8, N=8192, C=128, H=8, D=16,
                               M=64, x="mesh2d", seed=1),
    # FLARE (fixed queries) B=4, N=65536, C=128, H=8, D=16, M=256; seed 2
    "flare_n64k": dict(variant="flare", B=4, N=65536, C=128, H=8, D=16, M=256,
                       x="normal", seed=2),
    # FLARE++ same shape; seed 2
    "flarepp_n64k": dict(variant="flarepp", B=4, N=65536, C=128, H=8, D=16,
                         M=256, x="normal", seed=2),
    # FLARE++ B=1, N=1,048,576 (3-D point cloud), C=128, H=8, D=16, M=512; seed 3
    "flarepp_n1m_mesh3d": dict(variant="flarepp", B=1, N=1048576, C=128, H=8,
                               D=16, M=512, x="mesh3d", seed=3),
    # FLARE++ with key padding: B=32, N=4096 max, valid length U[1024,4096],
    # C=256, H=8, D=32, M=128; seed 4
    "flarepp_masked_n4k": dict(variant="flarepp", B=32, N=4096, C=256, H=8,
                               D=32, M=128, x="normal", seed=4,
                               lengths=(1024, 4096)),
    # Diagnostic (not a graded workload): the N=8192 shape with all weights
    # ~ N(0, 16/C), which gives routing scores with a spread of several units.
    "flarepp_n8k_sharp": dict(variant="flarepp", B=8, N=8192, C=128, H=8, D=16,
                              M=64, x="mesh2d", seed=1, weight_gain=4.0),
}


def to_bf16_bits(x) -> np.ndarray:
    """Round to float32, then to bf16 (round-to-nearest-even); return uint16 bits."""
    f = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    u = f.view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return bf16_bits_to_f32(b).astype(np.float64)


@dataclasses.dataclass
class Workload:
    name: str
    variant: str            # "flare" or "flarepp"
    B: int
    N: int
    C: int
    H: int
    D: int
    M: int
    seed: int
    # FLARE++ inputs (bf16 bits)
    X: Optional[np.ndarray] = None        # [B][N][C]
    Wk: Optional[np.ndarray] = None       # [C][C]
    Wv: Optional[np.ndarray] = None
    Wk_syn: Optional[np.ndarray] = None
    Wv_syn: Optional[np.ndarray] = None
    Q0: Optional[np.ndarray] = None       # [H][M][D]
    Wo: Optional[np.ndarray] = None       # [C][C] output projection
    # FLARE inputs (bf16 bits)
    K: Optional[np.ndarray] = None        # [B][H][N][D]
    V: Optional[np.ndarray] = None
    Q: Optional[np.ndarray] = None        # [H][M][D]
    lengths: Optional[np.ndarray] = None  # int32 [B] or None

    @property
    def scale(self) -> float:
        return 1.0 / float(np.sqrt(self.D))

    def valid_tokens(self) -> int:
        if self.lengths is None:
            return self.B * self.N
        return int(np.sum(self.lengths))


def _features(rng, kind, B, N, C):
    if kind == "normal":
        return rng.standard_normal((B, N, C), dtype=np.float32)
    dim = {"mesh2d": 2, "mesh3d": 3}[kind]
    P = rng.random((B, N, dim), dtype=np.float64)           # coordinates
    A = rng.standard_normal((dim, C), dtype=np.float64)      # random lift
    E = rng.standard_normal((B, N, C), dtype=np.float32)     # noise
    X = np.empty((B, N, C), dtype=np.float32)
    for b in range(B):
        X[b] = (P[b] @ A).astype(np.float32) + E[b]
    return X


def make_workload(name: str, N: Optional[int] = None, B: Optional[int] = None,
                  M: Optional[int] = None, lengths: Optional[np.ndarray] = None,
                  seed: Optional[int] = None) -> Workload:
    """Draw the named workload.  N, B, M and seed may be overridden to get a
    reduced case with the same distributions; explicit ``lengths`` replace the
    drawn ones."""
    spec = dict(WORKLOADS[name])
    if N is not None:
        spec["N"] = int(N)
    if B is not None:
        spec["B"] = int(B)
    if M is not None:
        spec["M"] = int(M)
    if seed is not None:
        spec["seed"] = int(seed)
    Bv, Nv, C, H, D, Mv = (spec[k] for k in ("B", "N", "C", "H", "D", "M"))
    assert C == H * D
    rng = np.random.Generator(np.random.PCG64(spec["seed"]))
    gain = float(spec.get("weight_gain", 1.0))
    wstd = gain / np.sqrt(C)
    w = Workload(name=name, variant=spec["variant"], B=Bv, N=Nv, C=C, H=H, D=D,
                 M=Mv, seed=spec["seed"])
    if spec["variant"] == "flarepp":
        w.X = to_bf16_bits(_features(rng, spec["x"], Bv, Nv, C))
        w.Wk = to_bf16_bits(rng.standard_normal((C, C), dtype=np.float32) * wstd)
        w.Wv = to_bf16_bits(rng.standard_normal((C, C), dtype=np.float32) * wstd)
        w.Wk_syn = to_bf16_bits(rng.standard_normal((C, C), dtype=np.float32) * wstd)
        w.Wv_syn = to_bf16_bits(rng.standard_normal((C, C), dtype=np.float32) * wstd)
        w.Q0 = to_bf16_bits(rng.standard_normal((H, Mv, D), dtype=np.float32))
    else:
        # K = X W and V = X W for X ~ N(0,1), W ~ N(0,1/C) have N(0,1) entries;
        # FLARE's inputs are drawn from that distribution directly.
        w.K = to_bf16_bits(rng.standard_normal((Bv, H, Nv, D), dtype=np.float32))
        w.V = to_bf16_bits(rng.standard_normal((Bv, H, Nv, D), dtype=np.float32))
        w.Q = to_bf16_bits(rng.standard_normal((H, Mv, D), dtype=np.float32))
    if lengths is not None:
        w.lengths = np.ascontiguousarray(lengths, dtype=np.int32)
    elif "lengths" in spec:
        lo, hi = spec["lengths"]
        n0 = WORKLOADS[name]["N"]
        if Nv != n0:  # reduced case: keep the same fraction of valid tokens
            lo, hi = max(1, lo * Nv // n0), max(1, hi * Nv // n0)
        w.lengths = rng.integers(lo, hi + 1, size=Bv, dtype=np.int64).astype(np.int32)
    if spec["variant"] == "flarepp":  # drawn last, so the draws above do not depend on it
        w.Wo = to_bf16_bits(rng.standard_normal((C, C), dtype=np.float32) * wstd)
    return w


def make_upstream_grad(w: Workload, seed: Optional[int] = None) -> np.ndarray:
    """Upstream gradient dY = dLoss/dY [B][H][N][D] for the backward, N(0,1)
    in bf16 bits, from its own generator (seed: the workload's seed + 7919,
    unless given), so the workload's draws are unchanged.  Rows of padding
    tokens are drawn too: the backward must ignore them."""
    s = w.seed + 7919 if seed is None else int(seed)
    rng = np.random.Generator(np.random.PCG64(s))
    return to_bf16_bits(rng.standard_normal((w.B, w.H, w.N, w.D), dtype=np.float32))
