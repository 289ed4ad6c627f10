"""Shared helpers of the GPU tests: move workload bytes to the device, call the
CUDA library through its binding, and compare with the fp64 oracle."""
import numpy as np
import torch

import rank_latent_routing_flare_b200 as fl
from workloads import bf16_bits_to_f64

# Tolerance on the bf16 outputs with fp32 accumulation (stated target).
REL_L2 = 5e-3
MAX_ABS = 3e-2


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def host_f64(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return bf16_bits_to_f64(t.view(torch.int16).cpu().numpy().view(np.uint16))
    return t.double().cpu().numpy()


def rel_l2(a, b) -> float:
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def max_abs(a, b) -> float:
    return float(np.max(np.abs(np.asarray(a, np.float64) - np.asarray(b, np.float64))))


def run_gpu(w, debug: bool = True):
    """Run the CUDA path on a workload; returns dict of float64 numpy arrays."""
    lengths = None if w.lengths is None else torch.from_numpy(w.lengths).cuda()
    out = {}
    if w.variant == "flare":
        K, V, Q = dev_bf16(w.K), dev_bf16(w.V), dev_bf16(w.Q)
        Z = torch.empty((w.B, w.H, w.M, w.D), dtype=torch.float32, device="cuda") if debug else None
        Y = fl.flare_mixer_fwd(K, V, Q, lengths=lengths, Z_out=Z)
        torch.cuda.synchronize()
        out["Y"] = host_f64(Y)
        if debug:
            out["Z"] = host_f64(Z)
    else:
        X = dev_bf16(w.X)
        Ws = [dev_bf16(a) for a in (w.Wk, w.Wv, w.Wk_syn, w.Wv_syn)]
        Q0 = dev_bf16(w.Q0)
        Qx = torch.empty((w.B, w.H, w.M, w.D), dtype=torch.float32, device="cuda") if debug else None
        Z = torch.empty((w.B, w.H, w.M, w.D), dtype=torch.float32, device="cuda") if debug else None
        Y = fl.flarepp_mixer_fwd(X, *Ws, Q0, lengths=lengths, Qx_out=Qx, Z_out=Z)
        torch.cuda.synchronize()
        out["Y"] = host_f64(Y)
        if debug:
            out["Qx"] = host_f64(Qx)
            out["Z"] = host_f64(Z)
    return out


def compare(gpu: dict, ref: dict, rows=None, label=""):
    """Assert the stated tolerance on Y (and on the Q(X) / Z diagnostics);
    returns the measured errors."""
    errs = {}
    Yg = gpu["Y"] if rows is None else gpu["Y"][:, :, rows]
    errs["Y_rel_l2"] = rel_l2(Yg, ref["Y"])
    errs["Y_max_abs"] = max_abs(Yg, ref["Y"])
    for k in ("Qx", "Z"):
        if k in gpu and k in ref:
            errs[f"{k}_rel_l2"] = rel_l2(gpu[k], ref[k])
    print(label, {k: f"{v:.3e}" for k, v in errs.items()})
    assert np.all(np.isfinite(Yg)), label
    assert errs["Y_rel_l2"] <= REL_L2, (label, errs)
    assert errs["Y_max_abs"] <= MAX_ABS, (label, errs)
    for k in ("Qx_rel_l2", "Z_rel_l2"):
        if k in errs:
            assert errs[k] <= REL_L2, (label, errs)
    return errs
