"""Shared helpers of the GPU tests: move workload bytes to the device, call the
CUDA library through its binding, and compare with the fp64 oracle (the
criteria live in ``parity.py``)."""
import numpy as np
import torch

import rank_latent_routing_flare_b200 as fl
from workloads import bf16_bits_to_f64

from .parity import MAX_ABS, REL_L2, check, max_abs, rel_l2  # noqa: F401


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def host_f64(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return bf16_bits_to_f64(t.view(torch.int16).cpu().numpy().view(np.uint16))
    return t.double().cpu().numpy()


def run_gpu(w, debug: bool = True):
    """Run the CUDA path on a workload; returns dict of float64 numpy arrays
    (with ``debug``: also Q(X), Z and the fp32 Y of the inspection call)."""
    lengths = None if w.lengths is None else torch.from_numpy(w.lengths).cuda()
    out = {"lengths": w.lengths}
    Y32 = torch.empty((w.B, w.H, w.N, w.D), dtype=torch.float32, device="cuda") if debug else None
    if w.variant == "flare":
        K, V, Q = dev_bf16(w.K), dev_bf16(w.V), dev_bf16(w.Q)
        Z = torch.empty((w.B, w.H, w.M, w.D), dtype=torch.float32, device="cuda") if debug else None
        Y = fl.flare_mixer_fwd(K, V, Q, lengths=lengths, Z_out=Z, Y_f32_out=Y32)
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
        Y = fl.flarepp_mixer_fwd(X, *Ws, Q0, lengths=lengths, Qx_out=Qx, Z_out=Z, Y_f32_out=Y32)
        torch.cuda.synchronize()
        out["Y"] = host_f64(Y)
        if debug:
            out["Qx"] = host_f64(Qx)
            out["Z"] = host_f64(Z)
    if debug:
        out["Y32"] = host_f64(Y32)
        # the bf16 output is the fp32 one rounded to nearest even
        from .parity import bf16_round
        assert np.array_equal(bf16_round(out["Y32"]), out["Y"])
    return out


def compare(gpu: dict, ref: dict, rows=None, label="", lengths=None, extra_rounding=None):
    """Assert the stated tolerance on Y, the bound on its token-centred part
    (bf16 and, when present, fp32) and the tolerance on the Q(X) / Z
    diagnostics; returns the measured errors."""
    if lengths is None:
        lengths = gpu.get("lengths")
    return check(gpu, ref, rows=rows, lengths=lengths, label=label, extra_rounding=extra_rounding)
