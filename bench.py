#!/usr/bin/env python
"""Benchmark of the FLARE++ mixer forward on B200.

One step = one ``flarepp_mixer_fwd`` call over the N = 1,048,576-token
workload (B=1, C=128, H=8, D=16, M=512; 3-D point cloud lifted to C features):
the four per-head projections, the query-synthesis encode, the encode with
the synthesised queries, both log-sum-exp merges and the decode.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    python bench.py --backward [--workload NAME] ...   # the backward: its own JSON line
    python bench.py --train [--workload NAME] ...      # a training step (forward + backward)

Prints one JSON line (rank 0).  ``value`` is whole-job token*heads/s with the
inputs resident in HBM, timed with CUDA events on the launching stream over
exactly K steps (max over ranks).  ``e2e`` is the same metric with every
step's host->device copy of its inputs (pinned memory) and device->host copy
of Y inside the timed region; the copies run on their own streams into double
buffers, so those of neighbouring steps overlap the current step's compute.
The timed steps run without events between the kernels; the per-stage times
come from as many steps with stage events, run after the timed region.
``roofline`` reports the dominant kernel against the exp-unit bound, from the
ex2 and fp32-fma rates measured on the device by the library's probe: ``frac``
(= ``frac_combined``) against the best split of the exponentials between the
special-function unit and an FMA-pipe polynomial, ``frac_mufu_only`` against
the special-function unit alone.  ``cpu_baseline`` is the fp64 oracle on a
bounded sample of the same workload on this host's cores.  ``--impl
reference`` times the oracle itself as the reference arm.

With ``--gpus N`` (launched through torch.distributed.run) every rank runs an
independent copy of the workload on its own synthetic input (weak scaling; the
heads and samples of the mixer are independent, so there is no data-path
collective).

``--backward`` times one ``flarepp_mixer_bwd`` call (``flare_mixer_bwd`` for a
FLARE workload) per step with a seeded upstream gradient dY, against the
backward's own roofline (three exponentials per score, the tensor term at half
the bf16 rate, HBM); ``e2e`` then copies the inputs and dY in and every
gradient out.
``--train`` times a training step instead: the training forward
(``flarepp_mixer_fwd_train``), which keeps its state, and the backward that
reuses it (``flarepp_mixer_bwd_train``), against the sum of the forward's and
the backward's rooflines; ``compare`` gives the plain forward + the
self-contained backward (which runs the forward's kernels again) on the same
inputs, timed after the timed region.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from workloads import make_workload  # noqa: E402

METRIC = "mixer fwd token·heads/s at N=1M (1×B200) and % of roofline (HBM/MMA/MUFU)"
UNIT = "token·heads/s"
WORKLOAD = "flarepp_n1m_mesh3d"
MUFU_PER_CLK_PER_SM = 16          # nominal ex2 results per clock per SM (used only if the probe fails)
FMA_PER_CLK_PER_SM = 128          # nominal fp32 fma per clock per SM (ditto)
NUM_SM = 148
# Issue-slot cost of the softmax's own arithmetic per score (the kernels'
# exponential step, thread instructions, with the paired fp32x2 forms the
# kernels use): half a paired FFMA for the scale-and-shift and half a bf16x2
# pack, plus the exponential itself -- one MUFU instruction, or 6 for the
# FMA-pipe polynomial (per pair of scores: 2 clamps, 2 paired adds for the
# range reduction, 4 paired FFMAs for the remainder and the cubic, 2 shifts
# and 2 integer adds for the exponent: 12).
SOFTMAX_BASE_OPS = 1.0
POLY_EXP_OPS = 6.0
STAGES_PP = ["project", "synth_encode", "synth_merge", "encode", "merge", "decode"]
KERNEL_SOURCES = {"project": "project.cu", "synth_encode": "encode.cu", "encode": "encode.cu",
                  "synth_merge": "merge.cu", "merge": "merge.cu", "decode": "decode.cu"}


def log(*a):
    print(*a, file=sys.stderr, flush=True)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]),
                "sm_max_mhz": d.get("sm_max_mhz", 1965.0), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0,
            "source": "fallback"}


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML, read only)
# ---------------------------------------------------------------------------

class ClockSampler:
    """Samples SM clock, power and clock-event reasons with ``nvidia-smi -lms``
    (a separate process, read only) while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, device_index: int, period_ms: int = 20, path: str | None = None):
        import tempfile
        self.dev = device_index
        self.period = period_ms
        self.path = path or tempfile.mktemp(prefix="flare_clocks_", suffix=".csv")
        self.proc = None
        self.lines = []

    def __enter__(self):
        import shutil
        import subprocess
        if shutil.which("nvidia-smi") is None:
            log("nvidia-smi not found: no clock samples")
            return self
        self.fh = open(self.path, "w")
        self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                      f"-lms={self.period}", "-i", str(self.dev)], stdout=self.fh,
                                     stderr=subprocess.DEVNULL)
        t0 = time.time()
        while time.time() - t0 < 10 and os.path.getsize(self.path) == 0:
            time.sleep(0.01)
        self.skip = sum(1 for _ in open(self.path))   # samples taken before the timed region
        return self

    def __exit__(self, *exc):
        if self.proc is None:
            return
        time.sleep(self.period / 1000.0)
        self.proc.terminate()
        self.proc.wait(timeout=10)
        self.fh.close()
        self.lines = [ln.strip() for ln in open(self.path) if ln.strip()][self.skip:]
        try:
            os.remove(self.path)
        except OSError:
            pass

    def summary(self):
        mhz, mx, pw, reasons = [], None, [], set()
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                mhz.append(float(f[1]))
                mx = float(f[2])
                pw.append(float(f[3]))
            except ValueError:
                continue
            for name, val in zip(self.NAMES, f[5:9]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": float(statistics.median(mhz)) if mhz else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(mhz),
                "power_w_median": float(statistics.median(pw)) if pw else None}


# ---------------------------------------------------------------------------
# algorithmic work per stage (FLARE++), per launch
# ---------------------------------------------------------------------------

def stage_work(w):
    B, N, C, H, D, M = w.B, w.N, w.C, w.H, w.D, w.M
    Nv = w.valid_tokens() // B if w.lengths is not None else N
    th = B * H * Nv                                   # token*heads
    proj_bytes = B * N * C * 2 + 4 * C * C * 2 + 4 * B * H * N * D * 2
    enc_exps = th * M                                 # one exponential per (latent, token) score
    enc_flops = 4 * th * M * D                        # Q K^T and P V
    enc_bytes = 2 * B * H * N * D * 2
    dec_bytes = 2 * B * H * N * D * 2                 # read K, write Y
    return {
        "project": {"bytes": proj_bytes, "flops": 8 * B * N * C * C, "exps": 0},
        "synth_encode": {"bytes": enc_bytes, "flops": enc_flops, "exps": enc_exps},
        "synth_merge": {"bytes": 0, "flops": 0, "exps": 0},
        "encode": {"bytes": enc_bytes, "flops": enc_flops, "exps": enc_exps},
        "merge": {"bytes": 0, "flops": 0, "exps": 0},
        "decode": {"bytes": dec_bytes, "flops": enc_flops, "exps": enc_exps},
    }


def pipe_rates(fl, dev) -> dict:
    """ex2 (MUFU) and fp32 fma (FMA pipe) results per clock per SM, measured
    on this device by the library's probe kernels; nominal values if the
    probe fails (then labelled so)."""
    try:
        r = fl.flare_probe_pipe_rates(dev)
        if r["ex2"] > 0 and r["ffma"] > 0:
            return {"ex2": r["ex2"], "ffma": r["ffma"], "source": "measured (flare_probe_pipe_rates)"}
    except Exception as e:  # noqa: BLE001
        log(f"pipe probe failed: {e}")
    return {"ex2": float(MUFU_PER_CLK_PER_SM), "ffma": float(FMA_PER_CLK_PER_SM), "source": "nominal"}


def exp_unit_bounds(rates: dict) -> dict:
    """Clocks per score per SM of the softmax's exponential step under two
    bounds:

    - mufu_only: every exponential on the special-function unit (1 / ex2 rate);
    - combined: a fraction f of the exponentials on the FMA-pipe polynomial,
      chosen to balance the MUFU against the issue slots (one instruction per
      clock per sub-partition, measured as the fma rate), which every
      instruction of the step takes: t = max((1 - f) / ex2, (base + (1 - f)
      + poly * f) / issue).  The best any MUFU/polynomial split of this
      arithmetic can reach."""
    ex2, issue = rates["ex2"], rates["ffma"]
    r = issue / ex2
    f = min(1.0, max(0.0, (r - SOFTMAX_BASE_OPS - 1.0) / (r + POLY_EXP_OPS - 1.0)))
    t_comb = max((1.0 - f) / ex2, (SOFTMAX_BASE_OPS + (1.0 - f) + POLY_EXP_OPS * f) / issue)
    return {"mufu_only": 1.0 / ex2, "combined": t_comb, "poly_fraction": f}


def kernel_traffic(kernel_file: str, workload: str):
    """dram bytes per launch from a committed ncu summary, if that summary was
    taken on the current source of the kernel (its .cu file, ptx.cuh and
    flare_internal.h); else None."""
    prof = os.path.join(ROOT, "profiles")
    csrc = os.path.join(ROOT, "rank_latent_routing_flare_b200", "csrc")
    srcs = [os.path.join(csrc, f) for f in (kernel_file, "ptx.cuh", "flare_internal.h")]
    if not os.path.isdir(prof) or not all(os.path.exists(f) for f in srcs):
        return None
    h = hashlib.sha256()
    for f in srcs:
        h.update(open(f, "rb").read())
    sha = h.hexdigest()[:16]
    for f in sorted(os.listdir(prof)):
        if not f.endswith(".md"):
            continue
        text = open(os.path.join(prof, f)).read()
        m_src = re.search(r"kernel_source_sha256_16:\s*(\w+)", text)
        m_w = re.search(r"workload:\s*(\S+)", text)
        m_k = re.search(r"kernel_file:\s*(\S+)", text)
        m_t = re.search(r"dram_bytes_per_launch_full_size:\s*([0-9.eE+]+)", text)
        if m_src and m_t and m_k and m_w and m_src.group(1) == sha and m_k.group(1) == kernel_file \
                and m_w.group(1) == workload:
            return float(m_t.group(1))
    return None


# ---------------------------------------------------------------------------
# ranks (weak scaling: every rank runs its own copy of the workload)
# ---------------------------------------------------------------------------

LAUNCHES_PER_STEP = 7   # project, synth encode, synth merge, encode, merge, decode, decode fallback


def rank_seed(rank: int):
    """Seed of a rank's synthetic input: rank 0 uses the workload's own seed."""
    return None if rank == 0 else 1000 + rank


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest value of x over all ranks (every rank gets it)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, units_per_rank: float, ms: float) -> float:
    """Units processed by all ranks per second, timed by the slowest rank."""
    return world * units_per_rank / (ms * 1e-3)


# ---------------------------------------------------------------------------
# CPU baseline: the fp64 oracle on a bounded sample of the workload
# ---------------------------------------------------------------------------

def oracle_sample_rate(w, target_s: float):
    import oracle
    from workloads import bf16_bits_to_f64 as f64
    oracle.build()
    W = [f64(a) for a in (w.Wk, w.Wv, w.Wk_syn, w.Wv_syn)]
    Q0 = f64(w.Q0)

    def run(ns):
        X = f64(w.X[:, :ns])
        t0 = time.perf_counter()
        oracle.flarepp_forward(X, *W, Q0, w.H, None, w.scale)
        return time.perf_counter() - t0

    ns = min(4096, w.N)
    t = run(ns)
    while t < target_s / 4 and ns < w.N:
        ns = min(w.N, int(ns * min(8.0, max(2.0, target_s / max(t, 1e-3)))))
        t = run(ns)
    rate = w.B * w.H * ns / t
    return rate, ns, t, oracle.num_threads()


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


# ---------------------------------------------------------------------------
# backward (gradients): a separate line, not the headline
# ---------------------------------------------------------------------------

BWD_METRIC = "mixer bwd token·heads/s at N=1M (1×B200) and % of roofline (HBM/MMA/MUFU)"
# a training step, by (variant, D): the training forward (the forward's
# kernels; at D = 16 plus the fp16 copy of Z) and the training backward (mark
# check, conversions, pads, the decoder's delta or statistics, the latent- and
# token-parallel passes with their sums and operand splits, the projection
# gradients)
TRAIN_LAUNCHES = {("flarepp", 16): 8 + 24, ("flarepp", 32): 7 + 24, ("flare", 16): 6 + 14, ("flare", 32): 5 + 14}
# a self-contained backward call runs the same launches without the mark check
BWD_LAUNCHES = {k: v - 1 for k, v in TRAIN_LAUNCHES.items()}
TRAIN_METRIC = "mixer training step (fwd+bwd) token·heads/s at N=1M (1×B200) and % of roofline"
# The backward's products take one operand (Z, dZ, dQ(X), dS or the gradient
# rows, fp32) as two bf16 parts, so most of them cost two bf16 MMAs: half the
# bf16 rate per useful flop (the nominal dense tf32 : bf16 ratio as well)
SPLIT_PER_BF16 = 0.5


def backward_work(w):
    """Algorithmic work of one backward call: one exponential per score of
    each SDPA call (three for FLARE++, two for FLARE); per call the score
    recompute and the four gradient products (5 x 2MD flop per token·head);
    FLARE++ adds the projection gradients dX and dW (2 x 4 x 2 C D flop per
    token·head).  HBM: FLARE++ reads X and dY and writes dX; FLARE reads K, V
    and dY and writes dK and dV.  Token counts are valid (unpadded) tokens,
    as in the forward's work model."""
    th = w.H * w.valid_tokens()
    if w.variant == "flare":
        return {"exps": 2 * w.M * th, "flops": 2 * 5 * 2 * w.M * w.D * th, "bytes": 5 * th * w.D * 2}
    return {"exps": 3 * w.M * th, "flops": (3 * 5 * 2 * w.M * w.D + 16 * w.C * w.D) * th,
            "bytes": 3 * w.valid_tokens() * w.C * 2}


def oracle_backward_rate(w, dY, target_s: float):
    import oracle
    from workloads import bf16_bits_to_f64 as f64
    oracle.build()
    W = [f64(a) for a in (w.Wk, w.Wv, w.Wk_syn, w.Wv_syn)] if w.variant != "flare" else None
    Q0 = f64(w.Q0) if w.variant != "flare" else None

    def run(ns):
        t0 = time.perf_counter()
        if w.variant == "flare":
            oracle.flare_backward(f64(w.K[:, :, :ns]), f64(w.V[:, :, :ns]), f64(w.Q), f64(dY[:, :, :ns]), None,
                                  w.scale)
        else:
            oracle.flarepp_backward(f64(w.X[:, :ns]), *W, Q0, f64(dY[:, :, :ns]), w.H, None, w.scale)
        return time.perf_counter() - t0

    ns = min(2048, w.N)
    t = run(ns)
    while t < target_s / 4 and ns < w.N:
        ns = min(w.N, int(ns * min(8.0, max(2.0, target_s / max(t, 1e-3)))))
        t = run(ns)
    return w.B * w.H * ns / t, ns, t, oracle.num_threads()


def run_backward(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    import rank_latent_routing_flare_b200 as fl
    from workloads import make_upstream_grad

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    fl.load_library()
    w = make_workload(args.workload, N=args.tokens, seed=rank_seed(rank))
    dY_bits = make_upstream_grad(w)

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    flare = w.variant == "flare"
    train = args.train
    dY = to_dev(dY_bits)
    if flare:
        host_inputs = (w.K, w.V, w.Q)
        K, V, Q = (to_dev(a) for a in host_inputs)
        dev_inputs = (K, V, Q)
        nbytes = fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLARE_BWD, w.B, w.H, w.N, w.M, w.D)
    else:
        host_inputs = (w.X, w.Wk, w.Wv, w.Wk_syn, w.Wv_syn, w.Q0)
        dev_inputs = tuple(to_dev(a) for a in host_inputs)
        nbytes = fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLAREPP_BWD, w.B, w.H, w.N, w.M, w.D, w.C)
    lengths = None if w.lengths is None else torch.from_numpy(w.lengths).to(dev)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    grads = None
    Y = torch.empty((w.B, w.H, w.N, w.D), dtype=torch.bfloat16, device=dev)

    def step(training=train, with_forward=train):
        """One backward call; with ``with_forward`` a training step: the
        forward, then the backward (the training pair if ``training``, else
        the plain forward and the recomputing backward)."""
        nonlocal grads
        if flare:
            if with_forward:
                if training:
                    fl.flare_mixer_fwd_train(*dev_inputs, lengths=lengths, Y=Y, workspace=ws, stream=stream,
                                             check=False)
                else:
                    fl.flare_mixer_fwd(*dev_inputs, lengths=lengths, Y=Y, workspace=ws, stream=stream, check=False)
            out = (None, None, None) if grads is None else (grads["dK"], grads["dV"], grads["dQ"])
            if training:
                dK, dV, dQ = fl.flare_mixer_bwd_train(*dev_inputs, dY, ws, lengths=lengths, stream=stream,
                                                      dK=out[0], dV=out[1], dQ=out[2], check=False)
            else:
                dK, dV, dQ = fl.flare_mixer_bwd(*dev_inputs, dY, lengths=lengths, workspace=ws, stream=stream,
                                                dK=out[0], dV=out[1], dQ=out[2], check=False)
            grads = {"dK": dK, "dV": dV, "dQ": dQ}
        else:
            if with_forward:
                if training:
                    fl.flarepp_mixer_fwd_train(*dev_inputs, lengths=lengths, Y=Y, workspace=ws, stream=stream,
                                               check=False)
                else:
                    fl.flarepp_mixer_fwd(*dev_inputs, lengths=lengths, Y=Y, workspace=ws, stream=stream,
                                         check=False)
            if training:
                grads = fl.flarepp_mixer_bwd_train(*dev_inputs, dY, ws, lengths=lengths, stream=stream,
                                                   grads=grads, check=False)
            else:
                grads = fl.flarepp_mixer_bwd(*dev_inputs, dY, lengths=lengths, workspace=ws, stream=stream,
                                             grads=grads, check=False)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    st = fl.flare_last_device_status(ws)
    if st != fl.Status.OK:
        raise RuntimeError(f"device status after warm-up: {st!r}")

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clocks:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        ev0.record(stream)
        for _ in range(args.steps):
            step()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1) / args.steps, world, dev)
    th_per_rank = w.B * w.H * (w.valid_tokens() // w.B if w.lengths is not None else w.N)
    value = whole_job_rate(world, th_per_rank, ms)
    compare = None
    if train:
        # the same training step with the plain forward and the recomputing
        # backward, for comparison (after the timed region)
        n_cmp = min(args.steps, 10)
        step(training=False, with_forward=True)
        torch.cuda.synchronize(dev)
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record(stream)
        for _ in range(n_cmp):
            step(training=False, with_forward=True)
        c1.record(stream)
        torch.cuda.synchronize(dev)
        compare = {"recomputing_pair_ms": round(max_over_ranks(c0.elapsed_time(c1) / n_cmp, world, dev), 4),
                   "steps": n_cmp, "what": "flare(pp)_mixer_fwd + flare(pp)_mixer_bwd on the same inputs"}

    peaks = load_peaks()
    rates = pipe_rates(fl, dev)
    mufu_peak = rates["ex2"] * NUM_SM * peaks["sm_max_mhz"] * 1e6
    split_peak = peaks["bf16_tflops"] * 1e12 * SPLIT_PER_BF16
    wk = backward_work(w)
    terms = {"hbm": wk["bytes"] / (peaks["hbm_gbs"] * 1e9), "mma": wk["flops"] / split_peak,
             "mufu": wk["exps"] / mufu_peak}
    if train:
        # plus the forward: its exponentials, its bf16 tensor products and its
        # HBM traffic (the stage model of the forward; FLARE: encode + decode)
        sw = stage_work(w)
        keys = ("encode", "merge", "decode") if flare else tuple(sw)
        terms["hbm"] += sum(sw[k]["bytes"] for k in keys) / (peaks["hbm_gbs"] * 1e9)
        terms["mma"] += sum(sw[k]["flops"] for k in keys) / (peaks["bf16_tflops"] * 1e12)
        terms["mufu"] += sum(sw[k]["exps"] for k in keys) / mufu_peak
    t_roof = max(terms.values())
    bound = {"hbm": "hbm", "mma": "tensor", "mufu": "alu"}[max(terms, key=terms.get)]

    # end to end: inputs and dY in from pinned host memory, gradients back out,
    # all inside the timed region on the call's stream
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).pin_memory()  # noqa: E731
    h_in = [pin(a) for a in (*host_inputs, dY_bits)]
    d_in = [t.view(torch.int16) for t in (*dev_inputs, dY)]
    h_out = {k: torch.empty(v.shape, dtype=v.dtype).pin_memory() for k, v in grads.items()}
    h2d = sum(a.numel() * 2 for a in h_in)
    d2h = sum(v.numel() * v.element_size() for v in grads.values())

    def e2e_step():
        for d, h in zip(d_in, h_in):
            d.copy_(h, non_blocking=True)
        step()
        for k, v in grads.items():
            h_out[k].copy_(v, non_blocking=True)

    e2e_ms = float("nan")
    if args.e2e_steps > 0:
        e2e_step()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = e0.elapsed_time(e1) / args.e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, world, dev)

    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            rate, ns, t, threads = oracle_backward_rate(w, dY_bits, args.cpu_seconds)
            cpu = {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle",
                   "sample": f"fp64 oracle, full {'FLARE' if flare else 'FLARE++'} backward (which computes the "
                             f"forward's values on the way) on the first {ns} "
                             f"of {w.N} tokens (B={w.B} H={w.H} M={w.M} D={w.D} C={w.C}) in {t:.1f} s; "
                             f"{cpu_model()}"}
        line = {
            "metric": TRAIN_METRIC if train else BWD_METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "pass": "training step" if train else "backward", "B": w.B, "N": w.N, "C": w.C, "H": w.H,
                       "D": w.D, "M": w.M, "parallelism": f"replicas{world}" if world > 1 else "single",
                       "l2": ("inputs larger than L2 (K, V, dY: " +
                              f"{3 * w.B * w.H * w.N * w.D * 2 / 2**20:.0f} MiB together)" if flare else
                              "inputs larger than L2 (X 256 MiB, dY 256 MiB, gradient rows 2 GiB)")},
            "step_roofline": {"t_roof_ms": round(t_roof * 1e3, 4), "frac": round(t_roof / (ms * 1e-3), 4),
                              "bound": bound, "terms_ms": {k: round(v * 1e3, 4) for k, v in terms.items()},
                              "peak_basis": f"MUFU {rates['ex2']:.2f} ex2/clk/SM ({rates['source']}) x {NUM_SM} x "
                                            f"{peaks['sm_max_mhz']:.0f} MHz; tensor = {SPLIT_PER_BF16} x measured "
                                            f"bf16 {peaks['bf16_tflops']} TFLOP/s (fp32 operands as two bf16 parts); "
                                            f"HBM {peaks['hbm_gbs']} GB/s "
                                            f"({peaks['source']})"},
            "cpu_baseline": cpu,
            "e2e": {"value": whole_job_rate(world, th_per_rank, e2e_ms), "unit": UNIT,
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": (TRAIN_LAUNCHES if train else BWD_LAUNCHES)[(w.variant, w.D)] * args.steps,
            "compare": compare,
            "clocks": clocks.summary(),
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ---------------------------------------------------------------------------
# reference arm: the oracle timed as it stands
# ---------------------------------------------------------------------------

def run_reference(args, rank, world):
    if rank != 0:
        return 0
    w = make_workload(args.workload)
    import oracle
    from workloads import bf16_bits_to_f64 as f64
    oracle.build()
    W = [f64(a) for a in (w.Wk, w.Wv, w.Wk_syn, w.Wv_syn)]
    Q0 = f64(w.Q0)
    # each step: the full FLARE++ forward on a bounded token sample, sized so
    # that the whole run stays within a few minutes
    budget = 150.0 / max(1, args.steps + args.warmup)
    rate, ns, t, threads = oracle_sample_rate(w, min(budget, 20.0))
    X = f64(w.X[:, :ns])
    for _ in range(args.warmup):
        oracle.flarepp_forward(X, *W, Q0, w.H, None, w.scale)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.flarepp_forward(X, *W, Q0, w.H, None, w.scale)
    dt = (time.perf_counter() - t0) / args.steps
    value = w.B * w.H * ns / dt
    sample = (f"FLARE++ forward (projections, synthesis, encode, decode) on the first {ns} of "
              f"{w.N} tokens, B={w.B} H={w.H} M={w.M} D={w.D} C={w.C}; fp64 oracle, {threads} threads, "
              f"{cpu_model()}")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "N": w.N, "C": w.C, "H": w.H, "D": w.D, "M": w.M,
                       "sample_tokens": ns},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--tokens", type=int, default=None,
                    help="override N (smaller cases for profiling; not a bench line)")
    ap.add_argument("--e2e-steps", type=int, default=8)
    ap.add_argument("--cpu-seconds", type=float, default=15.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--backward", action="store_true",
                    help="time the FLARE++ backward (gradients) instead of the forward; its own JSON line")
    ap.add_argument("--train", action="store_true",
                    help="with --backward: time a training step, the training forward that keeps its state and "
                         "the backward that reuses it (and, for comparison, the plain forward + backward)")
    ap.add_argument("--graph", action="store_true",
                    help="time replays of one step captured as a CUDA graph (no per-launch host cost); the "
                         "stage times come from as many eager steps with stage events after the timed region")
    args = ap.parse_args()
    if args.warmup < 3:
        log("warm-up raised to the minimum of 3 steps")
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.backward or args.train:
        return run_backward(args, rank, world, local_rank)

    import torch
    import torch.distributed as dist
    import rank_latent_routing_flare_b200 as fl

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    fl.load_library()

    # inputs: each rank its own synthetic sample of the workload (weak scaling)
    w = make_workload(args.workload, N=args.tokens, seed=rank_seed(rank))
    assert w.variant == "flarepp"

    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(dev)

    X = to_dev(w.X)
    Ws = [to_dev(a) for a in (w.Wk, w.Wv, w.Wk_syn, w.Wv_syn)]
    Q0 = to_dev(w.Q0)
    lengths = None if w.lengths is None else torch.from_numpy(w.lengths).to(dev)
    Y = torch.empty((w.B, w.H, w.N, w.D), dtype=torch.bfloat16, device=dev)
    nbytes = fl.flare_workspace_bytes(fl.FLARE_VARIANT_FLAREPP, w.B, w.H, w.N, w.M, w.D, w.C)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    stage_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(7)] for _ in range(args.steps)]

    def step(events=None, st=None):
        fl.flarepp_mixer_fwd(X, *Ws, Q0, lengths=lengths, Y=Y, workspace=ws, stream=st or stream, check=False,
                             stage_events=events)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    st = fl.flare_last_device_status(ws)
    if st != fl.Status.OK:
        raise RuntimeError(f"device status after warm-up: {st!r}")

    graph = None
    if args.graph:  # one step captured once and replayed
        graph = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream(dev)
        cap.wait_stream(stream)
        with torch.cuda.graph(graph, stream=cap):
            step(None, st=cap)
        stream.wait_stream(cap)
        for _ in range(args.warmup):
            graph.replay()
        torch.cuda.synchronize(dev)

    # ---------------- timed region (inputs resident in HBM) ----------------
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clocks:
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        ev0.record(stream)
        for i in range(args.steps):
            if graph is not None:
                graph.replay()
            else:
                step()
        ev1.record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
    ms = max_over_ranks(ev0.elapsed_time(ev1) / args.steps, world, dev)
    th_per_rank = w.B * w.H * (w.valid_tokens() // w.B if w.lengths is not None else w.N)
    value = whole_job_rate(world, th_per_rank, ms)

    # per-stage device times: as many steps again, after the timed region,
    # with CUDA events between the stages (the timed steps run without them:
    # an event between two kernels keeps the second from starting early)
    for i in range(args.steps):
        step(stage_ev[i])
    torch.cuda.synchronize(dev)
    stage_ms = {s: 0.0 for s in STAGES_PP}
    for evs in stage_ev:
        for j, s in enumerate(STAGES_PP):
            stage_ms[s] += evs[j].elapsed_time(evs[j + 1]) / args.steps
    work = stage_work(w)
    peaks = load_peaks()
    clk = clocks.summary()
    rates = pipe_rates(fl, dev)
    bounds = exp_unit_bounds(rates)
    sm_hz = NUM_SM * peaks["sm_max_mhz"] * 1e6
    exp_peak = {k: sm_hz / bounds[k] for k in ("mufu_only", "combined")}   # exps/s at the maximum clock
    mufu_peak_max = exp_peak["mufu_only"]
    stages = {}
    for s in STAGES_PP:
        t = stage_ms[s] * 1e-3
        wk = work[s]
        stages[s] = {"ms": round(stage_ms[s], 4),
                     "GB_s": round(wk["bytes"] / t / 1e9, 1) if wk["bytes"] else None,
                     "TFLOP_s": round(wk["flops"] / t / 1e12, 2) if wk["flops"] else None,
                     "Gexp_s": round(wk["exps"] / t / 1e9, 1) if wk["exps"] else None}
    # the dominant kernel: largest share of the step (the two encoder launches
    # are one kernel)
    kern_ms = {"encode": stage_ms["synth_encode"] + stage_ms["encode"], "decode": stage_ms["decode"],
               "project": stage_ms["project"], "merge": stage_ms["synth_merge"] + stage_ms["merge"]}
    dom = max(kern_ms, key=kern_ms.get)
    if dom in ("encode", "decode"):
        per_launch_ms = kern_ms[dom] / (2 if dom == "encode" else 1)
        exps = work["encode" if dom == "encode" else "decode"]["exps"]
        achieved = exps / (per_launch_ms * 1e-3) / 1e9
        roof = {"kernel": f"{dom}_kernel", "bound": "alu", "achieved": round(achieved, 1),
                "peak": round(exp_peak["combined"] / 1e9, 1), "unit": "Gexp/s",
                "frac": round(achieved / (exp_peak["combined"] / 1e9), 4),
                "frac_combined": round(achieved / (exp_peak["combined"] / 1e9), 4),
                "frac_mufu_only": round(achieved / (exp_peak["mufu_only"] / 1e9), 4),
                "peak_mufu_only": round(exp_peak["mufu_only"] / 1e9, 1),
                "peak_basis": (f"ex2 {rates['ex2']:.2f}/clk/SM and fma (issue) {rates['ffma']:.2f}/clk/SM "
                               f"({rates['source']}) x {NUM_SM} SMs x {peaks['sm_max_mhz']:.0f} MHz; combined: "
                               f"{bounds['poly_fraction']:.3f} of the exps on a {POLY_EXP_OPS:g}-instruction "
                               f"polynomial, {SOFTMAX_BASE_OPS:g} more instructions per score"),
                "per_launch_ms": round(per_launch_ms, 4),
                "traffic": kernel_traffic(f"{dom}.cu", w.name)}
        if clk.get("sm_mhz"):
            roof["frac_at_observed_clock"] = round(
                achieved / (exp_peak["combined"] / 1e9 * clk["sm_mhz"] / peaks["sm_max_mhz"]), 4)
    elif dom == "project":
        per = kern_ms[dom]
        achieved = work["project"]["bytes"] / (per * 1e-3) / 1e9
        roof = {"kernel": "project_kernel", "bound": "hbm", "achieved": round(achieved, 1),
                "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(achieved / peaks["hbm_gbs"], 4),
                "per_launch_ms": round(per, 4), "traffic": kernel_traffic("project.cu", w.name)}
    else:
        roof = {"kernel": "merge_kernel", "bound": "hbm", "achieved": None, "peak": peaks["hbm_gbs"],
                "unit": "GB/s", "frac": None, "traffic": None}
    roof["peak_source"] = rates["source"] if roof["bound"] == "alu" else peaks["source"]
    # whole-step roofline: max(bytes / HBM peak, MMA flops / tensor peak, exps / MUFU peak)
    tot_bytes = 3 * w.B * w.N * w.C * 2 + w.B * w.H * w.N * w.D * 2
    tot_exps = sum(work[s]["exps"] for s in STAGES_PP)
    tot_flops = sum(work[s]["flops"] for s in STAGES_PP)
    t_hbm, t_mma = tot_bytes / (peaks["hbm_gbs"] * 1e9), tot_flops / (peaks["bf16_tflops"] * 1e12)
    t_roof = max(t_hbm, t_mma, tot_exps / exp_peak["combined"])
    t_roof_mufu = max(t_hbm, t_mma, tot_exps / exp_peak["mufu_only"])
    step_roofline = {"t_roof_ms": round(t_roof * 1e3, 4), "frac": round(t_roof / (ms * 1e-3), 4),
                     "frac_combined": round(t_roof / (ms * 1e-3), 4),
                     "frac_mufu_only": round(t_roof_mufu / (ms * 1e-3), 4),
                     "terms_ms": {"hbm": round(t_hbm * 1e3, 4), "mma": round(t_mma * 1e3, 4),
                                  "exp_combined": round(tot_exps / exp_peak["combined"] * 1e3, 4),
                                  "exp_mufu_only": round(tot_exps / exp_peak["mufu_only"] * 1e3, 4)},
                     "pipe_rates": {"ex2_per_clk_sm": round(rates["ex2"], 3),
                                    "ffma_per_clk_sm": round(rates["ffma"], 3), "source": rates["source"]}}

    # ---------------- end to end through the public API ----------------
    # Every step copies its inputs (X, the four weights, Q0) in from pinned host
    # memory and its output Y back out, each on its own stream.  Inputs and
    # outputs are double-buffered on the device, so the copies of neighbouring
    # steps overlap the current step's compute, as a serving loop would run.
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).pin_memory()  # noqa: E731
    hX = pin(w.X)
    hW = [pin(a) for a in (w.Wk, w.Wv, w.Wk_syn, w.Wv_syn)]
    hQ0 = pin(w.Q0)
    hY = [torch.empty((w.B, w.H, w.N, w.D), dtype=torch.int16).pin_memory() for _ in range(2)]
    dX = [X.view(torch.int16), torch.empty_like(X).view(torch.int16)]
    dW = [[a.view(torch.int16) for a in Ws], [torch.empty_like(a).view(torch.int16) for a in Ws]]
    dQ0 = [Q0.view(torch.int16), torch.empty_like(Q0).view(torch.int16)]
    dY = [Y, torch.empty_like(Y)]
    h2d = hX.numel() * 2 + sum(a.numel() * 2 for a in hW) + hQ0.numel() * 2
    d2h = hY[0].numel() * 2
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_done = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(i):
        k = i % 2
        if i >= 2:
            s_in.wait_event(ev_done[k])      # step i-2 has finished reading buffer k
        with torch.cuda.stream(s_in):
            dX[k].copy_(hX, non_blocking=True)
            for d, h in zip(dW[k], hW):
                d.copy_(h, non_blocking=True)
            dQ0[k].copy_(hQ0, non_blocking=True)
            ev_in[k].record(s_in)
        stream.wait_event(ev_in[k])
        if i >= 2:
            stream.wait_event(ev_out[k])     # Y buffer k has been copied out
        fl.flarepp_mixer_fwd(dX[k].view(torch.bfloat16), *[a.view(torch.bfloat16) for a in dW[k]],
                             dQ0[k].view(torch.bfloat16), lengths=lengths, Y=dY[k], workspace=ws, stream=stream,
                             check=False)
        ev_done[k].record(stream)
        s_out.wait_event(ev_done[k])
        with torch.cuda.stream(s_out):
            hY[k].copy_(dY[k].view(torch.int16), non_blocking=True)
            ev_out[k].record(s_out)

    e2e_ms = float("nan")
    if args.e2e_steps > 0:
        for i in range(2):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(s_in)
        for i in range(args.e2e_steps):
            e2e_step(i)
        e1.record(s_out)
        torch.cuda.synchronize(dev)
        e2e_ms = e0.elapsed_time(e1) / args.e2e_steps
    e2e_ms = max_over_ranks(e2e_ms, world, dev)
    if world > 1:
        dist.barrier()
    e2e_value = whole_job_rate(world, th_per_rank, e2e_ms)

    line = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            rate, ns, t, threads = oracle_sample_rate(w, args.cpu_seconds)
            cpu = {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle",
                   "sample": f"fp64 oracle, full FLARE++ forward on the first {ns} of {w.N} tokens "
                             f"(B={w.B} H={w.H} M={w.M} D={w.D} C={w.C}) in {t:.1f} s; {cpu_model()}"}
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": w.name, "B": w.B, "N": w.N, "C": w.C, "H": w.H, "D": w.D, "M": w.M,
                       "parallelism": f"replicas{world}" if world > 1 else "single",
                       "launch": "cuda_graph" if args.graph else "eager",
                       "l2": "inputs larger than L2 (X 256 MiB; K~,V~,K,V 1 GiB per step)"},
            "roofline": roof,
            "step_roofline": step_roofline,
            "stages": stages,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": e2e_ms},
            "gpu_launches": LAUNCHES_PER_STEP * args.steps,
            "clocks": clk,
        }
    del graph
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
