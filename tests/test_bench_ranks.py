"""Host logic of bench.py's multi-rank path (weak scaling), on CPU.

With --gpus N every rank runs its own copy of the workload on its own seed;
the step time is the slowest rank's and the whole-job rate counts the units
of all ranks.  The reference arm does its work on rank 0 only.  The timing
reduction runs here on two gloo ranks."""
import datetime
import multiprocessing
import os
import socket
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from workloads import make_workload  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, ms, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        got = bench.max_over_ranks(ms[rank], world, "cpu")
        out.put((rank, got, bench.whole_job_rate(world, 8 * 1024, got)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_step_time_is_the_slowest_rank_and_rate_counts_all_ranks():
    world, ms = 2, [3.0, 5.0]
    ctx = multiprocessing.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, ms, out)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, rate in results:
        assert got == 5.0
        assert rate == world * 8 * 1024 / 5e-3


def test_single_rank_needs_no_process_group():
    assert bench.max_over_ranks(4.5, 1, None) == 4.5
    assert bench.whole_job_rate(1, 1000, 2.0) == 500_000.0


def test_each_rank_draws_its_own_input_of_the_same_shape():
    w0 = make_workload(bench.WORKLOAD, N=256, seed=bench.rank_seed(0))
    w1 = make_workload(bench.WORKLOAD, N=256, seed=bench.rank_seed(1))
    assert w0.seed == 3 and w1.seed != w0.seed
    assert w0.X.shape == w1.X.shape and not np.array_equal(w0.X, w1.X)
    assert np.array_equal(w0.Wk, make_workload(bench.WORKLOAD, N=256).Wk)


def test_reference_arm_works_on_rank_zero_only(capsys):
    class Args:
        workload, steps, warmup = bench.WORKLOAD, 1, 3
    assert bench.run_reference(Args, rank=1, world=2) == 0
    assert capsys.readouterr().out == ""


def test_backward_work_counts():
    """Algorithmic work of one FLARE++ backward call: three exponentials per
    token-head-latent (one per score of each SDPA call), per SDPA call the
    score recompute and four gradient products (5 x 2 M D flops per
    token-head), the projection gradients dX and dW of four C x C weights
    (2 x 4 x 2 C D per token-head); HBM: X and dY read, dX written."""
    import bench
    from workloads import make_workload
    w = make_workload("flarepp_n1k", N=256)
    wk = bench.backward_work(w)
    th = w.B * w.H * w.N
    assert wk["exps"] == 3 * w.M * th
    assert wk["flops"] == (30 * w.M * w.D + 16 * w.C * w.D) * th
    assert wk["bytes"] == 3 * w.B * w.N * w.C * 2


def test_backward_work_counts_flare():
    import bench
    from workloads import make_workload
    w = make_workload("flare_n64k", N=512, B=1)
    wk = bench.backward_work(w)
    th = w.B * w.H * w.N
    assert wk["exps"] == 2 * w.M * th and wk["flops"] == 20 * w.M * w.D * th
    assert wk["bytes"] == 5 * th * w.D * 2


def test_exp_unit_bounds_balance_the_two_pipes():
    """The combined bound puts the fraction f of exponentials on the
    polynomial where the special-function unit and the issue slots take
    equally long; it is never above the MUFU-only bound, and with a MUFU as
    fast as the issue rate nothing is moved."""
    b = bench.exp_unit_bounds({"ex2": 16.0, "ffma": 128.0})
    f = b["poly_fraction"]
    assert 0.0 < f < 1.0
    t_mufu = (1 - f) / 16.0
    t_issue = (bench.SOFTMAX_BASE_OPS + (1 - f) + bench.POLY_EXP_OPS * f) / 128.0
    assert abs(t_mufu - t_issue) < 1e-12 and abs(b["combined"] - t_mufu) < 1e-12
    assert b["combined"] < b["mufu_only"] == 1 / 16.0
    fast = bench.exp_unit_bounds({"ex2": 128.0, "ffma": 128.0})
    assert fast["poly_fraction"] == 0.0
    assert fast["combined"] == max(1 / 128.0, (bench.SOFTMAX_BASE_OPS + 1) / 128.0)
