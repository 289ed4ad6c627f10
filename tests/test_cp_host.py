"""Host side of the context-parallel forward: the partials of every rank are
all-gathered in rank order (two gloo ranks on CPU)."""
import datetime
import multiprocessing
import os
import socket

import torch


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    from rank_latent_routing_flare_b200 import cp
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        part = torch.arange(5, dtype=torch.float32) + 100 * rank
        got = cp.allgather_partials(part, world)
        out.put((rank, got.tolist(), cp._group_info(None)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_partials_are_gathered_in_rank_order():
    world = 2
    ctx = multiprocessing.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    want = [float(x) for x in range(5)] + [100.0 + x for x in range(5)]
    for rank, got, info in results:
        assert got == want
        assert info == (rank, world)


def test_single_rank_without_process_group():
    from rank_latent_routing_flare_b200 import cp
    part = torch.ones(3)
    assert cp._group_info(None) == (0, 1)
    assert cp.allgather_partials(part, 1) is part


class _FakeLib:
    """Stands in for libflare.so: records the backward phases and fills each
    exchange buffer with (rank, phase) markers, and records what each phase
    was handed as `gathered`."""

    def __init__(self, rank):
        self.rank = rank
        self.calls = []

    def flarepp_cp_bwd_exchange_bytes(self, phase, B, N, C, H, M, D):
        return 4 * (3 + phase) if 0 <= phase < 6 else 0

    def flarepp_cp_bwd_phase(self, phase, *args):
        import ctypes
        gathered, exchange = args[7], args[8]
        rank_arg, world_arg = args[22], args[23]   # after B, N, C, H, M, D and lengths
        seen = None
        if gathered:
            n = 2 * (3 + phase - 1)
            seen = list((ctypes.c_float * n).from_address(gathered))
        if exchange:
            n = 3 + phase
            buf = (ctypes.c_float * n).from_address(exchange)
            for i in range(n):
                buf[i] = 100 * self.rank + 10 * phase + i
        self.calls.append((phase, rank_arg, world_arg, seen, bool(exchange)))
        return 0

    def flare_last_device_status(self, workspace, stream):
        self.calls.append(("status",))
        return 0


def _bwd_rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    from rank_latent_routing_flare_b200 import _binding, cp
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        fake = _FakeLib(rank)
        _binding.load_library = lambda *a, **k: fake
        _binding.flare_workspace_bytes = lambda *a, **k: 256

        class _Stream:
            cuda_stream = 0
        B, N, C, H, M, D = 1, 4, 64, 4, 2, 16
        X = torch.zeros((B, N, C), dtype=torch.bfloat16)
        W = torch.zeros((C, C), dtype=torch.bfloat16)
        Q0 = torch.zeros((H, M, D), dtype=torch.bfloat16)
        dY = torch.zeros((B, H, N, D), dtype=torch.bfloat16)
        cp.flarepp_mixer_cp_bwd(X, W, W, W, W, Q0, dY, stream=_Stream())
        out.put((rank, fake.calls))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_backward_phases_run_in_order_with_rank_ordered_gathers():
    world = 2
    ctx = multiprocessing.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_bwd_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, calls in results:
        assert calls[-1] == ("status",)      # the device word is read after the last phase
        calls = calls[:-1]
        assert [c[0] for c in calls] == list(range(7))
        assert all(c[1] == rank and c[2] == world for c in calls)
        assert calls[0][3] is None                       # nothing gathered before phase 0
        assert [c[4] for c in calls] == [True] * 6 + [False]   # no exchange after the last phase
        for phase in range(1, 7):
            n = 3 + phase - 1
            want = [float(10 * (phase - 1) + i) for i in range(n)] + \
                   [float(100 + 10 * (phase - 1) + i) for i in range(n)]
            assert calls[phase][3] == want, (rank, phase)


class _StatusLib(_FakeLib):
    """A fake library whose device error word reports a bad length."""

    def __init__(self, word):
        super().__init__(0)
        self.word = word

    def flare_last_device_status(self, workspace, stream):
        self.calls.append(("status",))
        return self.word

    def flare_status_string(self, status):
        return b"FLARE_ERR_SHAPE (fake)"


def _run_single_rank_bwd(monkeypatch, fake, workspace=None, device_check=None):
    from rank_latent_routing_flare_b200 import _binding, cp
    monkeypatch.setattr(_binding, "load_library", lambda *a, **k: fake)
    monkeypatch.setattr(_binding, "flare_workspace_bytes", lambda *a, **k: 256)
    # a CPU tensor stands in for the caller's device workspace
    monkeypatch.setattr(_binding, "_workspace", lambda ws, n, dev: ws if ws is not None else torch.empty(n, dtype=torch.uint8))

    class _Stream:
        cuda_stream = 0
    B, N, C, H, M, D = 1, 4, 64, 4, 2, 16
    X = torch.zeros((B, N, C), dtype=torch.bfloat16)
    W = torch.zeros((C, C), dtype=torch.bfloat16)
    return cp.flarepp_mixer_cp_bwd(X, W, W, W, W, torch.zeros((H, M, D), dtype=torch.bfloat16),
                                   torch.zeros((B, H, N, D), dtype=torch.bfloat16), stream=_Stream(),
                                   workspace=workspace, device_check=device_check)


def test_device_error_word_raises_when_the_workspace_is_internal(monkeypatch):
    import pytest
    from rank_latent_routing_flare_b200 import FlareError, Status
    fake = _StatusLib(int(Status.ERR_SHAPE))
    with pytest.raises(FlareError) as e:
        _run_single_rank_bwd(monkeypatch, fake)
    assert e.value.status == Status.ERR_SHAPE
    assert fake.calls[-1] == ("status",)


def test_a_caller_workspace_is_left_for_the_caller_to_check(monkeypatch):
    fake = _StatusLib(2)
    ws = torch.empty(256, dtype=torch.uint8)
    _run_single_rank_bwd(monkeypatch, fake, workspace=ws)
    assert ("status",) not in fake.calls
    fake2 = _StatusLib(0)
    _run_single_rank_bwd(monkeypatch, fake2, workspace=ws, device_check=True)
    assert fake2.calls[-1] == ("status",)


class _FakeFlareLib(_FakeLib):
    """Stands in for libflare.so in the FLARE backward: exchange buffers get
    (rank, phase) markers, and what each phase was handed is recorded."""

    def flare_cp_bwd_exchange_bytes(self, phase, B, H, N, M, D):
        return 4 * (2 + phase) if 0 <= phase < 3 else 0

    def flare_cp_bwd_phase(self, phase, *args):
        import ctypes
        gathered, exchange = args[4], args[5]
        rank_arg, world_arg = args[15], args[16]   # after B, H, N, M, D and lengths
        seen = None
        if gathered:
            n = 2 * (2 + phase - 1)
            seen = list((ctypes.c_float * n).from_address(gathered))
        if exchange:
            n = 2 + phase
            buf = (ctypes.c_float * n).from_address(exchange)
            for i in range(n):
                buf[i] = 100 * self.rank + 10 * phase + i
        self.calls.append((phase, rank_arg, world_arg, seen, bool(exchange)))
        return 0


def _flare_bwd_rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import torch.distributed as dist
    from rank_latent_routing_flare_b200 import _binding, cp
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        fake = _FakeFlareLib(rank)
        _binding.load_library = lambda *a, **k: fake
        _binding.flare_workspace_bytes = lambda *a, **k: 256

        class _Stream:
            cuda_stream = 0
        B, H, N, M, D = 1, 2, 4, 16, 16
        K = torch.zeros((B, H, N, D), dtype=torch.bfloat16)
        Q = torch.zeros((H, M, D), dtype=torch.bfloat16)
        cp.flare_mixer_cp_bwd(K, K, Q, K, stream=_Stream())
        out.put((rank, fake.calls))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_flare_backward_phases_run_in_order_with_rank_ordered_gathers():
    world = 2
    ctx = multiprocessing.get_context("spawn")
    out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_flare_bwd_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    results = sorted(out.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, calls in results:
        assert calls[-1] == ("status",)
        calls = calls[:-1]
        assert [c[0] for c in calls] == list(range(4))
        assert all(c[1] == rank and c[2] == world for c in calls)
        assert calls[0][3] is None
        assert [c[4] for c in calls] == [True] * 3 + [False]
        for phase in range(1, 4):
            n = 2 + phase - 1
            want = [float(10 * (phase - 1) + i) for i in range(n)] + \
                   [float(100 + 10 * (phase - 1) + i) for i in range(n)]
            assert calls[phase][3] == want, (rank, phase)
