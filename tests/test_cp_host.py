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
