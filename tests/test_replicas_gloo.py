"""Multi-GPU runs are independent replicas (no collective on the data path);
bench.py only reduces its timing and token counts over ranks.  Checked here
with two gloo ranks on CPU: MAX of the device times, SUM of committed tokens."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, q):
    import torch
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    ms, e2e, committed = bench.reduce_over_ranks(1.0 + rank, 2.0 + 3 * rank, 60 + rank, torch.device("cpu"))
    q.put((rank, ms, e2e, committed))
    dist.barrier()
    dist.destroy_process_group()


def test_reduce_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ms, e2e, committed in out:
        assert ms == 2.0 and e2e == 5.0 and committed == 121


def test_single_process_returns_its_own_numbers():
    import torch
    import bench
    assert bench.reduce_over_ranks(1.5, 2.5, 63, torch.device("cpu")) == (1.5, 2.5, 63)
