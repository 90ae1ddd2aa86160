"""Data-parallel plumbing on CPU: two gloo ranks sum their adapter gradients
through one flat buffer and agree on the max of their timings."""
import os
import socket

import pytest


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    import torch
    import torch.distributed as dist
    from qlora_linear_layers_nf4_b200.dp import AdapterGradBuffer, max_over_ranks
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, k, n = 8, 64, 32
        g = AdapterGradBuffer(r, k, n, "cpu")
        g.dA.fill_(float(rank + 1))
        g.dB.copy_(torch.arange(n * r, dtype=torch.float32).view(n, r) * (rank + 1))
        g.all_reduce()
        total = sum(range(1, world + 1))
        ok = bool(torch.all(g.dA == total)) and bool(
            torch.equal(g.dB, torch.arange(n * r, dtype=torch.float32).view(n, r) * total))
        ok = ok and g.flat.data_ptr() == g.dA.data_ptr()          # views of one buffer
        m = max_over_ranks(10.0 * (rank + 1))
        q.put((rank, ok, m))
    finally:
        dist.destroy_process_group()


def test_two_rank_gradient_allreduce():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 2
    procs = [ctx.Process(target=_worker, args=(i, world, port, q)) for i in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    assert all(ok for _, ok, _ in res)
    assert all(m == 10.0 * world for _, _, m in res)
