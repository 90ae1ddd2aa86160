"""Data-parallel plumbing on CPU: two gloo ranks sum their adapter gradients
through one flat buffer and agree on the max of their timings; two ranks
quantize their row shards of one weight with the double quant's global max
exchanged by an all-reduce, and together give the single-device result."""
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


class _OracleOps:
    """The three steps of a sharded quantization, by the CPU oracle (test
    stand-ins for the CUDA calls; the exchange between them is real)."""

    @staticmethod
    def quantize(w, bs):
        import types
        import torch
        from oracle import nf4_oracle as O
        ref = O.quantize(w.numpy(), bs, double=False)
        return types.SimpleNamespace(codes=torch.from_numpy(ref["codes"]),
                                     absmax=torch.from_numpy(ref["absmax"]),
                                     absmax_q=None, absmax_scale=None, double_quant=False)

    @staticmethod
    def absmax_max(absmax):
        import torch
        return torch.tensor([float(absmax.max()) if absmax.numel() else 0.0], dtype=torch.float32)

    @staticmethod
    def double_quant(absmax, g):
        import numpy as np
        import torch
        from oracle import nf4_oracle as O
        q, s = O.double_quant(absmax.numpy(), g=np.float32(g.item()))
        return torch.from_numpy(q), torch.tensor([s], dtype=torch.float32)


def _quant_worker(rank, world, port, q):
    import numpy as np
    import torch
    import torch.distributed as dist
    from qlora_linear_layers_nf4_b200 import workloads as WL
    from qlora_linear_layers_nf4_b200.dp import quantize_sharded
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = WL.draw_weight((64, 128), seed=77)
        w[48:] *= np.float32(8.0)                 # the global max is on the last rank only
        rows = 64 // world
        shard = torch.from_numpy(np.ascontiguousarray(w[rank * rows:(rank + 1) * rows]))
        qs = quantize_sharded(shard, 64, True, ops=_OracleOps)
        q.put((rank, qs.codes.numpy().tobytes(), qs.absmax_q.numpy().tobytes(),
               float(qs.absmax_scale.item())))
    finally:
        dist.destroy_process_group()


def test_two_rank_sharded_double_quant():
    import numpy as np
    import torch.multiprocessing as mp
    from oracle import nf4_oracle as O
    from qlora_linear_layers_nf4_b200 import workloads as WL
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 2
    procs = [ctx.Process(target=_quant_worker, args=(i, world, port, q)) for i in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(world))
    w = WL.draw_weight((64, 128), seed=77)
    w[48:] *= np.float32(8.0)
    whole = O.quantize(w, 64, double=True)
    codes = np.frombuffer(b"".join(r[1] for r in res), dtype=np.uint8)
    aq = np.frombuffer(b"".join(r[2] for r in res), dtype=np.uint8)
    assert np.array_equal(codes, whole["codes"])
    assert np.array_equal(aq, whole["absmax_q"])
    assert all(np.float32(r[3]) == np.float32(whole["absmax_scale"]) for r in res)


def test_sharded_quantize_refuses_a_shard_that_splits_a_block():
    import torch
    from qlora_linear_layers_nf4_b200.dp import quantize_sharded
    with pytest.raises(ValueError):
        quantize_sharded(torch.zeros(3, 40), 64, True, ops=_OracleOps)      # 120 elements: not whole blocks
    q = quantize_sharded(torch.zeros(2, 64), 64, True, ops=_OracleOps)    # one rank, no process group
    assert q.double_quant and float(q.absmax_scale.item()) == 0.0 and int(q.absmax_q.max()) == 0
