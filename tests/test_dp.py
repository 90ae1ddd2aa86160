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


def _grad_worker(rank, world, port, q, split):
    """Each rank takes its token shard of the tiny layer, computes the adapter
    gradients of its shard (the CPU oracle stands in for the GPU call), and
    sums them with the other ranks through AdapterGradBuffer."""
    import numpy as np
    import torch
    import torch.distributed as dist
    from oracle import nf4_oracle as O
    from qlora_linear_layers_nf4_b200 import workloads as WL
    from qlora_linear_layers_nf4_b200.dp import AdapterGradBuffer
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        case = WL.TINY
        inp = WL.draw_linear(case)
        w_hat = O.bf16_to_f32(O.dequantize(O.quantize(inp.w, 64), "bf16"))
        f = WL.bf16_bits_to_f32
        x, a, b, dy = (f(v).astype(np.float64) for v in (inp.x, inp.a, inp.b, inp.dy))
        lo, hi = split[rank], split[rank + 1]
        d_a, d_b, _ = O.qlora_backward(x[lo:hi], w_hat, a, b, case.alpha, dy[lo:hi])
        g = AdapterGradBuffer(case.r, case.k, case.n, "cpu", dtype=torch.float64)
        g.dA.copy_(torch.from_numpy(d_a))
        g.dB.copy_(torch.from_numpy(d_b))
        g.all_reduce()
        q.put((rank, g.dA.numpy().copy(), g.dB.numpy().copy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("split", [(0, 8, 16), (0, 3, 16)])
def test_token_sharded_gradients_sum_to_the_full_batch(split):
    # Data parallelism over tokens is exact: dA = s sum_m u_m^T x_m and
    # dB = s sum_m dy_m^T t_m are sums over tokens, so the per-rank sums,
    # added by the all-reduce, equal the full-batch gradients (up to fp64
    # rounding of the summation order).  An uneven split gives the same.
    import numpy as np
    import torch.multiprocessing as mp
    from oracle import nf4_oracle as O
    from qlora_linear_layers_nf4_b200 import workloads as WL
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    world = 2
    procs = [ctx.Process(target=_grad_worker, args=(i, world, port, q, split)) for i in range(world)]
    for p in procs:
        p.start()
    # read the results before joining: a child cannot exit while its queued
    # arrays are still waiting in the pipe
    res = sorted((q.get(timeout=120) for _ in range(world)), key=lambda t: t[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    case = WL.TINY
    inp = WL.draw_linear(case)
    w_hat = O.bf16_to_f32(O.dequantize(O.quantize(inp.w, 64), "bf16"))
    f = WL.bf16_bits_to_f32
    x, a, b, dy = (f(v).astype(np.float64) for v in (inp.x, inp.a, inp.b, inp.dy))
    d_a, d_b, _ = O.qlora_backward(x, w_hat, a, b, case.alpha, dy)
    for _, got_a, got_b in res:
        assert np.max(np.abs(got_a - d_a)) <= 1e-12 * np.max(np.abs(d_a))
        assert np.max(np.abs(got_b - d_b)) <= 1e-12 * np.max(np.abs(d_b))
    # both ranks hold the same sum
    assert np.array_equal(res[0][1], res[1][1]) and np.array_equal(res[0][2], res[1][2])


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
