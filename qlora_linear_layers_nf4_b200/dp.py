"""Data-parallel training of the QLoRA linear over tokens, and row-sharded
quantization of its weight.

Every rank holds the same frozen NF4 weight and adapters and runs forward and
backward on its own tokens; the only exchange is the sum of the adapter
gradients dA [r, K] and dB [N, r] over ranks (one all-reduce of a single flat
fp32 buffer, NCCL over NVLink on GPUs, gloo on CPU).

Quantizing a weight whose rows are spread over the ranks needs no exchange
for the codes and block scales; the simplified double quant needs one: the
global max of the block scales (an all-reduce of one float with MAX).
"""
from __future__ import annotations


class AdapterGradBuffer:
    """dA and dB as views of one contiguous fp32 buffer, so the gradient
    exchange is a single all-reduce with no packing copy."""

    def __init__(self, r: int, k: int, n: int, device, dtype=None):
        import torch
        dtype = torch.float32 if dtype is None else dtype
        self.flat = torch.empty(r * k + n * r, dtype=dtype, device=device)
        self.dA = self.flat[: r * k].view(r, k)
        self.dB = self.flat[r * k:].view(n, r)

    def all_reduce(self, group=None):
        """Sum the gradients over the ranks of `group` (in place)."""
        import torch.distributed as dist
        if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
            dist.all_reduce(self.flat, op=dist.ReduceOp.SUM, group=group)
        return self


def max_over_ranks(value: float, device=None, group=None) -> float:
    """The largest of one float across ranks (timing is reported as the max)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size(group) == 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())


def quantize_sharded(w_shard, block_size: int = 64, double_quant: bool = False, group=None,
                     ops=None):
    """NF4-quantize this rank's rows of a weight whose rows are spread over the
    ranks of `group`; with double_quant the u8 block scales use the scale of
    scales of the whole weight.

    Steps: local quantize keeping the fp32 block scales; their max on the
    device; one all-reduce(MAX) of that float; the double-quant stage against
    it.  With shards that start on block boundaries the result is the rows of
    a single-device quantization of the whole weight, bit for bit.

    `ops` supplies quantize(w, block_size) -> QuantizedWeight (with absmax),
    absmax_max(absmax) -> 1-element tensor and double_quant(absmax, gmax) ->
    (absmax_q, absmax_scale); by default the CUDA library's calls.
    """
    import torch.distributed as dist
    if ops is None:
        from . import nf4qlora as ops_mod

        class _Cuda:
            @staticmethod
            def quantize(w, bs):
                return ops_mod.quantize(w, bs, False, keep_absmax=True)

            absmax_max = staticmethod(ops_mod.absmax_max)
            double_quant = staticmethod(ops_mod.double_quant)
        ops = _Cuda
    if w_shard.numel() % block_size != 0:
        raise ValueError("a shard must hold whole blocks so that its blocks are the weight's blocks")
    q = ops.quantize(w_shard, block_size)
    if not double_quant:
        return q
    g = ops.absmax_max(q.absmax)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(g, op=dist.ReduceOp.MAX, group=group)
    q.absmax_q, q.absmax_scale = ops.double_quant(q.absmax, g)
    q.double_quant = True
    return q
