"""Data-parallel training of the QLoRA linear over tokens.

Every rank holds the same frozen NF4 weight and adapters and runs forward and
backward on its own tokens; the only exchange is the sum of the adapter
gradients dA [r, K] and dB [N, r] over ranks (one all-reduce of a single flat
fp32 buffer, NCCL over NVLink on GPUs, gloo on CPU).
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
