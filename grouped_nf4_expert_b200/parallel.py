"""Data-parallel plumbing: one process per GPU, each running the whole block on its own tokens.

The frozen NF4 base is replicated and has no gradient, so the only exchange
of a data-parallel training step is the sum of the four LoRA gradient tensors
over all ranks (NCCL over NVLink on GPUs; any torch.distributed backend works).
"""

from __future__ import annotations


def allreduce_lora_grads(grads, group=None):
    """Sums each gradient tensor over all ranks of ``group``, in place."""
    import torch.distributed as dist
    for g in grads:
        dist.all_reduce(g, op=dist.ReduceOp.SUM, group=group)
    return grads
