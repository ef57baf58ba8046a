"""Data-parallel plumbing for the QLoRA linear (one process per GPU).

Each rank holds the full NF4 + double-quantized weight and its own tokens.
The only exchange of a training step is the sum of the adapter gradients
dA and dB over ranks: both are sums over tokens ("LoRA 与 QLoRA", section
LoRA: only A and B are trained; deck "3 QLoRA Finetuning", card 1), so the
rank-wise sums equal the gradients of the concatenated batch.  dX stays
per rank (it belongs to that rank's tokens) and W0 has no gradient.

torch.distributed carries the collective (NCCL on GPUs, gloo on CPU); the
helpers work with either backend.
"""
from typing import Tuple

import torch
import torch.distributed as dist


def token_range(n_global: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous share [t0, t1) of a global batch of n_global tokens."""
    base, extra = divmod(n_global, world)
    t0 = rank * base + min(rank, extra)
    return t0, t0 + base + (1 if rank < extra else 0)


def allreduce_adapter_grads(dA: torch.Tensor, dB: torch.Tensor, group=None) -> None:
    """In place: dA, dB <- their sums over all ranks of `group`."""
    dist.all_reduce(dA, op=dist.ReduceOp.SUM, group=group)
    dist.all_reduce(dB, op=dist.ReduceOp.SUM, group=group)


def max_over_ranks(value: float, device=None, group=None) -> float:
    """The largest `value` over all ranks (e.g. a per-rank elapsed time)."""
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return float(t.item())
