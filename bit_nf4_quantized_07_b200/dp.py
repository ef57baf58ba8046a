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
import datetime
import os
from typing import Callable, Tuple

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


def init_from_env(device_type: str = "cuda", timeout_s: float = 120.0) -> Tuple[int, int, int]:
    """(rank, world, local_rank) from the launcher's environment (RANK,
    WORLD_SIZE, LOCAL_RANK; MASTER_ADDR and MASTER_PORT for the rendezvous).
    With more than one rank this joins the default process group: NCCL bound
    to this rank's GPU for CUDA devices, gloo otherwise.  A short timeout
    turns a rank that never arrives into an error on the others."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1 and not dist.is_initialized():
        timeout = datetime.timedelta(seconds=timeout_s)
        if device_type == "cuda":
            dist.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=timeout)
    return rank, world, local


def train_step(backward: Callable[[], None], update: Callable[[], None], dA: torch.Tensor, dB: torch.Tensor,
               world: int, group=None) -> None:
    """One data-parallel training step, the same on every rank: this rank's
    forward and backward over its own tokens (`backward`, which leaves the
    adapter gradients in dA and dB), their sum over the ranks, then the
    optimizer update (`update`), which every rank applies to identical
    gradients, so the replicas of A and B stay identical."""
    backward()
    if world > 1:
        allreduce_adapter_grads(dA, dB, group=group)
    update()


def barrier(world: int) -> None:
    """Meet every rank (nothing with one rank)."""
    if world > 1:
        dist.barrier()


def finish(world: int) -> None:
    """Meet every rank, then leave the process group (nothing with one rank)."""
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
