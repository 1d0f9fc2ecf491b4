"""Shape sharding across ranks (one process per GPU).

Shapes are independent vecsets, so a batch is split across ranks with no
exchange on the data path; the only collectives are the timing barrier and
the max/sum reductions of scalars done here (NCCL on GPUs, gloo on CPU).
"""
from __future__ import annotations

from typing import List


def shapes_for_rank(n_shapes: int, rank: int, world: int) -> List[int]:
    """Contiguous block of shape ids owned by ``rank`` (sizes differ by <= 1)."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank / world size")
    base, extra = divmod(n_shapes, world)
    start = rank * base + min(rank, extra)
    return list(range(start, start + base + (1 if rank < extra else 0)))


def _reduce(x: float, op_name: str, device) -> float:
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=getattr(dist.ReduceOp, op_name))
    return float(t.item())


def max_over_ranks(x: float, device="cpu") -> float:
    return _reduce(x, "MAX", device)


def sum_over_ranks(x: float, device="cpu") -> float:
    return _reduce(x, "SUM", device)


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and str(device).startswith("cuda"):
            dist.barrier(device_ids=[int(str(device).split(":")[1]) if ":" in str(device) else 0])
        else:
            dist.barrier()
