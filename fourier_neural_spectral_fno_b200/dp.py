"""Data parallelism over the batch (one process per GPU).

Samples are independent through every step of the FNO block and network (the
per-mode mixing contracts channels, never samples), so the forward pass shards
the batch with no exchange at all; training adds one exchange, an all-reduce
of the parameter gradients.  This mirrors the all-reduce data parallelism of
"Efficient multi-GPU distributed training strategies for neural operator
networks: Application to magnetotelluric forward modeling" (key methods),
with the gradient buffer reduced by NCCL over NVLink/NVSwitch on B200 nodes
(gloo on CPU for the tests).

Host logic only: the per-rank compute runs through ``capi``.
"""

from __future__ import annotations

from typing import Dict, List, Tuple


def shard_range(batch: int, rank: int, world: int) -> Tuple[int, int]:
    """Contiguous [lo, hi) slice of the global batch owned by ``rank``."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("bad rank / world size")
    base, extra = divmod(batch, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def mse_scale(local_elems: int, global_elems: int) -> float:
    """Factor turning the local-mean MSE cotangent 2 (u - t) / n_local into the
    global-mean one 2 (u - t) / n_global (apply to du before the backward)."""
    return float(local_elems) / float(global_elems)


def _leaves(grads: Dict[str, object]) -> List:
    out = []
    for key in sorted(grads):
        val = grads[key]
        out.extend(val if isinstance(val, (list, tuple)) else [val])
    return out


def flatten(grads: Dict[str, object]):
    """Copy every gradient tensor into one contiguous float32 buffer."""
    import torch
    leaves = _leaves(grads)
    return torch.cat([t.reshape(-1).to(torch.float32) for t in leaves])


def unflatten_(grads: Dict[str, object], flat) -> None:
    """Write ``flat`` back into the gradient tensors (inverse of flatten)."""
    off = 0
    for t in _leaves(grads):
        n = t.numel()
        t.copy_(flat[off:off + n].view_as(t).to(t.dtype))
        off += n
    if off != flat.numel():
        raise ValueError("gradient buffer size mismatch")


def allreduce_grads(grads: Dict[str, object], group=None, average: bool = False) -> None:
    """Sum (or average) the gradients over the process group in one collective."""
    import torch.distributed as dist
    flat = flatten(grads)
    dist.all_reduce(flat, op=dist.ReduceOp.SUM, group=group)
    if average:
        flat /= dist.get_world_size(group)
    unflatten_(grads, flat)
