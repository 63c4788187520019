"""Data-parallel POET-X training step across ranks (one process per GPU).

Tokens are sharded across ranks; theta, G and the merged weight W0' are replicated.  The
layer's gradients in theta are sums over tokens ([POET-X] technical summary section 4:
distributed data-parallel training), so the only exchange of a step is one sum
all-reduce.  It carries dtheta after the CNP backward: that backward is linear in dG, so
reducing dtheta equals reducing dG before it, at about half the bytes ((n + m)(b - 1) / 2
fp32 values per layer against (n + m) b).  The collective is NCCL over NVLink / NVSwitch
for GPU tensors (gloo for CPU tensors in tests).
"""
from __future__ import annotations


def token_shard(T_global: int, world: int, rank: int) -> tuple[int, int]:
    """(first token, token count) of `rank`'s shard: contiguous, sizes differ by <= 1."""
    if world <= 0 or not 0 <= rank < world or T_global < 0:
        raise ValueError("bad shard request")
    base, extra = divmod(T_global, world)
    start = rank * base + min(rank, extra)
    return start, base + (1 if rank < extra else 0)


def allreduce_dtheta(dtheta, group=None) -> None:
    """Sums dtheta (one contiguous tensor holding every block of the layer) over ranks in
    place.  A no-op without an initialised process group of more than one rank."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return
    if dist.get_world_size(group) == 1:
        return
    if not dtheta.is_contiguous():
        raise ValueError("dtheta must be contiguous (one collective per step)")
    dist.all_reduce(dtheta, op=dist.ReduceOp.SUM, group=group)


def dp_step(layer, x, dy, y, dx, stream=None, group=None) -> None:
    """One data-parallel step of a PoetxLinear (or, with lists of tensors, a
    PoetxLinearGroup) on this rank's tokens: CNP forward, layer forward and backward, CNP
    backward, then the all-reduce of dtheta (every block of the layer or group at once)."""
    layer.step(x, dy, y, dx, stream)
    allreduce_dtheta(layer.cnp.dtheta if hasattr(layer, "layers") else layer.dtheta, group)
