"""Head sharding of one layer over the ranks of a process group (tensor-parallel style).

The heads of a layer are independent: a head's q, k, v, g, beta, state and output rows are read and
written by that head alone.  The two-node setup of the Ferrite project page (Design section 05)
splits each layer between the two machines; here rank r of W runs the library on a contiguous block
of heads of its own, with no exchange.  Only a caller that wants a whole layer's output or state on every rank
gathers the blocks, with one all-gather per tensor (NCCL on GPUs, gloo on the host).

This module is host plumbing: it slices and gathers tensors and calls ``torch.distributed``.  Every
step of the method runs in the library's kernels on each rank's own heads.
"""
from __future__ import annotations

__all__ = ["head_range", "shard_heads", "gather_heads"]


def head_range(rank: int, world: int, H: int) -> tuple[int, int]:
    """Heads [h0, h1) of rank `rank` out of `world` ranks: contiguous blocks that cover 0..H-1 once,
    the first H % world ranks taking one head more than the others."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank %d out of range for world size %d" % (rank, world))
    if H < world:
        raise ValueError("%d heads cannot be sharded over %d ranks" % (H, world))
    base, extra = divmod(H, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def shard_heads(tensors: dict, rank: int, world: int, head_dim: int = 1) -> dict:
    """A rank's heads of a layer's inputs: every tensor with a head axis at `head_dim` (q, k, v, g,
    beta: axis 1; a state ``[N, H, dv, dk]``: axis 1) is sliced to the rank's block and made
    contiguous, as the library requires; other entries (cu_seqlens, None) pass through."""
    H = None
    for t in tensors.values():
        if hasattr(t, "dim") and t.dim() > head_dim and t.dim() >= 2:
            H = t.shape[head_dim]
            break
    if H is None:
        raise ValueError("no tensor with a head axis")
    h0, h1 = head_range(rank, world, H)
    out = {}
    for name, t in tensors.items():
        if name == "cu_seqlens" or t is None or not hasattr(t, "dim") or t.dim() <= head_dim:
            out[name] = t
        else:
            if t.shape[head_dim] != H:
                raise ValueError("%s has %d heads, expected %d" % (name, t.shape[head_dim], H))
            out[name] = t.narrow(head_dim, h0, h1 - h0).contiguous()
    return out


def gather_heads(local, world: int, head_dim: int = 1, group=None):
    """The whole layer's tensor on every rank, from each rank's block of heads along `head_dim`
    (one all-gather).  The blocks must have equal shapes (H divisible by the world size): the ranks
    first exchange their block shapes, and every rank raises ValueError when they differ, before
    the data all-gather, so that no rank is left waiting in a collective with mismatched sizes."""
    import torch
    import torch.distributed as dist
    if world == 1:
        return local
    local = local.contiguous()
    dev = local.device if dist.get_backend(group) == "nccl" else torch.device("cpu")
    mine = torch.tensor(list(local.shape), dtype=torch.int64, device=dev)
    shapes = [torch.empty_like(mine) for _ in range(world)]
    dist.all_gather(shapes, mine, group=group)
    if any(not torch.equal(x, shapes[0]) for x in shapes):
        raise ValueError("gather_heads needs equal head blocks on every rank; got shapes %s (the heads "
                         "must divide evenly over the %d ranks)" % ([tuple(x.tolist()) for x in shapes], world))
    parts = [torch.empty_like(local) for _ in range(world)]
    dist.all_gather(parts, local, group=group)
    return torch.cat(parts, dim=head_dim)
