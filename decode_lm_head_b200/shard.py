"""Vocab sharding of an LM head over the ranks of a process group (host-side plumbing).

The head's output rows split into G contiguous stripes, one per rank: rank r holds weight
rows [r * S, min((r + 1) * S, N)) with S = ceil(N / G) and computes logits[:, stripe].  The
activation rows are replicated.  The exchange is one all-gather of the BF16 stripes into a
rank-major buffer [G, M, S] (a stripe shorter than S is zero-padded); `assemble` turns that
into the row-major [M, N] logits when a consumer needs them whole.  No arithmetic of the
method lives here.
"""

import torch


def stripe(n, world, rank):
    """(start, stop) of rank's weight rows; every rank's stripe is at most ceil(n / world)."""
    if world < 1 or not 0 <= rank < world or n < 0:
        raise ValueError("need world >= 1, 0 <= rank < world, n >= 0")
    s = -(-n // world)
    start = min(rank * s, n)
    return start, min(start + s, n)


def stripe_width(n, world):
    return -(-n // world)


def gather_buffer(m, n, world, device, dtype=torch.bfloat16):
    """The all-gather destination [world, m, ceil(n / world)]."""
    return torch.empty(world, m, stripe_width(n, world), dtype=dtype, device=device)


def all_gather_stripes(local, out, group=None, async_op=False):
    """All-gather every rank's [m, S] stripe (zero-padded to S) into out [world, m, S].

    NCCL takes the one-buffer all-gather; gloo the list form (same result)."""
    import torch.distributed as dist

    if dist.get_backend(group) == "nccl":
        return dist.all_gather_into_tensor(out.view(-1), local.reshape(-1), group=group, async_op=async_op)
    parts = list(out.unbind(0))
    return dist.all_gather(parts, local.contiguous(), group=group, async_op=async_op)


def assemble(gathered, n):
    """[world, m, S] rank-major stripes -> [m, n] logits."""
    world, m, s = gathered.shape
    return gathered.permute(1, 0, 2).reshape(m, world * s)[:, :n]
