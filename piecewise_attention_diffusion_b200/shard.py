"""Head-sharded runs over several GPUs: host-side partition and the optional gather of O.

Every (batch, head) pair is independent in all four calls of the path: block statistics,
routing and the attention of one head read only that head's Q, K and V and its own block
lists ("PISA: Piecewise Sparse Attention Is Wiser for Efficient Diffusion Transformers",
§2: the centroids, H_j and H-bar are statistics of one head; the fixed multimodal mask of
"多模态 DiT 上的块稀疏 Attention", §4.2, is one pattern that every head only reads). A run over
N GPUs therefore gives each rank one contiguous range of the flattened (batch * heads)
index and calls the library on that range alone: no data crosses GPUs on the path. The one
collective a caller may want afterwards is the all-gather of O, which `gather_heads` does
(uneven ranges padded to the largest, then trimmed).

Ranks are processes with a `torch.distributed` group (NCCL between GPUs, gloo on CPU).
"""
from __future__ import annotations

import torch


def head_range(n_heads: int, world: int, rank: int) -> tuple[int, int]:
    """The contiguous range [h0, h1) of flattened (batch * heads) indices of `rank`.

    The first n_heads % world ranks take one head more than the others, so range sizes
    differ by at most one; a rank past the last head (world > n_heads) gets an empty range.
    """
    if n_heads < 0 or world < 1 or not 0 <= rank < world:
        raise ValueError(f"bad partition: {n_heads} heads, world {world}, rank {rank}")
    base, extra = divmod(n_heads, world)
    h0 = rank * base + min(rank, extra)
    return h0, h0 + base + (1 if rank < extra else 0)


def shard_of(x: torch.Tensor, world: int, rank: int) -> torch.Tensor:
    """This rank's heads of a [batch, heads, L, d] tensor, as [1, h1 - h0, L, d] (a view
    when the range lies within one batch entry, else a copy)."""
    Bt, H, L, d = x.shape
    h0, h1 = head_range(Bt * H, world, rank)
    return x.reshape(Bt * H, L, d)[h0:h1].unsqueeze(0)


def gather_heads(o_local: torch.Tensor, n_heads: int, world: int, rank: int,
                 group=None) -> torch.Tensor:
    """All-gather the ranks' outputs [1, h1 - h0, L, d] into [n_heads, L, d] on every rank.

    Each rank's range comes from `head_range`; the pieces are padded to the largest range
    for one all-gather, then the padding is dropped. With world == 1 this is
    a reshape.
    """
    import torch.distributed as dist

    h0, h1 = head_range(n_heads, world, rank)
    if o_local.dim() != 4 or o_local.shape[0] != 1 or o_local.shape[1] != h1 - h0:
        raise ValueError(f"rank {rank}: expected [1, {h1 - h0}, L, d], got {tuple(o_local.shape)}")
    L, d = o_local.shape[2], o_local.shape[3]
    if world == 1:
        return o_local.reshape(n_heads, L, d)
    width = head_range(n_heads, world, 0)[1]  # rank 0 holds the largest range
    buf = o_local.new_zeros(width, L, d)
    buf[: h1 - h0] = o_local[0]
    pieces = [torch.empty_like(buf) for _ in range(world)]
    dist.all_gather(pieces, buf, group=group)
    parts = []
    for r in range(world):
        a, b = head_range(n_heads, world, r)
        parts.append(pieces[r][: b - a])
    return torch.cat(parts)
