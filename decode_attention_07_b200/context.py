"""Context parallelism for decode: one long key/value cache sharded along
its token positions over the ranks of a process group.

Rank r holds cache positions [lo_r, hi_r) of every sequence (an equal,
contiguous split of [0, Lmax)). Each rank runs the ordinary split kernel on
its shard, which yields, for every (sequence, query head) row, the attention
over its own tokens and the log-sum-exp of those logits; the ranks then
exchange these partials (one all-gather of rows x (D + 1) fp32 per rank) and
each merges them with fd_merge_partials, the same log-sum-exp reduction the
split kernel uses across splits ("Flash-Decoding for long-context
inference", section "A faster attention for decoding: Flash-Decoding"). The
DISTFLASHATTN abstract on the "Related papers: Glinthawk" page distributes
attention over GPUs along the sequence in this way.

The exchange uses torch.distributed (NCCL between GPUs, gloo on CPU in the
tests); every compute step runs in the library's CUDA kernels.
"""
import torch

from . import _lib


def token_range(Lmax: int, rank: int, world: int):
    """Cache positions [lo, hi) held by `rank`: equal contiguous parts of
    [0, Lmax), the first Lmax % world parts one position longer."""
    if world < 1 or not 0 <= rank < world or Lmax < 0:
        raise ValueError("need 0 <= rank < world and Lmax >= 0")
    base, extra = divmod(Lmax, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def local_seqlens(seqlens: torch.Tensor, lo: int) -> torch.Tensor:
    """Lengths as seen by the shard starting at `lo`: seqlens - lo (the split
    kernel clamps them to [0, shard length])."""
    return seqlens - int(lo)


def gather_partials(out: torch.Tensor, lse: torch.Tensor, group=None):
    """All-gather every rank's (out, lse) partials into [world, ...] tensors
    in rank order."""
    world = torch.distributed.get_world_size(group)
    outs = [torch.empty_like(out) for _ in range(world)]
    lses = [torch.empty_like(lse) for _ in range(world)]
    torch.distributed.all_gather(outs, out.contiguous(), group=group)
    torch.distributed.all_gather(lses, lse.contiguous(), group=group)
    return torch.stack(outs), torch.stack(lses)


def cp_decode(q, k_shard, v_shard, seqlens, lo, scale, group=None, num_splits=None, stream=None):
    """Decode attention of q over a cache sharded across `group`: this rank
    holds positions [lo, lo + k_shard.shape[2]). Returns the merged (out,
    lse), the same on every rank."""
    part_o, part_l = _lib.decode(q, k_shard, v_shard, local_seqlens(seqlens, lo), scale, num_splits, stream)
    if group is None and not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        all_o, all_l = part_o[None], part_l[None]
    else:
        all_o, all_l = gather_partials(part_o, part_l, group)
    out = torch.empty_like(part_o)
    lse = torch.empty_like(part_l)
    _lib.fd_merge_partials(all_o, all_l, out, lse, stream)
    return out, lse
