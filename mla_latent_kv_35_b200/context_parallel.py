"""Context parallelism for long sequences: the token range of each sequence
is split over the ranks of a process group (one GPU each), every rank decodes
its own range of the cache with mla_decode_partial, the per-rank (o_lat, lse)
parts are all-gathered, and mla_combine_parts merges them on every rank.

The exchange is the only collective: one all-gather of B*S_q*H*(d_latent + 1)
fp32 numbers per rank per step (0.26 MB at B=1, S_q=2, H=128).
"""

from __future__ import annotations

import torch

from . import binding as _b


def token_ranges(L: int, world: int, page_size: int = 64):
    """Split tokens [0, L) of one sequence into `world` contiguous ranges of
    whole pages (the last non-empty one may end mid-page).  Returns
    [(first, count, tail)] per rank: rank r holds tokens first .. first+count-1,
    and `tail` tokens of the sequence lie after its range."""
    if L < 0 or world < 1:
        raise ValueError("need L >= 0 and world >= 1")
    n_pages = -(-L // page_size)
    per = -(-n_pages // world) if n_pages else 0
    out = []
    for r in range(world):
        first = min(L, r * per * page_size)
        end = min(L, (r + 1) * per * page_size)
        out.append((first, end - first, L - end))
    return out


def gather_parts(o_local: torch.Tensor, lse_local: torch.Tensor, group=None):
    """All-gather every rank's (o_lat, lse) part: returns tensors
    [world, *o_local.shape] and [world, *lse_local.shape], rank-ordered."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    o_all = [torch.empty_like(o_local) for _ in range(world)]
    l_all = [torch.empty_like(lse_local) for _ in range(world)]
    dist.all_gather(o_all, o_local.contiguous(), group=group)
    dist.all_gather(l_all, lse_local.contiguous(), group=group)
    return torch.stack(o_all), torch.stack(l_all)


def decode_context_parallel(dims, qbuf, pool, n_pages, page_table, max_pages, seq_lens,
                            seq_tail, B: int, S_q: int, workspace, o_lat, lse, group=None,
                            num_workers: int = 0):
    """This rank's part of the decode, the all-gather, and the merge.

    pool / page_table / seq_lens / seq_tail describe this rank's token range
    of every sequence (see token_ranges and mla_decode_partial); qbuf holds
    the full queries on every rank.  o_lat [B, S_q, H, d_latent] and lse
    [B, S_q, H] receive the attention over the whole sequences."""
    o_part = torch.empty_like(o_lat)
    l_part = torch.empty_like(lse)
    _b.mla_decode_partial(dims, qbuf, pool, n_pages, page_table, max_pages, seq_lens, seq_tail,
                          B, S_q, num_workers, workspace, o_part, l_part)
    o_parts, l_parts = gather_parts(o_part, l_part, group)
    rows = B * S_q * dims.n_heads
    _b.mla_combine_parts(dims, o_parts, l_parts, o_parts.shape[0], rows, o_lat, lse)
