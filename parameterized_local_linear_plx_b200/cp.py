"""Context parallelism over torch.distributed: one rank per GPU, each holding
a contiguous slice of every sequence.

Decode: every rank computes the state record of its slice of the KV cache
per (b, h) (plx_decode_partial), the ranks all-gather them in rank order (the
one exchange step: B * Hq * (2d + 4) fp32 per rank, over NCCL on NVLink), and
every rank merges them (plx_decode_merge).  The slices follow
one another: rank r holds keys r * slice_len .. (r + 1) * slice_len - 1 of
every sequence.

Prefill: rank r holds positions r * C .. (r + 1) * C - 1 of the queries,
probes, keys and values.  The ranks all-gather the key and value chunks (the
exchange step: 2 * B * Hkv * C * d bf16 per rank); rank r then computes the
partial states of its queries block by block with plx_fwd_partial and merges
them with plx_fwd_merge.  Causal: its own chunk (causal) and each earlier
chunk (in full), r + 1 blocks, so later ranks do more blocks and the causal
work is not balanced across ranks.  Non-causal: every chunk in full, `world`
blocks on every rank.

The arithmetic runs in the library's kernels; this module only plans the
slices and moves the data.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def slice_start(rank: int, slice_len: int) -> int:
    """Global index of the first key of `rank`'s slice."""
    return rank * slice_len


def gather_partials(partial: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather one block per rank (partial states, or a key / value chunk)
    into [world, *partial.shape], rank-major."""
    world = dist.get_world_size(group)
    part = partial.contiguous()
    # the ranks' blocks concatenated along the first dimension (the layout every
    # backend accepts), then viewed rank-major
    out = torch.empty((world * part.shape[0],) + tuple(part.shape[1:]), dtype=part.dtype, device=part.device)
    dist.all_gather_into_tensor(out, part, group=group)
    return out.view((world,) + tuple(part.shape))


def context_parallel_decode(q, kslice, vslice, seqlens, r=None, scale=None, num_splits=0, group=None,
                            return_lse=True, stream=None):
    """One decode step with the KV cache split along the sequence over the ranks of `group`.

    q, r [B, Hq, d] bf16 (the same on every rank); kslice, vslice
    [B, Hkv, slice_len, d] bf16: this rank's slice; seqlens [B] int32: the full
    lengths (the same on every rank).  Every rank returns the full (out, lse).
    num_splits: the work partitions of this rank's decode kernel (0:
    automatic); ranks may differ, since each sends one record per (b, h).
    """
    from . import plx

    rank = dist.get_rank(group)
    slice_len = kslice.shape[2]
    partial = plx.plx_decode_partial(q, kslice, vslice, seqlens, r, key_offset=slice_start(rank, slice_len),
                                     scale=scale, num_splits=num_splits, stream=stream)
    gathered = gather_partials(partial, group)
    return plx.plx_decode_merge(gathered, return_lse=return_lse, stream=stream)


def context_parallel_prefill(q, k, v, r=None, causal=True, scale=None, group=None, return_lse=True, stream=None):
    """Prefill with every sequence cut into consecutive chunks over the ranks of `group`.

    q, r [B, Hq, C, d]; k, v [B, Hkv, C, d] bf16: this rank's chunk, positions
    rank * C .. rank * C + C - 1 (the same C on every rank).  causal: the
    queries attend their own chunk causally and the earlier chunks in full;
    otherwise every chunk in full.  Returns this rank's (out [B, Hq, C, d],
    lse [B, Hq, C]).
    """
    from . import plx

    rank = dist.get_rank(group)
    ks = gather_partials(k, group)  # [world, B, Hkv, C, d]
    vs = gather_partials(v, group)
    B, Hq, C, d = q.shape
    blocks = rank + 1 if causal else ks.shape[0]
    partials = torch.empty((blocks, B, Hq, C, 2 * d + 4), dtype=torch.float32, device=q.device)
    for j in range(blocks):
        plx.plx_fwd_partial(q, ks[j], vs[j], r, causal=(causal and j == rank), scale=scale, partial=partials[j],
                            stream=stream)
    return plx.plx_fwd_merge(partials, return_lse=return_lse, stream=stream)
