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
blocks on every rank.  The zig-zag layout (context_parallel_prefill_zigzag)
balances the causal case: 2 * world chunks, two per rank, 2 * world + 1
blocks on every rank, with the exchange overlapped by the local blocks.

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


# ---------------------------------------------------------------- zig-zag layout
# With consecutive chunks, rank r computes r + 1 blocks of the causal
# attention: the last rank does `world` times the work of the first.  The
# zig-zag layout cuts the sequence into 2 * world chunks of c positions and
# gives rank r chunks r and 2 * world - 1 - r: its early chunk attends r
# earlier chunks plus itself, its late chunk 2 * world - 1 - r earlier chunks
# plus itself, so every rank computes 2 * world + 1 blocks (two of them
# causal), the same amount.


def zigzag_chunks(rank: int, world: int):
    """The two global chunk indices rank `rank` holds (early, late)."""
    return rank, 2 * world - 1 - rank


def zigzag_shard(x: torch.Tensor, rank: int, world: int, dim: int = 2) -> torch.Tensor:
    """This rank's part of a full-sequence tensor: its early chunk followed by
    its late chunk along `dim` (the sequence length must divide by 2 * world)."""
    n = x.shape[dim]
    if n % (2 * world):
        raise ValueError(f"sequence length {n} is not a multiple of 2 * world = {2 * world}")
    c = n // (2 * world)
    a, b = zigzag_chunks(rank, world)
    return torch.cat([x.narrow(dim, a * c, c), x.narrow(dim, b * c, c)], dim=dim).contiguous()


def zigzag_unshard(parts, dim: int = 2) -> torch.Tensor:
    """The full-sequence tensor from every rank's part (rank order), the
    inverse of zigzag_shard."""
    world = len(parts)
    c = parts[0].shape[dim] // 2
    chunks = [None] * (2 * world)
    for rk, part in enumerate(parts):
        a, b = zigzag_chunks(rk, world)
        chunks[a] = part.narrow(dim, 0, c)
        chunks[b] = part.narrow(dim, c, c)
    return torch.cat(chunks, dim=dim)


def zigzag_blocks(rank: int, world: int):
    """The (query chunk, key chunk, causal) blocks of rank `rank`, local ones
    (which need no exchanged key / value) first."""
    a, b = zigzag_chunks(rank, world)
    local = [(a, a, True), (b, b, True), (b, a, False)]
    remote = [(a, j, False) for j in range(a)] + [(b, j, False) for j in range(b) if j != a]
    return local, remote


def context_parallel_prefill_zigzag(q, k, v, r=None, scale=None, group=None, return_lse=True, stream=None):
    """Causal prefill over the ranks of `group` in the zig-zag layout.

    q, r [B, Hq, 2c, d]; k, v [B, Hkv, 2c, d] bf16: this rank's early chunk
    followed by its late chunk (zigzag_shard of the full tensors).  The key /
    value chunks are all-gathered asynchronously while the three blocks that
    need only local keys run; then the remote blocks, then one merge per query
    chunk.  Returns (out [B, Hq, 2c, d], lse [B, Hq, 2c]) in the same local
    order (zigzag_unshard of every rank's out gives the full output).
    """
    from . import plx

    rank = dist.get_rank(group)
    world = dist.get_world_size(group)
    B, Hq, n2, d = q.shape
    c = n2 // 2
    a, b = zigzag_chunks(rank, world)

    def halves(t):
        return [t[:, :, :c].contiguous(), t[:, :, c:].contiguous()]

    qh = halves(q)
    rh = halves(r) if r is not None else [None, None]
    kh, vh = halves(k), halves(v)
    # the exchange: every rank's two key and two value chunks, chunk-major
    send = torch.stack(kh + vh)  # [4, B, Hkv, c, d]
    gathered = torch.empty((world,) + tuple(send.shape), dtype=send.dtype, device=send.device)
    work = dist.all_gather_into_tensor(gathered.view((world * send.shape[0],) + tuple(send.shape[1:])), send,
                                       group=group, async_op=True)

    own = {a: 0, b: 1}  # chunk -> local half

    def key_chunk(j):
        if j in own:
            return kh[own[j]], vh[own[j]]
        owner = j if j < world else 2 * world - 1 - j
        half = 0 if j < world else 1
        return gathered[owner, half], gathered[owner, 2 + half]

    local, remote = zigzag_blocks(rank, world)
    n_blocks = {a: sum(1 for qc, _, _ in local + remote if qc == a), b: sum(1 for qc, _, _ in local + remote if qc == b)}
    partials = {qc: torch.empty((n, B, Hq, c, 2 * d + 4), dtype=torch.float32, device=q.device)
                for qc, n in n_blocks.items()}
    used = {a: 0, b: 0}

    def run(blocks):
        for qc, kc, causal in blocks:
            kk, vv = key_chunk(kc)
            plx.plx_fwd_partial(qh[own[qc]], kk, vv, rh[own[qc]], causal=causal, scale=scale,
                                partial=partials[qc][used[qc]], stream=stream)
            used[qc] += 1

    run(local)
    work.wait()
    run(remote)
    oa, la = plx.plx_fwd_merge(partials[a], return_lse=return_lse, stream=stream)
    ob, lb = plx.plx_fwd_merge(partials[b], return_lse=return_lse, stream=stream)
    out = torch.cat([oa, ob], dim=2)
    lse = torch.cat([la, lb], dim=2) if return_lse else None
    return out, lse
