"""Seeded synthetic inputs for the Parallax forward pass.

This module draws random tensors and nothing else: it holds none of the
method's arithmetic. Both the tests (for the CPU oracle and the CUDA path)
and the benchmark take their inputs from here, so both sides see the same
values.

Recipe (one ``torch.Generator`` per call, seeded, tensors drawn in the fixed
order q, k, v, r, then seqlens):
  * q, k, v ~ N(0, 1); r = r_scale * N(0, 1) (r_scale = 0.1 unless stated);
  * prefill layout [B, H, N, d] (q, r on Hq heads; k, v on Hkv heads);
  * decode layout q, r [B, Hq, d]; k, v caches [B, Hkv, S_max, d];
  * seqlens int32 [B]: all equal to S_max ("equal"), or uniform integers in
    [S_max // 2, S_max] ("ragged");
  * draws are fp32 and then rounded to the requested dtype (bf16 by default).

The shapes follow the pages' workloads: LM pretraining at context 4096 with a
Qwen-3-shaped attention layer, and decode over batch 1..2048 x context
128..32768 (news.chathome.org, "Experiments" and "Hardware argument").
"""
from __future__ import annotations

import torch

__all__ = ["prefill_inputs", "decode_inputs", "draw"]


_CHUNK = 1 << 27  # fp32 elements drawn at a time (512 MB), so large caches fit


def draw(shape, gen, device, scale=1.0, dtype=torch.bfloat16):
    """N(0, scale^2) fp32 draws rounded to dtype; large tensors are drawn in
    slices along dim 0 (deterministic for a given shape and seed)."""
    shape = tuple(int(s) for s in shape)
    numel = 1
    for s in shape:
        numel *= s
    if numel <= _CHUNK or len(shape) == 1:
        x = torch.randn(*shape, generator=gen, device=device, dtype=torch.float32)
        if scale != 1.0:
            x.mul_(scale)
        return x.to(dtype)
    out = torch.empty(shape, device=device, dtype=dtype)
    flat = out.view(-1, *shape[-2:]) if len(shape) > 2 else out
    per = max(1, _CHUNK // (flat[0].numel()))
    for i0 in range(0, flat.shape[0], per):
        i1 = min(flat.shape[0], i0 + per)
        x = torch.randn((i1 - i0,) + tuple(flat.shape[1:]), generator=gen, device=device,
                        dtype=torch.float32)
        if scale != 1.0:
            x.mul_(scale)
        flat[i0:i1].copy_(x)
    return out


def _gen(seed, device):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def prefill_inputs(B, Hq, Hkv, N, d, seed=0, r_scale=0.1, dtype=torch.bfloat16,
                   device="cpu"):
    """(q, k, v, r) for causal/non-causal prefill, drawn in that order."""
    g = _gen(seed, device)
    q = draw((B, Hq, N, d), g, device, 1.0, dtype)
    k = draw((B, Hkv, N, d), g, device, 1.0, dtype)
    v = draw((B, Hkv, N, d), g, device, 1.0, dtype)
    r = draw((B, Hq, N, d), g, device, r_scale, dtype)
    return q, k, v, r


def decode_inputs(B, Hq, Hkv, S_max, d, seed=0, r_scale=0.1, seqlens="equal",
                  dtype=torch.bfloat16, device="cpu"):
    """(q, kcache, vcache, r, seqlens) for one decode step, drawn in that order.

    seqlens: "equal" (every entry S_max), "ragged" (uniform in [S_max//2, S_max])
    or an explicit list of ints.
    """
    g = _gen(seed, device)
    q = draw((B, Hq, d), g, device, 1.0, dtype)
    kc = draw((B, Hkv, S_max, d), g, device, 1.0, dtype)
    vc = draw((B, Hkv, S_max, d), g, device, 1.0, dtype)
    r = draw((B, Hq, d), g, device, r_scale, dtype)
    if isinstance(seqlens, str):
        if seqlens == "equal":
            sl = torch.full((B,), S_max, dtype=torch.int32, device=device)
        elif seqlens == "ragged":
            sl = torch.randint(S_max // 2, S_max + 1, (B,), generator=g,
                               device=device, dtype=torch.int32)
        else:
            raise ValueError(f"unknown seqlens mode {seqlens!r}")
    else:
        sl = torch.tensor(list(seqlens), dtype=torch.int32, device=device)
    return q, kc, vc, r, sl


def paged_decode_inputs(B, Hq, Hkv, max_pages, page_size, d, seed=0, r_scale=0.1, seqlens="ragged",
                        spare_pages=3, dtype=torch.bfloat16, device="cpu"):
    """Decode inputs on a paged cache: (q, kpool, vpool, r, block_table, seqlens).

    The pools hold B * max_pages + spare_pages pages of [Hkv, page_size, d]
    (drawn like the contiguous caches); page slots are assigned to pool pages
    by a seeded random permutation, so neighbouring slots sit in unrelated
    pages.  seqlens as in decode_inputs with S_max = max_pages * page_size.
    """
    S_max = max_pages * page_size
    g = _gen(seed, device)
    num_pages = B * max_pages + spare_pages
    q = draw((B, Hq, d), g, device, 1.0, dtype)
    kpool = draw((num_pages, Hkv, page_size, d), g, device, 1.0, dtype)
    vpool = draw((num_pages, Hkv, page_size, d), g, device, 1.0, dtype)
    r = draw((B, Hq, d), g, device, r_scale, dtype)
    perm = torch.randperm(num_pages, generator=g, device=device)[: B * max_pages]
    table = perm.to(torch.int32).reshape(B, max_pages).contiguous()
    if isinstance(seqlens, str):
        if seqlens == "equal":
            sl = torch.full((B,), S_max, dtype=torch.int32, device=device)
        elif seqlens == "ragged":
            sl = torch.randint(S_max // 2, S_max + 1, (B,), generator=g, device=device, dtype=torch.int32)
        else:
            raise ValueError(f"unknown seqlens mode {seqlens!r}")
    else:
        sl = torch.tensor(list(seqlens), dtype=torch.int32, device=device)
    return q, kpool, vpool, r, table, sl


def gather_pages(pool, table):
    """The contiguous cache [B, Hkv, max_pages * page_size, d] a block table
    describes (page slot n of sequence b = pool page table[b, n])."""
    B, max_pages = table.shape
    _, Hkv, page_size, d = pool.shape
    pages = pool[table.long().reshape(-1)].reshape(B, max_pages, Hkv, page_size, d)
    return pages.permute(0, 2, 1, 3, 4).reshape(B, Hkv, max_pages * page_size, d).contiguous()
