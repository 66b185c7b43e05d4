"""Sequence-sharded decode over several GPUs, one process per GPU.

A very long sequence's latent pages can be spread over the GPUs of a node: each GPU holds a
contiguous range of the sequence's tokens in its own page pool and decodes the query rows
against its range with the single-GPU library; the GPUs then exchange their partial results
(out_k bf16, lse_k fp32: R x 512 x 2 + R x 4 bytes per sequence and GPU) with one all-gather
and merge them locally with the log-sum-exp merge (mla_merge_partials), which is the method's
split-KV combine applied across GPUs.  This is the one exchange step of the path; the pages
never cross NVLink.

Causal masking with s_q > 1 (the s_q new tokens are the last s_q cache entries) only ever
hides keys in the last s_q - 1 positions.  shard_bounds keeps those in the last shard, so
every earlier shard's keys are visible to every row (decoded with causal off) and the last
shard is decoded with the usual bottom-right causal rule in its own coordinates.

The decode and merge steps run in the library's CUDA kernels (ops); decode_fn / merge_fn
exist only so that host logic can be exercised without a GPU.
"""

from __future__ import annotations

from typing import Callable, Optional, Sequence

import torch

PAGE = 64


def shard_bounds(length: int, n_shards: int, s_q: int = 1, page: int = PAGE) -> list[tuple[int, int]]:
    """Token ranges [start, end) of a sequence of `length` tokens over n_shards shards.

    Contiguous, disjoint and covering [0, length); boundaries fall on page multiples; pages are
    dealt out as evenly as possible, the earlier shards taking the extra ones; the last shard
    holds every token at position >= length - s_q + 1 (the only keys a causal row can fail to
    see).  Empty shards are (x, x)."""
    if n_shards < 1 or length < 0 or s_q < 1:
        raise ValueError("n_shards, s_q >= 1 and length >= 0")
    pages = (length + page - 1) // page
    base, extra = divmod(pages, n_shards)
    bounds, p = [], 0
    for k in range(n_shards):
        n = base + (1 if k < extra else 0)
        bounds.append((min(p * page, length), min((p + n) * page, length)))
        p += n
    # the causal tail: keys >= length - s_q + 1 belong to the last shard
    tail = max(0, (length - s_q + 1) // page * page)
    last_start = min(bounds[-1][0], tail)
    bounds = [(min(a, last_start), min(b, last_start)) for a, b in bounds[:-1]] + [(last_start, length)]
    return bounds


def shard_block_table(block_table: torch.Tensor, seqlens: Sequence[int], n_shards: int, shard: int,
                      s_q: int = 1) -> tuple[torch.Tensor, torch.Tensor]:
    """This shard's view of a batch: (block_table rows of its pages [b, w], its token counts
    [b]) from a global block table whose pages this shard holds for its ranges."""
    rows, lens = [], []
    for b, L in enumerate(int(x) for x in seqlens):
        a, e = shard_bounds(L, n_shards, s_q)[shard]
        pa, pe = a // PAGE, (e + PAGE - 1) // PAGE
        rows.append(block_table[b, pa:pe])
        lens.append(e - a)
    width = max(1, max(int(r.numel()) for r in rows))
    bt = torch.zeros(len(rows), width, dtype=torch.int32, device=block_table.device)
    for b, r in enumerate(rows):
        bt[b, :r.numel()] = r
    return bt, torch.tensor(lens, dtype=torch.int32, device=block_table.device)


def _cuda_decode(q, k_cache, block_table, seqlens, causal, softmax_scale):
    from . import ops
    R = q.shape[1] * q.shape[2] // k_cache.shape[2]
    tile, splits = ops.get_mla_metadata(seqlens, R, k_cache.shape[2])
    return ops.mla_decode_paged(q, k_cache, block_table, seqlens, 512, tile, splits,
                                softmax_scale=softmax_scale, causal=causal)


def _cuda_merge(o_parts, lse_parts):
    from . import ops
    return ops.mla_merge_partials(o_parts, lse_parts)


def sharded_decode(q: torch.Tensor, k_cache: torch.Tensor, block_table: torch.Tensor, seqlens: torch.Tensor,
                   is_last_shard: bool, causal: bool, group=None, softmax_scale: Optional[float] = None,
                   decode_fn: Optional[Callable] = None, merge_fn: Optional[Callable] = None):
    """Decode this rank's shard of every sequence and merge with the other ranks' shards.

    q [b, s_q, h_q, 576] (the same on every rank); k_cache / block_table / seqlens describe this
    rank's pages and token counts (see shard_block_table); is_last_shard: this rank holds the
    sequences' final tokens (shard_bounds' last shard).  group: a torch.distributed process
    group (None = the default group).  Returns (out [b, s_q, h_q, 512] bf16, lse [b, h_q, s_q]).
    """
    import torch.distributed as dist
    decode_fn = decode_fn or _cuda_decode
    merge_fn = merge_fn or _cuda_merge
    out, lse = decode_fn(q, k_cache, block_table, seqlens, bool(causal and is_last_shard), softmax_scale)
    world = dist.get_world_size(group)
    # gathered along dim 0 (the form every backend accepts), then viewed as [world, ...]
    o_all = torch.empty((world * out.shape[0],) + tuple(out.shape[1:]), dtype=out.dtype, device=out.device)
    l_all = torch.empty((world * lse.shape[0],) + tuple(lse.shape[1:]), dtype=lse.dtype, device=lse.device)
    dist.all_gather_into_tensor(o_all, out.contiguous(), group=group)
    dist.all_gather_into_tensor(l_all, lse.contiguous(), group=group)
    return merge_fn(o_all.view((world,) + tuple(out.shape)), l_all.view((world,) + tuple(lse.shape)))
