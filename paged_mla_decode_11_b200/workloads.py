"""Seeded synthetic inputs for paged MLA decode.

This module only draws inputs: sequence lengths, absorbed queries, the shared pool of
64-token latent pages and the block table that maps each sequence's logical pages onto
that pool.  It holds none of the attention arithmetic, so both the CUDA path and the
fp64 oracle can consume what it produces.

Layouts (FlashMLA call shape, "OpenSourceWeek Day 1 - FlashMLA" section V.2 and the
q-reshape / params-struct listings of section II):

    q            [batch, s_q, h_q, 576]           bf16  (512 latent + 64 rope columns)
    k_cache      [num_pages + 1, 64, h_kv, 576]   bf16  (last page = poison page)
    block_table  [batch, max_pages]               int32 (unused entries -> poison page)
    cache_seqlens[batch]                          int32

Draw order for one workload, all from one CPU ``torch.Generator`` seeded with ``seed``:

    1. cache_seqlens (uniform integers where the workload draws them)
    2. q ~ N(0, 1), rounded to bf16
    3. pool ~ N(0, 1) for the real pages, rounded to bf16; the extra last page = POISON
    4. outlier rows (only workloads with ``outlier_frac`` > 0): that fraction of the real
       pool's token rows, chosen by ``randperm``, multiplied by 8 (exact in bf16)
    5. perm = randperm(num_pages); sequence b's logical page p -> perm[offset_b + p]
    6. tail slots of every sequence's last page (token >= L_b) set to POISON

POISON is large but finite, so any read of a slot that should be masked shows up as a
parity failure without producing NaN (0 * NaN would poison a correct P.V product).
"""

from __future__ import annotations

import dataclasses
from typing import Optional, Sequence

import torch

PAGE = 64
D_QK = 576
D_V = 512
POISON = 256.0


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic decode batch.

    ``seqlens`` selects how cache_seqlens is produced:
      ("fixed", (L0, L1, ...))      given lengths, nothing drawn
      ("const", L)                  every sequence has length L, nothing drawn
      ("uniform", lo, hi)           torch.randint(lo, hi + 1)
      ("skewed", L0, lo, hi)        uniform draw for all, then sequence 0 set to L0
    """

    name: str
    batch: int
    s_q: int
    h_q: int
    h_kv: int
    seqlens: tuple
    causal: bool = True
    outlier_frac: float = 0.0
    softmax_scale: Optional[float] = None  # None -> 576 ** -0.5

    @property
    def rows_per_kv_head(self) -> int:
        return self.s_q * self.h_q // self.h_kv

    @property
    def scale(self) -> float:
        return self.softmax_scale if self.softmax_scale is not None else D_QK ** -0.5


# The five decode workloads, named by what they are.
TINY = Workload("tiny b2 h16 L{37,130}", 2, 1, 16, 1, ("fixed", (37, 130)))
MEMORY_BOUND = Workload("memory-bound b64 h16 L~U[1,4096]", 64, 1, 16, 1, ("uniform", 1, 4096))
COMPUTE_BOUND = Workload("compute-bound b128 h128 L=4096", 128, 1, 128, 1, ("const", 4096))
CAUSAL_MTP = Workload("causal s_q=2 b32 h128 L~U[2,16384] 5% x8 rows", 32, 2, 128, 1,
                      ("uniform", 2, 16384), causal=True, outlier_frac=0.05)
SKEWED = Workload("skewed b132 h64 L0=65536 others~U[256,2048]", 132, 1, 64, 1,
                  ("skewed", 65536, 256, 2048))

WORKLOADS = {
    "tiny": TINY,
    "memory_bound": MEMORY_BOUND,
    "compute_bound": COMPUTE_BOUND,
    "causal_mtp": CAUSAL_MTP,
    "skewed": SKEWED,
}


def _draw_seqlens(w: Workload, g: torch.Generator) -> torch.Tensor:
    kind = w.seqlens[0]
    if kind == "fixed":
        vals = list(w.seqlens[1])
        if len(vals) != w.batch:
            raise ValueError("fixed seqlens must list one length per sequence")
        return torch.tensor(vals, dtype=torch.int32)
    if kind == "const":
        return torch.full((w.batch,), int(w.seqlens[1]), dtype=torch.int32)
    if kind == "uniform":
        lo, hi = w.seqlens[1], w.seqlens[2]
        return torch.randint(lo, hi + 1, (w.batch,), generator=g, dtype=torch.int64).to(torch.int32)
    if kind == "skewed":
        first, lo, hi = w.seqlens[1], w.seqlens[2], w.seqlens[3]
        s = torch.randint(lo, hi + 1, (w.batch,), generator=g, dtype=torch.int64).to(torch.int32)
        s[0] = first
        return s
    raise ValueError(f"unknown seqlen rule {kind!r}")


def make_inputs(w: Workload, seed: int = 0, max_pages: Optional[int] = None) -> dict:
    """Draw one workload's inputs on the CPU (see the module docstring for the order).

    Returns a dict with q, k_cache, block_table, cache_seqlens (CPU tensors), plus
    num_pages (real pages, the poison page has index num_pages), max_pages and the
    workload's scalar parameters.
    """
    g = torch.Generator().manual_seed(seed)
    seqlens = _draw_seqlens(w, g)
    if w.h_q % w.h_kv != 0:
        raise ValueError("h_q must be a multiple of h_kv")
    if int(seqlens.min()) < 0:
        raise ValueError("negative sequence length")
    pages = [(int(L) + PAGE - 1) // PAGE for L in seqlens.tolist()]
    num_pages = sum(pages)
    width = max(pages) if pages else 0
    if max_pages is not None:
        if max_pages < width:
            raise ValueError("max_pages smaller than the longest sequence")
        width = max_pages
    width = max(width, 1)

    q = torch.randn(w.batch, w.s_q, w.h_q, D_QK, generator=g).to(torch.bfloat16)

    pool = torch.empty(num_pages + 1, PAGE, w.h_kv, D_QK, dtype=torch.bfloat16)
    pool[:num_pages] = torch.randn(num_pages, PAGE, w.h_kv, D_QK, generator=g).to(torch.bfloat16)
    pool[num_pages] = POISON

    if w.outlier_frac > 0 and num_pages > 0:
        n_rows = num_pages * PAGE
        n_out = int(round(w.outlier_frac * n_rows))
        rows = torch.randperm(n_rows, generator=g)[:n_out]
        flat = pool[:num_pages].view(n_rows, w.h_kv, D_QK)
        flat[rows] = flat[rows] * 8

    perm = torch.randperm(num_pages, generator=g).to(torch.int32)
    block_table = torch.full((w.batch, width), num_pages, dtype=torch.int32)
    off = 0
    for b, n in enumerate(pages):
        block_table[b, :n] = perm[off:off + n]
        off += n

    for b, L in enumerate(seqlens.tolist()):
        if L % PAGE and pages[b] > 0:
            last = int(block_table[b, pages[b] - 1])
            pool[last, L % PAGE:] = POISON

    return dict(q=q, k_cache=pool, block_table=block_table, cache_seqlens=seqlens,
                num_pages=num_pages, max_pages=width, s_q=w.s_q, h_q=w.h_q, h_kv=w.h_kv,
                causal=w.causal, softmax_scale=w.scale, dv=D_V)


E4M3_MAX = 448.0  # largest finite OCP E4M3 value


def to_fp8_cache(k_cache: torch.Tensor) -> tuple[torch.Tensor, torch.Tensor]:
    """Store a bf16 latent cache in the FP8 format (the cache writer's side, not the decode
    path): one fp32 scale per token and latent head, amax(|row|) / 448 (1 for an all-zero
    row), and the row divided by it rounded to OCP E4M3 by torch's float8_e4m3fn conversion.

    Returns (k8 [num_pages, page, h_kv, d] uint8 codes, k_scale [h_kv, num_pages, page] fp32).
    """
    rows = k_cache.float()
    amax = rows.abs().amax(dim=-1)                                    # [pages, page, h_kv]
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    k8 = (rows / scale[..., None]).to(torch.float8_e4m3fn).view(torch.uint8)
    return k8.contiguous(), scale.permute(2, 0, 1).contiguous()


def make_inputs_fp8(w: Workload, seed: int = 0, max_pages: Optional[int] = None) -> dict:
    """make_inputs, with the latent cache stored in the FP8 format (to_fp8_cache): adds
    k8 and k_scale; k_cache stays the bf16 source the codes were made from."""
    x = make_inputs(w, seed, max_pages)
    x["k8"], x["k_scale"] = to_fp8_cache(x["k_cache"])
    return x


# Token-level sparse decode: the memory-bound query shape (64 sequences, 16 heads) over
# longer contexts, each query token keeping 2,048 key positions (Top-K) of its sequence.
SPARSE = Workload("sparse b64 h16 L~U[4096,32768] top-2048", 64, 1, 16, 1, ("uniform", 4096, 32768))
SPARSE_TOPK = 2048


def make_sparse_lists(seqlens: Sequence[int], s_q: int, topk: int, seed: int = 0, causal: bool = True,
                      pad: bool = False) -> tuple[torch.Tensor, torch.Tensor]:
    """Key lists in CSR form for the token-level sparse decode.

    Query token (b, s) keeps min(topk, n) distinct positions drawn uniformly from [0, n) (n =
    L_b, less s_q - 1 - s under the causal rule), in increasing order; with ``pad`` every
    list is filled up to topk entries with -1 (a fixed-width Top-K buffer).  Drawn with
    torch.randperm from one CPU generator seeded with ``seed``, token by token in (b, s)
    order.  Returns (row_ptr [batch * s_q + 1], col_idx [nnz]) int32."""
    g = torch.Generator().manual_seed(seed)
    lists = []
    for L in (int(x) for x in seqlens):
        for s in range(s_q):
            n = max(0, L - (s_q - 1 - s)) if causal else L
            k = min(topk, n)
            pos = torch.sort(torch.randperm(n, generator=g)[:k])[0].to(torch.int32) if k else torch.zeros(0, dtype=torch.int32)
            if pad and k < topk:
                pos = torch.cat([pos, torch.full((topk - k,), -1, dtype=torch.int32)])
            lists.append(pos)
    row_ptr = torch.zeros(len(lists) + 1, dtype=torch.int32)
    row_ptr[1:] = torch.cumsum(torch.tensor([len(x) for x in lists], dtype=torch.int64), 0).to(torch.int32)
    col_idx = torch.cat(lists) if int(row_ptr[-1]) else torch.zeros(0, dtype=torch.int32)
    return row_ptr, col_idx


def make_inputs_sparse(w: Workload, topk: int, seed: int = 0, pad: bool = False) -> dict:
    """make_inputs plus the key lists (make_sparse_lists, drawn with seed + 1): adds row_ptr,
    col_idx and topk."""
    x = make_inputs(w, seed)
    x["row_ptr"], x["col_idx"] = make_sparse_lists(x["cache_seqlens"].tolist(), w.s_q, topk, seed + 1, w.causal, pad)
    x["topk"] = topk
    return x


def sparse_work(row_ptr, col_idx, cache_seqlens, s_q: int, h_q: int, h_kv: int, causal: bool,
                d: int = D_QK, dv: int = D_V) -> tuple[int, int]:
    """Algorithmic (bytes, flops) of one sparse decode call: every visible listed key row read
    once per latent head (d * 2 bytes) plus its 4-byte list entry, the query read and the
    output written once; flops 2 (d + dv) per visible key and query head."""
    rp = [int(v) for v in row_ptr]
    ci = col_idx.tolist() if hasattr(col_idx, "tolist") else list(col_idx)
    lens = [int(v) for v in cache_seqlens]
    keys = 0
    entries = rp[-1] - rp[0]
    for i in range(len(rp) - 1):
        b, s = divmod(i, s_q)
        n = max(0, lens[b] - (s_q - 1 - s)) if causal else lens[b]
        keys += sum(1 for j in ci[rp[i]:rp[i + 1]] if 0 <= j < n)
    batch = len(lens)
    g = h_q // h_kv
    byts = keys * h_kv * d * 2 + entries * 4 + batch * s_q * h_q * (d * 2 + dv * 2 + 4)
    flops = keys * g * 2 * (d + dv) * h_kv
    return byts, flops


D_NOPE = 128   # non-positional query / key columns per head
D_ROPE = 64    # positional (rope) columns, stored in the cache as they are
D_HEAD_V = 128  # value columns per head after the output up-projection


def make_absorb_inputs(tokens: int, heads: int, seed: int = 0) -> dict:
    """Per-head query halves and random-init up-projections for the absorption products.

    Draw order from one CPU generator: q_nope ~ N(0, 1) [T, H, 128], q_rope ~ N(0, 1)
    [T, H, 64], w_uk ~ N(0, 1/128) [H, 128, 512], w_uv ~ N(0, 1/512) [H, 128, 512] (variance
    1 / fan-in), o_latent ~ N(0, 1) [T, H, 512]; all rounded to bf16.  q_nope and q_rope are
    the two column ranges of one [T, H, 192] projection output, as a model produces them.
    """
    g = torch.Generator().manual_seed(seed)
    qkv = torch.randn(tokens, heads, D_NOPE + D_ROPE, generator=g).to(torch.bfloat16)
    w_uk = (torch.randn(heads, D_NOPE, D_V, generator=g) * D_NOPE ** -0.5).to(torch.bfloat16)
    w_uv = (torch.randn(heads, D_HEAD_V, D_V, generator=g) * D_V ** -0.5).to(torch.bfloat16)
    o_lat = torch.randn(tokens, heads, D_V, generator=g).to(torch.bfloat16)
    return dict(q_nope=qkv[..., :D_NOPE], q_rope=qkv[..., D_NOPE:], w_uk=w_uk, w_uv=w_uv, o_latent=o_lat)


def custom(batch: int, s_q: int, h_q: int, h_kv: int, seqlens: Sequence[int],
           causal: bool = True, scale: Optional[float] = None, outlier_frac: float = 0.0,
           name: str = "custom") -> Workload:
    """A workload with given lengths (used for small parity cases and edge cases)."""
    return Workload(name, batch, s_q, h_q, h_kv, ("fixed", tuple(int(x) for x in seqlens)),
                    causal=causal, outlier_frac=outlier_frac, softmax_scale=scale)


def algorithmic_work(seqlens: Sequence[int], s_q: int, h_q: int, h_kv: int, causal: bool,
                     d: int = D_QK, dv: int = D_V, batch_meta: bool = True,
                     token_bytes: Optional[int] = None) -> tuple[int, int]:
    """Algorithmic (bytes, flops) of one decode call.

    Bytes: every valid token's latent row (h_kv heads x d bf16, or token_bytes per token
    and latent head for another cache format) read once, q read once, out (bf16) and lse
    (fp32) written once, plus cache_seqlens and the block-table rows actually addressed.
    Flops: 2 * (d + dv) per (query row, unmasked key).
    """
    per_token = d * 2 if token_bytes is None else int(token_bytes)
    nbytes = 0
    flops = 0
    for L in seqlens:
        L = int(L)
        nbytes += L * h_kv * per_token
        nbytes += s_q * h_q * d * 2 + s_q * h_q * dv * 2 + s_q * h_q * 4
        if batch_meta:
            nbytes += 4 + ((L + PAGE - 1) // PAGE) * 4
        for s in range(s_q):
            n = L - (s_q - 1 - s) if causal else L
            n = max(n, 0)
            flops += 2 * (d + dv) * n * h_q
    return nbytes, flops


def whole_page_bytes(seqlens: Sequence[int], h_kv: int, d: int = D_QK) -> int:
    """Bytes of the whole 64-token pages a kernel streams (tail padding included)."""
    return sum(((int(L) + PAGE - 1) // PAGE) * PAGE * h_kv * d * 2 for L in seqlens)

