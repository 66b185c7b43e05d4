"""Split-KV scheduler specification -- TEST INFRASTRUCTURE ONLY (oracle side).

What the pages fix: "OpenSourceWeek Day 1 - FlashMLA", section V.2, calls
``get_mla_metadata(cache_seqlens, s_q * h_q // h_kv, h_kv)`` once per decode step and
passes the returned ``tile_metadata`` and ``num_splits`` to the kernel; the Baidu page
"Flash MLA: variable-length sequence decode kernels", sections 1-2, gives the purpose:
variable-length sequences over a paged cache, without padding work.  The pages print no
algorithm, so the plan below is this library's own specification, written out here in
plain Python.  Parity unpinned against the pages: it is pinned by its coverage invariants
(every page of every sequence covered exactly once, in order), its load bound and
hand-worked cases.

Specification ("balanced cuts")
  PAGE = 64 tokens; OVH = max(1, ceil(R / 32)) with R = rows per latent head: the cost of
  one split in pages (its fp32 partial of R rows grows with R; at least one page for the
  query tile and the epilogue)
  Lay the sequences end to end on a cost axis: sequence b occupies OVH + ceil(L_b / 64)
  units, its OVH units first, then one unit per page.  T = total length of the axis.
  payload = ceil(T / num_parts).  Part p covers the axis interval
  [min(p * payload, T), min((p + 1) * payload, T)).
  An axis position x maps to the cursor (sequence i, page k): x >= T -> (B, 0); otherwise
  i is the sequence whose interval holds x and k = max(0, x - start_i - OVH), so a cut
  inside a sequence's OVH units moves the whole sequence to the next part.
  Part p runs from the cursor of its first position up to (excluding) the cursor of its
  end, so each part does at most payload + OVH units of work.

Outputs
  tile_metadata[p] = (begin_i, begin_k * PAGE, end_i, end_k * PAGE, begin_split_ord, 0, 0, 0)
      begin_split_ord = how many earlier parts touched begin_i.
  num_splits[0] = 0; num_splits[b + 1] = num_splits[b] + (parts touching b).
"""

from __future__ import annotations

PAGE = 64
FIELDS = 8


def overhead_pages(rows_per_kv_head: int) -> int:
    """Fixed cost of one split, in pages: max(1, ceil(R / 32))."""
    return max(1, -(-int(rows_per_kv_head) // 32))


def num_parts_for(num_sms: int, rows_per_kv_head: int, h_kv: int, rows_per_sm: int = 64) -> int:
    """Scheduling granularity: one part per SM group that serves all query rows of all
    latent heads, 64 query rows per SM: max(1, num_sms // (h_kv * ceil(R / 64)))."""
    m_blocks = -(-rows_per_kv_head // rows_per_sm)
    return max(1, num_sms // (h_kv * m_blocks))


def schedule(cache_seqlens, num_parts: int, rows_per_kv_head: int = 16):
    """Return (tile_metadata: list of num_parts 8-int lists, num_splits: list of B+1)."""
    OVH = overhead_pages(rows_per_kv_head)
    lens = [int(x) for x in cache_seqlens]
    B = len(lens)
    cost = [OVH + -(-L // PAGE) for L in lens]
    start = []
    acc = 0
    for c in cost:
        start.append(acc)
        acc += c
    T = acc
    payload = -(-T // num_parts)

    def cursor(x):
        if x >= T:
            return B, 0
        i = 0
        while i + 1 < B and start[i + 1] <= x:
            i += 1
        return i, max(0, x - start[i] - OVH)

    cuts = [cursor(min(p * payload, T)) for p in range(num_parts + 1)]
    touched = [0] * B
    tiles = []
    for p in range(num_parts):
        (bi, bk), (ei, ek) = cuts[p], cuts[p + 1]
        ordinal = touched[bi] if bi < B else 0
        last = ei if ek > 0 else ei - 1          # last sequence this part touches
        for s in range(bi, min(last, B - 1) + 1):
            touched[s] += 1
        tiles.append([bi, bk * PAGE, ei, ek * PAGE, ordinal, 0, 0, 0])
    num_splits = [0]
    for b in range(B):
        num_splits.append(num_splits[-1] + touched[b])
    return tiles, num_splits


def payload_of(cache_seqlens, num_parts: int, rows_per_kv_head: int = 16) -> int:
    OVH = overhead_pages(rows_per_kv_head)
    T = sum(OVH + -(-int(L) // PAGE) for L in cache_seqlens)
    return -(-T // num_parts)


def segments(tiles, cache_seqlens):
    """Expand each part into its (sequence, token begin, token end, split ordinal) pieces."""
    lens = [int(x) for x in cache_seqlens]
    out = []
    for t in tiles:
        bi, bt, ei, et, bord = t[0], t[1], t[2], t[3], t[4]
        segs = []
        s = bi
        while s < ei or (s == ei and et > 0 and s < len(lens)):
            t0 = bt if s == bi else 0
            t1 = et if s == ei else lens[s]
            segs.append((s, t0, t1, bord if s == bi else 0))
            s += 1
        out.append(segs)
    return out
