"""Split-KV scheduler specification -- TEST INFRASTRUCTURE ONLY (oracle side).

What the pages fix: "OpenSourceWeek Day 1 - FlashMLA", section V.2, calls
``get_mla_metadata(cache_seqlens, s_q * h_q // h_kv, h_kv)`` once per decode step and
passes the returned ``tile_metadata`` and ``num_splits`` to the kernel; the Baidu page
"Flash MLA: variable-length sequence decode kernels", sections 1-2, gives the purpose:
variable-length sequences over a paged cache, without padding work.  The pages print no
algorithm, so the plan below is this library's own specification, written out here in
plain Python.  Parity unpinned against the pages: it is pinned by its coverage invariants
(every page of every sequence covered exactly once, in order) and by hand-worked cases.

Specification
  PAGE = 64 tokens, OVH = 5 (fixed cost of one split, in pages)
  pages_b  = ceil(L_b / PAGE);  total = sum_b (pages_b + OVH)
  payload  = ceil(total / num_parts) + OVH
  Walk the sequences with a cursor (i, k) = (sequence, page within it), starting at (0, 0).
  For each part in order: begin = cursor, rem = payload, then repeat while i < B:
      left = pages_i - k
      if left + OVH <= rem:  the part finishes sequence i (rem -= left + OVH; i += 1; k = 0)
      else: if rem - OVH > 0 the part takes the next rem - OVH pages of sequence i
            (k += rem - OVH); stop.
  end = cursor.  A part touches sequence i when it finishes it or takes pages of it;
  num_splits[b] counts the parts touching b.

Outputs
  tile_metadata[p] = (begin_i, begin_k * PAGE, end_i, end_k * PAGE, begin_split_ord, 0, 0, 0)
      The part covers tokens from (begin_i, begin_k*PAGE) up to, excluding,
      (end_i, end_k*PAGE).  begin_split_ord = how many earlier parts touched begin_i.
  num_splits[0] = 0; num_splits[b + 1] = num_splits[b] + (parts touching b).
"""

from __future__ import annotations

PAGE = 64
OVH = 5
FIELDS = 8


def num_parts_for(num_sms: int, rows_per_kv_head: int, h_kv: int, rows_per_sm: int = 64) -> int:
    """Scheduling granularity: one part per SM group that serves all query rows of all
    latent heads, 64 query rows per SM: max(1, num_sms // (h_kv * ceil(R / 64)))."""
    m_blocks = -(-rows_per_kv_head // rows_per_sm)
    return max(1, num_sms // (h_kv * m_blocks))


def schedule(cache_seqlens, num_parts: int):
    """Return (tile_metadata: list of num_parts 8-int lists, num_splits: list of B+1)."""
    lens = [int(x) for x in cache_seqlens]
    B = len(lens)
    pages = [-(-L // PAGE) for L in lens]
    total = sum(p + OVH for p in pages)
    payload = -(-total // num_parts) + OVH
    touched = [0] * B
    i, k = 0, 0
    tiles = []
    for _ in range(num_parts):
        begin_i, begin_k = i, k
        begin_ord = touched[i] if i < B else 0
        rem = payload
        while i < B:
            left = pages[i] - k
            if left + OVH <= rem:
                rem -= left + OVH
                touched[i] += 1
                i, k = i + 1, 0
            else:
                if rem - OVH > 0:
                    k += rem - OVH
                    touched[i] += 1
                break
        tiles.append([begin_i, begin_k * PAGE, i, k * PAGE, begin_ord, 0, 0, 0])
    num_splits = [0]
    for b in range(B):
        num_splits.append(num_splits[-1] + touched[b])
    return tiles, num_splits


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
