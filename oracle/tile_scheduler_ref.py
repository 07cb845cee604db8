"""Oracle (test infrastructure): the tile-scheduler rule, integer only.

The pages say only that get_mla_metadata(cache_seqlens, s_q*h_q/h_kv, h_kv) returns
tile_scheduler_metadata [num_sm_parts x TileSchedulerMetaDataSize] and num_splits
[batch + 1] ("flash_api.cpp" excerpt, mmssai.com page), and that the tile scheduler
spreads requests and blocks evenly over the SMs so that the load is balanced
(wmrh.cn page, "计算流水线设计").  The exact rule is this library's own reading,
written once here and once in the CUDA scheduler kernel:

  unit          a block of 128 tokens (two 64-token pages); request b has
                n_b = ceil(L_b / 128) blocks (0 when L_b = 0)
  cost          every chunk costs F + (its blocks); F = FIXED_SPLIT_COST = 2 blocks
  T             sum over requests with n_b > 0 of (n_b + F)
  payload       ceil(T / num_sm_parts) + F
  walk          parts p = 0 .. num_sm_parts-1 in order, with a cursor (b, blk) that
                starts at the first request with n_b > 0.  Part p gets budget =
                payload; while budget > F and requests remain it takes
                k = min(n_b - blk, budget - F) blocks of request b as one chunk,
                budget -= F + k, and moves the cursor (to the next request with
                n_b > 0 when b is finished).
  metadata row  {begin_b, begin_blk, end_b, end_blk, first_split, 0, 0, 0}: the part
                covers the cursor range [begin, end) in (b, blk) order; a part with
                no work has begin = end.
  num_splits    num_splits[0] = 0, num_splits[b+1] = num_splits[b] + (chunks of b)
  split index   of a chunk = num_splits[b] + its ordinal among b's chunks;
                first_split = that index for the part's first chunk.

Every block of every request lands in exactly one chunk: a part that ends inside a
request has spent its whole payload, of which F pays for the extra chunk the
next part opens, so each part covers at least ceil(T / num_sm_parts) of T.
``schedule`` asserts it.

num_sm_parts: a CTA handles at most 64 query rows, so rows_per_kv_head rows need
G = ceil(rows / 64) CTAs per chunk and num_sm_parts = max(1, sm_count // (h_kv * G)).
"""
from __future__ import annotations

import numpy as np

BLOCK_TOKENS = 128
FIXED_SPLIT_COST = 2
MD_INTS = 8
ROWS_PER_CTA = 64


def row_groups_for(rows_per_kv_head: int) -> int:
    return max(1, (int(rows_per_kv_head) + ROWS_PER_CTA - 1) // ROWS_PER_CTA)


def num_sm_parts_for(rows_per_kv_head: int, h_kv: int, sm_count: int) -> int:
    return max(1, int(sm_count) // (int(h_kv) * row_groups_for(rows_per_kv_head)))


def _blocks(L: int) -> int:
    return (int(L) + BLOCK_TOKENS - 1) // BLOCK_TOKENS if L > 0 else 0


def schedule(cache_seqlens, num_sm_parts: int, fixed_cost: int = FIXED_SPLIT_COST):
    """Return (tile_md int32 [num_sm_parts, 8], num_splits int32 [batch + 1])."""
    L = [int(x) for x in np.asarray(cache_seqlens).reshape(-1)]
    B = len(L)
    P = int(num_sm_parts)
    assert P >= 1
    n = [_blocks(x) for x in L]
    T = sum(nb + fixed_cost for nb in n if nb > 0)
    payload = (T + P - 1) // P + fixed_cost

    chunks_of = [0] * B
    rows = []

    def skip_empty(b):
        while b < B and n[b] == 0:
            b += 1
        return b

    b, blk = skip_empty(0), 0
    for _ in range(P):
        begin_b, begin_blk = b, blk
        first_ordinal = chunks_of[b] if b < B else 0
        budget = payload
        while budget > fixed_cost and b < B:
            k = min(n[b] - blk, budget - fixed_cost)
            chunks_of[b] += 1
            budget -= fixed_cost + k
            blk += k
            if blk == n[b]:
                b, blk = skip_empty(b + 1), 0
        rows.append([begin_b, begin_blk, b, blk, first_ordinal])
    assert b == B, "scheduler rule left work uncovered"

    num_splits = np.zeros(B + 1, dtype=np.int32)
    num_splits[1:] = np.cumsum(chunks_of)
    md = np.zeros((P, MD_INTS), dtype=np.int32)
    for p, (bb, bk, eb, ek, ordn) in enumerate(rows):
        md[p, :5] = [bb, bk, eb, ek, int(num_splits[bb]) + ordn]
    return md, num_splits


def iterate_part(md_row, cache_seqlens, num_splits):
    """The chunks (b, blk_begin, blk_end, split_index) that one part walks, in order."""
    L = [int(x) for x in np.asarray(cache_seqlens).reshape(-1)]
    begin_b, begin_blk, end_b, end_blk, first_split = (int(v) for v in md_row[:5])
    out = []
    b, blk, split = begin_b, begin_blk, first_split
    while b < end_b or (b == end_b and blk < end_blk):
        stop = end_blk if b == end_b else _blocks(L[b])
        if stop > blk:
            out.append((b, blk, stop, split))
        b += 1
        blk = 0
        if b < len(L):
            split = int(num_splits[b])
    return out
