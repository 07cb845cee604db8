"""Oracle (test infrastructure): the tile-scheduler rule, integer only.

The pages say only that get_mla_metadata(cache_seqlens, s_q*h_q/h_kv, h_kv) returns
tile_scheduler_metadata [num_sm_parts x TileSchedulerMetaDataSize] and num_splits
[batch + 1] ("flash_api.cpp" excerpt, mmssai.com page), and that the tile scheduler
spreads requests and blocks evenly over the SMs so that the load is balanced
(wmrh.cn page, "计算流水线设计").  The exact rule is this library's own reading,
written once here and once in the CUDA scheduler kernel:

  unit          a block of 128 tokens (two 64-token pages); request b has
                n_b = ceil(L_b / 128) blocks (0 when L_b <= 0)
  cost line     requests with n_b > 0 are laid end to end, each taking F + n_b cost
                units (F = FIXED_SPLIT_COST = 2: the cost of opening a chunk, then one
                unit per block); C_b is where request b starts, block j of request b
                sits at position C_b + F + j, and T is the total length
  parts         q = ceil(T / num_sm_parts); part p owns the positions [p*q, (p+1)*q)
  chunks        part p gets, for every request, the blocks whose positions it owns
                (a contiguous run in (b, block) order)
  metadata row  {begin_b, begin_blk, end_b, end_blk, first_split, 0, 0, 0}: the part
                covers the cursor range [begin, end) in (b, block) order; a part with
                no block has begin = end
  num_splits    num_splits[0] = 0, num_splits[b+1] = num_splits[b] + (chunks of b)
  split index   of a chunk = num_splits[b] + (number of earlier parts holding blocks of b)

Each part's cost (its blocks plus F per chunk) is at most q + F: the F units of every
request that starts inside the part are on its interval, and only the first chunk of a
part can be the continuation of a request started earlier.  Every block lands in
exactly one chunk by construction.  Everything is a closed form of prefix sums, so the
GPU kernel computes it in parallel.

num_sm_parts: up to 64 query rows run on one SM; more rows run on pairs of SMs that each
carry 128 rows, so a chunk needs G = 1 SM (rows <= 64) or G = 2 * ceil(rows / 128) SMs, and
num_sm_parts = max(1, sm_count // (h_kv * G)).
"""
from __future__ import annotations

import numpy as np

BLOCK_TOKENS = 128
FIXED_SPLIT_COST = 2
MD_INTS = 8
ROWS_PER_CTA = 64


def row_groups_for(rows_per_kv_head: int) -> int:
    return max(1, (int(rows_per_kv_head) + ROWS_PER_CTA - 1) // ROWS_PER_CTA)


PAIR_ROWS = 128


def sms_per_part(rows_per_kv_head: int) -> int:
    rows = int(rows_per_kv_head)
    return 1 if rows <= ROWS_PER_CTA else 2 * ((rows + PAIR_ROWS - 1) // PAIR_ROWS)


def num_sm_parts_for(rows_per_kv_head: int, h_kv: int, sm_count: int) -> int:
    return max(1, int(sm_count) // (int(h_kv) * sms_per_part(rows_per_kv_head)))


def _blocks(L: int) -> int:
    return (int(L) + BLOCK_TOKENS - 1) // BLOCK_TOKENS if L > 0 else 0


def schedule(cache_seqlens, num_sm_parts: int, fixed_cost: int = FIXED_SPLIT_COST):
    """Return (tile_md int32 [num_sm_parts, 8], num_splits int32 [batch + 1])."""
    L = [int(x) for x in np.asarray(cache_seqlens).reshape(-1)]
    B = len(L)
    P = int(num_sm_parts)
    assert P >= 1
    F = int(fixed_cost)
    n = [_blocks(x) for x in L]
    start = []                      # C_b
    pos = 0
    for nb in n:
        start.append(pos)
        if nb > 0:
            pos += F + nb
    T = pos
    q = max(1, -(-T // P))

    # which part owns each block, by walking every block of every request
    owner_runs = []                 # per request: list of (part, first_blk, end_blk)
    for b in range(B):
        runs = []
        for j in range(n[b]):
            part = (start[b] + F + j) // q
            if runs and runs[-1][0] == part:
                runs[-1][2] = j + 1
            else:
                runs.append([part, j, j + 1])
        owner_runs.append(runs)

    chunks_of = [len(r) for r in owner_runs]
    num_splits = np.zeros(B + 1, dtype=np.int32)
    num_splits[1:] = np.cumsum(chunks_of)

    md = np.zeros((P, MD_INTS), dtype=np.int32)
    for p in range(P):
        begin, end = (B, 0), (B, 0)
        found = False
        for b in range(B):
            for k, (part, s, e) in enumerate(owner_runs[b]):
                if part == p and not found:
                    begin = (b, s)
                    first_split = int(num_splits[b]) + k
                    found = True
        # end: the first block (in (b, blk) order) owned by a later part
        done = False
        for b in range(B):
            for part, s, e in owner_runs[b]:
                if part > p and not done:
                    end = (b, s)
                    done = True
        if not found:
            begin = end
            first_split = int(num_splits[end[0]]) if end[0] < B else int(num_splits[B])
        md[p, :5] = [begin[0], begin[1], end[0], end[1], first_split]
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
