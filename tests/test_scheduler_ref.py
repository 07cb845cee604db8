"""Pins of the tile-scheduler rule (oracle/tile_scheduler_ref.py) by its properties:
every block of every request is covered exactly once and in order, split indices
are a bijection onto [0, num_splits[b]), no part exceeds its payload, and the
special cases (batch 1, all lengths 1, one huge request among tiny ones, more parts
than blocks, empty requests) hold."""
import numpy as np
import pytest

from oracle import tile_scheduler_ref as ts


def _check(seqlens, parts, fixed=ts.FIXED_SPLIT_COST):
    md, ns = ts.schedule(seqlens, parts, fixed)
    B = len(seqlens)
    nblk = [ts._blocks(L) for L in seqlens]
    assert md.shape == (parts, 8) and ns.shape == (B + 1,)
    assert ns[0] == 0 and np.all(np.diff(ns) >= 0)
    covered = [[] for _ in range(B)]
    seen_splits = set()
    T = sum(n + fixed for n in nblk if n > 0)
    payload = -(-T // parts) + fixed
    prev_end = None
    for p in range(parts):
        chunks = ts.iterate_part(md[p], seqlens, ns)
        cost = sum(fixed + (e - s) for _, s, e, _ in chunks)
        assert cost <= payload + 0, (p, cost, payload)
        begin = (int(md[p, 0]), int(md[p, 1]))
        if prev_end is not None:
            assert begin == prev_end                   # parts tile the cursor range
        prev_end = (int(md[p, 2]), int(md[p, 3]))
        for b, s, e, split in chunks:
            assert 0 <= s < e <= nblk[b]
            covered[b].append((s, e))
            assert ns[b] <= split < ns[b + 1]
            assert split not in seen_splits
            seen_splits.add(split)
    for b in range(B):
        spans = covered[b]
        assert len(spans) == ns[b + 1] - ns[b]
        pos = 0
        for s, e in spans:
            assert s == pos
            pos = e
        assert pos == nblk[b]
    assert len(seen_splits) == ns[-1]
    return md, ns


@pytest.mark.parametrize("seed", range(20))
def test_random_batches(seed):
    rng = np.random.default_rng(seed)
    B = int(rng.integers(1, 200))
    seqlens = rng.integers(0, 20000, size=B)
    parts = int(rng.integers(1, 160))
    fixed = int(rng.integers(0, 6))
    _check(list(seqlens), parts, fixed)


def test_special_cases():
    _check([8192], 148)                      # batch 1, more parts than blocks
    _check([1] * 64, 37)                     # every request one token
    _check([16384] + [1] * 127, 74)          # one huge request among tiny ones
    _check([5, 0, 0, 300, 0], 3)             # empty requests
    _check([0, 0], 4)                        # nothing at all
    _check([128 * 7] * 3, 1)                 # a single part takes everything
    md, ns = _check([8192] * 128, 148)
    assert ns[-1] <= 128 + 148


def test_single_part_has_one_split_per_request():
    md, ns = _check([100, 5000, 17], 1)
    assert list(np.diff(ns)) == [1, 1, 1]


def test_workload_shapes_balance():
    # memory-bound shape: 128 requests x 64 blocks over 148 parts; the busiest part
    # carries at most payload = ceil(T / parts) + F cost units
    md, ns = _check([8192] * 128, 148)
    costs = [sum(ts.FIXED_SPLIT_COST + e - s for _, s, e, _ in ts.iterate_part(md[p], [8192] * 128, ns))
             for p in range(148)]
    T = 128 * (64 + ts.FIXED_SPLIT_COST)
    assert max(costs) <= -(-T // 148) + ts.FIXED_SPLIT_COST


def test_num_sm_parts_rule():
    assert ts.num_sm_parts_for(16, 1, 148) == 148
    assert ts.num_sm_parts_for(64, 1, 148) == 148
    assert ts.num_sm_parts_for(128, 1, 148) == 74
    assert ts.num_sm_parts_for(256, 1, 148) == 37
    assert ts.num_sm_parts_for(256, 1, 2) == 1
    assert ts.num_sm_parts_for(65, 1, 148) == 74      # one SM pair
    assert ts.num_sm_parts_for(192, 1, 148) == 37     # two SM pairs
    assert ts.num_sm_parts_for(300, 1, 148) == 24     # three SM pairs


def test_planted_floor_division_is_caught():
    """With q = floor(T / parts) instead of the ceiling, some block's owner would be a part
    index >= num_sm_parts for the memory-bound shape, i.e. left uncovered."""
    seqlens = [8192] * 128
    F, P = ts.FIXED_SPLIT_COST, 148
    n = [ts._blocks(L) for L in seqlens]
    T = sum(x + F for x in n)
    q_bad = T // P
    last_pos = T - 1
    assert last_pos // q_bad >= P                       # the planted rule loses blocks
    assert last_pos // (-(-T // P)) < P                 # the rule as written does not
