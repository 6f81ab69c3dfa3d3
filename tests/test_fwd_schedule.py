"""Host logic of the forward's item deal (gpt2_attn_fwd_item_schedule).

The forward runs one work item per (b, h) and pair of adjacent 128-row query
tiles, over a persistent grid of at most one CTA per SM. Which CTA runs
which item is decided on the host (longest processing time first) and passed
to the kernel; these tests check that deal on the CPU, through the library's
own host code: every item is dealt exactly once, each CTA's list is in
heaviest-first order and fits the kernel's list, the deal is the greedy one
it claims to be, and it balances better than the round-robin (snake) deal
the kernel used before. What the deal cannot change (the result of an item)
is checked on the GPU by the parity tests.
"""
import heapq

import numpy as np
import pytest

from causal_self_attention_flashattention_b200 import ops

SLOTS = 64        # items one CTA can hold
MAX_CTAS = 160    # CTAs one deal can describe
MAX_ITEMS = 6144  # items one deal can describe


def items_of(B, T, H):
    n_qt = -(-T // 128)
    n_pairs = (n_qt + 1) // 2
    bh = B * H
    # key tiles per item, items numbered heaviest first
    nkv = []
    for k in range(bh * n_pairs):
        p = n_pairs - 1 - k // bh
        nkv.append(2 * p + 2 if 2 * p + 1 < n_qt else 2 * p + 1)
    return np.array(nkv)


def cost2(nkv):
    return 2 * nkv + 5  # n key tiles + 2.5 tile steps, in half-tile units


SHAPES = [(16, 1024, 12), (2, 4096, 12), (20, 640, 8), (1, 1, 1), (1, 128, 3),
          (3, 1000, 5), (7, 128, 1000), (64, 8192, 12)]


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("num_sms", [148, 7])
def test_every_item_once_in_heaviest_first_lists(shape, num_sms):
    B, T, H = shape
    launch, cta, pos, n_launch = ops.fwd_item_schedule(B, T, H, num_sms)
    nkv = items_of(B, T, H)
    assert len(launch) == len(nkv)
    assert (launch >= 0).all() and (cta >= 0).all() and (pos >= 0).all()
    # launches take consecutive runs of items
    assert (np.diff(launch) >= 0).all() and launch[-1] == n_launch - 1
    for L in range(n_launch):
        sel = np.flatnonzero(launch == L)
        assert len(sel) <= MAX_ITEMS
        grid = min(len(sel), num_sms, MAX_CTAS)
        assert set(cta[sel]) <= set(range(grid))
        for c in range(grid):
            mine = sel[cta[sel] == c]
            assert len(mine) <= SLOTS
            # the CTA's list holds its items in increasing item number
            # (heaviest first), at places 0 .. len - 1
            assert list(pos[mine]) == list(range(len(mine)))


@pytest.mark.parametrize("shape", SHAPES[:6])
def test_deal_is_longest_processing_time_first(shape):
    """Re-deal with a heap: each item, heaviest first, to the least-loaded CTA
    (lowest index on ties); the library's deal must be the same."""
    B, T, H = shape
    launch, cta, pos, n_launch = ops.fwd_item_schedule(B, T, H, 148)
    assert n_launch == 1
    nkv = items_of(B, T, H)
    grid = min(len(nkv), 148)
    heap = [(0, c) for c in range(grid)]
    want = []
    for n in nkv:
        load, c = heapq.heappop(heap)
        want.append(c)
        heapq.heappush(heap, (load + cost2(n), c))
    assert list(cta) == want


def loads(nkv, cta, grid):
    out = np.zeros(grid, dtype=np.int64)
    np.add.at(out, cta, cost2(nkv))
    return out


@pytest.mark.parametrize("shape", SHAPES[:6])
def test_makespan_within_greedy_bound(shape):
    """A greedy deal ends no later than the mean load plus the largest item."""
    B, T, H = shape
    _, cta, _, _ = ops.fwd_item_schedule(B, T, H, 148)
    nkv = items_of(B, T, H)
    grid = min(len(nkv), 148)
    ld = loads(nkv, cta, grid)
    assert ld.max() <= ld.sum() / grid + cost2(nkv).max()


def test_beats_snake_deal_on_gpt2_batch():
    """B=16, T=1024, H=12 on 148 SMs: the round-robin deal (round r takes
    items r*148 .. r*148 + 147, forward in even rounds, backward in odd ones)
    gives CTA 147 items 147, 148 (8 key tiles each), 443, 444 (4 each), 739
    and 740 (2 each): 28 tiles and 6 item costs, 43 tile steps. The greedy
    deal's busiest CTA has 41 (the mean is 38.9)."""
    nkv = items_of(16, 1024, 12)
    _, cta, _, _ = ops.fwd_item_schedule(16, 1024, 12, 148)
    k = np.arange(len(nkv))
    r, i = k // 148, k % 148
    snake = np.where(r % 2 == 0, i, 147 - i)
    assert loads(nkv, snake, 148).max() == 2 * 43
    assert loads(nkv, cta, 148).max() == 2 * 41


def test_split_into_launches_when_the_table_is_full():
    launch, cta, pos, n = ops.fwd_item_schedule(7, 128, 1000, 148)
    assert n == 2
    assert (launch[:MAX_ITEMS] == 0).all() and (launch[MAX_ITEMS:] == 1).all()


@pytest.mark.parametrize("args", [(0, 128, 1, 148), (1, 0, 1, 148), (1, 128, 0, 148),
                                  (1, 128, 1, 0)])
def test_bad_arguments(args):
    with pytest.raises(ValueError):
        ops.fwd_item_schedule(*args)


def test_cached_deal_is_the_built_one():
    """The first call builds and caches the deal; later calls (the cache hit,
    as every forward after the first takes) return the same one."""
    first = ops.fwd_item_schedule(5, 896, 7, 148)
    for _ in range(3):
        again = ops.fwd_item_schedule(5, 896, 7, 148)
        assert again[3] == first[3]
        for a, b in zip(again[:3], first[:3]):
            assert (a == b).all()


def test_more_sms_than_one_table_describes():
    """On a device with more than 160 SMs a launch uses 160 CTAs."""
    launch, cta, pos, n = ops.fwd_item_schedule(16, 1024, 12, 200)
    assert n == 1 and cta.max() == MAX_CTAS - 1
    nkv = items_of(16, 1024, 12)
    ld = loads(nkv, cta, MAX_CTAS)
    assert ld.max() <= ld.sum() / MAX_CTAS + cost2(nkv).max()
