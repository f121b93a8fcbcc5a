"""The work dealing behind the grouping's per-SM shares (host-side model).

The grouping lays a batch's work items out largest first -- an id with c
tokens makes c // 16 items of 16 tokens and one of c % 16 -- and a
one-CTA-per-SM layer kernel of G CTAs takes them in rounds of G, round m in
alternating direction (CTA b takes position b of the round when m is even,
G - 1 - b when odd), processing its items in the order rounds 0, last, 1,
last - 1, ...  Each CTA's share is sized by the bound 16 + ceil(T / G) on its
tokens (its item of round m >= 1 is no larger than any item of round m - 1,
so all rounds after the first hold at most T / G of its tokens).  These tests
restate the dealing and check that every item is dealt exactly once, that
the processing order is a permutation of the CTA's rounds, and that the bound
holds on the batch shapes of the benchmark and on degenerate ones.
"""
import numpy as np
import pytest

from mixture_lookup_experts_b200 import inputs

ITEM = 16


def item_sizes(ids):
    """Item token counts laid out largest first (16, then 15, ..., then 1)."""
    _, counts = np.unique(ids, return_counts=True)
    full = int(np.sum(counts // ITEM))
    rest = counts % ITEM
    sizes = [ITEM] * full
    for n in range(ITEM - 1, 0, -1):
        sizes += [n] * int(np.sum(rest == n))
    return np.array(sizes, dtype=np.int64)


def item_of(m, b, G):
    return m * G + ((G - 1 - b) if (m & 1) else b)


def items_of(n_items, b, G):
    full = n_items // G
    return full + (1 if item_of(full, b, G) < n_items else 0)


def cta_item(k, my_n, b, G):
    return item_of(my_n - 1 - (k >> 1) if (k & 1) else (k >> 1), b, G)


def share_cap(T, G):
    return (ITEM + (T + G - 1) // G + 15) // 16 * 16


def deal(sizes, T, G):
    n = len(sizes)
    seen = np.zeros(n, dtype=np.int64)
    worst = 0
    for b in range(G):
        my_n = items_of(n, b, G)
        order = [cta_item(k, my_n, b, G) for k in range(my_n)]
        rounds = sorted(item_of(m, b, G) for m in range(my_n))
        assert sorted(order) == rounds  # the processing order is a permutation of the CTA's rounds
        for it in order:
            assert 0 <= it < n
            seen[it] += 1
        tokens = int(sizes[order].sum()) if my_n else 0
        assert tokens <= ITEM + -(-T // G), (b, tokens)
        assert my_n <= tokens or my_n == 0
        worst = max(worst, tokens)
    assert (seen == 1).all()
    assert worst <= share_cap(T, G)
    return worst


@pytest.mark.parametrize("T,kind", [(4096, "zipf"), (4096, "uniform"), (14080, "zipf"), (2500, "zipf"),
                                    (1024, "uniform"), (16384, "zipf")])
@pytest.mark.parametrize("G", [148, 132, 7])
def test_dealing_covers_every_item_once_within_the_share_bound(T, kind, G):
    rng = np.random.default_rng(T + G)
    ids = inputs.draw_ids(rng, T, 50304, kind)
    sizes = item_sizes(ids)
    assert sizes.sum() == T
    assert (np.diff(sizes) <= 0).all()
    deal(sizes, T, G)


@pytest.mark.parametrize("ids", [
    np.zeros(5000, dtype=np.int32),                  # one id: 313 items of that id
    np.arange(4096, dtype=np.int32),                 # every id distinct: 4096 one-token items
    np.repeat(np.arange(300, dtype=np.int32), 17),   # every id 17 times: a 16-token and a 1-token item each
    np.repeat(np.arange(148, dtype=np.int32), 15),   # one 15-token item per CTA
])
def test_dealing_degenerate_batches(ids):
    T = len(ids)
    deal(item_sizes(ids), T, 148)


def test_bound_is_reached_by_construction():
    """The bound is tight up to rounding: one 16-token item per CTA in round 0
    and one-token items after it."""
    G = 148
    ids = np.concatenate([np.repeat(np.arange(G), ITEM), np.arange(G, G + 10 * G)]).astype(np.int32)
    T = len(ids)
    worst = deal(item_sizes(ids), T, G)
    assert worst == ITEM + 10
    assert ITEM + 10 <= ITEM + -(-T // G)
