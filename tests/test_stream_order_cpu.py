"""The entry order of the interleaved layer kernel (host-side model).

A CTA of the interleaved kernel streams two kinds of entries through one
ring: router tiles (16 consecutive tokens of its share) and work items (the
share's items in processing order, item k owning share tokens loff[k] ..
loff[k+1]-1).  Both the producer and the consumers derive the order from one
rule: the next entry is tile t while t < n_tiles and 16 t < loff[k+1] (a
tile holds a token of item k or of an earlier item), else item k.  These
tests restate the rule on the shares the dealing gives (the same model as
test_shares_cpu.py) and check that every tile and item appears once, that
each item's tokens are all routed before the item, that no tile comes
earlier than the first item that needs it, and that the gates a tile writes
are never overwritten before their last item.
"""
import numpy as np
import pytest

from mixture_lookup_experts_b200 import inputs
from test_shares_cpu import cta_item, item_sizes, items_of

TILE = 16


def entry_order(loff):
    """The entries of one CTA: ('t', t) and ('i', k) in ring order."""
    my_n = len(loff) - 1
    n_tok = loff[-1]
    n_tiles = (n_tok + TILE - 1) // TILE
    out, t, k = [], 0, 0
    for _ in range(n_tiles + my_n):
        # (the kernel's expression: once every item is placed, t == n_tiles,
        # so loff[k + 1] is never read past the end -- an IndexError here
        # would say otherwise)
        if t < n_tiles and t * TILE < loff[k + 1]:
            out.append(("t", t))
            t += 1
        else:
            out.append(("i", k))
            k += 1
    return out, n_tiles


def check_order(loff):
    order, n_tiles = entry_order(loff)
    my_n = len(loff) - 1
    tiles = [x for kind, x in order if kind == "t"]
    items = [x for kind, x in order if kind == "i"]
    assert tiles == list(range(n_tiles)) and items == list(range(my_n))
    routed = 0  # tokens whose gates exist
    for pos, (kind, x) in enumerate(order):
        if kind == "t":
            # not earlier than needed: the next item has a token at or past the tile
            nxt = next((y for kd, y in order[pos + 1:] if kd == "i"), None)
            assert nxt is not None and loff[nxt + 1] > x * TILE
            routed = min((x + 1) * TILE, loff[-1])
        else:
            assert routed >= loff[x + 1]  # all of the item's tokens are routed
    return order


def shares(ids, G):
    """Per CTA: the token offsets of its items in processing order."""
    sizes = item_sizes(ids)
    n = len(sizes)
    out = []
    for b in range(G):
        my_n = items_of(n, b, G)
        order = [cta_item(k, my_n, b, G) for k in range(my_n)]
        loff = np.concatenate([[0], np.cumsum([sizes[i] for i in order])]).astype(np.int64)
        out.append(loff)
    return out


@pytest.mark.parametrize("T,kind", [(16384, "zipf"), (16384, "uniform"), (14208, "zipf"), (20011, "uniform")])
def test_entry_order_on_benchmark_shares(T, kind):
    rng = np.random.default_rng(T)
    ids = inputs.draw_ids(rng, T, 50304, kind)
    for loff in shares(ids, 148):
        check_order(loff)


def test_entry_order_degenerate():
    check_order(np.array([0], dtype=np.int64))                    # no items
    check_order(np.array([0, 1], dtype=np.int64))                 # one token
    check_order(np.array([0, 16, 32, 48], dtype=np.int64))        # items aligned with tiles
    check_order(np.array([0, 16, 17, 33, 34], dtype=np.int64))    # large, small, large, small
    order = check_order(np.array([0, 1, 2, 3, 4], dtype=np.int64))  # four single tokens: one tile first
    assert order[0] == ("t", 0) and [k for k, _ in order[1:]] == ["i"] * 4


def test_tile_gates_outlive_their_items():
    """The gate array is indexed by share position, one row per token, so a
    tile's gates stay until the kernel ends; the interleaving only decides
    when they are written.  Every item's tokens lie in tiles that precede it
    and that no later tile rewrites (tiles cover disjoint 16-token ranges)."""
    rng = np.random.default_rng(5)
    ids = inputs.draw_ids(rng, 16384, 50304, "zipf")
    for loff in shares(ids, 148)[:16]:
        order, _ = entry_order(loff)
        written = {}
        for pos, (kind, x) in enumerate(order):
            if kind == "t":
                for tok in range(x * TILE, min((x + 1) * TILE, loff[-1])):
                    assert tok not in written
                    written[tok] = pos
            else:
                assert all(written[tok] < pos for tok in range(loff[x], loff[x + 1]))
