"""Properties of the attention's split plan that the workspace and the kernels rely on,
checked on the host over many length mixes.

The plan (decode_attention_10_b200/csrc/attn_plan.cuh) lays every sequence's 128-position
tiles end to end (NT tiles in all) and gives CTA g of a grid of G = min(grid, NT) CTAs the
tiles [bound(g), bound(g + 1)), bound(g) = floor(g NT / G). The owner of tile t is
cta_of(t) = floor(((t + 1) G - 1) / NT). A sequence whose tiles fall to n > 1 CTAs gets n
partial slots. The two formulas are restated below, and the test checks:
- every tile belongs to exactly one CTA, and cta_of agrees with bound;
- no CTA is empty, and tile counts differ by at most one;
- the slots of all sequences fit the workspace's grid + batch slots, since the workspace is
  sized for exactly that many.
"""

import numpy as np
import pytest

TILE = 128


def bound(g, G, NT):
    return (g * NT) // G


def cta_of(t, G, NT):
    return ((t + 1) * G - 1) // NT


def plan(lens, grid):
    tiles = [(L + TILE - 1) // TILE if L > 0 else 0 for L in lens]
    start = np.concatenate([[0], np.cumsum(tiles)]).astype(np.int64)
    NT = int(start[-1])
    G = min(grid, NT)
    return tiles, start, NT, G


def _check(lens, grid):
    tiles, start, NT, G = plan(lens, grid)
    if NT == 0:
        return
    owner = np.array([cta_of(t, G, NT) for t in range(NT)])
    for g in range(G):
        lo, hi = bound(g, G, NT), bound(g + 1, G, NT)
        assert hi > lo, "empty CTA"
        assert (owner[lo:hi] == g).all()
    counts = np.bincount(owner, minlength=G)
    assert counts.sum() == NT and counts.max() - counts.min() <= 1
    slots = 0
    for b, n in enumerate(tiles):
        if n == 0:
            continue
        ns = cta_of(int(start[b + 1]) - 1, G, NT) - cta_of(int(start[b]), G, NT) + 1
        assert ns >= 1
        slots += ns if ns > 1 else 0
    assert slots <= grid + len(lens)


@pytest.mark.parametrize("grid", [1, 7, 148, 296])
def test_plan_covers_balances_and_fits_the_slots(grid):
    rng = np.random.default_rng(grid)
    for _ in range(150):
        batch = int(rng.integers(1, 300))
        kind = rng.integers(0, 4)
        if kind == 0:    # uniform
            lens = [int(rng.integers(1, 9000))] * batch
        elif kind == 1:  # ragged up to 64K
            lens = rng.integers(1, 65537, batch).tolist()
        elif kind == 2:  # mostly short, a few long
            lens = [int(x) if rng.random() < 0.9 else int(x) * 200
                    for x in rng.integers(1, 300, batch)]
        else:            # with rejected (zero-length) sequences
            lens = [int(x) if rng.random() < 0.8 else 0 for x in rng.integers(1, 5000, batch)]
        _check(lens, grid)


def test_plan_edge_cases():
    _check([1], 148)                      # one tile: one CTA
    _check([0, 0, 0], 148)                # all rejected: no work
    _check([65536], 148)                  # one sequence over every CTA
    _check([128] * 148, 148)              # one tile per CTA, no split
    _check([129] * 148, 148)              # two tiles per sequence over 148 CTAs
    _check([1] * 1024, 148)               # the largest batch
    _check([65536] * 16, 148)
