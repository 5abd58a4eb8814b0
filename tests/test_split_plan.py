"""The attention's length-aware split plan, read back from the device (mfa_split_plan runs
the same plan_build / plan_get the attention kernels run), checked over many length mixes
for what the kernels and the workspace rely on:
- every accepted sequence (1 <= length <= capacity) is covered by its items exactly once,
  in whole 128-position tiles; rejected sequences get no items;
- G = min(grid, NT) CTAs get work, none of them empty, and their tile counts differ by at
  most one (NT counted here from the lengths);
- a sequence with n > 1 items has split indices 0 .. n-1 in CTA order and n partial slots,
  distinct over all sequences and inside the workspace's grid + batch slots; a sequence with
  one item has no slot."""

import ctypes

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

TILE = 128


@pytest.fixture(scope="module")
def lib():
    from decode_attention_10_b200 import build, mfa
    build.build()
    return mfa.load()


class _Table:
    """A KV table with the given capacities. Only mfa_split_plan reads it (the capacities):
    every entry points at one small buffer, so no attention may ever run on it."""

    def __init__(self, lib, caps):
        from decode_attention_10_b200 import mfa
        self.batch = len(caps)
        self.buf = torch.zeros(4096, dtype=torch.bfloat16, device="cuda")
        nbytes = lib.mfa_kv_table_bytes(self.batch)
        self.table = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
        arr = ctypes.c_void_p * self.batch
        ptrs = arr(*([self.buf.data_ptr()] * self.batch))
        cp = (ctypes.c_int32 * self.batch)(*caps)
        assert lib.mfa_kv_table_init(self.table.data_ptr(), nbytes, self.batch, 0,
                                     ctypes.cast(ptrs, ctypes.c_void_p),
                                     ctypes.cast(ptrs, ctypes.c_void_p),
                                     ctypes.cast(cp, ctypes.c_void_p), None) == 0
        self.desc = mfa.KvCacheDesc(self.batch, 0, 1.0, 1.0, self.table.data_ptr(), 0)


def _check(lib, lens, grid, caps=None):
    from decode_attention_10_b200 import mfa
    batch = len(lens)
    caps = caps or [max(1, L) for L in lens]
    tab = _Table(lib, caps)
    G, NT, items = mfa.split_plan(tab, torch.tensor(lens, dtype=torch.int32, device="cuda"),
                                  grid)
    items = items.numpy()
    accepted = [1 <= L <= c for L, c in zip(lens, caps)]
    nt = sum((L + TILE - 1) // TILE for L, ok in zip(lens, accepted) if ok)
    assert NT == nt and G == min(grid, nt)
    if nt == 0:
        assert len(items) == 0
        return
    assert len(items) <= grid + batch
    ctas = items[:, 0]
    assert (np.diff(ctas) >= 0).all(), "items listed CTA by CTA"
    assert set(ctas.tolist()) == set(range(G)), "every CTA of the plan has work, no other"
    # tiles per CTA differ by at most one
    tiles = np.zeros(G, np.int64)
    for cta, b, t0, t1, slot, ns, sp in items:
        assert t0 % TILE == 0 and t1 > t0
        tiles[cta] += (t1 + TILE - 1) // TILE - t0 // TILE
    assert tiles.sum() == nt and tiles.max() - tiles.min() <= 1
    # coverage, splits and slots per sequence
    slots = []
    for b in range(batch):
        mine = items[items[:, 1] == b]
        if not accepted[b]:
            assert len(mine) == 0
            continue
        pos = 0
        for k, (cta, _, t0, t1, slot, ns, sp) in enumerate(mine):
            assert t0 == pos, f"sequence {b}: gap or overlap at {pos}"
            pos = t1
            assert ns == len(mine) and sp == k
            if ns == 1:
                assert slot == -1
            else:
                slots.append(slot)
        assert pos == lens[b], f"sequence {b}: covered to {pos} of {lens[b]}"
        if len(mine) > 1:
            assert (np.diff(mine[:, 4]) == 1).all(), "a sequence's slots are consecutive"
    assert len(set(slots)) == len(slots) and all(0 <= s < grid + batch for s in slots)


@pytest.mark.parametrize("grid", [1, 7, 148, 256])
def test_device_plan_covers_balances_and_fits_the_slots(lib, grid):
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
        else:            # with rejected sequences: length 0, or beyond a smaller capacity
            lens = [int(x) if rng.random() < 0.8 else 0 for x in rng.integers(1, 5000, batch)]
            caps = [max(1, L) if rng.random() < 0.9 else max(1, L // 2) for L in lens]
            _check(lib, lens, grid, caps)
            continue
        _check(lib, lens, grid)


def test_device_plan_edge_cases(lib):
    _check(lib, [1], 148)                      # one tile: one CTA
    _check(lib, [0, 0, 0], 148)                # all rejected: no work
    _check(lib, [65536], 148)                  # one sequence over every CTA
    _check(lib, [128] * 148, 148)              # one tile per CTA, no split
    _check(lib, [129] * 148, 148)              # two tiles per sequence over 148 CTAs
    _check(lib, [1] * 1024, 148)               # the largest batch
    _check(lib, [65536] * 16, 148)
    _check(lib, [4096] * 32, 148)              # the 4K workload: 6.92 tiles per CTA
    _check(lib, [300, 0, 65536, 2], 148, caps=[300, 10, 65536, 1])  # 2 > capacity 1
