"""Pins of the oracle's dynamic memory update ("MemLong: Memory-Augmented
Retrieval for Long Text Modeling", section 2.3.2, dynamic memory update)
against things other than itself: the rule's proportions in tests/golden,
exhaustive search over every possible kept set on tiny memories, the page's
one-at-a-time deletion process, closed forms, and library counting.

A plausible slip (newest and oldest swapped, the tie rule reversed, the
threshold off by one, the pinned front counted, the tail dropped) fails at
least one of them."""
import itertools
import os

import numpy as np
import pytest

import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden():
    rows = []
    with open(os.path.join(GOLDEN, "memory_update.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                rows.append(tuple(int(v) for v in line.split()))
    return rows


@pytest.mark.parametrize("row", _golden(), ids=lambda r: f"n{r[0]}")
def test_rule_proportions_match_golden(row):
    n, newest, oldest, middle, total, from_mid = row
    assert O.memory_rule(n) == (newest, oldest, total)
    assert n - newest - oldest == middle
    assert total - newest == from_mid


def _deletion_process(counts, nb, pinned, newest, oldest, total):
    """The page's process taken literally: drop the oldest, protect the
    newest, then delete the least-retrieved middle entry one at a time (the
    older of equal ones) until the memory holds `total` entries."""
    kept = list(range(pinned + oldest, nb))
    protected = set(range(nb - newest, nb))
    while len(kept) > total:
        victim = None
        for j in kept:
            if j in protected:
                continue
            if victim is None or counts[j] < counts[victim]:
                victim = j
        kept.remove(victim)
    return kept


def _exhaustive(counts, nb, pinned, newest, oldest, total):
    """Every kept set of the right size; exactly one has every kept middle
    entry ranked above every deleted one under (count, then newer)."""
    lo, hi = pinned + oldest, nb - newest
    mid = list(range(lo, hi))
    winners = []
    for keep in itertools.combinations(mid, total - newest):
        gone = [j for j in mid if j not in keep]
        if all((counts[a], a) > (counts[b], b) for a in keep for b in gone):
            winners.append(list(keep) + list(range(hi, nb)))
    assert len(winners) == 1
    return winners[0]


@pytest.mark.parametrize("seed", range(40))
def test_keep_exhaustive_and_process_tiny(seed):
    rng = np.random.default_rng(seed)
    nb = int(rng.integers(1, 13))
    pinned = int(rng.integers(0, min(nb, 3) + 1))
    n = nb - pinned
    if seed % 2:
        newest, oldest, total = O.memory_rule(n)
    else:
        oldest = int(rng.integers(0, n + 1))
        newest = int(rng.integers(0, n - oldest + 1))
        total = int(rng.integers(newest, n - oldest + 1))
    counts = rng.integers(0, 3, size=nb + 2)   # few values: many ties
    got = O.memory_keep(counts, nb, pinned, newest, oldest, total).tolist()
    assert got == _exhaustive(counts, nb, pinned, newest, oldest, total)
    assert got == _deletion_process(counts, nb, pinned, newest, oldest, total)


def test_keep_closed_forms():
    nb, pinned = 60, 4
    newest, oldest, total = O.memory_rule(nb - pinned)     # 5, 5, 28
    assert (newest, oldest, total) == (5, 5, 28)
    # all counts equal: recency decides, the newest `total` entries remain
    got = O.memory_keep(np.full(nb, 7), nb, pinned, newest, oldest, total)
    assert got.tolist() == list(range(nb - total, nb))
    # counts falling with age reversed (older = more retrieved): the oldest
    # middle entries win, then the protected newest
    c = np.arange(nb)[::-1].copy()
    got = O.memory_keep(c, nb, pinned, newest, oldest, total)
    lo = pinned + oldest
    assert got.tolist() == list(range(lo, lo + total - newest)) + list(range(nb - newest, nb))
    # a heavily retrieved entry among the oldest 10% is still dropped
    c = np.zeros(nb, dtype=np.int64)
    c[pinned] = 10 ** 6
    assert pinned not in O.memory_keep(c, nb, pinned, newest, oldest, total)
    # an entry among the newest 10% with no retrievals is still kept
    c = np.ones(nb, dtype=np.int64)
    c[nb - 1] = 0
    assert nb - 1 in O.memory_keep(c, nb, pinned, newest, oldest, total)


@pytest.mark.parametrize("seed", range(5))
def test_keep_invariants_large(seed):
    rng = np.random.default_rng(100 + seed)
    nb, pinned = 5000, 3
    newest, oldest, total = O.memory_rule(nb - pinned)
    counts = rng.poisson(2.0, size=nb)
    got = O.memory_keep(counts, nb, pinned, newest, oldest, total)
    assert got.shape == (total,)
    assert np.all(np.diff(got) > 0)
    assert got.min() >= pinned + oldest
    assert set(range(nb - newest, nb)) <= set(got.tolist())
    lo, hi = pinned + oldest, nb - newest
    kept_mid = got[got < hi]
    gone = np.setdiff1d(np.arange(lo, hi), kept_mid)
    worst_kept = min(kept_mid.tolist(), key=lambda j: (counts[j], j))
    best_gone = max(gone.tolist(), key=lambda j: (counts[j], j))
    assert (counts[worst_kept], worst_kept) > (counts[best_gone], best_gone)


def test_keep_rejects_bad_counts():
    with pytest.raises(ValueError):
        O.memory_keep(np.zeros(10), 10, 0, 6, 5, 6)       # newest + oldest > n
    with pytest.raises(ValueError):
        O.memory_keep(np.zeros(10), 10, 0, 3, 1, 2)       # total < newest
    with pytest.raises(ValueError):
        O.memory_keep(np.zeros(10), 10, 0, 1, 3, 8)       # total > n - oldest
    with pytest.raises(ValueError):
        O.memory_keep(np.zeros(10), 10, 11, 0, 0, 0)      # pinned > nb


def test_count_retrievals_library_and_closed_form():
    rng = np.random.default_rng(3)
    U, cap, G, k = 3, 50, 7, 9
    idx = np.stack([np.stack([np.sort(rng.choice(cap, k, replace=False)) for _ in range(U)])
                    for _ in range(G)])                    # [G][U][k]
    c, bad = O.count_retrievals(idx, U, cap)
    assert bad == 0
    for u in range(U):
        np.testing.assert_array_equal(c[u], np.bincount(idx[:, u].ravel(), minlength=cap))
    assert c.sum() == G * U * k
    # every row the same selection: each selected block counted G times per unit
    same = np.broadcast_to(np.arange(k), (G, U, k))
    c, _ = O.count_retrievals(same, U, cap)
    assert np.all(c[:, :k] == G) and np.all(c[:, k:] == 0)
    # out-of-range entries are skipped and reported
    c, bad = O.count_retrievals(np.array([[0, cap, -1, 2]]), 1, cap)
    assert bad == 2 and c[0, 0] == 1 and c[0, 2] == 1 and c.sum() == 2


def test_compact_moves_rows_blocks_tail_and_counters():
    bs, D, nb, tail, pinned = 4, 2, 12, 3, 1
    cap_blocks = 16
    T = nb * bs + tail
    # every token row holds its own position: the compacted store says where it came from
    K = np.zeros((2, cap_blocks * bs, D))
    K[:, :T, 0] = np.arange(T)
    K[:, :, 1] = np.arange(2)[:, None]                     # head id
    rep = np.arange(cap_blocks, dtype=np.float64)[:, None] * np.ones((1, 3))
    counts = np.arange(100, 100 + cap_blocks)
    keep = np.array([3, 5, 6, 10, 11])
    T_new, (K2,), (rep2,), c2 = O.memory_compact(keep, pinned=pinned, nb=nb, tail=tail, bs=bs,
                                                  kv=[K], per_block=[rep], counters=counts)
    assert T_new == (pinned + len(keep)) * bs + tail
    src = list(range(pinned)) + keep.tolist()
    expect = [s * bs + o for s in src for o in range(bs)] + [nb * bs + o for o in range(tail)]
    for h in range(2):
        np.testing.assert_array_equal(K2[h, :T_new, 0], expect)
        assert np.all(K2[h, :, 1] == h)
    np.testing.assert_array_equal(rep2[:pinned + len(keep), 0], src)
    np.testing.assert_array_equal(c2[:pinned + len(keep)], counts[src])
    new_nb = pinned + len(keep)
    assert np.all(c2[new_nb:nb + 1] == 0)                  # vacated, up to the old tail block
    np.testing.assert_array_equal(c2[nb + 1:], counts[nb + 1:])
