"""Plain statement of MemLong's dynamic memory update and its retrieval counters.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Source: "MemLong: Memory-Augmented Retrieval for Long Text Modeling" (summary
page), section 2.3.2, "dynamic memory update": when the memory overflows,
counters of how often each entry was retrieved decide what stays.  The newest
10% of the entries are kept (likely still relevant), the oldest 10% are
dropped (likely stale), and in the middle 80% the least retrieved entries are
deleted until the memory holds 50% of what it held.

Readings taken where the page is silent:
  * an entry is one block of the store (one token when the block size is 1);
    the update runs per memory unit: per (batch, kv head) for the dot-product
    modes, per batch row for the cosine bank, whose K/V of every kv head
    follow the bank entry;
  * the percentages are taken with floor: newest = oldest = n // 10 and the
    total kept = n // 2 (the default; every count may also be given);
  * among entries with equal counts the older one (lower index) is deleted
    first -- the same preference for recency as the rule itself;
  * kept entries keep their order and their counters; entries pinned at the
    front (attention-sink blocks) are outside the rule and stay in place; the
    partial block after the last full block (tokens not yet memorised) moves
    with the kept entries, right after them; vacated counters read zero.
"""
from __future__ import annotations

import numpy as np

__all__ = ["memory_rule", "count_retrievals", "memory_keep", "memory_compact"]


def memory_rule(n: int):
    """Counts of the page's rule for n entries: (keep_newest, drop_oldest,
    keep_total) = (floor(n/10), floor(n/10), floor(n/2))."""
    if n < 0:
        raise ValueError("n < 0")
    return n // 10, n // 10, n // 2


def count_retrievals(idx, n_units: int, cap_blocks: int, counters=None):
    """Retrieval-frequency counters: every entry j of a selected row adds one
    to counters[u][j], where the rows are laid out [G][n_units][k] (row r
    belongs to unit r % n_units).  Entries outside [0, cap_blocks) are
    skipped and reported as the second return value."""
    idx = np.asarray(idx)
    idx = idx.reshape(-1, idx.shape[-1]) if idx.ndim else idx.reshape(0, 0)
    c = np.zeros((n_units, cap_blocks), dtype=np.int64) if counters is None else \
        np.array(counters, dtype=np.int64, copy=True)
    bad = 0
    for r in range(idx.shape[0]):
        u = r % n_units
        for j in idx[r]:
            if 0 <= j < cap_blocks:
                c[u, j] += 1
            else:
                bad += 1
    return c, bad


def memory_keep(counts, nb: int, pinned: int, keep_newest: int, drop_oldest: int,
                keep_total: int):
    """Entries kept by the update of one memory unit, in destination order.

    counts[j] is entry j's retrieval count.  The entries under the rule are
    blocks [pinned, nb).  Following the page's steps: the drop_oldest oldest
    are dropped, the keep_newest newest are kept, and from the middle the
    least retrieved are deleted (equal counts: the older first) until
    keep_total entries remain.  Returns the kept absolute indices ascending
    (the pinned blocks, which never move, are not listed)."""
    n = nb - pinned
    if not (0 <= pinned <= nb and keep_newest >= 0 and drop_oldest >= 0
            and keep_newest + drop_oldest <= n and keep_newest <= keep_total <= n - drop_oldest):
        raise ValueError("invalid memory-update counts")
    lo, hi = pinned + drop_oldest, nb - keep_newest
    middle = np.arange(lo, hi)
    c = np.asarray(counts, dtype=np.int64)[lo:hi]
    n_delete = (hi - lo) - (keep_total - keep_newest)
    # deletion order: fewest retrievals first, then oldest first
    order = np.lexsort((middle, c))
    deleted = set(middle[order[:n_delete]].tolist())
    kept_mid = [j for j in middle.tolist() if j not in deleted]
    return np.array(kept_mid + list(range(hi, nb)), dtype=np.int64)


def memory_compact(keep, *, pinned: int, nb: int, tail: int, bs: int, kv=(), per_block=(),
                   counters=None):
    """The store after the update of one memory unit.

    keep: memory_keep's result; kv: arrays [..., T_cap, D] of token rows (the
    unit's K and V pools, every kv head); per_block: arrays [..., cap_blocks,
    ...] indexed by block on their first axis (representations, positions);
    counters [cap_blocks].
    Destination block pinned + t receives block keep[t]; the tail's tokens
    follow the kept blocks.  Returns (T_new, kv', per_block', counters')."""
    nk = len(keep)
    new_nb = pinned + nk
    kv_out = []
    for a in kv:
        b = np.array(a, copy=True)
        for t, s in enumerate(keep):
            d = pinned + t
            b[..., d * bs:(d + 1) * bs, :] = a[..., s * bs:(s + 1) * bs, :]
        if tail:
            b[..., new_nb * bs:new_nb * bs + tail, :] = a[..., nb * bs:nb * bs + tail, :]
        kv_out.append(b)
    pb_out = []
    for a in per_block:
        b = np.array(a, copy=True)
        for t, s in enumerate(keep):
            b[pinned + t] = a[s]
        pb_out.append(b)
    c_out = None
    if counters is not None:
        c = np.asarray(counters)
        c_out = np.array(c, copy=True)
        for t, s in enumerate(keep):
            c_out[pinned + t] = c[s]
        end = min(nb + 1, c.shape[0])
        c_out[new_nb:end] = 0
    return new_nb * bs + tail, kv_out, pb_out, c_out
