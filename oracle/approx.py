"""Plain statement of two-stage approximate token retrieval (block size 1).

TEST INFRASTRUCTURE ONLY (see the package docstring).

Source: RetrievalAttention summary (arXiv 2409.10516), "proposed method": the
attention of a query is computed over the few keys that matter, found by an
approximate nearest-neighbour search instead of a scan of every key, and a
search adapted to the query/key distribution gap reads only 1-3% of the
keys.  The page names no index structure; the reading taken here is the
plainest one that the rest supports:

  * index: consecutive groups of c candidate tokens (the blocks of size c of
    the candidate rule), each represented by the mean of its keys;
  * stage 1: score every group by its mean key against the queries that
    share the selection (the GQA group summed), keep the best C groups;
  * stage 2: score every token of the kept groups exactly, keep the best k;
  * ties go to the lower index in both stages.

The keys read are the group means plus C * c tokens.  Recall is measured
against the exact top-k over every candidate token.
"""
from __future__ import annotations

import numpy as np

from .retrieval import candidate_blocks, rep_mean, score_dot, top_k

__all__ = ["exact_token_select", "two_stage_select", "recall"]


def exact_token_select(qs, K, T: int, sink: int, window: int, k: int):
    """The k best candidate tokens by sum_q q . k_t (block size 1), ascending."""
    cand = candidate_blocks(T, 1, sink, window)
    s = score_dot(qs, np.asarray(K, dtype=np.float64)[cand][:, None, :])
    return cand[top_k(s, k)]


def two_stage_select(qs, K, T: int, *, group: int, sink: int, window: int, groups_kept: int,
                     k: int):
    """Approximate selection of k tokens (see the module docstring).

    qs [m][D] the queries sharing the selection; K [>= T][D] the keys (fp64).
    Returns dict: tokens (k, ascending), groups (kept group ids, ascending),
    scanned (keys read: one mean per candidate group + the kept groups' tokens),
    and the two stages' inputs: cand_groups (candidate group ids), group_scores
    (their stage-1 scores), kept_tokens (the kept groups' candidate tokens,
    ascending) and token_scores (their stage-2 scores)."""
    K = np.asarray(K, dtype=np.float64)
    w0 = max(T - window, 0)
    groups = candidate_blocks(T, group, sink, window)
    means = np.stack([rep_mean(K[g * group:(g + 1) * group])[0] for g in groups]) \
        if groups.size else np.zeros((0, K.shape[1]))
    s1 = score_dot(qs, means[:, None, :]) if groups.size else np.zeros(0)
    kept = groups[top_k(s1, min(groups_kept, groups.size))]
    toks = np.array([t for g in kept for t in range(g * group, (g + 1) * group)
                     if sink <= t < w0], dtype=np.int64)
    if toks.size < k:
        raise ValueError("the kept groups hold fewer than k candidate tokens")
    s2 = score_dot(qs, K[toks][:, None, :])
    return {"tokens": toks[top_k(s2, k)], "groups": kept,
            "scanned": int(groups.size + toks.size),
            "cand_groups": groups, "group_scores": s1, "kept_tokens": toks, "token_scores": s2}


def recall(approx_tokens, exact_tokens) -> float:
    """Fraction of the exact top-k found by the approximate selection."""
    exact = set(np.asarray(exact_tokens).tolist())
    return len(exact & set(np.asarray(approx_tokens).tolist())) / max(len(exact), 1)
