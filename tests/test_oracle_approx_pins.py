"""Pins of the oracle's two-stage approximate token retrieval (RetrievalAttention
summary, "proposed method": retrieval of the few keys that matter by an
approximate search that reads 1-3% of them), against things other than
itself: the exact search it approximates in its limiting cases, the closed
form of its recall, and brute force on a tiny input.

A plausible slip (scoring groups by a sum instead of a mean, keeping the wrong
end of the ranking, dropping the last kept group, letting tokens outside the
candidate range in) fails at least one of them."""
import numpy as np
import pytest

import oracle as O
from retrieval_block_sparse_b200 import synth


def _inputs(T=4096, D=32, m=4, seed=0, recipe="drift"):
    w = synth.WORKLOADS["token-retrieval-decode-1m"].scaled(
        context=T, head_dim=64 if D <= 64 else 128, n_q_heads=m, n_kv_heads=1, top_k=32,
        sink=64, window=128, recipe=recipe, seed=seed)
    x = synth.decode_inputs(w)
    K = O.widen(x["K"][0, 0], "bf16")
    qs = O.widen(x["q"][0, :m], "bf16")
    return w, K, qs


@pytest.mark.parametrize("group", [16, 64])
def test_keeping_every_group_is_the_exact_search(group):
    w, K, qs = _inputs(seed=1)
    n_groups = O.candidate_blocks(w.context, group, w.sink, w.window).size
    r = O.two_stage_select(qs, K, w.context, group=group, sink=w.sink, window=w.window,
                           groups_kept=n_groups, k=w.top_k)
    exact = O.exact_token_select(qs, K, w.context, w.sink, w.window, w.top_k)
    np.testing.assert_array_equal(r["tokens"], exact)
    assert O.recall(r["tokens"], exact) == 1.0


def test_groups_of_one_token_are_the_exact_search():
    w, K, qs = _inputs(T=2048, seed=2, recipe="shifted")
    r = O.two_stage_select(qs, K, w.context, group=1, sink=w.sink, window=w.window,
                           groups_kept=w.top_k, k=w.top_k)
    exact = O.exact_token_select(qs, K, w.context, w.sink, w.window, w.top_k)
    np.testing.assert_array_equal(r["tokens"], exact)


def test_recall_is_the_share_of_exact_tokens_in_kept_groups_and_grows_with_groups():
    w, K, qs = _inputs(seed=3)
    exact = O.exact_token_select(qs, K, w.context, w.sink, w.window, w.top_k)
    last = -1.0
    for kept in (1, 2, 4, 8, 16, 32):
        r = O.two_stage_select(qs, K, w.context, group=64, sink=w.sink, window=w.window,
                               groups_kept=kept, k=w.top_k)
        covered = {t for g in r["groups"] for t in range(g * 64, (g + 1) * 64)}
        closed = len(set(exact.tolist()) & covered) / w.top_k
        rec = O.recall(r["tokens"], exact)
        assert rec == pytest.approx(closed)
        assert rec >= last
        last = rec
        assert r["scanned"] == O.candidate_blocks(w.context, 64, w.sink, w.window).size + \
            sum(1 for g in r["groups"] for t in range(g * 64, (g + 1) * 64)
                if w.sink <= t < w.context - w.window)
        assert np.all(np.diff(r["tokens"]) > 0)
        assert np.all((r["tokens"] >= w.sink) & (r["tokens"] < w.context - w.window))


def test_brute_force_tiny():
    rng = np.random.default_rng(4)
    T, D, group, sink, window = 40, 3, 4, 5, 7
    K = rng.standard_normal((T, D))
    qs = rng.standard_normal((2, D))
    r = O.two_stage_select(qs, K, T, group=group, sink=sink, window=window, groups_kept=3, k=4)
    q = qs.sum(axis=0)
    w0 = T - window
    groups = [g for g in range(T // group)
              if (g + 1) * group > sink and g * group < w0]      # full groups meeting [sink, w0)
    gs = sorted(groups, key=lambda g: (-(K[g * group:(g + 1) * group].mean(axis=0) @ q), g))[:3]
    toks = [t for g in sorted(gs) for t in range(g * group, (g + 1) * group) if sink <= t < w0]
    best = sorted(sorted(toks, key=lambda t: (-(K[t] @ q), t))[:4])
    assert sorted(gs) == r["groups"].tolist()
    assert best == r["tokens"].tolist()


def test_drift_keys_make_group_means_informative():
    # on keys that drift along the sequence, a 2% scan recovers much of the
    # exact top-k; on independent keys the group means carry little signal
    out = {}
    for recipe in ("drift", "shifted"):
        w, K, qs = _inputs(T=16384, seed=5, recipe=recipe)
        exact = O.exact_token_select(qs, K, w.context, w.sink, w.window, w.top_k)
        r = O.two_stage_select(qs, K, w.context, group=64, sink=w.sink, window=w.window,
                               groups_kept=3, k=w.top_k)
        out[recipe] = O.recall(r["tokens"], exact)
        assert r["scanned"] / (w.context - w.sink - w.window) < 0.04
    assert out["drift"] > 2 * out["shifted"]
    assert out["drift"] >= 0.3
