"""Pins of the fp64 oracle against things other than itself: closed forms,
invariants the method fixes, library routines for special cases, brute force
on tiny inputs, and the derived workload sizes in tests/golden.

Each pin is chosen so that a plausible slip (an off-by-one block bound, a
dropped term, a transposed operand, a wrong GQA grouping, a wrong tie rule,
a softmax over the wrong axis) fails at least one of them.
"""
import itertools
import math
import os

import numpy as np
import pytest
import scipy.special
import scipy.spatial.distance
import torch

import oracle as O
from retrieval_block_sparse_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _sdpa(q, K, V, scale, mask=None):
    """torch's scaled_dot_product_attention in fp64 (library routine)."""
    qt = torch.from_numpy(np.atleast_2d(q))[None, None]
    kt = torch.from_numpy(K)[None, None]
    vt = torch.from_numpy(V)[None, None]
    m = None if mask is None else torch.from_numpy(mask)[None, None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=m, scale=scale)
    return o[0, 0].numpy()


# ---------------------------------------------------------------------------
# sizes: golden fixture + brute-force token enumeration


def _golden_rows():
    rows = []
    with open(os.path.join(GOLDEN, "workload_sizes.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                p = line.split()
                rows.append((p[0], *map(int, p[1:])))
    return rows


@pytest.mark.parametrize("row", _golden_rows(), ids=lambda r: r[0])
def test_candidate_and_attended_sizes_match_golden(row):
    name, T, bs, S, W, k, nb, nc, first, last, att, att_is_max = row
    cand = O.candidate_blocks(T, bs, S, W)
    assert T // bs == nb
    assert cand.shape[0] == nc and cand[0] == first and cand[-1] == last
    assert np.all(np.diff(cand) == 1)
    w = synth.WORKLOADS[name]
    assert (w.context, w.block_size, w.sink, w.window, w.top_k) == (T, bs, S, W, k)
    if att_is_max:
        # the block straddling the window start is the only one overlapping it
        worst = O.attended_tokens(T, bs, S, W, cand[:k])
        best_case = O.attended_tokens(T, bs, S, W, cand[-k:])
        assert worst.shape[0] == att and best_case.shape[0] < att
    else:
        sel = cand[np.linspace(0, nc - 1, k).astype(int)] if nc else cand[:0]
        assert O.attended_tokens(T, bs, S, W, sel).shape[0] == att


@pytest.mark.parametrize("T,bs,S,W", [(37, 5, 3, 7), (40, 8, 0, 0), (40, 8, 8, 8),
                                      (41, 8, 9, 2), (12, 4, 20, 0), (16, 4, 0, 16),
                                      (9, 1, 2, 3), (50, 7, 6, 13)])
def test_candidates_brute_force(T, bs, S, W):
    w0 = max(T - W, 0)
    expect = []
    for j in range(T):
        toks = list(range(j * bs, (j + 1) * bs))
        if toks[-1] >= T:
            continue
        if any(S <= t < w0 for t in toks):
            expect.append(j)
    assert O.candidate_blocks(T, bs, S, W).tolist() == expect


def test_attended_union_counts_each_token_once():
    T, bs, S, W = 100, 10, 15, 25
    got = O.attended_tokens(T, bs, S, W, [1, 4, 7])
    expect = sorted(set(range(15)) | set(range(10, 20)) | set(range(40, 50)) |
                    set(range(70, 80)) | set(range(75, 100)))
    assert got.tolist() == expect
    # MemLong 2.3.4: with no sink/window the attention window is k * block size
    assert O.attended_tokens(T, bs, 0, 0, [0, 3, 9]).shape[0] == 3 * bs


# ---------------------------------------------------------------------------
# representations


def test_rep_mean_arithmetic_progression():
    a, d = _rng(0).normal(size=8), _rng(1).normal(size=8)
    bs = 13
    K = np.stack([a + t * d for t in range(bs)])
    np.testing.assert_allclose(O.rep_mean(K)[0], a + (bs - 1) / 2 * d, rtol=0, atol=1e-12)
    np.testing.assert_allclose(O.rep_mean(np.tile(a, (5, 1)))[0], a, atol=1e-15)


def test_rep_topr_single_probe_is_argmax():
    K = _rng(2).normal(size=(32, 16))
    p = _rng(3).normal(size=16)
    c, keys, recv = O.rep_topr_attention(K, p[None], 1, 0.25)
    assert c.tolist() == [int(np.argmax(K @ p))]
    np.testing.assert_array_equal(keys[0], K[c[0]])
    # softmax over the block: received attention of one probe sums to 1
    assert abs(recv.sum() - 1.0) < 1e-12


def test_rep_topr_zero_probe_ties_take_first_tokens():
    K = _rng(4).normal(size=(20, 8))
    c, _, recv = O.rep_topr_attention(K, np.zeros((3, 8)), 4, 0.3)
    assert c.tolist() == [0, 1, 2, 3]
    np.testing.assert_allclose(recv, np.full(20, 3 / 20), atol=1e-15)


def test_rep_topr_probes_each_pick_their_token_and_output_is_sorted():
    D, bs = 16, 24
    K = _rng(5).normal(size=(bs, D)) * 0.01
    K[17] = 50 * np.eye(D)[0]
    K[3] = 50 * np.eye(D)[1]
    probe = np.stack([np.eye(D)[0], np.eye(D)[1]])
    c, keys, recv = O.rep_topr_attention(K, probe, 2, 1.0)
    assert c.tolist() == [3, 17]
    np.testing.assert_array_equal(keys, K[[3, 17]])
    assert abs(recv.sum() - 2.0) < 1e-12
    # r = bs keeps every token in order
    c_all, _, _ = O.rep_topr_attention(K, probe, bs, 1.0)
    assert c_all.tolist() == list(range(bs))


def test_rep_topr_softmax_is_over_tokens_not_probes():
    # two tokens, two probes: probe 0 prefers token 0 weakly, probe 1 prefers
    # token 1 strongly.  Per-probe softmax over tokens gives token 1 the larger
    # total; a softmax over probes (wrong axis) would tie them at 1 each.
    K = np.array([[1.0, 0.0], [0.0, 1.0]])
    probe = np.array([[0.2, 0.0], [0.0, 3.0]])
    c, _, recv = O.rep_topr_attention(K, probe, 1, 1.0)
    e0 = 1 / (1 + math.exp(-0.2))
    e1 = 1 / (1 + math.exp(-3.0))
    np.testing.assert_allclose(recv, [e0 + (1 - e1), (1 - e0) + e1], atol=1e-15)
    assert c.tolist() == [1]


def test_rep_embedding_unit_norm_and_direction():
    e = _rng(6).normal(size=768) * 7.3
    m = O.rep_embedding(e)
    assert abs(np.linalg.norm(m) - 1) < 1e-14
    assert 1 - scipy.spatial.distance.cosine(e, m) > 1 - 1e-14


def test_memorize_modes_shapes_and_identity():
    K = _rng(7).normal(size=(64, 8))
    reps, chosen = O.memorize(K, "identity", 1)
    np.testing.assert_array_equal(reps[:, 0], K)
    assert chosen is None
    L = _rng(8).normal(size=(4, 8))
    reps, _ = O.memorize(K[:60], "external", 15, landmarks=L)
    np.testing.assert_array_equal(reps[:, 0], L)
    reps, chosen = O.memorize(K, "topr_attn", 16, r=3, probe=_rng(9).normal(size=(5, 8)))
    assert reps.shape == (4, 3, 8) and chosen.shape == (4, 3)
    for j in range(4):
        np.testing.assert_array_equal(reps[j], K[16 * j + chosen[j]])
    reps, _ = O.memorize(K, "mean", 16)
    np.testing.assert_allclose(reps[2, 0], K[32:48].sum(0) / 16, atol=1e-14)


# ---------------------------------------------------------------------------
# scoring


def test_score_dot_basis_closed_form():
    # rep key (j, i) = c_{j,i} e_{d(j,i)}: s_j = sum_q sum_i c_{j,i} q[d(j,i)]
    D, n, r, m = 12, 7, 3, 4
    rng = _rng(10)
    qs = rng.normal(size=(m, D))
    dsel = rng.integers(0, D, size=(n, r))
    c = rng.normal(size=(n, r))
    reps = np.zeros((n, r, D))
    for j in range(n):
        for i in range(r):
            reps[j, i, dsel[j, i]] = c[j, i]
    expect = [sum(c[j, i] * qs[q, dsel[j, i]] for q in range(m) for i in range(r)) for j in range(n)]
    np.testing.assert_allclose(O.score_dot(qs, reps), expect, atol=1e-12)


def test_score_dot_max_variant_closed_form():
    # the same basis keys: the max variant takes, per block, the largest of its
    # r keys' group-summed dot products (not their sum)
    D, n, r, m = 12, 7, 3, 4
    rng = _rng(11)
    qs = rng.normal(size=(m, D))
    dsel = rng.integers(0, D, size=(n, r))
    c = rng.normal(size=(n, r))
    reps = np.zeros((n, r, D))
    for j in range(n):
        for i in range(r):
            reps[j, i, dsel[j, i]] = c[j, i]
    expect = [max(sum(c[j, i] * qs[q, dsel[j, i]] for q in range(m)) for i in range(r))
              for j in range(n)]
    np.testing.assert_allclose(O.score_dot(qs, reps, "max"), expect, atol=1e-12)
    # one key per block: max and sum agree; the order of the keys does not matter
    np.testing.assert_allclose(O.score_dot(qs, reps[:, :1], "max"), O.score_dot(qs, reps[:, :1]))
    perm = reps[:, ::-1]
    np.testing.assert_allclose(O.score_dot(qs, perm, "max"), O.score_dot(qs, reps, "max"))
    # a block whose keys are all equal scores max = sum / r
    same = np.repeat(reps[:, :1], r, axis=1)
    np.testing.assert_allclose(O.score_dot(qs, same, "max") * r, O.score_dot(qs, same), atol=1e-12)
    with pytest.raises(ValueError):
        O.score_dot(qs, reps, "mean")


def test_decode_gqa_grouping_closed_form():
    # q head i = (i+1) u, every rep key = u: kv head h sums q heads h*g..h*g+g-1
    B, Hq, Hkv, D, T, bs = 1, 8, 2, 4, 32, 4
    g = Hq // Hkv
    u = np.array([1.0, 0.0, 0.0, 0.0])
    q = np.stack([(i + 1) * u for i in range(Hq)])[None].astype(np.float32)
    K = np.zeros((B, Hkv, T, D), dtype=np.float32)
    reps = np.tile(u, (B, Hkv, T // bs, 2, 1))
    res = O.decode(q, K, K, reps, dtype="f32", block_size=bs, sink=0, window=0,
                   top_k_blocks=1)
    for h in range(Hkv):
        expect = 2 * sum(i + 1 for i in range(h * g, (h + 1) * g))
        np.testing.assert_allclose(res["scores"][0, h], expect, atol=1e-12)


def test_score_cosine_library_and_range():
    rng = _rng(11)
    M = rng.normal(size=(9, 30))
    rq = rng.normal(size=30) * 3
    s = O.score_cosine(rq, M)
    lib = [1 - scipy.spatial.distance.cosine(rq, M[j]) for j in range(9)]
    np.testing.assert_allclose(s, lib, atol=1e-14)
    assert np.all(np.abs(s) <= 1 + 1e-15)
    M2 = np.stack([rq * 2.5, -rq, rq + 0.0])
    np.testing.assert_allclose(O.score_cosine(rq, M2), [1, -1, 1], atol=1e-14)


# ---------------------------------------------------------------------------
# selection


def _topk_brute(s, k):
    """Rank counting: i is chosen iff fewer than k entries beat it, where a
    beats b iff s_a > s_b, or s_a == s_b and a < b."""
    n = len(s)
    out = []
    for i in range(n):
        beaten_by = sum(1 for j in range(n) if s[j] > s[i] or (s[j] == s[i] and j < i))
        if beaten_by < k:
            out.append(i)
    return out


@pytest.mark.parametrize("seed", range(12))
def test_topk_brute_force_with_ties(seed):
    rng = _rng(100 + seed)
    n = int(rng.integers(1, 40))
    levels = rng.normal(size=int(rng.integers(1, 6)))
    s = levels[rng.integers(0, len(levels), size=n)]
    for k in sorted({0, 1, n // 2, n - 1, n} - {-1}):
        if 0 <= k <= n:
            assert O.top_k(s, k).tolist() == _topk_brute(s, k)


def test_topk_subsets_exhaustive_tiny():
    # every k-subset: the chosen one maximises the sorted score vector
    s = np.array([0.5, -1.0, 0.5, 2.0, 0.5, -1.0])
    for k in range(len(s) + 1):
        best = max(itertools.combinations(range(len(s)), k),
                   key=lambda c: (sorted((s[i] for i in c), reverse=True), [-i for i in c]))
        assert O.top_k(s, k).tolist() == sorted(best)


def test_topk_signed_zero_is_a_tie():
    s = np.array([-0.0, 0.0, -0.0, 1.0])
    assert O.top_k(s, 2).tolist() == [0, 3]


# ---------------------------------------------------------------------------
# attention


def test_attention_matches_library_and_lse():
    rng = _rng(12)
    q, K, V = rng.normal(size=16), rng.normal(size=(50, 16)), rng.normal(size=(50, 16))
    o, lse, p = O.softmax_attention(q, K, V, 0.25)
    np.testing.assert_allclose(o, _sdpa(q, K, V, 0.25)[0], atol=1e-13)
    assert abs(lse - scipy.special.logsumexp(0.25 * K @ q)) < 1e-12
    np.testing.assert_allclose(p, scipy.special.softmax(0.25 * K @ q), atol=1e-15)


def test_attention_special_cases():
    rng = _rng(13)
    K, V = rng.normal(size=(9, 8)), rng.normal(size=(9, 8))
    # one attended token -> its value
    o, lse, _ = O.softmax_attention(rng.normal(size=8), K[:1], V[:1], 0.5)
    np.testing.assert_allclose(o, V[0], atol=1e-15)
    # zero query -> mean of the values, lse = ln n
    o, lse, p = O.softmax_attention(np.zeros(8), K, V, 0.5)
    np.testing.assert_allclose(o, V.mean(0), atol=1e-14)
    assert abs(lse - math.log(9)) < 1e-14
    # one-hot values -> the weights themselves; weights sum to 1
    q = rng.normal(size=8)
    o, _, p = O.softmax_attention(q, K, np.eye(9), 0.5)
    np.testing.assert_allclose(o, p, atol=1e-15)
    assert abs(p.sum() - 1) < 1e-14
    # convex hull: each coordinate within [min V, max V]
    o, _, _ = O.softmax_attention(q * 40, K, V, 1.0)
    assert np.all(o >= V.min(0) - 1e-12) and np.all(o <= V.max(0) + 1e-12)


@pytest.mark.parametrize("nsplit", [1, 2, 3, 7, 40])
def test_merge_split_invariance(nsplit):
    rng = _rng(14)
    q, K, V = rng.normal(size=32) * 2, rng.normal(size=(40, 32)), rng.normal(size=(40, 32))
    o_ref, lse_ref, _ = O.softmax_attention(q, K, V, 0.3)
    cuts = np.linspace(0, 40, nsplit + 1).astype(int)
    parts = [O.split_partial(q, K[a:b], V[a:b], 0.3) for a, b in zip(cuts[:-1], cuts[1:])]
    o, lse = O.merge_partials(parts)
    np.testing.assert_allclose(o, o_ref, atol=1e-12)
    assert abs(lse - lse_ref) < 1e-12


def test_decode_all_candidates_equals_full_attention():
    # invariant (a): k = every candidate, tail inside the window -> dense
    # softmax attention over all T tokens, per q head (GQA, g = 2)
    B, Hq, Hkv, D, T, bs, S, W = 2, 4, 2, 16, 70, 8, 5, 14
    rng = _rng(15)
    q = rng.normal(size=(B, Hq, D)).astype(np.float32)
    K = rng.normal(size=(B, Hkv, T, D)).astype(np.float32)
    V = rng.normal(size=(B, Hkv, T, D)).astype(np.float32)
    Kd = K.astype(np.float64)
    reps = np.stack([np.stack([O.memorize(Kd[b, h], "mean", bs)[0] for h in range(Hkv)])
                     for b in range(B)])
    nc = O.candidate_blocks(T, bs, S, W).shape[0]
    res = O.decode(q, K, V, reps, dtype="f32", block_size=bs, sink=S, window=W,
                   top_k_blocks=nc)
    for b in range(B):
        for i in range(Hq):
            h = i // 2
            full = _sdpa(q[b, i].astype(np.float64), Kd[b, h], V[b, h].astype(np.float64), D ** -0.5)
            np.testing.assert_allclose(res["out"][b, i], full[0], atol=1e-12)
            lse = scipy.special.logsumexp(D ** -0.5 * Kd[b, h] @ q[b, i].astype(np.float64))
            assert abs(res["lse"][b, i] - lse) < 1e-12


def test_prefill_all_blocks_equals_causal_attention():
    # retrieval-causal attention with every past block retrieved is ordinary
    # causal attention over [past ; chunk] (MemLong 2.3.3, Figure 3)
    Hq, Hkv, D, T, bs, Nq = 4, 2, 8, 24, 6, 5
    rng = _rng(16)
    Q = rng.normal(size=(1, Hq, Nq, D)).astype(np.float32)
    K = rng.normal(size=(1, Hkv, T, D)).astype(np.float32)
    V = rng.normal(size=(1, Hkv, T, D)).astype(np.float32)
    Kc = rng.normal(size=(1, Hkv, Nq, D)).astype(np.float32)
    Vc = rng.normal(size=(1, Hkv, Nq, D)).astype(np.float32)
    reps = np.stack([O.memorize(K[0, h].astype(np.float64), "mean", bs)[0] for h in range(Hkv)])[None]
    res = O.prefill(Q, K, V, Kc, Vc, dtype="f32", block_size=bs, sink=0, window=0,
                    top_k_blocks=T // bs, score_mode="dot", reps=reps)
    n = T + Nq
    mask = np.zeros((Nq, n), dtype=bool)
    for i in range(Nq):
        mask[i, :T + i + 1] = True
    for hq in range(Hq):
        h = hq // 2
        Kall = np.concatenate([K[0, h], Kc[0, h]]).astype(np.float64)
        Vall = np.concatenate([V[0, h], Vc[0, h]]).astype(np.float64)
        full = _sdpa(Q[0, hq].astype(np.float64), Kall, Vall, D ** -0.5, mask)
        np.testing.assert_allclose(res["out"][0, hq], full, atol=1e-12)


def test_prefill_dot_scores_are_chunk_summed_query():
    Hq, Hkv, D, T, bs, Nq = 2, 1, 4, 12, 3, 3
    rng = _rng(17)
    Q = rng.normal(size=(1, Hq, Nq, D)).astype(np.float32)
    K = rng.normal(size=(1, Hkv, T, D)).astype(np.float32)
    Kc = np.zeros((1, Hkv, Nq, D), dtype=np.float32)
    reps = O.memorize(K[0, 0].astype(np.float64), "mean", bs)[0][None, None]
    res = O.prefill(Q, K, K, Kc, Kc, dtype="f32", block_size=bs, sink=0, window=0,
                    top_k_blocks=2, score_mode="dot", reps=reps)
    expect = [sum(float(Q[0, hq, i].astype(np.float64) @ reps[0, 0, j, 0])
                  for hq in range(Hq) for i in range(Nq)) for j in range(T // bs)]
    np.testing.assert_allclose(res["scores"][0, 0], expect, atol=1e-12)


def _cosine_prefill_case(seed):
    """Memory of 10 blocks of 4 tokens, sink 6, window 10: block 0 lies in the
    sink, blocks 8 and 9 in the window, so the candidates are blocks 1..7 and
    candidate c is block c + 1 (a non-zero candidate offset).  Bank entry j is
    the one-hot vector e_j (orthogonal entries: cosines are closed forms)."""
    Hq, Hkv, D, T, bs, Nq, S, W = 4, 2, 8, 40, 4, 3, 6, 10
    rng = _rng(seed)
    Q = rng.normal(size=(2, Hq, Nq, D)).astype(np.float32)
    K = rng.normal(size=(1, Hkv, T, D)).astype(np.float32)
    V = rng.normal(size=(1, Hkv, T, D)).astype(np.float32)
    Kc = rng.normal(size=(2, Hkv, Nq, D)).astype(np.float32)
    Vc = rng.normal(size=(2, Hkv, Nq, D)).astype(np.float32)
    bank = np.eye(T // bs)
    return Q, K, V, Kc, Vc, bank, bs, S, W


def test_prefill_cosine_selection_is_shared_and_offset():
    # MemLong 2.3.2: each query chunk retrieves by cosine(r_q, M_j) over the
    # memory's candidate blocks, one selection for all heads.  r_q mixes bank
    # directions with known weights, so the cosines are weight / |r_q|; the
    # heaviest directions include a sink block (0) and a window block (9),
    # which are not candidates and must not be selected.
    Q, K, V, Kc, Vc, bank, bs, S, W = _cosine_prefill_case(18)
    T, D, Nq = K.shape[2], K.shape[3], Q.shape[2]
    weights = [{0: 5.0, 2: 3.0, 5: 2.0, 9: 4.0, 6: 0.5},
               {7: 2.5, 1: 2.0, 9: 6.0, 3: 1.0, 0: 3.0}]
    expect = [[2, 5], [1, 7]]
    qe = np.zeros((2, bank.shape[1]))
    for c, wc in enumerate(weights):
        for j, a in wc.items():
            qe[c, j] = a
    res = O.prefill(Q, K, V, Kc, Vc, dtype="f32", block_size=bs, sink=S, window=W,
                    top_k_blocks=2, score_mode="cosine", query_embed=qe, bank=bank)
    np.testing.assert_array_equal(res["cand"], np.arange(1, 8))
    assert res["idx"].shape == (2, 1, 2)
    for c in range(2):
        norm = math.sqrt(sum(a * a for a in weights[c].values()))
        closed = [weights[c].get(j, 0.0) / norm for j in range(1, 8)]
        np.testing.assert_allclose(res["scores"][c, 0], closed, atol=1e-15)
        np.testing.assert_array_equal(res["idx"][c, 0], expect[c])
        # every q head attends sink U the chunk's selected blocks U window,
        # then its own chunk causally (torch fp64 attention, explicit mask)
        toks = sorted(set(range(S)) | set(range(T - W, T)) |
                      {t for j in expect[c] for t in range(j * bs, (j + 1) * bs)})
        for hq in range(Q.shape[1]):
            h = hq // 2
            Kall = np.concatenate([K[0, h, toks], Kc[c, h]]).astype(np.float64)
            Vall = np.concatenate([V[0, h, toks], Vc[c, h]]).astype(np.float64)
            n = len(toks)
            mask = np.zeros((Nq, n + Nq), dtype=bool)
            for i in range(Nq):
                mask[i, :n + i + 1] = True
            ref = _sdpa(Q[c, hq].astype(np.float64), Kall, Vall, D ** -0.5, mask)
            np.testing.assert_allclose(res["out"][c, hq], ref, atol=1e-12)


def test_prefill_cosine_every_candidate_is_causal_attention():
    # k = every candidate: sink U blocks 1..7 U window covers all T past
    # tokens, so every row is causal attention over [past ; chunk], for every
    # q head, whatever the query embedding
    Q, K, V, Kc, Vc, bank, bs, S, W = _cosine_prefill_case(19)
    T, D, Nq = K.shape[2], K.shape[3], Q.shape[2]
    qe = _rng(20).normal(size=(2, bank.shape[1]))
    res = O.prefill(Q, K, V, Kc, Vc, dtype="f32", block_size=bs, sink=S, window=W,
                    top_k_blocks=7, score_mode="cosine", query_embed=qe, bank=bank)
    mask = np.zeros((Nq, T + Nq), dtype=bool)
    for i in range(Nq):
        mask[i, :T + i + 1] = True
    for c in range(2):
        np.testing.assert_array_equal(res["idx"][c, 0], np.arange(1, 8))
        for hq in range(Q.shape[1]):
            h = hq // 2
            Kall = np.concatenate([K[0, h], Kc[c, h]]).astype(np.float64)
            Vall = np.concatenate([V[0, h], Vc[c, h]]).astype(np.float64)
            full = _sdpa(Q[c, hq].astype(np.float64), Kall, Vall, D ** -0.5, mask)
            np.testing.assert_allclose(res["out"][c, hq], full, atol=1e-12)
            lse = scipy.special.logsumexp(
                np.where(mask, D ** -0.5 * (Kall @ Q[c, hq].astype(np.float64).T).T, -np.inf),
                axis=1)
            np.testing.assert_allclose(res["lse"][c, hq], lse, atol=1e-12)


# ---------------------------------------------------------------------------
# retrieval sanity on the synthetic recipes (statistical, not parity)


def test_planted_blocks_are_retrieved():
    w = synth.WORKLOADS["infllm-decode-128k"].scaled(context=16384, window=1024, top_k=16,
                                                     n_planted=8)
    x = synth.decode_inputs(w)
    reps = np.zeros((1, w.n_kv_heads, w.n_blocks, w.n_rep, w.head_dim))
    K = O.widen(x["K"], "bf16")
    probe = O.widen(x["probe"], "bf16")
    for h in range(w.n_kv_heads):
        reps[0, h] = O.memorize(K[0, h], "topr_attn", w.block_size, w.n_rep, probe=probe[h])[0]
    res = O.decode(x["q"], x["K"], x["V"], reps, dtype="bf16", block_size=w.block_size,
                   sink=w.sink, window=w.window, top_k_blocks=w.top_k)
    hits = sum(len(set(res["idx"][0, h]) & set(x["planted_blocks"][0, h]))
               for h in range(w.n_kv_heads))
    nc = res["cand"].shape[0]
    chance = w.n_kv_heads * w.n_planted * w.top_k / nc
    assert hits > 4 * chance


def test_landmark_query_retrieves_its_block():
    w = synth.WORKLOADS["landmark-decode-b16"].scaled(batch=2, n_q_heads=4, n_kv_heads=4,
                                                      context=5000)
    x = synth.decode_inputs(w)
    L = O.widen(x["landmarks"], "bf16")[..., None, :]
    res = O.decode(x["q"], x["K"], x["V"], L, dtype="bf16", block_size=w.block_size,
                   sink=w.sink, window=w.window, top_k_blocks=w.top_k)
    hit = [x["landmark_pick"][b, h] in res["idx"][b, h] for b in range(2) for h in range(4)]
    assert all(hit)


def test_cosine_query_retrieves_its_source_chunk():
    w = synth.WORKLOADS["memlong-cosine-prefill"].scaled(context=40 * 64, block_size=64,
                                                         chunk_len=4, n_q_heads=2, n_kv_heads=2,
                                                         head_dim=8)
    x = synth.prefill_inputs(w)
    bank = np.stack([O.rep_embedding(e) for e in x["bank_embed"]])
    for c in range(w.n_chunks):
        s = O.score_cosine(x["query_embed"][c], bank)
        assert int(np.argmax(s)) == x["query_source"][c]
        assert s.max() > 0.9
