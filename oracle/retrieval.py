"""Plain fp64 statement of context-memory retrieval attention.

TEST INFRASTRUCTURE ONLY (see the package docstring).  Slow on purpose: every
step is written the way the method defines it, on fp64 values widened exactly
from the stored fp32 / bf16 inputs, with numpy primitives (matmul, sort, exp)
as the only library steps.

Sources (pages, by title and section):
  [ML]  "MemLong: Memory-Augmented Retrieval for Long Text Modeling" (summary
        page): section 2.2.1 task definition (fixed-size chunks), 2.2.2 modules
        (memory = K-V pairs + representation embeddings), 2.3.2 retrieval
        process (cosine against the memory, top-k chunk indices) and
        memorisation process M(k, v; r^m), 2.3.3 / Figure 3 retrieval-causal
        attention (local causal + bidirectional over retrieved chunks),
        2.3.4 inference (attention window k * chunk size).
  [IL]  InfLLM article (Tsinghua NLP, "1024K context, 100% recall"), sections
        "method" / "overall framework": sliding window of local tokens plus a
        few memory units; memory units are contiguous token blocks; each unit
        is represented by the tokens that received the highest attention.
  [LM]  "Landmark Attention: Random-Access Infinite Context Length for
        Transformers" (review), section "proposed method": fixed-length blocks,
        one landmark key per block, blocks retrieved by query-landmark
        similarity, then standard attention over the retrieved tokens.
  [RA]  RetrievalAttention summary (arXiv 2409.10516), "proposed method":
        token-level retrieval (every key its own unit) by vector search.

Readings taken where the pages are silent:
  * candidate rule: a block is scored iff it is a full block with at least one
    token in [sink, T - window);
  * attended set: sink U retrieved blocks U window as a set (each token once);
  * r > 1 representative keys are combined by summing their dot products;
    GQA groups sum their q heads' dot products;
  * "received attention" = per probe query, softmax over the block's own
    tokens with scale 1/sqrt(D), summed over the probe queries;
  * ties (top-k and top-r) go to the lowest index;
  * prefill dot-mode selection is shared by the chunk: the chunk's summed
    query (over its tokens and the group's q heads) against each key.
"""
from __future__ import annotations

import math

import numpy as np

__all__ = [
    "widen", "candidate_blocks", "attended_tokens",
    "rep_mean", "rep_topr_attention", "rep_landmark", "rep_embedding", "memorize",
    "score_dot", "score_cosine", "top_k",
    "softmax_attention", "split_partial", "merge_partials",
    "decode", "prefill_chunk", "prefill",
]


def widen(x: np.ndarray, dtype: str) -> np.ndarray:
    """Stored value -> fp64, exactly.  bf16 arrives as uint16 bit patterns."""
    if dtype == "bf16":
        return (np.asarray(x).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    if dtype == "f32":
        return np.asarray(x, dtype=np.float32).astype(np.float64)
    if dtype == "f64":
        return np.asarray(x, dtype=np.float64)
    raise ValueError(dtype)


# ---------------------------------------------------------------------------
# blocks, candidates, attended tokens


def candidate_blocks(T: int, bs: int, sink: int, window: int) -> np.ndarray:
    """Blocks eligible for retrieval.

    [ML] 2.2.1 cuts the past into non-overlapping fixed-size chunks; [IL] keeps
    the local window and the initial tokens outside the memory; [LM] uses
    fixed-length blocks.  Block j holds tokens [j*bs, (j+1)*bs); it is a
    candidate iff it is full ((j+1)*bs <= T) and its token range meets
    [sink, T - window).
    """
    w0 = max(T - window, 0)
    j = np.arange(T // bs)
    full = (j + 1) * bs <= T
    meets = ((j + 1) * bs > sink) & (j * bs < w0)
    return j[full & meets]


def attended_tokens(T: int, bs: int, sink: int, window: int, blocks) -> np.ndarray:
    """Sorted token positions one decode query attends to.

    [IL] overall framework: local tokens plus a few memory units; [ML] 2.3.4:
    the retrieved blocks' tokens; the sink is the first ``sink`` tokens.
    Taken as a set union, so a token is attended at most once.
    """
    w0 = max(T - window, 0)
    toks = set(range(0, min(sink, T)))
    toks |= set(range(w0, T))
    for j in blocks:
        toks |= set(range(int(j) * bs, (int(j) + 1) * bs))
    return np.array(sorted(toks), dtype=np.int64)


# ---------------------------------------------------------------------------
# representations (memorisation)


def rep_mean(Kb: np.ndarray) -> np.ndarray:
    """Mean key of a block: (1/bs) * sum_t k_t.  Returns [1][D]."""
    bs = Kb.shape[0]
    acc = np.zeros(Kb.shape[1])
    for t in range(bs):
        acc += Kb[t]
    return (acc / bs)[None, :]


def rep_topr_attention(Kb: np.ndarray, probe: np.ndarray, r: int, scale: float):
    """[IL] method: represent a memory unit by the tokens that received the
    highest attention scores.

    For each probe query p, the attention it pays to the block's tokens is
    softmax_t(scale * p . k_t) over the block; a token's received attention is
    the sum over probe queries.  The r tokens with the largest received
    attention are kept (ties -> lowest position), returned in ascending
    position with their keys.
    """
    bs = Kb.shape[0]
    received = np.zeros(bs)
    for p in probe:
        x = scale * (Kb @ p)
        e = np.exp(x - x.max())
        received += e / e.sum()
    order = sorted(range(bs), key=lambda t: (-received[t], t))
    chosen = np.array(sorted(order[:r]), dtype=np.int64)
    return chosen, Kb[chosen], received


def rep_landmark(L: np.ndarray) -> np.ndarray:
    """[LM] proposed method: the block's landmark key is its representation."""
    return np.asarray(L, dtype=np.float64).reshape(1, -1).copy()


def rep_embedding(e: np.ndarray) -> np.ndarray:
    """[ML] 2.2.2 / 2.3.2: a chunk's representation embedding, stored
    L2-normalised so the cosine in retrieval is a plain dot product."""
    e = np.asarray(e, dtype=np.float64)
    return e / math.sqrt(float(np.sum(e * e)))


def memorize(K: np.ndarray, mode: str, bs: int, r: int = 1, probe=None,
             landmarks=None, scale: float | None = None):
    """[ML] 2.3.2 memorisation M(k, v; r^m) for one (batch, kv head): the
    representation of every full block of K ([T][D]).

    Returns (reps [nb][r][D], chosen [nb][r] positions or None).
    Modes: "mean", "topr_attn" (probe [P][D]), "external" (landmarks [nb][D]),
    "identity" (bs == 1: the key is its own representation).
    """
    T, D = K.shape
    nb = T // bs
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    reps = np.zeros((nb, r, D))
    chosen = None
    if mode == "mean":
        for j in range(nb):
            reps[j] = rep_mean(K[j * bs:(j + 1) * bs])
    elif mode == "topr_attn":
        chosen = np.zeros((nb, r), dtype=np.int64)
        for j in range(nb):
            c, keys, _ = rep_topr_attention(K[j * bs:(j + 1) * bs], probe, r, scale)
            chosen[j] = c
            reps[j] = keys
    elif mode == "external":
        for j in range(nb):
            reps[j] = rep_landmark(landmarks[j])
    elif mode == "identity":
        if bs != 1 or r != 1:
            raise ValueError("identity representation needs block size 1, r = 1")
        reps[:, 0, :] = K[:nb]
    else:
        raise ValueError(mode)
    return reps, chosen


# ---------------------------------------------------------------------------
# scoring and selection


def score_dot(qs: np.ndarray, reps: np.ndarray, reduce: str = "sum") -> np.ndarray:
    """Block score by dot product, [LM] query-landmark similarity and [IL]
    relevance against representative tokens.

    qs [m][D] are the query vectors that share the selection (the q heads of a
    GQA group); reps [n][r][D].  reduce="sum": s_j = sum_q sum_i q . rep_{j,i};
    reduce="max" (variant): s_j = max_i sum_q q . rep_{j,i}, a block as relevant
    as its most relevant representative key.
    """
    pair = reps @ qs.T                    # [n][r][m]: one dot product per (key, query)
    per_key = pair.sum(axis=2)            # [n][r]: the group's queries summed
    if reduce == "sum":
        return per_key.sum(axis=1)
    if reduce == "max":
        return per_key.max(axis=1)
    raise ValueError(reduce)


def score_cosine(rq: np.ndarray, M: np.ndarray) -> np.ndarray:
    """[ML] 2.3.2 retrieval process: cosine similarity between the query
    chunk's embedding r^q and every embedding stored in the memory."""
    rq = np.asarray(rq, dtype=np.float64)
    nq = math.sqrt(float(rq @ rq))
    out = np.empty(M.shape[0])
    for j in range(M.shape[0]):
        m = M[j]
        out[j] = (rq @ m) / (nq * math.sqrt(float(m @ m)))
    return out


def top_k(s: np.ndarray, k: int) -> np.ndarray:
    """[ML] 2.3.2: z^q = TopK{Cos(r^q)}; [ML] 2.3.4: the k most relevant blocks.
    Order: larger score first, equal scores -> lower index first.  Returns the
    k chosen positions in ascending order."""
    s = np.asarray(s, dtype=np.float64)
    if not 0 <= k <= s.shape[0]:
        raise ValueError("k out of range")
    order = np.lexsort((np.arange(s.shape[0]), -s))
    return np.sort(order[:k])


# ---------------------------------------------------------------------------
# attention


def softmax_attention(q: np.ndarray, Kt: np.ndarray, Vt: np.ndarray, scale: float):
    """Exact softmax attention of one query over the rows Kt/Vt.

    x_t = scale * q . k_t;  p_t = exp(x_t - max x) / sum;  o = sum_t p_t v_t;
    lse = max x + ln sum exp(x - max x).  Returns (o, lse, p).
    """
    x = scale * (Kt @ q)
    m = x.max()
    e = np.exp(x - m)
    Z = e.sum()
    p = e / Z
    return p @ Vt, m + math.log(Z), p


def split_partial(q, Kt, Vt, scale):
    """Split-K partial over a subset of the attended tokens: (m, l, o~) with
    m = max logit, l = sum exp(x - m), o~ = sum exp(x - m) v / l."""
    x = scale * (Kt @ q)
    m = x.max()
    e = np.exp(x - m)
    l = e.sum()
    return m, l, (e @ Vt) / l


def merge_partials(parts):
    """Log-sum-exp merge of split partials (m_s, l_s, o~_s):
    m = max m_s; L = sum l_s e^(m_s - m); o = sum l_s e^(m_s - m) o~_s / L;
    lse = m + ln L."""
    m = max(p[0] for p in parts)
    L = sum(p[1] * math.exp(p[0] - m) for p in parts)
    o = sum(p[1] * math.exp(p[0] - m) * p[2] for p in parts) / L
    return o, m + math.log(L)


# ---------------------------------------------------------------------------
# whole decode step


def decode(q, K, V, reps, *, dtype, block_size, sink, window, top_k_blocks,
           scale=None, score_reduce="sum"):
    """One decode step for every (batch, q head).

    q [B][Hq][D], K, V [B][Hkv][T][D] as stored (``dtype``, widened here one
    head at a time); reps [B][Hkv][nb][r][D] fp64 from ``memorize``, or None
    when every key is its own block ([RA]: block size 1).
    Per (b, kv head h): score the candidate blocks with the group's q heads
    (q heads h*g .. h*g+g-1), keep the top k, attend each q head of the group
    over sink U selected blocks U window.

    Returns dict: cand (block ids), scores [B][Hkv][nc], idx [B][Hkv][k]
    (ascending block ids), out [B][Hq][D], lse [B][Hq].
    """
    B, Hq, D = q.shape
    Hkv, T = K.shape[1], K.shape[2]
    g = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    cand = candidate_blocks(T, block_size, sink, window)
    nc = cand.shape[0]
    scores = np.zeros((B, Hkv, nc))
    idx = np.zeros((B, Hkv, top_k_blocks), dtype=np.int64)
    out = np.zeros((B, Hq, D))
    lse = np.zeros((B, Hq))
    for b in range(B):
        for h in range(Hkv):
            qg = widen(q[b, h * g:(h + 1) * g], dtype)
            if reps is None:
                if block_size != 1:
                    raise ValueError("reps=None needs block size 1")
                R = widen(K[b, h, cand], dtype)[:, None, :]
            else:
                R = reps[b, h, cand]
            s = score_dot(qg, R, score_reduce) if nc else np.zeros(0)
            scores[b, h] = s
            sel = cand[top_k(s, top_k_blocks)]
            idx[b, h] = sel
            toks = attended_tokens(T, block_size, sink, window, sel)
            Kt = widen(K[b, h, toks], dtype)
            Vt = widen(V[b, h, toks], dtype)
            for i in range(g):
                o, l, _ = softmax_attention(qg[i], Kt, Vt, scale)
                out[b, h * g + i] = o
                lse[b, h * g + i] = l
    return {"cand": cand, "scores": scores, "idx": idx, "out": out, "lse": lse}


# ---------------------------------------------------------------------------
# chunked prefill


def prefill_chunk(Q, K_ret, V_ret, Kc, Vc, scale, rows=None):
    """[ML] 2.3.3 / Figure 3 retrieval-causal attention for one (chunk, q head).

    Q [Nq][D] query rows; K_ret/V_ret [n][D] retrieved (past) tokens, attended
    bidirectionally by every row; Kc/Vc [Nq][D] the chunk's own tokens, row i
    attends own token i' iff i' <= i.  One joint softmax per row.
    Returns (out [len(rows)][D], lse [len(rows)]).
    """
    Nq, D = Q.shape
    rows = range(Nq) if rows is None else rows
    outs, lses = [], []
    for i in rows:
        keys = np.concatenate([K_ret, Kc[:i + 1]], axis=0)
        vals = np.concatenate([V_ret, Vc[:i + 1]], axis=0)
        o, l, _ = softmax_attention(Q[i], keys, vals, scale)
        outs.append(o)
        lses.append(l)
    return np.array(outs), np.array(lses)


def prefill(Q, K, V, Kc, Vc, *, dtype, block_size, sink, window, top_k_blocks,
            score_mode, reps=None, query_embed=None, bank=None, scale=None,
            rows=None, heads=None):
    """Chunked prefill for every (chunk, q head).

    Q [Bq][Hq][Nq][D]; K, V [1][Hkv][T][D] the memory; Kc, Vc [Bq][Hkv][Nq][D];
    all as stored (``dtype``).
    Selection:
      cosine: [ML] 2.3.2 -- per query chunk, top-k blocks by
              cosine(query_embed[c], bank[j]), shared by all heads;
      dot:    per (chunk, kv head), the chunk's summed query (over its rows and
              the group's q heads) dotted with each candidate's rep keys
              (reps fp64, or None when every key is its own block).
    Attention per row: sink U selected blocks U window (all past tokens,
    bidirectional) plus the chunk's own tokens causally.
    Returns dict: idx [Bq][1 or Hkv][k], out [Bq][Hq][len(rows)][D], lse.
    """
    Bq, Hq, Nq, D = Q.shape
    Hkv, T = K.shape[1], K.shape[2]
    g = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    cand = candidate_blocks(T, block_size, sink, window)
    rows = list(range(Nq)) if rows is None else list(rows)
    heads = list(range(Hq)) if heads is None else list(heads)
    nsel = 1 if score_mode == "cosine" else Hkv
    out = np.zeros((Bq, Hq, len(rows), D))
    lse = np.zeros((Bq, Hq, len(rows)))
    idx = np.zeros((Bq, nsel, top_k_blocks), dtype=np.int64)
    scores = np.zeros((Bq, nsel, cand.shape[0]))
    for c in range(Bq):
        if score_mode == "cosine":
            bank64 = np.asarray(bank, dtype=np.float64)
            s = score_cosine(np.asarray(query_embed[c], dtype=np.float64), bank64[cand])
            scores[c, 0] = s
            idx[c, 0] = cand[top_k(s, top_k_blocks)]
        elif score_mode == "dot":
            for h in range(Hkv):
                qsum = widen(Q[c, h * g:(h + 1) * g], dtype).reshape(-1, D).sum(axis=0)
                if reps is None:
                    if block_size != 1:
                        raise ValueError("reps=None needs block size 1")
                    R = widen(K[0, h, cand], dtype)[:, None, :]
                else:
                    R = reps[0, h, cand]
                s = score_dot(qsum[None, :], R)
                scores[c, h] = s
                idx[c, h] = cand[top_k(s, top_k_blocks)]
        else:
            raise ValueError(score_mode)
        for hq in heads:
            h = hq // g
            sel = idx[c, 0 if score_mode == "cosine" else h]
            toks = attended_tokens(T, block_size, sink, window, sel)
            o, l = prefill_chunk(widen(Q[c, hq], dtype), widen(K[0, h, toks], dtype),
                                 widen(V[0, h, toks], dtype), widen(Kc[c, h], dtype),
                                 widen(Vc[c, h], dtype), scale, rows)
            out[c, hq] = o
            lse[c, hq] = l
    return {"cand": cand, "scores": scores, "idx": idx, "out": out, "lse": lse}
