"""Plain statement of landmark-gated attention.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Source: "Landmark Attention: Random-Access Infinite Context Length for
Transformers" (review), "proposed method": the input is cut into fixed-length
blocks; each block is represented by a landmark token that acts as the gate
through which attention reaches the block; the attention score of the
landmark decides which blocks are retrieved and attended.

The page gives no formula for the gate.  The reading taken here is the
plainest one that the rest supports: the landmark takes the block's place in
the query's softmax.  For one query q with logits x_t = scale * q . k_t:
  * local tokens (sink U window) enter the softmax with their own logits;
  * retrieved block j enters it once, with the landmark's logit
    y_j = scale * q . L_j, and the mass it receives is spread over the block's
    tokens (those outside sink and window) by a softmax over the block alone;
  * out = (sum_local e^{x_t} v_t + sum_j e^{y_j} o_j) / Z,
    o_j = sum_{t in block j} softmax_block(x)_t v_t,
    Z = sum_local e^{x_t} + sum_j e^{y_j},  lse = ln Z.
When every y_j equals its block's log-sum-exp of x this is ordinary softmax
attention over sink U blocks U window (pinned in the tests).
"""
from __future__ import annotations

import math

import numpy as np

from .retrieval import attended_tokens

__all__ = ["gated_attention", "gated_decode"]


def gated_attention(q, K, V, L, blocks, T: int, bs: int, sink: int, window: int,
                    scale: float):
    """One query over the store rows K, V ([>= T][D], fp64) of one (batch, kv
    head), with landmark keys L ([nb][D]) and the retrieved block ids
    `blocks`.  Returns (out [D], lse)."""
    q = np.asarray(q, dtype=np.float64)
    local = attended_tokens(T, bs, sink, window, [])
    local_set = set(local.tolist())
    logits, values = [], []
    for t in local:                       # local tokens: their own logits
        logits.append(scale * float(K[t] @ q))
        values.append(V[t])
    for j in blocks:                      # a retrieved block: the landmark's logit
        toks = [t for t in range(int(j) * bs, (int(j) + 1) * bs) if t not in local_set]
        if not toks:
            continue
        x = np.array([scale * float(K[t] @ q) for t in toks])
        p = np.exp(x - x.max())
        p /= p.sum()
        logits.append(scale * float(L[int(j)] @ q))
        values.append(p @ V[toks])
    if not logits:
        return np.zeros(K.shape[1]), -math.inf
    y = np.array(logits)
    m = y.max()
    w = np.exp(y - m)
    Z = w.sum()
    return (w @ np.array(values)) / Z, m + math.log(Z)


def gated_decode(q, K, V, L, idx, *, dtype, block_size, sink, window, scale=None):
    """Every (batch, q head) of a decode step: q [B][Hq][D], K, V
    [B][Hkv][T][D] and L [B][Hkv][nb][D] as stored (``dtype``), idx
    [B][Hkv][k] the retrieved blocks.  Returns (out [B][Hq][D], lse [B][Hq])."""
    from .retrieval import widen
    B, Hq, D = q.shape
    Hkv, T = K.shape[1], K.shape[2]
    g = Hq // Hkv
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    out = np.zeros((B, Hq, D))
    lse = np.zeros((B, Hq))
    for b in range(B):
        for h in range(Hkv):
            Kb, Vb = widen(K[b, h], dtype), widen(V[b, h], dtype)
            Lb = widen(L[b, h], dtype)
            for i in range(h * g, (h + 1) * g):
                out[b, i], lse[b, i] = gated_attention(widen(q[b, i], dtype), Kb, Vb, Lb,
                                                       idx[b, h], T, block_size, sink, window,
                                                       scale)
    return out, lse
