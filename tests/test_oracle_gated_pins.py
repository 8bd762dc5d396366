"""Pins of the oracle's landmark-gated attention (Landmark Attention review,
"proposed method": a block's landmark token is the gate through which
attention reaches the block), against things other than itself: torch's fp64
attention in the cases where the gate reduces to ordinary softmax attention,
closed forms of the gate's weights, and scipy's logsumexp.

A plausible slip (gating by the block's own keys instead of the landmark,
normalising each block against the whole row, counting a token that is both
local and in a block twice, a dropped local term) fails at least one of them."""
import math

import numpy as np
import scipy.special
import torch

import oracle as O


def _rng(s):
    return np.random.default_rng(s)


def _sdpa(q, K, V, scale):
    o = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None, None, None], torch.from_numpy(K)[None, None],
        torch.from_numpy(V)[None, None], scale=scale)
    return o[0, 0, 0].numpy()


def _case(seed, T=96, bs=8, D=16):
    r = _rng(seed)
    return (r.normal(size=D), r.normal(size=(T, D)), r.normal(size=(T, D)),
            r.normal(size=(T // bs, D)))


def test_landmarks_at_block_logsumexp_give_plain_attention():
    # y_j = ln sum_{t in block j} e^{x_t}: each block then receives exactly the
    # mass plain softmax gives its tokens
    q, K, V, L = _case(1)
    T, bs, S, W, scale = 96, 8, 5, 13, 0.3
    blocks = [2, 5, 9]
    w0 = T - W
    for j in blocks:
        toks = [t for t in range(j * bs, (j + 1) * bs) if S <= t < w0]
        lse_j = scipy.special.logsumexp(scale * K[toks] @ q)
        L[j] = lse_j / (scale * (q @ q)) * q
    out, lse = O.gated_attention(q, K, V, L, blocks, T, bs, S, W, scale)
    toks = O.attended_tokens(T, bs, S, W, blocks)
    np.testing.assert_allclose(out, _sdpa(q, K[toks], V[toks], scale), atol=1e-12)
    assert abs(lse - scipy.special.logsumexp(scale * K[toks] @ q)) < 1e-12


def test_no_block_is_attention_over_sink_and_window():
    q, K, V, L = _case(2)
    T, bs, S, W, scale = 96, 8, 7, 20, 0.25
    out, lse = O.gated_attention(q, K, V, L, [], T, bs, S, W, scale)
    toks = O.attended_tokens(T, bs, S, W, [])
    np.testing.assert_allclose(out, _sdpa(q, K[toks], V[toks], scale), atol=1e-12)
    assert abs(lse - scipy.special.logsumexp(scale * K[toks] @ q)) < 1e-12


def test_one_block_alone_is_attention_inside_the_block():
    # no sink, no window: the only softmax term is the block, whose mass is
    # all of it: the gate's logit drops out
    q, K, V, L = _case(3)
    T, bs, scale = 96, 8, 0.4
    out, lse = O.gated_attention(q, K, V, L, [4], T, bs, 0, 0, scale)
    toks = np.arange(4 * bs, 5 * bs)
    np.testing.assert_allclose(out, _sdpa(q, K[toks], V[toks], scale), atol=1e-12)
    assert abs(lse - scale * L[4] @ q) < 1e-12


def test_gate_weights_are_the_landmark_softmax():
    # blocks whose values are one-hot per block: the output is the softmax of
    # the landmark logits (and of the local logits) over those directions,
    # whatever the blocks' own keys
    T, bs, D = 64, 8, 6
    q, K, V, L = _case(4, T=T, bs=bs, D=D)
    S, W, scale = 0, 8, 0.5
    V[:] = 0
    V[1 * bs:2 * bs, 0] = 1.0
    V[3 * bs:4 * bs, 1] = 1.0
    V[T - W:, 2] = 1.0
    out, lse = O.gated_attention(q, K, V, L, [1, 3], T, bs, S, W, scale)
    y = np.array([scale * L[1] @ q, scale * L[3] @ q])
    xl = scale * K[T - W:] @ q
    Z = np.exp(y).sum() + np.exp(xl).sum()
    np.testing.assert_allclose(out[:3], [math.exp(y[0]) / Z, math.exp(y[1]) / Z,
                                         np.exp(xl).sum() / Z], atol=1e-12)
    np.testing.assert_allclose(out[3:], 0, atol=0)
    assert abs(lse - math.log(Z)) < 1e-12


def test_block_tokens_inside_the_window_count_once_as_local():
    # block 10 of 12 straddles the window start: its tokens in the window are
    # local tokens; the gate covers only its tokens before the window
    q, K, V, L = _case(5)
    T, bs, S, W, scale = 96, 8, 0, 12, 0.3
    out, lse = O.gated_attention(q, K, V, L, [10], T, bs, S, W, scale)
    w0 = T - W                                 # 84: block 10 is tokens 80..87
    inner = np.arange(80, w0)
    x_in = scale * K[inner] @ q
    p = np.exp(x_in - x_in.max())
    p /= p.sum()
    local = np.arange(w0, T)
    y = np.concatenate([scale * K[local] @ q, [scale * L[10] @ q]])
    vals = np.concatenate([V[local], (p @ V[inner])[None]])
    w = np.exp(y - y.max())
    np.testing.assert_allclose(out, (w @ vals) / w.sum(), atol=1e-12)
    assert abs(lse - scipy.special.logsumexp(y)) < 1e-12


def test_gated_decode_groups_q_heads_by_kv_head():
    # every q head of a group uses its kv head's rows, landmarks and blocks
    r = _rng(6)
    B, Hq, Hkv, T, bs, D = 2, 4, 2, 48, 8, 8
    q = r.normal(size=(B, Hq, D)).astype(np.float32)
    K = r.normal(size=(B, Hkv, T, D)).astype(np.float32)
    V = r.normal(size=(B, Hkv, T, D)).astype(np.float32)
    L = r.normal(size=(B, Hkv, T // bs, D)).astype(np.float32)
    idx = np.array([[[1, 3], [2, 4]], [[0, 1], [3, 4]]])
    out, lse = O.gated_decode(q, K, V, L, idx, dtype="f32", block_size=bs, sink=4, window=8,
                              scale=D ** -0.5)
    for b in range(B):
        for i in range(Hq):
            h = i // 2
            o, l = O.gated_attention(q[b, i].astype(np.float64), K[b, h].astype(np.float64),
                                     V[b, h].astype(np.float64), L[b, h].astype(np.float64),
                                     idx[b, h], T, bs, 4, 8, D ** -0.5)
            np.testing.assert_array_equal(out[b, i], o)
            assert lse[b, i] == l
