"""GPU parity of chunked prefill (selection + retrieval-causal tensor-core
attention) against the fp64 oracle, through the C ABI.

Selections are computed on the GPU (rba_score + rba_topk) and checked against
the oracle's; the attention is then run on the oracle's selection so that
outputs are compared on identical token sets.  Full-size workloads compare a
seeded sample of query rows (24 random rows plus the first and last row of
every 128-row tile) and heads (the oracle walks rows one by one)."""
import numpy as np
import pytest
import torch

import oracle as O
from retrieval_block_sparse_b200 import synth

from parity import OUT_TOL, dev, selection_check

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS
CASES = {
    # MemLong-style cosine retrieval: whole 256-token chunks, direct tiles
    "cosine-small": W["memlong-cosine-prefill"].scaled(n_chunks=3, n_q_heads=4, n_kv_heads=4,
                                                       chunk_len=256, context=12 * 256,
                                                       block_size=256, top_k=3),
    # token-level retrieval (block size 1): gathered past tokens, GQA 4
    "token-small": W["token-retrieval-prefill-1m"].scaled(n_q_heads=8, n_kv_heads=2,
                                                          chunk_len=256, context=16384,
                                                          top_k=384),
    # ragged: chunk not a multiple of 128, sink/window partial tiles, mean reps
    "ragged": W["token-retrieval-prefill-1m"].scaled(n_q_heads=4, n_kv_heads=2, chunk_len=200,
                                                     context=40 * 160, block_size=160,
                                                     sink=64, window=100, top_k=5,
                                                     recipe="shifted"),
    "no-retrieval": W["token-retrieval-prefill-1m"].scaled(n_q_heads=2, n_kv_heads=1,
                                                           chunk_len=384, context=4096,
                                                           block_size=128, top_k=0),
    "memlong-cosine-prefill": W["memlong-cosine-prefill"],
    "token-retrieval-prefill-1m": W["token-retrieval-prefill-1m"],
}
FULL = {"memlong-cosine-prefill", "token-retrieval-prefill-1m"}


def _mode(w):
    if w.score_mode == "cosine":
        return "embed_cosine"
    return "identity" if w.block_size == 1 else "mean"


def _run(rba, name):
    w = CASES[name]
    x = synth.prefill_inputs(w)
    mode = _mode(w)
    st = rba.Store(batch=1, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, head_dim=w.head_dim,
                   block_size=w.block_size, capacity_tokens=w.context, dtype="bf16", mode=mode,
                   d_ret=w.d_ret)
    st.k.copy_(dev(x["K"], "bf16"))
    st.v.copy_(dev(x["V"], "bf16"))
    nb = w.context // w.block_size
    reps = None
    if mode == "embed_cosine":
        st.memorize(None, None, first_block=0, n_blocks=nb,
                    aux=torch.from_numpy(x["bank_embed"]).cuda().reshape(1, nb, w.d_ret))
    elif mode == "mean":
        st.memorize(None, None, first_block=0, n_blocks=nb)
        reps = np.stack([O.memorize(O.widen(x["K"][0, h], "bf16"), "mean", w.block_size)[0]
                         for h in range(w.n_kv_heads)])[None]
    Q = dev(x["Q"], "bf16")
    Kc, Vc = dev(x["chunk_K"], "bf16"), dev(x["chunk_V"], "bf16")
    rng = np.random.default_rng(7)
    rows = heads = None
    if name in FULL:
        # 24 random rows plus the first and last row of every 128-row query
        # tile (the tile edges and the causal diagonal's ends)
        edges = {r for t in range(0, w.chunk_len, 128) for r in (t, t + 127) if r < w.chunk_len}
        rows = sorted(set(rng.choice(w.chunk_len, 24, replace=False).tolist()) | edges)
        heads = sorted(rng.choice(w.n_q_heads, 3, replace=False).tolist())
    ref = O.prefill(x["Q"], x["K"], x["V"], x["chunk_K"], x["chunk_V"], dtype="bf16",
                    block_size=w.block_size, sink=w.sink, window=w.window,
                    top_k_blocks=w.top_k, score_mode=w.score_mode, reps=reps,
                    query_embed=x.get("query_embed"), bank=x.get("bank_embed"), rows=rows,
                    heads=heads)
    # GPU selection
    first, nc = st.candidates(w.context, w.sink, w.window)
    if w.top_k > 0:
        if w.score_mode == "cosine":
            sc = st.score(torch.from_numpy(x["query_embed"]).cuda(), w.context, w.sink, w.window)
        else:
            sc = st.score(Q, w.context, w.sink, w.window)
        gidx = rba.topk(sc.reshape(-1, nc), w.top_k, index_base=first).cpu().numpy()
        gidx = gidx.reshape(ref["idx"].shape)
        for c in range(ref["idx"].shape[0]):
            for s in range(ref["idx"].shape[1]):
                selection_check(ref["scores"][c, s], w.top_k, first, gidx[c, s])
    # attention on the oracle's selection
    idx = torch.from_numpy(ref["idx"].astype(np.int32)).cuda()
    out, lse = st.attend_prefill(Q, idx, Kc, Vc, w.context, w.sink, w.window)
    st.check()
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    rows = list(range(w.chunk_len)) if rows is None else rows
    heads = list(range(w.n_q_heads)) if heads is None else heads
    g = w.n_q_heads // w.n_kv_heads
    worst = 0.0
    for c in range(w.n_chunks):
        for hi, hq in enumerate(heads):
            h = hq // g
            sel = ref["idx"][c, 0 if w.score_mode == "cosine" else h]
            toks = O.attended_tokens(w.context, w.block_size, w.sink, w.window, sel)
            vmax = max(float(np.abs(O.widen(x["V"][0, h, toks], "bf16")).max()) if toks.size else 0,
                       float(np.abs(O.widen(x["chunk_V"][c, h], "bf16")).max()))
            err = np.abs(out[c, hq, rows] - ref["out"][c, hq]).max() / vmax
            worst = max(worst, float(err))
            np.testing.assert_allclose(lse[c, hq, rows], ref["lse"][c, hq], rtol=0, atol=2e-3)
    assert worst <= OUT_TOL["bf16"], worst
    return worst


@pytest.mark.parametrize("name", list(CASES))
def test_prefill(rba, name):
    _run(rba, name)


def test_prefill_all_blocks_is_causal_attention(rba):
    # every past block retrieved: the chunk's rows see [past ; own chunk]
    # causally -- torch's fp64 attention with the causal mask on CPU
    w = CASES["cosine-small"].scaled(n_chunks=1, context=4 * 256, top_k=4)
    x = synth.prefill_inputs(w)
    st = rba.Store(batch=1, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, head_dim=w.head_dim,
                   block_size=w.block_size, capacity_tokens=w.context, dtype="bf16",
                   mode="embed_cosine", d_ret=w.d_ret)
    st.k.copy_(dev(x["K"], "bf16"))
    st.v.copy_(dev(x["V"], "bf16"))
    idx = torch.arange(4, dtype=torch.int32, device="cuda").reshape(1, 1, 4)
    out, _ = st.attend_prefill(dev(x["Q"], "bf16"), idx, dev(x["chunk_K"], "bf16"),
                               dev(x["chunk_V"], "bf16"), w.context, 0, 0)
    st.check()
    out = out.cpu().numpy()
    T, N = w.context, w.chunk_len
    for hq in range(w.n_q_heads):
        Kall = np.concatenate([O.widen(x["K"][0, hq], "bf16"), O.widen(x["chunk_K"][0, hq], "bf16")])
        Vall = np.concatenate([O.widen(x["V"][0, hq], "bf16"), O.widen(x["chunk_V"][0, hq], "bf16")])
        mask = np.arange(T + N)[None, :] <= (T + np.arange(N))[:, None]
        qv = torch.from_numpy(O.widen(x["Q"][0, hq], "bf16"))[None, None]
        ref = torch.nn.functional.scaled_dot_product_attention(
            qv, torch.from_numpy(Kall)[None, None], torch.from_numpy(Vall)[None, None],
            attn_mask=torch.from_numpy(mask)[None, None], scale=w.head_dim ** -0.5)[0, 0].numpy()
        assert np.abs(out[0, hq] - ref).max() / np.abs(Vall).max() <= OUT_TOL["bf16"]
