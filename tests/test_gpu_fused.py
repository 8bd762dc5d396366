"""The whole decode step (rba_decode_step: one cooperative launch, or score,
top-k and the persistent attention kernel with the last two launched as
programmatic dependents) against the same three calls made one after the
other (rba_score -> rba_topk -> rba_attend) on the same store: identical
selections, outputs within the attention tolerance.  A cross-check of the
library's paths against each other; parity with the oracle is tested in
test_gpu_decode*.py.  Shapes cover one CTA per
SM, grids smaller than the SM count, several heads per CTA, GQA groups of 1, 2
and 4, ragged block sizes, and repeated calls on one workspace (its merge
tickets must come back to zero)."""
import numpy as np
import pytest
import torch

from retrieval_block_sparse_b200 import synth

from parity import OUT_TOL, dev, make_decode_store

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS
CASES = {
    "infllm-decode-128k": W["infllm-decode-128k"],
    "infllm-2k-window": W["infllm-decode-128k"].scaled(context=32768, window=2048, top_k=64),
    "landmark-decode-b16": W["landmark-decode-b16"],
    "tiny-decode-f32": W["tiny-decode-f32"],
    "gqa2-bs24-f32": W["tiny-decode-f32"].scaled(n_q_heads=8, n_kv_heads=4, context=1000,
                                                 block_size=24, sink=30, window=70, top_k=7),
    "one-head": W["infllm-decode-128k"].scaled(n_q_heads=4, n_kv_heads=1, context=16384,
                                               window=512, top_k=8),
    "batch4-d64": W["landmark-decode-b16"].scaled(batch=4, n_q_heads=8, n_kv_heads=8,
                                                  head_dim=64, context=3000, top_k=6),
}


@pytest.mark.parametrize("one_launch", [False, True])
@pytest.mark.parametrize("name", list(CASES))
def test_fused_step_equals_three_launches(rba, name, one_launch):
    w = CASES[name]
    x = synth.decode_inputs(w)
    st = make_decode_store(rba, w, x, one_launch)
    q = dev(x["q"], w.dtype)
    first, nc = st.candidates(w.context, w.sink, w.window)
    scores = st.score(q, w.context, w.sink, w.window)
    idx3 = rba.topk(scores.reshape(-1, nc), w.top_k, index_base=first).reshape(
        w.batch, w.n_kv_heads, w.top_k)
    out3, lse3 = st.attend(q, idx3, w.context, w.sink, w.window)
    plan = st.decode_plan(w.top_k, w.context, w.sink, w.window)
    # bf16 always takes a persistent kernel: the one-launch step (plan 3, when
    # asked for) or the whole-block tensor-core attention kernel (plan 2) when
    # blocks are whole 64-row tiles; fp32 with one q head per kv head has
    # tiles too large for shared memory and runs split-K (plan -2)
    whole = w.block_size % 64 == 0
    if w.dtype == "bf16":
        assert plan == ((3 if one_launch else 2) if whole else 1), plan
    else:
        assert plan in (1, -2), plan
    ws = st.decode_workspace(w.top_k, w.context, w.sink, w.window)
    vmax = float(st.v.float().abs().max())
    for rep in range(3):
        sc = torch.empty_like(scores)
        idx, out, lse = st.decode_step(q, w.top_k, w.context, w.sink, w.window, workspace=ws,
                                       scores=sc)
        st.check()
        assert torch.equal(idx, idx3), rep
        assert torch.allclose(sc, scores, rtol=1e-5, atol=1e-5)
        err = float((out - out3).abs().max()) / vmax
        assert err <= OUT_TOL[w.dtype], (rep, err)
        assert float((lse - lse3).abs().max()) <= OUT_TOL[w.dtype]


@pytest.mark.parametrize("n_distinct", [1, 2, 3, 40])
def test_fused_selection_with_tied_scores(rba, n_distinct):
    # Landmark keys drawn from n_distinct vectors: scores repeat exactly, so
    # the k-th largest value is shared by many candidates and the tie goes to
    # the lowest block ids.  With ~650 candidates, 3 values leave ~220 tied
    # candidates at the boundary (exact ranking inside the boundary value
    # bin), 2 values ~325 (more than the in-bin ranking takes: radix select),
    # 1 value a zero score range (radix select).
    w = W["landmark-decode-b16"].scaled(batch=2, n_q_heads=4, n_kv_heads=4, top_k=9)
    x = synth.decode_inputs(w)
    rng = np.random.default_rng(11)
    lm = x["landmarks"].copy()
    for b in range(w.batch):
        for h in range(w.n_kv_heads):
            lm[b, h] = x["landmarks"][b, h, rng.integers(0, n_distinct, w.n_blocks)]
    x = dict(x, landmarks=lm)
    st = make_decode_store(rba, w, x)
    q = dev(x["q"], w.dtype)
    first, nc = st.candidates(w.context, w.sink, w.window)
    scores = st.score(q, w.context, w.sink, w.window)
    idx3 = rba.topk(scores.reshape(-1, nc), w.top_k, index_base=first).reshape(
        w.batch, w.n_kv_heads, w.top_k)
    out3, _ = st.attend(q, idx3, w.context, w.sink, w.window)
    assert st.decode_plan(w.top_k, w.context, w.sink, w.window) in (1, 2)
    idx, out, _ = st.decode_step(q, w.top_k, w.context, w.sink, w.window)
    st.check()
    assert torch.equal(idx, idx3)
    # ties really go to the lowest ids: brute force on the GPU's own scores
    s = scores.reshape(w.batch * w.n_kv_heads, nc).cpu().numpy()
    for r in range(s.shape[0]):
        order = sorted(range(nc), key=lambda j: (-s[r, j], j))[:w.top_k]
        assert idx.reshape(-1, w.top_k)[r].tolist() == [first + j for j in sorted(order)]
    vmax = float(st.v.float().abs().max())
    assert float((out - out3).abs().max()) / vmax <= OUT_TOL[w.dtype]
