"""GPU parity of landmark-gated attention (rba_attend_landmark_gated; Landmark
Attention review, "proposed method": the landmark is the gate through which
attention reaches its block) against the oracle's gated_decode, through the
C ABI, on the oracle's own block selection.

Cases: the Landmark decode workload at full size (16 x 32 heads, 50-token
blocks, a 256-token window), GQA with a sink and fp32, head dim 100 (padded
pool rows), and the reduction to ordinary attention: with every landmark's
logit set to its block's log-sum-exp the gated output equals rba_attend's."""
import numpy as np
import pytest
import torch
import scipy.special

import oracle as O
from retrieval_block_sparse_b200 import synth

from parity import OUT_TOL, dev, make_decode_store, oracle_reps, out_error

pytestmark = pytest.mark.gpu
BASE = synth.WORKLOADS["landmark-decode-b16"]
CASES = {
    "landmark-decode-b16": BASE,
    "gqa-sink-f32": BASE.scaled(dtype="f32", batch=2, n_q_heads=8, n_kv_heads=4, context=3000,
                                top_k=6, sink=40, window=120, seed=91),
    "d100": BASE.scaled(batch=2, n_q_heads=4, n_kv_heads=4, head_dim=100, context=2018,
                        top_k=5, sink=20, window=100, seed=92),
}


@pytest.mark.parametrize("name", list(CASES))
def test_gated_matches_oracle(rba, name):
    w = CASES[name]
    x = synth.decode_inputs(w)
    reps, _ = oracle_reps(w, x)
    st = make_decode_store(rba, w, x)
    ref = O.decode(x["q"], x["K"], x["V"], reps, dtype=w.dtype, block_size=w.block_size,
                   sink=w.sink, window=w.window, top_k_blocks=w.top_k)
    idx = torch.from_numpy(ref["idx"].astype(np.int32)).cuda()
    out, lse = st.attend_gated(dev(x["q"], w.dtype), idx, w.context, w.sink, w.window)
    st.check()
    o_ref, l_ref = O.gated_decode(x["q"], x["K"], x["V"], x["landmarks"], ref["idx"],
                                  dtype=w.dtype, block_size=w.block_size, sink=w.sink,
                                  window=w.window)
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    g = w.n_q_heads // w.n_kv_heads
    worst = 0.0
    for b in range(w.batch):
        for h in range(w.n_kv_heads):
            va = O.widen(x["V"][b, h, O.attended_tokens(w.context, w.block_size, w.sink,
                                                          w.window, ref["idx"][b, h])], w.dtype)
            for i in range(h * g, (h + 1) * g):
                worst = max(worst, out_error(out[b, i], o_ref[b, i], va))
    assert worst <= OUT_TOL[w.dtype], worst
    np.testing.assert_allclose(lse, l_ref, rtol=0, atol=OUT_TOL[w.dtype])
    # the gate changes the result: plain attention differs on these inputs
    assert np.abs(out - ref["out"]).max() > 10 * OUT_TOL[w.dtype]


def test_landmarks_at_block_logsumexp_reduce_to_attention(rba):
    # one q head per kv head: set each retrieved block's landmark key so that
    # its logit is the block's log-sum-exp; the gated output is then plain
    # attention over sink U blocks U window (rba_attend)
    w = BASE.scaled(batch=2, n_q_heads=4, n_kv_heads=4, context=2018, top_k=5, sink=20,
                    window=100, seed=93)
    x = synth.decode_inputs(w)
    reps, _ = oracle_reps(w, x)
    ref = O.decode(x["q"], x["K"], x["V"], reps, dtype=w.dtype, block_size=w.block_size,
                   sink=w.sink, window=w.window, top_k_blocks=w.top_k)
    scale = w.head_dim ** -0.5
    lm = O.widen(x["landmarks"], w.dtype)
    w0 = w.context - w.window
    for b in range(w.batch):
        for h in range(w.n_kv_heads):
            q = O.widen(x["q"][b, h], w.dtype)
            K = O.widen(x["K"][b, h], w.dtype)
            for j in ref["idx"][b, h]:
                toks = [t for t in range(j * w.block_size, (j + 1) * w.block_size)
                        if w.sink <= t < w0]
                lse_j = scipy.special.logsumexp(scale * K[toks] @ q)
                lm[b, h, j] = lse_j / (scale * (q @ q)) * q
    st = make_decode_store(rba, w, dict(x, landmarks=synth.bf16_round(lm.astype(np.float32))))
    # (bf16 rounding of the constructed landmark moves y_j by ~1e-2: compare on
    # the rounded landmarks through the oracle, and plain attention loosely)
    idx = torch.from_numpy(ref["idx"].astype(np.int32)).cuda()
    q = dev(x["q"], w.dtype)
    o_g, _ = st.attend_gated(q, idx, w.context, w.sink, w.window)
    o_a, _ = st.attend(q, idx, w.context, w.sink, w.window)
    st.check()
    vmax = float(np.abs(O.widen(x["V"], w.dtype)).max())
    assert float((o_g - o_a).abs().max()) / vmax <= 0.05
    o_ref, _ = O.gated_decode(x["q"], x["K"], x["V"], synth.bf16_round(lm.astype(np.float32)),
                              ref["idx"], dtype=w.dtype, block_size=w.block_size, sink=w.sink,
                              window=w.window)
    assert np.abs(o_g.cpu().numpy() - o_ref).max() / vmax <= OUT_TOL[w.dtype]


def test_gated_rejects_other_stores(rba):
    w = synth.WORKLOADS["infllm-decode-128k"].scaled(context=4096, window=512, top_k=4,
                                                     n_planted=2)
    st = rba.Store(batch=1, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, head_dim=128,
                   block_size=128, capacity_tokens=4096, dtype="bf16", mode="mean")
    q = torch.zeros((1, w.n_q_heads, 128), dtype=torch.bfloat16, device="cuda")
    idx = torch.ones((1, w.n_kv_heads, 4), dtype=torch.int32, device="cuda")
    with pytest.raises(rba.RbaError):
        st.attend_gated(q, idx, 4096, w.sink, w.window)
