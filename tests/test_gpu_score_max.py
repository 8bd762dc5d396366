"""GPU parity of the max-over-representative-keys block score variant
(rba_store_set_score_reduce(RBA_SCORE_MAX)): the score kernel, and the whole
decode step that ranks blocks by it, against the oracle's
score_dot(..., "max") and decode(..., score_reduce="max").

The cases cover the kernel's two lane layouts of a key: keys spanning part of
a lane group (bf16: 16 or 8 lanes per key) and keys spanning whole vector
slots (fp32, D = 128), with 2, 4 and 8 keys per block."""
import numpy as np
import pytest

import oracle as O
from retrieval_block_sparse_b200 import synth

from parity import check_decode_step, dev, oracle_reps, score_tolerance

pytestmark = pytest.mark.gpu
BASE = synth.WORKLOADS["infllm-decode-128k"]
CASES = {
    "bf16-d128-r4": BASE.scaled(context=16384, window=1024, top_k=16, n_planted=8, seed=51),
    "bf16-d64-r8": BASE.scaled(n_q_heads=8, n_kv_heads=4, head_dim=64, context=8192,
                               block_size=64, n_rep=8, window=512, top_k=12, n_planted=4,
                               seed=52),
    "f32-d128-r2": BASE.scaled(dtype="f32", n_q_heads=8, n_kv_heads=4, context=8192,
                               n_rep=2, window=512, top_k=8, n_planted=4, seed=53),
    "f32-d64-r2": BASE.scaled(dtype="f32", n_q_heads=4, n_kv_heads=4, head_dim=64,
                              context=4096, block_size=64, n_rep=2, window=256, top_k=6,
                              n_planted=2, seed=54),
}


def _store(rba, w, x):
    st = rba.Store(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                   head_dim=w.head_dim, block_size=w.block_size, capacity_tokens=w.context,
                   dtype=w.dtype, mode=w.rep_mode, n_rep=w.n_rep, score_reduce="max")
    st.k.copy_(dev(x["K"], w.dtype))
    st.v.copy_(dev(x["V"], w.dtype))
    st.memorize(None, None, first_block=0, n_blocks=w.n_blocks, aux=dev(x["probe"], w.dtype))
    return st


@pytest.mark.parametrize("one_launch", [False, True])
@pytest.mark.parametrize("name", list(CASES))
def test_max_scores_and_decode_step(rba, name, one_launch):
    w = CASES[name]
    x = synth.decode_inputs(w)
    reps, _ = oracle_reps(w, x)
    ref = O.decode(x["q"], x["K"], x["V"], reps, dtype=w.dtype, block_size=w.block_size,
                   sink=w.sink, window=w.window, top_k_blocks=w.top_k, score_reduce="max")
    st = _store(rba, w, x)
    if one_launch:
        st.set_decode_step_one_launch(True)
    q = dev(x["q"], w.dtype)
    s = st.score(q, w.context, w.sink, w.window).cpu().numpy().astype(np.float64)
    st.check()
    g = w.n_q_heads // w.n_kv_heads
    cand = ref["cand"]
    for b in range(w.batch):
        for h in range(w.n_kv_heads):
            qa = np.abs(O.widen(x["q"][b, h * g:(h + 1) * g], w.dtype)).sum(axis=0)
            tol = score_tolerance(qa, np.abs(reps[b, h, cand]))
            err = np.abs(s[b, h] - ref["scores"][b, h])
            assert np.all(err <= tol), (b, h, float(err.max()))
    # the variant ranks differently from the sum on these inputs
    ref_sum = O.decode(x["q"], x["K"], x["V"], reps, dtype=w.dtype, block_size=w.block_size,
                       sink=w.sink, window=w.window, top_k_blocks=w.top_k)
    assert not np.array_equal(ref_sum["idx"], ref["idx"])
    idx, out, lse = st.decode_step(q, w.top_k, w.context, w.sink, w.window)
    st.check()
    check_decode_step(w, x["q"], x["K"], x["V"], ref, idx.cpu().numpy(), out.cpu().numpy(),
                      lse.cpu().numpy())
