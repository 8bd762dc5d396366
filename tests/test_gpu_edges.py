"""Edge geometry of the decode path on the GPU: no retrieval (k = 0), every
candidate retrieved (= dense attention), window covering everything, sink
swallowing the candidates, copy-in memorisation, malformed selections, host
argument errors."""
import numpy as np
import pytest
import torch

import oracle as O
from retrieval_block_sparse_b200 import synth

from parity import OUT_TOL, dev, make_decode_store, oracle_reps, out_error

pytestmark = pytest.mark.gpu
BASE = synth.WORKLOADS["infllm-decode-128k"].scaled(context=4096, window=512, top_k=8,
                                                    n_planted=4, seed=21)


def _run_case(rba, w, k):
    x = synth.decode_inputs(w)
    reps, _ = oracle_reps(w, x)
    st = make_decode_store(rba, w, x)
    ref = O.decode(x["q"], x["K"], x["V"], reps, dtype=w.dtype, block_size=w.block_size,
                   sink=w.sink, window=w.window, top_k_blocks=k)
    idx, out, lse = st.decode_step(dev(x["q"], w.dtype), k, w.context, w.sink, w.window)
    st.check()
    out = out.cpu().numpy()
    np.testing.assert_array_equal(idx.cpu().numpy(), ref["idx"])
    vmax = np.abs(O.widen(x["V"], w.dtype)).max()
    assert float(np.abs(out - ref["out"]).max()) / vmax <= OUT_TOL[w.dtype]
    return x, ref, out


def test_no_retrieval_sink_and_window_only(rba):
    _run_case(rba, BASE.scaled(top_k=0), 0)


def test_all_candidates_is_dense_attention(rba):
    w = BASE.scaled(sink=128, window=512)
    nc = O.candidate_blocks(w.context, w.block_size, w.sink, w.window).shape[0]
    x, ref, out = _run_case(rba, w, nc)
    # invariant (a): equals softmax attention over all T tokens
    g = w.n_q_heads // w.n_kv_heads
    q = O.widen(x["q"], w.dtype)
    for i in range(0, w.n_q_heads, 5):
        K = O.widen(x["K"][0, i // g], w.dtype)
        V = O.widen(x["V"][0, i // g], w.dtype)
        o, _, _ = O.softmax_attention(q[0, i], K, V, w.head_dim ** -0.5)
        assert out_error(out[0, i], o, V) <= OUT_TOL["bf16"]


def test_window_covers_context(rba):
    _run_case(rba, BASE.scaled(window=5000, sink=0, top_k=0), 0)


def test_sink_swallows_candidates(rba):
    _run_case(rba, BASE.scaled(sink=3700, window=512, top_k=0), 0)


def test_memorize_copy_in(rba):
    w = synth.WORKLOADS["tiny-decode-f32"].scaled(context=1024)
    x = synth.decode_inputs(w)
    st = rba.Store(batch=1, n_q_heads=4, n_kv_heads=4, head_dim=64, block_size=64,
                   capacity_tokens=2048, dtype="f32", mode="mean")
    K, V = dev(x["K"], "f32"), dev(x["V"], "f32")
    st.memorize(K[:, :, :512].contiguous(), V[:, :, :512].contiguous(), first_block=0)
    st.memorize(K[:, :, 512:].contiguous(), V[:, :, 512:].contiguous(), first_block=8)
    st.check()
    assert torch.equal(st.k[:, :, :1024], K) and torch.equal(st.v[:, :, :1024], V)
    reps, _ = oracle_reps(w, x)
    np.testing.assert_allclose(st.rep[:, :, :16].cpu().numpy(), reps, atol=1e-6)


def test_malformed_selection_is_reported_not_faulted(rba):
    w = BASE
    x = synth.decode_inputs(w)
    st = make_decode_store(rba, w, x)
    idx = torch.tensor([[[1, 2, 3, 4, 5, 6, 7, 10_000]] * w.n_kv_heads], dtype=torch.int32).cuda()
    st.attend(dev(x["q"], w.dtype), idx, w.context, w.sink, w.window)
    with pytest.raises(rba.RbaError) as e:
        st.check()
    assert e.value.status == rba.ERR_BOUNDS
    st.check()  # cleared


def test_host_errors(rba):
    w = BASE
    x = synth.decode_inputs(w)
    st = make_decode_store(rba, w, x)
    q = dev(x["q"], w.dtype)
    with pytest.raises(rba.RbaError):
        st.decode_step(q, 10_000, w.context, w.sink, w.window)      # k > candidates
    with pytest.raises(rba.RbaError):
        st.decode_step(q, 4, w.context + 10, w.sink, 0)             # beyond capacity
    tiny = torch.zeros(8, dtype=torch.uint8, device="cuda")
    with pytest.raises(rba.RbaError) as e:
        st.decode_step(q, 4, w.context, w.sink, w.window, workspace=tiny)
    assert e.value.status == rba.ERR_WORKSPACE
