"""GPU parity of the whole-block tensor-core decode kernel (bf16 stores whose
block size is a multiple of 64 rows) against the fp64 oracle.

The cases cover what that kernel has to get right: one, two and four q heads
per kv head (the padded rows of the A tile), head dims 64 and 128 (one or two
64-column halves of the swizzled tiles), blocks of one, two and three tiles,
blocks clipped by a sink or window that is not block-aligned (pieces that
start mid-block and partial tiles), a tail block inside the window, more kv
heads than SMs (each CTA holds whole heads) and fewer (heads cut into parts).
"""
import numpy as np
import pytest
import torch

import oracle as O
from retrieval_block_sparse_b200 import synth

from parity import (OUT_TOL, attended_v_max, check_decode_step, dev, make_decode_store,
                    oracle_reps, out_error)

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS
BASE = W["infllm-decode-128k"]
CASES = {
    "g1-d64-bs64": BASE.scaled(batch=2, n_q_heads=8, n_kv_heads=8, head_dim=64,
                               context=8192 + 37, block_size=64, n_rep=1, rep_mode="mean",
                               top_k=12, sink=100, window=300, n_planted=4, seed=21),
    "g2-bs192-topr": BASE.scaled(n_q_heads=16, n_kv_heads=8, context=20000, block_size=192,
                                 n_rep=2, top_k=10, sink=64, window=1000, n_planted=4, seed=22),
    "many-heads-g2": BASE.scaled(batch=8, n_q_heads=64, n_kv_heads=32, context=4096,
                                 block_size=64, n_rep=1, rep_mode="mean", top_k=8, sink=64,
                                 window=256, n_planted=2, seed=23),
    "g4-d64-bs128": BASE.scaled(n_q_heads=16, n_kv_heads=4, head_dim=64, context=30000,
                                block_size=128, n_rep=1, rep_mode="mean", top_k=24, sink=0,
                                window=2000, n_planted=8, seed=24),
}

_cache = {}


def _prepared(name):
    if name not in _cache:
        w = CASES[name]
        x = synth.decode_inputs(w)
        reps, _ = oracle_reps(w, x)
        ref = O.decode(x["q"], x["K"], x["V"], reps, dtype=w.dtype, block_size=w.block_size,
                       sink=w.sink, window=w.window, top_k_blocks=w.top_k)
        _cache.clear()
        _cache[name] = (w, x, ref)
    return _cache[name]


@pytest.mark.parametrize("name", list(CASES))
def test_attend_on_oracle_selection(rba, name):
    w, x, ref = _prepared(name)
    st = make_decode_store(rba, w, x)
    # rba_attend runs the whole-block kernel, as the default decode step does
    assert st.decode_plan(w.top_k, w.context, w.sink, w.window) == 2
    idx = torch.from_numpy(ref["idx"].astype(np.int32)).cuda()
    out, lse = st.attend(dev(x["q"], w.dtype), idx, w.context, w.sink, w.window)
    st.check()
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    g = w.n_q_heads // w.n_kv_heads
    worst = 0.0
    for b in range(w.batch):
        for h in range(w.n_kv_heads):
            va = attended_v_max(w, x, b, h, ref["idx"][b, h])
            for i in range(h * g, (h + 1) * g):
                worst = max(worst, out_error(out[b, i], ref["out"][b, i], va))
    assert worst <= OUT_TOL[w.dtype], worst
    np.testing.assert_allclose(lse, ref["lse"], rtol=0, atol=OUT_TOL[w.dtype])


@pytest.mark.parametrize("one_launch", [False, True])
@pytest.mark.parametrize("name", list(CASES))
def test_decode_step(rba, name, one_launch):
    w, x, ref = _prepared(name)
    st = make_decode_store(rba, w, x, one_launch)
    # 8 x 32 (batch, kv head) units are more than the one launch takes (at most
    # half as many as SMs): that case keeps the three-kernel step
    one = one_launch and w.batch * w.n_kv_heads * 2 <= torch.cuda.get_device_properties(
        0).multi_processor_count
    assert st.decode_plan(w.top_k, w.context, w.sink, w.window) == (3 if one else 2)
    q = dev(x["q"], w.dtype)
    ws = st.decode_workspace(w.top_k, w.context, w.sink, w.window)
    for _ in range(2):  # the workspace is reusable call after call
        idx, out, lse = st.decode_step(q, w.top_k, w.context, w.sink, w.window, workspace=ws)
        st.check()
    check_decode_step(w, x["q"], x["K"], x["V"], ref, idx.cpu().numpy(), out.cpu().numpy(),
                      lse.cpu().numpy())


def test_two_key_weights_keep_full_precision(rba):
    # q puts almost all weight on two keys in the ratio 1 : e^-0.4; the output
    # is their weighted mean.  Weights rounded once to bf16 would move it by
    # ~1e-3 of |v|; the split weights (hi + lo) keep it within 1e-4.
    w = CASES["g4-d64-bs128"]
    x = synth.decode_inputs(w)
    st = make_decode_store(rba, w, x)
    g = w.n_q_heads // w.n_kv_heads
    scale = w.head_dim ** -0.5
    K = O.widen(x["K"][0, 0], w.dtype)
    V = O.widen(x["V"][0, 0], w.dtype)
    t1, t2 = w.context - 7, w.context - 300           # both inside the window
    A = np.array([[K[t1] @ K[t1], K[t1] @ K[t2]], [K[t2] @ K[t1], K[t2] @ K[t2]]])
    ab = np.linalg.solve(A, np.array([40.0, 39.6]) / scale)
    qv = np.zeros((1, w.n_q_heads, w.head_dim), dtype=np.float32)
    qv[0, :g] = ab[0] * K[t1] + ab[1] * K[t2]
    qb = synth.bf16_round(qv)
    sel = np.arange(1, w.top_k + 1)
    idx = torch.from_numpy(np.tile(sel, (1, w.n_kv_heads, 1)).astype(np.int32)).cuda()
    out, _ = st.attend(dev(qb, w.dtype), idx, w.context, w.sink, w.window)
    st.check()
    qw = O.widen(qb, w.dtype)
    toks = O.attended_tokens(w.context, w.block_size, w.sink, w.window, sel)
    got = out.cpu().numpy()
    for i in range(g):
        o_ref, _, _ = O.softmax_attention(qw[0, i], K[toks], V[toks], scale)
        assert np.abs(got[0, i] - o_ref).max() <= 1e-4 * np.abs(V[toks]).max()
