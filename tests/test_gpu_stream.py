"""Streaming decode through the C ABI (rba_stream_step): the context grows by
one token per step, the block each append completes is memorised then, and
each step's selection and output are checked against the fp64 oracle run on
the whole context of that step (representations recomputed from scratch).

The streams start at 256 tokens and run 40 steps, crossing two 16-token block
boundaries and moving the window and the candidate range; representations
cover the mean, the InfLLM top-r-by-attention and the Landmark (external)
modes.  Acceptance as in the other decode tests: selections exact except at
near-ties, outputs within 2e-3 of max |V| (bf16)."""
import numpy as np
import pytest
import torch

import oracle as O
from retrieval_block_sparse_b200 import synth

from parity import check_decode_step, dev

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS
T0, STEPS = 256, 40
CASES = {
    "mean": W["infllm-decode-128k"].scaled(n_q_heads=8, n_kv_heads=2, context=T0 + STEPS,
                                           block_size=16, n_rep=1, rep_mode="mean", top_k=4,
                                           sink=16, window=64, recipe="normal", seed=31),
    "topr": W["infllm-decode-128k"].scaled(n_q_heads=8, n_kv_heads=2, context=T0 + STEPS,
                                           block_size=16, n_rep=2, rep_mode="topr_attn",
                                           top_k=3, sink=16, window=48, n_probe=8,
                                           recipe="normal", seed=32),
    "landmark": W["landmark-decode-b16"].scaled(batch=2, n_q_heads=4, n_kv_heads=4,
                                                context=T0 + STEPS, block_size=16, top_k=4,
                                                sink=0, window=40, seed=33),
}


def _reps(w, x, T):
    """Oracle representations of the full blocks among the first T tokens."""
    nb = T // w.block_size
    reps = np.zeros((w.batch, w.n_kv_heads, nb, w.n_rep, w.head_dim))
    for b in range(w.batch):
        for h in range(w.n_kv_heads):
            if w.rep_mode == "external":
                reps[b, h, :, 0] = O.widen(x["landmarks"][b, h, :nb], w.dtype)
                continue
            probe = O.widen(x["probe"][h], w.dtype) if w.rep_mode == "topr_attn" else None
            reps[b, h] = O.memorize(O.widen(x["K"][b, h, :nb * w.block_size], w.dtype),
                                    w.rep_mode, w.block_size, w.n_rep, probe=probe)[0]
    return reps


@pytest.mark.parametrize("name", list(CASES))
def test_stream_steps_match_oracle(rba, name):
    w = CASES[name]
    x = synth.decode_inputs(w)
    st = rba.Store(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                   head_dim=w.head_dim, block_size=w.block_size, capacity_tokens=w.context,
                   dtype=w.dtype, mode=w.rep_mode, n_rep=w.n_rep)
    K, V = dev(x["K"], w.dtype), dev(x["V"], w.dtype)
    nb0 = T0 // w.block_size
    aux_all = None
    if w.rep_mode == "topr_attn":
        aux_all = dev(x["probe"], w.dtype)
    elif w.rep_mode == "external":
        aux_all = dev(x["landmarks"], w.dtype).reshape(w.batch, w.n_kv_heads, w.n_blocks, 1,
                                                        w.head_dim)
    # the first T0 tokens: pools and representations in one call
    st.memorize(K[:, :, :T0].contiguous(), V[:, :, :T0].contiguous(), first_block=0,
                n_blocks=nb0,
                aux=(aux_all[:, :, :nb0].contiguous() if w.rep_mode == "external" else aux_all))
    rng = np.random.default_rng(w.seed)
    ws = st.decode_workspace(w.top_k, w.context, w.sink, w.window)
    checked = 0
    for i in range(STEPS):
        T = T0 + i
        qn = synth.bf16_round(rng.standard_normal((w.batch, w.n_q_heads, w.head_dim))
                              .astype(np.float32))
        q = dev(qn, w.dtype)
        aux = aux_all
        if w.rep_mode == "external":
            blk = (T + 1) // w.block_size - 1
            aux = aux_all[:, :, blk:blk + 1].contiguous()
        idx, out, lse = st.stream_step(q, K[:, :, T].contiguous(), V[:, :, T].contiguous(), T,
                                       w.top_k, w.sink, w.window, aux=aux, workspace=ws)
        st.check()
        if i % 7 != 6 and i != STEPS - 1:
            continue
        checked += 1
        Tn = T + 1
        first, nc = st.candidates(Tn, w.sink, w.window)
        ke = min(w.top_k, nc)
        assert idx.shape[-1] == ke
        ref = O.decode(qn, x["K"][:, :, :Tn], x["V"][:, :, :Tn], _reps(w, x, Tn), dtype=w.dtype,
                       block_size=w.block_size, sink=w.sink, window=w.window, top_k_blocks=ke)
        check_decode_step(w, qn, x["K"], x["V"], ref, idx.cpu().numpy(), out.cpu().numpy(),
                          lse.cpu().numpy(), T=Tn, k=ke)
    assert checked >= 6


def test_stream_rejects_growth_beyond_capacity(rba):
    w = CASES["mean"]
    st = rba.Store(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                   head_dim=w.head_dim, block_size=w.block_size, capacity_tokens=64,
                   dtype=w.dtype, mode=w.rep_mode, n_rep=w.n_rep)
    q = torch.zeros((w.batch, w.n_q_heads, w.head_dim), dtype=torch.bfloat16, device="cuda")
    kv = torch.zeros((w.batch, w.n_kv_heads, w.head_dim), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rba.RbaError):
        st.stream_step(q, kv, kv, 64, w.top_k, w.sink, w.window)
