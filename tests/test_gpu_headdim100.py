"""Head dim 100 (MemLong summary, 2.4.1: OpenLLaMA-3B, 32 heads of dimension
100), against the fp64 oracle, through the C ABI.

The library holds such rows in pools of 128-element rows (rba_row_pitch), the
28 columns past the head dim zero; every other tensor (q, out, K/V inputs,
probes, landmarks, prefill Q and chunk K/V) is dense with rows of 100.  The
oracle needs no change: it reads the same dense inputs.  Covered: memorise
(top-r by attention, landmarks), the decode step on its three attention paths
(one launch; three kernels with the whole-block tensor-core kernel; fp32 with
the CUDA-core or split-K kernel), streaming appends, two-stage token
selection, and chunked prefill (cosine chunks; token-level retrieval through
the gathered past), each on rows that span several tiles and ragged tails."""
import numpy as np
import pytest
import torch

import oracle as O
from retrieval_block_sparse_b200 import synth

from parity import (OUT_TOL, check_decode_step, dev, make_decode_store, oracle_reps, out_error,
                    scale_of, selection_check)

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS
D = 100
DECODE = {
    # one launch (asked for): 32 MHA heads of 100 (B = 1), top-r representative keys
    "step-mha32": (W["infllm-decode-128k"].scaled(n_q_heads=32, n_kv_heads=32, head_dim=D,
                                                  context=16384, window=1024, top_k=16,
                                                  n_planted=8, seed=81), 3),
    # three kernels, whole-block tensor-core attention: 4 x 32 MHA heads
    "mma-b4": (W["infllm-decode-128k"].scaled(batch=4, n_q_heads=32, n_kv_heads=32,
                                              head_dim=D, context=4096, block_size=64, n_rep=1,
                                              rep_mode="mean", window=512, top_k=8,
                                              n_planted=4, seed=82), 2),
    # fp32 landmarks, ragged blocks: CUDA-core persistent or split-K attention
    "f32-landmark": (W["landmark-decode-b16"].scaled(dtype="f32", batch=2, n_q_heads=8,
                                                     n_kv_heads=4, head_dim=D, context=3000,
                                                     top_k=6, seed=83), None),
}


@pytest.mark.parametrize("name", list(DECODE))
def test_decode_step_d100(rba, name):
    w, plan = DECODE[name]
    x = synth.decode_inputs(w)
    reps, pos = oracle_reps(w, x)
    st = make_decode_store(rba, w, x, one_launch=plan == 3)
    assert st.pitch == 128 and st.k.shape[-1] == 128
    if plan is not None:
        assert st.decode_plan(w.top_k, w.context, w.sink, w.window) == plan
    torch.cuda.synchronize()
    st.check()
    # representations: the first 100 columns as the oracle's, the padding zero
    if w.rep_mode == "external":
        np.testing.assert_array_equal(st.rep[..., :D].cpu().float().numpy(), reps)
    elif w.rep_mode == "mean":
        got = st.rep[..., :D].cpu().numpy().astype(np.float64)
        np.testing.assert_allclose(got, reps, rtol=0, atol=1e-6 * np.abs(reps).max())
    elif w.rep_mode == "topr_attn":
        gpos = st.rep_pos.cpu().numpy()
        assert (gpos == pos).mean() >= 0.99
    assert float(st.rep[..., D:].abs().max()) == 0.0
    ref = O.decode(x["q"], x["K"], x["V"], reps, dtype=w.dtype, block_size=w.block_size,
                   sink=w.sink, window=w.window, top_k_blocks=w.top_k)
    ws = st.decode_workspace(w.top_k, w.context, w.sink, w.window)
    for _ in range(2):
        idx, out, lse = st.decode_step(dev(x["q"], w.dtype), w.top_k, w.context, w.sink,
                                       w.window, workspace=ws)
        st.check()
    assert out.shape[-1] == D
    check_decode_step(w, x["q"], x["K"], x["V"], ref, idx.cpu().numpy(), out.cpu().numpy(),
                      lse.cpu().numpy())
    # the attention call alone on the oracle's selection
    o2, l2 = st.attend(dev(x["q"], w.dtype), torch.from_numpy(ref["idx"].astype(np.int32)).cuda(),
                       w.context, w.sink, w.window)
    st.check()
    check_decode_step(w, x["q"], x["K"], x["V"], ref, ref["idx"], o2.cpu().numpy(),
                      l2.cpu().numpy(), min_exact=1.0)


def test_stream_step_d100(rba):
    # rows appended one at a time land in padded pool rows; blocks they
    # complete are memorised; every few steps the step matches the oracle
    T0, steps = 256, 24
    w = W["infllm-decode-128k"].scaled(n_q_heads=8, n_kv_heads=2, head_dim=D,
                                       context=T0 + steps, block_size=16, n_rep=1,
                                       rep_mode="mean", top_k=4, sink=16, window=64,
                                       recipe="normal", seed=84)
    x = synth.decode_inputs(w)
    st = rba.Store(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                   head_dim=D, block_size=w.block_size, capacity_tokens=w.context,
                   dtype=w.dtype, mode="mean")
    K, V = dev(x["K"], w.dtype), dev(x["V"], w.dtype)
    st.memorize(K[:, :, :T0].contiguous(), V[:, :, :T0].contiguous(), first_block=0,
                n_blocks=T0 // w.block_size)
    ws = st.decode_workspace(w.top_k, w.context, w.sink, w.window)
    rng = np.random.default_rng(5)
    for i in range(steps):
        T = T0 + i
        qn = synth.bf16_round(rng.standard_normal((1, w.n_q_heads, D)).astype(np.float32))
        idx, out, lse = st.stream_step(dev(qn, w.dtype), K[:, :, T].contiguous(),
                                       V[:, :, T].contiguous(), T, w.top_k, w.sink, w.window,
                                       workspace=ws)
        st.check()
        if i % 8 != 7:
            continue
        Tn = T + 1
        nb = Tn // w.block_size
        reps = np.stack([O.memorize(O.widen(x["K"][0, h, :nb * w.block_size], w.dtype), "mean",
                                    w.block_size)[0] for h in range(w.n_kv_heads)])[None]
        ref = O.decode(qn, x["K"][:, :, :Tn], x["V"][:, :, :Tn], reps, dtype=w.dtype,
                       block_size=w.block_size, sink=w.sink, window=w.window,
                       top_k_blocks=idx.shape[-1])
        check_decode_step(w, qn, x["K"], x["V"], ref, idx.cpu().numpy(), out.cpu().numpy(),
                          lse.cpu().numpy(), T=Tn, k=idx.shape[-1])
    assert float(st.k[..., D:].abs().max()) == 0.0


def test_two_stage_selection_d100(rba):
    w = W["token-retrieval-decode-1m"].scaled(head_dim=D, context=32768, top_k=128,
                                              recipe="drift", seed=85)
    group, kept = 32, 16
    x = synth.decode_inputs(w)
    st = rba.Store(batch=1, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, head_dim=D,
                   block_size=1, capacity_tokens=w.context, dtype="bf16", mode="identity")
    st.kv_rows(st.k).copy_(dev(x["K"], "bf16"))
    st.kv_rows(st.v).copy_(dev(x["V"], "bf16"))
    means = st.group_means(group)
    idx, groups, _ = st.approx_select(dev(x["q"], "bf16"), w.context, w.sink, w.window, group,
                                      kept, w.top_k, means)
    st.check()
    idx, groups = idx.cpu().numpy(), groups.cpu().numpy()
    g = w.n_q_heads // w.n_kv_heads
    for h in range(w.n_kv_heads):
        K = O.widen(x["K"][0, h], "bf16")
        qs = O.widen(x["q"][0, h * g:(h + 1) * g], "bf16")
        r = O.two_stage_select(qs, K, w.context, group=group, sink=w.sink, window=w.window,
                               groups_kept=kept, k=w.top_k)
        assert selection_check(r["group_scores"], kept, int(r["cand_groups"][0]),
                               groups[0, h]) == "exact"
        p = np.searchsorted(r["kept_tokens"], idx[0, h])
        selection_check(r["token_scores"], w.top_k, 0, p)


PREFILL = {
    "cosine-d100": W["memlong-cosine-prefill"].scaled(n_chunks=2, n_q_heads=4, n_kv_heads=4,
                                                      head_dim=D, chunk_len=200,
                                                      context=12 * 256, block_size=256,
                                                      top_k=3),
    "token-d100": W["token-retrieval-prefill-1m"].scaled(n_q_heads=8, n_kv_heads=2, head_dim=D,
                                                         chunk_len=256, context=16384,
                                                         top_k=384),
}


@pytest.mark.parametrize("name", list(PREFILL))
def test_prefill_d100(rba, name):
    w = PREFILL[name]
    x = synth.prefill_inputs(w)
    cosine = w.score_mode == "cosine"
    mode = "embed_cosine" if cosine else "identity"
    st = rba.Store(batch=1, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads, head_dim=D,
                   block_size=w.block_size, capacity_tokens=w.context, dtype="bf16", mode=mode,
                   d_ret=w.d_ret)
    st.kv_rows(st.k).copy_(dev(x["K"], "bf16"))
    st.kv_rows(st.v).copy_(dev(x["V"], "bf16"))
    nb = w.context // w.block_size
    if cosine:
        st.memorize(None, None, first_block=0, n_blocks=nb,
                    aux=torch.from_numpy(x["bank_embed"]).cuda().reshape(1, nb, w.d_ret))
    Q = dev(x["Q"], "bf16")
    ref = O.prefill(x["Q"], x["K"], x["V"], x["chunk_K"], x["chunk_V"], dtype="bf16",
                    block_size=w.block_size, sink=w.sink, window=w.window,
                    top_k_blocks=w.top_k, score_mode=w.score_mode,
                    query_embed=x.get("query_embed"), bank=x.get("bank_embed"))
    first, nc = st.candidates(w.context, w.sink, w.window)
    sc = st.score(torch.from_numpy(x["query_embed"]).cuda() if cosine else Q, w.context, w.sink,
                  w.window)
    gidx = rba.topk(sc.reshape(-1, nc), w.top_k, index_base=first).cpu().numpy()
    gidx = gidx.reshape(ref["idx"].shape)
    for c in range(gidx.shape[0]):
        for s_ in range(gidx.shape[1]):
            selection_check(ref["scores"][c, s_], w.top_k, first, gidx[c, s_])
    idx = torch.from_numpy(ref["idx"].astype(np.int32)).cuda()
    out, lse = st.attend_prefill(Q, idx, dev(x["chunk_K"], "bf16"), dev(x["chunk_V"], "bf16"),
                                 w.context, w.sink, w.window)
    st.check()
    assert out.shape[-1] == D
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    g = w.n_q_heads // w.n_kv_heads
    worst = 0.0
    for c in range(w.n_chunks):
        for hq in range(w.n_q_heads):
            h = hq // g
            sel = ref["idx"][c, 0 if cosine else h]
            toks = O.attended_tokens(w.context, w.block_size, w.sink, w.window, sel)
            vmax = max(float(np.abs(O.widen(x["V"][0, h, toks], "bf16")).max()),
                       float(np.abs(O.widen(x["chunk_V"][c, h], "bf16")).max()))
            worst = max(worst, float(np.abs(out[c, hq] - ref["out"][c, hq]).max()) / vmax)
            np.testing.assert_allclose(lse[c, hq], ref["lse"][c, hq], rtol=0, atol=2e-3)
    assert worst <= OUT_TOL["bf16"], worst
