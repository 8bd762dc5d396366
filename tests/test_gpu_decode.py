"""GPU parity of the decode path (memorise, score, top-k, attend, whole step)
against the fp64 oracle on the same seeded inputs, through the C ABI.

Workloads: the four decode configurations at full size (the sizes the bench
times), plus reduced-size variants of the same recipes that the oracle
finishes quickly and that still span many tiles, several splits and ragged
tails."""
import numpy as np
import pytest
import torch

import oracle as O
from retrieval_block_sparse_b200 import synth

from parity import (OUT_TOL, attended_v_max, check_decode_step, dev, make_decode_store,
                    oracle_reps, out_error, scale_of, score_tolerance)

W = synth.WORKLOADS
CASES = {
    "tiny-decode-f32": W["tiny-decode-f32"],
    "infllm-small": W["infllm-decode-128k"].scaled(context=16384, window=1024, top_k=16,
                                                   n_planted=8),
    "infllm-decode-128k": W["infllm-decode-128k"],
    "landmark-small": W["landmark-decode-b16"].scaled(batch=2, n_q_heads=4, n_kv_heads=4,
                                                      context=5018),
    "landmark-decode-b16": W["landmark-decode-b16"],
    "token-small": W["token-retrieval-decode-1m"].scaled(context=65536, top_k=256),
    "token-retrieval-decode-1m": W["token-retrieval-decode-1m"],
    # edge geometry: odd block size, sink and window not block-aligned, GQA 2
    "ragged-f32": W["tiny-decode-f32"].scaled(n_q_heads=8, n_kv_heads=4, context=1000,
                                              block_size=24, sink=30, window=70, top_k=7, seed=11),
}

_cache = {}


def _prepared(name):
    if name not in _cache:
        w = CASES[name]
        x = synth.decode_inputs(w)
        reps, pos = oracle_reps(w, x)
        ref = O.decode(x["q"], x["K"], x["V"], reps, dtype=w.dtype, block_size=w.block_size,
                       sink=w.sink, window=w.window, top_k_blocks=w.top_k)
        _cache.clear()  # keep one full-size workload in host memory at a time
        _cache[name] = (w, x, reps, pos, ref)
    return _cache[name]


pytestmark = pytest.mark.gpu
NAMES = list(CASES)


@pytest.mark.parametrize("name", NAMES)
def test_memorize(rba, name):
    w, x, reps, pos, _ = _prepared(name)
    st = make_decode_store(rba, w, x)
    torch.cuda.synchronize()
    st.check()
    if w.rep_mode == "identity":
        return
    got = st.rep.cpu().float().numpy().astype(np.float64)
    if w.rep_mode == "mean":
        np.testing.assert_allclose(got, reps, rtol=0, atol=1e-6 * np.abs(reps).max())
    elif w.rep_mode == "external":
        np.testing.assert_array_equal(got, reps)
    elif w.rep_mode == "topr_attn":
        gpos = st.rep_pos.cpu().numpy()
        bad = np.argwhere((gpos != pos).any(axis=-1))
        # a differing block is only accepted at a near-tie of received attention
        probe = O.widen(x["probe"], w.dtype)
        for b, h, j in bad:
            Kb = O.widen(x["K"][b, h, j * w.block_size:(j + 1) * w.block_size], w.dtype)
            _, _, recv = O.rep_topr_attention(Kb, probe[h], w.n_rep, scale_of(w))
            order = np.sort(recv)[::-1]
            ar, ar1 = order[w.n_rep - 1], order[w.n_rep]
            assert ar - ar1 <= 1e-5 * ar, (b, h, j, gpos[b, h, j], pos[b, h, j])
            for t in set(gpos[b, h, j]) ^ set(pos[b, h, j]):
                assert abs(recv[t] - ar) <= 1e-5 * ar
        assert len(bad) <= max(1, gpos.shape[2] // 100)
        # rep keys are exact copies of the chosen keys
        for b in range(w.batch):
            for h in range(w.n_kv_heads):
                kk = O.widen(x["K"][b, h], w.dtype)
                rows = (np.arange(w.n_blocks)[:, None] * w.block_size + gpos[b, h]).reshape(-1)
                np.testing.assert_array_equal(got[b, h].reshape(-1, w.head_dim), kk[rows])


@pytest.mark.parametrize("name", NAMES)
def test_score(rba, name):
    w, x, reps, pos, ref = _prepared(name)
    st = make_decode_store(rba, w, x)
    q = dev(x["q"], w.dtype)
    s = st.score(q, w.context, w.sink, w.window).cpu().numpy().astype(np.float64)
    st.check()
    g = w.n_q_heads // w.n_kv_heads
    cand = ref["cand"]
    for b in range(w.batch):
        for h in range(w.n_kv_heads):
            qa = np.abs(O.widen(x["q"][b, h * g:(h + 1) * g], w.dtype)).sum(axis=0)
            if reps is None:
                ra = np.abs(O.widen(x["K"][b, h, cand], w.dtype))[:, None, :]
            else:
                ra = np.abs(reps[b, h, cand])
            tol = score_tolerance(qa, ra)
            err = np.abs(s[b, h] - ref["scores"][b, h])
            assert np.all(err <= tol), (b, h, float(err.max()), float(tol.min()))


@pytest.mark.parametrize("name", NAMES)
def test_attend_on_oracle_selection(rba, name):
    w, x, reps, pos, ref = _prepared(name)
    st = make_decode_store(rba, w, x)
    q = dev(x["q"], w.dtype)
    idx = torch.from_numpy(ref["idx"].astype(np.int32)).cuda()
    out, lse = st.attend(q, idx, w.context, w.sink, w.window)
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
@pytest.mark.parametrize("name", NAMES)
def test_decode_step(rba, name, one_launch):
    w, x, reps, pos, ref = _prepared(name)
    st = make_decode_store(rba, w, x, one_launch)
    q = dev(x["q"], w.dtype)
    ws = st.decode_workspace(w.top_k, w.context, w.sink, w.window)
    for _ in range(2):  # the workspace must be reusable call after call
        idx, out, lse = st.decode_step(q, w.top_k, w.context, w.sink, w.window, workspace=ws)
        st.check()
    check_decode_step(w, x["q"], x["K"], x["V"], ref, idx.cpu().numpy(), out.cpu().numpy(),
                      lse.cpu().numpy())


def test_planted_blocks_retrieved_on_gpu(rba):
    w, x, _, _, ref = _prepared("infllm-decode-128k")
    st = make_decode_store(rba, w, x)
    idx, _, _ = st.decode_step(dev(x["q"], w.dtype), w.top_k, w.context, w.sink, w.window)
    idx = idx.cpu().numpy()
    hits = sum(len(set(idx[0, h]) & set(x["planted_blocks"][0, h])) for h in range(w.n_kv_heads))
    chance = w.n_kv_heads * w.n_planted * w.top_k / ref["cand"].shape[0]
    assert hits > 4 * chance


@pytest.mark.parametrize("name", ["infllm-decode-128k", "landmark-decode-b16",
                                  "token-retrieval-decode-1m", "ragged-f32"])
def test_decode_step_host(rba, name):
    """The step through rba_decode_step_host, the entry point the bench's
    end-to-end figure uses: q from pinned host memory, out, lse and the
    selection copied back to pinned host buffers, the call synchronising.
    The host outputs are checked against the oracle as the device step's are,
    on two calls over one workspace."""
    w, x, reps, pos, ref = _prepared(name)
    st = make_decode_store(rba, w, x)
    q = dev(x["q"], w.dtype)
    q_host = q.cpu().pin_memory()
    B, Hq, Hkv, D = w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim
    q_dev = torch.empty_like(q)
    idx_dev = torch.empty((B, Hkv, w.top_k), dtype=torch.int32, device="cuda")
    out_dev = torch.empty((B, Hq, D), dtype=torch.float32, device="cuda")
    lse_dev = torch.empty((B, Hq), dtype=torch.float32, device="cuda")
    out_h = torch.empty(out_dev.shape, dtype=torch.float32).pin_memory()
    lse_h = torch.empty(lse_dev.shape, dtype=torch.float32).pin_memory()
    idx_h = torch.empty(idx_dev.shape, dtype=torch.int32).pin_memory()
    ws = st.decode_workspace(w.top_k, w.context, w.sink, w.window)
    for _ in range(2):
        out_h.fill_(float("nan"))
        idx_h.fill_(-1)
        st.decode_step_host(q_host, w.top_k, w.context, w.sink, w.window, q_dev=q_dev,
                            idx_dev=idx_dev, out_dev=out_dev, lse_dev=lse_dev, out_host=out_h,
                            lse_host=lse_h, idx_host=idx_h, workspace=ws)
    st.check()
    check_decode_step(w, x["q"], x["K"], x["V"], ref, idx_h.numpy(), out_h.numpy(),
                      lse_h.numpy())
