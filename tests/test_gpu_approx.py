"""GPU parity of two-stage approximate token retrieval (rba_group_means,
rba_approx_select; RetrievalAttention summary, "proposed method") against the
oracle's two_stage_select on the same seeded inputs, through the C ABI.

Per (batch, kv head): the kept groups must be the oracle's stage-1 top groups
(exactly, or an accepted near-tie swap); the selected tokens must be the
oracle's stage-2 top tokens over the kept groups' candidate tokens (taken on
the GPU's kept groups, so a near-tie swap in stage 1 is followed through); the
keys read must be the oracle's count; and attention over sink U tokens U
window (rba_attend) must match the oracle's attention over the same tokens.

Cases: drift keys (nearby keys resemble each other, the regime the index
exploits) at 64K and at the full 1M-token shape with k = 2048; a ragged case
whose sink and window cut groups (partly outside kept groups) in fp32."""
import numpy as np
import pytest
import torch

import oracle as O
from retrieval_block_sparse_b200 import synth

from parity import OUT_TOL, dev, out_error, scale_of, selection_check

pytestmark = pytest.mark.gpu
BASE = synth.WORKLOADS["token-retrieval-decode-1m"]
CASES = {
    "drift-64k": (BASE.scaled(context=65536, top_k=256, recipe="drift", seed=71), 64, 16),
    "ragged-f32": (BASE.scaled(dtype="f32", n_q_heads=8, n_kv_heads=2, head_dim=64,
                               context=20000, top_k=100, sink=100, window=300,
                               recipe="drift", seed=72), 48, 8),
    "drift-1m": (BASE.scaled(recipe="drift", seed=73), 64, 256),
}


def _positions(tokens, within):
    """Positions of `tokens` in the ascending array `within` (all must be there)."""
    p = np.searchsorted(within, tokens)
    assert np.all(p < within.size) and np.array_equal(within[p], tokens), "token not a candidate"
    return p


@pytest.mark.parametrize("name", list(CASES))
def test_two_stage_selection_and_attention(rba, name):
    w, group, kept = CASES[name]
    x = synth.decode_inputs(w)
    st = rba.Store(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                   head_dim=w.head_dim, block_size=1, capacity_tokens=w.context,
                   dtype=w.dtype, mode="identity")
    st.k.copy_(dev(x["K"], w.dtype))
    st.v.copy_(dev(x["V"], w.dtype))
    means = st.group_means(group)
    q = dev(x["q"], w.dtype)
    idx, groups, scanned = st.approx_select(q, w.context, w.sink, w.window, group, kept,
                                            w.top_k, means)
    out, lse = st.attend(q, idx, w.context, w.sink, w.window)
    st.check()
    idx, groups, scanned = idx.cpu().numpy(), groups.cpu().numpy(), scanned.cpu().numpy()
    out, lse = out.cpu().numpy(), lse.cpu().numpy()
    g = w.n_q_heads // w.n_kv_heads
    w0 = w.context - w.window
    for b in range(w.batch):
        for h in range(w.n_kv_heads):
            K = O.widen(x["K"][b, h], w.dtype)
            qs = O.widen(x["q"][b, h * g:(h + 1) * g], w.dtype)
            r = O.two_stage_select(qs, K, w.context, group=group, sink=w.sink,
                                   window=w.window, groups_kept=kept, k=w.top_k)
            # stage 1: the kept groups
            kind = selection_check(r["group_scores"], kept, int(r["cand_groups"][0]),
                                   groups[b, h])
            if kind == "exact":
                toks, s2 = r["kept_tokens"], r["token_scores"]
            else:  # follow the GPU's (near-tie) choice into stage 2
                toks = np.array([t for gg in groups[b, h]
                                 for t in range(gg * group, (gg + 1) * group)
                                 if w.sink <= t < w0], dtype=np.int64)
                s2 = O.score_dot(qs, K[toks][:, None, :])
            # stage 2: the tokens, as positions among the kept candidate tokens
            selection_check(s2, w.top_k, 0, _positions(idx[b, h], toks))
            assert scanned[b, h] == r["cand_groups"].size + toks.size
            # attention over sink U the GPU's tokens U window
            att = O.attended_tokens(w.context, 1, w.sink, w.window, idx[b, h])
            Kt, Vt = K[att], O.widen(x["V"][b, h, att], w.dtype)
            for i in range(h * g, (h + 1) * g):
                o, l, _ = O.softmax_attention(qs[i - h * g], Kt, Vt, scale_of(w))
                assert out_error(out[b, i], o, Vt) <= OUT_TOL[w.dtype]
                assert abs(lse[b, i] - l) <= OUT_TOL[w.dtype]


def test_every_group_kept_is_the_exact_selection(rba):
    # keeping every candidate group makes stage 2 the exact search: the GPU's
    # tokens equal the exact top-k of rba_score + rba_topk
    w = BASE.scaled(context=8192, top_k=64, recipe="drift", seed=74)
    group = 32
    x = synth.decode_inputs(w)
    st = rba.Store(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                   head_dim=w.head_dim, block_size=1, capacity_tokens=w.context,
                   dtype=w.dtype, mode="identity")
    st.k.copy_(dev(x["K"], w.dtype))
    st.v.copy_(dev(x["V"], w.dtype))
    means = st.group_means(group)
    q = dev(x["q"], w.dtype)
    n_groups = O.candidate_blocks(w.context, group, w.sink, w.window).size
    idx, _, scanned = st.approx_select(q, w.context, w.sink, w.window, group, n_groups,
                                       w.top_k, means)
    first, nc = st.candidates(w.context, w.sink, w.window)
    exact = rba.topk(st.score(q, w.context, w.sink, w.window).reshape(-1, nc), w.top_k,
                     index_base=first)
    st.check()
    assert torch.equal(idx.reshape(-1, w.top_k), exact)
    assert (scanned.cpu().numpy() == n_groups + nc).all()


def test_argument_checks(rba):
    w = BASE.scaled(context=4096, top_k=64)
    st = rba.Store(batch=1, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                   head_dim=w.head_dim, block_size=1, capacity_tokens=w.context, dtype="bf16",
                   mode="identity")
    means = st.group_means(64)
    q = torch.zeros((1, w.n_q_heads, w.head_dim), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(rba.RbaError):  # 1 group of 64 cannot hold k = 64 + 2 * 64
        st.approx_select(q, w.context, w.sink, w.window, 64, 1, 64, means)
    with pytest.raises(rba.RbaError):  # more groups kept than candidates
        st.approx_select(q, w.context, w.sink, w.window, 64, 1000, 64, means)
    blocked = rba.Store(batch=1, n_q_heads=4, n_kv_heads=4, head_dim=64, block_size=64,
                        capacity_tokens=4096, dtype="bf16", mode="mean")
    with pytest.raises(rba.RbaError):  # not a block-size-1 store
        blocked.group_means(64)
