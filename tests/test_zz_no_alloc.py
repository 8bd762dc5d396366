"""rba_attend_noalloc: decode attention for callers that cannot allocate.

Some hosts own all device memory through their own allocator (a serving
engine that reserves HBM at start-up), and some call sites cannot afford the
device-wide synchronisation a cudaMalloc may cause.  Those callers cannot hand
rba_attend a workspace; rba_attend_noalloc keeps the scratch in a fixed
device array inside the library instead.

This test calls it through the C ABI twice in a row (different queries, the
second call reusing whatever the first left in the shared array) and checks
each output against rba_attend's, within the attention tolerance the other
tests use (2e-3 of max |V| for bf16).  It also checks the size limit: a
problem whose split-K scratch (computed here from the documented layout) fits
runs and matches rba_attend, one just over it is rejected.  This
file is collected last, and it passes on its own in a fresh process too (its
first call is the first use of the array on the device).
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
from retrieval_block_sparse_b200 import synth

from parity import OUT_TOL, dev, make_decode_store, oracle_reps

pytestmark = pytest.mark.gpu


def _noalloc(rba, st, q, idx, w, out, lse):
    L = rba.lib()
    s = L.rba_attend_noalloc(st.handle, q.data_ptr(), idx.data_ptr(), idx.shape[-1], w.context,
                             w.sink, w.window, ctypes.c_float(w.head_dim ** -0.5),
                             out.data_ptr(), lse.data_ptr(),
                             torch.cuda.current_stream().cuda_stream)
    return s


def test_noalloc_matches_attend_twice(rba):
    w = synth.WORKLOADS["infllm-decode-128k"]
    x = synth.decode_inputs(w)
    reps, _ = oracle_reps(w, x)
    st = make_decode_store(rba, w, x)
    ref = O.decode(x["q"], x["K"], x["V"], reps, dtype=w.dtype, block_size=w.block_size,
                   sink=w.sink, window=w.window, top_k_blocks=w.top_k)
    idx = torch.from_numpy(ref["idx"].astype(np.int32)).cuda()
    vmax = float(np.abs(O.widen(x["V"], w.dtype)).max())
    q1 = dev(x["q"], w.dtype)
    q2 = (q1.float() * -0.75).to(torch.bfloat16).contiguous()
    for q in (q1, q2):
        out = torch.full((w.batch, w.n_q_heads, w.head_dim), float("nan"), device="cuda")
        lse = torch.full((w.batch, w.n_q_heads), float("nan"), device="cuda")
        assert _noalloc(rba, st, q, idx, w, out, lse) == rba.OK
        st.check()
        o_ref, l_ref = st.attend(q, idx, w.context, w.sink, w.window)
        err = float((out - o_ref).abs().max()) / vmax
        assert err <= OUT_TOL[w.dtype], err
        assert float((lse - l_ref).abs().max()) <= OUT_TOL[w.dtype]


def _split_k_scratch_bytes(batch, n_kv_heads, n_q_heads, head_dim, nsplit):
    """The split-K kernel's scratch as the library lays it out: merge tickets
    (one uint32 per (batch, kv head), 256-byte aligned), then one partial state
    (m, l, o[D]) of fp32 per (batch, q head, split), 256-byte aligned."""
    up = lambda n: (n + 255) // 256 * 256  # noqa: E731
    return up(4 * batch * n_kv_heads) + up(batch * n_q_heads * nsplit * (head_dim + 2) * 4)


@pytest.mark.parametrize("batch,fits", [(125, True), (126, False)])
def test_noalloc_limit_is_the_split_k_scratch(rba, batch, fits):
    # 32 MHA heads of 100 tokens per batch row: with more (batch, kv head)
    # units than SMs and rows this short the split-K kernel uses one split, so
    # its scratch is 4 B of ticket plus 32 * 130 * 4 B of partials per row:
    # 125 rows fit in the fixed array, 126 do not
    w = synth.WORKLOADS["landmark-decode-b16"].scaled(batch=batch, context=100)
    need = _split_k_scratch_bytes(batch, w.n_kv_heads, w.n_q_heads, w.head_dim, 1)
    assert (need <= (2 << 20)) == fits
    st = rba.Store(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                   head_dim=w.head_dim, block_size=w.block_size, capacity_tokens=w.context,
                   dtype="bf16", mode="external")
    gen = torch.Generator(device="cuda").manual_seed(batch)
    st.k.copy_(torch.randn(st.k.shape, generator=gen, device="cuda").to(torch.bfloat16))
    st.v.copy_(torch.randn(st.v.shape, generator=gen, device="cuda").to(torch.bfloat16))
    q = torch.randn((w.batch, w.n_q_heads, w.head_dim), generator=gen,
                    device="cuda").to(torch.bfloat16)
    idx = torch.zeros((w.batch, w.n_kv_heads, 0), dtype=torch.int32, device="cuda")
    out = torch.full((w.batch, w.n_q_heads, w.head_dim), float("nan"), device="cuda")
    lse = torch.full((w.batch, w.n_q_heads), float("nan"), device="cuda")
    s = _noalloc(rba, st, q, idx, w, out, lse)
    if not fits:
        assert s == rba.ERR_WORKSPACE
        assert torch.isnan(out).all()  # nothing launched
        return
    assert s == rba.OK
    st.check()
    o_ref, l_ref = st.attend(q, idx, w.context, w.sink, w.window)
    vmax = float(st.v.float().abs().max())
    assert float((out - o_ref).abs().max()) / vmax <= OUT_TOL["bf16"]
    assert float((lse - l_ref).abs().max()) <= OUT_TOL["bf16"]


SPLIT_K_CASES = {
    "tiny-decode-f32": synth.WORKLOADS["tiny-decode-f32"],
    "ragged-f32": synth.WORKLOADS["tiny-decode-f32"].scaled(
        n_q_heads=8, n_kv_heads=4, context=1000, block_size=24, sink=30, window=70, top_k=7,
        seed=11),
    "landmark-small": synth.WORKLOADS["landmark-decode-b16"].scaled(
        batch=2, n_q_heads=4, n_kv_heads=4, context=5018),
    "token-small": synth.WORKLOADS["token-retrieval-decode-1m"].scaled(context=65536,
                                                                         top_k=256),
}


@pytest.mark.parametrize("name", list(SPLIT_K_CASES))
def test_noalloc_split_k_matches_oracle(rba, name):
    # rba_attend_noalloc always runs the split-K kernel (rba_attend takes the
    # persistent kernel where it applies): this is that kernel's parity
    # against the oracle, on the oracle's own selection
    from parity import attended_v_max, out_error
    w = SPLIT_K_CASES[name]
    x = synth.decode_inputs(w)
    reps, _ = oracle_reps(w, x)
    st = make_decode_store(rba, w, x)
    ref = O.decode(x["q"], x["K"], x["V"], reps, dtype=w.dtype, block_size=w.block_size,
                   sink=w.sink, window=w.window, top_k_blocks=w.top_k)
    idx = torch.from_numpy(ref["idx"].astype(np.int32)).cuda()
    q = dev(x["q"], w.dtype)
    out = torch.empty((w.batch, w.n_q_heads, w.head_dim), device="cuda")
    lse = torch.empty((w.batch, w.n_q_heads), device="cuda")
    assert _noalloc(rba, st, q, idx, w, out, lse) == rba.OK
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
