"""GPU parity of the decode step's selection paths against the fp64 oracle,
through the C ABI: the one-launch step (rba_decode_step on a store with
rba_store_set_decode_step_one_launch(store, 1), plan 3; one selecting warp
per part) and, on the same tie cases, the default score -> top-k ->
attention step (rba_topk's kernel).

The whole-step tests of test_gpu_decode.py, test_gpu_decode_mma.py,
test_gpu_fused.py and test_gpu_score_max.py run this kernel and the default
three-kernel step on the configurations they cover
(GQA 1, 2 and 4, head dims 64 and 128, mean / top-r representations with 1, 2,
4 and 8 keys, sum and max scores).  This file adds what those random inputs do
not reach: exact score ties at the k-th place (the lower block index must win,
as in the oracle), a row of equal scores and a row whose k-th score sits
among many near-equal scores (long radix searches), a part count
that leaves some parts without candidates, and the bounded waits: with a wait
limit of 1 ns the step must report RBA_ERR_TIMEOUT in the status word and
return, and the next call on the same workspace must match the oracle."""
import numpy as np
import pytest
import torch

import oracle as O
from retrieval_block_sparse_b200 import synth

from parity import check_decode_step, dev, make_decode_store, oracle_reps

pytestmark = pytest.mark.gpu
BASE = synth.WORKLOADS["infllm-decode-128k"]
SMALL = BASE.scaled(context=16384, window=1024, top_k=16, n_planted=8, seed=61)


def _run_with_reps(rba, w, x, reps, one_launch):
    """Store with the given representations written into its rep pool, one
    decode step (one launch, or the default score -> top-k -> attention), and
    the oracle on the same representations."""
    st = make_decode_store(rba, w, x, one_launch=one_launch)
    assert st.decode_plan(w.top_k, w.context, w.sink, w.window) == (3 if one_launch else 2)
    assert st.decode_launches(w.top_k, w.context, w.sink, w.window) == (1 if one_launch else 3)
    rb = torch.from_numpy(reps.astype(np.float32)).to(torch.bfloat16)
    st.rep.copy_(rb.cuda())
    reps_stored = rb.float().numpy().astype(np.float64)  # the values the GPU reads
    ref = O.decode(x["q"], x["K"], x["V"], reps_stored, dtype=w.dtype,
                   block_size=w.block_size, sink=w.sink, window=w.window,
                   top_k_blocks=w.top_k)
    idx, out, lse = st.decode_step(dev(x["q"], w.dtype), w.top_k, w.context, w.sink, w.window)
    st.check()
    return st, ref, idx.cpu().numpy(), out.cpu().numpy(), lse.cpu().numpy()


def test_plan_at_128k(rba):
    w = BASE
    x = synth.decode_inputs(w.scaled(context=8192, window=1024, n_planted=4))
    st = rba.Store(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                   head_dim=w.head_dim, block_size=w.block_size, capacity_tokens=w.context,
                   dtype=w.dtype, mode=w.rep_mode, n_rep=w.n_rep)
    del x
    # by default score -> top-k -> whole-block attention; one launch when
    # asked for
    assert st.decode_plan(w.top_k, w.context, w.sink, w.window) == 2
    assert st.decode_launches(w.top_k, w.context, w.sink, w.window) == 3
    st.set_decode_step_one_launch(True)
    assert st.decode_plan(w.top_k, w.context, w.sink, w.window) == 3
    assert st.decode_launches(w.top_k, w.context, w.sink, w.window) == 1
    st.set_decode_step_one_launch(False)
    assert st.decode_plan(w.top_k, w.context, w.sink, w.window) == 2


@pytest.mark.parametrize("one_launch", [True, False])
def test_exact_ties_take_the_lower_block(rba, one_launch):
    # copy the representation of the oracle's k-th block onto candidates just
    # below and just above it in index: their scores equal the k-th exactly,
    # so the lower index must be selected, bit for bit as in the oracle
    w = SMALL
    x = synth.decode_inputs(w)
    reps, _ = oracle_reps(w, x)
    reps = synth.bf16_to_f32(synth.bf16_round(reps.astype(np.float32))).astype(np.float64)
    ref = O.decode(x["q"], x["K"], x["V"], reps, dtype=w.dtype, block_size=w.block_size,
                   sink=w.sink, window=w.window, top_k_blocks=w.top_k)
    cand = ref["cand"]
    for h in range(w.n_kv_heads):
        s = ref["scores"][0, h]
        order = np.lexsort((np.arange(s.size), -s))
        kth = cand[order[w.top_k - 1]]
        for j in (kth - 3, kth + 5):  # neighbours outside the selection
            if cand[0] <= j < cand[0] + cand.size and j not in ref["idx"][0, h]:
                reps[0, h, j] = reps[0, h, kth]
    st, ref2, idx, out, lse = _run_with_reps(rba, w, x, reps, one_launch)
    np.testing.assert_array_equal(idx, ref2["idx"])
    check_decode_step(w, x["q"], x["K"], x["V"], ref2, idx, out, lse, min_exact=1.0)


@pytest.mark.parametrize("one_launch", [True, False])
def test_equal_scores_select_the_first_candidates(rba, one_launch):
    # every block represented by the same keys: one score per head, a zero
    # value range; the k lowest candidate blocks are selected
    w = SMALL
    x = synth.decode_inputs(w)
    reps, _ = oracle_reps(w, x)
    reps[:] = reps[:, :, :1]
    st, ref, idx, out, lse = _run_with_reps(rba, w, x, reps, one_launch)
    first = int(ref["cand"][0])
    np.testing.assert_array_equal(idx, np.broadcast_to(np.arange(first, first + w.top_k),
                                                       idx.shape))
    check_decode_step(w, x["q"], x["K"], x["V"], ref, idx, out, lse, min_exact=1.0)


@pytest.mark.parametrize("one_launch", [True, False])
def test_crowded_boundary_bin(rba, one_launch):
    # two far outliers stretch the value range while the remaining scores
    # crowd near one value: the k-th score shares its high bits with most of
    # the row, so the radix search runs down to the low bits (and a binning
    # select would hold them in one bin)
    w = SMALL
    x = synth.decode_inputs(w)
    reps, _ = oracle_reps(w, x)
    rng = np.random.default_rng(62)
    base = reps[:, :, :1].copy()
    reps[:] = base + 1e-2 * rng.standard_normal(reps.shape)
    q = O.widen(x["q"], w.dtype)
    g = w.n_q_heads // w.n_kv_heads
    for h in range(w.n_kv_heads):
        qs = q[0, h * g:(h + 1) * g].sum(axis=0)
        u = qs / np.linalg.norm(qs)
        reps[0, h, 10] = base[0, h, 0] + 400.0 * u / w.n_rep   # far above
        reps[0, h, 20] = base[0, h, 0] - 400.0 * u / w.n_rep   # far below
    st, ref, idx, out, lse = _run_with_reps(rba, w, x, reps, one_launch)
    check_decode_step(w, x["q"], x["K"], x["V"], ref, idx, out, lse)
    assert all(10 in idx[0, h] and 20 not in idx[0, h] for h in range(w.n_kv_heads))


def test_parts_without_candidates(rba):
    # 4 kv heads x 37 parts and only 6 candidates per head: most parts score
    # nothing, the selection still covers every candidate it must
    w = BASE.scaled(n_q_heads=8, n_kv_heads=4, context=2048, window=1024, top_k=3,
                    n_planted=2, seed=63)
    x = synth.decode_inputs(w)
    reps, _ = oracle_reps(w, x)
    st = make_decode_store(rba, w, x, one_launch=True)
    assert st.decode_plan(w.top_k, w.context, w.sink, w.window) == 3
    ref = O.decode(x["q"], x["K"], x["V"], reps, dtype=w.dtype, block_size=w.block_size,
                   sink=w.sink, window=w.window, top_k_blocks=w.top_k)
    ws = st.decode_workspace(w.top_k, w.context, w.sink, w.window)
    for _ in range(3):
        idx, out, lse = st.decode_step(dev(x["q"], w.dtype), w.top_k, w.context, w.sink,
                                       w.window, workspace=ws)
        st.check()
    check_decode_step(w, x["q"], x["K"], x["V"], ref, idx.cpu().numpy(), out.cpu().numpy(),
                      lse.cpu().numpy())


def test_wait_that_runs_out_reports_timeout_and_next_call_is_correct(rba):
    w = SMALL
    x = synth.decode_inputs(w)
    reps, _ = oracle_reps(w, x)
    st = make_decode_store(rba, w, x, one_launch=True)
    assert st.decode_plan(w.top_k, w.context, w.sink, w.window) == 3
    q = dev(x["q"], w.dtype)
    ws = st.decode_workspace(w.top_k, w.context, w.sink, w.window)
    # a 1 ns bound: a part whose selector finds the head's slices not all
    # published yet gives up at once
    st.set_wait_limit_ns(1)
    st.decode_step(q, w.top_k, w.context, w.sink, w.window, workspace=ws)
    with pytest.raises(rba.RbaError) as e:
        st.check()
    assert e.value.status == rba.ERR_TIMEOUT
    st.check()  # the status word was cleared by the read
    # back to the default bound: the same workspace serves a correct step
    st.set_wait_limit_ns(0)
    ref = O.decode(x["q"], x["K"], x["V"], reps, dtype=w.dtype, block_size=w.block_size,
                   sink=w.sink, window=w.window, top_k_blocks=w.top_k)
    for _ in range(2):
        idx, out, lse = st.decode_step(q, w.top_k, w.context, w.sink, w.window, workspace=ws)
        st.check()
        check_decode_step(w, x["q"], x["K"], x["V"], ref, idx.cpu().numpy(),
                          out.cpu().numpy(), lse.cpu().numpy())
