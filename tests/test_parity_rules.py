"""The acceptance rules of the GPU parity tests (tests/parity.py), exercised on
the CPU with outputs made by the oracle itself.

Where two candidate blocks score exactly the same at the k-th place, either
one is a correct selection.  check_decode_step must then compare the step's
output with the oracle evaluated on the selection actually made (not skip
the unit), and reject a selection that differs outside such a near-tie."""
import numpy as np
import pytest

import oracle as O
from retrieval_block_sparse_b200 import synth

from parity import check_decode_step, selection_check


def _tied_case():
    w = synth.WORKLOADS["tiny-decode-f32"].scaled(n_q_heads=2, n_kv_heads=1, head_dim=8,
                                                  context=512, block_size=32, sink=32,
                                                  window=64, top_k=3, seed=41)
    x = synth.decode_inputs(w)
    K = O.widen(x["K"][0, 0], "f32")
    reps = O.memorize(K, "mean", w.block_size)[0][None, None]
    ref = O.decode(x["q"], x["K"], x["V"], reps, dtype="f32", block_size=w.block_size,
                   sink=w.sink, window=w.window, top_k_blocks=w.top_k)
    # give the best unselected candidate the representation of the k-th
    # selected block: an exact tie at the k-th place, broken by the index
    cand, s = ref["cand"], ref["scores"][0, 0]
    order = np.lexsort((np.arange(s.size), -s))
    kth, nxt = cand[order[w.top_k - 1]], cand[order[w.top_k]]
    reps[0, 0, nxt] = reps[0, 0, kth]
    ref = O.decode(x["q"], x["K"], x["V"], reps, dtype="f32", block_size=w.block_size,
                   sink=w.sink, window=w.window, top_k_blocks=w.top_k)
    lo, hi = min(kth, nxt), max(kth, nxt)
    assert lo in ref["idx"][0, 0] and hi not in ref["idx"][0, 0]
    swapped = np.sort(np.array([j for j in ref["idx"][0, 0] if j != lo] + [hi]))
    return w, x, ref, swapped


def _oracle_outputs(w, x, sel):
    """out / lse of every q head over sink U sel U window (oracle)."""
    toks = O.attended_tokens(w.context, w.block_size, w.sink, w.window, sel)
    Kt, Vt = O.widen(x["K"][0, 0, toks], "f32"), O.widen(x["V"][0, 0, toks], "f32")
    out = np.zeros((1, w.n_q_heads, w.head_dim))
    lse = np.zeros((1, w.n_q_heads))
    for i in range(w.n_q_heads):
        out[0, i], lse[0, i], _ = O.softmax_attention(O.widen(x["q"][0, i], "f32"), Kt, Vt,
                                                      w.head_dim ** -0.5)
    return out, lse


def test_tie_swap_is_accepted_and_checked_on_its_own_selection():
    w, x, ref, swapped = _tied_case()
    first = int(ref["cand"][0])
    assert selection_check(ref["scores"][0, 0], w.top_k, first, swapped) == "tie"
    out, lse = _oracle_outputs(w, x, swapped)
    n = check_decode_step(w, x["q"], x["K"], x["V"], ref, swapped[None, None], out, lse,
                          min_exact=0)
    assert n == 0
    # outputs of the oracle's selection do not pass for the swapped one
    with pytest.raises(AssertionError):
        check_decode_step(w, x["q"], x["K"], x["V"], ref, swapped[None, None], ref["out"],
                          ref["lse"], min_exact=0)
    # nor does an output off by more than the tolerance
    bad = out.copy()
    bad[0, 1, 3] += 3e-5 * np.abs(O.widen(x["V"], "f32")).max()
    with pytest.raises(AssertionError):
        check_decode_step(w, x["q"], x["K"], x["V"], ref, swapped[None, None], bad, lse,
                          min_exact=0)


def test_exact_selection_is_compared_with_the_oracle_step():
    w, x, ref, _ = _tied_case()
    n = check_decode_step(w, x["q"], x["K"], x["V"], ref, ref["idx"], ref["out"], ref["lse"])
    assert n == 1
    bad = ref["lse"].copy()
    bad[0, 0] += 1e-4
    with pytest.raises(AssertionError):
        check_decode_step(w, x["q"], x["K"], x["V"], ref, ref["idx"], ref["out"], bad)


def test_swap_outside_a_near_tie_is_rejected():
    w, x, ref, _ = _tied_case()
    s = ref["scores"][0, 0]
    worst = ref["cand"][int(np.argmin(s))]
    sel = np.sort(np.array(list(ref["idx"][0, 0][1:]) + [worst]))
    out, lse = _oracle_outputs(w, x, sel)
    with pytest.raises(AssertionError):
        check_decode_step(w, x["q"], x["K"], x["V"], ref, sel[None, None], out, lse,
                          min_exact=0)
