"""Shared helpers of the GPU parity tests: moving seeded inputs to the device,
building stores, running the oracle on the same inputs, and the acceptance
rules.

Tolerances (stated by the method's accuracy target):
  * attention outputs: max |o_gpu - o_ref| / max |V over the attended set|
    <= 2e-3 for bf16 inputs, 1e-5 for fp32 inputs;
  * selections: bit-exact, except where the oracle's k-th and (k+1)-th scores
    differ by less than 1e-5 relative -- there either choice is accepted, and
    only indices inside that near-tie may differ; the outputs of such a unit
    are compared with the oracle evaluated on the GPU's own selection, so
    every unit is checked against the oracle;
  * scores (no stated bound; derived from fp32 accumulation of n products):
    |s_gpu - s_ref| <= 1e-5 * sum |products|, about 10x the expected fp32
    rounding of an n <= 2048 term dot product.
"""
import math

import numpy as np
import torch

import oracle as O

OUT_TOL = {"bf16": 2e-3, "f32": 1e-5}
SEL_REL = 1e-5


def dev(x, dtype):
    """Stored numpy array -> CUDA tensor of the store dtype (same bits)."""
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()


def host_bits(t, dtype):
    if dtype == "bf16":
        return t.detach().cpu().view(torch.int16).numpy().view(np.uint16)
    return t.detach().cpu().numpy()


def make_decode_store(rba, w, x, one_launch=False):
    """Store holding the whole context of workload w, representations memorised;
    one_launch lets its decode step run as one cooperative launch."""
    st = rba.Store(batch=w.batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                   head_dim=w.head_dim, block_size=w.block_size, capacity_tokens=w.context,
                   dtype=w.dtype, mode=w.rep_mode, n_rep=w.n_rep)
    if one_launch:
        st.set_decode_step_one_launch(True)
    st.kv_rows(st.k).copy_(dev(x["K"], w.dtype))  # (pool rows may be padded past D)
    st.kv_rows(st.v).copy_(dev(x["V"], w.dtype))
    aux = None
    if w.rep_mode == "topr_attn":
        aux = dev(x["probe"], w.dtype)
    elif w.rep_mode == "external":
        aux = dev(x["landmarks"], w.dtype).reshape(w.batch, w.n_kv_heads, w.n_blocks, 1,
                                                    w.head_dim)
    st.memorize(None, None, first_block=0, n_blocks=w.n_blocks, aux=aux)
    return st


def oracle_reps(w, x):
    """Oracle representations [B][Hkv][nb][r][D] (fp64) and top-r positions."""
    if w.rep_mode == "identity":
        return None, None
    B, Hkv, nb, r, D = w.batch, w.n_kv_heads, w.n_blocks, w.n_rep, w.head_dim
    reps = np.zeros((B, Hkv, nb, r, D))
    pos = np.zeros((B, Hkv, nb, r), dtype=np.int64) if w.rep_mode == "topr_attn" else None
    probe = O.widen(x["probe"], w.dtype) if w.rep_mode == "topr_attn" else None
    for b in range(B):
        for h in range(Hkv):
            if w.rep_mode == "external":
                reps[b, h, :, 0] = O.widen(x["landmarks"][b, h], w.dtype)
                continue
            K = O.widen(x["K"][b, h, :nb * w.block_size], w.dtype)
            rr, ch = O.memorize(K, w.rep_mode, w.block_size, r,
                                probe=None if probe is None else probe[h])
            reps[b, h] = rr
            if pos is not None:
                pos[b, h] = ch
    return reps, pos


def selection_check(s_ref, k, first, gpu_idx):
    """Returns 'exact' or 'tie' (accepted near-tie swap); raises on mismatch.

    s_ref: oracle scores of the candidates (fp64), first: block id of
    candidate 0, gpu_idx: the GPU's k block ids (ascending)."""
    n = s_ref.shape[0]
    ref = (O.top_k(s_ref, k) + first).tolist()
    got = [int(i) for i in gpu_idx]
    if got == ref:
        return "exact"
    assert len(set(got)) == k and got == sorted(got), f"not k distinct ascending: {got}"
    assert all(first <= j < first + n for j in got), "index outside the candidates"
    order = np.sort(s_ref)[::-1]
    sk = order[k - 1]
    sk1 = order[k] if k < n else -np.inf
    tol = SEL_REL * max(abs(sk), abs(sk1), 1e-30)
    assert sk - sk1 < tol, f"selection differs without a near-tie: {sorted(set(got) ^ set(ref))}"
    for j in set(got) ^ set(ref):
        assert abs(s_ref[j - first] - sk) <= tol, f"index {j} not part of the near-tie"
    return "tie"


def out_error(o_gpu, o_ref, v_att):
    return float(np.max(np.abs(o_gpu - o_ref)) / max(float(np.max(np.abs(v_att))), 1e-30))


def attended_v_max(w, x, b, h, sel):
    toks = O.attended_tokens(w.context, w.block_size, w.sink, w.window, sel)
    return O.widen(x["V"][b, h, toks], w.dtype)


def score_tolerance(qsum_abs, reps_abs):
    """1e-5 * sum |q . rep| products for every candidate: [nc]."""
    return 1e-5 * (reps_abs @ qsum_abs).reshape(reps_abs.shape[0], -1).sum(axis=1)


def scale_of(w):
    return 1.0 / math.sqrt(w.head_dim)


def check_decode_step(w, q, K, V, ref, idx, out, lse, *, T=None, k=None, min_exact=0.9):
    """Acceptance of a whole decode step against the oracle, per (b, kv head).

    The GPU selection idx[b, h] must equal the oracle's, or be an accepted
    near-tie swap (selection_check).  Every q head's output and lse are then
    compared with the oracle's attention over the GPU-chosen token set: for an
    exact selection that is ref["out"] / ref["lse"]; for a near-tie swap the
    oracle's softmax_attention is evaluated on the attended tokens of the
    GPU's blocks.  q, K, V: the stored inputs (numpy, store dtype bits).
    Returns the number of units whose selection matched exactly; at least
    min_exact of them must (near-ties are rare on these inputs)."""
    T = w.context if T is None else T
    k = w.top_k if k is None else k
    g = w.n_q_heads // w.n_kv_heads
    scale = scale_of(w)
    tol = OUT_TOL[w.dtype]
    first = int(ref["cand"][0]) if ref["cand"].size else 0
    exact = 0
    for b in range(w.batch):
        for h in range(w.n_kv_heads):
            kind = selection_check(ref["scores"][b, h], k, first, idx[b, h])
            toks = O.attended_tokens(T, w.block_size, w.sink, w.window, idx[b, h])
            Kt = O.widen(K[b, h, toks], w.dtype)
            Vt = O.widen(V[b, h, toks], w.dtype)
            for i in range(h * g, (h + 1) * g):
                if kind == "exact":
                    o_ref, l_ref = ref["out"][b, i], ref["lse"][b, i]
                else:
                    o_ref, l_ref, _ = O.softmax_attention(O.widen(q[b, i], w.dtype), Kt, Vt,
                                                          scale)
                err = out_error(out[b, i], o_ref, Vt)
                assert err <= tol, (b, h, i, kind, err)
                assert abs(lse[b, i] - l_ref) <= tol, (b, h, i, kind, lse[b, i], l_ref)
            exact += kind == "exact"
    assert exact >= min_exact * w.batch * w.n_kv_heads
    return exact
