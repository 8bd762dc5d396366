"""GPU parity of the dynamic memory update ("MemLong: Memory-Augmented Retrieval
for Long Text Modeling", section 2.3.2) through the C ABI: retrieval counters
(rba_count_retrievals), the counter-driven keep set and the in-place
compaction of the store (rba_memory_update), against the oracle's
memory_keep / memory_compact.  Everything here is integer or data movement:
the comparison is bit-exact.

Counter values follow a retrieval-frequency shape (most blocks rarely
retrieved, some often), with many ties and a few counts above 2^31 so that
every byte of the 32-bit threshold search is exercised."""
import zlib

import numpy as np
import pytest
import torch

import oracle as O
from retrieval_block_sparse_b200 import synth

from parity import OUT_TOL, dev, host_bits, out_error, selection_check

pytestmark = pytest.mark.gpu

CASES = {
    "mean-bf16": dict(mode="mean", dtype="bf16", B=1, Hkv=2, D=128, bs=64, r=1, d_ret=0,
                      nb=120, tail=17, pinned=1),
    "topr-f32": dict(mode="topr_attn", dtype="f32", B=2, Hkv=1, D=64, bs=16, r=2, d_ret=0,
                     nb=333, tail=0, pinned=0),
    "external-bf16": dict(mode="external", dtype="bf16", B=1, Hkv=3, D=64, bs=32, r=1, d_ret=0,
                          nb=77, tail=31, pinned=2),
    "cosine": dict(mode="embed_cosine", dtype="bf16", B=2, Hkv=2, D=128, bs=256, r=1, d_ret=48,
                   nb=40, tail=100, pinned=0),
    "identity-large": dict(mode="identity", dtype="bf16", B=1, Hkv=2, D=64, bs=1, r=1, d_ret=0,
                           nb=150000, tail=0, pinned=4),
}
EXTRA_BLOCKS = 3  # capacity beyond the held blocks: counters there must stay untouched


def _store(rba, c, rng):
    cap = (c["nb"] + EXTRA_BLOCKS) * c["bs"]
    st = rba.Store(batch=c["B"], n_q_heads=c["Hkv"], n_kv_heads=c["Hkv"], head_dim=c["D"],
                   block_size=c["bs"], capacity_tokens=cap, dtype=c["dtype"], mode=c["mode"],
                   n_rep=c["r"], d_ret=c["d_ret"])
    st.k.copy_(torch.randn(st.k.shape).to(st.k.dtype))
    st.v.copy_(torch.randn(st.v.shape).to(st.v.dtype))
    if st.rep is not None:
        st.rep.copy_(torch.randn(st.rep.shape).to(st.rep.dtype))
    if st.rep_pos is not None:
        st.rep_pos.copy_(torch.from_numpy(rng.integers(0, c["bs"], st.rep_pos.shape,
                                                       dtype=np.int32)))
    return st


def _bits(t):
    if t.dtype == torch.bfloat16:
        return t.cpu().view(torch.int16).numpy()
    return t.cpu().numpy()


COUNT_VARIANTS = {
    "rule": lambda n: O.memory_rule(n),
    "no-oldest": lambda n: (n // 10, 0, n // 2),
    "newest-only": lambda n: (n // 10, n // 10, n // 10),
    "whole-middle": lambda n: (n // 10, n // 10, n - n // 10),
    "keep-all": lambda n: (0, 0, n),
}


@pytest.mark.parametrize("variant", list(COUNT_VARIANTS))
@pytest.mark.parametrize("name", list(CASES))
def test_memory_update_matches_oracle(rba, name, variant):
    c = CASES[name]
    if variant in ("no-oldest", "keep-all") and c["nb"] > 1000:
        pytest.skip("one move launch per kept entry without dropped oldest entries")
    torch.manual_seed(11)
    rng = np.random.default_rng(zlib.crc32(f"{name}/{variant}".encode()))
    st = _store(rba, c, rng)
    U = st.memory_units()
    assert U == (c["B"] if c["mode"] == "embed_cosine" else c["B"] * c["Hkv"])
    counts = synth.retrieval_counts(zlib.crc32(name.encode()), U, st.cap_blocks, huge=0.01)
    counters = torch.from_numpy(counts.view(np.int32)).cuda()
    nb, bs, pinned, tail = c["nb"], c["bs"], c["pinned"], c["tail"]
    T = nb * bs + tail
    newest, oldest, total = COUNT_VARIANTS[variant](nb - pinned)

    K0, V0 = _bits(st.k), _bits(st.v)
    rep0 = None if st.rep is None else _bits(st.rep)
    pos0 = None if st.rep_pos is None else st.rep_pos.cpu().numpy()
    T_new, kmap = st.memory_update(T, counters, pinned_blocks=pinned, keep_newest=newest,
                                   drop_oldest=oldest, keep_total=total)
    st.check()
    assert T_new == (pinned + total) * bs + tail
    kmap = kmap.cpu().numpy()
    K1, V1 = _bits(st.k), _bits(st.v)
    rep1 = None if st.rep is None else _bits(st.rep)
    pos1 = None if st.rep_pos is None else st.rep_pos.cpu().numpy()
    cnt1 = counters.cpu().numpy().view(np.uint32)
    cosine = c["mode"] == "embed_cosine"
    for u in range(U):
        keep = O.memory_keep(counts[u].astype(np.int64), nb, pinned, newest, oldest, total)
        np.testing.assert_array_equal(kmap[u], keep)
        if cosine:      # the bank entry of batch row u carries every kv head
            kv = [K0[u], V0[u]]
            pb = [rep0[u]]
        else:
            b, h = divmod(u, c["Hkv"])
            kv = [K0[b, h], V0[b, h]]
            pb = [] if rep0 is None else [rep0[b, h]]
            if pos0 is not None:
                pb.append(pos0[b, h])
        t_ref, kv_ref, pb_ref, c_ref = O.memory_compact(
            keep, pinned=pinned, nb=nb, tail=tail, bs=bs, kv=kv, per_block=pb,
            counters=counts[u])
        assert t_ref == T_new
        got_kv = [K1[u], V1[u]] if cosine else [K1[b, h], V1[b, h]]
        for g, r in zip(got_kv, kv_ref):
            np.testing.assert_array_equal(g[..., :T_new, :], r[..., :T_new, :])
        new_nb = pinned + total
        if cosine:
            got_pb = [rep1[u]]
        else:
            got_pb = [] if rep1 is None else [rep1[b, h]]
            if pos1 is not None:
                got_pb.append(pos1[b, h])
        for g, r in zip(got_pb, pb_ref):
            np.testing.assert_array_equal(g[:new_nb], r[:new_nb])
        np.testing.assert_array_equal(cnt1[u], c_ref)


def test_count_retrievals_matches_oracle(rba):
    rng = np.random.default_rng(5)
    st = rba.Store(batch=2, n_q_heads=4, n_kv_heads=2, head_dim=64, block_size=16,
                   capacity_tokens=16 * 300, dtype="bf16", mode="mean")
    U, cap = st.memory_units(), st.cap_blocks
    counters = st.new_counters()
    ref = np.zeros((U, cap), dtype=np.int64)
    for step in range(6):                     # decode-shaped selections [B][Hkv][k]
        k = 8 + step
        idx = np.stack([np.sort(rng.choice(cap, k, replace=False)) for _ in range(U)])
        idx = idx.reshape(2, 2, k).astype(np.int32)
        st.count_retrievals(torch.from_numpy(idx).cuda(), counters)
        ref, bad = O.count_retrievals(idx, U, cap, ref)
        assert bad == 0
    # prefill-shaped: [n_chunks][n_sel = U][k], a million entries, heavy collisions
    idx = rng.integers(0, 40, size=(2000, U, 128)).astype(np.int32)
    st.count_retrievals(torch.from_numpy(idx).cuda(), counters)
    for u in range(U):
        ref[u] += np.bincount(idx[:, u].ravel(), minlength=cap)
    st.check()
    np.testing.assert_array_equal(counters.cpu().numpy().astype(np.int64), ref)


def test_count_retrievals_flags_out_of_range(rba):
    st = rba.Store(batch=1, n_q_heads=2, n_kv_heads=1, head_dim=64, block_size=16,
                   capacity_tokens=16 * 10, dtype="bf16", mode="mean")
    counters = st.new_counters()
    idx = torch.tensor([[0, 3, 10, -1, 9]], dtype=torch.int32, device="cuda")
    st.count_retrievals(idx, counters)
    with pytest.raises(rba.RbaError) as e:
        st.check()
    assert e.value.status == rba.ERR_BOUNDS
    ref = np.zeros(10, dtype=np.int64)
    ref[[0, 3, 9]] = 1
    np.testing.assert_array_equal(counters.cpu().numpy()[0], ref)


def test_decode_count_update_decode_matches_oracle(rba):
    """Decode steps feed the counters; the update prunes the store; decoding
    continues on the compacted store.  The oracle runs the same sequence on
    its own selections and its own compacted copy, with representations
    recomputed from the moved keys."""
    w = synth.WORKLOADS["infllm-decode-128k"].scaled(
        batch=1, n_q_heads=4, n_kv_heads=2, context=1024, block_size=16, n_rep=1,
        rep_mode="mean", top_k=6, sink=16, window=64, recipe="normal", seed=41)
    x = synth.decode_inputs(w)
    st = rba.Store(batch=1, n_q_heads=4, n_kv_heads=2, head_dim=w.head_dim, block_size=16,
                   capacity_tokens=1024, dtype="bf16", mode="mean")
    st.k.copy_(dev(x["K"], "bf16"))
    st.v.copy_(dev(x["V"], "bf16"))
    st.memorize(None, None, first_block=0, n_blocks=64)
    rng = np.random.default_rng(42)
    counters = st.new_counters()
    K, V = x["K"].copy(), x["V"].copy()
    T, pinned, k = 1024, 1, w.top_k
    cnt = np.zeros((2, st.cap_blocks), dtype=np.int64)

    def step(T, K, V, cnt):
        q = synth.bf16_round(rng.standard_normal((1, 4, w.head_dim)))
        reps = np.stack([O.memorize(O.widen(K[0, h, :(T // 16) * 16], "bf16"), "mean", 16)[0]
                         for h in range(2)])[None]
        ref = O.decode(q, K[:, :, :T], V[:, :, :T], reps, dtype="bf16", block_size=16,
                       sink=w.sink, window=w.window, top_k_blocks=k)
        idx, out, _ = st.decode_step(dev(q, "bf16"), k, T, w.sink, w.window)
        st.count_retrievals(idx, counters)
        got = idx.cpu().numpy()
        for h in range(2):
            assert selection_check(ref["scores"][0, h], k, int(ref["cand"][0]), got[0, h]) == \
                "exact"
        vmax = np.abs(O.widen(V[0, :, :T], "bf16")).max()
        assert out_error(out.cpu().numpy(), ref["out"], np.array([vmax])) <= OUT_TOL["bf16"]
        cnt, _ = O.count_retrievals(ref["idx"], 2, st.cap_blocks, cnt)
        return cnt

    for _ in range(12):
        cnt = step(T, K, V, cnt)
    st.check()
    np.testing.assert_array_equal(counters.cpu().numpy().astype(np.int64), cnt)

    T_new, kmap = st.memory_update(T, counters, pinned_blocks=pinned)
    st.check()
    nb = T // 16
    newest, oldest, total = O.memory_rule(nb - pinned)
    K2, V2 = K.copy(), V.copy()
    for h in range(2):
        keep = O.memory_keep(cnt[h], nb, pinned, newest, oldest, total)
        np.testing.assert_array_equal(kmap.cpu().numpy()[h], keep)
        t_ref, (k2, v2), _, c2 = O.memory_compact(keep, pinned=pinned, nb=nb, tail=0, bs=16,
                                                  kv=[K[0, h], V[0, h]], counters=cnt[h])
        K2[0, h], V2[0, h], cnt[h] = k2, v2, c2
        assert t_ref == T_new
    np.testing.assert_array_equal(host_bits(st.k, "bf16")[:, :, :T_new], K2[:, :, :T_new])
    np.testing.assert_array_equal(counters.cpu().numpy().astype(np.int64), cnt)
    for _ in range(6):
        cnt = step(T_new, K2, V2, cnt)
    st.check()
    np.testing.assert_array_equal(counters.cpu().numpy().astype(np.int64), cnt)


@pytest.mark.parametrize("name", ["infllm-decode-128k", "memlong-cosine-prefill"])
def test_memory_update_full_size(rba, name):
    """The update of the full 128K store (8 kv heads x 1023 blocks after the
    sink) and of the full MemLong bank (160 chunks x 512 tokens x 32 heads),
    with the counters, rule and launch configuration the bench times.  Keep
    maps equal the oracle's memory_keep entry for entry; on sampled
    destinations (the first and last three and 40 drawn at random per unit)
    K, V, representation, positions and counter hold the bits of their source
    block; vacated counters are zero and the pinned blocks are untouched."""
    w = synth.WORKLOADS[name]
    cosine = getattr(w, "score_mode", "dot") == "cosine"
    if cosine:
        mode, r, d_ret, batch = "embed_cosine", 1, w.d_ret, 1
    else:
        mode, r, d_ret, batch = w.rep_mode, w.n_rep, 0, w.batch
    st = rba.Store(batch=batch, n_q_heads=w.n_q_heads, n_kv_heads=w.n_kv_heads,
                   head_dim=w.head_dim, block_size=w.block_size, capacity_tokens=w.context,
                   dtype=w.dtype, mode=mode, n_rep=r, d_ret=d_ret)
    gen = torch.Generator(device="cuda").manual_seed(w.seed)
    for t in (st.k, st.v, st.rep):
        if t is not None:
            t.copy_(torch.randn(t.shape, generator=gen, device="cuda", dtype=torch.float32))
    if st.rep_pos is not None:
        st.rep_pos.random_(0, w.block_size, generator=gen)
    U = st.memory_units()
    counts = synth.retrieval_counts(w.seed, U, st.cap_blocks)
    counters = torch.from_numpy(counts.view(np.int32)).cuda()
    T, bs = w.context, w.block_size
    nb = T // bs
    pinned = -(-w.sink // bs) if w.sink else 0
    newest, oldest, total = O.memory_rule(nb - pinned)
    before = [t.clone() for t in (st.k, st.v, st.rep, st.rep_pos) if t is not None]
    T_new, kmap = st.memory_update(T, counters, pinned_blocks=pinned)
    st.check()
    assert T_new == (pinned + total) * bs + (T - nb * bs)
    kmap = kmap.cpu().numpy()
    cnt1 = counters.cpu().numpy().view(np.uint32)
    after = [t for t in (st.k, st.v, st.rep, st.rep_pos) if t is not None]
    rng = np.random.default_rng(w.seed)
    bits = lambda t: t.view(torch.int16) if t.dtype == torch.bfloat16 else t  # noqa: E731
    for u in range(U):
        keep = O.memory_keep(counts[u].astype(np.int64), nb, pinned, newest, oldest, total)
        np.testing.assert_array_equal(kmap[u], keep)
        sample = sorted(set([0, 1, 2, total - 3, total - 2, total - 1]) |
                        set(rng.integers(0, total, 40).tolist()))
        b, h = (u, slice(None)) if cosine else divmod(u, w.n_kv_heads)
        for t in sample:
            src, dst = int(keep[t]), pinned + t
            for a0, a1 in zip(before[:2], after[:2]):  # K, V rows of the block
                assert torch.equal(bits(a1[b, h, dst * bs:(dst + 1) * bs]),
                                   bits(a0[b, h, src * bs:(src + 1) * bs])), (u, t)
            for a0, a1 in zip(before[2:], after[2:]):  # representation, positions
                ix = (b, dst) if cosine else (b, h, dst)
                jx = (b, src) if cosine else (b, h, src)
                assert torch.equal(bits(a1[ix]), bits(a0[jx])), (u, t)
            assert cnt1[u, dst] == counts[u, src], (u, t)
        assert not cnt1[u, pinned + total:nb].any()
        for j in range(pinned):
            for a0, a1 in zip(before[:2], after[:2]):
                assert torch.equal(bits(a1[b, h, j * bs:(j + 1) * bs]),
                                   bits(a0[b, h, j * bs:(j + 1) * bs]))
