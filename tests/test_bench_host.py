"""Host-side logic of bench.py, on CPU: size bookkeeping, the max-over-ranks
reduction on two gloo ranks, the traffic lookup, and the reference arm's
JSON line."""
import io
import json
import os
import contextlib

import numpy as np
import pytest
import torch.multiprocessing as mp

import bench
import oracle as O


def test_attended_counts_match_oracle():
    rng = np.random.default_rng(0)
    for T, bs, S, W, k in [(32768, 50, 0, 256, 4), (131072, 128, 128, 4096, 32),
                           (1000, 24, 30, 70, 7), (4096, 64, 64, 128, 4)]:
        cand = O.candidate_blocks(T, bs, S, W)
        idx = np.stack([np.sort(rng.choice(cand, k, replace=False)) for _ in range(6)])[None]
        got = bench.attended_counts(idx, T, bs, S, W)
        for i in range(6):
            assert got[0, i] == O.attended_tokens(T, bs, S, W, idx[0, i]).shape[0]


def _rank(rank, world, port, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    q.put((rank, bench.reduce_max(1.5 + rank, "cpu")))
    dist.destroy_process_group()


def test_reduce_max_over_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    ps = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in ps:
        p.start()
    for p in ps:
        p.join(120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert got == [(0, 2.5), (1, 2.5)]
    assert bench.reduce_max(3.25, "cpu") == 3.25  # no process group: identity


def test_traffic_lookup_requires_current_source(tmp_path):
    p = tmp_path / "t.txt"
    h = bench.source_hash("attend_decode_kernel")
    p.write_text(f"# kernel sha workload bytes\nattend_decode_kernel {h} w1 1234\n"
                 f"attend_decode_kernel 0000000000000000 w2 99\n")
    assert bench.traffic_lookup("attend_decode_kernel", "w1", str(p)) == 1234.0
    assert bench.traffic_lookup("attend_decode_kernel", "w2", str(p)) is None
    assert bench.traffic_lookup("attend_decode_kernel", "w3", str(p)) is None


def test_reference_arm_line():
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.main(["--impl", "reference", "--steps", "6", "--warmup", "1",
                    "--workload", "tiny-decode-f32"])
    line = json.loads(buf.getvalue().strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["value"] > 0
    assert line["unit"] == bench.UNIT and line["metric"] == bench.METRIC
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1


def test_prefill_pairs_match_brute_force_and_published_sizes():
    from retrieval_block_sparse_b200 import synth
    W = synth.WORKLOADS
    # brute force on a tiny case: count (row, key) pairs of the oracle's own
    # attended-token rule (past set per selection) plus the causal chunk
    w = W["token-retrieval-prefill-1m"].scaled(n_chunks=2, n_q_heads=4, n_kv_heads=2,
                                               chunk_len=5, context=200, block_size=10,
                                               sink=7, window=23, top_k=3)
    rng = np.random.default_rng(0)
    first = w.sink // w.block_size
    nc = -(-(w.context - w.window) // w.block_size) - first
    idx = np.stack([np.stack([np.sort(rng.choice(nc, 3, replace=False)) + first
                              for _ in range(w.n_kv_heads)]) for _ in range(w.n_chunks)])
    brute = 0
    for c in range(w.n_chunks):
        for hq in range(w.n_q_heads):
            toks = O.attended_tokens(w.context, w.block_size, w.sink, w.window,
                                     idx[c, hq // (w.n_q_heads // w.n_kv_heads)])
            for i in range(w.chunk_len):
                brute += len(toks) + i + 1
    assert bench.prefill_pairs(w, idx) == brute
    # the two full prefill workloads: 4 x 512 retrieved tokens shared by all
    # heads; 128 sink + 2048 single tokens + 512 window per kv head
    c2 = W["memlong-cosine-prefill"]
    idx2 = np.tile(np.arange(4), (c2.n_chunks, 1, 1))
    assert bench.prefill_pairs(c2, idx2) == 8 * 32 * (512 * 2048 + 512 * 513 // 2)
    c5 = W["token-retrieval-prefill-1m"]
    idx5 = np.tile(np.arange(128, 128 + 2048), (1, c5.n_kv_heads, 1))
    assert bench.prefill_pairs(c5, idx5) == 32 * (2048 * 2688 + 2048 * 2049 // 2)


def test_kernel_source_hash_ignores_comments_only():
    import bench
    code = "int f(int x) {\n  return x + 1;  // one more\n}\n/* block\n comment */\n"
    same = "// header\nint f(int x) {\n  return x + 1;\n}\n"
    other = "int f(int x) {\n  return x + 2;\n}\n"
    assert bench._code_only(code) == bench._code_only(same)
    assert bench._code_only(code) != bench._code_only(other)
