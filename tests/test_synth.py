"""The seeded generators: determinism, rounding, recipe structure."""
import numpy as np

from retrieval_block_sparse_b200 import synth


def _rne_reference(x):
    """bf16 round-to-nearest-even written from the definition: keep the upper
    16 bits, add one ulp when the dropped half is > 1/2 ulp or == 1/2 ulp with
    an odd kept part."""
    u = x.astype(np.float32).view(np.uint32)
    hi = u >> 16
    lo = u & 0xFFFF
    up = (lo > 0x8000) | ((lo == 0x8000) & ((hi & 1) == 1))
    return (hi + up).astype(np.uint16)


def test_bf16_round_is_nearest_even():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.normal(size=100000).astype(np.float32),
                        # exact halfway cases, both parities
                        np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, -(1 + 2 ** -8), 0.0, -0.0],
                                 dtype=np.float32)])
    np.testing.assert_array_equal(synth.bf16_round(x), _rne_reference(x))
    back = synth.bf16_to_f32(synth.bf16_round(x))
    assert np.all(np.abs(back - x) <= np.abs(x) * 2 ** -8 + 1e-38)


def test_generators_are_deterministic_and_seeded():
    w = synth.WORKLOADS["infllm-decode-128k"].scaled(context=4096, window=512)
    a = synth.decode_inputs(w)
    b = synth.decode_inputs(w)
    for k in a:
        np.testing.assert_array_equal(a[k], b[k])
    c = synth.decode_inputs(w.scaled(seed=99))
    assert not np.array_equal(a["K"], c["K"])


def test_shapes_and_dtypes():
    w = synth.WORKLOADS["landmark-decode-b16"].scaled(batch=2, n_q_heads=3, n_kv_heads=3,
                                                      context=1000)
    x = synth.decode_inputs(w)
    assert x["K"].shape == (2, 3, 1000, 128) and x["K"].dtype == np.uint16
    assert x["landmarks"].shape == (2, 3, 20, 128)
    assert x["q"].shape == (2, 3, 128)
    w1 = synth.WORKLOADS["tiny-decode-f32"]
    x1 = synth.decode_inputs(w1)
    assert x1["K"].dtype == np.float32 and x1["K"].shape == (1, 4, 4096, 64)
    p = synth.prefill_inputs(synth.WORKLOADS["memlong-cosine-prefill"].scaled(
        context=8 * 512, chunk_len=16, n_q_heads=2, n_kv_heads=2))
    assert p["bank_embed"].shape == (8, 768) and p["query_embed"].shape == (8, 768)
    assert p["Q"].shape == (8, 2, 16, 128) and p["chunk_K"].shape == (8, 2, 16, 128)


def test_shifted_query_distribution():
    w = synth.WORKLOADS["token-retrieval-decode-1m"].scaled(context=2048, n_q_heads=256,
                                                            n_kv_heads=8)
    x = synth.decode_inputs(w)
    q = synth.bf16_to_f32(x["q"])
    assert abs(q.mean() - 0.5) < 0.045 and abs(q.std() - 1.5) < 0.03
    k = synth.bf16_to_f32(x["K"])
    assert abs(k.mean()) < 0.01 and abs(k.std() - 1) < 0.01


def test_random_scores_ties():
    s = synth.random_scores(3, 4, 500, ties=7)
    for row in s:
        assert len(np.unique(row)) <= 7
