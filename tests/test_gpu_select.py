"""GPU top-k against the oracle's top_k on identical fp32 score rows:
bit-exact, ties included (both decide on the same fp32 values)."""
import numpy as np
import pytest
import torch

import oracle as O
from retrieval_block_sparse_b200 import synth

pytestmark = pytest.mark.gpu


def _run(rba, s, k, base=0):
    t = torch.from_numpy(s).cuda()
    return rba.topk(t, k, index_base=base).cpu().numpy()


@pytest.mark.parametrize("n,k,ties", [(1, 1, 0), (2, 1, 0), (61, 4, 0), (991, 32, 0),
                                      (991, 32, 5), (1000, 1000, 3), (4096, 4096, 0),
                                      (8192, 100, 2), (5000, 1, 0), (7, 7, 1),
                                      (8193, 2048, 0), (16383, 256, 3), (16384, 2048, 0)])
def test_topk_small_rows(rba, n, k, ties):
    s = synth.random_scores(20 + n + k, 6, n, ties=ties)
    got = _run(rba, s, k, base=3)
    for r in range(s.shape[0]):
        np.testing.assert_array_equal(got[r], O.top_k(s[r].astype(np.float64), k) + 3)


@pytest.mark.parametrize("n,k,ties", [(16385, 2048, 0), (65536, 256, 0), (1 << 20, 2048, 0),
                                      (100000, 2048, 4), (50000, 16384, 0), (16400, 16384, 0)])
def test_topk_large_rows(rba, n, k, ties):
    s = synth.random_scores(7 + k, 3, n, ties=ties)
    got = _run(rba, s, k)
    for r in range(s.shape[0]):
        np.testing.assert_array_equal(got[r], O.top_k(s[r].astype(np.float64), k))


@pytest.mark.parametrize("n,k", [(1024, 600), (1024, 1), (700, 69), (33, 32), (991, 32),
                                 (129, 128)])
def test_topk_warp_rows_skewed_and_tied(rba, n, k):
    # rows of at most 1024 scores are selected by one warp: cover a value
    # range dominated by a few outliers (crowded boundary bin), two-level ties
    # (radix path), infinities (radix path) and plain normal rows
    rng = np.random.default_rng(n * 7 + k)
    rows = [rng.standard_normal(n),
            np.where(rng.random(n) < 0.02, 1e4, rng.standard_normal(n) * 1e-3),
            rng.integers(0, 2, n).astype(np.float64),
            np.where(rng.random(n) < 0.05, np.inf, rng.standard_normal(n)),
            np.where(rng.random(n) < 0.05, -np.inf, rng.standard_normal(n))]
    s = np.stack(rows).astype(np.float32)
    got = _run(rba, s, k, base=11)
    for r in range(s.shape[0]):
        np.testing.assert_array_equal(got[r], O.top_k(s[r].astype(np.float64), k) + 11)


def test_topk_signed_zero_and_constant_rows(rba):
    s = np.zeros((2, 300), dtype=np.float32)
    s[0, ::2] = -0.0
    s[1, 50] = 1.0
    got = _run(rba, s, 5)
    assert got[0].tolist() == [0, 1, 2, 3, 4]
    assert got[1].tolist() == [0, 1, 2, 3, 50]
    big = np.zeros((1, 20000), dtype=np.float32)  # all tied, radix path
    assert _run(rba, big, 7)[0].tolist() == list(range(7))


def test_topk_rejects_k_above_n(rba):
    with pytest.raises(rba.RbaError):
        _run(rba, np.zeros((1, 5), dtype=np.float32), 6)
