"""The C-ABI library: it loads without a GPU, exports every symbol the header
declares, and its host-only logic (argument checks, candidate geometry,
workspace sizes) behaves as documented.  No kernel is launched here."""
import ctypes
import os
import re

import pytest

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rba.h")


@pytest.fixture(scope="module")
def L():
    from retrieval_block_sparse_b200 import build
    build.build()
    import retrieval_block_sparse_b200 as m
    return m.lib()


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(rba_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(L):
    import retrieval_block_sparse_b200 as m
    names = _declared()
    assert len(names) >= 15
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(m.SIGNATURES), set(names) ^ set(m.SIGNATURES)


def test_status_strings_and_version(L):
    assert L.rba_status_string(0) == b"ok"
    assert L.rba_status_string(3) == b"workspace too small"
    assert L.rba_version() >= 100


class _Desc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("block_size", ctypes.c_int32), ("n_rep", ctypes.c_int32),
                ("d_ret", ctypes.c_int32), ("capacity_tokens", ctypes.c_int64),
                ("dtype", ctypes.c_int32), ("mode", ctypes.c_int32)]


FAKE = ctypes.c_void_p(0x10000)  # never dereferenced: nothing is launched


def _create(L, **kw):
    d = dict(batch=1, n_q_heads=4, n_kv_heads=2, head_dim=128, block_size=16, n_rep=1, d_ret=0,
             capacity_tokens=1024, dtype=1, mode=0)
    d.update(kw)
    h = ctypes.c_void_p()
    s = L.rba_store_create(ctypes.byref(_Desc(**d)), FAKE, FAKE, FAKE, None, None,
                           ctypes.byref(h))
    return s, h


def test_store_create_validates(L):
    s, h = _create(L)
    assert s == 0 and h.value
    L.rba_store_destroy(h)
    assert _create(L, head_dim=130)[0] == 2         # head dim above the 128-element row
    assert _create(L, head_dim=98)[0] == 2          # not a multiple of 4
    for hd, pitch in ((64, 64), (128, 128), (100, 128), (96, 128), (48, 64)):
        s, h = _create(L, head_dim=hd)               # held in rows of the pitch
        assert s == 0 and L.rba_row_pitch(hd) == pitch, hd
        L.rba_store_destroy(h)
    assert _create(L, n_q_heads=3)[0] == 1          # Hq not a multiple of Hkv
    assert _create(L, mode=4)[0] == 1               # identity needs block size 1
    assert _create(L, mode=4, block_size=1)[0] == 0
    assert _create(L, mode=1, n_rep=17)[0] == 1     # more rep keys than tokens
    assert _create(L, mode=3, d_ret=0)[0] == 1      # embedding size missing
    assert _create(L, capacity_tokens=0)[0] == 1


@pytest.mark.parametrize("T,bs,S,W", [(4096, 64, 64, 128), (131072, 128, 128, 4096),
                                      (32768, 50, 0, 256), (1 << 20, 1, 128, 512),
                                      (81920, 512, 0, 0), (37, 5, 3, 7), (40, 8, 8, 8),
                                      (41, 8, 9, 2), (12, 4, 20, 0), (16, 4, 0, 16),
                                      (100, 10, 95, 10), (50, 7, 6, 13), (0, 4, 0, 0)])
def test_candidate_geometry_matches_oracle(L, T, bs, S, W):
    s, h = _create(L, block_size=bs, capacity_tokens=max(T, 1) + 64,
                   mode=4 if bs == 1 else 0)
    assert s == 0
    f, n = ctypes.c_int32(), ctypes.c_int32()
    st = L.rba_candidates(h, T, S, W, ctypes.byref(f), ctypes.byref(n))
    cand = O.candidate_blocks(T, bs, S, W)
    if T - (T // bs) * bs > W:
        assert st == 1
    else:
        assert st == 0
        assert n.value == cand.shape[0]
        if n.value:
            assert f.value == cand[0]
    L.rba_store_destroy(h)


def test_tail_outside_window_is_rejected(L):
    s, h = _create(L, block_size=50, capacity_tokens=40000)
    f, n = ctypes.c_int32(), ctypes.c_int32()
    assert L.rba_candidates(h, 32768, 0, 10, ctypes.byref(f), ctypes.byref(n)) == 1
    assert L.rba_candidates(h, 32768, 0, 18, ctypes.byref(f), ctypes.byref(n)) == 0
    assert L.rba_candidates(h, 50000, 0, 18, ctypes.byref(f), ctypes.byref(n)) == 1  # > capacity
    L.rba_store_destroy(h)


def test_host_argument_checks_launch_nothing(L):
    s, h = _create(L)
    # k larger than the candidate count
    assert L.rba_attend(h, FAKE, FAKE, 1000, 1024, 0, 0, ctypes.c_float(0.1), FAKE, None, FAKE,
                        ctypes.c_size_t(1 << 20), None) == 1
    # workspace too small
    assert L.rba_attend(h, FAKE, FAKE, 4, 1024, 0, 0, ctypes.c_float(0.1), FAKE, None, FAKE,
                        ctypes.c_size_t(8), None) == 3
    assert L.rba_topk(FAKE, 2, 10, 11, 0, FAKE, None, ctypes.c_size_t(0), None) == 1
    assert L.rba_memorize(h, FAKE, None, 0, 1, None, 0, ctypes.c_float(1), None) == 1
    L.rba_store_destroy(h)


def test_workspace_sizes_are_positive(L):
    s, h = _create(L)
    assert L.rba_attend_workspace_size(h, 8, 1024, 16, 64) > 0
    assert L.rba_decode_step_workspace_size(h, 8, 1024, 16, 64) > 0
    assert L.rba_topk_workspace_size(8, 1 << 20, 2048) > 8 * (1 << 20) * 8
    assert L.rba_topk_workspace_size(8, 1000, 32) == 0
    L.rba_store_destroy(h)


def test_memory_rule_matches_oracle(L):
    a, b, c = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
    for n in list(range(0, 64)) + [99, 100, 101, 7936, 1 << 20, (1 << 31) - 3]:
        assert L.rba_memory_rule(n, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)) == 0
        assert (a.value, b.value, c.value) == O.memory_rule(n)
    assert L.rba_memory_rule(-1, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)) == 1


def test_memory_units_per_mode(L):
    s, h = _create(L, batch=3, n_kv_heads=2, n_q_heads=4)
    assert L.rba_memory_units(h) == 6
    L.rba_store_destroy(h)
    s, h = _create(L, batch=3, n_kv_heads=2, n_q_heads=4, mode=3, d_ret=32)
    assert L.rba_memory_units(h) == 3                     # the cosine bank is per batch row
    L.rba_store_destroy(h)
    assert L.rba_memory_units(None) == -1


def test_memory_update_argument_checks_launch_nothing(L):
    s, h = _create(L, block_size=16, capacity_tokens=1024)  # U = 2, cap_blocks = 64
    i64 = ctypes.c_int64
    T = 40 * 16 + 5                                         # nb = 40, tail 5
    upd = lambda T, pin, nw, od, kt, cnt=FAKE, km=FAKE: L.rba_memory_update(  # noqa: E731
        h, i64(T), pin, i64(nw), i64(od), i64(kt), cnt, km, None, None)
    assert upd(T, 0, 4, 4, 37) == 1                         # keep_total > n - drop_oldest
    assert upd(T, 0, 4, 4, 3) == 1                          # keep_total < keep_newest
    assert upd(T, 0, 30, 11, 30) == 1                       # newest + oldest > n
    assert upd(T, 41, 0, 0, 0) == 1                         # pinned beyond the full blocks
    assert upd(2000, 0, 0, 0, 0) == 1                       # T above the capacity
    assert upd(T, 0, 4, 4, 20, cnt=None) == 1               # no counters
    assert upd(T, 0, 4, 4, 20, km=None) == 1                # no keep map
    assert upd(T, -1, 4, 4, 20) == 1
    # counting: rows must be a whole number of units; an empty selection is a no-op
    assert L.rba_count_retrievals(h, FAKE, 3, 4, FAKE, None) == 1
    assert L.rba_count_retrievals(h, FAKE, 2, 0, FAKE, None) == 0
    assert L.rba_count_retrievals(h, FAKE, 2, 4, None, None) == 1
    L.rba_store_destroy(h)


def test_score_reduce_setter_checks(L):
    s, h = _create(L, mode=1, n_rep=4)                  # top-r keys
    assert L.rba_store_set_score_reduce(h, 1) == 0
    assert L.rba_store_set_score_reduce(h, 0) == 0
    assert L.rba_store_set_score_reduce(h, 2) == 1      # unknown value
    L.rba_store_destroy(h)
    s, h = _create(L, mode=4, block_size=1)             # identity: nothing to reduce
    assert L.rba_store_set_score_reduce(h, 1) == 1
    L.rba_store_destroy(h)
    assert L.rba_store_set_score_reduce(None, 1) == 1


def test_step_setters_check_their_arguments(L):
    # the one-launch switch takes 0 or 1; the wait bound takes any value (0:
    # the default); both reject a NULL store.  Host only: nothing launches.
    L.rba_store_set_decode_step_one_launch.argtypes = [ctypes.c_void_p, ctypes.c_int32]
    L.rba_store_set_wait_limit_ns.argtypes = [ctypes.c_void_p, ctypes.c_uint64]
    s, h = _create(L)
    assert L.rba_store_set_decode_step_one_launch(h, 1) == 0
    assert L.rba_store_set_decode_step_one_launch(h, 0) == 0
    assert L.rba_store_set_decode_step_one_launch(h, 2) == 1
    assert L.rba_store_set_decode_step_one_launch(h, -1) == 1
    assert L.rba_store_set_wait_limit_ns(h, 0) == 0
    assert L.rba_store_set_wait_limit_ns(h, 1000) == 0
    L.rba_store_destroy(h)
    assert L.rba_store_set_decode_step_one_launch(None, 1) == 1
    assert L.rba_store_set_wait_limit_ns(None, 0) == 1
