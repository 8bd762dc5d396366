"""Python binding of librba.so (include/rba.h): argument marshalling only.

Every computation runs in the CUDA library.  torch supplies device memory
(caller-owned pools, outputs, workspaces) and the current CUDA stream.  If
the library is missing the calls raise; there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "librba.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA, ERR_TIMEOUT, ERR_BOUNDS = range(7)
F32, BF16 = 0, 1
MODES = {"mean": 0, "topr_attn": 1, "external": 2, "embed_cosine": 3, "identity": 4}
SCORE_REDUCE = {"sum": 0, "max": 1}

_c_i32, _c_i64, _c_f32, _c_size, _p = (ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                                        ctypes.c_size_t, ctypes.c_void_p)

# name -> (restype, argtypes), mirroring include/rba.h
SIGNATURES = {
    "rba_store_create": (_c_i32, [_p, _p, _p, _p, _p, _p, ctypes.POINTER(_p)]),
    "rba_store_destroy": (_c_i32, [_p]),
    "rba_store_set_score_reduce": (_c_i32, [_p, _c_i32]),
    "rba_store_set_wait_limit_ns": (_c_i32, [_p, ctypes.c_uint64]),
    "rba_store_set_decode_step_one_launch": (_c_i32, [_p, _c_i32]),
    "rba_candidates": (_c_i32, [_p, _c_i64, _c_i32, _c_i32, ctypes.POINTER(_c_i32),
                                ctypes.POINTER(_c_i32)]),
    "rba_memorize": (_c_i32, [_p, _p, _p, _c_i64, _c_i32, _p, _c_i32, _c_f32, _p]),
    "rba_score": (_c_i32, [_p, _p, _c_i32, _c_i64, _c_i32, _c_i32, _p, _p, _p]),
    "rba_topk": (_c_i32, [_p, _c_i32, _c_i32, _c_i32, _c_i32, _p, _p, _c_size, _p]),
    "rba_topk_workspace_size": (_c_size, [_c_i32, _c_i32, _c_i32]),
    "rba_attend": (_c_i32, [_p, _p, _p, _c_i32, _c_i64, _c_i32, _c_i32, _c_f32, _p, _p, _p,
                            _c_size, _p]),
    "rba_attend_workspace_size": (_c_size, [_p, _c_i32, _c_i64, _c_i32, _c_i32]),
    "rba_attend_noalloc": (_c_i32, [_p, _p, _p, _c_i32, _c_i64, _c_i32, _c_i32, _c_f32, _p, _p,
                                    _p]),
    "rba_attend_landmark_gated": (_c_i32, [_p, _p, _p, _c_i32, _c_i64, _c_i32, _c_i32, _c_f32,
                                           _p, _p, _p]),
    "rba_attend_prefill": (_c_i32, [_p, _p, _c_i32, _c_i32, _p, _c_i32, _c_i32, _c_i64, _c_i32,
                                    _c_i32, _p, _p, _c_f32, _p, _p, _p, _c_size, _p]),
    "rba_attend_prefill_workspace_size": (_c_size, [_p, _c_i32, _c_i32, _c_i32, _c_i32, _c_i64,
                                                    _c_i32, _c_i32]),
    "rba_decode_step": (_c_i32, [_p, _p, _c_i32, _c_i64, _c_i32, _c_i32, _c_f32, _p, _p, _p, _p,
                                 _p, _c_size, _p]),
    "rba_decode_step_workspace_size": (_c_size, [_p, _c_i32, _c_i64, _c_i32, _c_i32]),
    "rba_decode_step_plan": (_c_i32, [_p, _c_i32, _c_i64, _c_i32, _c_i32]),
    "rba_decode_step_launches": (_c_i32, [_p, _c_i32, _c_i64, _c_i32, _c_i32]),
    "rba_stream_step": (_c_i32, [_p, _p, _p, _p, _c_i64, _c_i32, _c_i32, _c_i32, _c_f32, _p,
                                 _c_i32, _p, _p, _p, ctypes.POINTER(_c_i32), _p, _c_size, _p]),
    "rba_group_means": (_c_i32, [_p, _c_i64, _c_i32, _c_i32, _p, _p]),
    "rba_approx_select": (_c_i32, [_p, _p, _c_i64, _c_i32, _c_i32, _c_i32, _c_i32, _c_i32, _p,
                                   _p, _p, _p, _p, _c_size, _p]),
    "rba_approx_select_workspace_size": (_c_size, [_p, _c_i64, _c_i32, _c_i32, _c_i32, _c_i32,
                                                   _c_i32]),
    "rba_memory_rule": (_c_i32, [_c_i64, ctypes.POINTER(_c_i64), ctypes.POINTER(_c_i64),
                                 ctypes.POINTER(_c_i64)]),
    "rba_memory_units": (_c_i32, [_p]),
    "rba_count_retrievals": (_c_i32, [_p, _p, _c_i32, _c_i32, _p, _p]),
    "rba_memory_update": (_c_i32, [_p, _c_i64, _c_i32, _c_i64, _c_i64, _c_i64, _p, _p,
                                   ctypes.POINTER(_c_i64), _p]),
    "rba_decode_step_host": (_c_i32, [_p, _p, _p, _c_i32, _c_i64, _c_i32, _c_i32, _c_f32, _p, _p,
                                      _p, _p, _p, _p, _p, _c_size, _p]),
    "rba_store_check": (_c_i32, [_p, _p]),
    "rba_row_pitch": (_c_i32, [_c_i32]),
    "rba_status_string": (ctypes.c_char_p, [_c_i32]),
    "rba_version": (_c_i32, []),
}

_LIB = None


class RbaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def lib() -> ctypes.CDLL:
    """Loads librba.so (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m retrieval_block_sparse_b200.build`"
                " (the CUDA library is required; there is no CPU fallback)")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = L
    return _LIB


def status_string(s: int) -> str:
    return lib().rba_status_string(s).decode()


def _check(s: int, where: str):
    if s != OK:
        raise RbaError(s, where)


def _ptr(t) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _tdtype(dtype: int):
    return torch.bfloat16 if dtype == BF16 else torch.float32


class _Desc(ctypes.Structure):
    _fields_ = [("batch", _c_i32), ("n_q_heads", _c_i32), ("n_kv_heads", _c_i32),
                ("head_dim", _c_i32), ("block_size", _c_i32), ("n_rep", _c_i32),
                ("d_ret", _c_i32), ("capacity_tokens", _c_i64), ("dtype", _c_i32),
                ("mode", _c_i32)]


class Store:
    """A block store: caller-owned device pools described to the library.

    Pools (allocated here with torch, owned by this object), rows of P =
    rba_row_pitch(D) elements (P = D for D = 64 or 128; else the first D are
    the row and the rest stay zero -- write rows through `kv_rows`):
      k, v     [B][Hkv][capacity][P]         store dtype
      rep      mean: fp32 [B][Hkv][cap_blocks][1][P]; topr_attn / external:
               dtype [B][Hkv][cap_blocks][r][P]; embed_cosine: fp32
               [B][cap_blocks][d_ret]; identity: none
      rep_pos  int32 [B][Hkv][cap_blocks][r] (topr_attn)
      status   int32[4] device status word
    score_reduce: "sum" (default) or "max" -- how a block's r representative
    keys combine into its score (rba_store_set_score_reduce).
    """

    def __init__(self, *, batch, n_q_heads, n_kv_heads, head_dim, block_size, capacity_tokens,
                 dtype="bf16", mode="mean", n_rep=1, d_ret=0, device="cuda", score_reduce="sum"):
        self.dtype = BF16 if dtype in ("bf16", torch.bfloat16) else F32
        self.mode = mode
        self.B, self.Hq, self.Hkv, self.D = batch, n_q_heads, n_kv_heads, head_dim
        self.bs, self.r, self.d_ret, self.cap = block_size, n_rep, d_ret, capacity_tokens
        self.cap_blocks = capacity_tokens // block_size
        # pool rows hold `pitch` elements: the head dim, then zero padding
        self.pitch = lib().rba_row_pitch(head_dim)
        if self.pitch < 0:
            raise RbaError(ERR_UNSUPPORTED, f"head_dim {head_dim}")
        P = self.pitch
        td = _tdtype(self.dtype)
        dev = torch.device(device)
        self.k = torch.zeros((batch, n_kv_heads, capacity_tokens, P), dtype=td, device=dev)
        self.v = torch.zeros_like(self.k)
        self.rep = None
        self.rep_pos = None
        if mode == "mean":
            self.rep = torch.zeros((batch, n_kv_heads, self.cap_blocks, 1, P),
                                   dtype=torch.float32, device=dev)
        elif mode in ("topr_attn", "external"):
            self.rep = torch.zeros((batch, n_kv_heads, self.cap_blocks, n_rep, P), dtype=td,
                                   device=dev)
            if mode == "topr_attn":
                self.rep_pos = torch.full((batch, n_kv_heads, self.cap_blocks, n_rep), -1,
                                          dtype=torch.int32, device=dev)
        elif mode == "embed_cosine":
            self.rep = torch.zeros((batch, self.cap_blocks, d_ret), dtype=torch.float32, device=dev)
        elif mode != "identity":
            raise ValueError(mode)
        self.status = torch.zeros(4, dtype=torch.int32, device=dev)
        d = _Desc(batch, n_q_heads, n_kv_heads, head_dim, block_size, n_rep, d_ret,
                  capacity_tokens, self.dtype, MODES[mode])
        h = _p()
        _check(lib().rba_store_create(ctypes.byref(d), _ptr(self.k), _ptr(self.v), _ptr(self.rep),
                                      _ptr(self.rep_pos), _ptr(self.status), ctypes.byref(h)),
               "rba_store_create")
        self.handle = h
        if score_reduce != "sum":
            _check(lib().rba_store_set_score_reduce(h, SCORE_REDUCE[score_reduce]),
                   "rba_store_set_score_reduce")
        self.score_reduce = score_reduce

    def set_wait_limit_ns(self, ns):
        """Bound of the one-launch decode step's device waits (0: the default 2 s)."""
        _check(lib().rba_store_set_wait_limit_ns(self.handle, int(ns)),
               "rba_store_set_wait_limit_ns")

    def set_decode_step_one_launch(self, on=True):
        """Let decode_step run as one cooperative launch where eligible (plan 3)."""
        _check(lib().rba_store_set_decode_step_one_launch(self.handle, int(bool(on))),
               "rba_store_set_decode_step_one_launch")

    def __del__(self):
        h = getattr(self, "handle", None)
        if h is not None and _LIB is not None:
            _LIB.rba_store_destroy(h)
            self.handle = None

    @property
    def tdtype(self):
        return _tdtype(self.dtype)

    def kv_rows(self, t):
        """The first D elements of every row of a pool tensor (a view to write into)."""
        return t[..., :self.D]

    # -- geometry ------------------------------------------------------------
    def candidates(self, T, sink, window):
        f, n = _c_i32(), _c_i32()
        _check(lib().rba_candidates(self.handle, T, sink, window, ctypes.byref(f), ctypes.byref(n)),
               "rba_candidates")
        return f.value, n.value

    # -- memorise --------------------------------------------------------------
    def memorize(self, k_src=None, v_src=None, *, first_block=0, n_blocks=None, aux=None,
                 scale=None):
        if n_blocks is None:
            n_blocks = k_src.shape[2] // self.bs if k_src is not None else aux.shape[2]
        n_aux = 0
        if aux is not None and self.mode == "topr_attn":
            n_aux = aux.shape[1]
        if scale is None:
            scale = 1.0 / math.sqrt(self.D)
        _check(lib().rba_memorize(self.handle, _ptr(k_src), _ptr(v_src), first_block, n_blocks,
                                  _ptr(aux), n_aux, scale, _stream()), "rba_memorize")

    # -- score -------------------------------------------------------------------
    def score(self, q, T, sink, window, *, n_q=None, out=None, qsum_ws=None):
        first, nc = self.candidates(T, sink, window)
        if self.mode == "embed_cosine":
            n_q = q.shape[0]
            shape = (n_q, nc)
        else:
            n_q = 1 if q.dim() == 3 else q.shape[2]
            shape = (self.B, self.Hkv, nc)
            if (self.Hq // self.Hkv) * n_q > 64 and qsum_ws is None:
                qsum_ws = torch.empty((self.B, self.Hkv, self.D), dtype=torch.float32,
                                      device=q.device)
        if out is None:
            out = torch.empty(shape, dtype=torch.float32, device=q.device)
        _check(lib().rba_score(self.handle, _ptr(q), n_q, T, sink, window, _ptr(out),
                               _ptr(qsum_ws), _stream()), "rba_score")
        return out

    # -- attend ----------------------------------------------------------------
    def attend_workspace(self, k, T, sink, window):
        n = lib().rba_attend_workspace_size(self.handle, k, T, sink, window)
        return torch.zeros(max(n, 16), dtype=torch.uint8, device=self.k.device)

    def attend(self, q, idx, T, sink, window, *, scale=None, out=None, lse=None, workspace=None):
        k = idx.shape[-1] if idx is not None else 0
        if scale is None:
            scale = 1.0 / math.sqrt(self.D)
        if out is None:
            out = torch.empty((self.B, self.Hq, self.D), dtype=torch.float32, device=q.device)
        if lse is None:
            lse = torch.empty((self.B, self.Hq), dtype=torch.float32, device=q.device)
        if workspace is None:
            workspace = self.attend_workspace(k, T, sink, window)
        _check(lib().rba_attend(self.handle, _ptr(q), _ptr(idx), k, T, sink, window, scale,
                                _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(),
                                _stream()), "rba_attend")
        return out, lse

    def attend_gated(self, q, idx, T, sink, window, *, scale=None, out=None, lse=None):
        """Landmark-gated attention (landmark stores): each retrieved block enters
        the softmax once, with its landmark's logit (see rba.h)."""
        k = idx.shape[-1] if idx is not None else 0
        if scale is None:
            scale = 1.0 / math.sqrt(self.D)
        if out is None:
            out = torch.empty((self.B, self.Hq, self.D), dtype=torch.float32, device=q.device)
        if lse is None:
            lse = torch.empty((self.B, self.Hq), dtype=torch.float32, device=q.device)
        _check(lib().rba_attend_landmark_gated(self.handle, _ptr(q), _ptr(idx), k, T, sink,
                                               window, scale, _ptr(out), _ptr(lse), _stream()),
               "rba_attend_landmark_gated")
        return out, lse

    def prefill_workspace(self, n_chunks, chunk_len, n_sel, k, T, sink, window):
        n = lib().rba_attend_prefill_workspace_size(self.handle, n_chunks, chunk_len, n_sel, k, T,
                                                    sink, window)
        return torch.zeros(max(n, 16), dtype=torch.uint8, device=self.k.device)

    def attend_prefill(self, q, idx, chunk_k, chunk_v, T, sink, window, *, scale=None, out=None,
                       lse=None, workspace=None):
        n_chunks, _, chunk_len, _ = q.shape
        n_sel, k = idx.shape[1], idx.shape[2]
        if scale is None:
            scale = 1.0 / math.sqrt(self.D)
        if out is None:
            out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
        if lse is None:
            lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
        if workspace is None:
            workspace = self.prefill_workspace(n_chunks, chunk_len, n_sel, k, T, sink, window)
        _check(lib().rba_attend_prefill(self.handle, _ptr(q), n_chunks, chunk_len, _ptr(idx), n_sel,
                                        k, T, sink, window, _ptr(chunk_k), _ptr(chunk_v), scale,
                                        _ptr(out), _ptr(lse), _ptr(workspace), workspace.numel(),
                                        _stream()), "rba_attend_prefill")
        return out, lse

    # -- whole decode step -----------------------------------------------------------
    def decode_workspace(self, k, T, sink, window):
        n = lib().rba_decode_step_workspace_size(self.handle, k, T, sink, window)
        return torch.zeros(max(n, 16), dtype=torch.uint8, device=self.k.device)

    def decode_plan(self, k, T, sink, window):
        """3: the whole step in one cooperative launch; 2: score -> top-k ->
        whole-block tensor-core attention kernel, overlapped (programmatic
        dependent launches); 1: the same with the CUDA-core attention kernel;
        0: score -> top-k -> split-K in stream order; <0: see rba.h."""
        return lib().rba_decode_step_plan(self.handle, k, T, sink, window)

    def decode_launches(self, k, T, sink, window):
        """Kernels one decode_step enqueues (-4: invalid arguments)."""
        return lib().rba_decode_step_launches(self.handle, k, T, sink, window)

    def decode_step(self, q, k, T, sink, window, *, scale=None, workspace=None, out=None,
                    lse=None, idx=None, scores=None):
        if scale is None:
            scale = 1.0 / math.sqrt(self.D)
        dev = q.device
        if out is None:
            out = torch.empty((self.B, self.Hq, self.D), dtype=torch.float32, device=dev)
        if lse is None:
            lse = torch.empty((self.B, self.Hq), dtype=torch.float32, device=dev)
        if idx is None:
            idx = torch.empty((self.B, self.Hkv, k), dtype=torch.int32, device=dev)
        if workspace is None:
            workspace = self.decode_workspace(k, T, sink, window)
        _check(lib().rba_decode_step(self.handle, _ptr(q), k, T, sink, window, scale, _ptr(scores),
                                     _ptr(idx), _ptr(out), _ptr(lse), _ptr(workspace),
                                     workspace.numel(), _stream()), "rba_decode_step")
        return idx, out, lse

    def stream_step(self, q, k_new, v_new, T, k, sink, window, *, aux=None, scale=None,
                    workspace=None, out=None, lse=None, idx=None):
        """Append one token's K/V at position T, memorise the block it completes,
        decode q over T + 1 tokens.  Returns (idx [B][Hkv][k'], out, lse) with
        k' = min(k, candidates at T + 1)."""
        if scale is None:
            scale = 1.0 / math.sqrt(self.D)
        dev = q.device
        if out is None:
            out = torch.empty((self.B, self.Hq, self.D), dtype=torch.float32, device=dev)
        if lse is None:
            lse = torch.empty((self.B, self.Hq), dtype=torch.float32, device=dev)
        if idx is None:
            idx = torch.empty((self.B, self.Hkv, max(k, 1)), dtype=torch.int32, device=dev)
        if workspace is None:
            workspace = self.decode_workspace(k, T + 1, sink, window)
        n_aux = aux.shape[1] if (aux is not None and self.mode == "topr_attn") else 0
        used = ctypes.c_int32(0)
        _check(lib().rba_stream_step(self.handle, _ptr(q), _ptr(k_new), _ptr(v_new), T, k, sink,
                                     window, scale, _ptr(aux), n_aux, _ptr(idx), _ptr(out),
                                     _ptr(lse), ctypes.byref(used), _ptr(workspace),
                                     workspace.numel(), _stream()), "rba_stream_step")
        kk = used.value
        sel = idx.reshape(-1)[: self.B * self.Hkv * kk].reshape(self.B, self.Hkv, kk)
        return sel, out, lse

    # -- two-stage approximate token retrieval (block size 1) ---------------------
    def group_means(self, group, *, first_group=0, n_groups=None, out=None):
        """Mean key of every group of `group` consecutive tokens (fp32 index
        [B][Hkv][capacity // group][P]); groups [first_group, first_group + n_groups)."""
        cap_groups = self.cap // group
        if n_groups is None:
            n_groups = cap_groups - first_group
        if out is None:
            out = torch.zeros((self.B, self.Hkv, cap_groups, self.pitch), dtype=torch.float32,
                              device=self.k.device)
        _check(lib().rba_group_means(self.handle, first_group, n_groups, group, _ptr(out),
                                     _stream()), "rba_group_means")
        return out

    def approx_select(self, q, T, sink, window, group, groups_kept, k, means, *, idx=None,
                      groups_out=None, scanned=None, workspace=None):
        """Two-stage selection of k tokens per (batch, kv head).  Returns
        (idx [B][Hkv][k], kept groups [B][Hkv][groups_kept], keys read [B][Hkv])."""
        dev = q.device
        if idx is None:
            idx = torch.empty((self.B, self.Hkv, k), dtype=torch.int32, device=dev)
        if groups_out is None:
            groups_out = torch.empty((self.B, self.Hkv, groups_kept), dtype=torch.int32,
                                     device=dev)
        if scanned is None:
            scanned = torch.empty((self.B, self.Hkv), dtype=torch.int32, device=dev)
        if workspace is None:
            n = lib().rba_approx_select_workspace_size(self.handle, T, sink, window, group,
                                                       groups_kept, k)
            workspace = torch.empty(max(n, 16), dtype=torch.uint8, device=dev)
        _check(lib().rba_approx_select(self.handle, _ptr(q), T, sink, window, group,
                                       groups_kept, k, _ptr(means), _ptr(idx), _ptr(groups_out),
                                       _ptr(scanned), _ptr(workspace), workspace.numel(),
                                       _stream()), "rba_approx_select")
        return idx, groups_out, scanned

    # -- dynamic memory update ---------------------------------------------------
    def memory_units(self):
        """Memory units U: B * Hkv (dot modes) or B (cosine bank)."""
        return lib().rba_memory_units(self.handle)

    def new_counters(self):
        """Zeroed retrieval counters [U][cap_blocks] (uint32 in the library; held
        here as int32 with the same bits)."""
        return torch.zeros((self.memory_units(), self.cap_blocks), dtype=torch.int32,
                           device=self.k.device)

    def count_retrievals(self, idx, counters):
        """Adds the selection idx ([..., U, k] int32, row r -> unit r % U) to counters."""
        k = idx.shape[-1]
        rows = idx.numel() // k if k else 0
        _check(lib().rba_count_retrievals(self.handle, _ptr(idx), rows, k, _ptr(counters),
                                          _stream()), "rba_count_retrievals")

    def memory_update(self, T, counters, *, pinned_blocks=0, keep_newest=None, drop_oldest=None,
                      keep_total=None, keep_map=None):
        """Counter-driven prune and in-place compaction of the T tokens held.
        Counts not given follow memory_rule(n) for the n = T // bs - pinned_blocks
        entries.  Returns (T_new, keep_map [U][keep_total])."""
        n = T // self.bs - pinned_blocks
        rule = memory_rule(max(n, 0))
        keep_newest = rule[0] if keep_newest is None else keep_newest
        drop_oldest = rule[1] if drop_oldest is None else drop_oldest
        keep_total = rule[2] if keep_total is None else keep_total
        if keep_map is None:
            keep_map = torch.empty((self.memory_units(), max(keep_total, 1)), dtype=torch.int32,
                                   device=self.k.device)
        t_new = _c_i64(0)
        _check(lib().rba_memory_update(self.handle, T, pinned_blocks, keep_newest, drop_oldest,
                                       keep_total, _ptr(counters), _ptr(keep_map),
                                       ctypes.byref(t_new), _stream()), "rba_memory_update")
        return t_new.value, keep_map[:, :keep_total]

    def decode_step_host(self, q_host, k, T, sink, window, *, q_dev, idx_dev, out_dev, lse_dev,
                         out_host, lse_host=None, idx_host=None, workspace, scale=None):
        """Host buffers in and out; synchronises the current stream."""
        if scale is None:
            scale = 1.0 / math.sqrt(self.D)
        hp = lambda t: None if t is None else t.data_ptr()  # noqa: E731
        _check(lib().rba_decode_step_host(self.handle, hp(q_host), _ptr(q_dev), k, T, sink, window,
                                          scale, _ptr(idx_dev), _ptr(out_dev), _ptr(lse_dev),
                                          hp(out_host), hp(lse_host), hp(idx_host),
                                          _ptr(workspace), workspace.numel(), _stream()),
               "rba_decode_step_host")

    def check(self):
        """Synchronises and raises if a kernel recorded a device-side error."""
        _check(lib().rba_store_check(self.handle, _stream()), "device status")


def memory_rule(n):
    """(keep_newest, drop_oldest, keep_total) for n memory entries (host only)."""
    a, b, c = _c_i64(), _c_i64(), _c_i64()
    _check(lib().rba_memory_rule(n, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c)),
           "rba_memory_rule")
    return a.value, b.value, c.value


def topk(scores, k, *, index_base=0, out=None, workspace=None):
    """Top-k per row of a 2-D (or [..., n]) fp32 score tensor; ascending positions."""
    n = scores.shape[-1]
    rows = scores.numel() // n if n else 0
    if out is None:
        out = torch.empty(scores.shape[:-1] + (k,), dtype=torch.int32, device=scores.device)
    if workspace is None:
        nb = lib().rba_topk_workspace_size(rows, n, k)
        workspace = torch.empty(max(nb, 16), dtype=torch.uint8, device=scores.device)
    _check(lib().rba_topk(_ptr(scores), rows, n, k, index_base, _ptr(out), _ptr(workspace),
                          workspace.numel(), _stream()), "rba_topk")
    return out
