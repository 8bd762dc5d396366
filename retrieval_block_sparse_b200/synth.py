"""Seeded synthetic inputs for retrieval block-sparse attention.

The pages describe their workloads as model activations on long-text datasets;
none of those are available or needed here.  This module draws random inputs
with the shapes, value distributions and structure of the five workloads the
library is measured on, and nothing else: it holds none of the retrieval
method's arithmetic (no representative keys, no scores, no selection, no
attention).  Both the CUDA path and the fp64 CPU oracle read the arrays it
returns, and it imports neither of them.

Determinism: every tensor is drawn slice by slice from its own PCG64 stream,
keyed by ``(seed, tensor id, slice index)``, so the values do not depend on the
number of threads used to draw them.  bf16 tensors are drawn in fp32 and
rounded once, round-to-nearest-even, to bf16; they are returned as ``uint16``
bit patterns, which both sides widen exactly.

Layouts (row-major):
  K, V          [B][Hkv][T][D]           past keys / values of the memory
  q             [B][Hq][D]               decode queries (q head i -> kv head i // (Hq/Hkv))
  probe         [Hkv][P][D]              attention probe used to rank tokens
  landmarks     [B][Hkv][nb][D]          one landmark key per full block
  bank_embed    [nb][d_ret]              raw (unnormalised) chunk embeddings
  query_embed   [Bq][d_ret]              raw query-chunk embeddings
  Q, chunk K/V  [Bq][H][Nq][D]           prefill query chunk and its own K/V
"""
from __future__ import annotations

import dataclasses
import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

__all__ = [
    "DecodeWorkload", "PrefillWorkload", "WORKLOADS",
    "decode_inputs", "prefill_inputs", "bf16_round", "bf16_to_f32",
    "random_scores",
]

# ---------------------------------------------------------------------------
# workload descriptions


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    """One decode configuration: a single query token per (batch, q head)."""
    name: str
    dtype: str            # "f32" or "bf16": storage type of q, K, V and rep keys
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    context: int          # T: past tokens held in the store
    block_size: int       # bs
    n_rep: int            # r: representative keys per block
    rep_mode: str         # "mean" | "topr_attn" | "external" | "identity"
    top_k: int            # k: blocks retrieved per (batch, kv head)
    sink: int             # S: leading tokens always attended
    window: int           # W: trailing tokens always attended
    seed: int
    recipe: str           # "normal" | "planted" | "landmark" | "shifted"
    n_probe: int = 16     # P: probe queries ranking tokens (topr_attn only)
    n_planted: int = 16   # planted high-scoring blocks per kv head ("planted")

    def scaled(self, **kw) -> "DecodeWorkload":
        return dataclasses.replace(self, **kw)

    @property
    def n_blocks(self) -> int:
        return self.context // self.block_size


@dataclasses.dataclass(frozen=True)
class PrefillWorkload:
    """A chunk of Nq query tokens per (query chunk, q head) attending to
    retrieved blocks of a memory plus its own chunk (causally)."""
    name: str
    dtype: str
    n_chunks: int         # Bq: query chunks processed together
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    chunk_len: int        # Nq: query tokens per chunk (= tokens per own chunk)
    context: int          # T: tokens in the memory
    block_size: int
    top_k: int
    sink: int
    window: int
    score_mode: str       # "cosine" (per-chunk embedding) | "dot" (chunk-summed q)
    seed: int
    recipe: str           # "bank" | "shifted"
    d_ret: int = 0
    noise: float = 0.0    # sigma of the noisy-copy query embedding ("bank")

    def scaled(self, **kw) -> "PrefillWorkload":
        return dataclasses.replace(self, **kw)

    @property
    def n_blocks(self) -> int:
        return self.context // self.block_size


# The five measured workloads, named by what they are.
WORKLOADS = {
    # fp32 MHA decode: 4096-token context in 64-token blocks, mean rep keys.
    "tiny-decode-f32": DecodeWorkload(
        name="tiny-decode-f32", dtype="f32", batch=1, n_q_heads=4, n_kv_heads=4,
        head_dim=64, context=4096, block_size=64, n_rep=1, rep_mode="mean",
        top_k=4, sink=64, window=128, seed=1, recipe="normal"),
    # MemLong-style cosine chunk retrieval + chunked prefill over a 160-chunk bank.
    "memlong-cosine-prefill": PrefillWorkload(
        name="memlong-cosine-prefill", dtype="bf16", n_chunks=8, n_q_heads=32,
        n_kv_heads=32, head_dim=128, chunk_len=512, context=160 * 512,
        block_size=512, top_k=4, sink=0, window=0, score_mode="cosine", seed=2,
        recipe="bank", d_ret=768, noise=0.3),
    # InfLLM-style GQA decode at a 128K context: the headline workload.
    "infllm-decode-128k": DecodeWorkload(
        name="infllm-decode-128k", dtype="bf16", batch=1, n_q_heads=32, n_kv_heads=8,
        head_dim=128, context=131072, block_size=128, n_rep=4, rep_mode="topr_attn",
        top_k=32, sink=128, window=4096, seed=3, recipe="planted"),
    # Landmark-style batched MHA decode, 50-token blocks with an 18-token tail.
    "landmark-decode-b16": DecodeWorkload(
        name="landmark-decode-b16", dtype="bf16", batch=16, n_q_heads=32, n_kv_heads=32,
        head_dim=128, context=32768, block_size=50, n_rep=1, rep_mode="external",
        top_k=4, sink=0, window=256, seed=4, recipe="landmark"),
    # RetrievalAttention-style token-level (block size 1) retrieval over 1M keys.
    "token-retrieval-decode-1m": DecodeWorkload(
        name="token-retrieval-decode-1m", dtype="bf16", batch=1, n_q_heads=32,
        n_kv_heads=8, head_dim=128, context=1 << 20, block_size=1, n_rep=1,
        rep_mode="identity", top_k=2048, sink=128, window=512, seed=5, recipe="shifted"),
    "token-retrieval-prefill-1m": PrefillWorkload(
        name="token-retrieval-prefill-1m", dtype="bf16", n_chunks=1, n_q_heads=32,
        n_kv_heads=8, head_dim=128, chunk_len=2048, context=1 << 20, block_size=1,
        top_k=2048, sink=128, window=512, score_mode="dot", seed=5, recipe="shifted"),
}

# ---------------------------------------------------------------------------
# number generation

_TENSOR_IDS = {"K": 1, "V": 2, "q": 3, "probe": 4, "landmarks": 5, "u": 6,
               "planted": 7, "bank_embed": 8, "query_embed": 9, "Q": 10,
               "chunk_K": 11, "chunk_V": 12, "pick": 13, "scores": 14, "counts": 15}


def _stream(seed: int, tensor: str, index: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(
        np.random.SeedSequence([seed, _TENSOR_IDS[tensor], index])))


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def _normal(seed: int, tensor: str, shape, mean: float = 0.0, std: float = 1.0) -> np.ndarray:
    """fp32 N(mean, std^2) array; axis 0..-3 form independent slices."""
    shape = tuple(int(s) for s in shape)
    out = np.empty(shape, dtype=np.float32)
    flat = out.reshape((-1,) + shape[-2:]) if len(shape) >= 3 else out.reshape(1, -1)

    def fill(i):
        _stream(seed, tensor, i).standard_normal(out=flat[i], dtype=np.float32)
        if std != 1.0:
            flat[i] *= np.float32(std)
        if mean != 0.0:
            flat[i] += np.float32(mean)

    if flat.shape[0] == 1:
        fill(0)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(fill, range(flat.shape[0])))
    return out


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even); returns the uint16 bit patterns."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def _store(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return bf16_round(x)
    if dtype == "f32":
        return np.ascontiguousarray(x, dtype=np.float32)
    raise ValueError(f"unknown dtype {dtype!r}")


def _unit_rows(x: np.ndarray) -> np.ndarray:
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


# ---------------------------------------------------------------------------
# decode inputs


def decode_inputs(w: DecodeWorkload) -> dict:
    """Inputs of one decode step of workload ``w``.

    Recipes:
      normal    q, K, V ~ N(0, 1).
      planted   K, V ~ N(0, 1); per kv head a unit direction u_h; ``n_planted``
                blocks lying wholly between the sink and the window get +2 u_h
                added to every key; the q heads of group h are z + 3 u_h.
      landmark  q, K, V, landmark keys ~ N(0, 1); per (batch, head) one block
                j* before the window is drawn and q = 0.5 L[j*] + sqrt(0.75) z.
      shifted   K, V ~ N(0, 1); q ~ N(0.5, 1.5^2) (query/key distribution gap).
      drift     as shifted, but each key channel drifts slowly along the sequence
                (first-order autoregression, correlation 0.97 between neighbouring
                tokens, unit variance): nearby keys resemble each other.
    """
    B, Hq, Hkv, D, T, bs = (w.batch, w.n_q_heads, w.n_kv_heads, w.head_dim,
                            w.context, w.block_size)
    if Hq % Hkv:
        raise ValueError("n_q_heads must be a multiple of n_kv_heads")
    g = Hq // Hkv
    s = w.seed
    out = {}
    K = _normal(s, "K", (B, Hkv, T, D))
    V = _normal(s, "V", (B, Hkv, T, D))
    if w.recipe == "normal":
        q = _normal(s, "q", (B, Hq, D))
    elif w.recipe == "shifted":
        q = _normal(s, "q", (B, Hq, D), mean=0.5, std=1.5)
    elif w.recipe == "drift":
        from scipy.signal import lfilter
        rho = 0.97

        def drift(bh):
            # one (batch, kv head) slice at a time; slices are independent, so
            # the threads change no value
            z = K[bh // Hkv, bh % Hkv]
            zi = (rho * z[0])[None, :]
            z[1:] = lfilter([math.sqrt(1.0 - rho * rho)], [1.0, -rho], z[1:], axis=0, zi=zi)[0]
        with ThreadPoolExecutor(max(1, min(B * Hkv, os.cpu_count() or 1))) as ex:
            list(ex.map(drift, range(B * Hkv)))
        q = _normal(s, "q", (B, Hq, D), mean=0.5, std=1.5)
    elif w.recipe == "planted":
        u = _unit_rows(_normal(s, "u", (Hkv, D)).astype(np.float64)).astype(np.float32)
        lo = -(-w.sink // bs)                       # first block starting at/after the sink
        hi = max(T - w.window, 0) // bs             # blocks ending at/before the window
        n_pl = min(w.n_planted, max(hi - lo, 0))
        planted = np.zeros((B, Hkv, n_pl), dtype=np.int64)
        for b in range(B):
            for h in range(Hkv):
                if n_pl:
                    pick = _stream(s, "planted", b * Hkv + h).choice(hi - lo, n_pl, replace=False)
                    planted[b, h] = np.sort(pick + lo)
                    for j in planted[b, h]:
                        K[b, h, j * bs:(j + 1) * bs] += 2.0 * u[h]
        q = _normal(s, "q", (B, Hq, D))
        for i in range(Hq):
            q[:, i] += 3.0 * u[i // g]
        out["planted_blocks"] = planted
        out["u"] = u
    elif w.recipe == "landmark":
        nb = T // bs
        L = _normal(s, "landmarks", (B, Hkv, nb, D))
        hi = max(T - w.window, 0) // bs
        q = _normal(s, "q", (B, Hq, D))
        star = np.zeros((B, Hq), dtype=np.int64)
        for b in range(B):
            for i in range(Hq):
                star[b, i] = _stream(s, "pick", b * Hq + i).integers(0, max(hi, 1))
        # q is built from the stored (rounded) landmark, so the correlation
        # holds for the values the method actually reads.
        Ls = _store(L, w.dtype)
        Lr = bf16_to_f32(Ls) if w.dtype == "bf16" else Ls
        for b in range(B):
            for i in range(Hq):
                q[b, i] = 0.5 * Lr[b, i // g, star[b, i]] + math.sqrt(0.75) * q[b, i]
        out["landmarks"] = Ls
        out["landmark_pick"] = star
    else:
        raise ValueError(f"unknown recipe {w.recipe!r}")
    if w.rep_mode == "topr_attn":
        out["probe"] = _store(_normal(s, "probe", (Hkv, w.n_probe, D)), w.dtype)
    out["K"] = _store(K, w.dtype)
    del K
    out["V"] = _store(V, w.dtype)
    del V
    out["q"] = _store(q, w.dtype)
    return out


# ---------------------------------------------------------------------------
# prefill inputs


def prefill_inputs(w: PrefillWorkload) -> dict:
    """Inputs of one chunked-prefill step of workload ``w``.

    Recipes:
      bank     memory K/V ~ N(0, 1) stored as ``nb`` chunks of ``block_size``
               tokens; raw chunk embeddings g_j ~ N(0, I_dret); query chunk i
               copies bank entry j_i (uniform) with noise: g_{j_i} + noise * z.
               Query-chunk Q and its own K/V ~ N(0, 1).
      shifted  memory K/V ~ N(0, 1); Q ~ N(0.5, 1.5^2); own-chunk K/V ~ N(0, 1).
    """
    Bq, Hq, Hkv, D, Nq, T = (w.n_chunks, w.n_q_heads, w.n_kv_heads, w.head_dim,
                             w.chunk_len, w.context)
    s = w.seed
    out = {}
    out["K"] = _store(_normal(s, "K", (1, Hkv, T, D)), w.dtype)
    out["V"] = _store(_normal(s, "V", (1, Hkv, T, D)), w.dtype)
    if w.recipe == "bank":
        nb = T // w.block_size
        gbank = _normal(s, "bank_embed", (nb, w.d_ret))
        src = _stream(s, "pick").integers(0, nb, size=Bq)
        z = _normal(s, "query_embed", (Bq, w.d_ret))
        out["bank_embed"] = gbank
        out["query_embed"] = (gbank[src] + np.float32(w.noise) * z).astype(np.float32)
        out["query_source"] = src
        out["Q"] = _store(_normal(s, "Q", (Bq, Hq, Nq, D)), w.dtype)
    elif w.recipe == "shifted":
        out["Q"] = _store(_normal(s, "Q", (Bq, Hq, Nq, D), mean=0.5, std=1.5), w.dtype)
    else:
        raise ValueError(f"unknown recipe {w.recipe!r}")
    out["chunk_K"] = _store(_normal(s, "chunk_K", (Bq, Hkv, Nq, D)), w.dtype)
    out["chunk_V"] = _store(_normal(s, "chunk_V", (Bq, Hkv, Nq, D)), w.dtype)
    return out


# ---------------------------------------------------------------------------
# bare score rows (for the selector alone)


def random_scores(seed: int, rows: int, n: int, ties: int = 0) -> np.ndarray:
    """fp32 score rows ~ N(0, 1).  With ``ties`` > 0, each row's values are
    drawn from only ``ties`` distinct levels, so equal scores are frequent."""
    x = _normal(seed, "scores", (rows, n))
    if ties:
        lv = np.sort(_normal(seed + 1, "scores", (1, ties))[0])
        x = lv[np.floor((x - x.min()) / (x.max() - x.min() + 1e-9) * ties).astype(np.int64).clip(0, ties - 1)]
    return np.ascontiguousarray(x, dtype=np.float32)


# ---------------------------------------------------------------------------
# retrieval counters (for the dynamic memory update)


def retrieval_counts(seed: int, units: int, n: int, huge: float = 0.0) -> np.ndarray:
    """uint32 retrieval-frequency counters [units][n]: most entries rarely
    retrieved (Poisson mean 0.7), about 30% often (Poisson mean 20), so equal
    counts are frequent.  A fraction ``huge`` of the entries gets a count in
    [2^31, 2^32) (exercises every byte of a 32-bit count)."""
    g = _stream(seed, "counts")
    c = g.poisson(0.7, size=(units, n)).astype(np.uint64)
    hot = g.random((units, n)) < 0.3
    c[hot] = g.poisson(20.0, size=int(hot.sum()))
    if huge > 0:
        big = g.random((units, n)) < huge
        c[big] = g.integers(1 << 31, (1 << 32) - 1, size=int(big.sum()))
    return c.astype(np.uint32)
