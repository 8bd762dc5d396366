"""Retrieval block-sparse attention on B200 (sm_100a).

Context-memory retrieval attention for long-context decode and chunked
prefill: blocks of past K/V are scored by representative keys or embeddings,
the top-k blocks per KV head are selected, and exact softmax attention runs
over sink tokens, retrieved blocks and the local window.  Around that path:
a streaming decode step (append a token, memorise the block it completes,
decode), counter-driven dynamic memory update with in-place compaction, and
a max-over-representative-keys score variant.

All computation is in the CUDA library ``librba.so`` (C ABI:
``include/rba.h``); ``rba`` is its Python binding.  ``synth`` draws the seeded
synthetic inputs.
"""
from .rba import (Store, RbaError, topk, memory_rule, lib, status_string,  # noqa: F401
                  OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_CUDA,
                  ERR_TIMEOUT, ERR_BOUNDS, LIB_PATH, SIGNATURES)

__all__ = ["Store", "RbaError", "topk", "memory_rule", "lib", "status_string", "LIB_PATH", "SIGNATURES"]
