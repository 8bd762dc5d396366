/*
 * rba.h -- retrieval block-sparse attention on NVIDIA B200 (sm_100a), C ABI.
 *
 * Context-memory retrieval attention for long-context decoding and chunked
 * prefill.  Past K/V is cut into fixed-size blocks; each block carries
 * representative keys (or an embedding); a query scores the blocks, keeps the
 * top k per KV head, and runs exact softmax attention over the sink tokens,
 * the retrieved blocks and the local window.
 *
 * Sources (pages, by title and section):
 *   [ML] "MemLong: Memory-Augmented Retrieval for Long Text Modeling"
 *        (summary page) -- 2.2.1 fixed-size chunks, 2.2.2 memory of K-V pairs
 *        plus representation embeddings, 2.3.2 retrieval (cosine, TopK) and
 *        memorisation M(k, v; r^m), 2.3.3 / Figure 3 retrieval-causal
 *        attention, 2.3.4 inference (attention window k * chunk size).
 *   [IL] InfLLM article (Tsinghua NLP, "1024K context, 100% recall") --
 *        "method" and "overall framework": sliding window + memory units of
 *        contiguous tokens, represented by the tokens that received the most
 *        attention.
 *   [LM] "Landmark Attention: Random-Access Infinite Context Length for
 *        Transformers" (review) -- "proposed method": one landmark key per
 *        fixed-length block, retrieval by query-landmark similarity.
 *   [RA] RetrievalAttention summary (arXiv 2409.10516) -- "proposed method":
 *        every key its own unit (block size 1), retrieved by vector search.
 *
 * Conventions for every call:
 *   - Every device buffer is owned by the caller.  The library never
 *     allocates or frees device memory; calls that need scratch take a
 *     caller-provided workspace whose size a *_workspace_size() call reports.
 *   - Pointers marked "device" must be device pointers (cudaMalloc / torch);
 *     "host" pointers are host memory.  All tensors are dense, row-major,
 *     with the layout given in brackets.
 *   - Work is asynchronous on the given stream; no call synchronises except
 *     rba_store_check and rba_decode_step_host, which say so.
 *   - Arguments are validated on the host before anything is launched; a
 *     failed check returns a status and launches nothing.  Errors found on
 *     the device (index out of range, a bounded wait that gave up) set the
 *     store's status word, read back by rba_store_check.
 *   - No C++ exception crosses this interface.
 *
 * Block / token vocabulary used below (T = tokens currently in the store):
 *   block j            tokens [j*bs, (j+1)*bs) of one (batch, kv head)
 *   w0                 max(T - window, 0): first token of the local window
 *   sink               tokens [0, min(sink, w0))
 *   candidate block    a full block whose tokens meet [sink, w0); candidates
 *                      form the contiguous range [first_cand, first_cand+nc)
 *   attended set       sink U retrieved blocks U window, each token once
 *   T - nb*bs > window (a partial tail block outside the window) is rejected.
 */
#ifndef RBA_H_
#define RBA_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RBA_OK = 0,
  RBA_ERR_INVALID_ARG = 1,  /* bad size, pointer, mode or layout; nothing launched */
  RBA_ERR_UNSUPPORTED = 2,  /* valid but not built (e.g. a head dim above 128) */
  RBA_ERR_WORKSPACE = 3,    /* workspace smaller than *_workspace_size() */
  RBA_ERR_CUDA = 4,         /* a CUDA runtime call failed */
  RBA_ERR_TIMEOUT = 5,      /* a bounded device-side wait gave up (status word) */
  RBA_ERR_BOUNDS = 6        /* a device-side index check failed (status word) */
} rba_status;

typedef enum { RBA_F32 = 0, RBA_BF16 = 1 } rba_dtype;

/* How a block is represented for scoring ([ML] 2.3.2 memorisation). */
typedef enum {
  RBA_REP_MEAN = 0,         /* mean of the block's keys; rep pool fp32 [B][Hkv][cap_blocks][1][P] */
  RBA_REP_TOPR_ATTN = 1,    /* [IL] method: the n_rep keys that received the most attention from a
                               probe; rep pool dtype [B][Hkv][cap_blocks][n_rep][P], positions
                               int32 [B][Hkv][cap_blocks][n_rep] */
  RBA_REP_EXTERNAL = 2,     /* [LM] landmark keys given by the caller; rep pool dtype
                               [B][Hkv][cap_blocks][n_rep][P] */
  RBA_REP_EMBED_COSINE = 3, /* [ML] 2.2.2: L2-normalised chunk embedding; rep pool fp32
                               [B][cap_blocks][d_ret]; scored by cosine */
  RBA_REP_IDENTITY = 4      /* [RA]: block size 1, each key is its own representation; no rep pool */
} rba_rep_mode;

typedef struct {
  int32_t batch;            /* B */
  int32_t n_q_heads;        /* Hq (a multiple of n_kv_heads; q head i reads kv head i / (Hq/Hkv)) */
  int32_t n_kv_heads;       /* Hkv */
  int32_t head_dim;         /* D: a multiple of 4 up to 128; pool rows hold rba_row_pitch(D) */
  int32_t block_size;       /* bs >= 1 */
  int32_t n_rep;            /* r: representative keys per block (1 except RBA_REP_TOPR_ATTN / EXTERNAL) */
  int32_t d_ret;            /* embedding size (RBA_REP_EMBED_COSINE), else 0 */
  int64_t capacity_tokens;  /* tokens per (batch, kv head) the K/V pools hold (cap_blocks = cap / bs) */
  rba_dtype dtype;          /* storage type of q, K, V and (except fp32 pools above) rep keys */
  rba_rep_mode mode;
} rba_store_desc;

/* How the dot-product modes combine a block's n_rep representative keys into one
 * score (rba_store_set_score_reduce). */
typedef enum {
  RBA_SCORE_SUM = 0,  /* default: sum over the keys of the group-summed dot products */
  RBA_SCORE_MAX = 1   /* variant: the largest of the keys' group-summed dot products */
} rba_score_reduce;

/* Opaque: host-side description of caller-owned device pools. */
typedef struct rba_store rba_store;

/* Describe a block store ([ML] 2.2.2: memory = K-V pairs + representations).
 * P = rba_row_pitch(D) is the row length of every pool (P = D for D = 64 or 128).
 *   k_pool, v_pool  device, dtype [B][Hkv][capacity_tokens][P]
 *   rep_pool        device, layout per mode above (NULL for RBA_REP_IDENTITY)
 *   rep_pos         device int32 [B][Hkv][cap_blocks][n_rep] for RBA_REP_TOPR_ATTN (may be
 *                   NULL: positions are then not recorded), else ignored
 *   status_word     device int32[4], zeroed by the caller; first error code, where, detail
 *   out             host: receives the handle (free with rba_store_destroy)
 * Nothing is launched.  Errors: INVALID_ARG, UNSUPPORTED. */
rba_status rba_store_create(const rba_store_desc* desc, void* k_pool, void* v_pool,
                            void* rep_pool, int32_t* rep_pos, int32_t* status_word,
                            rba_store** out);
rba_status rba_store_destroy(rba_store* store);

/* Block-score variant of a store (host only; the default is RBA_SCORE_SUM).  With
 * RBA_SCORE_MAX, rba_score, rba_decode_step and rba_stream_step score candidate j as
 * max over the block's keys i of sum over the scoring q rows of q . rep_{j,i}: a block
 * as relevant as its most relevant representative token ([IL] method: units are
 * represented by their most-attended tokens; this reading weighs the best one alone).
 * Errors: INVALID_ARG (unknown value; RBA_SCORE_MAX on cosine or identity stores). */
rba_status rba_store_set_score_reduce(rba_store* store, int32_t reduce);

/* Bound, in nanoseconds, of every device-side wait of the one-launch decode step on
 * this store (host only; 0 restores the default of 2 s).  A wait that runs out
 * records RBA_ERR_TIMEOUT in the status word; the kernel then stops issuing work,
 * waits for its own copies in flight and returns, and every (batch, kv head) of the
 * call still leaves its synchronisation words zero, so the next call on the same
 * workspace runs normally.  Outputs of a call that timed out are undefined.  Meant
 * for tests of that path and for callers that prefer a short bound.
 * Errors: INVALID_ARG (NULL store). */
rba_status rba_store_set_wait_limit_ns(rba_store* store, uint64_t ns);

/* Whether rba_decode_step may run the whole step as one cooperative launch on this
 * store (host only; on = 1), where rba_decode_step_plan() then reports 3; 0 (the
 * default) keeps the three-kernel step.  On B200 the three-kernel step is the faster
 * of the two at the 128K-token InfLLM decode shape; the one-launch step is kept for
 * shapes and callers that prefer a single launch.  Results are the same either way
 * (same definitions; floating-point sums may differ in rounding order).
 * Errors: INVALID_ARG (NULL store, on not 0 or 1). */
rba_status rba_store_set_decode_step_one_launch(rba_store* store, int32_t on);

/* Candidate range for a store holding T tokens with the given sink/window
 * (host only; see the vocabulary above).  Errors: INVALID_ARG (tail block
 * outside the window, negative sizes, T > capacity). */
rba_status rba_candidates(const rba_store* store, int64_t T, int32_t sink, int32_t window,
                          int32_t* first_cand, int32_t* n_cand);

/* [ML] 2.3.2 memorisation M(k, v; r^m); [IL] method (representative tokens);
 * [LM] proposed method (landmarks).  Writes blocks [first_block,
 * first_block + n_blocks) of every (batch, kv head):
 *   k_src, v_src  device dtype [B][Hkv][n_blocks*bs][D], copied into the pools; both NULL when
 *                 the pools already hold those tokens (representations only)
 *   aux           RBA_REP_TOPR_ATTN: probe queries, device dtype [Hkv][n_aux][D]
 *                 RBA_REP_EXTERNAL:  landmark keys, device dtype [B][Hkv][n_blocks][n_rep][D]
 *                 RBA_REP_EMBED_COSINE: raw embeddings, device fp32 [B][n_blocks][d_ret]
 *                 otherwise NULL
 *   scale         logit scale for the probe softmax (RBA_REP_TOPR_ATTN), typically 1/sqrt(D)
 * RBA_REP_TOPR_ATTN: per probe query p, softmax over the block's bs tokens of
 * scale * p.k_t; a token's received attention is the sum over probes; the
 * n_rep tokens with the most (ties -> lower position) are kept in ascending
 * position.  RBA_REP_MEAN: (1/bs) sum_t k_t.  RBA_REP_EMBED_COSINE: e/|e|.
 * Errors: INVALID_ARG (range beyond capacity, missing aux), CUDA. */
rba_status rba_memorize(rba_store* store, const void* k_src, const void* v_src,
                        int64_t first_block, int32_t n_blocks, const void* aux, int32_t n_aux,
                        float scale, cudaStream_t stream);

/* Block scores ([ML] 2.3.2 cosine retrieval; [LM] query-landmark similarity;
 * [IL] relevance against representative tokens).
 *   dot modes: q device dtype [B][Hq][n_q][D]; for candidate c of (b, kv head h)
 *     scores[b][h][c] = sum over the group's q heads, over the n_q rows, and over the
 *     block's n_rep keys of q . rep  (n_q > 1: a prefill chunk shares one selection);
 *     with RBA_SCORE_MAX the sum over the keys becomes a max
 *   cosine mode: q = query embeddings, device fp32 [n_q][d_ret]; store batch must be 1;
 *     scores[i][c] = cos(q_i, M_{first_cand + c})
 *   scores  device fp32 [B][Hkv][nc] (dot) or [n_q][nc] (cosine)
 *   qsum_ws device fp32 [B][Hkv][D] scratch for the summed queries (dot modes; may be NULL
 *           when Hq/Hkv * n_q <= 64)
 * Errors: INVALID_ARG, CUDA. */
rba_status rba_score(const rba_store* store, const void* q, int32_t n_q, int64_t T,
                     int32_t sink, int32_t window, float* scores, float* qsum_ws,
                     cudaStream_t stream);

/* Top-k selection ([ML] 2.3.2 z^q = TopK{Cos(r^q)}; 2.3.4 the k most relevant
 * chunks).  For each of `rows` rows of n fp32 scores, the k best positions
 * under (larger score first, equal scores -> lower position first; -0 == +0),
 * written in ascending order as index_base + position.
 *   scores  device fp32 [rows][n];  idx  device int32 [rows][k]
 *   workspace / ws_bytes  device scratch, >= rba_topk_workspace_size(rows, n, k)
 * NaN scores are not supported.  Errors: INVALID_ARG (k > n), WORKSPACE, CUDA. */
rba_status rba_topk(const float* scores, int32_t rows, int32_t n, int32_t k, int32_t index_base,
                    int32_t* idx, void* workspace, size_t ws_bytes, cudaStream_t stream);
size_t rba_topk_workspace_size(int32_t rows, int32_t n, int32_t k);

/* Decode attention with online softmax and a log-sum-exp merge of partial
 * states ([IL] overall framework: local window + a few memory units; [ML]
 * 2.3.3 retrieved chunks attended without a causal mask).  Runs the
 * persistent attention kernel (one CTA per SM, bulk-copy staging) where
 * rba_decode_step_plan() would report 1 or 2, else a split-K kernel.
 *   q    device dtype [B][Hq][D];  idx device int32 [B][Hkv][k] ascending candidate block ids
 *   out  device fp32 [B][Hq][D];   lse device fp32 [B][Hq] (natural log) or NULL
 *   For q head i of kv head h = i / (Hq/Hkv):
 *     out = sum_t softmax_t(scale * q.k_t) v_t over the attended set of (b, h).
 *   workspace >= rba_attend_workspace_size(); its first 2 * roundup256(4 * B * Hkv) bytes
 *   (merge tickets) must be zero before the first call (the kernels leave them zero after
 *   each call that completes).
 * Errors: INVALID_ARG (k > nc, T > capacity), WORKSPACE, CUDA; out-of-range idx
 * entries are skipped and flagged as RBA_ERR_BOUNDS in the status word. */
rba_status rba_attend(const rba_store* store, const void* q, const int32_t* idx, int32_t k,
                      int64_t T, int32_t sink, int32_t window, float scale, float* out,
                      float* lse, void* workspace, size_t ws_bytes, cudaStream_t stream);
size_t rba_attend_workspace_size(const rba_store* store, int32_t k, int64_t T, int32_t sink,
                                 int32_t window);

/* rba_attend without a workspace argument, for callers that cannot allocate
 * device memory.  The pages have no counterpart: this is an interface addition
 * of this library.
 * Meant for hosts that own all device memory through their own allocator (for
 * example a serving engine that reserves HBM when it starts) and for call sites
 * that cannot afford the device-wide synchronisation cudaMalloc may cause.
 * Same computation, arguments, layouts and errors as rba_attend, always on the
 * split-K kernel; its split partials and merge tickets live in a fixed device
 * array inside the library,
 * RBA_ATTEND_NOALLOC_SCRATCH_BYTES long, which every GPU that loads the library
 * holds until the process exits.
 *   - Allocates nothing: no cudaMalloc / cudaFree and no allocating library call.
 *     The array itself is reserved by the CUDA driver when it loads the part of
 *     the library that holds it on a device: under lazy module loading (the
 *     default of recent CUDA releases) that happens at the first call on that
 *     device, otherwise when the library's kernels are loaded.
 *   - The first call on each device looks up the array's device address, with
 *     that device current; that lookup may load the module (above), which can
 *     reserve memory and synchronise.  Make the first call on each device at
 *     start-up: before any stream capture and outside latency-sensitive paths.
 *   - Each call zeroes the array's ticket region on `stream`, then launches.
 *   - Every call shares the one array, which keeps the last call's contents:
 *     calls that overlap on the GPU (other streams, other host threads) race and
 *     must be serialised by the caller.
 *   - A call whose split-K scratch exceeds the limit returns RBA_ERR_WORKSPACE and
 *     launches nothing. */
#define RBA_ATTEND_NOALLOC_SCRATCH_BYTES ((size_t)2 << 20)
rba_status rba_attend_noalloc(const rba_store* store, const void* q, const int32_t* idx,
                              int32_t k, int64_t T, int32_t sink, int32_t window, float scale,
                              float* out, float* lse, cudaStream_t stream);

/* Landmark-gated decode attention ([LM] proposed method: a block's landmark token
 * is the gate through which attention reaches the block).  The page gives no formula;
 * the reading taken: the landmark takes the block's place in the query's softmax.
 * For q head i of kv head h, with x_t = scale q . k_t:
 *   out = (sum_{t local} e^{x_t} v_t + sum_j e^{y_j} o_j) / Z,   lse = ln Z,
 *   local = sink U window tokens; j over the retrieved blocks idx[b][h][.];
 *   y_j = scale q . L_j with L_j the block's landmark key (the rep pool);
 *   o_j = sum over the block's tokens in [sink, w0) of softmax_block(x)_t v_t;
 *   Z = sum_{t local} e^{x_t} + sum_j e^{y_j}.
 * With every y_j equal to its block's log-sum-exp of x this is rba_attend.
 * RBA_REP_EXTERNAL stores with n_rep = 1.  Arguments and layouts as rba_attend
 * (no workspace).  Errors: INVALID_ARG, CUDA; out-of-range idx entries are skipped
 * and flagged as RBA_ERR_BOUNDS in the status word. */
rba_status rba_attend_landmark_gated(const rba_store* store, const void* q, const int32_t* idx,
                                     int32_t k, int64_t T, int32_t sink, int32_t window,
                                     float scale, float* out, float* lse, cudaStream_t stream);

/* Chunked prefill, retrieval-causal ([ML] 2.3.3 / Figure 3): every row of a
 * query chunk attends bidirectionally to sink U retrieved blocks U window of
 * the memory, and causally to the chunk's own tokens (own token i' visible to
 * row i iff i' <= i), in one joint softmax.  Tensor-core (tcgen05) tiles.
 *   q          device bf16 [n_chunks][Hq][chunk_len][D]
 *   idx        device int32 [n_chunks][n_sel][k], n_sel = 1 (one selection per chunk, all
 *              heads: cosine mode) or Hkv (one per kv head)
 *   chunk_k/v  device bf16 [n_chunks][Hkv][chunk_len][D]
 *   out        device fp32 [n_chunks][Hq][chunk_len][D];  lse fp32 [n_chunks][Hq][chunk_len] or NULL
 *   The store's batch is 1 (one memory shared by all chunks) or n_chunks.
 *   workspace >= rba_attend_prefill_workspace_size().
 *   Head dims between 64 and 128 run on 128-wide tiles: Q and the chunk's K/V are
 *   copied, zero-padded, into the workspace (counted by the size call).
 * Errors: INVALID_ARG, UNSUPPORTED (dtype other than bf16, D <= 64), WORKSPACE, CUDA. */
rba_status rba_attend_prefill(const rba_store* store, const void* q, int32_t n_chunks,
                              int32_t chunk_len, const int32_t* idx, int32_t n_sel, int32_t k,
                              int64_t T, int32_t sink, int32_t window, const void* chunk_k,
                              const void* chunk_v, float scale, float* out, float* lse,
                              void* workspace, size_t ws_bytes, cudaStream_t stream);
size_t rba_attend_prefill_workspace_size(const rba_store* store, int32_t n_chunks,
                                         int32_t chunk_len, int32_t n_sel, int32_t k, int64_t T,
                                         int32_t sink, int32_t window);

/* One whole decode step: rba_score (dot modes) -> rba_topk per (b, kv head)
 * -> rba_attend, with the same definitions as those calls, on `stream`.
 * Where rba_decode_step_plan() reports 3 it is ONE cooperative launch of one CTA
 * per SM: the CTAs of a (batch, kv head) score slices of its candidates, each
 * selects the head's top k once all slices are published, and they stream the
 * sink/window rows meanwhile and the selected rows after.  Where it reports 1 or
 * 2 it is three kernels, the top-k kernel and the persistent attention kernel
 * programmatic dependents of the kernel before them; else three kernels in
 * stream order.
 *   q device dtype [B][Hq][D]; idx device int32 [B][Hkv][k] (written); scores device fp32
 *   [B][Hkv][nc] (written) or NULL; out/lse as rba_attend.
 *   workspace >= rba_decode_step_workspace_size(); zero it before the first call (its
 *   synchronisation words must start at zero; every call that completes leaves them
 *   zero, and their offsets depend on the store only, so one workspace of the largest
 *   size serves calls of every geometry).
 * Errors: as the three calls. */
rba_status rba_decode_step(const rba_store* store, const void* q, int32_t k, int64_t T,
                           int32_t sink, int32_t window, float scale, float* scores,
                           int32_t* idx, float* out, float* lse, void* workspace,
                           size_t ws_bytes, cudaStream_t stream);
size_t rba_decode_step_workspace_size(const rba_store* store, int32_t k, int64_t T,
                                      int32_t sink, int32_t window);

/* How rba_decode_step runs this problem (host only; queries the device, launches nothing):
 *   3   the whole step in one cooperative launch (only after
 *       rba_store_set_decode_step_one_launch(store, 1)): bf16 store, block size a multiple of 64,
 *       head dim 64 or 128, GQA group of 1, 2 or 4, dot-mode representations (mean, top-r,
 *       landmark) with at most 8 keys per block, 1 <= k <= 256, at most 4096 candidates
 *       per (batch, kv head), at most half as many (batch, kv head) units as SMs, and a
 *       part's slice of representative keys within 64 KiB
 *   2   score -> top-k -> persistent attention kernel, the last two as programmatic
 *       dependents (overlapped); the attention kernel is the whole-block one: bf16 store,
 *       block size a multiple of 64, head dim 64 or 128; inner products on tensor cores
 *   1   as 2 with the CUDA-core attention kernel (other block sizes of at least 2, fp32);
 *       k <= 2048, GQA group of 1, 2 or 4 in both
 *   0   score -> top-k -> split-K attention, in stream order: outside those limits, and
 *       token-level stores (block size 1, where gathered loads beat per-row bulk copies)
 *  -2   within the limits but no CTA of the persistent kernel fits on an SM (as 0)
 *  -3   a CUDA error while asking (as 0)
 *  -4   invalid arguments (as rba_decode_step would report) */
int32_t rba_decode_step_plan(const rba_store* store, int32_t k, int64_t T, int32_t sink,
                             int32_t window);

/* Number of kernels rba_decode_step enqueues for this problem (host only, launches
 * nothing): 1 where rba_decode_step_plan() reports 3; else block scores and top-k (one
 * kernel for rows of up to 16384 candidates, four above; neither when k = 0), then one
 * attention kernel (persistent or split-K).  -4 for invalid arguments. */
int32_t rba_decode_step_launches(const rba_store* store, int32_t k, int64_t T, int32_t sink,
                                 int32_t window);

/* One step of streaming decode ([IL] overall framework: the newest tokens form
 * the local window and the tokens before it stay in memory as units that are
 * represented once; [ML] 2.3.2: a completed chunk is memorised).  The store
 * holds T tokens.  The call
 *   1. appends the new token's K and V (device dtype [B][Hkv][D]) at position T,
 *   2. if T + 1 is a multiple of the block size, memorises block (T + 1) / bs - 1
 *      from the pools (aux / n_aux as rba_memorize for one block: probe queries
 *      [Hkv][n_aux][D] for RBA_REP_TOPR_ATTN, the landmark keys [B][Hkv][1][n_rep][D]
 *      for RBA_REP_EXTERNAL, NULL for RBA_REP_MEAN and RBA_REP_IDENTITY),
 *   3. runs rba_decode_step for q over the T + 1 tokens with k' = min(k, candidates)
 *      blocks (written to *k_used when k_used is not NULL, host); idx is
 *      [B][Hkv][k'], out / lse as rba_decode_step.
 * The caller advances T by one per call.  Everything is enqueued on `stream`.
 *   workspace >= rba_decode_step_workspace_size(store, k, T + 1, sink, window).
 * Errors: INVALID_ARG (T + 1 above the capacity, cosine stores, invalid
 * geometry), and those of rba_memorize and rba_decode_step. */
rba_status rba_stream_step(rba_store* store, const void* q, const void* k_new,
                           const void* v_new, int64_t T, int32_t k, int32_t sink, int32_t window,
                           float scale, const void* aux, int32_t n_aux, int32_t* idx, float* out,
                           float* lse, int32_t* k_used, void* workspace, size_t ws_bytes,
                           cudaStream_t stream);

/* Two-stage approximate token retrieval for block size 1 ([RA] proposed method:
 * the few keys that matter are found by an approximate search that reads 1-3 % of
 * the keys instead of all of them).  The page names no index; this one is the
 * plainest the rest supports: consecutive groups of `group` tokens represented by
 * the mean of their keys.
 *
 * rba_group_means: the index.  For groups j in [first_group, first_group + n_groups)
 * of every (batch, kv head), means[b][h][j] = (1 / group) sum_t K[j * group + t]
 * (fp32).  RBA_REP_IDENTITY stores only.
 *   means  device fp32 [B][Hkv][capacity_tokens / group][P], caller-owned
 * Errors: INVALID_ARG (not an identity store, groups beyond the capacity), CUDA. */
rba_status rba_group_means(const rba_store* store, int64_t first_group, int32_t n_groups,
                           int32_t group, float* means, cudaStream_t stream);

/* rba_approx_select: per (batch, kv head), with the GQA group's queries summed
 *   stage 1  every candidate group (a full group meeting [sink, T - window)) scored
 *            by its mean; the best `groups_kept` kept (ties -> lower group);
 *   stage 2  every token of the kept groups that lies in [sink, T - window) scored
 *            exactly (q . k_t); the best k kept (ties -> lower token).
 * The keys read are one mean per candidate group plus the kept groups' tokens.
 * Attend over the result with rba_attend (block size 1: token ids are block ids).
 *   q           device dtype [B][Hq][D]
 *   means       device fp32 index from rba_group_means, covering the candidate groups
 *   idx         device int32 [B][Hkv][k], written: the selected tokens, ascending
 *   groups_out  device int32 [B][Hkv][groups_kept] (kept groups, ascending) or NULL
 *   scanned     device int32 [B][Hkv] (keys read) or NULL
 *   workspace >= rba_approx_select_workspace_size()
 * Requires groups_kept * group >= k + 2 * group (enough candidate tokens in any
 * kept set) and groups_kept <= the candidate groups.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA. */
rba_status rba_approx_select(const rba_store* store, const void* q, int64_t T, int32_t sink,
                             int32_t window, int32_t group, int32_t groups_kept, int32_t k,
                             const float* means, int32_t* idx, int32_t* groups_out,
                             int32_t* scanned, void* workspace, size_t ws_bytes,
                             cudaStream_t stream);
size_t rba_approx_select_workspace_size(const rba_store* store, int64_t T, int32_t sink,
                                        int32_t window, int32_t group, int32_t groups_kept,
                                        int32_t k);

/* Dynamic memory update ([ML] 2.3.2, dynamic memory update): retrieval
 * counters decide what the memory keeps once it overflows.  The newest entries
 * are kept, the oldest are dropped, and from the entries between them the
 * least retrieved are deleted until the requested number remains.
 *
 * Memory unit: the update and its counters are per (batch, kv head) for the
 * dot-product modes and per batch row for RBA_REP_EMBED_COSINE, whose bank
 * entry carries the K/V of every kv head.  rba_memory_units() reports the
 * count U (B * Hkv or B).  Entry = one block (one token when bs = 1).
 *
 * Counters: device uint32 [U][cap_blocks], caller-owned, zeroed before first use.
 * Element j of unit u counts how often block j of that unit has been selected.
 *
 * rba_memory_rule (host only): the page's proportions for n entries, with floor:
 *   keep_newest = n / 10, drop_oldest = n / 10, keep_total = n / 2. */
rba_status rba_memory_rule(int64_t n_entries, int64_t* keep_newest, int64_t* drop_oldest,
                           int64_t* keep_total);
int32_t rba_memory_units(const rba_store* store);  /* U, or -1 for a NULL store */

/* Adds a selection to the counters: every entry j of row r of idx (device int32
 * [rows][k], laid out [G][U][k] so that row r belongs to unit r % U -- a decode
 * step's [B][Hkv][k] for dot modes, a prefill's [n_chunks][n_sel][k] with a
 * batch-1 store, or one row per batch row for the cosine bank) adds one to
 * counters[r % U][j].  Entries outside [0, cap_blocks) are skipped and flagged
 * as RBA_ERR_BOUNDS in the status word.  Integer atomics: the result does not
 * depend on the order.  Errors: INVALID_ARG (rows not a multiple of U), CUDA. */
rba_status rba_count_retrievals(const rba_store* store, const int32_t* idx, int32_t rows,
                                int32_t k, uint32_t* counters, cudaStream_t stream);

/* Prunes and compacts the store in place.  The store holds T tokens: full blocks
 * [0, nb = T / bs) and a partial tail of T - nb * bs tokens.  Blocks [0,
 * pinned_blocks) (for example attention-sink blocks) are outside the rule and
 * never move.  The n = nb - pinned_blocks entries after them are updated:
 *   - the drop_oldest oldest entries are deleted;
 *   - the keep_newest newest entries are kept;
 *   - from the entries between them, the least retrieved are deleted (equal
 *     counts: the older entry first) until keep_total entries remain.
 * Kept entries stay in order at blocks pinned_blocks, pinned_blocks + 1, ...
 * Each moves with its K/V rows (every kv head of the unit), its representation,
 * its positions (RBA_REP_TOPR_ATTN) and its counter.  The tail's tokens follow
 * the kept blocks.  Counters of the vacated blocks up to the old tail's block
 * are zeroed.  *T_new (host, may be NULL) receives
 * (pinned_blocks + keep_total) * bs + tail.
 *   keep_map  device int32 [U][keep_total], written: keep_map[u][t] = the old index
 *             of the block now at pinned_blocks + t (may be NULL when keep_total = 0)
 * Requires 0 <= pinned_blocks <= nb, keep_newest + drop_oldest <= n and
 * keep_newest <= keep_total <= n - drop_oldest.  Launches one selection kernel,
 * ceil(keep_total / max(drop_oldest, 1)) move kernels of as even a share of the
 * destinations as possible (each moves entries that are at least drop_oldest
 * blocks from their destination, so no move overwrites a block that is still to
 * be read; a share too large for one grid is cut into several launches), and one
 * kernel for the tail and counters; every kernel after the selection is a
 * programmatic dependent of the one before it.
 * Errors: INVALID_ARG, UNSUPPORTED (nb >= 2^31 - 1), CUDA. */
rba_status rba_memory_update(rba_store* store, int64_t T, int32_t pinned_blocks,
                             int64_t keep_newest, int64_t drop_oldest, int64_t keep_total,
                             uint32_t* counters, int32_t* keep_map, int64_t* T_new,
                             cudaStream_t stream);

/* rba_decode_step from and to host memory: copies q_host (host, dtype [B][Hq][D]) into
 * q_dev, runs the step, copies out/lse/idx back into the host buffers (any of lse_host,
 * idx_host may be NULL), then synchronises `stream`.  q_dev, idx_dev, out_dev, lse_dev are
 * device buffers of the sizes above.  Pinned host memory makes the copies asynchronous.
 * Errors: as rba_decode_step, plus CUDA for the copies. */
rba_status rba_decode_step_host(const rba_store* store, const void* q_host, void* q_dev,
                                int32_t k, int64_t T, int32_t sink, int32_t window, float scale,
                                int32_t* idx_dev, float* out_dev, float* lse_dev,
                                float* out_host, float* lse_host, int32_t* idx_host,
                                void* workspace, size_t ws_bytes, cudaStream_t stream);

/* Synchronises `stream`, reads the store's status word, clears it, and returns
 * the first device-side error recorded since the last check (RBA_OK if none). */
rba_status rba_store_check(const rba_store* store, cudaStream_t stream);

/* Row pitch (elements) of the K/V and representation pools for a head dim D
 * (host only): 64 for D <= 64, else 128; -1 for an unsupported D (not a multiple
 * of 4, or above 128).  Pools hold each row in `pitch` elements: the first D are
 * the row, the rest are padding that must hold zeros (the library's own writes
 * -- rba_memorize, rba_stream_step, rba_memory_update -- keep them zero).  Every
 * other tensor of the interface (q, out, K/V and key inputs, prefill chunks) is
 * dense with rows of D elements. */
int32_t rba_row_pitch(int32_t head_dim);

const char* rba_status_string(rba_status status);
int32_t rba_version(void);

#ifdef __cplusplus
}
#endif
#endif /* RBA_H_ */
