// Chunked prefill, retrieval-causal attention (MemLong summary, 2.3.3 and
// Figure 3): every row of a query chunk attends bidirectionally to the
// retrieved past tokens and causally to its own chunk, in one softmax.
#include "rba_internal.cuh"

extern "C" {

rba_status rba_attend_prefill(const rba_store* st, const void* q, int32_t n_chunks,
                              int32_t chunk_len, const int32_t* idx, int32_t n_sel, int32_t k,
                              int64_t T, int32_t sink, int32_t window, const void* chunk_k,
                              const void* chunk_v, float scale, float* out, float* lse,
                              void* workspace, size_t ws_bytes, cudaStream_t stream) {
  (void)st; (void)q; (void)n_chunks; (void)chunk_len; (void)idx; (void)n_sel; (void)k; (void)T;
  (void)sink; (void)window; (void)chunk_k; (void)chunk_v; (void)scale; (void)out; (void)lse;
  (void)workspace; (void)ws_bytes; (void)stream;
  return RBA_ERR_UNSUPPORTED;
}

size_t rba_attend_prefill_workspace_size(const rba_store* st, int32_t n_chunks,
                                         int32_t chunk_len, int32_t n_sel, int32_t k, int64_t T,
                                         int32_t sink, int32_t window) {
  (void)st; (void)n_chunks; (void)chunk_len; (void)n_sel; (void)k; (void)T; (void)sink;
  (void)window;
  return 0;
}

}  // extern "C"
