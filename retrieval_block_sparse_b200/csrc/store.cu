// Block store description, candidate geometry, status handling.
#include <atomic>
#include <mutex>
#include <new>
#include <unordered_map>

#include "rba_internal.cuh"

namespace rba {

rba_status geometry(const rba_store* st, int64_t T, int32_t sink, int32_t window, Geometry* g) {
  if (st == nullptr || g == nullptr) return RBA_ERR_INVALID_ARG;
  const int32_t bs = st->d.block_size;
  if (T < 0 || sink < 0 || window < 0 || T > st->d.capacity_tokens) return RBA_ERR_INVALID_ARG;
  const int64_t w0 = T > window ? T - window : 0;
  const int64_t nb = T / bs;
  if (nb > INT32_MAX) return RBA_ERR_INVALID_ARG;
  // the partial tail block must lie inside the window
  if (T - nb * bs > window) return RBA_ERR_INVALID_ARG;
  // candidate j: full, (j+1)*bs > sink and j*bs < w0
  const int64_t lo = sink / bs;
  int64_t hi = (w0 + bs - 1) / bs;
  if (hi > nb) hi = nb;
  g->T = T;
  g->bs = bs;
  g->sink = sink;
  g->sink_end = static_cast<int32_t>(sink < w0 ? sink : w0);
  g->w0 = w0;
  g->nb = static_cast<int32_t>(nb);
  g->first = static_cast<int32_t>(lo < hi ? lo : 0);
  g->nc = static_cast<int32_t>(hi > lo ? hi - lo : 0);
  return RBA_OK;
}

// SM count of the current device, cached per device (devices may differ).
int num_sms() {
  constexpr int kDevices = 64;
  static std::atomic<int> cached[kDevices];  // 0: not looked up yet
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev < 0 || dev >= kDevices) {
    int n = 0;
    return cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0
               ? n
               : 148;
  }
  int n = cached[dev].load(std::memory_order_relaxed);
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev].store(n, std::memory_order_relaxed);
  }
  return n;
}

cudaError_t ensure_smem(const void* kernel, size_t bytes) {
  if (bytes <= 48 * 1024) return cudaSuccess;
  static std::mutex mu;
  static std::unordered_map<uint64_t, size_t> done;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t key = reinterpret_cast<uint64_t>(kernel) ^ (uint64_t(dev) << 56);
  std::lock_guard<std::mutex> lock(mu);
  auto it = done.find(key);
  if (it != done.end() && it->second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(bytes));
  if (e == cudaSuccess) done[key] = bytes;
  return e;
}

int occupancy(const void* kernel, int threads, size_t smem) {
  static std::mutex mu;
  static std::unordered_map<uint64_t, int> done;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  const uint64_t key = reinterpret_cast<uint64_t>(kernel) ^ (uint64_t(dev) << 56) ^
                       (uint64_t(smem) << 20) ^ uint64_t(threads);
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = done.find(key);
    if (it != done.end()) return it->second;
  }
  if (ensure_smem(kernel, smem) != cudaSuccess) {
    (void)cudaGetLastError();
    return -1;
  }
  int occ = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kernel, threads, smem) != cudaSuccess) {
    (void)cudaGetLastError();
    return -1;
  }
  std::lock_guard<std::mutex> lock(mu);
  done[key] = occ;
  return occ;
}

}  // namespace rba

extern "C" {

rba_status rba_store_create(const rba_store_desc* d, void* k_pool, void* v_pool, void* rep_pool,
                            int32_t* rep_pos, int32_t* status_word, rba_store** out) {
  if (d == nullptr || out == nullptr) return RBA_ERR_INVALID_ARG;
  *out = nullptr;
  if (d->batch <= 0 || d->n_q_heads <= 0 || d->n_kv_heads <= 0 || d->block_size <= 0 ||
      d->n_rep <= 0 || d->capacity_tokens <= 0 || d->n_q_heads % d->n_kv_heads != 0)
    return RBA_ERR_INVALID_ARG;
  if (d->dtype != RBA_F32 && d->dtype != RBA_BF16) return RBA_ERR_INVALID_ARG;
  if (rba::pool_pitch(d->head_dim) < 0) return RBA_ERR_UNSUPPORTED;
  if (k_pool == nullptr || v_pool == nullptr) return RBA_ERR_INVALID_ARG;
  if (d->capacity_tokens >= (int64_t(1) << 31)) return RBA_ERR_INVALID_ARG;
  switch (d->mode) {
    case RBA_REP_MEAN:
      if (d->n_rep != 1 || rep_pool == nullptr) return RBA_ERR_INVALID_ARG;
      break;
    case RBA_REP_TOPR_ATTN:
      if (rep_pool == nullptr || d->n_rep > d->block_size || d->n_rep > 32 ||
          d->block_size > 1024)
        return RBA_ERR_INVALID_ARG;
      break;
    case RBA_REP_EXTERNAL:
      if (rep_pool == nullptr || d->n_rep > 32) return RBA_ERR_INVALID_ARG;
      break;
    case RBA_REP_EMBED_COSINE:
      if (rep_pool == nullptr || d->d_ret <= 0 || d->d_ret % 4 != 0 || d->d_ret > 8192 ||
          d->n_rep != 1)
        return RBA_ERR_INVALID_ARG;
      break;
    case RBA_REP_IDENTITY:
      if (d->block_size != 1 || d->n_rep != 1) return RBA_ERR_INVALID_ARG;
      break;
    default:
      return RBA_ERR_INVALID_ARG;
  }
  rba_store* s = new (std::nothrow) rba_store;
  if (s == nullptr) return RBA_ERR_INVALID_ARG;
  s->d = *d;
  s->pitch = rba::pool_pitch(d->head_dim);
  s->k = k_pool;
  s->v = v_pool;
  s->rep = rep_pool;
  s->rep_pos = rep_pos;
  s->status = status_word;
  s->cap_blocks = d->capacity_tokens / d->block_size;
  s->score_reduce = RBA_SCORE_SUM;
  s->wait_ns = rba::kDefaultWaitNs;
  s->one_launch = 0;
  *out = s;
  return RBA_OK;
}

rba_status rba_store_destroy(rba_store* store) {
  delete store;
  return RBA_OK;
}

rba_status rba_candidates(const rba_store* store, int64_t T, int32_t sink, int32_t window,
                          int32_t* first_cand, int32_t* n_cand) {
  rba::Geometry g;
  rba_status s = rba::geometry(store, T, sink, window, &g);
  if (s != RBA_OK) return s;
  if (first_cand) *first_cand = g.first;
  if (n_cand) *n_cand = g.nc;
  return RBA_OK;
}

rba_status rba_store_check(const rba_store* store, cudaStream_t stream) {
  if (store == nullptr) return RBA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize(stream) != cudaSuccess) return RBA_ERR_CUDA;
  if (store->status == nullptr) return RBA_OK;
  int32_t h[4] = {0, 0, 0, 0};
  if (cudaMemcpy(h, store->status, sizeof(h), cudaMemcpyDeviceToHost) != cudaSuccess)
    return RBA_ERR_CUDA;
  if (h[0] != 0) {
    if (cudaMemset(store->status, 0, sizeof(h)) != cudaSuccess) return RBA_ERR_CUDA;
    return static_cast<rba_status>(h[0]);
  }
  return RBA_OK;
}

int32_t rba_row_pitch(int32_t head_dim) { return rba::pool_pitch(head_dim); }

const char* rba_status_string(rba_status s) {
  switch (s) {
    case RBA_OK: return "ok";
    case RBA_ERR_INVALID_ARG: return "invalid argument";
    case RBA_ERR_UNSUPPORTED: return "unsupported configuration";
    case RBA_ERR_WORKSPACE: return "workspace too small";
    case RBA_ERR_CUDA: return "CUDA runtime error";
    case RBA_ERR_TIMEOUT: return "bounded device wait timed out";
    case RBA_ERR_BOUNDS: return "device-side index out of range";
  }
  return "unknown status";
}

int32_t rba_version(void) { return 100; }

}  // extern "C"

extern "C" rba_status rba_store_set_wait_limit_ns(rba_store* st, uint64_t ns) {
  if (st == nullptr) return RBA_ERR_INVALID_ARG;
  st->wait_ns = ns == 0 ? rba::kDefaultWaitNs : ns;
  return RBA_OK;
}

extern "C" rba_status rba_store_set_decode_step_one_launch(rba_store* st, int32_t on) {
  if (st == nullptr || (on != 0 && on != 1)) return RBA_ERR_INVALID_ARG;
  st->one_launch = on;
  return RBA_OK;
}

extern "C" rba_status rba_store_set_score_reduce(rba_store* st, int32_t reduce) {
  if (st == nullptr || (reduce != RBA_SCORE_SUM && reduce != RBA_SCORE_MAX))
    return RBA_ERR_INVALID_ARG;
  if (reduce == RBA_SCORE_MAX && (st->d.mode == RBA_REP_EMBED_COSINE ||
                                  st->d.mode == RBA_REP_IDENTITY))
    return RBA_ERR_INVALID_ARG;
  st->score_reduce = reduce;
  return RBA_OK;
}
