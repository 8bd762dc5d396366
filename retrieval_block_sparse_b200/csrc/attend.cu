// Split-K decode attention over sink U retrieved blocks U window, and the
// whole decode step (score -> top-k -> attend).
//
// InfLLM article, "overall framework" (local window plus a few memory units
// per step); MemLong summary, 2.3.3 (retrieved chunks attended without a
// causal mask); every split computes an online softmax over its share of the
// attended tokens and the last CTA of each (batch, kv head) merges the split
// partials by log-sum-exp (no CTA ever waits for another).
#include "attend_impl.cuh"
#include "decode_fused.cuh"
#include "decode_step.cuh"
#include "score_impl.cuh"
#include "topk_impl.cuh"

namespace rba {
namespace {

template <typename T, int D, int G>
__global__ void __launch_bounds__(kAttendThreads, 1) attend_decode_kernel(AttendArgs a) {
  using C = DecodeTile<T, D>;
  extern __shared__ __align__(16) char smem[];
  char* stages = smem;
  float* red = reinterpret_cast<float*>(smem + C::NS * C::STAGE);
  int* sstart = reinterpret_cast<int*>(red + kAttendWarps * G * (D + 2));
  int* svstart = sstart + (a.k + 2);
  float* wsm = reinterpret_cast<float*>(svstart + a.k + 3);
  __shared__ int s_warp[32];
  __shared__ bool s_last;
  const int split = blockIdx.x, bh = blockIdx.y;
  const int nseg = a.k + 2;
  const int n_att = build_segments(a, bh, sstart, svstart, s_warp);
  // token-level retrieval with every selected token in place: direct mapping
  const bool unit = a.bs == 1 && svstart[nseg - 1] == svstart[1] + a.k;
  const int v_lo = static_cast<int>(int64_t(n_att) * split / a.nsplit);
  const int v_hi = static_cast<int>(int64_t(n_att) * (split + 1) / a.nsplit);
  const int ntiles = (v_hi - v_lo + C::TT - 1) / C::TT;
  const int64_t row0 = int64_t(bh) * a.cap;
  LaneState<T, D, G> st;
  load_q<T, D, G>(a, bh, st);
#pragma unroll
  for (int s = 0; s < C::NS - 1; ++s) {
    if (s < ntiles)
      issue_tile<T, D>(a, row0, stages + s * C::STAGE, sstart, svstart, nseg, v_lo + s * C::TT,
                       v_hi, unit);
    cp_async_commit();
  }
  for (int t = 0; t < ntiles; ++t) {
    const int tn = t + C::NS - 1;
    if (tn < ntiles)
      issue_tile<T, D>(a, row0, stages + (tn % C::NS) * C::STAGE, sstart, svstart, nseg,
                       v_lo + tn * C::TT, v_hi, unit);
    cp_async_commit();
    cp_async_wait<C::NS - 1>();
    __syncthreads();
    consume_tile<T, D, G>(stages + (t % C::NS) * C::STAGE, min(C::TT, v_hi - v_lo - t * C::TT),
                          st, threadIdx.x >> 5);
    __syncthreads();
  }
  write_partial<T, D, G>(a, bh, split, st, red);
  merge_partials_last<D, G>(a, bh, wsm, &s_last);
}

template <typename T, int D, int G>
rba_status launch_t(const AttendArgs& a, int BH, cudaStream_t stream) {
  using C = DecodeTile<T, D>;
  const size_t smem = size_t(C::NS) * C::STAGE + size_t(kAttendWarps) * G * (D + 2) * 4 +
                      size_t(2 * a.k + 5) * 4 + size_t(G) * a.nsplit * 4 + 16;
  if (smem > 227 * 1024) return RBA_ERR_UNSUPPORTED;
  auto kfn = attend_decode_kernel<T, D, G>;
  RBA_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(kfn), smem));
  kfn<<<dim3(a.nsplit, BH), kAttendThreads, smem, stream>>>(a);
  RBA_LAUNCH_CHECK();
  return RBA_OK;
}

template <typename T, int D>
rba_status dispatch_g(const AttendArgs& a, int G, int BH, cudaStream_t s) {
  switch (G) {
    case 1: return launch_t<T, D, 1>(a, BH, s);
    case 2: return launch_t<T, D, 2>(a, BH, s);
    case 4: return launch_t<T, D, 4>(a, BH, s);
  }
  return RBA_ERR_UNSUPPORTED;
}

int64_t n_att_bound(const Geometry& g, int k) {
  return int64_t(g.sink_end) + (g.T - g.w0) + int64_t(k) * g.bs;
}

struct AttendWs {
  uint32_t* tickets;
  float* part;
  size_t bytes;
};

AttendWs attend_layout(void* ws, int BH, int Hq_total, int D, int nsplit) {
  AttendWs w;
  char* p = static_cast<char*>(ws);
  const size_t tb = align_up(size_t(BH) * 4, 256);
  w.tickets = reinterpret_cast<uint32_t*>(p);
  w.part = reinterpret_cast<float*>(p + tb);
  w.bytes = tb + align_up(size_t(Hq_total) * nsplit * (D + 2) * 4, 256);
  return w;
}

}  // namespace

int attend_nsplit(int BH, int64_t n_att_max) {
  int ns = num_sms() / (BH > 0 ? BH : 1);
  if (ns < 1) ns = 1;
  const int64_t by_len = n_att_max / 64;
  if (ns > by_len) ns = static_cast<int>(by_len < 1 ? 1 : by_len);
  return ns;
}

size_t attend_workspace_bytes(int BH, int Hq_total, int D, int nsplit) {
  return attend_layout(nullptr, BH, Hq_total, D, nsplit).bytes;
}

size_t splitk_workspace_bytes(const rba_store* st, const Geometry& g, int k) {
  const int BH = st->d.batch * st->d.n_kv_heads;
  const int nsplit = attend_nsplit(BH, n_att_bound(g, k));
  return attend_workspace_bytes(BH, st->d.batch * st->d.n_q_heads, st->pitch, nsplit);
}

rba_status launch_attend(const rba_store* st, const void* q, const int32_t* idx, int k,
                         const Geometry& g, float scale, float* out, float* lse, void* ws,
                         size_t ws_bytes, cudaStream_t stream) {
  const rba_store_desc& d = st->d;
  const int BH = d.batch * d.n_kv_heads;
  const int G = d.n_q_heads / d.n_kv_heads;
  const int nsplit = attend_nsplit(BH, n_att_bound(g, k));
  AttendWs w = attend_layout(ws, BH, d.batch * d.n_q_heads, st->pitch, nsplit);
  if (ws == nullptr || ws_bytes < w.bytes) return RBA_ERR_WORKSPACE;
  AttendArgs a;
  a.K = st->k;
  a.V = st->v;
  a.q = q;
  a.idx = idx;
  a.out = out;
  a.lse = lse;
  a.part = w.part;
  a.tickets = w.tickets;
  a.status = st->status;
  a.cap = d.capacity_tokens;
  a.T = g.T;
  a.w0 = g.w0;
  a.Hq = d.n_q_heads;
  a.Hkv = d.n_kv_heads;
  a.k = k;
  a.bs = d.block_size;
  a.sink = g.sink;
  a.sink_end = g.sink_end;
  a.nsplit = nsplit;
  a.first = g.first;
  a.nc = g.nc;
  a.qd = d.head_dim;
  a.scale_log2 = scale * 1.4426950408889634f;
  if (d.dtype == RBA_BF16) {
    if (st->pitch == 128) return dispatch_g<__nv_bfloat16, 128>(a, G, BH, stream);
    return dispatch_g<__nv_bfloat16, 64>(a, G, BH, stream);
  }
  if (st->pitch == 128) return dispatch_g<float, 128>(a, G, BH, stream);
  return dispatch_g<float, 64>(a, G, BH, stream);
}

namespace {

// Attention workspace: [persistent-kernel tickets (zero)] [split-K tickets
// (zero) + partials] [persistent-kernel partial slots].  The zero words of
// the two kernels never overlap the other kernel's scratch.
struct AttendLayout {
  void* fused_sync;
  float* fused_slots;
  void* splitk_ws;
  size_t splitk_bytes;
  size_t total;
};

AttendLayout attend_layout_full(void* ws, const rba_store* st, const Geometry& g, int k) {
  const rba_store_desc& d = st->d;
  const int BH = d.batch * d.n_kv_heads;
  AttendLayout l;
  char* p = static_cast<char*>(ws);
  size_t off = 0;
  l.fused_sync = p + off;
  off += fused_sync_bytes(st);
  const int nsplit = attend_nsplit(BH, n_att_bound(g, k));
  l.splitk_bytes = attend_workspace_bytes(BH, d.batch * d.n_q_heads, st->pitch, nsplit);
  l.splitk_ws = p + off;
  off += align_up(l.splitk_bytes, 256);
  l.fused_slots = reinterpret_cast<float*>(p + off);
  if (fused_eligible(st, g, k)) off += fused_slot_bytes(st, g, k, nullptr);
  l.total = off;
  return l;
}

bool use_fused(const rba_store* st, const Geometry& g, int k) {
  return fused_eligible(st, g, k) && fused_occupancy(st) > 0;
}

// Attention over sink U selected blocks U window: the persistent kernel
// where it applies (pdl: behind the top-k kernel), else split-K.
rba_status attend_any(const rba_store* st, const void* q, const int32_t* idx, int k,
                      const Geometry& g, float scale, float* out, float* lse,
                      const AttendLayout& l, bool pdl, cudaStream_t stream) {
  if (use_fused(st, g, k)) {
    const rba_status s =
        launch_fused(st, q, k, g, scale, idx, out, lse, l.fused_sync, l.fused_slots, pdl, stream);
    if (s != RBA_ERR_UNSUPPORTED) return s;
  }
  return launch_attend(st, q, idx, k, g, scale, out, lse, l.splitk_ws, l.splitk_bytes, stream);
}

struct StepWs {
  AttendLayout att;
  bool one_launch;      // the one-launch decode step covers the problem
  void* step_sync;      // its synchronisation words (zero between calls)
  float* step_slots;    // its partial-state slots
  float* scores;
  void* topk_ws;
  size_t topk_bytes;
  size_t total;
};

// [one-launch step: sync words] [attention workspace] [one-launch step: slots]
// [scores] [top-k scratch].  The zero words (the step's, then the attention
// kernels' at the start of the attention workspace) sit at offsets that
// depend on the store alone, so calls of any geometry on one workspace agree
// on them.
StepWs step_layout(void* ws, const rba_store* st, const Geometry& g, int k, bool own_scores) {
  const int BH = st->d.batch * st->d.n_kv_heads;
  StepWs s;
  char* p = static_cast<char*>(ws);
  s.step_sync = p;
  size_t off = step_sync_bytes(st);
  s.att = attend_layout_full(p + off, st, g, k);
  off += align_up(s.att.total, 256);
  s.one_launch = step_eligible(st, g, k);
  s.step_slots = nullptr;
  if (s.one_launch) {
    s.step_slots = reinterpret_cast<float*>(p + off);
    off += step_slot_bytes(st);
  }
  s.scores = nullptr;
  if (own_scores) {
    s.scores = reinterpret_cast<float*>(p + off);
    off += align_up(size_t(BH) * (g.nc > 0 ? g.nc : 1) * 4, 256);
  }
  s.topk_bytes = topk_workspace(BH, g.nc, k);
  s.topk_ws = p + off;
  off += align_up(s.topk_bytes, 256);
  s.total = off;
  return s;
}

}  // namespace
}  // namespace rba

extern "C" {

rba_status rba_attend(const rba_store* st, const void* q, const int32_t* idx, int32_t k,
                      int64_t T, int32_t sink, int32_t window, float scale, float* out,
                      float* lse, void* workspace, size_t ws_bytes, cudaStream_t stream) {
  using namespace rba;
  if (st == nullptr || q == nullptr || out == nullptr || k < 0) return RBA_ERR_INVALID_ARG;
  if (st->d.mode == RBA_REP_EMBED_COSINE) return RBA_ERR_INVALID_ARG;
  Geometry g;
  rba_status s = geometry(st, T, sink, window, &g);
  if (s != RBA_OK) return s;
  if (k > g.nc || (k > 0 && idx == nullptr)) return RBA_ERR_INVALID_ARG;
  const AttendLayout l = attend_layout_full(workspace, st, g, k);
  if (workspace == nullptr || ws_bytes < l.total) return RBA_ERR_WORKSPACE;
  return attend_any(st, q, idx, k, g, scale, out, lse, l, false, stream);
}

size_t rba_attend_workspace_size(const rba_store* st, int32_t k, int64_t T, int32_t sink,
                                 int32_t window) {
  using namespace rba;
  Geometry g;
  if (st == nullptr || geometry(st, T, sink, window, &g) != RBA_OK || k < 0) return 0;
  return attend_layout_full(nullptr, st, g, k).total;
}

rba_status rba_decode_step(const rba_store* st, const void* q, int32_t k, int64_t T,
                           int32_t sink, int32_t window, float scale, float* scores,
                           int32_t* idx, float* out, float* lse, void* workspace,
                           size_t ws_bytes, cudaStream_t stream) {
  using namespace rba;
  if (st == nullptr || q == nullptr || out == nullptr || k < 0 || (k > 0 && idx == nullptr))
    return RBA_ERR_INVALID_ARG;
  if (st->d.mode == RBA_REP_EMBED_COSINE) return RBA_ERR_INVALID_ARG;
  Geometry g;
  rba_status s = geometry(st, T, sink, window, &g);
  if (s != RBA_OK) return s;
  if (k > g.nc) return RBA_ERR_INVALID_ARG;
  StepWs w = step_layout(workspace, st, g, k, scores == nullptr);
  if (workspace == nullptr || ws_bytes < w.total) return RBA_ERR_WORKSPACE;
  float* sc = scores != nullptr ? scores : w.scores;
  const int BH = st->d.batch * st->d.n_kv_heads;
  const int grp = st->d.n_q_heads / st->d.n_kv_heads;
  if (grp > 64) return RBA_ERR_UNSUPPORTED;
  if (w.one_launch)  // the whole step in one cooperative launch
    return launch_step(st, q, k, g, scale, sc, idx, out, lse, w.step_sync, w.step_slots, stream);
  // score -> top-k -> attention; the top-k kernel and the persistent
  // attention kernel start early (programmatic dependent launch) and wait
  // for their inputs on the device
  const bool fused = use_fused(st, g, k);
  if (k > 0) {
    // before the persistent kernel: at most one score CTA per SM, so that
    // some SMs are empty from the start and the score CTAs retire together;
    // the attention CTAs (which cannot share an SM with a score CTA: their
    // registers fill an SM sub-partition) then start earlier and stream the
    // sink/window rows while the top-k runs (128K step 21.5 -> 20.8 us)
    s = launch_score_dot(st, q, 1, nullptr, g, sc, stream, fused ? 1 : 4);
    if (s != RBA_OK) return s;
    s = launch_topk(sc, BH, g.nc, k, g.first, idx, w.topk_ws, w.topk_bytes, stream, fused);
    if (s != RBA_OK) return s;
  }
  return attend_any(st, q, idx, k, g, scale, out, lse, w.att, fused && k > 0, stream);
}

rba_status rba_stream_step(rba_store* st, const void* q, const void* k_new, const void* v_new,
                           int64_t T, int32_t k, int32_t sink, int32_t window, float scale,
                           const void* aux, int32_t n_aux, int32_t* idx, float* out, float* lse,
                           int32_t* k_used, void* workspace, size_t ws_bytes,
                           cudaStream_t stream) {
  using namespace rba;
  if (st == nullptr || q == nullptr || k_new == nullptr || v_new == nullptr || T < 0 || k < 0)
    return RBA_ERR_INVALID_ARG;
  const rba_store_desc& d = st->d;
  if (d.mode == RBA_REP_EMBED_COSINE) return RBA_ERR_INVALID_ARG;
  if (T + 1 > d.capacity_tokens) return RBA_ERR_INVALID_ARG;
  // the step's geometry first: nothing is launched if it is invalid
  Geometry g;
  rba_status s = geometry(st, T + 1, sink, window, &g);
  if (s != RBA_OK) return s;
  const int32_t ke = k < g.nc ? k : g.nc;  // early in a stream fewer blocks are candidates
  if (k_used != nullptr) *k_used = ke;
  // 1. the new token's K and V at position T of every (batch, kv head)
  // (the new rows are head_dim long; pool rows are st->pitch long, their
  // padding columns stay zero)
  const size_t row = size_t(d.head_dim) * dtype_size(d.dtype);
  const size_t prow = size_t(st->pitch) * dtype_size(d.dtype);
  const size_t rows = size_t(d.batch) * d.n_kv_heads;
  const size_t pitch = size_t(d.capacity_tokens) * prow;
  char* kdst = static_cast<char*>(st->k) + size_t(T) * prow;
  char* vdst = static_cast<char*>(st->v) + size_t(T) * prow;
  RBA_CUDA_TRY(cudaMemcpy2DAsync(kdst, pitch, k_new, row, row, rows, cudaMemcpyDeviceToDevice,
                                 stream));
  RBA_CUDA_TRY(cudaMemcpy2DAsync(vdst, pitch, v_new, row, row, rows, cudaMemcpyDeviceToDevice,
                                 stream));
  // 2. the block this token completes becomes a memory unit: its representation
  if ((T + 1) % d.block_size == 0 && d.mode != RBA_REP_IDENTITY) {
    s = rba_memorize(st, nullptr, nullptr, (T + 1) / d.block_size - 1, 1, aux, n_aux, scale,
                     stream);
    if (s != RBA_OK) return s;
  }
  // 3. the decode step over the T + 1 tokens
  return rba_decode_step(st, q, ke, T + 1, sink, window, scale, nullptr, idx, out, lse,
                         workspace, ws_bytes, stream);
}

int32_t rba_decode_step_plan(const rba_store* st, int32_t k, int64_t T, int32_t sink,
                             int32_t window) {
  using namespace rba;
  Geometry g;
  if (st == nullptr || k < 0 || geometry(st, T, sink, window, &g) != RBA_OK || k > g.nc)
    return -4;
  if (step_eligible(st, g, k)) return 3;
  if (!fused_eligible(st, g, k)) return 0;
  const int occ = fused_occupancy(st);
  if (occ < 0) return -3;
  if (occ == 0) return -2;
  return fused_whole_blocks(st) ? 2 : 1;
}

int32_t rba_decode_step_launches(const rba_store* st, int32_t k, int64_t T, int32_t sink,
                                 int32_t window) {
  using namespace rba;
  Geometry g;
  if (st == nullptr || k < 0 || geometry(st, T, sink, window, &g) != RBA_OK || k > g.nc)
    return -4;
  if (step_eligible(st, g, k)) return 1;  // the whole step in one launch
  int32_t n = 0;
  if (k > 0) n += 1 + (g.nc <= kSmallN ? 1 : 4);  // scores; top-k (one kernel, or four)
  return n + 1;  // the attention kernel (persistent or split-K)
}

size_t rba_decode_step_workspace_size(const rba_store* st, int32_t k, int64_t T, int32_t sink,
                                      int32_t window) {
  using namespace rba;
  Geometry g;
  if (st == nullptr || geometry(st, T, sink, window, &g) != RBA_OK || k < 0) return 0;
  return step_layout(nullptr, st, g, k, true).total;
}

rba_status rba_decode_step_host(const rba_store* st, const void* q_host, void* q_dev, int32_t k,
                                int64_t T, int32_t sink, int32_t window, float scale,
                                int32_t* idx_dev, float* out_dev, float* lse_dev,
                                float* out_host, float* lse_host, int32_t* idx_host,
                                void* workspace, size_t ws_bytes, cudaStream_t stream) {
  using namespace rba;
  if (st == nullptr || q_host == nullptr || q_dev == nullptr || out_host == nullptr)
    return RBA_ERR_INVALID_ARG;
  const rba_store_desc& d = st->d;
  const size_t q_bytes = size_t(d.batch) * d.n_q_heads * d.head_dim * dtype_size(d.dtype);
  RBA_CUDA_TRY(cudaMemcpyAsync(q_dev, q_host, q_bytes, cudaMemcpyHostToDevice, stream));
  rba_status s = rba_decode_step(st, q_dev, k, T, sink, window, scale, nullptr, idx_dev, out_dev,
                                 lse_dev, workspace, ws_bytes, stream);
  if (s != RBA_OK) return s;
  const size_t rows = size_t(d.batch) * d.n_q_heads;
  RBA_CUDA_TRY(cudaMemcpyAsync(out_host, out_dev, rows * d.head_dim * 4, cudaMemcpyDeviceToHost,
                               stream));
  if (lse_host != nullptr && lse_dev != nullptr)
    RBA_CUDA_TRY(cudaMemcpyAsync(lse_host, lse_dev, rows * 4, cudaMemcpyDeviceToHost, stream));
  if (idx_host != nullptr)
    RBA_CUDA_TRY(cudaMemcpyAsync(idx_host, idx_dev, size_t(d.batch) * d.n_kv_heads * k * 4,
                                 cudaMemcpyDeviceToHost, stream));
  RBA_CUDA_TRY(cudaStreamSynchronize(stream));
  return RBA_OK;
}

}  // extern "C"
