// Two-stage approximate token retrieval for block size 1.
//
// RetrievalAttention summary (arXiv 2409.10516), "proposed method": a query
// attends over the few keys that matter, found by an approximate search that
// reads 1-3% of the keys instead of all of them.  The page names no index;
// the one built here is the plainest the rest supports:
//   index    consecutive groups of `group` tokens, each represented by the
//            mean of its keys (fp32), built once as tokens arrive;
//   stage 1  every candidate group (a full group meeting [sink, T - window))
//            scored by its mean against the summed GQA query; the best
//            `groups_kept` kept (ties -> lower group);
//   stage 2  every candidate token of the kept groups scored exactly; the
//            best k kept (ties -> lower token).
// The k tokens are then attended with sink and window as usual (rba_attend).
#include "rba_internal.cuh"
#include "score_impl.cuh"
#include "topk_impl.cuh"

namespace rba {
namespace {

// means[bh][j] = (1 / group) sum_t K[bh][j * group + t], fp32, for groups
// [first, first + n).  grid (n, B * Hkv), block D (the pools' row pitch).
template <typename T>
__global__ void group_mean_kernel(const T* __restrict__ K, float* __restrict__ means, int D,
                                  int group, int64_t cap_tokens, int64_t cap_groups,
                                  int64_t first) {
  const int64_t j = first + blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int d = threadIdx.x;
  const T* base = K + (bh * cap_tokens + j * group) * D + d;
  float acc = 0.f;
  for (int t = 0; t < group; ++t) acc += Elem<T>::to_f32(base[int64_t(t) * D]);
  means[(bh * cap_groups + j) * D + d] = acc / float(group);
}

// Stage 2: the tokens of kept group blockIdx.x of (b, kv head) blockIdx.y
// scored by the summed query; tokens outside [sink, w0) score -inf.
// scores2[bh][gi * group + t].  LPT lanes per token (16-byte loads), TPW
// tokens per warp iteration.
template <typename T, int D>
__global__ void __launch_bounds__(128) stage2_kernel(const T* __restrict__ K,
                                                     const T* __restrict__ q,
                                                     const int32_t* __restrict__ kept,
                                                     float* __restrict__ scores2, int Hq,
                                                     int Hkv, int qd, int64_t cap, int group,
                                                     int C, int sink, int64_t w0) {
  constexpr int EPV = Elem<T>::kPerVec;
  constexpr int LPT = D / EPV;
  constexpr int TPW = 32 / LPT;
  constexpr int U = 8;  // key loads in flight per lane
  __shared__ float qs[D];
  const int gi = blockIdx.x, bh = blockIdx.y;
  const int b = bh / Hkv, h = bh % Hkv, G = Hq / Hkv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
  const int sub = lane % LPT;
  const int stride = nwarp * TPW;  // tokens per load round of the CTA
  const int64_t t0 = int64_t(kept[int64_t(bh) * C + gi]) * group;
  const uint4* kb = reinterpret_cast<const uint4*>(K + int64_t(bh) * cap * D);
  float* out = scores2 + (int64_t(bh) * C + gi) * group;
  // this lane's token of load u of a batch: base + u * stride + (its slot)
  const int slot = warp * TPW + lane / LPT;
  uint4 kv[U];
  auto load_batch = [&](int base) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int tt = base + u * stride + slot;
      kv[u] = tt < group ? ld_stream(kb + (t0 + tt) * LPT + sub) : make_uint4(0, 0, 0, 0);
    }
  };
  // the first batch's loads are issued before the query is summed: the two
  // latencies overlap
  load_batch(0);
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float acc = 0.f;  // (q rows are qd long; the pools' padding columns score zero)
    if (d < qd)
      for (int i = 0; i < G; ++i) acc += Elem<T>::to_f32(q[(int64_t(b) * Hq + h * G + i) * qd + d]);
    qs[d] = acc;
  }
  __syncthreads();
  float qv[EPV];
#pragma unroll
  for (int e = 0; e < EPV; ++e) qv[e] = qs[sub * EPV + e];
  for (int base = 0; base < group; base += U * stride) {
    if (base > 0) load_batch(base);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int tt = base + u * stride + slot;
      float f[EPV];
      unpack(kv[u], f, T());
      float part = 0.f;
#pragma unroll
      for (int e = 0; e < EPV; ++e) part = fmaf(qv[e], f[e], part);
#pragma unroll
      for (int o = LPT / 2; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
      const int64_t tok = t0 + tt;
      if (tt < group && sub == 0) out[tt] = tok >= sink && tok < w0 ? part : -INFINITY;
    }
  }
}

// Stage-2 positions -> token ids; the kept groups and the keys read.
__global__ void approx_finish_kernel(const int32_t* __restrict__ pos,
                                     const int32_t* __restrict__ kept, int32_t* __restrict__ idx,
                                     int32_t* __restrict__ groups_out,
                                     int32_t* __restrict__ scanned, int k, int C, int group,
                                     int n_groups, int sink, int64_t w0) {
  const int bh = blockIdx.x;
  for (int j = threadIdx.x; j < k; j += blockDim.x) {
    const int p = pos[int64_t(bh) * k + j];
    idx[int64_t(bh) * k + j] = kept[int64_t(bh) * C + p / group] * group + p % group;
  }
  if (groups_out != nullptr)
    for (int j = threadIdx.x; j < C; j += blockDim.x)
      groups_out[int64_t(bh) * C + j] = kept[int64_t(bh) * C + j];
  if (scanned != nullptr) {
    __shared__ int s_cnt;
    if (threadIdx.x == 0) s_cnt = 0;
    __syncthreads();
    int cnt = 0;
    for (int j = threadIdx.x; j < C; j += blockDim.x) {
      const int64_t lo = max(int64_t(kept[int64_t(bh) * C + j]) * group, int64_t(sink));
      const int64_t hi = min(int64_t(kept[int64_t(bh) * C + j] + 1) * group, w0);
      cnt += hi > lo ? static_cast<int>(hi - lo) : 0;
    }
    atomicAdd(&s_cnt, cnt);
    __syncthreads();
    if (threadIdx.x == 0) scanned[bh] = n_groups + s_cnt;
  }
}

// Candidate groups: full groups of `group` tokens meeting [sink, w0).
void group_range(const Geometry& g, int group, int* first, int* n) {
  const int64_t lo = g.sink / group;
  int64_t hi = (g.w0 + group - 1) / group;
  if (hi > g.T / group) hi = g.T / group;
  *first = static_cast<int>(lo < hi ? lo : 0);
  *n = static_cast<int>(hi > lo ? hi - lo : 0);
}

struct ApproxWs {
  float* scores1;
  int32_t* kept;
  float* scores2;
  int32_t* pos;
  void* topk;
  size_t topk_bytes;
  size_t total;
};

ApproxWs approx_layout(void* ws, int BH, int n_groups, int C, int group, int k) {
  ApproxWs w;
  char* p = static_cast<char*>(ws);
  size_t off = 0;
  w.scores1 = reinterpret_cast<float*>(p + off);
  off += align_up(size_t(BH) * n_groups * 4, 256);
  w.kept = reinterpret_cast<int32_t*>(p + off);
  off += align_up(size_t(BH) * C * 4, 256);
  w.scores2 = reinterpret_cast<float*>(p + off);
  off += align_up(size_t(BH) * C * group * 4, 256);
  w.pos = reinterpret_cast<int32_t*>(p + off);
  off += align_up(size_t(BH) * k * 4, 256);
  w.topk = p + off;
  const size_t t1 = topk_workspace(BH, n_groups, C), t2 = topk_workspace(BH, C * group, k);
  w.topk_bytes = t1 > t2 ? t1 : t2;
  off += align_up(w.topk_bytes, 256);
  w.total = off;
  return w;
}

constexpr int kMaxGroup = 1024;

// Validates the arguments of rba_approx_select; fills the geometry.
rba_status approx_check(const rba_store* st, int64_t T, int32_t sink, int32_t window,
                        int32_t group, int32_t groups_kept, int32_t k, Geometry* g,
                        int* first_group, int* n_groups) {
  if (st == nullptr) return RBA_ERR_INVALID_ARG;
  if (st->d.mode != RBA_REP_IDENTITY) return RBA_ERR_INVALID_ARG;
  if (group < 1 || group > kMaxGroup || groups_kept < 1 || k < 1) return RBA_ERR_INVALID_ARG;
  rba_status s = geometry(st, T, sink, window, g);
  if (s != RBA_OK) return s;
  group_range(*g, group, first_group, n_groups);
  if (groups_kept > *n_groups) return RBA_ERR_INVALID_ARG;
  // at most two kept groups (the ones holding `sink` and w0) are partly
  // outside the candidate range: this many kept tokens always suffice
  if (int64_t(groups_kept) * group < int64_t(k) + 2 * int64_t(group)) return RBA_ERR_INVALID_ARG;
  if (int64_t(groups_kept) * group > (int64_t(1) << 30)) return RBA_ERR_UNSUPPORTED;
  return RBA_OK;
}

}  // namespace
}  // namespace rba

extern "C" {

rba_status rba_group_means(const rba_store* st, int64_t first_group, int32_t n_groups,
                           int32_t group, float* means, cudaStream_t stream) {
  using namespace rba;
  if (st == nullptr || means == nullptr || st->d.mode != RBA_REP_IDENTITY) return RBA_ERR_INVALID_ARG;
  if (group < 1 || group > kMaxGroup || n_groups < 0 || first_group < 0) return RBA_ERR_INVALID_ARG;
  const int64_t cap_groups = st->d.capacity_tokens / group;
  if (first_group + n_groups > cap_groups) return RBA_ERR_INVALID_ARG;
  if (n_groups == 0) return RBA_OK;
  const rba_store_desc& d = st->d;
  const dim3 grid(n_groups, d.batch * d.n_kv_heads);
  if (d.dtype == RBA_BF16)
    group_mean_kernel<__nv_bfloat16><<<grid, st->pitch, 0, stream>>>(
        static_cast<const __nv_bfloat16*>(st->k), means, st->pitch, group, d.capacity_tokens,
        cap_groups, first_group);
  else
    group_mean_kernel<float><<<grid, st->pitch, 0, stream>>>(
        static_cast<const float*>(st->k), means, st->pitch, group, d.capacity_tokens,
        cap_groups, first_group);
  RBA_LAUNCH_CHECK();
  return RBA_OK;
}

size_t rba_approx_select_workspace_size(const rba_store* st, int64_t T, int32_t sink,
                                        int32_t window, int32_t group, int32_t groups_kept,
                                        int32_t k) {
  using namespace rba;
  Geometry g;
  int fg = 0, ng = 0;
  if (approx_check(st, T, sink, window, group, groups_kept, k, &g, &fg, &ng) != RBA_OK) return 0;
  return approx_layout(nullptr, st->d.batch * st->d.n_kv_heads, ng, groups_kept, group, k).total;
}

rba_status rba_approx_select(const rba_store* st, const void* q, int64_t T, int32_t sink,
                             int32_t window, int32_t group, int32_t groups_kept, int32_t k,
                             const float* means, int32_t* idx, int32_t* groups_out,
                             int32_t* scanned, void* workspace, size_t ws_bytes,
                             cudaStream_t stream) {
  using namespace rba;
  Geometry g;
  int first_group = 0, n_groups = 0;
  rba_status s = approx_check(st, T, sink, window, group, groups_kept, k, &g, &first_group,
                              &n_groups);
  if (s != RBA_OK) return s;
  if (q == nullptr || means == nullptr || idx == nullptr) return RBA_ERR_INVALID_ARG;
  const rba_store_desc& d = st->d;
  const int BH = d.batch * d.n_kv_heads;
  if (d.n_q_heads / d.n_kv_heads > 64) return RBA_ERR_UNSUPPORTED;
  if (k > (1 << 16) || groups_kept > (1 << 16)) return RBA_ERR_UNSUPPORTED;
  const ApproxWs w = approx_layout(workspace, BH, n_groups, groups_kept, group, k);
  if (workspace == nullptr || ws_bytes < w.total) return RBA_ERR_WORKSPACE;
  // stage 1: the candidate groups' means against the summed query, top groups_kept
  ScoreArgs a = {};
  a.rep = means;
  a.rep_rows = d.capacity_tokens / group;
  a.q = q;
  a.qsum = nullptr;
  a.scores = w.scores1;
  a.Hq = d.n_q_heads;
  a.Hkv = d.n_kv_heads;
  a.n_q = 1;
  a.first = first_group;
  a.nc = n_groups;
  a.qd = d.head_dim;
  a.max_over_keys = false;
  s = dispatch_score_dot(a, d.dtype == RBA_BF16, true, st->pitch, 1, BH, stream);
  if (s != RBA_OK) return s;
  s = launch_topk(w.scores1, BH, n_groups, groups_kept, first_group, w.kept, w.topk,
                  w.topk_bytes, stream, false);
  if (s != RBA_OK) return s;
  // stage 2: the kept groups' tokens scored exactly, top k
  const dim3 grid(groups_kept, BH);
#define RBA_STAGE2(T_, D_)                                                                  \
  stage2_kernel<T_, D_><<<grid, 128, 0, stream>>>(                                          \
      static_cast<const T_*>(st->k), static_cast<const T_*>(q), w.kept, w.scores2,          \
      d.n_q_heads, d.n_kv_heads, d.head_dim, d.capacity_tokens, group, groups_kept, g.sink, g.w0)
  if (d.dtype == RBA_BF16) {
    if (st->pitch == 128) RBA_STAGE2(__nv_bfloat16, 128);
    else RBA_STAGE2(__nv_bfloat16, 64);
  } else {
    if (st->pitch == 128) RBA_STAGE2(float, 128);
    else RBA_STAGE2(float, 64);
  }
#undef RBA_STAGE2
  RBA_LAUNCH_CHECK();
  const int n2 = groups_kept * group;
  s = launch_topk(w.scores2, BH, n2, k, 0, w.pos, w.topk, w.topk_bytes, stream, false);
  if (s != RBA_OK) return s;
  approx_finish_kernel<<<BH, 256, 0, stream>>>(w.pos, w.kept, idx, groups_out, scanned, k,
                                               groups_kept, group, n_groups, g.sink, g.w0);
  RBA_LAUNCH_CHECK();
  return RBA_OK;
}

}  // extern "C"
