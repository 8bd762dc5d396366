// Block scoring.
//
// Dot modes (Landmark Attention review, "proposed method": query-landmark
// similarity; InfLLM article, "method": relevance against representative
// tokens): for candidate c of (b, kv head h),
//   s = sum_{q heads of the group} sum_{query rows} sum_{rep keys i} q . rep_i
// computed as (summed query) . rep_i, one pass over the rep keys.
// Cosine mode (MemLong summary, 2.3.2 retrieval process): cos(r^q, M_j) with
// M_j stored L2-normalised.
#include "rba_internal.cuh"
#include "score_impl.cuh"

namespace rba {
namespace {

// qsum[bh][d] = sum over the group's q heads and n_q rows of q[b][hq][t][d].
// The g * n_q rows of one (b, kv head) are contiguous; the CTA reads them as
// 16-byte vectors (LPR lanes per row, kQsumThreads / LPR rows in flight) and
// sums the per-thread partials in a fixed order (deterministic).
constexpr int kQsumThreads = 1024;

template <typename QT, int D>
__global__ void __launch_bounds__(kQsumThreads) qsum_kernel(const QT* __restrict__ q,
                                                            float* __restrict__ qsum, int Hq,
                                                            int Hkv, int n_q) {
  constexpr int EPV = Elem<QT>::kPerVec;
  constexpr int LPR = D / EPV;                  // lanes per row
  constexpr int RPP = kQsumThreads / LPR;       // rows per pass
  __shared__ float part[RPP][D + 1];
  const int bh = blockIdx.x;
  const int b = bh / Hkv, h = bh % Hkv, g = Hq / Hkv;
  const int64_t rows = int64_t(g) * n_q;
  const uint4* base = reinterpret_cast<const uint4*>(q + (int64_t(b) * Hq + h * g) * n_q * D);
  const int sub = threadIdx.x % LPR, r0 = threadIdx.x / LPR;
  float acc[EPV];
#pragma unroll
  for (int e = 0; e < EPV; ++e) acc[e] = 0.f;
#pragma unroll 4
  for (int64_t r = r0; r < rows; r += RPP) {
    float f[EPV];
    unpack(ld_stream(base + r * LPR + sub), f, QT());
#pragma unroll
    for (int e = 0; e < EPV; ++e) acc[e] += f[e];
  }
#pragma unroll
  for (int e = 0; e < EPV; ++e) part[r0][sub * EPV + e] = acc[e];
  __syncthreads();
  for (int d = threadIdx.x; d < D; d += kQsumThreads) {
    float s = 0.f;
    for (int i = 0; i < RPP; ++i) s += part[i][d];
    qsum[int64_t(bh) * D + d] = s;
  }
}

// qsum for q rows of qd < D elements (head dims below the pools' row pitch):
// one thread per column, rows summed in order; columns past qd are zero.
template <typename QT>
__global__ void qsum_rows_kernel(const QT* __restrict__ q, float* __restrict__ qsum, int Hq,
                                 int Hkv, int n_q, int qd, int D) {
  const int bh = blockIdx.x;
  const int b = bh / Hkv, h = bh % Hkv, g = Hq / Hkv;
  const int64_t rows = int64_t(g) * n_q;
  const QT* base = q + (int64_t(b) * Hq + h * g) * n_q * qd;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float acc = 0.f;
    if (d < qd)
      for (int64_t r = 0; r < rows; ++r) acc += Elem<QT>::to_f32(base[r * qd + d]);
    qsum[int64_t(bh) * D + d] = acc;
  }
}

__global__ void score_cos_kernel(const float* __restrict__ qe, const float* __restrict__ bank,
                                 float* __restrict__ scores, int d_ret, int first, int nc) {
  extern __shared__ float sq[];
  __shared__ float sred[32];
  const int i = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
  float ss = 0.f;
  for (int d = threadIdx.x; d < d_ret; d += blockDim.x) {
    const float v = qe[int64_t(i) * d_ret + d];
    sq[d] = v;
    ss = fmaf(v, v, ss);
  }
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  if (lane == 0) sred[warp] = ss;
  __syncthreads();
  float tot = 0.f;
  for (int w = 0; w < nwarp; ++w) tot += sred[w];
  const float nrm = sqrtf(tot);
  for (int c = warp; c < nc; c += nwarp) {
    const float4* m = reinterpret_cast<const float4*>(bank + (int64_t(first) + c) * d_ret);
    float acc = 0.f;
    for (int v = lane; v < d_ret / 4; v += 32) {
      const float4 x = m[v];
      acc = fmaf(sq[4 * v + 0], x.x, acc);
      acc = fmaf(sq[4 * v + 1], x.y, acc);
      acc = fmaf(sq[4 * v + 2], x.z, acc);
      acc = fmaf(sq[4 * v + 3], x.w, acc);
    }
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) scores[int64_t(i) * nc + c] = acc / nrm;
  }
}

}  // namespace

rba_status launch_qsum(const rba_store* st, const void* q, int n_q, float* qsum,
                       cudaStream_t stream) {
  const rba_store_desc& d = st->d;
  const int BH = d.batch * d.n_kv_heads;
  if (d.head_dim != st->pitch) {
    if (d.dtype == RBA_BF16)
      qsum_rows_kernel<__nv_bfloat16><<<BH, st->pitch, 0, stream>>>(
          static_cast<const __nv_bfloat16*>(q), qsum, d.n_q_heads, d.n_kv_heads, n_q, d.head_dim,
          st->pitch);
    else
      qsum_rows_kernel<float><<<BH, st->pitch, 0, stream>>>(
          static_cast<const float*>(q), qsum, d.n_q_heads, d.n_kv_heads, n_q, d.head_dim,
          st->pitch);
    RBA_LAUNCH_CHECK();
    return RBA_OK;
  }
#define RBA_QSUM(QT_, D_)                                                                \
  qsum_kernel<QT_, D_><<<BH, kQsumThreads, 0, stream>>>(static_cast<const QT_*>(q), qsum, \
                                                         d.n_q_heads, d.n_kv_heads, n_q)
  if (d.dtype == RBA_BF16) {
    if (d.head_dim == 128) RBA_QSUM(__nv_bfloat16, 128);
    else RBA_QSUM(__nv_bfloat16, 64);
  } else {
    if (d.head_dim == 128) RBA_QSUM(float, 128);
    else RBA_QSUM(float, 64);
  }
#undef RBA_QSUM
  RBA_LAUNCH_CHECK();
  return RBA_OK;
}

// Dot-mode launch: templated on query, rep element type, head dim and rep count.
rba_status launch_score_dot(const rba_store* st, const void* q, int n_q, const float* qsum,
                            const Geometry& g, float* scores, cudaStream_t stream,
                            int ctas_per_sm) {
  const rba_store_desc& d = st->d;
  const int BH = d.batch * d.n_kv_heads;
  const int grp = d.n_q_heads / d.n_kv_heads;
  if (qsum == nullptr && grp * n_q > 64) return RBA_ERR_INVALID_ARG;
  if (g.nc == 0) return RBA_OK;
  ScoreArgs a = {};
  a.q = q;
  a.qsum = qsum;
  a.scores = scores;
  a.Hq = d.n_q_heads;
  a.Hkv = d.n_kv_heads;
  a.n_q = n_q;
  a.first = g.first;
  a.nc = g.nc;
  a.qd = d.head_dim;
  a.max_over_keys = st->score_reduce == RBA_SCORE_MAX;
  a.ctas_per_sm = ctas_per_sm;
  if (d.mode == RBA_REP_IDENTITY) {
    a.rep = st->k;
    a.rep_rows = d.capacity_tokens;
  } else {
    a.rep = st->rep;
    a.rep_rows = st->cap_blocks;
  }
  const bool rep_f32 = d.mode == RBA_REP_MEAN || d.dtype == RBA_F32;
  return dispatch_score_dot(a, d.dtype == RBA_BF16, rep_f32, st->pitch, d.n_rep, BH, stream);
}

rba_status launch_score_cos(const rba_store* st, const float* qe, int n_q, const Geometry& g,
                            float* scores, cudaStream_t stream) {
  const int d_ret = st->d.d_ret;
  if (g.nc == 0 || n_q == 0) return RBA_OK;
  const size_t smem = size_t(d_ret) * sizeof(float);
  if (smem > 48 * 1024)
    RBA_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(score_cos_kernel), smem));
  score_cos_kernel<<<n_q, 256, smem, stream>>>(qe, static_cast<const float*>(st->rep), scores,
                                               d_ret, g.first, g.nc);
  RBA_LAUNCH_CHECK();
  return RBA_OK;
}

}  // namespace rba

extern "C" rba_status rba_score(const rba_store* st, const void* q, int32_t n_q, int64_t T,
                                int32_t sink, int32_t window, float* scores, float* qsum_ws,
                                cudaStream_t stream) {
  using namespace rba;
  if (st == nullptr || q == nullptr || scores == nullptr || n_q <= 0) return RBA_ERR_INVALID_ARG;
  Geometry g;
  rba_status s = geometry(st, T, sink, window, &g);
  if (s != RBA_OK) return s;
  if (st->d.mode == RBA_REP_EMBED_COSINE) {
    if (st->d.batch != 1) return RBA_ERR_INVALID_ARG;
    return launch_score_cos(st, static_cast<const float*>(q), n_q, g, scores, stream);
  }
  const int grp = st->d.n_q_heads / st->d.n_kv_heads;
  if (grp * n_q > 64) {
    if (qsum_ws == nullptr) return RBA_ERR_INVALID_ARG;
    s = launch_qsum(st, q, n_q, qsum_ws, stream);
    if (s != RBA_OK) return s;
    return launch_score_dot(st, q, n_q, qsum_ws, g, scores, stream);
  }
  return launch_score_dot(st, q, n_q, nullptr, g, scores, stream);
}
