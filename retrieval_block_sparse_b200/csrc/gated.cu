// Landmark-gated decode attention.
//
// Landmark Attention review, "proposed method": each block is represented by
// a landmark token that acts as the gate through which attention reaches the
// block.  The reading taken (no formula is given): the landmark takes the
// block's place in the query's softmax.  Local tokens (sink U window) enter
// with their own logits x_t = scale q . k_t; retrieved block j enters once,
// with the landmark's logit y_j = scale q . L_j, and carries the value
// o_j = sum over its tokens (outside sink and window) of softmax_block(x) v:
//   out = (sum_local e^{x_t} v_t + sum_j e^{y_j} o_j) / Z,  lse = ln Z.
//
// One CTA per (batch, q head), four warps.  A warp keeps one softmax state
// over its share of the terms: local rows t = warp, warp + 4, ... and blocks
// j = warp, warp + 4, ... (a block's o_j from a softmax over its rows inside
// the same warp).  Lane l holds columns [l EPL, (l + 1) EPL) of a row; a
// row's logit is a warp-wide sum.  The four warp states merge by log-sum-exp.
#include "rba_internal.cuh"

namespace rba {
namespace {

constexpr int kGWarps = 4;

struct GatedArgs {
  const void* K;        // [BH][cap][P]
  const void* V;
  const void* L;        // landmark keys [BH][cap_blocks][1][P]
  const void* q;        // [B][Hq][qd]
  const int32_t* idx;   // [BH][k]
  float* out;           // [B][Hq][qd]
  float* lse;           // [B][Hq] or nullptr
  int32_t* status;
  int64_t cap, cap_blocks, T, w0;
  int Hq, Hkv, k, bs, sink, sink_end, first, nc, qd;
  float scale_log2;
};

// online softmax state of one lane's EPL columns (log2 units)
template <int EPL>
struct State {
  float m, l;
  float o[EPL];
  __device__ void init() {
    m = -INFINITY;
    l = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) o[e] = 0.f;
  }
  // one term: logit x (log2 units), weight 2^x, value v
  __device__ void add(float x, const float (&v)[EPL]) {
    if (x > m) {
      const float c = m == -INFINITY ? 0.f : exp2f(m - x);
      l *= c;
#pragma unroll
      for (int e = 0; e < EPL; ++e) o[e] *= c;
      m = x;
    }
    const float p = exp2f(x - m);
    l += p;
#pragma unroll
    for (int e = 0; e < EPL; ++e) o[e] = fmaf(p, v[e], o[e]);
  }
};

template <typename T, int EPL>
__device__ __forceinline__ void load_row(const T* row, int lane, float (&f)[EPL]) {
#pragma unroll
  for (int e = 0; e < EPL; ++e) f[e] = Elem<T>::to_f32(row[lane * EPL + e]);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

template <typename T, int P>
__global__ void __launch_bounds__(kGWarps * 32) gated_kernel(GatedArgs a) {
  constexpr int EPL = P / 32;
  __shared__ float red[kGWarps][P + 2];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int bq = blockIdx.x;  // b * Hq + q head
  const int b = bq / a.Hq, hq = bq % a.Hq;
  const int G = a.Hq / a.Hkv, h = hq / G;
  const int64_t bh = int64_t(b) * a.Hkv + h;
  // q scaled to log2 units; columns past qd are zero
  float qv[EPL];
  const T* qp = static_cast<const T*>(a.q) + int64_t(bq) * a.qd;
#pragma unroll
  for (int e = 0; e < EPL; ++e) {
    const int d = lane * EPL + e;
    qv[e] = d < a.qd ? Elem<T>::to_f32(qp[d]) * a.scale_log2 : 0.f;
  }
  const T* Kb = static_cast<const T*>(a.K) + bh * a.cap * P;
  const T* Vb = static_cast<const T*>(a.V) + bh * a.cap * P;
  auto logit = [&](const T* row) {
    float f[EPL];
    load_row<T, EPL>(row, lane, f);
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) s = fmaf(qv[e], f[e], s);
    return warp_sum(s);
  };
  auto local_row = [&](State<EPL>& st, int64_t t) {
    float v[EPL];
    const float x = logit(Kb + t * P);
    load_row<T, EPL>(Vb + t * P, lane, v);
    st.add(x, v);
  };
  State<EPL> st;
  st.init();
  // local terms: sink rows [0, sink_end), window rows [w0, T)
  for (int t = warp; t < a.sink_end; t += kGWarps) local_row(st, t);
  for (int64_t t = a.w0 + warp; t < a.T; t += kGWarps) local_row(st, t);
  // gated terms: a retrieved block's rows inside [sink, w0) through their own
  // softmax, entering this warp's state once with the landmark's logit
  for (int i = warp; i < a.k; i += kGWarps) {
    const int j = a.idx[bh * a.k + i];
    if (j < a.first || j >= a.first + a.nc) {
      if (lane == 0) report(a.status, RBA_ERR_BOUNDS, kWhereAttend, j);
      continue;
    }
    const int64_t lo = max(int64_t(j) * a.bs, int64_t(a.sink));
    const int64_t hi = min(int64_t(j + 1) * a.bs, a.w0);
    if (hi <= lo) continue;
    State<EPL> blk;
    blk.init();
    for (int64_t t = lo; t < hi; ++t) local_row(blk, t);
    float ob[EPL];
    const float inv = blk.l > 0.f ? 1.f / blk.l : 0.f;
#pragma unroll
    for (int e = 0; e < EPL; ++e) ob[e] = blk.o[e] * inv;
    const float y = logit(static_cast<const T*>(a.L) + (bh * a.cap_blocks + j) * P);
    st.add(y, ob);
  }
  // merge the warps' states
  if (lane == 0) {
    red[warp][0] = st.m;
    red[warp][1] = st.l;
  }
#pragma unroll
  for (int e = 0; e < EPL; ++e) red[warp][2 + lane * EPL + e] = st.o[e];
  __syncthreads();
  float M = -INFINITY;
#pragma unroll
  for (int w = 0; w < kGWarps; ++w) M = fmaxf(M, red[w][0]);
  float f[kGWarps], L = 0.f;
#pragma unroll
  for (int w = 0; w < kGWarps; ++w) {
    f[w] = red[w][0] == -INFINITY ? 0.f : exp2f(red[w][0] - M);
    L = fmaf(f[w], red[w][1], L);
  }
  for (int d = threadIdx.x; d < a.qd; d += blockDim.x) {
    float O = 0.f;
#pragma unroll
    for (int w = 0; w < kGWarps; ++w) O = fmaf(f[w], red[w][2 + d], O);
    a.out[int64_t(bq) * a.qd + d] = L > 0.f ? O / L : 0.f;
  }
  if (threadIdx.x == 0 && a.lse != nullptr)
    a.lse[bq] = L > 0.f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
}

}  // namespace
}  // namespace rba

extern "C" rba_status rba_attend_landmark_gated(const rba_store* st, const void* q,
                                                const int32_t* idx, int32_t k, int64_t T,
                                                int32_t sink, int32_t window, float scale,
                                                float* out, float* lse, cudaStream_t stream) {
  using namespace rba;
  if (st == nullptr || q == nullptr || out == nullptr || k < 0) return RBA_ERR_INVALID_ARG;
  const rba_store_desc& d = st->d;
  if (d.mode != RBA_REP_EXTERNAL || d.n_rep != 1) return RBA_ERR_INVALID_ARG;
  Geometry g;
  rba_status s = geometry(st, T, sink, window, &g);
  if (s != RBA_OK) return s;
  if (k > g.nc || (k > 0 && idx == nullptr)) return RBA_ERR_INVALID_ARG;
  const int BQ = d.batch * d.n_q_heads;
  if (BQ == 0) return RBA_OK;
  GatedArgs a;
  a.K = st->k;
  a.V = st->v;
  a.L = st->rep;
  a.q = q;
  a.idx = idx;
  a.out = out;
  a.lse = lse;
  a.status = st->status;
  a.cap = d.capacity_tokens;
  a.cap_blocks = st->cap_blocks;
  a.T = g.T;
  a.w0 = g.w0;
  a.Hq = d.n_q_heads;
  a.Hkv = d.n_kv_heads;
  a.k = k;
  a.bs = d.block_size;
  a.sink = g.sink;
  a.sink_end = g.sink_end;
  a.first = g.first;
  a.nc = g.nc;
  a.qd = d.head_dim;
  a.scale_log2 = scale * 1.4426950408889634f;
  const dim3 grid(BQ), block(kGWarps * 32);
  if (d.dtype == RBA_BF16) {
    if (st->pitch == 128) gated_kernel<__nv_bfloat16, 128><<<grid, block, 0, stream>>>(a);
    else gated_kernel<__nv_bfloat16, 64><<<grid, block, 0, stream>>>(a);
  } else {
    if (st->pitch == 128) gated_kernel<float, 128><<<grid, block, 0, stream>>>(a);
    else gated_kernel<float, 64><<<grid, block, 0, stream>>>(a);
  }
  RBA_LAUNCH_CHECK();
  return RBA_OK;
}
