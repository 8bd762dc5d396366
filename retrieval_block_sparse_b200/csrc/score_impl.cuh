// Dot-mode block scoring kernel (HBM-bound stream over representative keys).
#pragma once

#include "rba_internal.cuh"

namespace rba {

struct ScoreArgs {
  const void* rep;      // [B*Hkv][rep_rows][R][D]
  int64_t rep_rows;     // rows (blocks) per (b, kv head) in the rep pool
  const void* q;        // [B][Hq][n_q][D] (used when qsum == nullptr)
  const float* qsum;    // [B*Hkv][D] or nullptr
  float* scores;        // [B*Hkv][nc]
  int Hq, Hkv, n_q, first, nc;
  int qd;               // row length of q (the rep rows hold D >= qd elements, the rest zero)
  bool max_over_keys;   // block score = max over its keys (else their sum)
  int ctas_per_sm;      // grid target (host side): CTAs per SM
};

// One CTA covers `cand_per_cta` consecutive candidates of one (b, kv head).
// A candidate's R*D rep elements are contiguous; LPC lanes share one
// candidate, each loading VPL 16-byte vectors, and U candidate groups are in
// flight per warp before any arithmetic.
template <typename QT, typename RT, int D, int R, int NW, int U, bool MAXR>
__global__ void __launch_bounds__(NW * 32) score_dot_kernel(ScoreArgs a, int cand_per_cta) {
  constexpr int EPV = Elem<RT>::kPerVec;
  constexpr int VPC = R * D / EPV;
  constexpr int LPC = VPC < 32 ? VPC : 32;
  constexpr int VPL = VPC / LPC;
  constexpr int CPW = 32 / LPC;
  static_assert(VPC % LPC == 0 && 32 % LPC == 0, "rep row must tile the warp");
  // a kernel launched behind this one as a programmatic dependent (the
  // top-k of the decode step) may start now; it waits for our completion
  // before it reads the scores
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  __shared__ float qs[D];
  const int bh = blockIdx.y;
  const int b = bh / a.Hkv, h = bh - b * a.Hkv, g = a.Hq / a.Hkv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int sub = lane % LPC, slot = lane / LPC;
  const uint4* base = reinterpret_cast<const uint4*>(
      static_cast<const RT*>(a.rep) + (int64_t(bh) * a.rep_rows + a.first) * (R * D));
  const int c_begin = blockIdx.x * cand_per_cta;
  const int c_end = min(a.nc, c_begin + cand_per_cta);
  float* out = a.scores + int64_t(bh) * a.nc;
  // U candidate groups of this warp's first iteration: their loads are issued
  // before the query is summed, so the two latencies overlap
  uint4 v[U][VPL];
  auto load_groups = [&](int c0) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int c = c0 + u * CPW + slot;
#pragma unroll
      for (int i = 0; i < VPL; ++i)
        v[u][i] = c < c_end ? ld_stream(base + int64_t(c) * VPC + sub + i * LPC)
                            : make_uint4(0, 0, 0, 0);
    }
  };
  const int c_first = c_begin + warp * CPW * U;
  load_groups(c_first);
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float acc = 0.f;
    if (a.qsum != nullptr) {
      acc = a.qsum[int64_t(bh) * D + d];
    } else if (d < a.qd) {
      const QT* q = static_cast<const QT*>(a.q);
      for (int i = 0; i < g; ++i)
        for (int t = 0; t < a.n_q; ++t)
          acc += Elem<QT>::to_f32(q[((int64_t(b) * a.Hq + h * g + i) * a.n_q + t) * a.qd + d]);
    }
    qs[d] = acc;
  }
  __syncthreads();
  float qr[VPL][EPV];
#pragma unroll
  for (int i = 0; i < VPL; ++i) {
    const int d0 = ((sub + i * LPC) * EPV) % D;
#pragma unroll
    for (int e = 0; e < EPV; ++e) qr[i][e] = qs[d0 + e];
  }
  for (int c0 = c_first; c0 < c_end; c0 += NW * CPW * U) {
    if (c0 != c_first) load_groups(c0);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      float part[VPL];  // this lane's share of the dot product, per loaded vector
#pragma unroll
      for (int i = 0; i < VPL; ++i) {
        float f[EPV];
        unpack(v[u][i], f, RT());
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < EPV; ++e) acc = fmaf(qr[i][e], f[e], acc);
        part[i] = acc;
      }
      float acc;
      if constexpr (!MAXR) {
        acc = 0.f;
#pragma unroll
        for (int i = 0; i < VPL; ++i) acc += part[i];
#pragma unroll
        for (int o = LPC / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
      } else {
        // vector (sub + i LPC) of the candidate belongs to key (sub + i LPC) / VPR
        constexpr int VPR = D / EPV;  // vectors per representative key
        if constexpr (VPR >= LPC) {
          // a key spans VPR / LPC whole vector slots of every lane
          constexpr int SPK = VPR / LPC;
          acc = -INFINITY;
#pragma unroll
          for (int r0 = 0; r0 < VPL; r0 += SPK) {
            float kd = 0.f;
#pragma unroll
            for (int i = r0; i < r0 + SPK; ++i) kd += part[i];
#pragma unroll
            for (int o = LPC / 2; o > 0; o >>= 1) kd += __shfl_xor_sync(0xffffffffu, kd, o);
            acc = fmaxf(acc, kd);
          }
        } else {
          // a key spans VPR lanes of one vector slot: sum inside those lane
          // segments, then the max over slots and segments
          acc = -INFINITY;
#pragma unroll
          for (int i = 0; i < VPL; ++i) {
            float kd = part[i];
#pragma unroll
            for (int o = VPR / 2; o > 0; o >>= 1) kd += __shfl_xor_sync(0xffffffffu, kd, o);
            acc = fmaxf(acc, kd);
          }
#pragma unroll
          for (int o = VPR; o < LPC; o <<= 1) acc = fmaxf(acc, __shfl_xor_sync(0xffffffffu, acc, o));
        }
      }
      const int c = c0 + u * CPW + slot;
      if (sub == 0 && c < c_end) out[c] = acc;
    }
  }
}

// NW warps per CTA and U candidate groups in flight per warp; about `want`
// CTAs in all (each warp at least one batch)
template <int NW, int U, typename QT, typename RT, int D, int R, bool MAXR>
rba_status launch_score_nw(const ScoreArgs& a, int BH, int64_t want, cudaStream_t stream) {
  constexpr int EPV = Elem<RT>::kPerVec;
  constexpr int VPC = R * D / EPV;
  constexpr int LPC = VPC < 32 ? VPC : 32;
  constexpr int per_iter = NW * (32 / LPC) * U;
  if (want < 1) want = 1;
  int64_t per_cta = (int64_t(a.nc) * BH + want - 1) / want;
  per_cta = (per_cta + per_iter - 1) / per_iter * per_iter;
  if (per_cta < per_iter) per_cta = per_iter;
  const int gx = static_cast<int>((a.nc + per_cta - 1) / per_cta);
  score_dot_kernel<QT, RT, D, R, NW, U, MAXR>
      <<<dim3(gx, BH), NW * 32, 0, stream>>>(a, static_cast<int>(per_cta));
  RBA_LAUNCH_CHECK();
  return RBA_OK;
}

template <typename QT, typename RT, int D, int R, bool MAXR>
rba_status launch_score_dot_t(const ScoreArgs& a, int BH, cudaStream_t stream) {
  constexpr int EPV = Elem<RT>::kPerVec;
  constexpr int VPC = R * D / EPV;
  constexpr int LPC = VPC < 32 ? VPC : 32;
  constexpr int per_iter = 8 * (32 / LPC) * 4;  // candidates of one batch of an 8-warp CTA
  // fewer than 4 CTAs per SM only where 4 would leave each CTA one batch of
  // loads anyway (a short, latency-bound scan); long scans keep 4
  int cps = a.ctas_per_sm > 0 ? a.ctas_per_sm : 4;
  if (cps < 4 && int64_t(a.nc) * BH > int64_t(num_sms()) * 4 * per_iter) cps = 4;
  // one CTA per SM: twice the candidate groups in flight per warp where a
  // lane holds at most two vectors of a group (the registers are there with
  // one CTA an SM; more vectors would spill), so that each warp's share is one
  // batch of loads (128K step 20.83 -> 20.65 us)
  if (cps == 1) {
    if constexpr (VPC / LPC <= 2)
      return launch_score_nw<8, 8, QT, RT, D, R, MAXR>(a, BH, num_sms(), stream);
    else
      return launch_score_nw<8, 4, QT, RT, D, R, MAXR>(a, BH, num_sms(), stream);
  }
  return launch_score_nw<8, 4, QT, RT, D, R, MAXR>(a, BH, int64_t(num_sms()) * cps, stream);
}

template <typename QT, typename RT, int D>
rba_status dispatch_r(const ScoreArgs& a, int R, int BH, cudaStream_t s) {
  // with one key per block the max over keys is the sum
  if (a.max_over_keys && R > 1) {
    switch (R) {
      case 2: return launch_score_dot_t<QT, RT, D, 2, true>(a, BH, s);
      case 4: return launch_score_dot_t<QT, RT, D, 4, true>(a, BH, s);
      case 8: return launch_score_dot_t<QT, RT, D, 8, true>(a, BH, s);
    }
    return RBA_ERR_UNSUPPORTED;
  }
  switch (R) {
    case 1: return launch_score_dot_t<QT, RT, D, 1, false>(a, BH, s);
    case 2: return launch_score_dot_t<QT, RT, D, 2, false>(a, BH, s);
    case 4: return launch_score_dot_t<QT, RT, D, 4, false>(a, BH, s);
    case 8: return launch_score_dot_t<QT, RT, D, 8, false>(a, BH, s);
  }
  return RBA_ERR_UNSUPPORTED;
}

template <typename QT, typename RT>
rba_status dispatch_d(const ScoreArgs& a, int D, int R, int BH, cudaStream_t s) {
  if (D == 128) return dispatch_r<QT, RT, 128>(a, R, BH, s);
  if (D == 64) return dispatch_r<QT, RT, 64>(a, R, BH, s);
  return RBA_ERR_UNSUPPORTED;
}

inline rba_status dispatch_score_dot(const ScoreArgs& a, bool q_bf16, bool rep_f32, int D, int R,
                                     int BH, cudaStream_t s) {
  if (q_bf16 && !rep_f32) return dispatch_d<__nv_bfloat16, __nv_bfloat16>(a, D, R, BH, s);
  if (q_bf16 && rep_f32) return dispatch_d<__nv_bfloat16, float>(a, D, R, BH, s);
  if (!q_bf16 && rep_f32) return dispatch_d<float, float>(a, D, R, BH, s);
  return RBA_ERR_UNSUPPORTED;
}

// ctas_per_sm: the grid's target CTAs per SM (4 keeps enough loads in flight
// for long scans; 1, for short scans, leaves some SMs empty and lets the CTAs
// retire together, so that a persistent kernel launched as a programmatic
// dependent gets SMs sooner)
rba_status launch_score_dot(const rba_store* st, const void* q, int n_q, const float* qsum,
                            const Geometry& g, float* scores, cudaStream_t stream,
                            int ctas_per_sm = 4);
rba_status launch_qsum(const rba_store* st, const void* q, int n_q, float* qsum,
                       cudaStream_t stream);

}  // namespace rba
