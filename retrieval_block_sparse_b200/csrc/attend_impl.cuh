// Decode attention internals: attended-set segments, tile staging, per-lane
// online softmax, split partials and their log-sum-exp merge.
//
// InfLLM article, "overall framework": each query attends to the local
// window and a few retrieved memory units; MemLong summary, 2.3.3: retrieved
// chunks are attended without a causal mask.  The attended set of one
// (batch, kv head) is the union sink U retrieved blocks U window, laid out as
// a list of disjoint physical token ranges ("segments"); its tokens are
// numbered 0..n_att-1 in segment order ("virtual" positions) and split evenly
// over the CTAs of that (batch, kv head).
#pragma once

#include "rba_internal.cuh"

namespace rba {

struct AttendArgs {
  const void* K;          // [B*Hkv][cap][D]
  const void* V;          // [B*Hkv][cap][D]
  const void* q;          // [B][Hq][D]
  const int32_t* idx;     // [B*Hkv][k] ascending candidate block ids
  float* out;             // [B*Hq][D]
  float* lse;             // [B*Hq] or nullptr
  float* part;            // [B*Hq][nsplit][D+2]  (m, l, unnormalised o)
  uint32_t* tickets;      // [B*Hkv], zero between calls
  int32_t* status;
  int64_t cap;
  int64_t T;
  int64_t w0;
  int Hq, Hkv, k, bs, sink, sink_end, nsplit, first, nc;
  int qd;                 // head dim: row length of q and out (the pools' rows hold D >= qd
                          // elements, the columns past qd zero)
  float scale_log2;       // scale * log2(e)
};

constexpr int kAttendWarps = 8;
constexpr int kAttendThreads = kAttendWarps * 32;

// Tile geometry for NW consuming warps: each warp takes TPW rows per step,
// NT steps per tile, LPR lanes per row and EPL elements per lane.
template <typename T, int D, int NW = kAttendWarps>
struct DecodeTile {
  static constexpr int ES = sizeof(T);
  static constexpr int EPL = 16;                  // elements of a row per lane
  static constexpr int LPR = D / EPL;             // lanes per row
  static constexpr int TPW = 32 / LPR;            // rows per warp step
  static constexpr int NT = 2;                    // steps per tile
  static constexpr int TT = NW * TPW * NT;        // tokens per tile
  static constexpr int ROWB = D * ES;
  static constexpr int CPR = ROWB / 16;           // 16-byte chunks per row
  static constexpr int CPL = EPL * ES / 16;       // chunks per lane per row
  static constexpr int EPC = 16 / ES;             // elements per chunk
  static constexpr int NS = ES == 2 ? 3 : 2;      // pipeline stages (split-K kernel)
  static constexpr int STAGE = 2 * TT * ROWB;     // K tile + V tile
  static constexpr int LOADS = 2 * TT * CPR / (NW * 32);  // cp.async per thread per tile
  static_assert((2 * TT * CPR) % (NW * 32) == 0, "tile must split over the warps");
};

// ---------------------------------------------------------------------------
// segments

// Exclusive scan of n ints in shared memory (block-wide), returns the total.
__device__ inline int block_exclusive_scan(int* v, int n, int* s_warp) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int lane = tid & 31, warp = tid >> 5, nw = nt >> 5;
  const int per = (n + nt - 1) / nt;
  const int b0 = min(n, tid * per), b1 = min(n, b0 + per);
  int local = 0;
  for (int i = b0; i < b1; ++i) local += v[i];
  int incl = local;
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) s_warp[warp] = incl;
  __syncthreads();
  int wbase = 0, total = 0;
  for (int w = 0; w < nw; ++w) {
    const int x = s_warp[w];
    if (w < warp) wbase += x;
    total += x;
  }
  int run = wbase + incl - local;
  for (int i = b0; i < b1; ++i) {
    const int x = v[i];
    v[i] = run;
    run += x;
  }
  __syncthreads();
  return total;
}

// Builds the k+2 segments of (b, kv head) `bh`: sstart (physical first
// token), svstart (virtual first position; svstart[k+2] = n_att).
// Malformed idx entries become empty segments and are reported.
__device__ inline int build_segments(const AttendArgs& a, int bh, int* sstart, int* svstart,
                                     int* s_warp) {
  const int nseg = a.k + 2;
  for (int i = threadIdx.x; i < nseg; i += blockDim.x) {
    int64_t start, len;
    if (i == 0) {
      start = 0;
      len = a.sink_end;
    } else if (i == nseg - 1) {
      start = a.w0;
      len = a.T - a.w0;
    } else {
      const int j = a.idx[int64_t(bh) * a.k + i - 1];
      const bool ok = j >= a.first && j < a.first + a.nc &&
                      (i == 1 || a.idx[int64_t(bh) * a.k + i - 2] < j);
      if (!ok) report(a.status, RBA_ERR_BOUNDS, kWhereAttend, j);
      const int64_t lo = max(int64_t(j) * a.bs, int64_t(a.sink));
      const int64_t hi = min(int64_t(j + 1) * a.bs, a.w0);
      start = lo;
      len = ok && hi > lo ? hi - lo : 0;
    }
    sstart[i] = static_cast<int>(start);
    svstart[i] = static_cast<int>(len);
  }
  __syncthreads();
  const int total = block_exclusive_scan(svstart, nseg, s_warp);
  if (threadIdx.x == 0) svstart[nseg] = total;
  __syncthreads();
  return total;
}

// physical token of virtual position v (0 <= v < n_att).  unit: every
// selected segment is one token (token-level retrieval), so segment i >= 1
// starts at virtual position svstart[1] + i - 1 and no search is needed.
__device__ __forceinline__ int seg_map(const int* sstart, const int* svstart, int nseg, int v,
                                       bool unit) {
  if (unit) {
    const int i = v < svstart[1] ? 0 : min(1 + v - svstart[1], nseg - 1);
    return sstart[i] + (v - svstart[i]);
  }
  int lo = 0, hi = nseg - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (svstart[mid] <= v) lo = mid; else hi = mid - 1;
  }
  return sstart[lo] + (v - svstart[lo]);
}

// ---------------------------------------------------------------------------
// staging

template <typename T, int D>
__device__ __forceinline__ void issue_tile(const AttendArgs& a, int64_t bh_row0, char* stage,
                                           const int* sstart, const int* svstart, int nseg,
                                           int v0, int v1, bool unit) {
  using C = DecodeTile<T, D>;
  const char* Kb = static_cast<const char*>(a.K);
  const char* Vb = static_cast<const char*>(a.V);
  constexpr int HALF = C::TT * C::CPR;
#pragma unroll
  for (int i = 0; i < C::LOADS; ++i) {
    const int c = threadIdx.x + i * kAttendThreads;
    const bool isv = c >= HALF;
    const int cc = isv ? c - HALF : c;
    const int row = cc / C::CPR, col = cc % C::CPR;
    const int v = v0 + row;
    if (v < v1) {
      const int64_t tok = bh_row0 + seg_map(sstart, svstart, nseg, v, unit);
      const char* src = (isv ? Vb : Kb) + tok * C::ROWB + col * 16;
      cp_async16(stage + (isv ? HALF * 16 : 0) + row * C::ROWB + col * 16, src);
    }
  }
}

// ---------------------------------------------------------------------------
// per-lane online softmax over staged tiles

template <typename T, int D, int G>
struct LaneState {
  using C = DecodeTile<T, D>;
  float2 q[G][C::EPL / 2];   // scaled query slice (rotated chunk order)
  float2 o[G][C::EPL / 2];   // unnormalised output slice
  float m[G];                // running max (base-2 logits)
  float l[G];                // running sum of exp2(x - m)
};

template <typename T, int D>
__device__ __forceinline__ int lane_rot(int part) {
  using C = DecodeTile<T, D>;
  return (part * C::CPL) / 8;
}

// Query heads g0 .. g0 + G - 1 of the group of (b, kv head) bh (the group
// has Hq / Hkv heads).
template <typename T, int D, int G>
__device__ __forceinline__ void load_q(const AttendArgs& a, int bh, LaneState<T, D, G>& st,
                                       int g0 = 0) {
  using C = DecodeTile<T, D>;
  const int lane = threadIdx.x & 31;
  const int part = lane % C::LPR;
  const int rot = lane_rot<T, D>(part);
  const int b = bh / a.Hkv, h = bh % a.Hkv;
  const int grp = a.Hq / a.Hkv;
  const T* q = static_cast<const T*>(a.q);
#pragma unroll
  for (int g = 0; g < G; ++g) {
    // q rows are qd long; columns past qd count as zero
    const T* qr = q + (int64_t(b) * a.Hq + h * grp + g0 + g) * a.qd;
#pragma unroll
    for (int j = 0; j < C::CPL; ++j) {
      const int jj = (j + rot) % C::CPL;
#pragma unroll
      for (int e = 0; e < C::EPC; e += 2) {
        const int col = part * C::EPL + jj * C::EPC + e;  // qd is even: col, col + 1 agree
        st.q[g][(j * C::EPC + e) / 2] =
            col < a.qd ? make_float2(Elem<T>::to_f32(qr[col]) * a.scale_log2,
                                     Elem<T>::to_f32(qr[col + 1]) * a.scale_log2)
                       : make_float2(0.f, 0.f);
      }
    }
    st.m[g] = -INFINITY;
    st.l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < C::EPL / 2; ++e) st.o[g][e] = make_float2(0.f, 0.f);
  }
}

template <typename T, int D>
__device__ __forceinline__ void load_slice(const char* row, int part, int rot, float2* f) {
  using C = DecodeTile<T, D>;
#pragma unroll
  for (int j = 0; j < C::CPL; ++j) {
    const int jj = (j + rot) % C::CPL;
    const uint4 u = *reinterpret_cast<const uint4*>(row + (part * C::CPL + jj) * 16);
    float tmp[C::EPC];
    unpack(u, tmp, T());
#pragma unroll
    for (int e = 0; e < C::EPC; e += 2) f[(j * C::EPC + e) / 2] = make_float2(tmp[e], tmp[e + 1]);
  }
}

// Consume one staged tile of `nvalid` rows; `warp` is this warp's index
// among the NW consuming warps (it owns rows [warp * TPW * NT, +TPW * NT)).
template <typename T, int D, int G, int NW = kAttendWarps>
__device__ __forceinline__ void consume_tile(const char* stage, int nvalid,
                                             LaneState<T, D, G>& st, int warp) {
  using C = DecodeTile<T, D, NW>;
  const int lane = threadIdx.x & 31;
  const int slot = lane / C::LPR, part = lane % C::LPR;
  const int rot = lane_rot<T, D>(part);
  const char* sK = stage;
  const char* sV = stage + C::TT * C::ROWB;
  float x[C::NT][G];
#pragma unroll
  for (int n = 0; n < C::NT; ++n) {
    const int row = warp * C::TPW * C::NT + n * C::TPW + slot;
    float2 kf[C::EPL / 2];
    load_slice<T, D>(sK + row * C::ROWB, part, rot, kf);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float2 acc = make_float2(0.f, 0.f);
#pragma unroll
      for (int e = 0; e < C::EPL / 2; ++e) acc = __ffma2_rn(st.q[g][e], kf[e], acc);
      x[n][g] = acc.x + acc.y;
    }
  }
#pragma unroll
  for (int n = 0; n < C::NT; ++n)
#pragma unroll
    for (int g = 0; g < G; ++g)
#pragma unroll
      for (int o = C::LPR / 2; o > 0; o >>= 1)
        x[n][g] += __shfl_xor_sync(0xffffffffu, x[n][g], o);
  bool valid[C::NT];
#pragma unroll
  for (int n = 0; n < C::NT; ++n) {
    const int row = warp * C::TPW * C::NT + n * C::TPW + slot;
    valid[n] = row < nvalid;
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float mt = -INFINITY;
#pragma unroll
    for (int n = 0; n < C::NT; ++n)
      if (valid[n]) mt = fmaxf(mt, x[n][g]);
    if (mt > st.m[g]) {
      const float c = exp2f(st.m[g] - mt);
      st.l[g] *= c;
      const float2 c2 = make_float2(c, c);
#pragma unroll
      for (int e = 0; e < C::EPL / 2; ++e) st.o[g][e] = __fmul2_rn(st.o[g][e], c2);
      st.m[g] = mt;
    }
  }
#pragma unroll
  for (int n = 0; n < C::NT; ++n) {
    if (!valid[n]) continue;
    const int row = warp * C::TPW * C::NT + n * C::TPW + slot;
    float2 vf[C::EPL / 2];
    load_slice<T, D>(sV + row * C::ROWB, part, rot, vf);
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float p = exp2f(x[n][g] - st.m[g]);
      st.l[g] += p;
      const float2 p2 = make_float2(p, p);
#pragma unroll
      for (int e = 0; e < C::EPL / 2; ++e) st.o[g][e] = __ffma2_rn(p2, vf[e], st.o[g][e]);
    }
  }
}

// Combine (m, l, o) of lanes `off` apart (same row slice, other slots).
template <typename T, int D, int G>
__device__ __forceinline__ void merge_slots(LaneState<T, D, G>& st) {
  using C = DecodeTile<T, D>;
#pragma unroll
  for (int off = C::LPR; off < 32; off <<= 1) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float mo = __shfl_xor_sync(0xffffffffu, st.m[g], off);
      const float lo = __shfl_xor_sync(0xffffffffu, st.l[g], off);
      const float mn = fmaxf(st.m[g], mo);
      const float ca = st.m[g] == -INFINITY ? 0.f : exp2f(st.m[g] - mn);
      const float cb = mo == -INFINITY ? 0.f : exp2f(mo - mn);
      st.l[g] = st.l[g] * ca + lo * cb;
      const float2 ca2 = make_float2(ca, ca), cb2 = make_float2(cb, cb);
#pragma unroll
      for (int e = 0; e < C::EPL / 2; ++e) {
        float2 oo;
        oo.x = __shfl_xor_sync(0xffffffffu, st.o[g][e].x, off);
        oo.y = __shfl_xor_sync(0xffffffffu, st.o[g][e].y, off);
        st.o[g][e] = __ffma2_rn(oo, cb2, __fmul2_rn(st.o[g][e], ca2));
      }
      st.m[g] = mn;
    }
  }
}

// Reduce the warps' states through shared memory `red` ([NW][G][D+2] floats)
// and write the CTA's partial for split `split` of (b, kv head) `bh`.
template <typename T, int D, int G>
__device__ __forceinline__ void write_partial(const AttendArgs& a, int bh, int split,
                                              LaneState<T, D, G>& st, float* red) {
  using C = DecodeTile<T, D>;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int slot = lane / C::LPR, part = lane % C::LPR;
  const int rot = lane_rot<T, D>(part);
  merge_slots<T, D, G>(st);
  if (slot == 0) {
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float* r = red + (warp * G + g) * (D + 2);
      if (part == 0) {
        r[0] = st.m[g];
        r[1] = st.l[g];
      }
#pragma unroll
      for (int j = 0; j < C::CPL; ++j) {
        const int jj = (j + rot) % C::CPL;
#pragma unroll
        for (int e = 0; e < C::EPC; e += 2) {
          const float2 v = st.o[g][(j * C::EPC + e) / 2];
          r[2 + part * C::EPL + jj * C::EPC + e] = v.x;
          r[2 + part * C::EPL + jj * C::EPC + e + 1] = v.y;
        }
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < G * (D + 2); i += blockDim.x) {
    const int g = i / (D + 2), c = i % (D + 2);
    float M = -INFINITY;
    for (int w = 0; w < kAttendWarps; ++w) M = fmaxf(M, red[(w * G + g) * (D + 2)]);
    float acc = 0.f;
    if (c == 0) {
      acc = M;
    } else {
      for (int w = 0; w < kAttendWarps; ++w) {
        const float mw = red[(w * G + g) * (D + 2)];
        const float f = mw == -INFINITY ? 0.f : exp2f(mw - M);
        acc += red[(w * G + g) * (D + 2) + c] * f;
      }
    }
    a.part[((int64_t(bh) * G + g) * a.nsplit + split) * (D + 2) + c] = acc;
  }
}

// The last CTA of (b, kv head) to finish merges the split partials.
// `wsm` is shared scratch of G * nsplit floats.
template <int D, int G>
__device__ __forceinline__ void merge_partials_last(const AttendArgs& a, int bh, float* wsm,
                                                    bool* s_last) {
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t t = atomicAdd(a.tickets + bh, 1u);
    *s_last = t == uint32_t(a.nsplit - 1);
  }
  __syncthreads();
  if (!*s_last) return;
  __threadfence();
  const int ns = a.nsplit;
  // per q head: max and weights exp2(m_s - M) / L
  for (int g = threadIdx.x >> 5; g < G; g += blockDim.x >> 5) {
    const int lane = threadIdx.x & 31;
    const float* p = a.part + (int64_t(bh) * G + g) * ns * (D + 2);
    float M = -INFINITY;
    for (int s = lane; s < ns; s += 32) M = fmaxf(M, __ldcg(p + s * (D + 2)));
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.f;
    for (int s = lane; s < ns; s += 32) {
      const float ms = __ldcg(p + s * (D + 2));
      const float w = ms == -INFINITY ? 0.f : exp2f(ms - M);
      wsm[g * ns + s] = w;
      L += w * __ldcg(p + s * (D + 2) + 1);
    }
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    __syncwarp();
    const float inv = L > 0.f ? 1.f / L : 0.f;
    for (int s = lane; s < ns; s += 32) wsm[g * ns + s] *= inv;
    if (lane == 0 && a.lse != nullptr) {
      const int b = bh / a.Hkv, h = bh % a.Hkv;
      a.lse[int64_t(b) * a.Hq + h * G + g] =
          L > 0.f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < G * a.qd; i += blockDim.x) {
    const int g = i / a.qd, d = i % a.qd;
    const float* p = a.part + (int64_t(bh) * G + g) * ns * (D + 2) + 2 + d;
    float acc = 0.f;
    for (int s = 0; s < ns; ++s) acc += wsm[g * ns + s] * __ldcg(p + s * (D + 2));
    const int b = bh / a.Hkv, h = bh % a.Hkv;
    a.out[(int64_t(b) * a.Hq + h * G + g) * a.qd + d] = acc;
  }
  if (threadIdx.x == 0) a.tickets[bh] = 0;
}

// host helpers
size_t attend_workspace_bytes(int BH, int Hq_total, int D, int nsplit);
// workspace of the split-K kernel alone for this problem
size_t splitk_workspace_bytes(const rba_store* st, const Geometry& g, int k);
int attend_nsplit(int BH, int64_t n_att_max);
rba_status launch_attend(const rba_store* st, const void* q, const int32_t* idx, int k,
                         const Geometry& g, float scale, float* out, float* lse, void* ws,
                         size_t ws_bytes, cudaStream_t stream);

}  // namespace rba
