// One decode step in one persistent launch: block scores -> top-k ->
// split attention over sink U retrieved blocks U window -> log-sum-exp merge.
//
// Same definitions as rba_score / rba_topk / rba_attend (InfLLM article,
// "method" and "overall framework"; Landmark Attention review, "proposed
// method"; MemLong summary, 2.3.2 TopK and 2.3.3).  What this launch adds is
// the schedule:
//   * one CTA per SM: warp 0 only stages data, warps 1..7 compute;
//   * every CTA gets an equal share of two flattened work lists, processed
//     in order: (1) candidate blocks to score, (2) attention rows, where each
//     head's share mixes sink + window rows (no selection needed) and rows of
//     the selected blocks in proportion;
//   * warp 0 walks the same item sequence as the compute warps and stages
//     each item with bulk asynchronous copies (whole contiguous runs: rep keys
//     of consecutive candidates, K/V rows of a segment) into a ring of
//     shared-memory stages guarded by full / empty mbarriers, waiting for a
//     head's selection only when it reaches that head's selected rows;
//   * the last CTA to finish scoring a (batch, kv head) selects its top-k and
//     publishes a ready flag; selection overlaps the sink/window stream;
//   * partial softmax states go to per-(head, CTA) slots; the last
//     contributor of a head merges them (no CTA waits for a merge).
// No wait can be circular: scoring depends only on a CTA's own stager, and
// every CTA scores before it attends.  All waits are bounded in time; on
// expiry the kernel records RBA_ERR_TIMEOUT in the status word, skips the
// remaining work, waits (bounded) for its copies in flight and terminates.
#include <cstdio>
#include <cstdlib>

#include "attend_impl.cuh"
#include "topk_impl.cuh"

namespace rba {
namespace {

constexpr int kCW = 7;                        // compute warps (warps 1..7)
constexpr int kCT = kCW * 32;                 // compute threads
constexpr int kFT = kCT + 32;                 // + warp 0, which stages
constexpr int kMaxN = 8192;                   // candidates per (b, kv head)
constexpr int kMaxK = 1024;
constexpr int kMaxTouch = 64;                 // heads one CTA's score range may touch
constexpr int kMaxStages = 6;
constexpr int kMaxSlots = 128;                // partial slots per head
constexpr int kMinRowsPerCta = 128;           // grid shrinks for small problems
constexpr int kMaxGrid = 256;                 // CTAs (one per SM)
constexpr int kBins = 256;                    // value bins of the top-k select
constexpr unsigned long long kTimeoutNs = 2000000000ull;
static_assert(kMaxTouch * 128 <= kMaxN, "summed queries share the top-k key buffer");

struct FusedArgs {
  AttendArgs at;            // K, V, q, out, lse, status, cap, T, w0, Hq, Hkv, k, bs, sink,
                            // sink_end, first, nc, scale_log2 (part/tickets/nsplit unused)
  const char* rep;          // rep rows: [BH][rep_rows][rep_bytes]
  int64_t rep_rows;
  int rep_bytes;            // bytes of one candidate's representation
  int score_cap;            // candidates per score item
  float* scores;            // [BH][nc]
  int32_t* idx;             // [BH][k]
  float* slots;             // [BH][MS][G][D+2] partial states, one per contributing CTA
  uint32_t* tickets;        // [BH]
  uint32_t* ready;          // [BH]
  uint32_t* score_cnt;      // [BH]
  int BH, L_st, U_sel, MS, NS;
  bool rep_f32;
};

// ---------------------------------------------------------------------------
// small PTX helpers

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ unsigned long long now_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint64_t* b, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(b)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive_tx(uint64_t* b, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                   smem_u32(b)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* b) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(b))
               : "memory");
}
__device__ __forceinline__ bool mbar_try(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Warp-uniform bounded wait on an mbarrier phase (every lane acquires it).
// False when the CTA is aborting or the wait ran out (then reported, and
// the abort flag set).
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity, volatile int* abort_flag,
                                          int32_t* status, int where) {
  bool ok = mbar_try(b, parity);
  if (__all_sync(0xffffffffu, ok)) return true;
  const unsigned long long t0 = now_ns();
  while (true) {
    if (!ok) ok = mbar_try(b, parity);
    if (__all_sync(0xffffffffu, ok)) return true;
    if (__any_sync(0xffffffffu, *abort_flag != 0)) return false;
    if (__shfl_sync(0xffffffffu, now_ns() - t0 > kTimeoutNs, 0)) {
      if ((threadIdx.x & 31) == 0) {
        report(status, RBA_ERR_TIMEOUT, kWhereFused, where);
        *abort_flag = 1;
      }
      __syncwarp();
      return false;
    }
  }
}
// bounded wait that ignores the abort flag (draining copies in flight)
__device__ __forceinline__ void mbar_drain(uint64_t* b, uint32_t parity) {
  const unsigned long long t0 = now_ns();
  while (!mbar_try(b, parity) && now_ns() - t0 <= kTimeoutNs) {
  }
}
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(uint32_t* p, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t* p, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;"
               : "=r"(old)
               : "l"(p), "r"(v)
               : "memory");
  return old;
}
// barrier of the compute warps only (warp 0 never joins it)
__device__ __forceinline__ void compute_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(kCT) : "memory");
}
__device__ __forceinline__ int ctid() { return static_cast<int>(threadIdx.x) - 32; }
__device__ __forceinline__ int cwarp() { return static_cast<int>(threadIdx.x >> 5) - 1; }

// ---------------------------------------------------------------------------
// work lists

__device__ __forceinline__ int64_t bnd(int p, int P, int64_t total) {
  return total * p / P;
}

// CTAs whose share of a phase list meets head bh's rows: how many (= the
// partials that head receives) and the ordinal of CTA `me` among them (its
// slot), or -1 if it is not one of them.  `B` holds the phase's CTA
// boundaries bnd(0..P) (no division here).
__device__ __forceinline__ int contributors(int bh, int64_t per_bh, int P, const int64_t* B,
                                            int me, int* ordinal) {
  *ordinal = -1;
  if (per_bh <= 0) return 0;
  const int64_t a = bh * per_bh, b = a + per_bh;
  // first CTA whose range ends after a: the largest p with B[p] <= a
  int lo = 0, hi = P - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (B[mid] <= a) lo = mid; else hi = mid - 1;
  }
  int c = 0;
  for (int p = lo; p < P && B[p] < b; ++p) {
    const int64_t s = max(B[p], a), e = min(B[p + 1], b);
    if (e > s) {
      if (p == me) *ordinal = c;
      ++c;
    }
  }
  return c;
}

struct Item {
  int kind;  // 0 score, 1 sink/window rows, 2 selected rows
  int bh;
  int v0, v1;
};

// A CTA's walk over its work, without divisions per item:
//   phase 0: its share of the flattened candidate list (BH x nc);
//   phase 1: its share of the flattened attention list, where head h
//     contributes Lh = L_st + U_sel rows; a share [x0, x1) of head h maps to
//     sink/window rows [st(x0), st(x1)) and selected rows
//     [x0 - st(x0), x1 - st(x1)) with st(x) = floor(x * L_st / Lh), so a CTA
//     streams both parts of one head with one softmax state.
struct Iter {
  int phase;          // 0 score, 1 attention, 2 done
  int64_t r, r1;      // remaining range of the current phase's list
  int bh, loc;        // score: position
  int kind, v, vend;  // attention: current part of head bh
  int sel0, sel1;
};

__device__ __forceinline__ void attn_head(const FusedArgs& a, Iter& it) {
  const int64_t Lh = a.L_st + a.U_sel;
  const int64_t h0 = int64_t(it.bh) * Lh;
  const int64_t x0 = max(it.r, h0) - h0, x1 = min(it.r1, h0 + Lh) - h0;
  const int64_t s0 = x0 * a.L_st / Lh, s1 = x1 * a.L_st / Lh;
  it.kind = 1;
  it.v = static_cast<int>(s0);
  it.vend = static_cast<int>(s1);
  it.sel0 = static_cast<int>(x0 - s0);
  it.sel1 = static_cast<int>(x1 - s1);
}

// B0: CTA boundaries bnd(0..P) of the candidate list
__device__ __forceinline__ void iter_begin(const FusedArgs& a, Iter& it, const int64_t* B0) {
  it.phase = 0;
  it.r = B0[blockIdx.x];
  it.r1 = B0[blockIdx.x + 1];
  if (it.r < it.r1) {
    it.bh = static_cast<int>(it.r / a.at.nc);
    it.loc = static_cast<int>(it.r - int64_t(it.bh) * a.at.nc);
  }
}

// B1: CTA boundaries of the attention list
template <int TT>
__device__ __forceinline__ bool next_item(const FusedArgs& a, Iter& it, Item& out,
                                          const int64_t* B1) {
  if (it.phase == 0) {
    if (it.r < it.r1) {
      const int L = a.at.nc;
      int n = min(L - it.loc, a.score_cap);
      if (n > it.r1 - it.r) n = static_cast<int>(it.r1 - it.r);
      out.kind = 0;
      out.bh = it.bh;
      out.v0 = it.loc;
      out.v1 = it.loc + n;
      it.loc += n;
      it.r += n;
      if (it.loc == L) {
        ++it.bh;
        it.loc = 0;
      }
      return true;
    }
    it.phase = 1;
    it.r = B1[blockIdx.x];
    it.r1 = B1[blockIdx.x + 1];
    if (it.r >= it.r1) {
      it.phase = 2;
      return false;
    }
    it.bh = static_cast<int>(it.r / (int64_t(a.L_st) + a.U_sel));
    attn_head(a, it);
  }
  while (it.phase == 1) {
    if (it.v < it.vend) {
      const int n = min(it.vend - it.v, TT);
      out.kind = it.kind;
      out.bh = it.bh;
      out.v0 = it.v;
      out.v1 = it.v + n;
      it.v += n;
      return true;
    }
    if (it.kind == 1) {
      it.kind = 2;
      it.v = it.sel0;
      it.vend = it.sel1;
      continue;
    }
    ++it.bh;
    if (int64_t(it.bh) * (int64_t(a.L_st) + a.U_sel) >= it.r1) {
      it.phase = 2;
      break;
    }
    attn_head(a, it);
  }
  return false;
}

// ---------------------------------------------------------------------------
// shared memory layout

struct __align__(16) Meta {
  int nrows;
  int pad[3];
};

template <typename T, int D, int G>
struct FusedSmem {
  using C = DecodeTile<T, D, kCW>;
  static constexpr int STAGE = C::STAGE;
  // regions after the stage ring (NS * STAGE, chosen at launch)
  static constexpr int up16(int x) { return (x + 15) & ~15; }
  static constexpr int RED = up16(kCW * G * (D + 2) * 4);       // warp states / merge sums
  static constexpr int SEL = (kMaxK + 4) * 4 * 2;               // selected prefix + starts
  static constexpr int SLOTS = up16((kMaxSlots + 3 * G * kMaxSlots) * 4);  // merge: m, l, w
  static constexpr int MISC = 4096;
  static constexpr int KEYS = kMaxN * 4;      // top-k values or keys; summed queries first
  static constexpr int FLAGS = kMaxN + kCT * 4;  // top-k: selected flags, boundary-bin members
  static constexpr int BOUNDS = 2 * (kMaxGrid + 1) * 8;         // CTA boundaries, 2 lists
  static size_t bytes(int NS) {
    return size_t(NS) * STAGE + RED + SEL + SLOTS + MISC + KEYS + FLAGS + BOUNDS;
  }
};

// ---------------------------------------------------------------------------
// compute-warp helpers

__device__ __forceinline__ int compute_exclusive_scan(int v, int* s_w, int* total) {
  const int lane = threadIdx.x & 31, cw = cwarp();
  int incl = v;
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) s_w[cw] = incl;
  compute_sync();
  int base = 0, tot = 0;
  for (int w = 0; w < kCW; ++w) {
    const int x = s_w[w];
    if (w < cw) base += x;
    tot += x;
  }
  compute_sync();
  *total = tot;
  return base + incl - v;
}

// Positions whose flag is set, written ascending to idx[bh] (first + j).
__device__ __forceinline__ void write_selected(const FusedArgs& a, int bh, const uint8_t* flag,
                                               int* s_w) {
  const int n = a.at.nc;
  const int per = (n + kCT - 1) / kCT;
  const int p0 = ctid() * per, p1 = min(n, p0 + per);
  int cnt = 0;
  for (int j = p0; j < p1; ++j) cnt += flag[j];
  int tot;
  int rank = compute_exclusive_scan(cnt, s_w, &tot);
  int32_t* dst = a.idx + int64_t(bh) * a.at.k;
  for (int j = p0; j < p1; ++j)
    if (flag[j]) dst[rank++] = a.at.first + j;
}

// Exact top-k of row bh by the radix select of the k-th largest
// order-preserving score value; ties at that value go to the lower
// positions.  `keys` holds kMaxN words.
__device__ __noinline__ void topk_radix(const FusedArgs& a, int bh, uint32_t* hist, int* s_w,
                                        int* s_misc, uint32_t* keys, uint8_t* flag) {
  const int n = a.at.nc, k = a.at.k;
  const int tid = ctid(), lane = threadIdx.x & 31;
  const float* s = a.scores + int64_t(bh) * n;
  for (int j = tid; j < n; j += kCT) keys[j] = ordered_f32(__ldcg(s + j));
  compute_sync();
  uint32_t prefix = 0, mask = 0;
  int kk = k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = tid; b < 256; b += kCT) hist[b] = 0;
    compute_sync();
    // lanes falling into the same bin add once
    for (int j0 = tid - lane; j0 < n; j0 += kCT) {
      const int j = j0 + lane;
      const uint32_t u = j < n ? keys[j] : 0u;
      const bool in = j < n && (u & mask) == prefix;
      const uint32_t bin = in ? ((u >> shift) & 255u) : 256u;
      const unsigned same = __match_any_sync(0xffffffffu, bin);
      if (in && lane == __ffs(same) - 1) atomicAdd(&hist[bin], uint32_t(__popc(same)));
    }
    compute_sync();
    if (tid < 32) {
      // lane l owns bins [8l, 8l+8); counts above a bin = all higher bins
      uint32_t c[8], tot = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        c[i] = hist[tid * 8 + i];
        tot += c[i];
      }
      uint32_t incl = tot;  // sum over lanes >= tid
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t t = __shfl_down_sync(0xffffffffu, incl, o);
        if (tid + o < 32) incl += t;
      }
      uint32_t above = incl - tot;
#pragma unroll
      for (int i = 7; i >= 0; --i) {
        if (above < uint32_t(kk) && uint32_t(kk) <= above + c[i]) {
          s_misc[0] = tid * 8 + i;
          s_misc[1] = static_cast<int>(above);
        }
        above += c[i];
      }
    }
    compute_sync();
    prefix |= uint32_t(s_misc[0]) << shift;
    mask |= 255u << shift;
    kk -= s_misc[1];
    compute_sync();
  }
  // prefix = the k-th largest value: every larger score, and the first kk
  // equal ones in position order
  const int per = (n + kCT - 1) / kCT;
  const int p0 = tid * per, p1 = min(n, p0 + per);
  int n_eq = 0;
  for (int j = p0; j < p1; ++j) n_eq += keys[j] == prefix;
  int tot;
  int e = compute_exclusive_scan(n_eq, s_w, &tot);
  for (int j = p0; j < p1; ++j) {
    const uint32_t u = keys[j];
    flag[j] = u > prefix || (u == prefix && e++ < kk);
  }
  compute_sync();
  write_selected(a, bh, flag, s_w);
  compute_sync();
}

// value bin of x: monotone non-decreasing in x, so every score in a higher
// bin is strictly larger than every score in a lower one
__device__ __forceinline__ int value_bin(float x, float lo, float scale) {
  const float t = __fmul_rn(__fsub_rn(x, lo), scale);
  return min(kBins - 1, static_cast<int>(t));
}

// Exact top-k of row bh (1 <= k < n) with one histogram pass: kBins bins
// linear in the score value between the row's min and max; every score in
// the bins above the bin holding the k-th largest is selected, and inside
// that bin the members are ranked exactly (value, then lower position).
// Returns false (nothing written) for rows it does not cover -- non-finite
// scores, a zero range, or more members in the boundary bin than compute
// threads -- which the radix select then takes.
__device__ __noinline__ bool topk_binned(const FusedArgs& a, int bh, uint32_t* hist, int* s_w,
                                         int* s_misc, float* s_f, float* vals, uint8_t* flag,
                                         int* cand) {
  const int n = a.at.nc, k = a.at.k;
  const int tid = ctid(), lane = threadIdx.x & 31, cw = cwarp();
  const float* s = a.scores + int64_t(bh) * n;
  float lo = INFINITY, hi = -INFINITY;
  int bad = 0;
  for (int j = tid; j < n; j += kCT) {
    const float v = __ldcg(s + j);
    vals[j] = v;
    bad |= !isfinite(v);
    lo = fminf(lo, v);
    hi = fmaxf(hi, v);
  }
  for (int b = tid; b < kBins; b += kCT) hist[b] = 0;
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  bad = __any_sync(0xffffffffu, bad);
  if (lane == 0) {
    s_f[2 * cw] = lo;
    s_f[2 * cw + 1] = hi;
    s_w[cw] = bad;
  }
  compute_sync();
  lo = s_f[0];
  hi = s_f[1];
  bad = s_w[0];
  for (int w = 1; w < kCW; ++w) {
    lo = fminf(lo, s_f[2 * w]);
    hi = fmaxf(hi, s_f[2 * w + 1]);
    bad |= s_w[w];
  }
  const float range = hi - lo;
  const float scale = float(kBins) / range;
  // (uniform: every compute thread decides on the same shared values)
  if (bad || !(range > 0.f) || !isfinite(range) || !isfinite(scale)) return false;
  for (int j0 = tid - lane; j0 < n; j0 += kCT) {
    const int j = j0 + lane;
    const int bin = j < n ? value_bin(vals[j], lo, scale) : kBins;
    const unsigned same = __match_any_sync(0xffffffffu, bin);
    if (j < n && lane == __ffs(same) - 1) atomicAdd(&hist[bin], uint32_t(__popc(same)));
  }
  compute_sync();
  if (cw == 0) {
    // lane l owns bins [8l, 8l+8); counts above a bin = all higher bins
    uint32_t c[8], tot = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      c[i] = hist[lane * 8 + i];
      tot += c[i];
    }
    uint32_t incl = tot;
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t t = __shfl_down_sync(0xffffffffu, incl, o);
      if (lane + o < 32) incl += t;
    }
    uint32_t above = incl - tot;
#pragma unroll
    for (int i = 7; i >= 0; --i) {
      if (above < uint32_t(k) && uint32_t(k) <= above + c[i]) {
        s_misc[0] = lane * 8 + i;
        s_misc[1] = static_cast<int>(above);
        s_misc[2] = static_cast<int>(c[i]);
      }
      above += c[i];
    }
    if (lane == 0) s_misc[3] = 0;
  }
  compute_sync();
  const int bstar = s_misc[0], n_above = s_misc[1], nb = s_misc[2];
  if (nb > kCT) return false;
  for (int j = tid; j < n; j += kCT) {
    const int bin = value_bin(vals[j], lo, scale);
    if (bin == bstar) cand[atomicAdd(&s_misc[3], 1)] = j;
    flag[j] = bin > bstar;
  }
  compute_sync();
  if (tid < nb) {
    const int j = cand[tid];
    const float x = vals[j];
    int rank = 0;  // boundary-bin members ahead of j
    for (int m = 0; m < nb; ++m) {
      const int jm = cand[m];
      const float y = vals[jm];
      rank += y > x || (y == x && jm < j);
    }
    flag[j] = rank < k - n_above;
  }
  compute_sync();
  write_selected(a, bh, flag, s_w);
  compute_sync();
  return true;
}

// Top-k of row bh into idx[bh], ascending (compute warps; ends with a barrier).
__device__ __forceinline__ void select_row(const FusedArgs& a, int bh, uint32_t* hist, int* s_w,
                                           int* s_misc, float* s_f, uint32_t* keys,
                                           uint8_t* flag, int* cand) {
  const int n = a.at.nc, k = a.at.k;
  if (k >= n) {  // every candidate
    for (int j = ctid(); j < n; j += kCT) a.idx[int64_t(bh) * k + j] = a.at.first + j;
    compute_sync();
    return;
  }
  if (!topk_binned(a, bh, hist, s_w, s_misc, s_f, reinterpret_cast<float*>(keys), flag, cand))
    topk_radix(a, bh, hist, s_w, s_misc, keys, flag);
}

// ---------------------------------------------------------------------------
// staging (warp 0)

// Stages one item into `stg`: bulk copies that complete on `bar`, whose
// transaction count is armed with the item's bytes.  Selected rows wait
// (bounded) for the head's selection.  False: aborting or timed out, nothing
// armed.
template <typename T, int D>
__device__ bool issue_item(const FusedArgs& a, const Item& item, char* stg, uint64_t* bar,
                           Meta* meta, int* sel_pref, int* sel_phys, int* sel_bh,
                           volatile int* abort_flag) {
  using C = DecodeTile<T, D, kCW>;
  const int lane = threadIdx.x & 31;
  if (item.kind == 0) {
    const int n = item.v1 - item.v0;
    if (lane == 0) {
      meta->nrows = n;
      const uint32_t bytes = uint32_t(n) * a.rep_bytes;
      mbar_arrive_tx(bar, bytes);
      bulk_g2s(stg, a.rep + (int64_t(item.bh) * a.rep_rows + a.at.first + item.v0) * a.rep_bytes,
               bytes, bar);
    }
    __syncwarp();
    return true;
  }
  const int* pref;
  const int* phys;
  int nseg;
  int st_pref[3], st_phys[2];
  if (item.kind == 1) {
    st_pref[0] = 0;
    st_pref[1] = a.at.sink_end;
    st_pref[2] = a.L_st;
    st_phys[0] = 0;
    st_phys[1] = static_cast<int>(a.at.w0);
    pref = st_pref;
    phys = st_phys;
    nseg = 2;
  } else {
    if (item.bh != *sel_bh) {
      // this head's selection (every lane acquires the flag), then the
      // layout of its blocks
      const uint32_t* flag = a.ready + item.bh;
      bool ok = ld_acquire(flag) != 0;
      if (!__all_sync(0xffffffffu, ok)) {
        const unsigned long long t0 = now_ns();
        while (true) {
          __nanosleep(32);
          if (!ok) ok = ld_acquire(flag) != 0;
          if (__all_sync(0xffffffffu, ok)) break;
          if (__any_sync(0xffffffffu, *abort_flag != 0)) return false;
          if (__shfl_sync(0xffffffffu, now_ns() - t0 > kTimeoutNs, 0)) {
            if (lane == 0) {
              report(a.at.status, RBA_ERR_TIMEOUT, kWhereFused, 2);
              *abort_flag = 1;
            }
            __syncwarp();
            return false;
          }
        }
      }
      const int k = a.at.k;
      int run = 0;
      for (int base = 0; base < k; base += 32) {
        const int j = base + lane;
        int len = 0, start = 0;
        if (j < k) {
          const int blk = __ldcg(a.idx + int64_t(item.bh) * k + j);
          const bool okb = blk >= a.at.first && blk < a.at.first + a.at.nc;
          const int64_t lo = max(int64_t(blk) * a.at.bs, int64_t(a.at.sink));
          const int64_t hi = min(int64_t(blk + 1) * a.at.bs, a.at.w0);
          start = static_cast<int>(lo);
          len = okb && hi > lo ? static_cast<int>(hi - lo) : 0;
          if (!okb) report(a.at.status, RBA_ERR_BOUNDS, kWhereFused, blk);
        }
        int incl = len;
        for (int o = 1; o < 32; o <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += t;
        }
        if (j < k) {
          sel_pref[j] = run + incl - len;
          sel_phys[j] = start;
        }
        run += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) sel_pref[k] = run;
      __syncwarp();
      *sel_bh = item.bh;
    }
    pref = sel_pref;
    phys = sel_phys;
    nseg = a.at.k;
  }
  const int total = pref[nseg];
  const int v0 = item.v0;
  const int v1 = min(item.v1, total);
  const int nrows = v1 > v0 ? v1 - v0 : 0;
  if (lane == 0) {
    meta->nrows = nrows;
    mbar_arrive_tx(bar, uint32_t(nrows) * C::ROWB * 2);
  }
  __syncwarp();
  if (nrows > 0) {
    // first segment holding v0: the last one with pref <= v0
    int lo = 0, hi = nseg - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pref[mid] <= v0) lo = mid; else hi = mid - 1;
    }
    const char* Kb = static_cast<const char*>(a.at.K);
    const char* Vb = static_cast<const char*>(a.at.V);
    for (int sg = lo + lane; sg < nseg && pref[sg] < v1; sg += 32) {
      const int a0 = max(v0, pref[sg]), a1 = min(v1, pref[sg + 1]);
      if (a1 <= a0) continue;
      const int64_t tok = int64_t(item.bh) * a.at.cap + phys[sg] + (a0 - pref[sg]);
      const uint32_t bytes = uint32_t(a1 - a0) * C::ROWB;
      const int row = a0 - v0;
      bulk_g2s(stg + row * C::ROWB, Kb + tok * C::ROWB, bytes, bar);
      bulk_g2s(stg + C::TT * C::ROWB + row * C::ROWB, Vb + tok * C::ROWB, bytes, bar);
    }
  }
  __syncwarp();
  return true;
}

// Warp 0: stage every item of this CTA, in order, into the stage ring.
template <typename T, int D>
__device__ __forceinline__ void produce(const FusedArgs& a, char* stages, uint64_t* full,
                                        uint64_t* empty, Meta* meta, int* sel_pref,
                                        int* sel_phys, volatile int* abort_flag,
                                        const int64_t* B0, const int64_t* B1) {
  using C = DecodeTile<T, D, kCW>;
  const int NS = a.NS;
  Iter it;
  iter_begin(a, it, B0);
  Item item;
  int j = 0, s = 0, sel_bh = -1;
  uint32_t ph = 0;  // phase parity of the stage's next fill
  while (next_item<C::TT>(a, it, item, B1)) {
    // stage s is free once every compute warp released its previous item
    if (j >= NS && !mbar_wait(&empty[s], ph ^ 1u, abort_flag, a.at.status, 1)) break;
    if (!issue_item<T, D>(a, item, stages + size_t(s) * C::STAGE, &full[s], &meta[s], sel_pref,
                          sel_phys, &sel_bh, abort_flag))
      break;
    ++j;
    if (++s == NS) {
      s = 0;
      ph ^= 1u;
    }
  }
  // no copy may still be landing in shared memory when the CTA exits
  if ((threadIdx.x & 31) == 0)
    for (int q = max(0, j - NS); q < j; ++q) mbar_drain(&full[q % NS], (q / NS) & 1u);
  __syncwarp();
}

// ---------------------------------------------------------------------------
// the kernel

template <typename T, int D, int G>
__global__ void __launch_bounds__(kFT, 1) decode_fused_kernel(FusedArgs a) {
  using C = DecodeTile<T, D, kCW>;
  using S = FusedSmem<T, D, G>;
  extern __shared__ __align__(128) char smem[];
  const int NS = a.NS;
  char* stages = smem;
  float* red = reinterpret_cast<float*>(smem + size_t(NS) * C::STAGE);
  int* sel_pref = reinterpret_cast<int*>(reinterpret_cast<char*>(red) + S::RED);
  int* sel_phys = sel_pref + (kMaxK + 1);
  float* wslot = reinterpret_cast<float*>(reinterpret_cast<char*>(sel_pref) + S::SEL);
  char* misc = reinterpret_cast<char*>(wslot) + S::SLOTS;
  uint64_t* full = reinterpret_cast<uint64_t*>(misc);               // [kMaxStages]
  uint64_t* empty = full + kMaxStages;                              // [kMaxStages]
  Meta* meta = reinterpret_cast<Meta*>(empty + kMaxStages);         // [kMaxStages]
  uint32_t* hist = reinterpret_cast<uint32_t*>(meta + kMaxStages);  // [kBins + 1]
  int* s_w = reinterpret_cast<int*>(hist + kBins + 1);              // [32]
  int* s_misc = s_w + 32;                                           // [16]
  int* owned = s_misc + 16;                                         // [kMaxTouch]
  volatile int* abort_flag = owned + kMaxTouch;                     // [4]
  float* s_f = reinterpret_cast<float*>(owned + kMaxTouch + 4);     // [32]
  uint32_t* keys = reinterpret_cast<uint32_t*>(misc + S::MISC);     // [kMaxN]
  uint8_t* flag = reinterpret_cast<uint8_t*>(misc + S::MISC + S::KEYS);  // [kMaxN]
  int* cand = reinterpret_cast<int*>(flag + kMaxN);                      // [kCT]
  int64_t* B0 = reinterpret_cast<int64_t*>(misc + S::MISC + S::KEYS + S::FLAGS);  // candidates
  int64_t* B1 = B0 + (kMaxGrid + 1);                                              // attention

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int P = gridDim.x, p = blockIdx.x;
  const int64_t Lh = int64_t(a.L_st) + a.U_sel;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCW);
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  for (int q = threadIdx.x; q <= P; q += kFT) {
    B0[q] = bnd(q, P, int64_t(a.at.k > 0 ? a.at.nc : 0) * a.BH);
    B1[q] = bnd(q, P, Lh * a.BH);
  }
  __syncthreads();
  if (warp == 0) {
    produce<T, D>(a, stages, full, empty, meta, sel_pref, sel_phys, abort_flag, B0, B1);
    return;
  }
  // ---- compute warps from here on (named barrier 1; no __syncthreads)
  const int cw = warp - 1, tid = ctid();

  // item i of this CTA sits in stage s with parity ph
  int s = 0;
  uint32_t ph = 0;
  auto wait_full = [&]() -> bool { return mbar_wait(&full[s], ph, abort_flag, a.at.status, 3); };
  auto release = [&]() {
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
  };
  auto advance = [&]() {
    if (++s == NS) {
      s = 0;
      ph ^= 1u;
    }
  };

  // summed query of every head this CTA scores (GQA: the group's q heads)
  const int64_t sr0 = B0[p], sr1 = B0[p + 1];
  const int bh_first = sr1 > sr0 ? static_cast<int>(sr0 / a.at.nc) : 0;
  const int n_touch = sr1 > sr0 ? static_cast<int>((sr1 - 1) / a.at.nc) - bh_first + 1 : 0;
  float* qsum = reinterpret_cast<float*>(keys);  // [n_touch][D]
  for (int x = tid; x < n_touch * D; x += kCT) {
    const int bh = bh_first + x / D, d = x % D;
    const int b = bh / a.at.Hkv, h = bh % a.at.Hkv;
    const T* qp = static_cast<const T*>(a.at.q) + (int64_t(b) * a.at.Hq + h * G) * D + d;
    float qs = 0.f;
    for (int gg = 0; gg < G; ++gg) qs += Elem<T>::to_f32(qp[gg * D]);
    qsum[x] = qs;
  }
  compute_sync();

  Iter it;
  iter_begin(a, it, B0);
  Item item;
  bool have = next_item<C::TT>(a, it, item, B1);

  // ---- phase 1: score this CTA's candidates
  while (have && item.kind == 0) {
    if (wait_full()) {
      const char* stg = stages + size_t(s) * C::STAGE;
      const int nrows = meta[s].nrows;
      const float* qv_ = qsum + (item.bh - bh_first) * D;
      const int vpc = a.rep_bytes / 16;     // vectors per candidate
      const int lpc = vpc < 32 ? vpc : 32;  // lanes per candidate
      const int cpw = 32 / lpc;
      const int sub = lane % lpc, slot = lane / lpc;
      for (int c = cw * cpw + slot; c - slot < nrows; c += kCW * cpw) {
        float acc = 0.f;
        if (c < nrows) {
          for (int v = sub; v < vpc; v += lpc) {
            const uint4 u =
                *reinterpret_cast<const uint4*>(stg + size_t(c) * a.rep_bytes + v * 16);
            float f[8];
            if (a.rep_f32) {
              const int d0 = (v * 4) % D;
              unpack(u, f, 0.f);
              const float4 qv = *reinterpret_cast<const float4*>(qv_ + d0);
              acc = fmaf(qv.x, f[0], acc);
              acc = fmaf(qv.y, f[1], acc);
              acc = fmaf(qv.z, f[2], acc);
              acc = fmaf(qv.w, f[3], acc);
            } else {
              const int d0 = (v * 8) % D;
              unpack(u, f, __nv_bfloat16());
              const float4 q0 = *reinterpret_cast<const float4*>(qv_ + d0);
              const float4 q1 = *reinterpret_cast<const float4*>(qv_ + d0 + 4);
              acc = fmaf(q0.x, f[0], acc);
              acc = fmaf(q0.y, f[1], acc);
              acc = fmaf(q0.z, f[2], acc);
              acc = fmaf(q0.w, f[3], acc);
              acc = fmaf(q1.x, f[4], acc);
              acc = fmaf(q1.y, f[5], acc);
              acc = fmaf(q1.z, f[6], acc);
              acc = fmaf(q1.w, f[7], acc);
            }
          }
        }
        for (int o = lpc / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (sub == 0 && c < nrows) a.scores[int64_t(item.bh) * a.at.nc + item.v0 + c] = acc;
      }
      release();
    }
    advance();
    have = next_item<C::TT>(a, it, item, B1);
  }

  // ---- selection: count this CTA's scores in; top-k the heads it completes
  compute_sync();
  if (tid == 0) {
    int n_owned = 0;
    if (sr1 > sr0) {
      const int64_t L = a.at.nc;
      for (int bh = bh_first; bh < bh_first + n_touch; ++bh) {
        const int64_t c0 = max(sr0, bh * L), c1 = min(sr1, (bh + 1) * L);
        const uint32_t cnt = static_cast<uint32_t>(c1 - c0);
        const uint32_t old = atom_add_acq_rel(a.score_cnt + bh, cnt);  // publishes our scores
        if (old + cnt == uint32_t(a.at.nc) && n_owned < kMaxTouch) owned[n_owned++] = bh;
      }
    }
    s_misc[8] = n_owned;
  }
  compute_sync();
  for (int o = 0; o < s_misc[8]; ++o) {
    const int bh = owned[o];
    select_row(a, bh, hist, s_w, s_misc, s_f, keys, flag, cand);  // ends with a barrier
    if (tid == 0) {
      __threadfence();
      st_release(a.ready + bh, 1u);
    }
  }

  // ---- attention over this CTA's rows, head by head
  LaneState<T, D, G> st;
  int cur_bh = -1;
  float* m_s = wslot + kMaxSlots;               // [nl][G]
  float* l_s = m_s + G * kMaxSlots;             // [nl][G]
  float* w_s = l_s + G * kMaxSlots;             // [G][nl]

  while (true) {
    const bool more = have;
    if (cur_bh >= 0 && (!more || item.bh != cur_bh)) {
      // ---- this CTA's state of head cur_bh -> its slot; the last
      // contributor of the head merges all of its slots
      merge_slots<T, D, G>(st);
      const int slot_lane = lane / C::LPR, part = lane % C::LPR;
      const int rot = lane_rot<T, D>(part);
      if (slot_lane == 0) {
#pragma unroll
        for (int gg = 0; gg < G; ++gg) {
          float* r = red + (cw * G + gg) * (D + 2);
          if (part == 0) {
            r[0] = st.m[gg];
            r[1] = st.l[gg];
          }
#pragma unroll
          for (int j = 0; j < C::CPL; ++j) {
            const int jj = (j + rot) % C::CPL;
#pragma unroll
            for (int e = 0; e < C::EPC; e += 2) {
              const float2 v = st.o[gg][(j * C::EPC + e) / 2];
              r[2 + part * C::EPL + jj * C::EPC + e] = v.x;
              r[2 + part * C::EPL + jj * C::EPC + e + 1] = v.y;
            }
          }
        }
      }
      compute_sync();
      int ord;
      const int ncontrib = contributors(cur_bh, Lh, P, B1, p, &ord);
      const bool slot_ok = ord >= 0 && ord < a.MS;
      if (!slot_ok && tid == 0) report(a.at.status, RBA_ERR_BOUNDS, kWhereFused, 4);
      float* base = a.slots + int64_t(cur_bh) * a.MS * G * (D + 2);
      float* slot = base + int64_t(slot_ok ? ord : 0) * G * (D + 2);
#pragma unroll 1
      for (int x = tid; x < G * (D + 2) && slot_ok; x += kCT) {
        const int gg = x / (D + 2), c = x % (D + 2);
        float M = -INFINITY;
        for (int w = 0; w < kCW; ++w) M = fmaxf(M, red[(w * G + gg) * (D + 2)]);
        float acc = 0.f;
        if (c == 0) {
          acc = M;
        } else {
          for (int w = 0; w < kCW; ++w) {
            const float mw = red[(w * G + gg) * (D + 2)];
            acc += red[(w * G + gg) * (D + 2) + c] * (mw == -INFINITY ? 0.f : exp2f(mw - M));
          }
        }
        slot[x] = acc;
      }
      compute_sync();
      if (tid == 0) {
        const uint32_t t = atom_add_acq_rel(a.tickets + cur_bh, 1u);  // publishes our slot
        s_misc[9] = t == uint32_t(ncontrib - 1);
      }
      compute_sync();
      if (s_misc[9]) {
        const int nl = min(ncontrib, a.MS);
        for (int x = tid; x < nl * G; x += kCT) {  // (m, l) of every slot, one round trip
          const int j = x / G, gg = x % G;
          const float* sp = base + (int64_t(j) * G + gg) * (D + 2);
          m_s[x] = __ldcg(sp);
          l_s[x] = __ldcg(sp + 1);
        }
        compute_sync();
        if (cw < G) {
          const int gg = cw;
          float M = -INFINITY;
          for (int j = lane; j < nl; j += 32) M = fmaxf(M, m_s[j * G + gg]);
          for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
          float L = 0.f;
          for (int j = lane; j < nl; j += 32) {
            const float ms_ = m_s[j * G + gg];
            const float wv = ms_ == -INFINITY ? 0.f : exp2f(ms_ - M);
            w_s[gg * kMaxSlots + j] = wv;
            L += wv * l_s[j * G + gg];
          }
          for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
          const float inv = L > 0.f ? 1.f / L : 0.f;
          for (int j = lane; j < nl; j += 32) w_s[gg * kMaxSlots + j] *= inv;
          if (lane == 0 && a.at.lse != nullptr) {
            const int b = cur_bh / a.at.Hkv, h = cur_bh % a.at.Hkv;
            a.at.lse[int64_t(b) * a.at.Hq + h * G + gg] =
                L > 0.f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
          }
        }
        compute_sync();
        // warps take slots round-robin and read each slot whole (coalesced)
        constexpr int PER = (G * D + 31) / 32;
        float acc[PER];
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[e] = 0.f;
#pragma unroll 1
        for (int j = cw; j < nl; j += kCW) {
          const float* sp = base + int64_t(j) * G * (D + 2);
          float v[PER];
#pragma unroll
          for (int e = 0; e < PER; ++e) {
            const int x = lane + 32 * e;  // output element (g, d)
            v[e] = x < G * D ? __ldcg(sp + (x / D) * (D + 2) + 2 + (x % D)) : 0.f;
          }
#pragma unroll
          for (int e = 0; e < PER; ++e) {
            const int x = lane + 32 * e;
            if (x < G * D) acc[e] += w_s[(x / D) * kMaxSlots + j] * v[e];
          }
        }
#pragma unroll
        for (int e = 0; e < PER; ++e) {
          const int x = lane + 32 * e;
          if (x < G * D) red[cw * G * D + x] = acc[e];
        }
        compute_sync();
        for (int x = tid; x < G * D; x += kCT) {
          float sum = 0.f;
          for (int w = 0; w < kCW; ++w) sum += red[w * G * D + x];
          const int gg = x / D, d = x % D;
          const int b = cur_bh / a.at.Hkv, h = cur_bh % a.at.Hkv;
          a.at.out[(int64_t(b) * a.at.Hq + h * G + gg) * D + d] = sum;
        }
        if (tid == 0) {  // leave the synchronisation state zero for the next call
          a.tickets[cur_bh] = 0;
          a.ready[cur_bh] = 0;
          a.score_cnt[cur_bh] = 0;
        }
      }
      compute_sync();
      cur_bh = -1;
    }
    if (!more) break;
    if (item.bh != cur_bh) {
      cur_bh = item.bh;
      load_q<T, D, G>(a.at, cur_bh, st);
    }
    if (wait_full()) {
      consume_tile<T, D, G, kCW>(stages + size_t(s) * C::STAGE, meta[s].nrows, st, cw);
      release();
    }
    advance();
    have = next_item<C::TT>(a, it, item, B1);
  }
}

template <typename T, int D, int G>
int fused_stages() {
  using S = FusedSmem<T, D, G>;
  int NS = kMaxStages;
  while (NS > 2 && S::bytes(NS) > 227 * 1024) --NS;
  return NS;
}

// CTAs of this kernel that fit on one SM (0: none; <0: a CUDA error)
template <typename T, int D, int G>
int fused_occupancy_t() {
  using S = FusedSmem<T, D, G>;
  const size_t smem = S::bytes(fused_stages<T, D, G>());
  auto kfn = decode_fused_kernel<T, D, G>;
  if (ensure_smem(reinterpret_cast<const void*>(kfn), smem) != cudaSuccess) return -1;
  int occ = 0;
  const cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kfn, kFT, smem);
  if (getenv("RBA_DEBUG") != nullptr) {
    cudaFuncAttributes fa = {};
    cudaFuncGetAttributes(&fa, kfn);
    fprintf(stderr,
            "rba: decode_fused_kernel regs=%d maxThreads=%d static_smem=%zu local=%zu "
            "max_dyn_smem=%d requested_smem=%zu threads=%d occupancy=%d (%s)\n",
            fa.numRegs, fa.maxThreadsPerBlock, fa.sharedSizeBytes, fa.localSizeBytes,
            fa.maxDynamicSharedSizeBytes, smem, kFT, occ, cudaGetErrorString(e));
  }
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return -2;
  }
  return occ;
}

template <typename T, int D, int G>
rba_status launch_fused_t(FusedArgs a, int P, cudaStream_t stream) {
  using S = FusedSmem<T, D, G>;
  using C = DecodeTile<T, D, kCW>;
  const int NS = fused_stages<T, D, G>();
  a.NS = NS;
  a.score_cap = C::STAGE / a.rep_bytes;
  if (a.score_cap < 1) return RBA_ERR_UNSUPPORTED;
  const size_t smem = S::bytes(NS);
  auto kfn = decode_fused_kernel<T, D, G>;
  const int occ = fused_occupancy_t<T, D, G>();
  if (occ < 0) return RBA_ERR_CUDA;
  if (occ < 1) return RBA_ERR_UNSUPPORTED;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(P);
  cfg.blockDim = dim3(kFT);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  RBA_CUDA_TRY(cudaLaunchKernelEx(&cfg, kfn, a));
  return RBA_OK;
}

}  // namespace

static int64_t phase_total(const rba_store* st, const Geometry& g, int k, int ph) {
  const int64_t BH = int64_t(st->d.batch) * st->d.n_kv_heads;
  const int64_t L = ph == 1 ? int64_t(g.sink_end) + (g.T - g.w0)
                            : (k > 0 ? int64_t(k) * st->d.block_size : 0);
  return BH * L;
}

// CTAs of the fused launch: one per SM, fewer for small problems.
int fused_grid(const rba_store* st, const Geometry& g, int k) {
  const int64_t rows = phase_total(st, g, k, 1) + phase_total(st, g, k, 2);
  int64_t P = (rows + kMinRowsPerCta - 1) / kMinRowsPerCta;
  if (P > num_sms()) P = num_sms();
  if (P > kMaxGrid) P = kMaxGrid;
  return static_cast<int>(P < 1 ? 1 : P);
}

// Bound on the CTAs whose share of a phase list meets one head's rows.
// (each contributor holds at least one of the head's rows, and at least
// floor(total / P) rows in all)
static int slots_bound(int64_t per_bh, int64_t total, int P) {
  if (per_bh <= 0) return 0;
  int64_t minlen = total / P;
  if (minlen < 1) minlen = 1;
  int64_t b = (per_bh + minlen - 1) / minlen + 1;
  if (b > per_bh) b = per_bh;
  return static_cast<int>(b);
}

size_t fused_slot_bytes(const rba_store* st, const Geometry& g, int k, int* ms) {
  const rba_store_desc& d = st->d;
  const int BH = d.batch * d.n_kv_heads;
  const int G = d.n_q_heads / d.n_kv_heads;
  const int P = fused_grid(st, g, k);
  const int64_t total = phase_total(st, g, k, 1) + phase_total(st, g, k, 2);
  const int m = slots_bound(total / BH, total, P);
  if (ms) *ms = m;
  return align_up(size_t(BH) * m * G * (d.head_dim + 2) * 4, 256);
}

size_t fused_sync_bytes(const rba_store* st) {
  return 3 * align_up(size_t(st->d.batch) * st->d.n_kv_heads * 4, 256);
}

// Whether the fused step covers this problem (else the three-launch path runs).
bool fused_eligible(const rba_store* st, const Geometry& g, int k) {
  const rba_store_desc& d = st->d;
  const int BH = d.batch * d.n_kv_heads;
  const int G = d.n_q_heads / d.n_kv_heads;
  if (d.mode == RBA_REP_EMBED_COSINE) return false;
  if (G != 1 && G != 2 && G != 4) return false;
  if (g.nc > kMaxN || k > kMaxK) return false;
  if (phase_total(st, g, k, 1) + phase_total(st, g, k, 2) == 0) return false;
  const int P = fused_grid(st, g, k);
  if (k > 0 && g.nc > 0) {
    const int64_t per_cta = (int64_t(BH) * g.nc + P - 1) / P;
    if (per_cta / g.nc + 2 > kMaxTouch) return false;
  }
  int ms = 0;
  fused_slot_bytes(st, g, k, &ms);
  return ms <= kMaxSlots;
}

int fused_occupancy(const rba_store* st) {
  const rba_store_desc& d = st->d;
  const int G = d.n_q_heads / d.n_kv_heads;
#define RBA_OCC(T_, D_)                                   \
  switch (G) {                                            \
    case 1: return fused_occupancy_t<T_, D_, 1>();        \
    case 2: return fused_occupancy_t<T_, D_, 2>();        \
    case 4: return fused_occupancy_t<T_, D_, 4>();        \
  }                                                       \
  return 0;
  if (d.dtype == RBA_BF16) {
    if (d.head_dim == 128) { RBA_OCC(__nv_bfloat16, 128) }
    RBA_OCC(__nv_bfloat16, 64)
  }
  if (d.head_dim == 128) { RBA_OCC(float, 128) }
  RBA_OCC(float, 64)
#undef RBA_OCC
}

rba_status launch_fused(const rba_store* st, const void* q, int k, const Geometry& g, float scale,
                        float* scores, int32_t* idx, float* out, float* lse, void* sync,
                        float* slots, cudaStream_t stream) {
  const rba_store_desc& d = st->d;
  const int P = fused_grid(st, g, k);
  const int BH = d.batch * d.n_kv_heads;
  FusedArgs a = {};
  AttendArgs& at = a.at;
  at.K = st->k;
  at.V = st->v;
  at.q = q;
  at.idx = idx;
  at.out = out;
  at.lse = lse;
  at.status = st->status;
  at.cap = d.capacity_tokens;
  at.T = g.T;
  at.w0 = g.w0;
  at.Hq = d.n_q_heads;
  at.Hkv = d.n_kv_heads;
  at.k = k;
  at.bs = d.block_size;
  at.sink = g.sink;
  at.sink_end = g.sink_end;
  at.nsplit = 1;
  at.first = g.first;
  at.nc = g.nc;
  at.scale_log2 = scale * 1.4426950408889634f;
  const size_t es = dtype_size(d.dtype);
  if (d.mode == RBA_REP_IDENTITY) {
    a.rep = static_cast<const char*>(st->k);
    a.rep_rows = d.capacity_tokens;
    a.rep_bytes = static_cast<int>(d.head_dim * es);
    a.rep_f32 = d.dtype == RBA_F32;
  } else {
    const bool f32 = d.mode == RBA_REP_MEAN || d.dtype == RBA_F32;
    a.rep = static_cast<const char*>(st->rep);
    a.rep_rows = st->cap_blocks;
    a.rep_bytes = static_cast<int>(d.n_rep * d.head_dim * (f32 ? 4 : es));
    a.rep_f32 = f32;
  }
  const size_t sb = align_up(size_t(BH) * 4, 256);
  a.tickets = static_cast<uint32_t*>(sync);
  a.ready = reinterpret_cast<uint32_t*>(static_cast<char*>(sync) + sb);
  a.score_cnt = reinterpret_cast<uint32_t*>(static_cast<char*>(sync) + 2 * sb);
  a.scores = scores;
  a.idx = idx;
  a.slots = slots;
  a.BH = BH;
  a.L_st = static_cast<int>(g.sink_end + (g.T - g.w0));
  a.U_sel = k > 0 ? k * d.block_size : 0;
  fused_slot_bytes(st, g, k, &a.MS);
  const int G = d.n_q_heads / d.n_kv_heads;
#define RBA_FUSED(T_, D_)                                               \
  switch (G) {                                                          \
    case 1: return launch_fused_t<T_, D_, 1>(a, P, stream);             \
    case 2: return launch_fused_t<T_, D_, 2>(a, P, stream);             \
    case 4: return launch_fused_t<T_, D_, 4>(a, P, stream);             \
  }                                                                     \
  return RBA_ERR_UNSUPPORTED;
  if (d.dtype == RBA_BF16) {
    if (d.head_dim == 128) { RBA_FUSED(__nv_bfloat16, 128) }
    RBA_FUSED(__nv_bfloat16, 64)
  }
  if (d.head_dim == 128) { RBA_FUSED(float, 128) }
  RBA_FUSED(float, 64)
#undef RBA_FUSED
}

}  // namespace rba
