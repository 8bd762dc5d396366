// Decode attention of one step in one persistent launch, overlapped with the
// selection that precedes it on the stream.
//
// Same definitions as rba_attend (InfLLM article, "overall framework";
// MemLong summary, 2.3.3: softmax attention over sink U retrieved blocks U
// window, one state per q head, log-sum-exp merge of partial states).  The
// decode step launches three kernels back to back -- block scores, top-k,
// this kernel -- the last two as programmatic dependents, so this kernel
// starts while the selection is still running:
//   * one CTA per SM (minus the SMs the top-k kernel holds): warp 0 stages,
//     warps 1..7 compute;
//   * every CTA gets an equal share of the flattened attention list; a
//     head's share mixes sink + window rows (known without the selection)
//     and rows of the selected blocks in proportion, sink/window first;
//   * warp 0 walks the same item sequence as the compute warps and stages
//     each item with bulk asynchronous copies (whole contiguous runs of K/V
//     rows) into a ring of shared-memory stages guarded by full / empty
//     mbarriers; before the first selected row it waits for the top-k
//     kernel to complete (griddepcontrol.wait);
//   * partial softmax states go to per-(head, CTA) slots; the last
//     contributor of a head merges them (no CTA waits for another).
// All mbarrier waits are bounded in time; on expiry the kernel records
// RBA_ERR_TIMEOUT in the status word, skips the remaining work, waits
// (bounded) for its copies in flight and terminates.
#include <cstdio>
#include <cstdlib>

#include "attend_impl.cuh"
#include "decode_fused.cuh"
#include "topk_impl.cuh"

namespace rba {
namespace {

constexpr int kCW = 14;                       // compute warps (warps 1..14)
constexpr int kCT = kCW * 32;                 // compute threads
constexpr int kFT = kCT + 32;                 // + warp 0, which stages

// The compute warps form NGRP groups of RW warps.  With G >= 2 q heads per kv
// head each group holds HS = G / 2 of them for every row of a tile (the tile
// is read by both groups; each lane keeps half the softmax state, so 15 warps
// fit the register file); with G = 1 one group of kCW warps splits the rows.
template <int G>
struct Groups {
  static constexpr int NGRP = G >= 2 ? 2 : 1;
  static constexpr int HS = G / NGRP;        // q heads per warp
  static constexpr int RW = kCW / NGRP;      // warps per group (rows of a tile)
  static_assert(G % NGRP == 0 && kCW % NGRP == 0, "even split");
};
constexpr int kMaxK = 2048;                   // selected blocks per (b, kv head)
constexpr int kMaxStages = 6;
constexpr int kMinRowsPerCta = 128;           // grid shrinks for small problems
constexpr int kMaxGrid = 256;                 // CTAs (one per SM)
constexpr unsigned long long kTimeoutNs = 2000000000ull;

// One partial state (G q heads x (m, l, o[D]) floats), padded to 16 bytes so
// that every slot can be moved by a bulk copy.
__host__ __device__ constexpr int slot_floats(int G, int D) { return (G * (D + 2) + 3) & ~3; }

struct FusedArgs {
  AttendArgs at;            // K, V, q, out, lse, status, cap, T, w0, Hq, Hkv, k, bs, sink,
                            // sink_end, first, nc, scale_log2 (part/tickets/nsplit unused)
  int32_t* idx;             // [BH][k], written by the top-k kernel before this one
  float* slots;             // [BH][m] partial states of slot_floats(G, D), one per part
  uint32_t* tickets;        // [BH], zero between calls
  int BH, L_st, U_sel, NS;
  int m;                    // parts per head (CTAs per head when BH <= CTAs, else 1)
  // part c of a head: attention rows [px[c], px[c+1]), of which sink/window
  // rows [ps[c], ps[c+1]) and selected rows [px[c] - ps[c], px[c+1] - ps[c+1])
  int px[kMaxGrid + 1];
  int ps[kMaxGrid + 1];
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
// Tests the phase; a thread whose phase is not complete is suspended until it
// completes or about 20 us pass (the hint), so waiting warps do not spin.
__device__ __forceinline__ bool mbar_try(uint64_t* b, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(b)), "r"(parity), "r"(20000u)
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

// ---------------------------------------------------------------------------
// work list
//
// The attention rows of head h (Lh = L_st + U_sel) are cut into m equal
// parts, "units" u = h * m + c, c < m; CTA p takes units
// [U * p / P, U * (p + 1) / P) of the U = BH * m units.  With BH <= P, m is
// chosen so that P = BH * m: every CTA holds exactly one part of one head and
// each head has exactly m partial states.  With BH > P, m = 1: every CTA holds
// whole heads and writes their outputs itself.  A part [x0, x1) of a head
// maps to sink/window rows [st(x0), st(x1)) and selected rows
// [x0 - st(x0), x1 - st(x1)) with st(x) = floor(x * L_st / Lh), so a CTA
// streams both kinds of one head with one softmax state, sink/window first.

struct Item {
  int kind;  // 1 sink/window rows, 2 selected rows
  int bh;
  int v0, v1;
};

struct Iter {
  int u, u1;              // current unit, end of this CTA's units
  int bh, part;           // head and part index of unit u
  int kind, v, vend, sel0, sel1;
  bool done;
};

__device__ __forceinline__ void unit_begin(const FusedArgs& a, Iter& it) {
  it.bh = it.u / a.m;
  it.part = it.u - it.bh * a.m;
  const int x0 = a.px[it.part], x1 = a.px[it.part + 1];
  const int s0 = a.ps[it.part], s1 = a.ps[it.part + 1];
  it.kind = 1;
  it.v = s0;
  it.vend = s1;
  it.sel0 = x0 - s0;
  it.sel1 = x1 - s1;
}

__device__ __forceinline__ void iter_begin(const FusedArgs& a, Iter& it) {
  const unsigned U = unsigned(a.BH) * a.m;  // < 2^24 (host-checked): no overflow below
  it.u = static_cast<int>(U * blockIdx.x / gridDim.x);
  it.u1 = static_cast<int>(U * (blockIdx.x + 1) / gridDim.x);
  it.done = it.u >= it.u1;
  if (!it.done) unit_begin(a, it);
}

template <int TT>
__device__ __forceinline__ bool next_item(const FusedArgs& a, Iter& it, Item& out) {
  while (!it.done) {
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
    if (++it.u >= it.u1) {
      it.done = true;
      break;
    }
    unit_begin(a, it);
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
  using C = DecodeTile<T, D, Groups<G>::RW>;
  static constexpr int STAGE = C::STAGE;
  static constexpr int up16(int x) { return (x + 15) & ~15; }
  // regions after the stage ring (NS * STAGE, chosen at launch)
  static constexpr int RED = up16(kCW * G * (D + 2) * 4);       // warp states
  static constexpr int SEL = (kMaxK + 4) * 4 * 2;               // selected prefix + starts
  static constexpr int MISC = 1024;
  static size_t bytes(int NS) { return size_t(NS) * STAGE + RED + SEL + MISC; }
};

// LaneState query slice from a [G][D] fp32 copy in shared memory (the same
// values and lane layout as load_q).
template <typename T, int D, int G>
__device__ __forceinline__ void load_q_smem(const float* qs, float scale_log2,
                                            LaneState<T, D, G>& st) {
  using C = DecodeTile<T, D>;
  const int part = (threadIdx.x & 31) % C::LPR;
  const int rot = lane_rot<T, D>(part);
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float* qr = qs + g * D + part * C::EPL;
#pragma unroll
    for (int j = 0; j < C::CPL; ++j) {
      const int jj = (j + rot) % C::CPL;
#pragma unroll
      for (int e = 0; e < C::EPC; e += 2)
        st.q[g][(j * C::EPC + e) / 2] = make_float2(qr[jj * C::EPC + e] * scale_log2,
                                                    qr[jj * C::EPC + e + 1] * scale_log2);
    }
    st.m[g] = -INFINITY;
    st.l[g] = 0.f;
#pragma unroll
    for (int e = 0; e < C::EPL / 2; ++e) st.o[g][e] = make_float2(0.f, 0.f);
  }
}

// ---------------------------------------------------------------------------
// staging (warp 0)

// Stages one item into `stg`: bulk copies that complete on `bar`, whose
// transaction count is armed with the item's bytes.  Selected rows need the
// selection, which the caller has waited for.
template <typename T, int D, int RW>
__device__ void issue_item(const FusedArgs& a, const Item& item, char* stg, uint64_t* bar,
                           Meta* meta, int* sel_pref, int* sel_phys, int* sel_bh) {
  using C = DecodeTile<T, D, RW>;
  const int lane = threadIdx.x & 31;
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
      // the layout of this head's selected blocks: prefix of their clipped
      // lengths and their first tokens
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
}

// Warp 0: stage every item of this CTA, in order, into the stage ring.
template <typename T, int D, int RW>
__device__ __forceinline__ void produce(const FusedArgs& a, char* stages, uint64_t* full,
                                        uint64_t* empty, Meta* meta, int* sel_pref,
                                        int* sel_phys, volatile int* abort_flag) {
  using C = DecodeTile<T, D, RW>;
  const int NS = a.NS;
  Iter it;
  iter_begin(a, it);
  Item item;
  int j = 0, s = 0, sel_bh = -1;
  uint32_t ph = 0;  // phase parity of the stage's next fill
  bool selection_visible = false;
  while (next_item<C::TT>(a, it, item)) {
    // stage s is free once every compute warp released its previous item
    if (j >= NS && !mbar_wait(&empty[s], ph ^ 1u, abort_flag, a.at.status, 1)) break;
    if (item.kind == 2 && !selection_visible) {
      // the selection comes from the kernel this one depends on: wait for
      // its completion (and its writes) before the first selected row
      asm volatile("griddepcontrol.wait;" ::: "memory");
      selection_visible = true;
    }
    issue_item<T, D, RW>(a, item, stages + size_t(s) * C::STAGE, &full[s], &meta[s], sel_pref,
                     sel_phys, &sel_bh);
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
  constexpr int HS = Groups<G>::HS, RW = Groups<G>::RW;
  constexpr int kSlotFloats = slot_floats(G, D);
  static_assert((kSlotFloats * 4) % 16 == 0, "bulk copies move 16-byte multiples");
  using C = DecodeTile<T, D, RW>;
  using S = FusedSmem<T, D, G>;
  extern __shared__ __align__(128) char smem[];
  const int NS = a.NS;
  char* stages = smem;
  float* red = reinterpret_cast<float*>(smem + size_t(NS) * C::STAGE);
  int* sel_pref = reinterpret_cast<int*>(reinterpret_cast<char*>(red) + S::RED);
  int* sel_phys = sel_pref + (kMaxK + 1);
  char* misc = reinterpret_cast<char*>(sel_pref) + S::SEL;
  uint64_t* full = reinterpret_cast<uint64_t*>(misc);               // [kMaxStages]
  uint64_t* empty = full + kMaxStages;                              // [kMaxStages]
  Meta* meta = reinterpret_cast<Meta*>(empty + kMaxStages);         // [kMaxStages]
  int* s_misc = reinterpret_cast<int*>(meta + kMaxStages);          // [16]
  volatile int* abort_flag = s_misc + 16;                           // [4]
  uint64_t* merge_bar = reinterpret_cast<uint64_t*>(s_misc + 84);   // [1] (s_f is [64] at +20)
  float* s_f = reinterpret_cast<float*>(s_misc + 20);               // [64]

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kCW);
    }
    mbar_init(merge_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();
  if (warp == 0) {
    produce<T, D, RW>(a, stages, full, empty, meta, sel_pref, sel_phys, abort_flag);
    return;
  }
  // ---- compute warps from here on (named barrier 1; no __syncthreads)
  const int cw = warp - 1, tid = ctid();
  const int grp = cw / RW, rw = cw % RW;  // head group, warp within the group
  const int g0 = grp * HS;                // first q head of this warp

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

  // the query heads of this CTA's first head, fp32, while the first tile loads
  Iter it;
  iter_begin(a, it);
  const int bh_att0 = it.done ? -1 : it.bh;
  float* q_first = red;  // [G][D]; red is not used before the first flush
  if (bh_att0 >= 0) {
    const int b = bh_att0 / a.at.Hkv, h = bh_att0 % a.at.Hkv;
    const T* qp = static_cast<const T*>(a.at.q) + (int64_t(b) * a.at.Hq + h * G) * D;
    for (int x = tid; x < G * D; x += kCT) q_first[x] = Elem<T>::to_f32(qp[x]);
  }
  compute_sync();

  Item item;
  bool have = next_item<C::TT>(a, it, item);

  // ---- attention over this CTA's rows, head by head
  LaneState<T, D, HS> st;
  int cur_bh = -1;
  int ord = 0;  // part index of head cur_bh held by this CTA (its slot)
  uint32_t merge_ph = 0;  // phase parity of merge_bar
  float* fac = s_f;         // [G][nw] factors exp2(m_w - M) of the nw warp states
  float* gmax = s_f + 60;   // [G] the max M
  // fac / gmax from nw per-warp states red[w][g][m, l, o[D]]
  auto combine = [&](int nw) {
    if (tid < G * nw) {
      const int gg = tid / nw, w = tid % nw;
      float M = -INFINITY;
      for (int v = 0; v < nw; ++v) M = fmaxf(M, red[(v * G + gg) * (D + 2)]);
      const float mw = red[(w * G + gg) * (D + 2)];
      fac[tid] = mw == -INFINITY ? 0.f : exp2f(mw - M);
      if (w == 0) gmax[gg] = M;
    }
  };
  // output (and lse) of head cur_bh from nw warp states combined by fac
  auto write_out = [&](int nw) {
    const int b = cur_bh / a.at.Hkv, h = cur_bh % a.at.Hkv;
    for (int x = tid; x < G * D; x += kCT) {
      const int gg = x / D, d = x % D;
      float num = 0.f, den = 0.f;
      for (int w = 0; w < nw; ++w) {
        const float f = fac[gg * nw + w];
        num += red[(w * G + gg) * (D + 2) + 2 + d] * f;
        den += red[(w * G + gg) * (D + 2) + 1] * f;
      }
      a.at.out[(int64_t(b) * a.at.Hq + h * G + gg) * D + d] = den > 0.f ? num / den : 0.f;
      if (d == 0 && a.at.lse != nullptr)
        a.at.lse[int64_t(b) * a.at.Hq + h * G + gg] =
            den > 0.f ? (gmax[gg] + log2f(den)) * 0.6931471805599453f : -INFINITY;
    }
  };
  while (true) {
    const bool more = have;
    if (cur_bh >= 0 && (!more || item.bh != cur_bh)) {
      // ---- this CTA's state of head cur_bh: warp states -> red[rw][g]
      merge_slots<T, D, HS>(st);
      const int slot_lane = lane / C::LPR, part = lane % C::LPR;
      const int rot = lane_rot<T, D>(part);
      if (slot_lane == 0) {
#pragma unroll
        for (int gg = 0; gg < HS; ++gg) {
          float* r = red + (rw * G + g0 + gg) * (D + 2);
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
      combine(RW);
      compute_sync();
      if (a.m == 1) {
        write_out(RW);  // this CTA holds the whole head
      } else {
        // this CTA's state -> slot `ord` of the head; the last of the head's
        // m parts to finish merges all m slots
        const bool slot_ok = ord >= 0 && ord < a.m;
        if (!slot_ok && tid == 0) report(a.at.status, RBA_ERR_BOUNDS, kWhereFused, 4);
        float* base = a.slots + int64_t(cur_bh) * a.m * kSlotFloats;
        float* slot = base + int64_t(slot_ok ? ord : 0) * kSlotFloats;
#pragma unroll 1
        for (int x = tid; x < G * (D + 2) && slot_ok; x += kCT) {
          const int gg = x / (D + 2), c = x % (D + 2);
          float acc = 0.f;
          if (c == 0) {
            acc = gmax[gg];
          } else {
#pragma unroll
            for (int w = 0; w < RW; ++w)
              acc += red[(w * G + gg) * (D + 2) + c] * fac[gg * RW + w];
          }
          slot[x] = acc;
        }
        compute_sync();
        if (tid == 0) {
          const uint32_t t = atom_add_acq_rel(a.tickets + cur_bh, 1u);  // publishes our slot
          s_misc[9] = t == uint32_t(a.m - 1);
        }
        compute_sync();
        if (s_misc[9]) {
          // the last part of the head merges the m slots.  The slots go to
          // shared memory by bulk copies into the stage ring (idle: with
          // m > 1 a CTA holds one part of one head, all of it consumed), a
          // chunk at a time; each thread then folds every slot's (m, l, o[d])
          // of its output elements (g, d) into a running (max, sum, output).
          constexpr int SLOT = kSlotFloats * 4;  // a multiple of 16 bytes
          const int nl = a.m;
          const int chunk = (NS * C::STAGE) / SLOT;
          const int b = cur_bh / a.at.Hkv, h = cur_bh % a.at.Hkv;
          float M[2], L[2], O[2];  // elements x = tid and tid + kCT
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            M[r] = -INFINITY;
            L[r] = 0.f;
            O[r] = 0.f;
          }
          for (int j0 = 0; j0 < nl; j0 += chunk) {
            const int n = min(chunk, nl - j0);
            if (tid == 0) {
              // (the compute warps' reads of the ring are ordered before the copies)
              asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
              mbar_arrive_tx(merge_bar, uint32_t(n) * SLOT);
              for (int j = 0; j < n; ++j)
                bulk_g2s(stages + size_t(j) * SLOT, base + int64_t(j0 + j) * kSlotFloats, SLOT,
                         merge_bar);
            }
            const bool ok = mbar_wait(merge_bar, merge_ph, abort_flag, a.at.status, 6);
            if (!ok && tid == 0) mbar_drain(merge_bar, merge_ph);  // no copy outlives the CTA
            merge_ph ^= 1u;
            const float* sm = reinterpret_cast<const float*>(stages);
#pragma unroll
            for (int r = 0; r < 2; ++r) {
              const int x = tid + r * kCT;
              if (!ok || x >= G * D) continue;
              const int gg = x / D, d = x % D;
              for (int j = 0; j < n; ++j) {
                const float* q = sm + j * kSlotFloats + gg * (D + 2);
                const float mj = q[0], lj = q[1], oj = q[2 + d];
                const float mn = fmaxf(M[r], mj);
                const float sa = M[r] == -INFINITY ? 0.f : exp2f(M[r] - mn);
                const float sb = mj == -INFINITY ? 0.f : exp2f(mj - mn);
                L[r] = L[r] * sa + lj * sb;
                O[r] = O[r] * sa + oj * sb;
                M[r] = mn;
              }
            }
            compute_sync();  // the chunk buffer is read before the next copy
          }
#pragma unroll
          for (int r = 0; r < 2; ++r) {
            const int x = tid + r * kCT;
            if (x >= G * D) continue;
            const int gg = x / D, d = x % D;
            a.at.out[(int64_t(b) * a.at.Hq + h * G + gg) * D + d] = L[r] > 0.f ? O[r] / L[r] : 0.f;
            if (d == 0 && a.at.lse != nullptr)
              a.at.lse[int64_t(b) * a.at.Hq + h * G + gg] =
                  L[r] > 0.f ? (M[r] + log2f(L[r])) * 0.6931471805599453f : -INFINITY;
          }
          if (tid == 0) a.tickets[cur_bh] = 0;  // zero again for the next call
        }
      }
      compute_sync();
      cur_bh = -1;
    }
    if (!more) break;
    if (item.bh != cur_bh) {
      cur_bh = item.bh;
      if (cur_bh == bh_att0)
        load_q_smem<T, D, HS>(q_first + g0 * D, a.at.scale_log2, st);
      else
        load_q<T, D, HS>(a.at, cur_bh, st, g0);
      ord = it.part;
    }
    if (wait_full()) {
      consume_tile<T, D, HS, RW>(stages + size_t(s) * C::STAGE, meta[s].nrows, st, rw);
      release();
    }
    advance();
    have = next_item<C::TT>(a, it, item);
  }
}

constexpr size_t kMaxSmem = 227 * 1024;  // dynamic shared memory of one CTA

template <typename T, int D, int G>
int fused_stages() {
  using S = FusedSmem<T, D, G>;
  int NS = kMaxStages;
  while (NS > 2 && S::bytes(NS) > kMaxSmem) --NS;
  return NS;
}

// CTAs of this kernel that fit on one SM (0: none; <0: a CUDA error)
template <typename T, int D, int G>
int fused_occupancy_t() {
  using S = FusedSmem<T, D, G>;
  const size_t smem = S::bytes(fused_stages<T, D, G>());
  if (smem > kMaxSmem) return 0;  // (large fp32 tiles) the split-K kernel runs instead
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
rba_status launch_fused_t(FusedArgs a, int P, bool pdl, cudaStream_t stream) {
  using S = FusedSmem<T, D, G>;
  const int NS = fused_stages<T, D, G>();
  a.NS = NS;
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
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  RBA_CUDA_TRY(cudaLaunchKernelEx(&cfg, kfn, a));
  return RBA_OK;
}

}  // namespace

static int64_t attention_rows(const rba_store* st, const Geometry& g, int k) {
  const int64_t BH = int64_t(st->d.batch) * st->d.n_kv_heads;
  return BH * (int64_t(g.sink_end) + (g.T - g.w0) + (k > 0 ? int64_t(k) * st->d.block_size : 0));
}

// CTAs available to the attention launch: one per SM, leaving the SMs that
// the top-k kernel (one CTA per row) holds while this kernel starts; fewer
// for small problems.
static int cta_budget(const rba_store* st, const Geometry& g, int k) {
  const int BH = st->d.batch * st->d.n_kv_heads;
  int sms = num_sms();
  if (k > 0 && g.nc <= kSmallN && BH <= sms / 4) sms -= BH;
  int64_t P = (attention_rows(st, g, k) + kMinRowsPerCta - 1) / kMinRowsPerCta;
  if (P > sms) P = sms;
  if (P > kMaxGrid) P = kMaxGrid;
  return static_cast<int>(P < 1 ? 1 : P);
}

// Parts per head (m) and CTAs (P): with BH <= budget, m = budget / BH and
// P = BH * m (each CTA one part of one head); else m = 1 and P = budget
// (each CTA whole heads).
static void partition(const rba_store* st, const Geometry& g, int k, int* m, int* P) {
  const int BH = st->d.batch * st->d.n_kv_heads;
  const int budget = cta_budget(st, g, k);
  if (BH <= budget) {
    *m = budget / BH;
    *P = BH * *m;
  } else {
    *m = 1;
    *P = budget;
  }
}

int fused_grid(const rba_store* st, const Geometry& g, int k) {
  int m, P;
  partition(st, g, k, &m, &P);
  return P;
}

size_t fused_slot_bytes(const rba_store* st, const Geometry& g, int k, int* ms) {
  const rba_store_desc& d = st->d;
  const int BH = d.batch * d.n_kv_heads;
  const int G = d.n_q_heads / d.n_kv_heads;
  int m, P;
  partition(st, g, k, &m, &P);
  if (ms) *ms = m;
  return m > 1 ? align_up(size_t(BH) * m * slot_floats(G, d.head_dim) * 4, 256) : 0;
}

size_t fused_sync_bytes(const rba_store* st) {
  return align_up(size_t(st->d.batch) * st->d.n_kv_heads * 4, 256);
}

// Whether the persistent attention kernel covers this problem (else the
// split-K kernel runs).
bool fused_eligible(const rba_store* st, const Geometry& g, int k) {
  const rba_store_desc& d = st->d;
  const int G = d.n_q_heads / d.n_kv_heads;
  if (d.mode == RBA_REP_EMBED_COSINE) return false;
  if (G != 1 && G != 2 && G != 4) return false;
  if (k > kMaxK) return false;
  if (attention_rows(st, g, k) == 0) return false;
  const int64_t BH = int64_t(d.batch) * d.n_kv_heads;
  if (BH >= (int64_t(1) << 24)) return false;
  if (attention_rows(st, g, k) / BH >= (int64_t(1) << 31)) return false;
  int ms = 0;
  fused_slot_bytes(st, g, k, &ms);
  return ms <= kMaxGrid;
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
                        const int32_t* idx, float* out, float* lse, void* sync, float* slots,
                        bool pdl, cudaStream_t stream) {
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
  a.idx = const_cast<int32_t*>(idx);
  a.tickets = static_cast<uint32_t*>(sync);
  a.slots = slots;
  a.BH = BH;
  a.L_st = static_cast<int>(g.sink_end + (g.T - g.w0));
  a.U_sel = k > 0 ? k * d.block_size : 0;
  fused_slot_bytes(st, g, k, &a.m);
  // part boundaries (host side: no 64-bit divisions on the device)
  const int64_t Lh = int64_t(a.L_st) + a.U_sel;
  for (int c = 0; c <= a.m; ++c) {
    const int64_t x = Lh * c / a.m;
    a.px[c] = static_cast<int>(x);
    a.ps[c] = static_cast<int>(x * a.L_st / Lh);
  }
  const int G = d.n_q_heads / d.n_kv_heads;
#define RBA_FUSED(T_, D_)                                               \
  switch (G) {                                                          \
    case 1: return launch_fused_t<T_, D_, 1>(a, P, pdl, stream);        \
    case 2: return launch_fused_t<T_, D_, 2>(a, P, pdl, stream);        \
    case 4: return launch_fused_t<T_, D_, 4>(a, P, pdl, stream);        \
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
