// Decode attention of one step in one persistent launch, overlapped with the
// selection that precedes it on the stream.
//
// Same definitions as rba_attend (InfLLM article, "overall framework";
// MemLong summary, 2.3.3: softmax attention over sink U retrieved blocks U
// window, one state per q head, log-sum-exp merge of partial states).  The
// decode step launches three kernels back to back -- block scores, top-k,
// this kernel -- the last two as programmatic dependents, so this kernel
// starts while the selection is still running.  Two kernels share the work
// list, the staging scheme and the end-of-head merge:
//   * decode_mma_kernel (bf16 stores whose blocks are whole 64-row tiles):
//     the staging warp loads single-segment pieces of up to 64 rows as
//     swizzled 2-D tensor boxes; eight compute warps run the inner products
//     on the tensor cores (mma.sync), two pieces at a time;
//   * decode_fused_kernel (other block sizes, fp32): the staging warp copies
//     whole contiguous runs of K/V rows into 56-row tiles; fourteen compute
//     warps run the online softmax on the CUDA cores.
// In both, one CTA runs per SM (minus the SMs the top-k kernel holds); every
// CTA gets an equal share of the flattened attention list, and a head's share
// mixes sink + window rows (known without the selection) and rows of the
// selected blocks in proportion, sink/window first.  The staging warp fills a
// ring of shared-memory stages guarded by full / empty mbarriers and waits
// for the top-k kernel (griddepcontrol.wait) only before the first selected
// row.  Partial softmax states go to per-(head, CTA) slots; the last
// contributor of a head merges them (no CTA waits for another).
// All mbarrier waits are bounded in time; on expiry the kernel records
// RBA_ERR_TIMEOUT in the status word, skips the remaining work, waits
// (bounded) for its copies in flight and terminates.
#include <cstdio>
#include <cstdlib>

#include "attend_impl.cuh"
#include "decode_fused.cuh"
#include "decode_persist.cuh"
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
// shared-memory table: prefix [kMaxK + 1], starts [kMaxK], sink/window [5]
static_assert((kMaxK + 1) + kMaxK + 5 <= 2 * (kMaxK + 4), "selection table room");
constexpr int kMinRowsPerCta = 128;           // grid shrinks for small problems
constexpr int kMaxGrid = 256;                 // CTAs (one per SM)

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

// Stage geometry: a stage holds TT rows of K then TT rows of V; rows are ROWB
// bytes long and RSTR bytes apart.  RSTR == ROWB: a contiguous run of rows is
// one bulk copy; RSTR > ROWB (padded rows): one bulk copy per row.
template <int TT_, int ROWB_, int RSTR_>
struct StageGeo {
  static constexpr int TT = TT_, ROWB = ROWB_, RSTR = RSTR_;
  static constexpr int VOFF = TT * RSTR;
  static constexpr int STAGE = 2 * TT * RSTR;
  static_assert(RSTR % 16 == 0 && ROWB % 16 == 0, "bulk copies move 16-byte multiples");
};


template <typename T, int D, int G>
struct FusedSmem {
  using C = DecodeTile<T, D, Groups<G>::RW>;
  static constexpr int STAGE = C::STAGE;
  static constexpr int up16(int x) { return (x + 15) & ~15; }
  // regions after the stage ring (NS * STAGE, chosen at launch)
  static constexpr int RED = up16(kCW * G * (D + 2) * 4);       // warp states
  static constexpr int SEL = (kMaxK + 4) * 4 * 2;  // selected prefix + starts, sink/window table
  static constexpr int MISC = kMiscBytes;
  static size_t bytes(int NS) { return size_t(NS) * STAGE + RED + SEL + MISC; }
};

// ---------------------------------------------------------------------------
// end of a head: NW per-warp states -> output, or -> a partial slot and the
// last part's merge

// red[w][g] = (m, l, o[D]) of warp w (log2 units, o unnormalised).  Combines
// the NW states of head bh held by this CTA; with m == 1 writes out and lse,
// else publishes the state to slot `ord` of the head and, if this CTA is the
// head's last part to finish (acq_rel ticket), merges the head's m slots,
// which arrive by bulk copies into the (idle) stage ring.  Called by all NCT
// compute threads; ends with them synchronised.
template <int G, int D, int NW, int NCT>
__device__ __forceinline__ void finish_head(const FusedArgs& a, int bh, int ord, float* red,
                            const MiscLayout& ms, char* stages, size_t ring_bytes,
                            uint32_t& merge_ph) {
  constexpr int kSlotFloats = slot_floats(G, D);
  static_assert(G * NW <= 112 && G <= 16, "merge factors fit the misc floats");
  const int tid = ctid();
  float* fac = ms.s_f;          // [G][NW] factors exp2(m_w - M) of the NW warp states
  float* gmax = ms.s_f + 112;   // [G] the max M
  compute_sync<NCT>();
  if (tid < G * NW) {
    const int gg = tid / NW, w = tid % NW;
    float M = -INFINITY;
    for (int v = 0; v < NW; ++v) M = fmaxf(M, red[(v * G + gg) * (D + 2)]);
    const float mw = red[(w * G + gg) * (D + 2)];
    fac[tid] = mw == -INFINITY ? 0.f : exp2f(mw - M);
    if (w == 0) gmax[gg] = M;
  }
  compute_sync<NCT>();
  const int b = bh / a.at.Hkv, h = bh % a.at.Hkv;
  if (a.m == 1) {
    // this CTA holds the whole head
    for (int x = tid; x < G * D; x += NCT) {
      const int gg = x / D, d = x % D;
      if (d >= a.at.qd) continue;  // padding columns of the pools
      float num = 0.f, den = 0.f;
      for (int w = 0; w < NW; ++w) {
        const float f = fac[gg * NW + w];
        num += red[(w * G + gg) * (D + 2) + 2 + d] * f;
        den += red[(w * G + gg) * (D + 2) + 1] * f;
      }
      a.at.out[(int64_t(b) * a.at.Hq + h * G + gg) * a.at.qd + d] = den > 0.f ? num / den : 0.f;
      if (d == 0 && a.at.lse != nullptr)
        a.at.lse[int64_t(b) * a.at.Hq + h * G + gg] =
            den > 0.f ? (gmax[gg] + log2f(den)) * 0.6931471805599453f : -INFINITY;
    }
  } else {
    // this CTA's state -> slot `ord` of the head; the last of the head's m
    // parts to finish merges all m slots
    const bool slot_ok = ord >= 0 && ord < a.m;
    if (!slot_ok && tid == 0) report(a.at.status, RBA_ERR_BOUNDS, kWhereFused, 4);
    float* base = a.slots + int64_t(bh) * a.m * kSlotFloats;
    float* slot = base + int64_t(slot_ok ? ord : 0) * kSlotFloats;
#pragma unroll 1
    for (int x = tid; x < G * (D + 2) && slot_ok; x += NCT) {
      const int gg = x / (D + 2), c = x % (D + 2);
      float acc = 0.f;
      if (c == 0) {
        acc = gmax[gg];
      } else {
#pragma unroll
        for (int w = 0; w < NW; ++w) acc += red[(w * G + gg) * (D + 2) + c] * fac[gg * NW + w];
      }
      slot[x] = acc;
    }
    compute_sync<NCT>();
    if (tid == 0) {
      const uint32_t t = atom_add_acq_rel(a.tickets + bh, 1u);  // publishes our slot
      ms.s_misc[9] = t == uint32_t(a.m - 1);
    }
    compute_sync<NCT>();
    if (ms.s_misc[9]) {
      // the last part of the head merges the m slots.  The slots go to shared
      // memory by bulk copies into the stage ring (idle: with m > 1 a CTA
      // holds one part of one head, all of it consumed), a chunk at a time.
      // Per chunk, warp g < G folds the slots' (m, l) of q head g into a
      // running max and denominator and leaves one factor per slot in `fac`
      // (red is free by now); then each thread folds its output elements
      // (g, d) with those factors.
      constexpr int SLOT = kSlotFloats * 4;  // a multiple of 16 bytes
      constexpr int NX = (G * D + NCT - 1) / NCT;
      const int nl = a.m;
      const int chunk = min(static_cast<int>(ring_bytes / SLOT), (NW * (D + 2)) / 2);
      float* mfac = const_cast<float*>(red);      // [chunk][G] factors
      float* mrun = ms.s_f;                       // [G] running max (replaces fac / gmax)
      float* lrun = ms.s_f + 16;                  // [G] running denominator
      float* rsc = ms.s_f + 32;                   // [G] rescale of the running sums
      const int lane = tid & 31, cw = tid >> 5;
      float O[NX];
#pragma unroll
      for (int r = 0; r < NX; ++r) O[r] = 0.f;
      for (int j0 = 0; j0 < nl; j0 += chunk) {
        const int n = min(chunk, nl - j0);
        if (tid == 0) {
          // (the compute warps' reads of the ring are ordered before the copies)
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
          mbar_arrive_tx(ms.merge_bar, uint32_t(n) * SLOT);
          for (int j = 0; j < n; ++j)
            bulk_g2s(stages + size_t(j) * SLOT, base + int64_t(j0 + j) * kSlotFloats, SLOT,
                     ms.merge_bar);
        }
        const bool ok = mbar_wait(ms.merge_bar, merge_ph, ms.abort_flag, a.at.status, 6);
        if (!ok && tid == 0) mbar_drain(ms.merge_bar, merge_ph);  // no copy outlives the CTA
        merge_ph ^= 1u;
        const float* sm = reinterpret_cast<const float*>(stages);
        if (cw < G) {
          const int g = cw;
          float cm = -INFINITY;
          for (int j = lane; j < n; j += 32) cm = fmaxf(cm, sm[j * kSlotFloats + g * (D + 2)]);
          for (int o = 16; o > 0; o >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, o));
          const float mo = j0 == 0 ? -INFINITY : mrun[g];  // (warp g alone writes mrun[g])
          const float lo = j0 == 0 ? 0.f : lrun[g];
          const float mn = fmaxf(mo, cm);
          float lsum = 0.f;
          for (int j = lane; j < n; j += 32) {
            const float mj = sm[j * kSlotFloats + g * (D + 2)];
            const float f = mj == -INFINITY ? 0.f : exp2f(mj - mn);
            mfac[j * G + g] = f;
            lsum += f * sm[j * kSlotFloats + g * (D + 2) + 1];
          }
          for (int o = 16; o > 0; o >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, o);
          if (lane == 0) {
            const float sc = mo == -INFINITY ? 0.f : exp2f(mo - mn);
            rsc[g] = sc;
            lrun[g] = lo * sc + lsum;
            mrun[g] = mn;
          }
        }
        compute_sync<NCT>();
#pragma unroll
        for (int r = 0; r < NX; ++r) {
          const int x = tid + r * NCT;
          if (!ok || x >= G * D) continue;
          const int gg = x / D, d = x % D;
          float acc = O[r] * rsc[gg];
          for (int j = 0; j < n; ++j) acc += mfac[j * G + gg] * sm[j * kSlotFloats + gg * (D + 2) + 2 + d];
          O[r] = acc;
        }
        compute_sync<NCT>();  // the chunk buffer and factors are read before the next copy
      }
#pragma unroll
      for (int r = 0; r < NX; ++r) {
        const int x = tid + r * NCT;
        if (x >= G * D) continue;
        const int gg = x / D, d = x % D;
        const float L = lrun[gg];
        if (d < a.at.qd)
          a.at.out[(int64_t(b) * a.at.Hq + h * G + gg) * a.at.qd + d] = L > 0.f ? O[r] / L : 0.f;
        if (d == 0 && a.at.lse != nullptr)
          a.at.lse[int64_t(b) * a.at.Hq + h * G + gg] =
              L > 0.f ? (mrun[gg] + log2f(L)) * 0.6931471805599453f : -INFINITY;
      }
      if (tid == 0) a.tickets[bh] = 0;  // zero again for the next call
    }
  }
  compute_sync<NCT>();
}

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
template <class Geo>
__device__ void issue_item(const FusedArgs& a, const Item& item, char* stg, uint64_t* bar,
                           Meta* meta, int* sel_pref, int* sel_phys, int* sel_bh) {
  const int lane = threadIdx.x & 31;
  const int* pref;
  const int* phys;
  int nseg;
  if (item.kind == 1) {
    pref = sel_phys + kMaxK;  // the sink/window table (written by produce)
    phys = pref + 3;
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
    mbar_arrive_tx(bar, uint32_t(nrows) * Geo::ROWB * 2);
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
    if constexpr (Geo::RSTR == Geo::ROWB) {
      // one copy per contiguous run (a lane per segment)
      for (int sg = lo + lane; sg < nseg && pref[sg] < v1; sg += 32) {
        const int a0 = max(v0, pref[sg]), a1 = min(v1, pref[sg + 1]);
        if (a1 <= a0) continue;
        const int64_t tok = int64_t(item.bh) * a.at.cap + phys[sg] + (a0 - pref[sg]);
        const uint32_t bytes = uint32_t(a1 - a0) * Geo::ROWB;
        const int row = a0 - v0;
        bulk_g2s(stg + row * Geo::RSTR, Kb + tok * Geo::ROWB, bytes, bar);
        bulk_g2s(stg + Geo::VOFF + row * Geo::RSTR, Vb + tok * Geo::ROWB, bytes, bar);
      }
    } else {
      // padded rows: one copy per row (a lane per row); the row's segment is
      // the last one starting at or before it
      for (int row = lane; row < nrows; row += 32) {
        const int v = v0 + row;
        int l2 = lo, h2 = nseg - 1;
        while (l2 < h2) {
          const int mid = (l2 + h2 + 1) >> 1;
          if (pref[mid] <= v) l2 = mid; else h2 = mid - 1;
        }
        const int64_t tok = int64_t(item.bh) * a.at.cap + phys[l2] + (v - pref[l2]);
        bulk_g2s(stg + row * Geo::RSTR, Kb + tok * Geo::ROWB, Geo::ROWB, bar);
        bulk_g2s(stg + Geo::VOFF + row * Geo::RSTR, Vb + tok * Geo::ROWB, Geo::ROWB, bar);
      }
    }
  }
  __syncwarp();
}

// Warp 0: stage every item of this CTA, in order, into the stage ring.
template <class Geo>
__device__ __forceinline__ void produce(const FusedArgs& a, char* stages, uint64_t* full,
                                        uint64_t* empty, Meta* meta, int* sel_pref,
                                        int* sel_phys, volatile int* abort_flag) {
  // the sink/window segments (prefix 0, sink_end, L_st; first rows 0, w0),
  // in shared memory after the selection's table: a small array indexed at
  // run time would live in local memory, and every access would wait on an
  // L2 kept busy by the copies
  if ((threadIdx.x & 31) == 0) {
    int* st_tab = sel_phys + kMaxK;
    st_tab[0] = 0;
    st_tab[1] = a.at.sink_end;
    st_tab[2] = a.L_st;
    st_tab[3] = 0;
    st_tab[4] = static_cast<int>(a.at.w0);
  }
  __syncwarp();
  const int NS = a.NS;
  Iter it;
  iter_begin(a, it);
  Item item;
  int j = 0, s = 0, sel_bh = -1;
  uint32_t ph = 0;  // phase parity of the stage's next fill
  bool selection_visible = false;
  while (next_item<Geo::TT>(a, it, item)) {
    // stage s is free once every compute warp released its previous item
    if (j >= NS && !mbar_wait(&empty[s], ph ^ 1u, abort_flag, a.at.status, 1)) break;
    if (item.kind == 2 && !selection_visible) {
      // the selection comes from the kernel this one depends on: wait for
      // its completion (and its writes) before the first selected row
      asm volatile("griddepcontrol.wait;" ::: "memory");
      selection_visible = true;
    }
    issue_item<Geo>(a, item, stages + size_t(s) * Geo::STAGE, &full[s], &meta[s], sel_pref,
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
  const MiscLayout ms(misc);
  uint64_t* full = ms.full;
  uint64_t* empty = ms.empty;
  Meta* meta = ms.meta;
  volatile int* abort_flag = ms.abort_flag;
  uint64_t* merge_bar = ms.merge_bar;

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
    produce<StageGeo<C::TT, C::ROWB, C::ROWB>>(a, stages, full, empty, meta, sel_pref, sel_phys,
                                               abort_flag);
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
    const T* qp = static_cast<const T*>(a.at.q) + (int64_t(b) * a.at.Hq + h * G) * a.at.qd;
    for (int x = tid; x < G * D; x += kCT) {
      const int gg = x / D, d = x % D;  // (columns past qd count as zero)
      q_first[x] = d < a.at.qd ? Elem<T>::to_f32(qp[gg * a.at.qd + d]) : 0.f;
    }
  }
  compute_sync<kCT>();

  Item item;
  bool have = next_item<C::TT>(a, it, item);

  // ---- attention over this CTA's rows, head by head
  LaneState<T, D, HS> st;
  int cur_bh = -1;
  int ord = 0;  // part index of head cur_bh held by this CTA (its slot)
  uint32_t merge_ph = 0;  // phase parity of merge_bar
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
      finish_head<G, D, RW, kCT>(a, cur_bh, ord, red, ms, stages, size_t(NS) * C::STAGE,
                                 merge_ph);
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

// ---------------------------------------------------------------------------
// bf16 with whole-block tiles: the inner products on the tensor cores
//
// Used when every retrieved block is a whole number of 64-row tiles.  The
// staging warp cuts the CTA's rows into pieces that never cross a segment
// (sink, window, one selected block) and are at most 64 rows long, and loads
// each piece as 64-row boxes of K and V (two 64-column halves each) with 2-D
// bulk tensor copies in the 128-byte swizzled layout; rows of a box past the
// piece are ignored.  It records each piece's head, part and row count in the
// stage's meta word, which drives the compute warps.
//
// Per warp and 16-row slice of a tile (mma.sync m16n8k16, bf16 in, fp32
// accumulate), with the q heads of the kv head padded to M = 16:
//   S^T[16][16 rows]  = Q[16][D] . K^T           (D/16 k-steps, 2 n-tiles of 8 rows)
//   online softmax per head over the rows (a lane holds 4 rows of head lane/4)
//   O[16][D]         += P^T[16][16 rows] . V     (D/8 n-tiles, one k-step)
// P^T comes straight from the S^T accumulators (the C layout of two 8-row
// n-tiles is the A layout of one 16-row k-step).  P is split as p = hi + lo,
// both bf16, and multiplied twice, so the weights keep ~16 mantissa bits.
// K and V fragments come from shared memory by ldmatrix (V transposed); the
// swizzle puts the eight rows of a matrix in distinct banks.

template <int D, int G>
struct MmaSmem {
  using Geo = MmaGeo<D>;
  static constexpr int up16(int x) { return (x + 15) & ~15; }
  static constexpr int RED = up16(kMW * G * (D + 2) * 4);       // warp states
  static constexpr int QF = kMW * (D / 16) * 32 * 8;            // per-warp Q fragments
  static constexpr int SEL = (kMaxK + 4) * 4 * 2;  // selected prefix + starts, sink/window table
  static constexpr int MISC = kMiscBytes;
  static constexpr int ALIGN = 1024;                            // ring base alignment slack
  static size_t bytes(int NS) {
    return size_t(NS) * Geo::STAGE + RED + QF + SEL + MISC + ALIGN;
  }
};

// Warp 0 of the whole-block kernel: cuts this CTA's rows into pieces (one
// segment, <= 64 rows) and stages each into the ring with bulk tensor copies.
// The last piece of each unit (head part) carries the flush flag; a unit
// without rows still gets one empty piece.
template <int D>
__device__ __forceinline__ void produce_pieces(const FusedArgs& a, const CUtensorMap* kmap,
                                               const CUtensorMap* vmap, char* stages,
                                               const MiscLayout& ms, int* sel_pref,
                                               int* sel_phys) {
  using Geo = MmaGeo<D>;
  const int lane = threadIdx.x & 31;
  // the sink/window segments (prefix 0, sink_end, L_st; first rows 0, w0),
  // in shared memory after the selection's table: a small array indexed at
  // run time would live in local memory, and every access would wait on an
  // L2 kept busy by the copies
  if ((threadIdx.x & 31) == 0) {
    int* st_tab = sel_phys + kMaxK;
    st_tab[0] = 0;
    st_tab[1] = a.at.sink_end;
    st_tab[2] = a.L_st;
    st_tab[3] = 0;
    st_tab[4] = static_cast<int>(a.at.w0);
  }
  __syncwarp();
  const int NS = a.NS;
  int j = 0, s = 0, sel_bh = -1;
  uint32_t ph = 0;
  bool selection_visible = false;
  // stages one piece of n rows starting at pool row y (n = 0: no copies)
  auto emit = [&](int n, int y, int bh, int part, bool flush) -> bool {
    // stage s is free once all compute warps released its previous piece
    if (j >= NS && !mbar_wait(&ms.empty[s], ph ^ 1u, ms.abort_flag, a.at.status, 1))
      return false;
    if (lane == 0) {
      Meta& mt = ms.meta[s];
      mt.nrows = n;
      mt.pad[0] = bh;
      mt.pad[1] = part;
      mt.pad[2] = flush ? kPieceFlush : 0;
      mbar_arrive_tx(&ms.full[s], n > 0 ? uint32_t(Geo::TX) : 0u);
      if (n > 0) {
        char* stg = stages + size_t(s) * Geo::STAGE;
#pragma unroll
        for (int hh = 0; hh < Geo::NH; ++hh) {
          tma_load_2d(stg + hh * kHalfBytes, kmap, hh * 64, y, &ms.full[s]);
          tma_load_2d(stg + Geo::VOFF + hh * kHalfBytes, vmap, hh * 64, y, &ms.full[s]);
        }
      }
    }
    __syncwarp();
    ++j;
    if (++s == NS) {
      s = 0;
      ph ^= 1u;
    }
    return true;
  };
  Iter it;
  iter_begin(a, it);
  bool alive = true;
  while (!it.done && alive) {
    const int bh = it.bh, part = it.part;
    const int s0 = a.ps[part], s1 = a.ps[part + 1];
    const int sel0 = a.px[part] - s0, sel1 = a.px[part + 1] - s1;
    bool pend = false;
    int pn = 0, py = 0;
    for (int kind = 1; kind <= 2 && alive; ++kind) {
      int v = kind == 1 ? s0 : sel0;
      const int vend = kind == 1 ? s1 : sel1;
      if (v >= vend) continue;
      const int* pref;
      const int* phys;
      int nseg;
      if (kind == 1) {
        pref = sel_phys + kMaxK;  // the sink/window table
        phys = pref + 3;
        nseg = 2;
      } else {
        if (!selection_visible) {
          // the selection comes from the kernel this one depends on: wait for
          // its completion (and its writes) before the first selected row
          asm volatile("griddepcontrol.wait;" ::: "memory");
          selection_visible = true;
        }
        if (bh != sel_bh) {
          // prefix of the clipped lengths of this head's selected blocks, and
          // their first tokens
          const int k = a.at.k;
          int run = 0;
          for (int base = 0; base < k; base += 32) {
            const int jj = base + lane;
            int len = 0, start = 0;
            if (jj < k) {
              const int blk = __ldcg(a.idx + int64_t(bh) * k + jj);
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
            if (jj < k) {
              sel_pref[jj] = run + incl - len;
              sel_phys[jj] = start;
            }
            run += __shfl_sync(0xffffffffu, incl, 31);
          }
          if (lane == 0) sel_pref[k] = run;
          __syncwarp();
          sel_bh = bh;
        }
        pref = sel_pref;
        phys = sel_phys;
        nseg = a.at.k;
      }
      const int vlim = min(vend, pref[nseg]);
      while (v < vlim) {
        // the segment holding v: the last one starting at or before it
        int lo2 = 0, hi2 = nseg - 1;
        while (lo2 < hi2) {
          const int mid = (lo2 + hi2 + 1) >> 1;
          if (pref[mid] <= v) lo2 = mid; else hi2 = mid - 1;
        }
        const int n = min(min(vlim, pref[lo2 + 1]), v + kMTT) - v;
        const int y = static_cast<int>(int64_t(bh) * a.at.cap + phys[lo2] + (v - pref[lo2]));
        if (pend && !emit(pn, py, bh, part, false)) {
          alive = false;
          break;
        }
        pend = true;
        pn = n;
        py = y;
        v += n;
      }
    }
    if (alive && !emit(pend ? pn : 0, py, bh, part, true)) alive = false;
    if (++it.u >= it.u1) it.done = true; else unit_begin(a, it);
  }
  // no copy may still be landing in shared memory when the CTA exits
  if (lane == 0)
    for (int q = max(0, j - NS); q < j; ++q) mbar_drain(&ms.full[q % NS], (q / NS) & 1u);
  __syncwarp();
}

template <int D, int G>
__global__ void __launch_bounds__(kMFT, 1)
    decode_mma_kernel(const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap vmap, FusedArgs a) {
  static_assert(G <= 8, "q heads of a kv head fit the rows 0..7 of the A tile");
  using Geo = MmaGeo<D>;
  using S = MmaSmem<D, G>;
  extern __shared__ char smem_raw[];
  // 1024-byte aligned base, offset from the shared array itself (an integer
  // round trip would hide from the compiler that the pointers address shared
  // memory and turn every access into a generic one)
  char* stages = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int NS = a.NS;
  float* red = reinterpret_cast<float*>(stages + size_t(NS) * Geo::STAGE);
  uint2* qfrag = reinterpret_cast<uint2*>(reinterpret_cast<char*>(red) + S::RED);
  int* sel_pref = reinterpret_cast<int*>(reinterpret_cast<char*>(qfrag) + S::QF);
  int* sel_phys = sel_pref + (kMaxK + 1);
  const MiscLayout ms(reinterpret_cast<char*>(sel_pref) + S::SEL);

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (warp == 0) {
    // the staging warp sets up the barriers, releases the compute warps
    // (named barrier 2, which it does not wait on) and starts copying
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&kmap))
                   : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&vmap))
                   : "memory");
      for (int s = 0; s < NS; ++s) {
        mbar_init(&ms.full[s], 1);
        mbar_init(&ms.empty[s], kMW);
      }
      mbar_init(ms.merge_bar, 1);
      *ms.abort_flag = 0;
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
    __syncwarp();
    asm volatile("bar.arrive 2, %0;" ::"n"(kMFT) : "memory");
    produce_pieces<D>(a, &kmap, &vmap, stages, ms, sel_pref, sel_phys);
    return;
  }
  asm volatile("bar.sync 2, %0;" ::"n"(kMFT) : "memory");
  // ---- compute warps: every warp reads every piece's meta; group grp
  // computes the pieces i with i % 2 == grp, warp wr of the group rows
  // [16 wr, 16 wr + 16) of each.  All warps release every stage.
  const int cw = warp - 1;
  const int grp = cw / kMGW, wr = cw % kMGW;
  Iter it;
  iter_begin(a, it);
  const int n_units = it.done ? 0 : it.u1 - it.u;
  const uint32_t ring = smem_u32(stages);
  MmaState<D> st;
  int cur_bh = -1, i = 0, s = 0, units = 0;
  uint32_t ph = 0, merge_ph = 0;
  bool ok = true;
  while (units < n_units) {
    int flags = kPieceFlush, bh = -1, part = 0, nrows = 0;
    if (ok) ok = mbar_wait(&ms.full[s], ph, ms.abort_flag, a.at.status, 3);
    if (ok) {
      const Meta& mt = ms.meta[s];
      nrows = mt.nrows;
      bh = mt.pad[0];
      part = mt.pad[1];
      flags = mt.pad[2];
      if (bh != cur_bh) {
        cur_bh = bh;
        mma_load_q<D, G>(a.at, bh, st, qfrag + cw * (MmaState<D>::KS * 32));
      }
      if ((i & 1) == grp)
        mma_consume<D>(ring + uint32_t(s) * Geo::STAGE, nrows, st, wr, a.at.scale_log2);
      __syncwarp();
      if (lane == 0) mbar_arrive(&ms.empty[s]);
    }
    ++i;
    if (++s == NS) {
      s = 0;
      ph ^= 1u;
    }
    if (flags & kPieceFlush) {
      // ---- this warp's state of the head -> red[cw][hq]; after a failed
      // wait every warp still takes part in one flush per unit (with its
      // state as it stands) so that the barriers inside match
      if (cur_bh < 0) {
        cur_bh = 0;
        mma_load_q<D, G>(a.at, 0, st, qfrag + cw * (MmaState<D>::KS * 32));
      }
      float lt = st.l;
      lt += __shfl_xor_sync(0xffffffffu, lt, 1);
      lt += __shfl_xor_sync(0xffffffffu, lt, 2);
      const int hq = lane >> 2, c = (lane & 3) * 2;
      if (hq < G) {
        float* r = red + (cw * G + hq) * (D + 2);
        if (c == 0) {
          r[0] = st.m;
          r[1] = lt;
        }
#pragma unroll
        for (int nt = 0; nt < MmaState<D>::NTD; ++nt) {
          r[2 + nt * 8 + c] = st.o[nt][0];
          r[2 + nt * 8 + c + 1] = st.o[nt][1];
        }
      }
      // the unit's head and part: from the meta, or from the work list when the wait failed
      int fbh = bh, fpart = part;
      if (!ok) {
        Iter iu;
        iter_begin(a, iu);
        iu.u += units;
        if (iu.u < iu.u1) unit_begin(a, iu);
        fbh = iu.bh;
        fpart = iu.part;
      }
      finish_head<G, D, kMW, kMCT>(a, fbh, fpart, red, ms, stages, size_t(NS) * Geo::STAGE,
                                   merge_ph);
      cur_bh = -1;
      ++units;
    }
  }
}

constexpr size_t kMaxSmem = 227 * 1024;  // dynamic shared memory of one CTA

// Kernel, threads and shared memory of one (T, D, G) and path: the
// whole-block tensor-core kernel (MMA) or the CUDA-core one.
template <typename T, int D, int G, bool MMA>
struct FusedKernel {
  static constexpr int kThreads = MMA ? kMFT : kFT;
  static size_t smem(int NS) {
    if constexpr (MMA) return MmaSmem<D, G>::bytes(NS);
    else return FusedSmem<T, D, G>::bytes(NS);
  }
  static const void* fn() {
    if constexpr (MMA) return reinterpret_cast<const void*>(decode_mma_kernel<D, G>);
    else return reinterpret_cast<const void*>(decode_fused_kernel<T, D, G>);
  }
  static int stages() {
    int NS = kMaxStages;
    while (NS > 2 && smem(NS) > kMaxSmem) --NS;
    return NS;
  }
};

// CTAs of this kernel that fit on one SM (0: none; <0: a CUDA error); the
// query is cached per device (every decode step asks)
template <typename T, int D, int G, bool MMA>
int fused_occupancy_t() {
  using K = FusedKernel<T, D, G, MMA>;
  const size_t smem = K::smem(K::stages());
  if (smem > kMaxSmem) return 0;  // (large fp32 tiles) the split-K kernel runs instead
  const int occ = occupancy(K::fn(), K::kThreads, smem);
  static const bool debug = getenv("RBA_DEBUG") != nullptr;
  if (debug) {
    static std::once_flag once;
    std::call_once(once, [&] {
      cudaFuncAttributes fa = {};
      cudaFuncGetAttributes(&fa, K::fn());
      fprintf(stderr,
              "rba: decode attention kernel (%s) regs=%d maxThreads=%d static_smem=%zu "
              "local=%zu max_dyn_smem=%d requested_smem=%zu threads=%d occupancy=%d\n",
              MMA ? "tensor-core, whole blocks" : "cuda-core", fa.numRegs, fa.maxThreadsPerBlock,
              fa.sharedSizeBytes, fa.localSizeBytes, fa.maxDynamicSharedSizeBytes, smem,
              K::kThreads, occ);
    });
  }
  return occ;
}

template <typename T, int D, int G, bool MMA>
rba_status launch_fused_t(FusedArgs a, const CUtensorMap* maps, int P, bool pdl,
                          cudaStream_t stream) {
  using K = FusedKernel<T, D, G, MMA>;
  const int NS = K::stages();
  a.NS = NS;
  const size_t smem = K::smem(NS);
  const int occ = fused_occupancy_t<T, D, G, MMA>();
  if (occ < 0) return RBA_ERR_CUDA;
  if (occ < 1) return RBA_ERR_UNSUPPORTED;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(P);
  cfg.blockDim = dim3(K::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if constexpr (MMA) {
    CUtensorMap km = maps[0], vm = maps[1];
    void* args[] = {&km, &vm, &a};
    RBA_CUDA_TRY(cudaLaunchKernelExC(&cfg, K::fn(), args));
  } else {
    void* args[] = {&a};
    RBA_CUDA_TRY(cudaLaunchKernelExC(&cfg, K::fn(), args));
  }
  return RBA_OK;
}

// The whole-block tensor-core kernel covers bf16 stores whose blocks are whole
// 64-row tiles (and whose pools fit 32-bit tensor coordinates).
bool use_mma(const rba_store* st) {
  const rba_store_desc& d = st->d;
  return d.dtype == RBA_BF16 && (st->pitch == 64 || st->pitch == 128) &&
         d.block_size % kMTT == 0 &&
         int64_t(d.batch) * d.n_kv_heads * d.capacity_tokens < (int64_t(1) << 31) - kMTT;
}

}  // namespace

static int64_t attention_rows(const rba_store* st, const Geometry& g, int k) {
  const int64_t BH = int64_t(st->d.batch) * st->d.n_kv_heads;
  return BH * (int64_t(g.sink_end) + (g.T - g.w0) + (k > 0 ? int64_t(k) * st->d.block_size : 0));
}

// CTAs available to the attention launch: one per SM, leaving the SMs that
// the top-k kernel holds while this kernel starts; fewer for small problems.
static int cta_budget(const rba_store* st, const Geometry& g, int k) {
  const int BH = st->d.batch * st->d.n_kv_heads;
  int sms = num_sms();
  const int held = k > 0 ? topk_ctas(BH, g.nc) : 0;
  if (held > 0 && held <= sms / 4) sms -= held;
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
  return m > 1 ? align_up(size_t(BH) * m * slot_floats(G, st->pitch) * 4, 256) : 0;
}

size_t fused_sync_bytes(const rba_store* st) {
  return align_up(size_t(st->d.batch) * st->d.n_kv_heads * 4, 256);
}

// Whether the persistent attention kernel covers this problem (else the
// split-K kernel runs).
// Token-level retrieval (one key per block) runs split-K: the persistent
// kernels stage each selected row with its own bulk copies, and the split-K
// kernel's gathered 16-byte loads cost less (1M-token decode 528 -> 508 us,
// two-stage retrieval 108 -> 91 us per step on B200).
constexpr int kFusedMinBlock = 2;
bool fused_eligible(const rba_store* st, const Geometry& g, int k) {
  const rba_store_desc& d = st->d;
  if (d.block_size < kFusedMinBlock) return false;
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

bool fused_whole_blocks(const rba_store* st) { return use_mma(st); }

int fused_occupancy(const rba_store* st) {
  const rba_store_desc& d = st->d;
  const int G = d.n_q_heads / d.n_kv_heads;
  const bool mma = use_mma(st);
#define RBA_OCC(T_, D_, M_)                                 \
  switch (G) {                                              \
    case 1: return fused_occupancy_t<T_, D_, 1, M_>();      \
    case 2: return fused_occupancy_t<T_, D_, 2, M_>();      \
    case 4: return fused_occupancy_t<T_, D_, 4, M_>();      \
  }                                                         \
  return 0;
  if (d.dtype == RBA_BF16) {
    if (mma) {
      if (st->pitch == 128) { RBA_OCC(__nv_bfloat16, 128, true) }
      RBA_OCC(__nv_bfloat16, 64, true)
    }
    if (st->pitch == 128) { RBA_OCC(__nv_bfloat16, 128, false) }
    RBA_OCC(__nv_bfloat16, 64, false)
  }
  if (st->pitch == 128) { RBA_OCC(float, 128, false) }
  RBA_OCC(float, 64, false)
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
  at.qd = d.head_dim;
  at.scale_log2 = scale * 1.4426950408889634f;
  a.idx = const_cast<int32_t*>(idx);
  a.tickets = static_cast<uint32_t*>(sync);
  a.slots = slots;
  a.BH = BH;
  a.L_st = static_cast<int>(g.sink_end + (g.T - g.w0));
  a.U_sel = k > 0 ? k * d.block_size : 0;
  fused_slot_bytes(st, g, k, &a.m);
  // part boundaries (host side: no 64-bit divisions on the device).  For the
  // whole-block kernel both kinds of rows are cut at multiples of its tile,
  // so that interior tiles stay whole.
  const bool mma = use_mma(st);
  const int64_t Lh = int64_t(a.L_st) + a.U_sel;
  for (int c = 0; c <= a.m; ++c) {
    const int64_t x = Lh * c / a.m;
    int64_t xs = x * a.L_st / Lh;  // sink/window rows before the boundary
    int64_t xq = x - xs;           // selected rows before it
    if (mma && c < a.m) {
      xs = xs / kMTT * kMTT;
      xq = xq / kMTT * kMTT;
    }
    a.px[c] = static_cast<int>(xs + xq);
    a.ps[c] = static_cast<int>(xs);
  }
  CUtensorMap maps[2];
  static_assert(kMTT == 64, "the store's cached tensor maps use 64-row boxes");
  if (mma && !store_tmaps64(st, &maps[0], &maps[1])) return RBA_ERR_CUDA;
  const int G = d.n_q_heads / d.n_kv_heads;
#define RBA_FUSED(T_, D_, M_)                                                   \
  switch (G) {                                                                  \
    case 1: return launch_fused_t<T_, D_, 1, M_>(a, maps, P, pdl, stream);      \
    case 2: return launch_fused_t<T_, D_, 2, M_>(a, maps, P, pdl, stream);      \
    case 4: return launch_fused_t<T_, D_, 4, M_>(a, maps, P, pdl, stream);      \
  }                                                                             \
  return RBA_ERR_UNSUPPORTED;
  if (d.dtype == RBA_BF16) {
    if (mma) {
      if (st->pitch == 128) { RBA_FUSED(__nv_bfloat16, 128, true) }
      RBA_FUSED(__nv_bfloat16, 64, true)
    }
    if (st->pitch == 128) { RBA_FUSED(__nv_bfloat16, 128, false) }
    RBA_FUSED(__nv_bfloat16, 64, false)
  }
  if (st->pitch == 128) { RBA_FUSED(float, 128, false) }
  RBA_FUSED(float, 64, false)
#undef RBA_FUSED
}

}  // namespace rba
