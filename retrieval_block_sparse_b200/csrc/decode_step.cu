// One decode step in one launch: block scores -> per-head top-k -> attention
// over sink U selected blocks U window.
//
// Same definitions as rba_score (dot modes), rba_topk and rba_attend
// (Landmark Attention review, "proposed method": blocks scored by query /
// representative-key similarity; MemLong summary, 2.3.2: the top-k blocks;
// InfLLM article, "overall framework": softmax attention over the local
// window, the initial tokens and a few retrieved memory units).  Used for
// bf16 stores whose blocks are whole 64-row tiles and whose (batch, kv head)
// units number at most half the SMs.
//
// One cooperative launch of one CTA per SM; the CTAs of a unit ("head") are
// its parts.  Every CTA:
//   * stager warp: bulk-copies this part's slice of the head's representative
//     keys into shared memory, then streams the part's sink/window rows into
//     a ring of 64-row K/V stages (2-D tensor copies, 128-byte swizzle), waits
//     for the selection, and streams the part's share of the selected rows;
//   * eight compute warps: score the slice (summed GQA query against each
//     candidate's keys), publish the scores and bump the head's slice counter,
//     then run the tensor-core online softmax over the staged tiles
//     (mma.sync, as the whole-block attention kernel);
//   * selector warp: waits until every part of the head has published its
//     scores, reads the head's scores and selects the top k with one warp
//     (bitwise radix select on keys held in registers);
//     every part of the head selects the same set, so no second exchange is
//     needed.  Part 0 writes the selection out.
// Each part's softmax state goes to a slot; the last part of the head to
// finish (acq_rel ticket) merges the head's slots straight from L2 and resets
// the head's synchronisation words for the next call.
// Every wait is bounded (a per-store limit, 2 s by default); on expiry the
// status word records RBA_ERR_TIMEOUT, the CTA stops issuing work, drains its
// copies in flight and returns.
#include "decode_persist.cuh"
#include "decode_step.cuh"
#include "topk_impl.cuh"

namespace rba {
namespace {

constexpr int kSelWarp = kMW + 1;        // warp 9: the selector
constexpr int kSThreads = (kMW + 2) * 32;  // stager + 8 compute warps + selector
constexpr int kStepMaxNc = 4096;         // candidates per head the selector holds
constexpr int kStepMaxK = 256;           // selected blocks per head
constexpr int kStepMaxRep = 64 * 1024;   // bytes of one part's representative-key slice
constexpr int kStepMaxGrid = 256;

struct StepArgs {
  AttendArgs at;         // K, V, q, out, lse, status, cap, T, w0, Hq, Hkv, k, bs, sink,
                         // sink_end, first, nc, scale_log2
  const void* rep;       // [BH][rep_rows][R][D]
  int64_t rep_rows;
  float* scores;         // [BH][nc]
  int32_t* idx;          // [BH][k]
  float* slots;          // [P][slot floats]
  uint32_t* sync;        // [BH][2]: score slices published, parts flushed; zero between calls
  int BH, P, R, L_st, U_sel;
  int NS;                // stages of the K/V ring
  int rep_cap;           // bytes reserved for a part's representative-key slice
  int max_over_keys;
  unsigned long long wait_ns;
};

__host__ __device__ constexpr int step_slot_floats(int G, int D) { return (G * (D + 2) + 3) & ~3; }

// Head and part of CTA p: head h owns CTAs [ceil(h P / BH), ceil((h + 1) P / BH)).
struct PartOf {
  int h, c, m, p0;
};
__device__ __forceinline__ PartOf part_of(int p, int P, int BH) {
  PartOf r;
  r.h = static_cast<int>(int64_t(p) * BH / P);
  r.p0 = static_cast<int>((int64_t(r.h) * P + BH - 1) / BH);
  const int p1 = static_cast<int>((int64_t(r.h + 1) * P + BH - 1) / BH);
  r.c = p - r.p0;
  r.m = p1 - r.p0;
  return r;
}

// Boundary c of m over a head's rows (Lh = L_st + U_sel): sink/window rows
// before it (xs) and selected rows before it (xq); interior boundaries fall
// on 64-row multiples of both kinds so that interior tiles stay whole.
__device__ __forceinline__ void boundary(int64_t L_st, int64_t Lh, int c, int m, int* xs,
                                         int* xq) {
  const int64_t x = Lh * c / m;
  int64_t s = Lh > 0 ? x * L_st / Lh : 0;
  int64_t q = x - s;
  if (c < m) {
    s = s / kMTT * kMTT;
    q = q / kMTT * kMTT;
  }
  *xs = static_cast<int>(s);
  *xq = static_cast<int>(q);
}

__device__ __forceinline__ uint32_t ld_acquire_u32(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_add(uint32_t* p, uint32_t v) {
  asm volatile("red.release.gpu.global.add.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
// (a plain intrinsic: the compiler may issue many of these before their uses;
// the acquire that orders them is a volatile asm with a memory clobber)
__device__ __forceinline__ float ld_cg_f32(const float* p) { return __ldcg(p); }

// ---------------------------------------------------------------------------
// scoring of one part's candidate slice (compute warps)

// Candidates [0, ns) of the slice sit in shared memory, R keys of D elements
// each.  Lane l of a warp covers elements (l % LPK) * EPV + [0, EPV) of key
// r0 + l / LPK; warp cw scores candidates cw, cw + kMW, ...  The block score
// is the sum over the keys of (summed query) . key, or their max.
template <typename RT, int D>
__device__ __forceinline__ void score_slice(const char* rep, int ns, int R, bool maxr,
                                            const float* qs, float* out, int cw) {
  constexpr int EPV = 16 / int(sizeof(RT));
  constexpr int LPK = D / EPV;   // lanes per key
  constexpr int KPI = 32 / LPK;  // keys per warp iteration
  const int lane = threadIdx.x & 31;
  const int col = (lane % LPK) * EPV, kof = lane / LPK;
  float qv[EPV];
#pragma unroll
  for (int e = 0; e < EPV; ++e) qv[e] = qs[col + e];
  for (int c = cw; c < ns; c += kMW) {
    const uint4* cv = reinterpret_cast<const uint4*>(rep + size_t(c) * R * D * sizeof(RT));
    float acc = maxr ? -INFINITY : 0.f;
    for (int r0 = 0; r0 < R; r0 += KPI) {
      const int r = r0 + kof;
      float part = 0.f;
      if (r < R) {
        float f[EPV];
        unpack(cv[r * LPK + lane % LPK], f, RT());
#pragma unroll
        for (int e = 0; e < EPV; ++e) part = fmaf(qv[e], f[e], part);
      }
      if (maxr) {
#pragma unroll
        for (int o = LPK / 2; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
        acc = fmaxf(acc, r < R ? part : -INFINITY);
      } else {
        acc += part;
      }
    }
    if (maxr) {
#pragma unroll
      for (int o = LPK; o < 32; o <<= 1) acc = fmaxf(acc, __shfl_xor_sync(0xffffffffu, acc, o));
    } else {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    }
    if (lane == 0) out[c] = acc;
  }
}

// ---------------------------------------------------------------------------
// one-warp top-k (selector)
//
// The k best positions of a head's n scores under (larger score first, equal
// scores -> lower position first), written ascending to pos[0, k).  Scores
// become order-preserving 32-bit keys (-0 == +0; infinities and NaNs keep the
// order of their bits).  The scores are copied to shared memory (coalesced,
// 32 loads in flight per lane); per chunk of 1024 positions lane l holds the
// keys of positions [1024 c + 32 l, +32) in registers (read rotated, so the
// 32 lanes hit 32 banks), and its selection bits of those positions form one
// word, so the ascending positions come from one scan over the lanes.
// A radix select finds the threshold tau two bits at a time, starting below
// the bits that the smallest and largest keys share: the three trial values
// of the next two bits are counted with independent compares and three warp
// reductions, and the largest one that at least k keys reach is kept.  Once
// at most 256 keys reach tau, they alone can reach a later trial value: they
// are compacted to 8 registers per lane.  The search stops as soon as exactly
// k keys reach tau; otherwise tau ends as the k-th largest key and its lowest
// positions fill the set.

constexpr int kSelRegs = 32;   // keys per lane of one 1024-position chunk
constexpr int kSelLive = 8;    // keys per lane once at most 256 reach tau
// (the live keys and the spare words use the positions and prefix scratch)
static_assert(kSelLive * 32 + 32 <= 2 * kStepMaxK + 2, "live key scratch");

template <int N>
__device__ __forceinline__ void count3(const uint32_t (&key)[N], uint32_t t1, uint32_t t2,
                                       uint32_t t3, int& c1, int& c2, int& c3) {
#pragma unroll
  for (int i = 0; i < N; ++i) {
    c1 += key[i] >= t1;
    c2 += key[i] >= t2;
    c3 += key[i] >= t3;
  }
}

// keys of lane l in chunk c: register i holds position 1024 c + 32 l +
// ((i + l) & 31); positions past n read as 0 (every trial value is >= 1)
__device__ __forceinline__ void chunk_keys(const float* sm, int n, int c, uint32_t (&key)[kSelRegs]) {
  const int lane = threadIdx.x & 31;
  const int base = c * (kSelRegs * 32) + lane * 32;
#pragma unroll
  for (int i = 0; i < kSelRegs; ++i) {
    const int p = base + ((i + lane) & 31);
    key[i] = ordered_f32(sm[min(p, n - 1)]) & (0u - uint32_t(p < n));
  }
}

// g: the head's n scores in global memory; sm: shared scratch of n floats;
// live_sm: shared scratch of 256 + 32 words
__device__ __forceinline__ void warp_topk(const float* g, float* sm, uint32_t* live_sm, int n,
                                          int k, int* pos) {
  const int lane = threadIdx.x & 31;
  if (k >= n) {
    for (int j = lane; j < n; j += 32) pos[j] = j;
    __syncwarp();
    return;
  }
  for (int base = 0; base < n; base += kSelRegs * 32) {
    float v[kSelRegs];
#pragma unroll
    for (int u = 0; u < kSelRegs; ++u) v[u] = ld_cg_f32(g + min(base + u * 32 + lane, n - 1));
#pragma unroll
    for (int u = 0; u < kSelRegs; ++u)
      if (base + u * 32 + lane < n) sm[base + u * 32 + lane] = v[u];
  }
  __syncwarp();
  const int nch = (n + kSelRegs * 32 - 1) / (kSelRegs * 32);
  uint32_t key0[kSelRegs];
  chunk_keys(sm, n, 0, key0);
  // smallest and largest key (padding keys: 0, raised for the minimum)
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  for (int c = 0; c < nch; ++c) {
    uint32_t key[kSelRegs];
    if (c == 0) {
#pragma unroll
      for (int i = 0; i < kSelRegs; ++i) key[i] = key0[i];
    } else {
      chunk_keys(sm, n, c, key);
    }
    const int cb = c * (kSelRegs * 32) + lane * 32;
#pragma unroll
    for (int i = 0; i < kSelRegs; ++i) {
      kmin = min(kmin, key[i] | (0u - uint32_t(cb + ((i + lane) & 31) >= n)));
      kmax = max(kmax, key[i]);
    }
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  // every key lies in [kmin, kmax]: the bits above their highest differing
  // bit are common, and all n keys reach that prefix
  uint32_t tau = kmin;
  int cnt = n;
  bool compact = false;
  uint32_t live[kSelLive];
#pragma unroll
  for (int j = 0; j < kSelLive; ++j) live[j] = 0u;
  const uint32_t diff = kmin ^ kmax;
  if (diff != 0u) {
    const int top = 31 - __clz(diff);
    tau = top == 31 ? 0u : (kmax & ~((2u << top) - 1u));
    for (int b = top; b >= 0 && cnt != k; b -= 2) {
      if (!compact && cnt <= kSelLive * 32) {
        // the keys >= tau, in any order, to live[] (cnt of them)
        int off = 0;
        for (int c = 0; c < nch; ++c) {
          uint32_t key[kSelRegs];
          if (c == 0) {
#pragma unroll
            for (int i = 0; i < kSelRegs; ++i) key[i] = key0[i];
          } else {
            chunk_keys(sm, n, c, key);
          }
          const int cb = c * (kSelRegs * 32) + lane * 32;
          uint32_t in = 0u;  // bit i: register i holds a key >= tau
#pragma unroll
          for (int i = 0; i < kSelRegs; ++i)
            in |= (uint32_t(key[i] >= tau) & uint32_t(cb + ((i + lane) & 31) < n)) << i;
          const int sc = __popc(in);
          int incl = sc;
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const int t = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += t;
          }
          int o2 = off + incl - sc;
          // every register is stored: a key that is out goes to this lane's
          // spare word past the 256
#pragma unroll
          for (int i = 0; i < kSelRegs; ++i) {
            const uint32_t b = (in >> i) & 1u;
            live_sm[b ? o2 : kSelLive * 32 + lane] = key[i];
            o2 += int(b);
          }
          off += __shfl_sync(0xffffffffu, incl, 31);
        }
        __syncwarp();
#pragma unroll
        for (int j = 0; j < kSelLive; ++j)
          live[j] = live_sm[j * 32 + lane] & (0u - uint32_t(j * 32 + lane < off));
        __syncwarp();
        compact = true;
      }
      // the next two bits (b, b - 1), or bit 0 alone
      const int sh = b >= 1 ? b - 1 : 0;
      const uint32_t t1 = tau | (1u << sh);
      const uint32_t t2 = b >= 1 ? tau | (2u << sh) : t1;
      const uint32_t t3 = b >= 1 ? tau | (3u << sh) : t1;
      int c1 = 0, c2 = 0, c3 = 0;
      if (compact) {
        count3(live, t1, t2, t3, c1, c2, c3);
      } else {
        count3(key0, t1, t2, t3, c1, c2, c3);
        for (int c = 1; c < nch; ++c) {
          uint32_t key[kSelRegs];
          chunk_keys(sm, n, c, key);
          count3(key, t1, t2, t3, c1, c2, c3);
        }
      }
      c1 = static_cast<int>(__reduce_add_sync(0xffffffffu, unsigned(c1)));
      c2 = static_cast<int>(__reduce_add_sync(0xffffffffu, unsigned(c2)));
      c3 = static_cast<int>(__reduce_add_sync(0xffffffffu, unsigned(c3)));
      if (c3 >= k) {
        tau = t3;
        cnt = c3;
      } else if (c2 >= k) {
        tau = t2;
        cnt = c2;
      } else if (c1 >= k) {
        tau = t1;
        cnt = c1;
      }
    }
  }
  // cnt == k: exactly the keys >= tau.  Otherwise tau is the k-th largest
  // key: every key > tau, then the lowest positions of the keys == tau.
  const bool exact = cnt == k;
  // selected outright: keys >= lo (none when tau is the largest key value)
  const bool none_above = !exact && tau == 0xffffffffu;
  const uint32_t lo = exact ? tau : tau + 1u;
  int need = 0;
  if (none_above) {
    need = k;
  } else if (!exact) {
    int c1 = 0, c2 = 0, c3 = 0;
    if (compact) {
      count3(live, lo, lo, lo, c1, c2, c3);
    } else {
      count3(key0, lo, lo, lo, c1, c2, c3);
      for (int c = 1; c < nch; ++c) {
        uint32_t key[kSelRegs];
        chunk_keys(sm, n, c, key);
        count3(key, lo, lo, lo, c1, c2, c3);
      }
    }
    need = k - static_cast<int>(__reduce_add_sync(0xffffffffu, unsigned(c1)));
  }
  const uint32_t take_above = none_above ? 0u : 1u;
  int written = 0;
  for (int c = 0; c < nch; ++c) {
    uint32_t key[kSelRegs];
    if (c == 0) {
#pragma unroll
      for (int i = 0; i < kSelRegs; ++i) key[i] = key0[i];
    } else {
      chunk_keys(sm, n, c, key);
    }
    // this lane's selection bits of positions [1024 c + 32 lane, +32)
    const int base = c * (kSelRegs * 32) + lane * 32;
    uint32_t word = 0u, ties = 0u;
#pragma unroll
    for (int i = 0; i < kSelRegs; ++i) {
      const int bit = (i + lane) & 31;
      word |= (uint32_t(key[i] >= lo) & take_above) << bit;
      ties |= (uint32_t(key[i] == tau) & uint32_t(base + bit < n)) << bit;
    }
    if (need > 0) {
      // the lowest positions of the ties: lanes in order, bits in order
      const int tc = __popc(ties);
      int incl = tc;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += t;
      }
      int r = min(max(need - (incl - tc), 0), tc);
      while (r-- > 0) {
        word |= ties & (0u - ties);
        ties &= ties - 1u;
      }
      need -= min(need, __shfl_sync(0xffffffffu, incl, 31));
    }
    const int wc = __popc(word);
    int incl = wc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += t;
    }
    int p = written + incl - wc;
    while (word) {
      pos[p++] = base + __ffs(word) - 1;
      word &= word - 1u;
    }
    written += __shfl_sync(0xffffffffu, incl, 31);
  }
  __syncwarp();
}

// ---------------------------------------------------------------------------
// shared memory

template <int D, int G>
struct StepSmem {
  using Geo = MmaGeo<D>;
  static constexpr int up16(int x) { return (x + 15) & ~15; }
  static constexpr int RED = up16(kMW * G * (D + 2) * 4);    // warp states
  static constexpr int QF = (D / 16) * 32 * 8;              // Q fragments (one copy)
  static constexpr int QS = D * 4;                           // summed query (fp32)
  static constexpr int SELL = (3 * kStepMaxK + 4) * 4;       // positions, prefix, starts
  static constexpr int MISC = kMiscBytes;
  static constexpr int ALIGN = 1024;
  // ring of NS stages, then the rep slice (rep_bytes), the head's scores
  // (nc floats), then the fixed regions
  static size_t bytes(int NS, int rep_bytes, int nc) {
    return size_t(NS) * Geo::STAGE + up16(rep_bytes) + up16(nc * 4) + RED + QF + QS +
           SELL + MISC + ALIGN;
  }
};

// misc words used by this kernel (after the MiscLayout fields, in s_misc):
// [10] is-last flag of the flush; the rep-slice and selection mbarriers
// follow the merge mbarrier.
struct StepBars {
  uint64_t* rep;
  uint64_t* sel;
  __device__ explicit StepBars(const MiscLayout& ms) {
    rep = reinterpret_cast<uint64_t*>(reinterpret_cast<char*>(ms.s_misc) + 152 * 4);
    sel = rep + 1;
  }
};
static_assert(2 * kMaxStages * 8 + kMaxStages * 16 + 152 * 4 + 16 <= kMiscBytes, "misc layout");

// ---------------------------------------------------------------------------
// the kernel

template <int D, int G, typename RT>
__global__ void __launch_bounds__(kSThreads, 1)
    decode_step_kernel(const __grid_constant__ CUtensorMap kmap,
                       const __grid_constant__ CUtensorMap vmap, StepArgs a) {
  static_assert(G <= 8, "q heads of a kv head fit the rows 0..7 of the A tile");
  using Geo = MmaGeo<D>;
  using S = StepSmem<D, G>;
  constexpr int kSlotF = step_slot_floats(G, D);
  extern __shared__ char smem_raw[];
  // 1024-byte aligned base, offset from the shared array itself (an integer
  // round trip would hide from the compiler that the pointers address shared
  // memory and turn every access into a generic one)
  char* ring = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const AttendArgs& at = a.at;
  const int NS = a.NS;
  const PartOf po = part_of(blockIdx.x, a.P, a.BH);
  const int bh = po.h;
  // this part's candidate slice [cs0, cs1) and its representative keys
  const int cs0 = static_cast<int>(int64_t(at.nc) * po.c / po.m);
  const int cs1 = static_cast<int>(int64_t(at.nc) * (po.c + 1) / po.m);
  const int ns = cs1 - cs0;
  const size_t cand_bytes = size_t(a.R) * D * sizeof(RT);
  const int rep_bytes = static_cast<int>(size_t(ns) * cand_bytes);
  char* rep = ring + size_t(NS) * Geo::STAGE;
  float* ssc = reinterpret_cast<float*>(rep + S::up16(a.rep_cap));
  float* red = reinterpret_cast<float*>(reinterpret_cast<char*>(ssc) + S::up16(at.nc * 4));
  uint2* qfrag = reinterpret_cast<uint2*>(reinterpret_cast<char*>(red) + S::RED);
  float* qs = reinterpret_cast<float*>(reinterpret_cast<char*>(qfrag) + S::QF);
  int* selpos = reinterpret_cast<int*>(reinterpret_cast<char*>(qs) + S::QS);
  int* sel_pref = selpos + kStepMaxK;
  int* sel_phys = sel_pref + kStepMaxK + 2;
  const MiscLayout ms(reinterpret_cast<char*>(selpos) + S::SELL);
  const StepBars sb(ms);

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t Lh = int64_t(a.L_st) + a.U_sel;
  if (warp == 0) {
    // ---- stager
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&kmap))
                   : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&vmap))
                   : "memory");
      for (int s = 0; s < NS; ++s) {
        mbar_init(&ms.full[s], 1);
        mbar_init(&ms.empty[s], kMW);
      }
      mbar_init(sb.rep, 1);
      mbar_init(sb.sel, 1);
      *ms.abort_flag = 0;
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      // the representative keys of this part's slice first: the scores are
      // on the critical path
      mbar_arrive_tx(sb.rep, uint32_t(rep_bytes));
      if (rep_bytes > 0)
        bulk_g2s(rep,
                 static_cast<const char*>(a.rep) +
                     (size_t(bh) * a.rep_rows + at.first + cs0) * cand_bytes,
                 uint32_t(rep_bytes), sb.rep);
    }
    __syncwarp();
    asm volatile("bar.arrive 2, %0;" ::"n"(kSThreads) : "memory");
    // the K/V stream starts once the slice has landed, so that the scores
    // (on the critical path) do not share the first microseconds of HBM
    // bandwidth with it
    bool alive = mbar_wait(sb.rep, 0, ms.abort_flag, at.status, 6, a.wait_ns, kWhereStep);
    int xs0, xq0, xs1, xq1;
    boundary(a.L_st, Lh, po.c, po.m, &xs0, &xq0);
    boundary(a.L_st, Lh, po.c + 1, po.m, &xs1, &xq1);
    int j = 0, s = 0;
    uint32_t ph = 0;
    bool pend = false;
    int pn = 0, py = 0;
    auto emit = [&](int n, int y, bool flush) -> bool {
      if (j >= NS &&
          !mbar_wait(&ms.empty[s], ph ^ 1u, ms.abort_flag, at.status, 1, a.wait_ns, kWhereStep))
        return false;
      if (lane == 0) {
        Meta& mt = ms.meta[s];
        mt.nrows = n;
        mt.pad[0] = bh;
        mt.pad[1] = po.c;
        mt.pad[2] = flush ? kPieceFlush : 0;
        mbar_arrive_tx(&ms.full[s], n > 0 ? uint32_t(Geo::TX) : 0u);
        if (n > 0) {
          char* stg = ring + size_t(s) * Geo::STAGE;
#pragma unroll
          for (int hh = 0; hh < Geo::NH; ++hh) {
            tma_load_2d(stg + hh * kHalfBytes, &kmap, hh * 64, y, &ms.full[s]);
            tma_load_2d(stg + Geo::VOFF + hh * kHalfBytes, &vmap, hh * 64, y, &ms.full[s]);
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
    // pieces of one kind: rows [v, vend) of the virtual layout given by the
    // segment prefix pref(i) (nseg segments starting at physical rows
    // phys(i)), cut at segment ends and at 64 rows.  (Accessors rather than
    // arrays: a small array indexed at run time would live in local memory,
    // and every access to it would wait on an L2 kept busy by the copies.)
    auto run = [&](int v, int vend, auto pref, auto phys, int nseg) {
      const int vlim = min(vend, pref(nseg));
      while (alive && v < vlim) {
        int lo2 = 0, hi2 = nseg - 1;
        while (lo2 < hi2) {
          const int mid = (lo2 + hi2 + 1) >> 1;
          if (pref(mid) <= v) lo2 = mid; else hi2 = mid - 1;
        }
        const int n = min(min(vlim, pref(lo2 + 1)), v + kMTT) - v;
        const int y = static_cast<int>(int64_t(bh) * at.cap + phys(lo2) + (v - pref(lo2)));
        if (pend && !emit(pn, py, false)) {
          alive = false;
          break;
        }
        pend = true;
        pn = n;
        py = y;
        v += n;
      }
    };
    {
      // sink rows [0, sink_end) then window rows [w0, T): two segments
      const int se = at.sink_end, lst = a.L_st, w0 = static_cast<int>(at.w0);
      run(xs0, xs1, [=](int i) { return i == 0 ? 0 : (i == 1 ? se : lst); },
          [=](int i) { return i == 0 ? 0 : w0; }, 2);
    }
    if (alive) {
      // the selector fills sel_pref / sel_phys and arrives on sel (also
      // when this part holds no selected rows: the flush piece, hence the
      // part's ticket, must follow the selector's last read of the head's
      // synchronisation words)
      if (!mbar_wait(sb.sel, 0, ms.abort_flag, at.status, 2, a.wait_ns, kWhereStep) ||
          *ms.abort_flag != 0)
        alive = false;
      else if (xq1 > xq0)
        run(xq0, xq1, [=](int i) { return sel_pref[i]; }, [=](int i) { return sel_phys[i]; }, at.k);
    }
    if (alive) emit(pend ? pn : 0, py, true);
    // no copy may still be landing in shared memory when the CTA exits
    if (lane == 0) {
      for (int q = max(0, j - NS); q < j; ++q) mbar_drain(&ms.full[q % NS], (q / NS) & 1u);
      mbar_drain(sb.rep, 0);
    }
    __syncwarp();
    return;
  }
  asm volatile("bar.sync 2, %0;" ::"n"(kSThreads) : "memory");

  if (warp == kSelWarp) {
    // ---- selector: wait until every part of the head has published its
    // scores, then select the head's top k (every part computes the same set)
    bool ok = true;
    if (lane == 0) {
      const unsigned long long t0 = now_ns();
      while (ld_acquire_u32(a.sync + 2 * bh) < uint32_t(po.m)) {
        if (*ms.abort_flag != 0) {
          ok = false;
          break;
        }
        if (now_ns() - t0 > a.wait_ns) {
          report(at.status, RBA_ERR_TIMEOUT, kWhereStep, 3);
          *ms.abort_flag = 1;
          ok = false;
          break;
        }
        __nanosleep(64);
      }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok) {
      // (live-key scratch: selpos and the start of sel_pref, both written after it)
      warp_topk(a.scores + int64_t(bh) * at.nc, ssc, reinterpret_cast<uint32_t*>(selpos), at.nc,
                at.k, selpos);
      // the selected blocks as segments of the attended set (clipped to
      // [sink, w0)), prefix of their lengths; part 0 writes the selection out
      int run = 0;
      for (int base = 0; base < at.k; base += 32) {
        const int jj = base + lane;
        int len = 0, start = 0;
        if (jj < at.k) {
          const int blk = at.first + selpos[jj];
          if (po.c == 0) a.idx[int64_t(bh) * at.k + jj] = blk;
          const int64_t lo = max(int64_t(blk) * at.bs, int64_t(at.sink));
          const int64_t hi = min(int64_t(blk + 1) * at.bs, at.w0);
          start = static_cast<int>(lo);
          len = hi > lo ? static_cast<int>(hi - lo) : 0;
        }
        int incl = len;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int t = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += t;
        }
        if (jj < at.k) {
          sel_pref[jj] = run + incl - len;
          sel_phys[jj] = start;
        }
        run += __shfl_sync(0xffffffffu, incl, 31);
      }
      if (lane == 0) sel_pref[at.k] = run;
      __syncwarp();
    }
    if (lane == 0) mbar_arrive(sb.sel);  // (after a failure the stager sees the abort flag)
    return;
  }

  // ---- compute warps (named barrier 1 among them)
  const int cw = warp - 1, tid = ctid();
  const int grp = cw / kMGW, wr = cw % kMGW;
  const int b = bh / at.Hkv, h = bh % at.Hkv;
  // one copy of the head's Q fragments serves all compute warps (they all
  // work on this CTA's head)
  MmaState<D> st;
  if (cw == 0) {
    MmaState<D> tmp;
    mma_load_q<D, G>(at, bh, tmp, qfrag);
  }
  st.qf = qfrag;
  st.m = -INFINITY;
  st.l = 0.f;
#pragma unroll
  for (int nt = 0; nt < MmaState<D>::NTD; ++nt) st.o[nt][0] = st.o[nt][1] = 0.f;
  if (tid < D) {
    const __nv_bfloat16* qp = static_cast<const __nv_bfloat16*>(at.q) +
                              (int64_t(b) * at.Hq + h * G) * at.qd + tid;
    float acc = 0.f;
    if (tid < at.qd) {  // (padding columns of the pools score zero)
#pragma unroll
      for (int i = 0; i < G; ++i) acc += __bfloat162float(qp[i * at.qd]);
    }
    qs[tid] = acc;
  }
  compute_sync<kMCT>();
  // scores of this part's slice -> global, then the head's slice counter
  if (mbar_wait(sb.rep, 0, ms.abort_flag, at.status, 4, a.wait_ns, kWhereStep))
    score_slice<RT, D>(rep, ns, a.R, a.max_over_keys != 0, qs,
                       a.scores + int64_t(bh) * at.nc + cs0, cw);
  compute_sync<kMCT>();
  if (tid == 0) red_release_add(a.sync + 2 * bh, 1u);  // published even after a failure

  // ---- attention over the staged pieces of this part
  const uint32_t ring_s = smem_u32(ring);
  int i = 0, s = 0;
  uint32_t ph = 0;
  while (true) {
    if (!mbar_wait(&ms.full[s], ph, ms.abort_flag, at.status, 5, a.wait_ns, kWhereStep)) break;
    const Meta& mt = ms.meta[s];
    const int nrows = mt.nrows, flags = mt.pad[2];
    if ((i & 1) == grp) mma_consume<D>(ring_s + uint32_t(s) * Geo::STAGE, nrows, st, wr,
                                       at.scale_log2);
    __syncwarp();
    if (lane == 0) mbar_arrive(&ms.empty[s]);
    ++i;
    if (++s == NS) {
      s = 0;
      ph ^= 1u;
    }
    if (flags & kPieceFlush) break;
  }

  // ---- flush: the 8 warp states -> this part's slot
  {
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
  }
  compute_sync<kMCT>();
  // this part's state: the kMW warp states combined into its global slot
  float* slot = a.slots + int64_t(blockIdx.x) * kSlotF;
  for (int x = tid; x < G * (D + 2); x += kMCT) {
    const int gg = x / (D + 2), col = x - gg * (D + 2);
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kMW; ++w) M = fmaxf(M, red[(w * G + gg) * (D + 2)]);
    float v = M;
    if (col > 0) {
      v = 0.f;
#pragma unroll
      for (int w = 0; w < kMW; ++w) {
        const float mw = red[(w * G + gg) * (D + 2)];
        const float f = mw == -INFINITY ? 0.f : exp2f(mw - M);
        v = fmaf(f, red[(w * G + gg) * (D + 2) + col], v);
      }
    }
    slot[x] = v;
  }
  compute_sync<kMCT>();
  if (tid == 0) {
    const uint32_t t = atom_add_acq_rel(a.sync + 2 * bh + 1, 1u);  // publishes the slot
    ms.s_misc[10] = t == uint32_t(po.m - 1);
  }
  compute_sync<kMCT>();
  if (!ms.s_misc[10]) return;

  // ---- the last part of the head: merge the head's m slots from L2, in
  // two rounds of independent loads.  Warp g < G: slot j's (m, l) of q head
  // g in lane j % 32, the head's max M and sum L, and one factor 2^(m_j - M)
  // per slot; then every thread folds its output elements over the slots.
  const float* slots = a.slots + int64_t(po.p0) * kSlotF;
  float* fac = red;  // [G][m] (the warp states are consumed)
  constexpr int kMaxSlotRegs = (kStepMaxGrid + 31) / 32;
  if (cw < G) {
    const int g = cw;
    float mj[kMaxSlotRegs], lj[kMaxSlotRegs];
    float M = -INFINITY;
#pragma unroll
    for (int r = 0; r < kMaxSlotRegs; ++r) {
      const int j = lane + 32 * r;
      const float* sl = slots + int64_t(j) * kSlotF + g * (D + 2);
      mj[r] = j < po.m ? ld_cg_f32(sl) : -INFINITY;
      lj[r] = j < po.m ? ld_cg_f32(sl + 1) : 0.f;
      M = fmaxf(M, mj[r]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
    float L = 0.f;
#pragma unroll
    for (int r = 0; r < kMaxSlotRegs; ++r) {
      const int j = lane + 32 * r;
      const float f = mj[r] == -INFINITY ? 0.f : exp2f(mj[r] - M);
      if (j < po.m) fac[g * po.m + j] = f;
      L = fmaf(f, lj[r], L);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) L += __shfl_xor_sync(0xffffffffu, L, o);
    if (lane == 0) {
      ms.s_f[g] = M;
      ms.s_f[16 + g] = L;
    }
  }
  compute_sync<kMCT>();
  for (int x = tid; x < G * at.qd; x += kMCT) {
    const int gg = x / at.qd, d = x - gg * at.qd;
    const float* col = slots + gg * (D + 2) + 2 + d;
    const float* fg = fac + gg * po.m;
    float O = 0.f;
    for (int j0 = 0; j0 < po.m; j0 += 16) {  // 16 loads in flight, then their terms
      float ov[16];
#pragma unroll
      for (int u = 0; u < 16; ++u)
        ov[u] = j0 + u < po.m ? ld_cg_f32(col + int64_t(j0 + u) * kSlotF) : 0.f;
#pragma unroll
      for (int u = 0; u < 16; ++u)
        if (j0 + u < po.m) O = fmaf(fg[j0 + u], ov[u], O);
    }
    const float M = ms.s_f[gg], L = ms.s_f[16 + gg];
    at.out[(int64_t(b) * at.Hq + h * G + gg) * at.qd + d] = L > 0.f ? O / L : 0.f;
    if (d == 0 && at.lse != nullptr)
      at.lse[int64_t(b) * at.Hq + h * G + gg] =
          L > 0.f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
  }
  if (tid == 0) {
    // every part of the head is past its selection and its flush: the
    // head's synchronisation words are free for the next call
    a.sync[2 * bh] = 0u;
    a.sync[2 * bh + 1] = 0u;
  }
}

// ---------------------------------------------------------------------------
// host side

constexpr size_t kStepMaxSmem = 227 * 1024;

template <int D, int G, typename RT>
const void* step_fn() {
  return reinterpret_cast<const void*>(decode_step_kernel<D, G, RT>);
}

const void* step_kernel(const rba_store* st) {
  const rba_store_desc& d = st->d;
  const int G = d.n_q_heads / d.n_kv_heads;
  const bool f32rep = d.mode == RBA_REP_MEAN;
#define RBA_STEP_FN(D_)                                                                \
  switch (G) {                                                                         \
    case 1: return f32rep ? step_fn<D_, 1, float>() : step_fn<D_, 1, __nv_bfloat16>(); \
    case 2: return f32rep ? step_fn<D_, 2, float>() : step_fn<D_, 2, __nv_bfloat16>(); \
    case 4: return f32rep ? step_fn<D_, 4, float>() : step_fn<D_, 4, __nv_bfloat16>(); \
  }                                                                                    \
  return nullptr;
  if (st->pitch == 128) { RBA_STEP_FN(128) }
  RBA_STEP_FN(64)
#undef RBA_STEP_FN
}

size_t step_cand_bytes(const rba_store* st) {
  const rba_store_desc& d = st->d;
  return size_t(d.n_rep) * st->pitch * (d.mode == RBA_REP_MEAN ? 4 : 2);
}

// How the step runs: a cooperative launch of one CTA per SM; a head has at
// least P / BH parts.
struct StepPlan {
  int P;          // CTAs
  int parts;      // fewest parts of a head
  int rep_cap;    // bytes of the representative keys of the largest part slice
  int NS;         // ring stages (0: does not fit)
  size_t smem;
};

// false: the step does not fit
bool step_plan(const rba_store* st, const Geometry& g, StepPlan* pl) {
  const int BH = st->d.batch * st->d.n_kv_heads;
  const int G = st->d.n_q_heads / st->d.n_kv_heads;
  int sms = num_sms();
  if (sms > kStepMaxGrid) sms = kStepMaxGrid;
  pl->P = sms;
  pl->parts = sms / BH;
  if (pl->parts < 2) return false;
  pl->rep_cap = static_cast<int>(size_t((g.nc + pl->parts - 1) / pl->parts) *
                                 step_cand_bytes(st));
  if (pl->rep_cap > kStepMaxRep) return false;
  pl->NS = 0;
  for (int NS = kMaxStages; NS >= 2 && pl->NS == 0; --NS) {
    size_t b = 0;
    if (st->pitch == 128) {
      b = G == 1 ? StepSmem<128, 1>::bytes(NS, pl->rep_cap, g.nc)
        : G == 2 ? StepSmem<128, 2>::bytes(NS, pl->rep_cap, g.nc)
                 : StepSmem<128, 4>::bytes(NS, pl->rep_cap, g.nc);
    } else {
      b = G == 1 ? StepSmem<64, 1>::bytes(NS, pl->rep_cap, g.nc)
        : G == 2 ? StepSmem<64, 2>::bytes(NS, pl->rep_cap, g.nc)
                 : StepSmem<64, 4>::bytes(NS, pl->rep_cap, g.nc);
    }
    if (b <= kStepMaxSmem) {
      pl->NS = NS;
      pl->smem = b;
    }
  }
  if (pl->NS < 2) return false;
  const void* fn = step_kernel(st);
  return fn != nullptr && occupancy(fn, kSThreads, pl->smem) >= 1;
}

}  // namespace

bool step_eligible(const rba_store* st, const Geometry& g, int k) {
  const rba_store_desc& d = st->d;
  if (st->one_launch == 0) return false;
  if (d.dtype != RBA_BF16 || (st->pitch != 64 && st->pitch != 128)) return false;
  if (d.block_size % kMTT != 0) return false;
  if (d.mode != RBA_REP_MEAN && d.mode != RBA_REP_TOPR_ATTN && d.mode != RBA_REP_EXTERNAL)
    return false;
  const int G = d.n_q_heads / d.n_kv_heads;
  if (G != 1 && G != 2 && G != 4) return false;
  if (d.n_rep > 8) return false;
  if (k < 1 || k > kStepMaxK || g.nc < 1 || g.nc > kStepMaxNc || k > g.nc) return false;
  if (int64_t(d.batch) * d.n_kv_heads * d.capacity_tokens >= (int64_t(1) << 31) - kMTT)
    return false;
  StepPlan pl;
  return step_plan(st, g, &pl);
}

size_t step_sync_bytes(const rba_store* st) {
  return align_up(size_t(st->d.batch) * st->d.n_kv_heads * 2 * 4, 256);
}

size_t step_slot_bytes(const rba_store* st) {
  const rba_store_desc& d = st->d;
  const int G = d.n_q_heads / d.n_kv_heads;
  int sms = num_sms();
  if (sms > kStepMaxGrid) sms = kStepMaxGrid;
  return align_up(size_t(sms) * step_slot_floats(G, st->pitch) * 4, 256);
}

rba_status launch_step(const rba_store* st, const void* q, int k, const Geometry& g, float scale,
                       float* scores, int32_t* idx, float* out, float* lse, void* sync,
                       float* slots, cudaStream_t stream) {
  const rba_store_desc& d = st->d;
  StepPlan pl;
  if (!step_plan(st, g, &pl)) return RBA_ERR_UNSUPPORTED;
  StepArgs a = {};
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
  a.rep = st->rep;
  a.rep_rows = st->cap_blocks;
  a.scores = scores;
  a.idx = idx;
  a.slots = slots;
  a.sync = static_cast<uint32_t*>(sync);
  a.BH = d.batch * d.n_kv_heads;
  a.P = pl.P;
  a.R = d.n_rep;
  a.L_st = static_cast<int>(g.sink_end + (g.T - g.w0));
  a.U_sel = k * d.block_size;
  a.NS = pl.NS;
  a.rep_cap = pl.rep_cap;
  a.max_over_keys = st->score_reduce == RBA_SCORE_MAX ? 1 : 0;
  a.wait_ns = st->wait_ns;
  CUtensorMap maps[2];
  static_assert(kMTT == 64, "the store's cached tensor maps use 64-row boxes");
  if (!store_tmaps64(st, &maps[0], &maps[1])) return RBA_ERR_CUDA;
  const void* fn = step_kernel(st);
  if (fn == nullptr) return RBA_ERR_UNSUPPORTED;
  RBA_CUDA_TRY(ensure_smem(fn, pl.smem));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(pl.P);
  cfg.blockDim = dim3(kSThreads);
  cfg.dynamicSmemBytes = pl.smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeCooperative;  // the parts of a head wait on one another
  attr[0].val.cooperative = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  void* args[] = {&maps[0], &maps[1], &a};
  RBA_CUDA_TRY(cudaLaunchKernelExC(&cfg, fn, args));
  return RBA_OK;
}

}  // namespace rba
