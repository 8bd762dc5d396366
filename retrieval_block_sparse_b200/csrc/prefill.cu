// Chunked prefill with retrieval-causal attention on the tensor cores.
//
// MemLong summary, 2.3.3 and Figure 3: every row of a query chunk attends
// bidirectionally to the retrieved past tokens (sink U selected blocks U
// window of the memory) and causally to its own chunk, in one softmax;
// 2.3.4: the retrieved window is k * block size.
//
// One CTA = one (chunk, q head, 256 query rows) = two 128-row query tiles A
// and B that share every K/V tile (half the K/V traffic per FLOP):
//   warp 8      TMA producer: both Q tiles once, then K/V tiles of 128 keys
//               (128B-swizzled) into a two-stage ring;
//   warp 9      MMA issuer (one lane): S_X = Q_X K^T into TMEM, then
//               O_X += P_X V with P_X read from TMEM (tcgen05.mma kind::f16,
//               bf16 in, fp32 accumulate), alternating between the tiles so
//               the tensor core works on one tile while the other's softmax
//               runs;
//   warps 0-3 / 4-7   softmax of tile A / B: thread t owns query row t; two
//               passes over its S row in 32-column chunks (max, then
//               exp2(scale s - m) packed to bf16 and stored back over the S
//               columns as P); O rows are rescaled in TMEM when the max grows
//               by more than 2^8; at the end O is normalised into the output.
// TMEM: S_A / P_A columns [0,128), S_B / P_B [128,256), O_A [256,384),
// O_B [384,512).
// Past blocks shorter than a tile (token-level retrieval) are first gathered
// into a contiguous staging buffer so that every tile is one TMA box.
// All waits on mbarriers are bounded; on expiry the kernel records
// RBA_ERR_TIMEOUT, stops issuing work, drains, frees TMEM and returns.
#include <cuda.h>
#include <cstring>

#include "rba_internal.cuh"

namespace rba {
namespace {

constexpr int kBM = 128;   // query rows per tile (two tiles per CTA)
constexpr int kBN = 128;   // keys per tile
constexpr int kHD = 128;   // head dim (bf16)
constexpr int kMaxTiles = 320;
constexpr int kThreads = 320;  // 8 softmax warps, TMA warp, MMA warp
constexpr unsigned long long kTimeoutNs = 2000000000ull;

enum MapId { kPool = 0, kStage = 1, kChunk = 2 };

struct PrefillArgs {
  const int32_t* idx;  // [n_chunks][n_sel][k]
  float* out;          // [n_chunks][Hq][Nq][D]
  float* lse;          // [n_chunks][Hq][Nq] or nullptr
  int32_t* status;
  int64_t cap, T, w0;
  int Hq, Hkv, G, Nq, n_chunks, n_sel, k, bs, sink, sink_end, first, nc;
  int store_batch;     // 1 (one memory for all chunks) or n_chunks
  int staged;          // past tokens come from the staging buffer
  int n_att_max;       // staging rows per (chunk, kv head)
  int pairs_outer;     // grid order: 1 = (head, chunk, pair), heaviest pairs first
  int od;              // row length of out (the head dim; tiles are kHD wide, zero-padded)
  float scale_log2;
};

// shared memory map (bytes, from a 1024-aligned base)
constexpr int kQOff = 0;                       // Q_A, Q_B  [2][2][128][128B]
constexpr int kKVOff = 65536;                  // 2 stages x (K [2][128][128B], V same)
constexpr int kStageBytes = 65536;
constexpr int kTileOff = kKVOff + 2 * kStageBytes;  // tile list int4[kMaxTiles]
constexpr int kBarOff = kTileOff + kMaxTiles * 16;
constexpr int kSmemBytes = kBarOff + 256 + 1024;  // + barriers, + alignment slack

struct Bars {
  uint64_t q_full;
  uint64_t kv_full[2];
  uint64_t kv_empty[2];
  uint64_t s_full[2];   // per query tile: S = Q K^T landed in TMEM
  uint64_t p_full[2];   // per query tile: P written to TMEM (128 arrivals)
  uint64_t o_done[2];   // per query tile: P V accumulated into O
  uint32_t tmem_base;
  int n_tiles;
  int abort;
};

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
// bounded wait; on expiry records the error, raises the CTA's abort flag
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity, Bars* bars,
                                          int32_t* status, int where) {
  if (mbar_try(b, parity)) return true;
  const unsigned long long t0 = now_ns();
  while (!mbar_try(b, parity)) {
    if (bars->abort || now_ns() - t0 > kTimeoutNs) {
      if (!bars->abort) report(status, RBA_ERR_TIMEOUT, kWherePrefill, where);
      atomicExch(&bars->abort, 1);
      return false;
    }
  }
  return true;
}
// bounded wait that ignores the abort flag (draining copies / MMAs at exit)
__device__ __forceinline__ void mbar_drain(uint64_t* b, uint32_t parity) {
  const unsigned long long t0 = now_ns();
  while (!mbar_try(b, parity) && now_ns() - t0 < kTimeoutNs) {
  }
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// shared-memory operand descriptor: 128B swizzle, sm100 version bits
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= uint64_t((saddr >> 4) & 0x3FFF);
  d |= uint64_t(lbo & 0x3FFF) << 16;
  d |= uint64_t(sbo & 0x3FFF) << 32;
  d |= uint64_t(1) << 46;  // descriptor version
  d |= uint64_t(2) << 61;  // SWIZZLE_128B
  return d;
}
// instruction descriptor: bf16 x bf16 -> fp32, M = 128, N = 128, K-major A,
// B K-major (b_mn = 0) or MN-major (b_mn = 1)
__host__ __device__ constexpr uint32_t idesc_bf16(int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (uint32_t(b_mn) << 16) | ((kBN >> 3) << 17) |
         ((kBM >> 4) << 24);
}
__device__ __forceinline__ void umma(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc,
                                     uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n}\n" ::"r"(
          tmem_d),
      "l"(da), "l"(db), "r"(idesc), "r"(accumulate), "r"(0u)
      : "memory");
}
// D (TMEM) += A (TMEM: M rows in lanes, K elements packed two per column) x B (smem)
__device__ __forceinline__ void umma_ta(uint32_t tmem_d, uint32_t tmem_a, uint64_t db,
                                        uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %5, %5, %5}, p;\n}\n" ::"r"(
          tmem_d),
      "r"(tmem_a), "l"(db), "r"(idesc), "r"(accumulate), "r"(0u)
      : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(
          taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,"
      "%13,%14,%15,%16};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15])
      : "memory");
}
// 2^x by the MUFU unit (PTX ex2.approx.ftz)
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// The registers of an in-flight tcgen05.ld pass through this empty asm after
// tcgen05.wait::ld, so the compiler cannot move their uses above the wait.
__device__ __forceinline__ void tmem_regs_ready(float* v) {
  asm volatile(""
               : "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]),
                 "+f"(v[6]), "+f"(v[7]), "+f"(v[8]), "+f"(v[9]), "+f"(v[10]), "+f"(v[11]),
                 "+f"(v[12]), "+f"(v[13]), "+f"(v[14]), "+f"(v[15]), "+f"(v[16]), "+f"(v[17]),
                 "+f"(v[18]), "+f"(v[19]), "+f"(v[20]), "+f"(v[21]), "+f"(v[22]), "+f"(v[23]),
                 "+f"(v[24]), "+f"(v[25]), "+f"(v[26]), "+f"(v[27]), "+f"(v[28]), "+f"(v[29]),
                 "+f"(v[30]), "+f"(v[31])
               :
               : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Tiles of keys one CTA attends: past segments (bidirectional), then its own
// chunk up to the diagonal.  int4 {map, first row, valid rows, own tile index
// (-1 for past tiles)}.
__device__ int build_tiles(const PrefillArgs& a, int c, int h, int qt, int4* tiles) {
  int n = 0;
  const int lane = threadIdx.x & 31;
  int64_t sel_rows = 0;  // staged: rows of the selected blocks (whole warp)
  if (a.staged) {
    const int32_t* sel = a.idx + (int64_t(c) * a.n_sel + (a.n_sel == 1 ? 0 : h)) * a.k;
    for (int i = lane; i < a.k; i += 32) {
      const int64_t j = sel[i];
      const int64_t lo = max(j * a.bs, int64_t(a.sink)), hi = min((j + 1) * a.bs, a.w0);
      if (j >= a.first && j < a.first + a.nc && hi > lo) sel_rows += hi - lo;
    }
    for (int o = 16; o > 0; o >>= 1) sel_rows += __shfl_xor_sync(0xffffffffu, sel_rows, o);
  }
  if (lane == 0) {
    if (a.staged) {
      // gathered past tokens: one segment of n_att rows
      const int64_t n_att = a.sink_end + (a.T - a.w0) + sel_rows;
      const int64_t row0 = (int64_t(c) * a.Hkv + h) * a.n_att_max;
      for (int64_t r = 0; r < n_att && n < kMaxTiles; r += kBN)
        tiles[n++] = make_int4(kStage, static_cast<int>(row0 + r),
                               static_cast<int>(n_att - r < kBN ? n_att - r : kBN), -1);
    } else {
      const int b = a.store_batch == 1 ? 0 : c;
      const int64_t bh_row = (int64_t(b) * a.Hkv + h) * a.cap;
      auto seg = [&](int64_t start, int64_t len) {
        for (int64_t r = 0; r < len && n < kMaxTiles; r += kBN)
          tiles[n++] = make_int4(kPool, static_cast<int>(bh_row + start + r),
                                 static_cast<int>(len - r < kBN ? len - r : kBN), -1);
      };
      seg(0, a.sink_end);
      const int32_t* sel = a.idx + (int64_t(c) * a.n_sel + (a.n_sel == 1 ? 0 : h)) * a.k;
      for (int i = 0; i < a.k; ++i) {
        const int64_t j = sel[i];
        const bool ok = j >= a.first && j < a.first + a.nc;
        if (!ok) report(a.status, RBA_ERR_BOUNDS, kWherePrefill, static_cast<int>(j));
        const int64_t lo = max(j * a.bs, int64_t(a.sink)), hi = min((j + 1) * a.bs, a.w0);
        if (ok && hi > lo) seg(lo, hi - lo);
      }
      seg(a.w0, a.T - a.w0);
    }
    const int64_t own0 = (int64_t(c) * a.Hkv + h) * a.Nq;
    for (int kt = 0; kt <= qt && n < kMaxTiles; ++kt)
      tiles[n++] = make_int4(kChunk, static_cast<int>(own0 + int64_t(kt) * kBN),
                             min(kBN, a.Nq - kt * kBN), kt);
  }
  return __shfl_sync(0xffffffffu, n, 0);
}

__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(PrefillArgs a, const __grid_constant__ CUtensorMap map_q,
                   const __grid_constant__ CUtensorMap map_pk,
                   const __grid_constant__ CUtensorMap map_pv,
                   const __grid_constant__ CUtensorMap map_sk,
                   const __grid_constant__ CUtensorMap map_sv,
                   const __grid_constant__ CUtensorMap map_ck,
                   const __grid_constant__ CUtensorMap map_cv) {
  extern __shared__ char smem_raw[];
  // 1024-byte aligned base, offset from the shared array itself (an integer
  // round trip would hide from the compiler that the pointers address shared
  // memory and turn every access into a generic one)
  char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  char* sQ = smem + kQOff;
  int4* tiles = reinterpret_cast<int4*>(smem + kTileOff);
  Bars* bars = reinterpret_cast<Bars*>(smem + kBarOff);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // grid order.  Many pairs per chunk (their causal work differs a lot): the
  // slowest index runs over the query-tile pairs, later (heavier) pairs first,
  // so the last partial wave holds light CTAs.  Else the pairs of one (head,
  // chunk) are neighbours and share its retrieved K/V in L2.
  const int pt = a.pairs_outer ? gridDim.z - 1 - blockIdx.z : blockIdx.x;
  const int hq = a.pairs_outer ? blockIdx.x : blockIdx.y;
  const int c = a.pairs_outer ? blockIdx.y : blockIdx.z;
  const int h = hq / a.G;
  // query tiles of this CTA: X = 0 (A) rows [256 pt, +128), X = 1 (B) the next 128
  const int qt0 = 2 * pt;
  const bool has_b = (qt0 + 1) * kBM < a.Nq;
  const int qt_last = has_b ? qt0 + 1 : qt0;
  // key tile j is active for query tile X unless it is an own-chunk tile past X's diagonal
  auto active = [&](const int4& t, int X) { return t.w < 0 || t.w <= qt0 + X; };

  if (warp == 8) {
    const int n = build_tiles(a, c, h, qt_last, tiles);
    if (lane == 0) {
      bars->n_tiles = n;
      bars->abort = 0;
      mbar_init(&bars->q_full, 1);
      for (int s = 0; s < 2; ++s) {
        mbar_init(&bars->kv_full[s], 1);
        mbar_init(&bars->kv_empty[s], 1);
        mbar_init(&bars->s_full[s], 1);
        mbar_init(&bars->p_full[s], 128);
        mbar_init(&bars->o_done[s], 1);
      }
      asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    }
  }
  if (warp == 9) {  // TMEM: S/P of A [0,128), of B [128,256); O_A [256,384), O_B [384,512)
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(&bars->tmem_base)),
                 "r"(512u)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;
  const int n = bars->n_tiles;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_arrive_tx(&bars->q_full, has_b ? 65536 : 32768);
      const int qrow = (c * a.Hq + hq) * a.Nq + qt0 * kBM;
      tma_load_2d(sQ, &map_q, 0, qrow, &bars->q_full);
      tma_load_2d(sQ + 16384, &map_q, 64, qrow, &bars->q_full);
      if (has_b) {
        tma_load_2d(sQ + 32768, &map_q, 0, qrow + kBM, &bars->q_full);
        tma_load_2d(sQ + 49152, &map_q, 64, qrow + kBM, &bars->q_full);
      }
      int issued = 0;
      for (int j = 0; j < n; ++j) {
        const int st = j & 1;
        if (j >= 2 && !mbar_wait(&bars->kv_empty[st], ((j >> 1) - 1) & 1, bars, a.status, 1))
          break;
        issued = j + 1;
        const int4 t = tiles[j];
        const CUtensorMap* mk = t.x == kPool ? &map_pk : t.x == kStage ? &map_sk : &map_ck;
        const CUtensorMap* mv = t.x == kPool ? &map_pv : t.x == kStage ? &map_sv : &map_cv;
        char* sK = smem + kKVOff + st * kStageBytes;
        char* sV = sK + 32768;
        mbar_arrive_tx(&bars->kv_full[st], 65536);
        tma_load_2d(sK, mk, 0, t.y, &bars->kv_full[st]);
        tma_load_2d(sK + 16384, mk, 64, t.y, &bars->kv_full[st]);
        tma_load_2d(sV, mv, 0, t.y, &bars->kv_full[st]);
        tma_load_2d(sV + 16384, mv, 64, t.y, &bars->kv_full[st]);
      }
      if (bars->abort) {  // every issued copy must have landed before the CTA exits
        mbar_drain(&bars->q_full, 0);
        for (int j = max(0, issued - 2); j < issued; ++j) mbar_drain(&bars->kv_full[j & 1], (j >> 1) & 1);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_qk = idesc_bf16(0), id_pv = idesc_bf16(1);
      bool ok = mbar_wait(&bars->q_full, 0, bars, a.status, 2);
      const int nx = has_b ? 2 : 1;
      int n_pv[2] = {0, 0};     // P V issued per query tile (o_done phases)
      int n_qk[2] = {0, 0};     // Q K^T issued per query tile (s_full phases)
      int n_commit = 0;         // commits of kv_empty
      int kv_seen = -1;         // last key tile whose K/V was waited for
      auto wait_kv = [&](int j) -> bool {
        if (j <= kv_seen) return true;
        kv_seen = j;
        return mbar_wait(&bars->kv_full[j & 1], (j >> 1) & 1, bars, a.status, 3);
      };
      auto issue_qk = [&](int j, int X) {
        const uint32_t q_base = smem_u32(sQ + X * 32768);
        const uint32_t k_base = smem_u32(smem + kKVOff + (j & 1) * kStageBytes);
#pragma unroll
        for (int kk = 0; kk < kHD / 16; ++kk) {
          const uint64_t da = sdesc(q_base + (kk >> 2) * 16384 + (kk & 3) * 32, 1, 64);
          const uint64_t db = sdesc(k_base + (kk >> 2) * 16384 + (kk & 3) * 32, 1, 64);
          umma(tmem + X * 128, da, db, id_qk, kk > 0 ? 1u : 0u);
        }
        umma_commit(&bars->s_full[X]);
        ++n_qk[X];
      };
      // first tile: S for both query tiles
      if (ok && n > 0) ok = wait_kv(0);
      for (int X = 0; X < nx && ok; ++X)
        if (active(tiles[0], X)) issue_qk(0, X);
      for (int j = 0; j < n && ok; ++j) {
        const int4 t = tiles[j];
        const uint32_t v_base = smem_u32(smem + kKVOff + (j & 1) * kStageBytes + 32768);
        int last_x = -1;
        for (int X = 0; X < nx; ++X)
          if (active(t, X)) last_x = X;
        for (int X = 0; X < nx && ok; ++X) {
          if (!active(t, X)) continue;
          // O_X += P_X V once the softmax has written P_X
          if (!mbar_wait(&bars->p_full[X], n_pv[X] & 1, bars, a.status, 5)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            // A = P (TMEM, 16 keys = 8 columns per step); B = V (MN-major)
            const uint64_t db = sdesc(v_base + kk * 2048, 1024, 64);
            umma_ta(tmem + 256 + X * 128, tmem + X * 128 + kk * 8, db, id_pv,
                    (n_pv[X] > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&bars->o_done[X]);
          ++n_pv[X];
          if (X == last_x) {
            umma_commit(&bars->kv_empty[j & 1]);
            ++n_commit;
          }
          // next S_X overwrites P_X: after this P V has completed
          if (j + 1 < n && active(tiles[j + 1], X)) {
            if (!wait_kv(j + 1) ||
                !mbar_wait(&bars->o_done[X], (n_pv[X] - 1) & 1, bars, a.status, 4)) {
              ok = false;
              break;
            }
            tc_fence_after();
            issue_qk(j + 1, X);
          }
        }
      }
      if (bars->abort) {  // no MMA may still be running when TMEM is freed
        for (int X = 0; X < nx; ++X) {
          if (n_qk[X] > 0) mbar_drain(&bars->s_full[X], (n_qk[X] - 1) & 1);
          if (n_pv[X] > 0) mbar_drain(&bars->o_done[X], (n_pv[X] - 1) & 1);
        }
      }
      (void)n_commit;
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ softmax
    const int X = warp >> 2;                       // query tile of this warpgroup
    const int r = tid & 127;                       // query row within the tile (TMEM lane)
    const int qpos = (qt0 + X) * kBM + r;
    const uint32_t lane_off = uint32_t((warp & 3) * 32) << 16;
    const uint32_t s_col = X * 128, o_col = 256 + X * 128;
    float m = -INFINITY, l = 0.f;  // running max (scaled log2 units) and sum
    bool ok = X == 0 || has_b;
    int n_s = 0;
    for (int j = 0; j < n && ok; ++j) {
      const int4 t = tiles[j];
      if (!active(t, X)) continue;
      if (!__all_sync(0xffffffffu, mbar_wait(&bars->s_full[X], n_s & 1, bars, a.status, 7))) {
        ok = false;
        break;
      }
      ++n_s;
      tc_fence_after();
      const int valid = t.z;
      const int lim = t.w >= 0 ? min(valid, qpos - t.w * kBN + 1) : valid;  // keys [0, lim) visible
      // pass 1: the row's max over its visible keys (two chunks in flight per wait)
      float mt = -INFINITY;
#pragma unroll 1
      for (int q8 = 0; q8 < 4; q8 += 2) {
        float va[32], vb[32];
        tmem_ld32(tmem + lane_off + s_col + q8 * 32, va);
        tmem_ld32(tmem + lane_off + s_col + (q8 + 1) * 32, vb);
        tmem_wait_ld();
        tmem_regs_ready(va);
        tmem_regs_ready(vb);
        if (lim >= (q8 + 2) * 32) {
          float m2 = mt;
#pragma unroll
          for (int x = 0; x < 32; ++x) {  // two chains
            mt = fmaxf(mt, va[x]);
            m2 = fmaxf(m2, vb[x]);
          }
          mt = fmaxf(mt, m2);
        } else {
#pragma unroll
          for (int x = 0; x < 32; ++x) {
            if (q8 * 32 + x < lim) mt = fmaxf(mt, va[x]);
            if ((q8 + 1) * 32 + x < lim) mt = fmaxf(mt, vb[x]);
          }
        }
      }
      const float m_new = fmaxf(m, mt * a.scale_log2);
      const bool rescale = m_new > m + 8.f;  // lazy: also when m is still -inf
      const float m_use = rescale ? m_new : m;
      const float corr = (rescale && m != -INFINITY) ? exp2f(m - m_use) : 1.f;
      // O rows whose max grew are rescaled; the warp loads and stores together
      // (O_X is idle: the next S_X was issued only after the last P_X V)
      if (__any_sync(0xffffffffu, corr != 1.f)) {
#pragma unroll 1
        for (int q4 = 0; q4 < 4; ++q4) {
          float o[32];
          tmem_ld32(tmem + lane_off + o_col + q4 * 32, o);
          tmem_wait_ld();
          tmem_regs_ready(o);
#pragma unroll
          for (int x = 0; x < 32; ++x) o[x] *= corr;
          tmem_st32(tmem + lane_off + o_col + q4 * 32, o);
        }
      }
      // pass 2: P = exp2(scale s - m), bf16 pairs stored over the S columns
      // (pairs through f32x2 FMA / add; masks only where keys are cut off)
      const float neg_m = m_use == -INFINITY ? 0.f : -m_use;
      const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
      const float2 nm2 = make_float2(neg_m, neg_m);
      const bool whole = lim >= kBN && m_use != -INFINITY;  // no key of this tile is masked
      float2 rs2[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                       make_float2(0.f, 0.f)};  // four independent sum chains
      // chunk q4 + 1 is loaded while chunk q4 is exponentiated (P chunk q4 goes to
      // columns [16 q4, 16 q4 + 16), below every chunk still to be read)
      float vbuf[2][32];
      tmem_ld32(tmem + lane_off + s_col, vbuf[0]);
      tmem_wait_ld();
      tmem_regs_ready(vbuf[0]);
#pragma unroll
      for (int q4 = 0; q4 < 4; ++q4) {
        const float* v = vbuf[q4 & 1];
        if (q4 < 3) tmem_ld32(tmem + lane_off + s_col + (q4 + 1) * 32, vbuf[(q4 + 1) & 1]);
        uint32_t pk[16];
        if (whole) {
#pragma unroll
          for (int x = 0; x < 32; x += 2) {
            const float2 e = __ffma2_rn(make_float2(v[x], v[x + 1]), sc2, nm2);
            const float2 pp = make_float2(ex2_approx(e.x), ex2_approx(e.y));
            rs2[(x >> 1) & 3] = __fadd2_rn(rs2[(x >> 1) & 3], pp);
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(pp.x, pp.y);
            pk[x / 2] = *reinterpret_cast<const uint32_t*>(&b2);
          }
        } else {
#pragma unroll
          for (int x = 0; x < 32; x += 2) {
            const bool in0 = q4 * 32 + x < lim && m_use != -INFINITY;
            const bool in1 = q4 * 32 + x + 1 < lim && m_use != -INFINITY;
            const float2 e = __ffma2_rn(make_float2(v[x], v[x + 1]), sc2, nm2);
            const float2 pp = make_float2(in0 ? ex2_approx(e.x) : 0.f, in1 ? ex2_approx(e.y) : 0.f);
            rs2[(x >> 1) & 3] = __fadd2_rn(rs2[(x >> 1) & 3], pp);
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(pp.x, pp.y);
            pk[x / 2] = *reinterpret_cast<const uint32_t*>(&b2);
          }
        }
        tmem_st16(tmem + lane_off + s_col + q4 * 16, pk);
        if (q4 < 3) {
          tmem_wait_ld();
          tmem_regs_ready(vbuf[(q4 + 1) & 1]);
        }
      }
      tmem_wait_st();
      const float2 r01 = __fadd2_rn(rs2[0], rs2[1]), r23 = __fadd2_rn(rs2[2], rs2[3]);
      const float2 r03 = __fadd2_rn(r01, r23);
      const float rs = r03.x + r03.y;
      l = l * corr + rs;
      m = m_use;
      tc_fence_before();
      mbar_arrive(&bars->p_full[X]);
    }
    // final: O / l into the output once the last P V has completed
    if (ok && n_s > 0 &&
        __all_sync(0xffffffffu, mbar_wait(&bars->o_done[X], (n_s - 1) & 1, bars, a.status, 9))) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
      float* orow = a.out + ((int64_t(c) * a.Hq + hq) * a.Nq + qpos) * a.od;
#pragma unroll 1
      for (int q4 = 0; q4 < 4; ++q4) {
        float o[32];
        tmem_ld32(tmem + lane_off + o_col + q4 * 32, o);  // whole warp, rows past Nq too
        tmem_wait_ld();
        tmem_regs_ready(o);
        if (qpos < a.Nq) {
#pragma unroll
          for (int x = 0; x < 32; x += 4)  // (od is a multiple of 4: whole float4s)
            if (q4 * 32 + x < a.od)
              *reinterpret_cast<float4*>(orow + q4 * 32 + x) =
                  make_float4(o[x] * inv, o[x + 1] * inv, o[x + 2] * inv, o[x + 3] * inv);
        }
      }
      if (qpos < a.Nq && a.lse != nullptr)
        a.lse[(int64_t(c) * a.Hq + hq) * a.Nq + qpos] =
            l > 0.f ? (m + log2f(l)) * 0.6931471805599453f : -INFINITY;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(512u)
                 : "memory");
  }
}

// Gathers the attended past tokens of each (chunk, kv head) into a
// contiguous staging buffer [n_chunks][Hkv][n_att_max][D] (K and V).
__global__ void gather_kernel(PrefillArgs a, const __nv_bfloat16* __restrict__ K,
                              const __nv_bfloat16* __restrict__ V, __nv_bfloat16* __restrict__ SK,
                              __nv_bfloat16* __restrict__ SV) {
  extern __shared__ int gsm[];
  const int c = blockIdx.y, h = blockIdx.z;
  int* start = gsm;             // [k + 2]
  int* pref = gsm + (a.k + 2);  // [k + 3]
  const int nseg = a.k + 2;
  const int32_t* sel = a.idx + (int64_t(c) * a.n_sel + (a.n_sel == 1 ? 0 : h)) * a.k;
  for (int i = threadIdx.x; i < nseg; i += blockDim.x) {
    int64_t s0, len;
    if (i == 0) {
      s0 = 0;
      len = a.sink_end;
    } else if (i == nseg - 1) {
      s0 = a.w0;
      len = a.T - a.w0;
    } else {
      const int64_t j = sel[i - 1];
      const bool ok = j >= a.first && j < a.first + a.nc;
      const int64_t lo = max(j * a.bs, int64_t(a.sink)), hi = min((j + 1) * a.bs, a.w0);
      s0 = lo;
      len = ok && hi > lo ? hi - lo : 0;
    }
    start[i] = static_cast<int>(s0);
    pref[i] = static_cast<int>(len);
  }
  __syncthreads();
  if (threadIdx.x == 0) {  // exclusive prefix (k + 2 entries)
    int run = 0;
    for (int i = 0; i < nseg; ++i) {
      const int x = pref[i];
      pref[i] = run;
      run += x;
    }
    pref[nseg] = run;
  }
  __syncthreads();
  const int total = pref[nseg];
  const int b = a.store_batch == 1 ? 0 : c;
  const int64_t src0 = (int64_t(b) * a.Hkv + h) * a.cap;
  const int64_t dst0 = (int64_t(c) * a.Hkv + h) * a.n_att_max;
  // 16 lanes per row (16 x 16 B = 256 B)
  const int sub = threadIdx.x & 15;
  for (int v = blockIdx.x * (blockDim.x / 16) + threadIdx.x / 16; v < total;
       v += gridDim.x * (blockDim.x / 16)) {
    int lo = 0, hi = nseg - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pref[mid] <= v) lo = mid; else hi = mid - 1;
    }
    const int64_t tok = src0 + start[lo] + (v - pref[lo]);
    const uint4* ks = reinterpret_cast<const uint4*>(K + tok * kHD) + sub;
    const uint4* vs = reinterpret_cast<const uint4*>(V + tok * kHD) + sub;
    reinterpret_cast<uint4*>(SK + (dst0 + v) * kHD)[sub] = *ks;
    reinterpret_cast<uint4*>(SV + (dst0 + v) * kHD)[sub] = *vs;
  }
}

// rows of D bf16 (dense) -> rows of kHD with zero padding, in 32-bit words
__global__ void pad_rows_kernel(const uint32_t* __restrict__ src, uint32_t* __restrict__ dst,
                                int64_t rows, int src_words) {
  constexpr int kDstWords = kHD / 2;
  const int64_t total = rows * kDstWords;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = i / kDstWords;
    const int w = static_cast<int>(i - r * kDstWords);
    dst[i] = w < src_words ? src[r * src_words + w] : 0u;
  }
}

// [rows][128] bf16 matrix, 128-byte-swizzled boxes of 64 columns x 128 rows
bool make_map(CUtensorMap* m, const void* base, int64_t rows) {
  return make_tmap_bf16(m, base, rows, kHD, 128);
}

struct Plan {
  bool staged;
  int n_att_max;
  size_t staged_bytes;  // staging buffers of the gathered past K and V
  bool padded;          // head dim below kHD: Q and the chunk's K/V padded to kHD columns
  size_t q_pad, kv_pad; // bytes of the padded Q and of each padded chunk K / V
  size_t ws_bytes;
};

Plan plan(const rba_store* st, const Geometry& g, int n_chunks, int chunk_len, int k) {
  Plan p;
  const rba_store_desc& d = st->d;
  const int64_t n_att = int64_t(g.sink_end) + (g.T - g.w0) + int64_t(k) * d.block_size;
  const int64_t direct_tiles = (g.sink_end + kBN - 1) / kBN +
                               int64_t(k) * ((d.block_size + kBN - 1) / kBN + 1) +
                               (g.T - g.w0 + kBN - 1) / kBN;
  p.staged = d.block_size < kBN || direct_tiles > kMaxTiles / 2;
  p.n_att_max = static_cast<int>(n_att);
  p.staged_bytes =
      p.staged ? align_up(size_t(n_chunks) * d.n_kv_heads * n_att * kHD * 2, 256) * 2 : 0;
  p.padded = d.head_dim != kHD;
  p.q_pad = p.padded ? align_up(size_t(n_chunks) * d.n_q_heads * chunk_len * kHD * 2, 256) : 0;
  p.kv_pad = p.padded ? align_up(size_t(n_chunks) * d.n_kv_heads * chunk_len * kHD * 2, 256) : 0;
  p.ws_bytes = p.staged_bytes + p.q_pad + 2 * p.kv_pad;
  return p;
}

}  // namespace
}  // namespace rba

extern "C" {

rba_status rba_attend_prefill(const rba_store* st, const void* q, int32_t n_chunks,
                              int32_t chunk_len, const int32_t* idx, int32_t n_sel, int32_t k,
                              int64_t T, int32_t sink, int32_t window, const void* chunk_k,
                              const void* chunk_v, float scale, float* out, float* lse,
                              void* workspace, size_t ws_bytes, cudaStream_t stream) {
  using namespace rba;
  if (st == nullptr || q == nullptr || out == nullptr || chunk_k == nullptr ||
      chunk_v == nullptr || n_chunks <= 0 || chunk_len <= 0 || k < 0)
    return RBA_ERR_INVALID_ARG;
  const rba_store_desc& d = st->d;
  // head dims below kHD run on kHD-wide tiles: pools are held with rows of kHD
  // elements (zero padding), Q and the chunk's K/V are padded into the workspace
  if (d.dtype != RBA_BF16 || st->pitch != kHD) return RBA_ERR_UNSUPPORTED;
  if (d.batch != 1 && d.batch != n_chunks) return RBA_ERR_INVALID_ARG;
  if (n_sel != 1 && n_sel != d.n_kv_heads) return RBA_ERR_INVALID_ARG;
  if (k > 0 && idx == nullptr) return RBA_ERR_INVALID_ARG;
  Geometry g;
  rba_status s = geometry(st, T, sink, window, &g);
  if (s != RBA_OK) return s;
  if (k > g.nc) return RBA_ERR_INVALID_ARG;
  const Plan p = plan(st, g, n_chunks, chunk_len, k);
  const int64_t own_tiles = (chunk_len + kBN - 1) / kBN;
  if ((int64_t(p.n_att_max) + kBN - 1) / kBN + own_tiles > kMaxTiles) return RBA_ERR_UNSUPPORTED;
  if (int64_t(n_chunks) * d.n_q_heads * chunk_len >= (int64_t(1) << 31) ||
      int64_t(d.batch) * d.n_kv_heads * d.capacity_tokens >= (int64_t(1) << 31))
    return RBA_ERR_UNSUPPORTED;
  if (ws_bytes < p.ws_bytes || (p.ws_bytes > 0 && workspace == nullptr)) return RBA_ERR_WORKSPACE;

  PrefillArgs a;
  a.idx = idx;
  a.out = out;
  a.lse = lse;
  a.status = st->status;
  a.cap = d.capacity_tokens;
  a.T = g.T;
  a.w0 = g.w0;
  a.Hq = d.n_q_heads;
  a.Hkv = d.n_kv_heads;
  a.G = d.n_q_heads / d.n_kv_heads;
  a.Nq = chunk_len;
  a.n_chunks = n_chunks;
  a.n_sel = n_sel;
  a.k = k;
  a.bs = d.block_size;
  a.sink = g.sink;
  a.sink_end = g.sink_end;
  a.first = g.first;
  a.nc = g.nc;
  a.store_batch = d.batch;
  a.staged = p.staged ? 1 : 0;
  a.n_att_max = p.n_att_max;
  a.od = d.head_dim;
  a.scale_log2 = scale * 1.4426950408889634f;

  __nv_bfloat16* SK = nullptr;
  __nv_bfloat16* SV = nullptr;
  if (p.staged) {
    SK = static_cast<__nv_bfloat16*>(workspace);
    SV = reinterpret_cast<__nv_bfloat16*>(static_cast<char*>(workspace) + p.staged_bytes / 2);
    const size_t gsmem = size_t(2 * k + 5) * sizeof(int);
    if (gsmem > 200 * 1024) return RBA_ERR_UNSUPPORTED;
    RBA_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(gather_kernel), gsmem));
    const int rows_per_block = 256 / 16;
    int gx = (p.n_att_max + rows_per_block - 1) / rows_per_block;
    if (gx > 64) gx = 64;
    gather_kernel<<<dim3(gx, n_chunks, d.n_kv_heads), 256, gsmem, stream>>>(
        a, static_cast<const __nv_bfloat16*>(st->k), static_cast<const __nv_bfloat16*>(st->v), SK,
        SV);
    RBA_LAUNCH_CHECK();
  }
  CUtensorMap mq, mpk, mpv, msk, msv, mck, mcv;
  const int64_t pool_rows = int64_t(d.batch) * d.n_kv_heads * d.capacity_tokens;
  const int64_t chunk_rows = int64_t(n_chunks) * d.n_kv_heads * chunk_len;
  if (p.padded) {
    char* base = static_cast<char*>(workspace) + p.staged_bytes;
    void* qp = base;
    void* kp = base + p.q_pad;
    void* vp = base + p.q_pad + p.kv_pad;
    const int64_t q_rows = int64_t(n_chunks) * d.n_q_heads * chunk_len;
    const int words = d.head_dim / 2;
    auto pad = [&](const void* src, void* dst, int64_t rows) {
      int64_t grid = (rows * (kHD / 2) + 255) / 256;
      if (grid > int64_t(num_sms()) * 16) grid = int64_t(num_sms()) * 16;
      pad_rows_kernel<<<static_cast<int>(grid), 256, 0, stream>>>(
          static_cast<const uint32_t*>(src), static_cast<uint32_t*>(dst), rows, words);
    };
    pad(q, qp, q_rows);
    pad(chunk_k, kp, chunk_rows);
    pad(chunk_v, vp, chunk_rows);
    RBA_LAUNCH_CHECK();
    q = qp;
    chunk_k = kp;
    chunk_v = vp;
  }
  if (!make_map(&mq, q, int64_t(n_chunks) * d.n_q_heads * chunk_len) ||
      !make_map(&mpk, st->k, pool_rows) || !make_map(&mpv, st->v, pool_rows) ||
      !make_map(&mck, chunk_k, chunk_rows) || !make_map(&mcv, chunk_v, chunk_rows))
    return RBA_ERR_CUDA;
  if (p.staged) {
    const int64_t srows = int64_t(n_chunks) * d.n_kv_heads * p.n_att_max;
    if (!make_map(&msk, SK, srows) || !make_map(&msv, SV, srows)) return RBA_ERR_CUDA;
  } else {
    msk = mpk;
    msv = mpv;
  }
  RBA_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(prefill_kernel), kSmemBytes));
  const unsigned n_pairs = static_cast<unsigned>((chunk_len + 2 * kBM - 1) / (2 * kBM));
  a.pairs_outer = n_pairs > 2 ? 1 : 0;
  const dim3 grid = a.pairs_outer
                        ? dim3(static_cast<unsigned>(d.n_q_heads),
                               static_cast<unsigned>(n_chunks), n_pairs)
                        : dim3(n_pairs, static_cast<unsigned>(d.n_q_heads),
                               static_cast<unsigned>(n_chunks));
  prefill_kernel<<<grid, kThreads, kSmemBytes, stream>>>(a, mq, mpk, mpv, msk, msv, mck, mcv);
  RBA_LAUNCH_CHECK();
  return RBA_OK;
}

size_t rba_attend_prefill_workspace_size(const rba_store* st, int32_t n_chunks,
                                         int32_t chunk_len, int32_t n_sel, int32_t k, int64_t T,
                                         int32_t sink, int32_t window) {
  using namespace rba;
  (void)n_sel;
  rba::Geometry g;
  if (st == nullptr || n_chunks <= 0 || k < 0 || geometry(st, T, sink, window, &g) != RBA_OK)
    return 0;
  return plan(st, g, n_chunks, chunk_len, k).ws_bytes;
}

}  // extern "C"
