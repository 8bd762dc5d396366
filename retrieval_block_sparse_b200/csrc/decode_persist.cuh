// Device helpers shared by the persistent decode kernels (the whole-block
// tensor-core attention kernel of the three-kernel decode step and the
// one-launch decode step): mbarrier and bulk-copy primitives with bounded
// waits, the shared-memory bookkeeping of a stage ring, and the mma.sync
// tile consumer of 128-byte-swizzled K/V tiles.
#pragma once

#include <cuda.h>

#include "attend_impl.cuh"

namespace rba {
namespace {

constexpr int kMaxStages = 6;
constexpr unsigned long long kTimeoutNs = 2000000000ull;  // default bound of every wait

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
// False when the CTA is aborting or the wait ran out after limit_ns (then
// reported as RBA_ERR_TIMEOUT with `kernel` and `where`, and the abort flag
// set).
__device__ __forceinline__ bool mbar_wait(uint64_t* b, uint32_t parity, volatile int* abort_flag,
                                          int32_t* status, int where,
                                          unsigned long long limit_ns = kTimeoutNs,
                                          int kernel = kWhereFused) {
  bool ok = mbar_try(b, parity);
  if (__all_sync(0xffffffffu, ok)) return true;
  const unsigned long long t0 = now_ns();
  while (true) {
    if (!ok) ok = mbar_try(b, parity);
    if (__all_sync(0xffffffffu, ok)) return true;
    if (__any_sync(0xffffffffu, *abort_flag != 0)) return false;
    if (__shfl_sync(0xffffffffu, now_ns() - t0 > limit_ns, 0)) {
      if ((threadIdx.x & 31) == 0) {
        report(status, RBA_ERR_TIMEOUT, kernel, where);
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
// barrier of the NCT compute threads only (warp 0 never joins it)
template <int NCT>
__device__ __forceinline__ void compute_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(NCT) : "memory");
}
__device__ __forceinline__ int ctid() { return static_cast<int>(threadIdx.x) - 32; }


struct __align__(16) Meta {
  int nrows;
  int pad[3];
};

// Small shared variables after the stage ring, the warp states and the
// selection layout (MISC bytes): full[kMaxStages], empty[kMaxStages] (mbarriers),
// meta[kMaxStages], then ints: [0..16) flags, [16..20) abort flag, [20..148)
// floats (merge factors and maxima), [148..150) the merge mbarrier.
struct MiscLayout {
  uint64_t* full;
  uint64_t* empty;
  Meta* meta;
  int* s_misc;
  volatile int* abort_flag;
  float* s_f;         // [128]: fac [G * NW] (<= 112), gmax [G] at +112
  uint64_t* merge_bar;
  __device__ explicit MiscLayout(char* misc) {
    full = reinterpret_cast<uint64_t*>(misc);
    empty = full + kMaxStages;
    meta = reinterpret_cast<Meta*>(empty + kMaxStages);
    s_misc = reinterpret_cast<int*>(meta + kMaxStages);
    abort_flag = s_misc + 16;
    s_f = reinterpret_cast<float*>(s_misc + 20);
    merge_bar = reinterpret_cast<uint64_t*>(s_misc + 148);
  }
};
constexpr int kMiscBytes = 1024;
static_assert(2 * kMaxStages * 8 + kMaxStages * 16 + 150 * 4 <= kMiscBytes, "misc layout");

constexpr int kMW = 8;                 // compute warps: two groups of four
constexpr int kMGW = 4;                // warps per tile (16 rows each)
constexpr int kMCT = kMW * 32;         // compute threads
constexpr int kMFT = kMCT + 32;        // + the staging warp
constexpr int kMTT = kMGW * 16;        // rows per tile
constexpr int kHalfBytes = kMTT * 128; // one 64-column half of a tile (1024-byte multiple)

enum : int { kPieceFlush = 1 };        // meta flag: last piece of this CTA's part of the head

template <int D>
struct MmaGeo {
  static constexpr int NH = D / 64;                  // 64-column halves
  static constexpr int VOFF = NH * kHalfBytes;
  static constexpr int STAGE = 2 * NH * kHalfBytes;  // K halves, then V halves
  static constexpr int TX = STAGE;                   // bytes each stage's copies deliver
};


__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}
__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
#pragma nv_diag_suppress 550  // the discarded accumulators of mma_rows8
// d[0..1] += A . B for the rows lane/4 of a 16x8 tile; A rows 8..15 are zero
// (a1 = a3 = 0) and their accumulators are not kept.
__device__ __forceinline__ void mma_rows8(float (&d)[2], uint32_t a0, uint32_t a2, uint32_t b0,
                                          uint32_t b1) {
  float d2, d3;  // rows 8..15: discarded
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%5}, "
      "{%7,%8}, {%0,%1,%9,%9};"
      : "+f"(d[0]), "+f"(d[1]), "=f"(d2), "=f"(d3)
      : "r"(a0), "r"(0u), "r"(a2), "r"(b0), "r"(b1), "f"(0.f));
}
__device__ __forceinline__ float ex2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ uint32_t pack_bf16(float lo_elem, float hi_elem) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo_elem, hi_elem);
  return *reinterpret_cast<const uint32_t*>(&v);
}
// byte offset of 16-byte chunk ch of row r in a 128-byte-swizzled half tile
__device__ __forceinline__ uint32_t swz(int r, int ch) {
  return uint32_t(r * 128 + ((ch ^ (r & 7)) << 4));
}

// One warp's softmax state: head hq = lane/4 (q heads >= G are padding).
// The warp's Q fragments live in its own shared-memory copy `qf`
// ([KS][32 lanes] x (a0, a2)), read back for every tile.
template <int D>
struct MmaState {
  static constexpr int KS = D / 16;  // k-steps of Q.K^T
  static constexpr int NTD = D / 8;  // n-tiles of P.V
  const uint2* qf;                   // this warp's Q fragments
  float m;                           // running max of head hq (log2 units)
  float l;                           // sum of this lane's weights of head hq
  float o[NTD][2];                   // O[hq][8 nt + 2 (lane % 4) + {0, 1}]
};

template <int D, int G>
__device__ __forceinline__ void mma_load_q(const AttendArgs& at, int bh, MmaState<D>& st,
                                           uint2* qf) {
  const int lane = threadIdx.x & 31, hq = lane >> 2, c = (lane & 3) * 2;
  const int b = bh / at.Hkv, h = bh % at.Hkv;
  // q rows are at.qd long (even); columns past it count as zero
  const __nv_bfloat16* qp =
      static_cast<const __nv_bfloat16*>(at.q) + (int64_t(b) * at.Hq + h * G + hq) * at.qd + c;
  auto word = [&](int col) -> uint32_t {  // q columns col + c, col + c + 1
    return hq < G && col + c < at.qd ? __ldg(reinterpret_cast<const uint32_t*>(qp + col)) : 0u;
  };
  // (each lane reads back only its own entries)
#pragma unroll
  for (int ks = 0; ks < MmaState<D>::KS; ++ks)
    qf[ks * 32 + lane] = make_uint2(word(ks * 16), word(ks * 16 + 8));
  st.qf = qf;
  st.m = -INFINITY;
  st.l = 0.f;
#pragma unroll
  for (int nt = 0; nt < MmaState<D>::NTD; ++nt) st.o[nt][0] = st.o[nt][1] = 0.f;
}

// keeps the bf16 halves of b whose rows (lo half: row, hi half: row + 1) are valid
__device__ __forceinline__ uint32_t keep_rows(uint32_t b, int row, int nvalid) {
  const uint32_t lo = row < nvalid ? 0x0000ffffu : 0u;
  const uint32_t hi = row + 1 < nvalid ? 0xffff0000u : 0u;
  return b & (lo | hi);
}

// Rows [16 wr, 16 wr + 16) of the tile at shared address `stage` (nvalid rows
// valid; the rest hold whatever the boxes brought and get zero weight).
template <int D>
__device__ __forceinline__ void mma_consume(uint32_t stage, int nvalid, MmaState<D>& st, int wr,
                                            float scale_log2) {
  using Geo = MmaGeo<D>;
  constexpr int KS = MmaState<D>::KS, NTD = MmaState<D>::NTD;
  const int lane = threadIdx.x & 31;
  const int r0 = wr * 16;
  if (r0 >= nvalid) return;
  // S^T: n-tile nt holds rows r0 + 8 nt + [0, 8).  K-steps ks, ks + 1 cover
  // columns [16 ks, 16 ks + 32): half ks / 4, chunks 2 (ks % 4) + [0, 4).
  float sc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
  for (int ks = 0; ks < KS; ks += 2) {
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      uint32_t bk[4];  // b0, b1 of k-steps ks and ks + 1
      const int r = r0 + 8 * nt + (lane & 7);
      ldsm_x4(bk, stage + (ks / 4) * kHalfBytes + swz(r, 2 * (ks % 4) + (lane >> 3)));
      const uint2 qa = st.qf[ks * 32 + lane], qb = st.qf[(ks + 1) * 32 + lane];
      mma_rows8(sc[nt], qa.x, qa.y, bk[0], bk[1]);
      mma_rows8(sc[nt], qb.x, qb.y, bk[2], bk[3]);
    }
  }
  // this lane's rows: r0 + c + {0, 1} (n-tile 0) and r0 + 8 + c + {0, 1} (n-tile 1)
  const int c = (lane & 3) * 2;
  float x[4];
#pragma unroll
  for (int nt = 0; nt < 2; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int row = r0 + 8 * nt + c + e;
      x[nt * 2 + e] = row < nvalid ? sc[nt][e] * scale_log2 : -INFINITY;
    }
  float mt = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
  mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 1));
  mt = fmaxf(mt, __shfl_xor_sync(0xffffffffu, mt, 2));
  if (mt > st.m) {  // per head (lanes differ); no collective inside
    const float cf = ex2_fast(st.m - mt);  // 0 while the state is empty
    st.l *= cf;
#pragma unroll
    for (int nt = 0; nt < NTD; ++nt) {
      st.o[nt][0] *= cf;
      st.o[nt][1] *= cf;
    }
    st.m = mt;
  }
  const float mu = st.m == -INFINITY ? 0.f : st.m;
  float p[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) p[e] = ex2_fast(x[e] - mu);
  st.l += (p[0] + p[1]) + (p[2] + p[3]);
  // A fragments of P^T: a0 = rows c, c+1 (n-tile 0), a2 = rows 8+c, 9+c (n-tile 1)
  const uint32_t h0 = pack_bf16(p[0], p[1]), h2 = pack_bf16(p[2], p[3]);
  const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&h0));
  const float2 f2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&h2));
  const uint32_t l0 = pack_bf16(p[0] - f0.x, p[1] - f0.y);
  const uint32_t l2 = pack_bf16(p[2] - f2.x, p[3] - f2.y);
  // V (transposed): n-tiles nt, nt + 1 cover columns [8 nt, 8 nt + 16): half
  // nt / 8, chunks nt % 8 + {0, 1}.  Rows past nvalid may hold non-finite
  // values from the boxes: a partial slice masks them out of its fragments.
  const bool partial = r0 + 16 > nvalid;
  const int vr = r0 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
  for (int nt = 0; nt < NTD; nt += 2) {
    uint32_t bv[4];  // b0, b1 of n-tiles nt and nt + 1
    ldsm_x4_t(bv, stage + Geo::VOFF + (nt / 8) * kHalfBytes + swz(vr, (nt % 8) + (lane >> 4)));
    if (partial) {
      bv[0] = keep_rows(bv[0], r0 + c, nvalid);
      bv[1] = keep_rows(bv[1], r0 + 8 + c, nvalid);
      bv[2] = keep_rows(bv[2], r0 + c, nvalid);
      bv[3] = keep_rows(bv[3], r0 + 8 + c, nvalid);
    }
    mma_rows8(st.o[nt], h0, h2, bv[0], bv[1]);
    mma_rows8(st.o[nt], l0, l2, bv[0], bv[1]);
    mma_rows8(st.o[nt + 1], h0, h2, bv[2], bv[3]);
    mma_rows8(st.o[nt + 1], l0, l2, bv[2], bv[3]);
  }
}

}  // namespace
}  // namespace rba
