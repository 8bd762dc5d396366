// Internal helpers shared by the rba kernels (device and host side).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <mutex>

#include <cuda.h>

#include "rba.h"

struct rba_store {
  rba_store_desc d;
  int32_t pitch;          // elements per row of the K/V and representation pools (64 or 128)
  void* k;
  void* v;
  void* rep;
  int32_t* rep_pos;
  int32_t* status;
  int64_t cap_blocks;
  int32_t score_reduce;   // rba_score_reduce: how a block's r representative keys combine
  unsigned long long wait_ns;  // bound of the one-launch decode step's waits (ns)
  int32_t one_launch;     // rba_decode_step may use the one-launch path (0: three kernels)
  // tensor maps of the K and V pools in 64-row boxes (the whole-block decode
  // kernels), encoded once on first use: the pools never move
  mutable std::once_flag tmap_once;
  mutable bool tmap_ok = false;
  mutable CUtensorMap kmap64 = {}, vmap64 = {};
};

namespace rba {

// ---------------------------------------------------------------------------
// status word: [0] first error code, [1] where, [2] detail, [3] error count

enum Where : int32_t {
  kWhereAttend = 1,
  kWhereScore = 2,
  kWhereTopk = 3,
  kWhereMemorize = 4,
  kWherePrefill = 5,
  kWhereFused = 6,
  kWhereMemory = 7,
  kWhereStep = 8,
};

__device__ __forceinline__ void report(int32_t* status, int32_t code, int32_t where,
                                       int32_t detail) {
  if (status == nullptr) return;
  if (atomicCAS(status, 0, code) == 0) {
    status[1] = where;
    status[2] = detail;
  }
  atomicAdd(status + 3, 1);
}

// ---------------------------------------------------------------------------
// element types

template <typename T> struct Elem;
template <> struct Elem<float> {
  static constexpr int kPerVec = 4;  // elements per 16-byte vector
  __device__ __forceinline__ static float to_f32(float x) { return x; }
};
template <> struct Elem<__nv_bfloat16> {
  static constexpr int kPerVec = 8;
  __device__ __forceinline__ static float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }
};

// 16-byte vector -> floats (exact widening)
__device__ __forceinline__ void unpack(const uint4& u, float* f, float) {
  f[0] = __uint_as_float(u.x);
  f[1] = __uint_as_float(u.y);
  f[2] = __uint_as_float(u.z);
  f[3] = __uint_as_float(u.w);
}
__device__ __forceinline__ void unpack(const uint4& u, float* f, __nv_bfloat16) {
  f[0] = __uint_as_float(u.x << 16);
  f[1] = __uint_as_float(u.x & 0xffff0000u);
  f[2] = __uint_as_float(u.y << 16);
  f[3] = __uint_as_float(u.y & 0xffff0000u);
  f[4] = __uint_as_float(u.z << 16);
  f[5] = __uint_as_float(u.z & 0xffff0000u);
  f[6] = __uint_as_float(u.w << 16);
  f[7] = __uint_as_float(u.w & 0xffff0000u);
}

// streaming 16-byte global load (read once: do not keep in L1)
__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

// ---------------------------------------------------------------------------
// top-k keys: larger key = better (higher score, then lower position)

// (straight-line arithmetic: a branch on the loaded value would make every
// load in an unrolled loop complete before the next one issues)
__device__ __forceinline__ uint32_t ordered_f32(float f) {
  uint32_t u = __float_as_uint(f);
  u &= 0u - uint32_t((u << 1) != 0u);  // -0 == +0
  const uint32_t flip = uint32_t(int32_t(u) >> 31) | 0x80000000u;  // negative: all bits
  return u ^ flip;
}
__device__ __forceinline__ uint64_t topk_key(float s, uint32_t pos) {
  return (static_cast<uint64_t>(ordered_f32(s)) << 32) | static_cast<uint32_t>(0xffffffffu - pos);
}
__device__ __forceinline__ uint32_t key_pos(uint64_t key) {
  return 0xffffffffu - static_cast<uint32_t>(key);
}

// ---------------------------------------------------------------------------
// cp.async (16 bytes, L2 only)

__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
  uint32_t s = static_cast<uint32_t>(__cvta_generic_to_shared(smem));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N)); }

// ---------------------------------------------------------------------------
// host side

// Default bound of a device-side wait (a store's wait limit until changed).
constexpr unsigned long long kDefaultWaitNs = 2000000000ull;

struct Geometry {
  int64_t T;
  int32_t bs;
  int32_t sink;       // requested sink (tokens below it are not in retrieved ranges)
  int32_t sink_end;   // min(sink, w0)
  int64_t w0;         // first window token
  int32_t nb;         // full blocks
  int32_t first;      // first candidate block
  int32_t nc;         // candidates
};

rba_status geometry(const rba_store* st, int64_t T, int32_t sink, int32_t window, Geometry* g);
int num_sms();

// Raises a kernel's dynamic shared-memory limit once per (device, kernel);
// later calls (including inside stream capture) make no CUDA call.
cudaError_t ensure_smem(const void* kernel, size_t bytes);
// CTAs of `kernel` that fit on one SM with this block size and dynamic shared
// memory (raising the kernel's limit first), cached per (device, kernel,
// size); -1 on a CUDA error.
int occupancy(const void* kernel, int threads, size_t smem);

#define RBA_CUDA_TRY(expr)                          \
  do {                                              \
    cudaError_t e_ = (expr);                        \
    if (e_ != cudaSuccess) return RBA_ERR_CUDA;     \
  } while (0)

#define RBA_LAUNCH_CHECK()                          \
  do {                                              \
    if (cudaPeekAtLastError() != cudaSuccess) {     \
      (void)cudaGetLastError();                     \
      return RBA_ERR_CUDA;                          \
    }                                               \
  } while (0)

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Tensor map of a row-major [rows][cols] bf16 matrix for 2-D bulk tensor
// copies: boxes of 64 columns (128 bytes) x box_rows rows, 128-byte swizzle,
// zero fill outside the matrix.  False if the driver's encoder is unavailable
// or rejects the arguments.
bool make_tmap_bf16(CUtensorMap* m, const void* base, int64_t rows, int cols, int box_rows);
// the store's K and V tensor maps in 64-row boxes (encoded once); false if
// they cannot be encoded
bool store_tmaps64(const rba_store* st, CUtensorMap* kmap, CUtensorMap* vmap);
inline size_t dtype_size(rba_dtype t) { return t == RBA_BF16 ? 2 : 4; }
// Row pitch (elements) of the pools for a head dim: 64 up to 64, else 128;
// -1 for head dims the library does not hold (not a multiple of 4, or > 128).
inline int32_t pool_pitch(int32_t head_dim) {
  if (head_dim < 4 || head_dim > 128 || head_dim % 4 != 0) return -1;
  return head_dim <= 64 ? 64 : 128;
}

}  // namespace rba
