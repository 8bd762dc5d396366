// Top-k block selection.
//
// MemLong summary, 2.3.2 (z^q = TopK{Cos(r^q)}) and 2.3.4 (the k most
// relevant chunks).  Order: larger score first; equal scores -> lower
// position first.  Each score becomes a 64-bit key (order-preserving score
// bits << 32 | ~position), so one unsigned comparison decides both, and the
// k largest keys are the selection.  Rows of up to kSmallN scores are sorted
// by one CTA in shared memory; longer rows go through a radix select.
#include "rba_internal.cuh"
#include "topk_impl.cuh"

namespace rba {
namespace {

constexpr int kThreads = 1024;

// Bitonic sort of P (power of two) keys in shared memory; descending.
__device__ void bitonic_desc(uint64_t* keys, int P) {
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < (P >> 1); i += blockDim.x) {
        const int lo = 2 * stride * (i / stride) + (i % stride);
        const int hi = lo + stride;
        const bool desc = (lo & size) == 0;
        const uint64_t a = keys[lo], b = keys[hi];
        if (desc ? (a < b) : (a > b)) {
          keys[lo] = b;
          keys[hi] = a;
        }
      }
      __syncthreads();
    }
  }
}

// Bitonic sort ascending of P uint32 values.
__device__ void bitonic_asc32(uint32_t* v, int P) {
  for (int size = 2; size <= P; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int i = threadIdx.x; i < (P >> 1); i += blockDim.x) {
        const int lo = 2 * stride * (i / stride) + (i % stride);
        const int hi = lo + stride;
        const bool asc = (lo & size) == 0;
        const uint32_t a = v[lo], b = v[hi];
        if (asc ? (a > b) : (a < b)) {
          v[lo] = b;
          v[hi] = a;
        }
      }
      __syncthreads();
    }
  }
}

__global__ void __launch_bounds__(kThreads) topk_small_kernel(const float* __restrict__ scores,
                                                              int n, int k, int P, int Pk,
                                                              int index_base,
                                                              int32_t* __restrict__ idx) {
  extern __shared__ uint64_t skeys[];
  const int64_t row = blockIdx.x;
  const float* s = scores + row * n;
  for (int i = threadIdx.x; i < P; i += blockDim.x)
    skeys[i] = i < n ? topk_key(s[i], static_cast<uint32_t>(i)) : 0ull;
  __syncthreads();
  bitonic_desc(skeys, P);
  // positions of the k best, sorted ascending (reuse the tail of shared memory)
  uint32_t* pos = reinterpret_cast<uint32_t*>(skeys + P);
  for (int i = threadIdx.x; i < Pk; i += blockDim.x)
    pos[i] = i < k ? key_pos(skeys[i]) : 0xffffffffu;
  __syncthreads();
  bitonic_asc32(pos, Pk);
  for (int i = threadIdx.x; i < k; i += blockDim.x)
    idx[row * k + i] = index_base + static_cast<int32_t>(pos[i]);
}

int pow2_at_least(int x) {
  int p = 1;
  while (p < x) p <<= 1;
  return p;
}

}  // namespace

rba_status launch_topk(const float* scores, int rows, int n, int k, int index_base, int32_t* idx,
                       void* ws, size_t ws_bytes, cudaStream_t stream) {
  if (rows == 0 || k == 0) return RBA_OK;
  if (n <= kSmallN) {
    const int P = pow2_at_least(n < 2 ? 2 : n);
    const int Pk = pow2_at_least(k < 2 ? 2 : k);
    const size_t smem = size_t(P) * 8 + size_t(Pk) * 4;
    if (smem > 48 * 1024)
      RBA_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(topk_small_kernel), smem));
    topk_small_kernel<<<rows, kThreads, smem, stream>>>(scores, n, k, P, Pk, index_base, idx);
    RBA_LAUNCH_CHECK();
    return RBA_OK;
  }
  if (ws_bytes < topk_large_workspace(rows, n, k)) return RBA_ERR_WORKSPACE;
  return launch_topk_large(scores, rows, n, k, index_base, idx, ws, stream);
}

size_t topk_workspace(int rows, int n, int k) {
  return n <= kSmallN ? 0 : topk_large_workspace(rows, n, k);
}

}  // namespace rba

extern "C" rba_status rba_topk(const float* scores, int32_t rows, int32_t n, int32_t k,
                               int32_t index_base, int32_t* idx, void* workspace, size_t ws_bytes,
                               cudaStream_t stream) {
  if (rows < 0 || n < 0 || k < 0 || k > n) return RBA_ERR_INVALID_ARG;
  if (rows > 0 && k > 0 && (scores == nullptr || idx == nullptr)) return RBA_ERR_INVALID_ARG;
  if (k > (1 << 16)) return RBA_ERR_UNSUPPORTED;
  return rba::launch_topk(scores, rows, n, k, index_base, idx, workspace, ws_bytes, stream);
}

extern "C" size_t rba_topk_workspace_size(int32_t rows, int32_t n, int32_t k) {
  if (rows <= 0 || n <= 0 || k <= 0) return 0;
  return rba::topk_workspace(rows, n, k);
}
