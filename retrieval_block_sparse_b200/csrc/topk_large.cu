// Exact top-k of long score rows (token-level retrieval: one unit per key,
// about a million candidates per kv head).
//
// Keys are 64-bit (order-preserving score bits << 32 | ~position), so the
// k-th largest key is unique and "ties -> lowest position" needs no extra
// pass.  Steps per row:
//   1. histogram of the top 11 score bits over the row;
//   2. the bin holding the k-th largest key; everything above it is selected;
//   3. compaction: positions above the bin, full keys inside the bin;
//   4. exact selection inside the bin (shared-memory sort, or an in-CTA radix
//      select over the compacted keys when heavy ties make it large), then
//      all k positions sorted ascending.
#include "rba_internal.cuh"
#include "topk_impl.cuh"

namespace rba {
namespace {

constexpr int kBins = 2048;
constexpr int kShift = 21;           // 32 - 11
constexpr int kChunk = 4096;         // scores per CTA in the scan passes
constexpr int kSortMax = 4096;       // compacted keys sorted in shared memory
constexpr int kFinishThreads = 1024;

struct RowState {
  uint32_t bin;      // bin holding the k-th largest key
  uint32_t kk;       // keys still to take from that bin
  uint32_t n_above;  // positions written to `above`
  uint32_t n_cand;   // keys written to `cand`
};

struct Layout {
  uint32_t* hist;   // [rows][kBins]
  RowState* state;  // [rows]
  uint32_t* above;  // [rows][k]
  uint64_t* cand;   // [rows][n]
  size_t zero_bytes;
  size_t total;
};

Layout layout(void* ws, int rows, int n, int k) {
  Layout L;
  char* p = static_cast<char*>(ws);
  size_t off = 0;
  L.hist = reinterpret_cast<uint32_t*>(p + off);
  off += align_up(size_t(rows) * kBins * 4, 256);
  L.state = reinterpret_cast<RowState*>(p + off);
  off += align_up(size_t(rows) * sizeof(RowState), 256);
  L.zero_bytes = off;
  L.above = reinterpret_cast<uint32_t*>(p + off);
  off += align_up(size_t(rows) * k * 4, 256);
  L.cand = reinterpret_cast<uint64_t*>(p + off);
  off += align_up(size_t(rows) * n * 8, 256);
  L.total = off;
  return L;
}

__global__ void hist_kernel(const float* __restrict__ scores, int n, uint32_t* __restrict__ hist) {
  __shared__ uint32_t h[kBins];
  for (int b = threadIdx.x; b < kBins; b += blockDim.x) h[b] = 0;
  __syncthreads();
  const int64_t row = blockIdx.y;
  const float* s = scores + row * n;
  const int i0 = blockIdx.x * kChunk;
  const int i1 = min(n, i0 + kChunk);
  // lanes falling into the same bin add once (neighbouring scores share their
  // top bits, so plain per-lane atomics would serialise)
  for (int base = i0; base < i1; base += blockDim.x) {
    const int i = base + threadIdx.x;
    const bool ok = i < i1;
    const uint32_t bin = ok ? ordered_f32(s[i]) >> kShift : uint32_t(kBins);
    const unsigned same = __match_any_sync(0xffffffffu, bin);
    if (ok && (threadIdx.x & 31) == __ffs(same) - 1) atomicAdd(&h[bin], uint32_t(__popc(same)));
  }
  __syncthreads();
  for (int b = threadIdx.x; b < kBins; b += blockDim.x)
    if (h[b]) atomicAdd(&hist[row * kBins + b], h[b]);
}

// One CTA of 1024 threads per row: suffix sums over the bins.
__global__ void pick_bin_kernel(const uint32_t* __restrict__ hist, RowState* __restrict__ state,
                                int k) {
  __shared__ uint32_t suf[kBins + 1];
  const int64_t row = blockIdx.x;
  // bins are scanned from the top: position p holds bin (kBins-1-p)
  for (int p = threadIdx.x; p < kBins; p += blockDim.x)
    suf[p] = hist[row * kBins + (kBins - 1 - p)];
  __syncthreads();
  // inclusive prefix over p (Hillis-Steele)
  for (int off = 1; off < kBins; off <<= 1) {
    uint32_t v[2];
    for (int j = 0; j < 2; ++j) {
      const int p = threadIdx.x + j * blockDim.x;
      v[j] = (p < kBins && p >= off) ? suf[p - off] : 0u;
    }
    __syncthreads();
    for (int j = 0; j < 2; ++j) {
      const int p = threadIdx.x + j * blockDim.x;
      if (p < kBins) suf[p] += v[j];
    }
    __syncthreads();
  }
  for (int p = threadIdx.x; p < kBins; p += blockDim.x) {
    const uint32_t incl = suf[p];
    const uint32_t excl = p ? suf[p - 1] : 0u;
    if (excl < uint32_t(k) && uint32_t(k) <= incl) {
      state[row].bin = kBins - 1 - p;
      state[row].kk = uint32_t(k) - excl;
    }
  }
}

__global__ void compact_kernel(const float* __restrict__ scores, int n, int k,
                               RowState* __restrict__ state, uint32_t* __restrict__ above,
                               uint64_t* __restrict__ cand) {
  const int64_t row = blockIdx.y;
  const float* s = scores + row * n;
  const uint32_t bin = state[row].bin;
  const int lane = threadIdx.x & 31;
  const int i0 = blockIdx.x * kChunk;
  const int i1 = min(n, i0 + kChunk);
  for (int base = i0; base < i1; base += blockDim.x) {
    const int i = base + threadIdx.x;
    uint32_t key32 = 0, d = 0;
    bool ok = i < i1;
    if (ok) {
      key32 = ordered_f32(s[i]);
      d = key32 >> kShift;
    }
    const bool up = ok && d > bin;
    const bool eq = ok && d == bin;
    // warp-aggregated appends
    const unsigned mu = __ballot_sync(0xffffffffu, up);
    if (mu) {
      uint32_t b0 = 0;
      if (lane == __ffs(mu) - 1) b0 = atomicAdd(&state[row].n_above, __popc(mu));
      b0 = __shfl_sync(0xffffffffu, b0, __ffs(mu) - 1);
      if (up) {
        const uint32_t slot = b0 + __popc(mu & ((1u << lane) - 1));
        if (slot < uint32_t(k)) above[row * k + slot] = uint32_t(i);
      }
    }
    const unsigned me = __ballot_sync(0xffffffffu, eq);
    if (me) {
      uint32_t b0 = 0;
      if (lane == __ffs(me) - 1) b0 = atomicAdd(&state[row].n_cand, __popc(me));
      b0 = __shfl_sync(0xffffffffu, b0, __ffs(me) - 1);
      if (eq) {
        const uint32_t slot = b0 + __popc(me & ((1u << lane) - 1));
        if (slot < uint32_t(n))
          cand[row * n + slot] = (uint64_t(key32) << 32) | (0xffffffffu - uint32_t(i));
      }
    }
  }
}

__device__ void bitonic_desc64(uint64_t* keys, int P) {
  for (int size = 2; size <= P; size <<= 1)
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

__device__ void bitonic_asc32(uint32_t* v, int P) {
  for (int size = 2; size <= P; size <<= 1)
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

__global__ void __launch_bounds__(kFinishThreads)
    finish_kernel(const RowState* __restrict__ state, const uint32_t* __restrict__ above,
                  const uint64_t* __restrict__ cand, int n, int k, int Pk, int index_base,
                  int32_t* __restrict__ idx) {
  extern __shared__ uint64_t sm64[];
  uint64_t* keys = sm64;                                          // [kSortMax]
  uint32_t* pos = reinterpret_cast<uint32_t*>(sm64 + kSortMax);  // [Pk]
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_cnt;
  __shared__ uint64_t s_prefix;
  __shared__ uint32_t s_need;
  const int64_t row = blockIdx.x;
  const uint32_t m = min(state[row].n_cand, uint32_t(n));
  const uint32_t kk = state[row].kk;
  const uint32_t na = uint32_t(k) - kk;
  const uint64_t* c = cand + row * n;
  for (int i = threadIdx.x; i < int(na); i += blockDim.x) pos[i] = above[row * k + i];
  if (m <= uint32_t(kSortMax)) {
    int P = 2;
    while (P < int(m)) P <<= 1;
    for (int i = threadIdx.x; i < P; i += blockDim.x) keys[i] = i < int(m) ? c[i] : 0ull;
    __syncthreads();
    bitonic_desc64(keys, P);
    for (int i = threadIdx.x; i < int(kk); i += blockDim.x) pos[na + i] = key_pos(keys[i]);
  } else {
    // radix select of the kk-th largest key among m, 8 bits at a time
    if (threadIdx.x == 0) {
      s_prefix = 0;
      s_need = kk;
      s_cnt = 0;
    }
    uint64_t mask = 0;
    for (int shift = 56; shift >= 0; shift -= 8) {
      for (int b = threadIdx.x; b < 256; b += blockDim.x) hist[b] = 0;
      __syncthreads();
      const uint64_t prefix = s_prefix;
      for (uint32_t j = threadIdx.x; j < m; j += blockDim.x) {
        const uint64_t key = c[j];
        if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
      }
      __syncthreads();
      if (threadIdx.x == 0) {
        uint32_t above_cnt = 0, need = s_need;
        for (int dgt = 255; dgt >= 0; --dgt) {
          if (above_cnt + hist[dgt] >= need) {
            s_prefix = prefix | (uint64_t(dgt) << shift);
            s_need = need - above_cnt;
            break;
          }
          above_cnt += hist[dgt];
        }
      }
      mask |= uint64_t(255) << shift;
      __syncthreads();
    }
    const uint64_t thr = s_prefix;  // the kk-th largest key: exactly kk keys are >= thr
    for (uint32_t j = threadIdx.x; j < m; j += blockDim.x) {
      const uint64_t key = c[j];
      if (key >= thr) {
        const uint32_t slot = atomicAdd(&s_cnt, 1u);
        if (slot < kk) pos[na + slot] = key_pos(key);
      }
    }
  }
  __syncthreads();
  for (int i = k + threadIdx.x; i < Pk; i += blockDim.x) pos[i] = 0xffffffffu;
  __syncthreads();
  bitonic_asc32(pos, Pk);
  for (int i = threadIdx.x; i < k; i += blockDim.x)
    idx[row * k + i] = index_base + static_cast<int32_t>(pos[i]);
}

}  // namespace

size_t topk_large_workspace(int rows, int n, int k) { return layout(nullptr, rows, n, k).total; }

rba_status launch_topk_large(const float* scores, int rows, int n, int k, int index_base,
                             int32_t* idx, void* ws, cudaStream_t stream) {
  if (k > kLargeMaxK) return RBA_ERR_UNSUPPORTED;
  if (ws == nullptr) return RBA_ERR_WORKSPACE;
  Layout L = layout(ws, rows, n, k);
  RBA_CUDA_TRY(cudaMemsetAsync(ws, 0, L.zero_bytes, stream));
  const dim3 scan_grid((n + kChunk - 1) / kChunk, rows);
  hist_kernel<<<scan_grid, 512, 0, stream>>>(scores, n, L.hist);
  RBA_LAUNCH_CHECK();
  pick_bin_kernel<<<rows, 1024, 0, stream>>>(L.hist, L.state, k);
  RBA_LAUNCH_CHECK();
  compact_kernel<<<scan_grid, 512, 0, stream>>>(scores, n, k, L.state, L.above, L.cand);
  RBA_LAUNCH_CHECK();
  int Pk = 2;
  while (Pk < k) Pk <<= 1;
  const size_t smem = size_t(kSortMax) * 8 + size_t(Pk) * 4;
  RBA_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(finish_kernel), smem));
  finish_kernel<<<rows, kFinishThreads, smem, stream>>>(L.state, L.above, L.cand, n, k, Pk,
                                                        index_base, idx);
  RBA_LAUNCH_CHECK();
  return RBA_OK;
}

}  // namespace rba
