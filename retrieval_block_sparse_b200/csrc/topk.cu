// Top-k block selection.
//
// MemLong summary, 2.3.2 (z^q = TopK{Cos(r^q)}) and 2.3.4 (the k most
// relevant chunks).  Order: larger score first; equal scores -> lower
// position first.  Each score becomes a 64-bit key (order-preserving score
// bits << 32 | ~position), so one unsigned comparison decides both, and the
// k largest keys are the selection.  Rows of up to kSmallN scores are
// selected by one CTA in shared memory (one value-binned histogram pass,
// radix select where that does not apply); longer rows go through a
// multi-CTA radix select.
#include "rba_internal.cuh"
#include "topk_impl.cuh"

namespace rba {
namespace {

constexpr int kRowThreads = 512;
constexpr int kRowWarps = kRowThreads / 32;
constexpr int kBins = 256;  // value bins of the one-pass select

__device__ __forceinline__ int block_exclusive_scan1(int v, int* s_w, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) s_w[warp] = incl;
  __syncthreads();
  int base = 0, tot = 0;
  for (int w = 0; w < kRowWarps; ++w) {
    const int x = s_w[w];
    if (w < warp) base += x;
    tot += x;
  }
  __syncthreads();
  *total = tot;
  return base + incl - v;
}

// Positions whose flag is set, written ascending (index_base + position).
__device__ __forceinline__ void write_flagged(const uint8_t* flag, int n, int index_base,
                                              int32_t* dst, int* s_w) {
  const int per = (n + kRowThreads - 1) / kRowThreads;
  const int p0 = threadIdx.x * per, p1 = min(n, p0 + per);
  int cnt = 0;
  for (int j = p0; j < p1; ++j) cnt += flag[j];
  int tot;
  int rank = block_exclusive_scan1(cnt, s_w, &tot);
  for (int j = p0; j < p1; ++j)
    if (flag[j]) dst[rank++] = index_base + j;
}

// Radix select of the k-th largest order-preserving key (4 passes of 8
// bits), then every larger key and the first equal ones in position order.
__device__ void select_radix(const float* s, int n, int k, int index_base, int32_t* dst,
                             uint32_t* keys, uint8_t* flag, uint32_t* hist, int* s_w,
                             int* s_misc) {
  const int tid = threadIdx.x, lane = tid & 31;
  for (int j = tid; j < n; j += kRowThreads) keys[j] = ordered_f32(s[j]);
  __syncthreads();
  uint32_t prefix = 0, mask = 0;
  int kk = k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = tid; b < 256; b += kRowThreads) hist[b] = 0;
    __syncthreads();
    // lanes falling into the same bin add once (keys often share top bits)
    for (int j0 = tid - lane; j0 < n; j0 += kRowThreads) {
      const int j = j0 + lane;
      const uint32_t u = j < n ? keys[j] : 0u;
      const bool in = j < n && (u & mask) == prefix;
      const uint32_t bin = in ? ((u >> shift) & 255u) : 256u;
      const unsigned same = __match_any_sync(0xffffffffu, bin);
      if (in && lane == __ffs(same) - 1) atomicAdd(&hist[bin], uint32_t(__popc(same)));
    }
    __syncthreads();
    if (tid < 32) {
      // lane l owns bins [8l, 8l+8); counts above a bin = all higher bins
      uint32_t c[8], tot = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        c[i] = hist[tid * 8 + i];
        tot += c[i];
      }
      uint32_t incl = tot;
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
    __syncthreads();
    prefix |= uint32_t(s_misc[0]) << shift;
    mask |= 255u << shift;
    kk -= s_misc[1];
    __syncthreads();
  }
  const int per = (n + kRowThreads - 1) / kRowThreads;
  const int p0 = tid * per, p1 = min(n, p0 + per);
  int n_eq = 0;
  for (int j = p0; j < p1; ++j) n_eq += keys[j] == prefix;
  int tot;
  int e = block_exclusive_scan1(n_eq, s_w, &tot);
  for (int j = p0; j < p1; ++j) {
    const uint32_t u = keys[j];
    flag[j] = u > prefix || (u == prefix && e++ < kk);
  }
  __syncthreads();
  write_flagged(flag, n, index_base, dst, s_w);
}

// value bin of x: monotone non-decreasing in x, so every score in a higher
// bin is strictly larger than every score in a lower one
__device__ __forceinline__ int value_bin(float x, float lo, float scale) {
  const float t = __fmul_rn(__fsub_rn(x, lo), scale);
  return min(kBins - 1, static_cast<int>(t));
}

// One histogram pass: kBins bins linear in the score value between the
// row's min and max.  Every score in the bins above the bin holding the k-th
// largest is selected; inside that bin the members are ranked exactly
// (value, then lower position).  False (nothing written) for rows it does
// not cover: non-finite scores, a zero range, or more members in the
// boundary bin than threads.
__device__ bool select_binned(const float* s, int n, int k, int index_base, int32_t* dst,
                              float* vals, uint8_t* flag, int* cand, uint32_t* hist, int* s_w,
                              int* s_misc, float* s_f) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  float lo = INFINITY, hi = -INFINITY;
  int bad = 0;
  // long rows: sixteen loads in flight per thread before any store (two
  // rounds at the longest rows instead of one per four scores); short rows
  // (the decode step's) keep the plain loop
  constexpr int kBatch = 16;
  if (n <= 8 * kRowThreads) {
#pragma unroll 4
    for (int j = tid; j < n; j += kRowThreads) {
      const float v = s[j];
      vals[j] = v;
      bad |= !isfinite(v);
      lo = fminf(lo, v);
      hi = fmaxf(hi, v);
    }
  }
  for (int j0 = n <= 8 * kRowThreads ? n : tid; j0 < n; j0 += kBatch * kRowThreads) {
    float v[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int j = j0 + u * kRowThreads;
      v[u] = j < n ? s[j] : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int j = j0 + u * kRowThreads;
      if (j < n) {
        vals[j] = v[u];
        bad |= !isfinite(v[u]);
        lo = fminf(lo, v[u]);
        hi = fmaxf(hi, v[u]);
      }
    }
  }
  for (int b = tid; b < kBins; b += kRowThreads) hist[b] = 0;
  for (int o = 16; o > 0; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  bad = __any_sync(0xffffffffu, bad);
  if (lane == 0) {
    s_f[2 * warp] = lo;
    s_f[2 * warp + 1] = hi;
    s_w[warp] = bad;
  }
  __syncthreads();
  lo = s_f[0];
  hi = s_f[1];
  bad = s_w[0];
  for (int w = 1; w < kRowWarps; ++w) {
    lo = fminf(lo, s_f[2 * w]);
    hi = fmaxf(hi, s_f[2 * w + 1]);
    bad |= s_w[w];
  }
  const float range = hi - lo;
  const float scale = float(kBins) / range;
  __syncthreads();  // s_w / s_f are reused below
  // (uniform: every thread decided on the same shared values)
  if (bad || !(range > 0.f) || !isfinite(range) || !isfinite(scale)) return false;
  for (int j = tid; j < n; j += kRowThreads) atomicAdd(&hist[value_bin(vals[j], lo, scale)], 1u);
  __syncthreads();
  if (warp == 0) {
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
  __syncthreads();
  const int bstar = s_misc[0], n_above = s_misc[1], nb = s_misc[2];
  if (nb > kRowThreads) return false;
  for (int j = tid; j < n; j += kRowThreads) {
    const int bin = value_bin(vals[j], lo, scale);
    if (bin == bstar) cand[atomicAdd(&s_misc[3], 1)] = j;
    flag[j] = bin > bstar;
  }
  __syncthreads();
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
  __syncthreads();
  write_flagged(flag, n, index_base, dst, s_w);
  return true;
}

// One CTA per row of n <= kSmallN scores.  Launched behind the kernel that
// writes the scores, it may start early (programmatic dependent launch) and
// waits for that kernel's completion before reading them.
__global__ void __launch_bounds__(kRowThreads) topk_rows_kernel(const float* __restrict__ scores,
                                                                int n, int k, int index_base,
                                                                int32_t* __restrict__ idx) {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  extern __shared__ __align__(16) char sm[];
  float* vals = reinterpret_cast<float*>(sm);                            // [n]
  uint8_t* flag = reinterpret_cast<uint8_t*>(sm + size_t(n) * 4);        // [n]
  __shared__ int cand[kRowThreads];
  __shared__ uint32_t hist[kBins];
  __shared__ int s_w[32];
  __shared__ int s_misc[8];
  __shared__ float s_f[2 * kRowWarps];
  const int64_t row = blockIdx.x;
  const float* s = scores + row * n;
  int32_t* dst = idx + row * k;
  if (k >= n) {
    for (int j = threadIdx.x; j < n; j += kRowThreads) dst[j] = index_base + j;
    return;
  }
  if (!select_binned(s, n, k, index_base, dst, vals, flag, cand, hist, s_w, s_misc, s_f))
    select_radix(s, n, k, index_base, dst, reinterpret_cast<uint32_t*>(vals), flag, hist, s_w,
                 s_misc);
}

}  // namespace

rba_status launch_topk(const float* scores, int rows, int n, int k, int index_base, int32_t* idx,
                       void* ws, size_t ws_bytes, cudaStream_t stream, bool pdl) {
  if (rows == 0 || k == 0) return RBA_OK;
  if (n <= kSmallN) {
    const size_t smem = size_t(n) * 5 + 16;
    RBA_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(topk_rows_kernel), smem));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(rows);
    cfg.blockDim = dim3(kRowThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = pdl ? 1 : 0;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    RBA_CUDA_TRY(cudaLaunchKernelEx(&cfg, topk_rows_kernel, scores, n, k, index_base, idx));
    return RBA_OK;
  }
  if (ws_bytes < topk_large_workspace(rows, n, k)) return RBA_ERR_WORKSPACE;
  return launch_topk_large(scores, rows, n, k, index_base, idx, ws, stream);
}

int topk_ctas(int rows, int n) { return n <= kSmallN ? rows : 0; }

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
  return rba::launch_topk(scores, rows, n, k, index_base, idx, workspace, ws_bytes, stream,
                          false);
}

extern "C" size_t rba_topk_workspace_size(int32_t rows, int32_t n, int32_t k) {
  if (rows <= 0 || n <= 0 || k <= 0) return 0;
  return rba::topk_workspace(rows, n, k);
}
