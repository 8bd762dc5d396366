// Memorisation: append blocks to the store and compute their representations.
//
// MemLong summary, 2.3.2 (memorisation M(k, v; r^m)): K-V pairs and the
// block's representation are written together, index-aligned.
// InfLLM article, "method": a memory unit is represented by the tokens that
// received the highest attention scores.
// Landmark Attention review, "proposed method": one landmark key per block.
#include "rba_internal.cuh"

namespace rba {
namespace {

// Copy `rows` rows of `vec_per_row` 16-byte vectors for each of `bh` slices from
// src [bh][rows] into dst [bh][dst_rows] at row offset `row0`.
__global__ void copy_rows_kernel(const uint4* __restrict__ src, uint4* __restrict__ dst,
                                 int64_t bh, int64_t rows, int64_t dst_rows, int64_t row0,
                                 int32_t vec_per_row) {
  const int64_t per_bh = rows * vec_per_row;
  const int64_t total = bh * per_bh;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t s = i / per_bh;
    const int64_t rem = i - s * per_bh;
    dst[(s * dst_rows + row0) * vec_per_row + rem] = src[i];
  }
}

// As copy_rows_kernel for rows of src_words 32-bit words into rows of
// dst_words >= src_words (head dims below the pools' row pitch): the words
// past src_words are written as zero.
__global__ void copy_rows_pad_kernel(const uint32_t* __restrict__ src, uint32_t* __restrict__ dst,
                                     int64_t bh, int64_t rows, int64_t dst_rows, int64_t row0,
                                     int32_t src_words, int32_t dst_words) {
  const int64_t per_bh = rows * dst_words;
  const int64_t total = bh * per_bh;
  for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < total;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int64_t s = i / per_bh;
    const int64_t rem = i - s * per_bh;
    const int64_t r = rem / dst_words;
    const int w = static_cast<int>(rem - r * dst_words);
    dst[(s * dst_rows + row0 + r) * dst_words + w] =
        w < src_words ? src[(s * rows + r) * src_words + w] : 0u;
  }
}

// RBA_REP_MEAN: rep[j] = (1/bs) sum_t k_t, fp32.  grid (n_blocks, B*Hkv), block D.
template <typename T>
__global__ void rep_mean_kernel(const T* __restrict__ K, float* __restrict__ rep, int D, int bs,
                                int64_t cap_tokens, int64_t cap_blocks, int64_t first_block) {
  const int64_t j = first_block + blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int d = threadIdx.x;
  const T* base = K + (bh * cap_tokens + j * bs) * D + d;
  float acc = 0.f;
  for (int t = 0; t < bs; ++t) acc += Elem<T>::to_f32(base[int64_t(t) * D]);
  rep[(bh * cap_blocks + j) * D + d] = acc / float(bs);
}

constexpr int kMaxProbe = 32;

// RBA_REP_TOPR_ATTN.  grid (n_blocks, B*Hkv), block = bs rounded up to 32 (<= 1024).
// Thread t owns token t of the block.
template <typename T, int D>
__global__ void rep_topr_kernel(const T* __restrict__ K, const T* __restrict__ probe,
                                T* __restrict__ rep, int32_t* __restrict__ rep_pos, int Hkv,
                                int bs, int r, int P, int qd, float scale_log2,
                                int64_t cap_tokens, int64_t cap_blocks, int64_t first_block) {
  extern __shared__ float sm[];
  float* sprobe = sm;                          // [P][D]
  float* sred = sm + P * D;                    // [32 warps][kMaxProbe]
  __shared__ uint64_t swin[32];
  __shared__ int32_t schosen[32];
  const int t = threadIdx.x;
  const int lane = t & 31, warp = t >> 5, nwarp = blockDim.x >> 5;
  const int64_t j = first_block + blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int h = static_cast<int>(bh % Hkv);
  for (int i = t; i < P * D; i += blockDim.x) {  // probe rows are qd long
    const int p = i / D, d = i - p * D;
    sprobe[i] = d < qd ? Elem<T>::to_f32(probe[(int64_t(h) * P + p) * qd + d]) : 0.f;
  }
  __syncthreads();

  const bool valid = t < bs;
  float x[kMaxProbe];
#pragma unroll
  for (int p = 0; p < kMaxProbe; ++p) x[p] = 0.f;
  if (valid) {
    const uint4* row = reinterpret_cast<const uint4*>(K + (bh * cap_tokens + j * bs + t) * D);
    constexpr int EPV = Elem<T>::kPerVec;
    for (int v = 0; v < D / EPV; ++v) {
      float kf[EPV];
      unpack(row[v], kf, T());
#pragma unroll
      for (int p = 0; p < kMaxProbe; ++p) {
        if (p < P) {
          float a = x[p];
#pragma unroll
          for (int e = 0; e < EPV; ++e) a = fmaf(sprobe[p * D + v * EPV + e], kf[e], a);
          x[p] = a;
        }
      }
    }
  }
  // per probe: softmax over the block's tokens (base-2 with scale folded in)
#pragma unroll
  for (int p = 0; p < kMaxProbe; ++p) x[p] = valid ? x[p] * scale_log2 : -INFINITY;

  // max over tokens, per probe
#pragma unroll
  for (int p = 0; p < kMaxProbe; ++p) {
    if (p < P) {
      float m = x[p];
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
      if (lane == 0) sred[warp * kMaxProbe + p] = m;
    }
  }
  __syncthreads();
  float mx[kMaxProbe];
#pragma unroll
  for (int p = 0; p < kMaxProbe; ++p) {
    float m = -INFINITY;
    if (p < P)
      for (int w = 0; w < nwarp; ++w) m = fmaxf(m, sred[w * kMaxProbe + p]);
    mx[p] = m;
  }
  __syncthreads();
  // sum of exp over tokens, per probe
  float e[kMaxProbe];
#pragma unroll
  for (int p = 0; p < kMaxProbe; ++p) {
    if (p < P) {
      e[p] = valid ? exp2f(x[p] - mx[p]) : 0.f;
      float s = e[p];
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) sred[warp * kMaxProbe + p] = s;
    }
  }
  __syncthreads();
  float received = 0.f;
#pragma unroll
  for (int p = 0; p < kMaxProbe; ++p) {
    if (p < P) {
      float z = 0.f;
      for (int w = 0; w < nwarp; ++w) z += sred[w * kMaxProbe + p];
      received += e[p] / z;
    }
  }
  // top-r tokens by received attention, ties -> lower position
  uint64_t key = valid ? topk_key(received, static_cast<uint32_t>(t)) : 0ull;
  for (int i = 0; i < r; ++i) {
    uint64_t m = key;
    for (int o = 16; o > 0; o >>= 1) {
      uint64_t other = __shfl_xor_sync(0xffffffffu, m, o);
      m = other > m ? other : m;
    }
    if (lane == 0) swin[warp] = m;
    __syncthreads();
    uint64_t best = 0;
    for (int w = 0; w < nwarp; ++w) best = swin[w] > best ? swin[w] : best;
    if (key == best) key = 0ull;  // unique: the position is part of the key
    if (t == 0) schosen[i] = static_cast<int32_t>(key_pos(best));
    __syncthreads();
  }
  if (t == 0) {  // ascending positions (r <= 32)
    for (int a = 1; a < r; ++a) {
      int32_t v = schosen[a];
      int b = a - 1;
      while (b >= 0 && schosen[b] > v) {
        schosen[b + 1] = schosen[b];
        --b;
      }
      schosen[b + 1] = v;
    }
  }
  __syncthreads();
  const int64_t rbase = (bh * cap_blocks + j) * r;
  if (rep_pos != nullptr && t < r) rep_pos[rbase + t] = schosen[t];
  for (int i = t; i < r * D; i += blockDim.x) {
    const int ri = i / D, d = i - ri * D;
    rep[(rbase + ri) * D + d] = K[(bh * cap_tokens + j * bs + schosen[ri]) * D + d];
  }
}

// RBA_REP_EMBED_COSINE: rep[b][j] = e / |e| (fp32).  One warp per embedding.
__global__ void rep_embed_kernel(const float* __restrict__ e, float* __restrict__ rep, int d_ret,
                                 int64_t rows, int32_t n_blocks, int64_t cap_blocks,
                                 int64_t first_block) {
  const int64_t w = (blockIdx.x * int64_t(blockDim.x) + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= rows) return;
  const int64_t b = w / n_blocks, j = w - b * n_blocks;
  const float* src = e + w * d_ret;
  float ss = 0.f;
  for (int d = lane; d < d_ret; d += 32) ss = fmaf(src[d], src[d], ss);
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float nrm = sqrtf(ss);
  float* dst = rep + (b * cap_blocks + first_block + j) * d_ret;
  for (int d = lane; d < d_ret; d += 32) dst[d] = src[d] / nrm;
}

int grid_for(int64_t work, int threads) {
  int64_t g = (work + threads - 1) / threads;
  const int64_t cap = int64_t(num_sms()) * 16;
  if (g > cap) g = cap;
  return static_cast<int>(g < 1 ? 1 : g);
}

}  // namespace
}  // namespace rba

extern "C" rba_status rba_memorize(rba_store* st, const void* k_src, const void* v_src,
                                   int64_t first_block, int32_t n_blocks, const void* aux,
                                   int32_t n_aux, float scale, cudaStream_t stream) {
  using namespace rba;
  if (st == nullptr || n_blocks < 0 || first_block < 0) return RBA_ERR_INVALID_ARG;
  if (n_blocks == 0) return RBA_OK;
  const rba_store_desc& d = st->d;
  if (first_block + n_blocks > st->cap_blocks) return RBA_ERR_INVALID_ARG;
  if ((k_src == nullptr) != (v_src == nullptr)) return RBA_ERR_INVALID_ARG;
  const int64_t BH = int64_t(d.batch) * d.n_kv_heads;
  const int64_t bs = d.block_size;
  const int D = st->pitch;  // pool rows; inputs are d.head_dim long
  const size_t es = dtype_size(d.dtype);
  const int vec_row = static_cast<int>(D * es / 16);
  const bool padded = d.head_dim != D;
  const int src_words = static_cast<int>(d.head_dim * es / 4), dst_words = static_cast<int>(D * es / 4);
  // rows of `rows` per (b, kv head) from a dense input into a pool at row0
  auto copy_in = [&](const void* src, void* dst, int64_t rows, int64_t dst_rows,
                     int64_t row0) -> rba_status {
    if (!padded) {
      const int g = grid_for(BH * rows * vec_row, 256);
      copy_rows_kernel<<<g, 256, 0, stream>>>(static_cast<const uint4*>(src),
                                              static_cast<uint4*>(dst), BH, rows, dst_rows, row0,
                                              vec_row);
    } else {
      const int g = grid_for(BH * rows * dst_words, 256);
      copy_rows_pad_kernel<<<g, 256, 0, stream>>>(static_cast<const uint32_t*>(src),
                                                  static_cast<uint32_t*>(dst), BH, rows, dst_rows,
                                                  row0, src_words, dst_words);
    }
    RBA_LAUNCH_CHECK();
    return RBA_OK;
  };

  if (k_src != nullptr) {
    const int64_t rows = int64_t(n_blocks) * bs;
    rba_status s = copy_in(k_src, st->k, rows, d.capacity_tokens, first_block * bs);
    if (s != RBA_OK) return s;
    s = copy_in(v_src, st->v, rows, d.capacity_tokens, first_block * bs);
    if (s != RBA_OK) return s;
  }

  const dim3 grid(static_cast<unsigned>(n_blocks), static_cast<unsigned>(BH));
  switch (d.mode) {
    case RBA_REP_MEAN: {
      if (d.dtype == RBA_F32)
        rep_mean_kernel<float><<<grid, D, 0, stream>>>(
            static_cast<const float*>(st->k), static_cast<float*>(st->rep), D,
            static_cast<int>(bs), d.capacity_tokens, st->cap_blocks, first_block);
      else
        rep_mean_kernel<__nv_bfloat16><<<grid, D, 0, stream>>>(
            static_cast<const __nv_bfloat16*>(st->k), static_cast<float*>(st->rep), D,
            static_cast<int>(bs), d.capacity_tokens, st->cap_blocks, first_block);
      RBA_LAUNCH_CHECK();
      break;
    }
    case RBA_REP_TOPR_ATTN: {
      if (aux == nullptr || n_aux <= 0 || n_aux > kMaxProbe) return RBA_ERR_INVALID_ARG;
      const int threads = static_cast<int>((bs + 31) / 32 * 32);
      const size_t smem = (size_t(n_aux) * D + 32 * kMaxProbe) * sizeof(float);
      const float sl2 = scale * 1.4426950408889634f;
#define RBA_TOPR(T_, D_)                                                                      \
  do {                                                                                        \
    auto kfn = rep_topr_kernel<T_, D_>;                                                       \
    RBA_CUDA_TRY(ensure_smem(reinterpret_cast<const void*>(kfn), smem));                       \
    kfn<<<grid, threads, smem, stream>>>(static_cast<const T_*>(st->k),                       \
                                         static_cast<const T_*>(aux), static_cast<T_*>(st->rep), \
                                         st->rep_pos, d.n_kv_heads, static_cast<int>(bs),     \
                                         d.n_rep, n_aux, d.head_dim, sl2, d.capacity_tokens,  \
                                         st->cap_blocks, first_block);                        \
  } while (0)
      if (d.dtype == RBA_BF16) {
        if (D == 128) RBA_TOPR(__nv_bfloat16, 128); else RBA_TOPR(__nv_bfloat16, 64);
      } else {
        if (D == 128) RBA_TOPR(float, 128); else RBA_TOPR(float, 64);
      }
#undef RBA_TOPR
      RBA_LAUNCH_CHECK();
      break;
    }
    case RBA_REP_EXTERNAL: {
      if (aux == nullptr) return RBA_ERR_INVALID_ARG;
      const int64_t rows = int64_t(n_blocks) * d.n_rep;
      const rba_status s =
          copy_in(aux, st->rep, rows, st->cap_blocks * d.n_rep, first_block * d.n_rep);
      if (s != RBA_OK) return s;
      break;
    }
    case RBA_REP_EMBED_COSINE: {
      if (aux == nullptr) return RBA_ERR_INVALID_ARG;
      const int64_t rows = int64_t(d.batch) * n_blocks;
      const int threads = 256;
      const int g = static_cast<int>((rows * 32 + threads - 1) / threads);
      rep_embed_kernel<<<g, threads, 0, stream>>>(static_cast<const float*>(aux),
                                                  static_cast<float*>(st->rep), d.d_ret, rows,
                                                  n_blocks, st->cap_blocks, first_block);
      RBA_LAUNCH_CHECK();
      break;
    }
    case RBA_REP_IDENTITY:
      break;
  }
  return RBA_OK;
}
