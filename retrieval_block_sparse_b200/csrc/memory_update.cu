// Dynamic memory update of a block store, after "MemLong: Memory-Augmented
// Retrieval for Long Text Modeling", section 2.3.2 (dynamic memory update):
// retrieval-frequency counters, and on overflow a counter-driven prune that
// keeps the newest entries, drops the oldest, and deletes the least retrieved
// of the middle until the requested number of entries remains.
//
//   retrieval_count_kernel  counters[u][j] += 1 for every selected block j of unit u
//   memory_select_kernel    one CTA per memory unit: radix select of the keep
//                           threshold on the 32-bit counts, then an ordered scan
//                           that writes the keep map (destination -> source block)
//   memory_move_kernel      in-place compaction, one launch per round of destinations,
//                           each a programmatic dependent of the kernel before it
//                           (a CTA copies 32 KB of one block, 8 loads in flight a thread)
//   memory_finish_kernel    moves the partial tail block, zeroes vacated counters
//
// In-place safety.  The keep map is strictly increasing and every kept entry
// t moves from block map[t] >= pinned + drop_oldest + t to block pinned + t,
// so each move spans at least g = drop_oldest blocks.  A round moves the
// destinations [t0, t0 + g): it writes blocks [pinned + t0, pinned + t0 + g)
// and reads blocks >= pinned + t0 + g, none of which a round writes before the
// source has been read (later rounds read higher blocks still); a round of
// fewer destinations is safe all the more.  With drop_oldest = 0 a round
// moves one entry.
#include "rba_internal.cuh"

namespace rba {
namespace {

constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kMoveThreads = 256;
constexpr int kMoveWarps = kMoveThreads / 32;
constexpr int kMoveVecs = 8;                           // loads in flight per thread
constexpr int kChunkVecs = kMoveThreads * kMoveVecs;   // vectors a CTA copies (32 KB)
constexpr int64_t kMaxMoveCtas = int64_t(1) << 30;      // K/V CTAs of one launch

int grid_cap(int64_t work, int threads) {
  int64_t g = (work + threads - 1) / threads;
  const int64_t cap = int64_t(num_sms()) * 16;
  if (g > cap) g = cap;
  return static_cast<int>(g < 1 ? 1 : g);
}

__global__ void retrieval_count_kernel(const int32_t* __restrict__ idx, int64_t n, int32_t k,
                                       int32_t units, int64_t cap_blocks,
                                       uint32_t* __restrict__ counters, int32_t* status) {
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += stride) {
    const int32_t j = idx[i];
    if (j < 0 || j >= cap_blocks) {
      report(status, RBA_ERR_BOUNDS, kWhereMemory, j);
      continue;
    }
    const int64_t u = (i / k) % units;
    atomicAdd(counters + u * cap_blocks + j, 1u);
  }
}

// Exclusive count of `flag` over the CTA's threads in thread order; *total
// receives the CTA's count.  Every thread of the CTA must call it.
__device__ __forceinline__ uint32_t cta_exclusive(bool flag, uint32_t* swarp, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned b = __ballot_sync(0xffffffffu, flag);
  if (lane == 0) swarp[warp] = __popc(b);
  __syncthreads();
  uint32_t before = 0, all = 0;
#pragma unroll 8
  for (int w = 0; w < kSelWarps; ++w) {
    const uint32_t c = swarp[w];
    before += w < warp ? c : 0u;
    all += c;
  }
  __syncthreads();
  *total = all;
  return before + __popc(b & ((1u << lane) - 1u));
}

// Keep map of one memory unit (blockIdx.x).  Middle entries are blocks
// [lo, lo + mid); kk of them are kept: those with the most retrievals, and
// among equal counts the newest.  map[0..kk) = kept middle blocks ascending,
// map[kk..kk + keep_newest) = the newest blocks [hi, hi + keep_newest).
__global__ void __launch_bounds__(kSelThreads)
    memory_select_kernel(const uint32_t* __restrict__ counters, int64_t cap_blocks, int32_t lo,
                  int32_t mid, int32_t kk, int32_t hi, int32_t keep_newest, int32_t keep_total,
                  int32_t* __restrict__ keep_map) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t swarp[kSelWarps];
  __shared__ uint32_t s_digit, s_rem;
  // the first move kernel may become resident now (it waits for our completion)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int tid = threadIdx.x;
  const uint32_t* cnt = counters + int64_t(blockIdx.x) * cap_blocks + lo;
  int32_t* map = keep_map + int64_t(blockIdx.x) * keep_total;

  // threshold count thr = the kk-th largest count of the middle; `need` of
  // the n_eq entries whose count equals thr are kept (the newest ones)
  const bool keep_none = kk == 0, keep_all = kk == mid;
  uint32_t thr = 0, need = 0, n_eq = 0;
  if (!keep_none && !keep_all) {
    // digits above the largest count's top digit are zero for every entry:
    // the select starts at that digit
    uint32_t cmax = 0;
    for (int64_t i = tid; i < mid; i += kSelThreads) cmax = max(cmax, cnt[i]);
    cmax = __reduce_max_sync(0xffffffffu, cmax);
    if ((tid & 31) == 0) swarp[tid >> 5] = cmax;
    __syncthreads();
    if (tid < 32) {
      uint32_t m = tid < kSelWarps ? swarp[tid] : 0u;
      m = __reduce_max_sync(0xffffffffu, m);
      if (tid == 0) s_digit = m;
    }
    __syncthreads();
    cmax = s_digit;
    int top = 0;
    while (top < 24 && (cmax >> (top + 8)) != 0u) top += 8;
    uint32_t prefix = 0, mask = 0, rem = static_cast<uint32_t>(kk);
    for (int shift = top; shift >= 0; shift -= 8) {
      for (int i = tid; i < 256; i += kSelThreads) hist[i] = 0;
      __syncthreads();
      for (int64_t base = 0; base < mid; base += kSelThreads) {
        const int64_t i = base + tid;
        const uint32_t c = i < mid ? cnt[i] : 0u;
        const int bin = (i < mid && (c & mask) == prefix) ? int((c >> shift) & 255u) : 256;
        const unsigned peers = __match_any_sync(0xffffffffu, bin);
        if (bin < 256 && (tid & 31) == __ffs(peers) - 1) atomicAdd(&hist[bin], __popc(peers));
      }
      __syncthreads();
      if (tid < 32) {
        // the highest digit d >= 1 whose suffix count S(d) = sum_{i >= d} hist[i]
        // reaches rem (else 0); lane l holds bins [8 l, 8 l + 8)
        uint32_t h8[8], own = 0;
#pragma unroll
        for (int b = 0; b < 8; ++b) {
          h8[b] = hist[tid * 8 + b];
          own += h8[b];
        }
        uint32_t incl = own;  // sum over lanes >= tid
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const uint32_t y = __shfl_down_sync(0xffffffffu, incl, o);
          if (tid + o < 32) incl += y;
        }
        uint32_t suf = incl - own;  // S(8 tid + 8)
        int found = -1;
        uint32_t above = 0;
#pragma unroll
        for (int b = 7; b >= 0; --b) {
          const int d = tid * 8 + b;
          if (found < 0 && d >= 1 && suf + h8[b] >= rem) {
            found = d;
            above = suf;
          }
          suf += h8[b];
        }
        const unsigned hits = __ballot_sync(0xffffffffu, found >= 0);
        if (hits == 0u) {
          if (tid == 0) {  // digit 0: every entry of bins 1..255 is above
            s_digit = 0;
            s_rem = rem - (incl - h8[0]);
          }
        } else if (tid == 31 - __clz(hits)) {
          s_digit = static_cast<uint32_t>(found);
          s_rem = rem - above;
        }
      }
      __syncthreads();
      prefix |= s_digit << shift;
      mask |= 255u << shift;
      rem = s_rem;
    }
    thr = prefix;
    need = rem;
    n_eq = hist[thr & 255u];  // the last pass counted exactly the entries equal to thr
  }

  if (!keep_none) {
    uint32_t eq_base = 0, keep_base = 0;
    for (int64_t base = 0; base < mid; base += kSelThreads) {
      const int64_t i = base + tid;
      const bool valid = i < mid;
      const uint32_t c = valid ? cnt[i] : 0u;
      const bool eq = valid && !keep_all && c == thr;
      uint32_t eq_total, keep_total_tile;
      const uint32_t eq_rank = eq_base + cta_exclusive(eq, swarp, &eq_total);
      const bool keep = valid && (keep_all || c > thr || (eq && eq_rank >= n_eq - need));
      const uint32_t pos = keep_base + cta_exclusive(keep, swarp, &keep_total_tile);
      if (keep && pos < static_cast<uint32_t>(kk)) map[pos] = static_cast<int32_t>(lo + i);
      eq_base += eq_total;
      keep_base += keep_total_tile;
    }
  }
  for (int j = tid; j < keep_newest; j += kSelThreads) map[kk + j] = hi + j;
}

struct MoveArgs {
  uint4* k;               // K pool as 16-byte vectors
  uint4* v;               // V pool
  int64_t cap_tokens;     // tokens per (batch, kv head)
  int32_t bs;             // block size
  int32_t row_vecs;       // 16-byte vectors per token row
  int32_t heads;          // kv heads per memory unit (all of them for the cosine bank, else 1)
  int32_t units;          // memory units
  uint32_t* rep;          // representation pool as 4-byte words, or null
  int32_t rep_words;      // words per block in the representation pool
  int32_t* rep_pos;       // representative positions, or null
  int32_t pos_words;      // positions per block
  uint32_t* counters;     // [units][cap_blocks]
  int64_t cap_blocks;
  const int32_t* keep_map;  // [units][keep_total]
  int32_t keep_total;
  int32_t pinned;         // blocks in front of the memory entries (never move)
  int32_t nb;             // full blocks before the update: every source is below it
  int32_t* status;        // store status word
};

// A keep-map entry is a valid source for destination dst iff dst <= src < nb;
// anything else is reported and skipped, so no access leaves the pools.
__device__ __forceinline__ bool source_ok(const MoveArgs& a, int32_t src, int32_t dst) {
  if (src >= dst && src < a.nb) return true;
  report(a.status, RBA_ERR_BOUNDS, kWhereMemory, src);
  return false;
}

// Launched as a programmatic dependent of the previous kernel of the update:
// it may become resident early, but touches no memory before that kernel has
// completed; it lets the next kernel do the same.
__device__ __forceinline__ void chain_entry() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Moves destinations [t0, t0 + nt) of every unit (see the safety note above).
// CTAs [0, word_ctas) come first (scheduled first, so they are not a round's
// tail): warp w of CTA b copies the per-block words of destination 8 b + w
// (representation, positions, counter), kMoveVecs loads in flight a lane.
// The other CTAs copy K/V rows: a row is one (unit, destination, head, K or
// V) block, bs * row_vecs contiguous 16-byte vectors at both ends, `chunks`
// CTAs a row, each thread holding kMoveVecs loads in flight before its stores.
// All index arithmetic is once per CTA or warp, in 32 bits.
__global__ void __launch_bounds__(kMoveThreads)
    memory_move_kernel(MoveArgs a, int32_t t0, int32_t nt, int32_t chunks, int32_t word_ctas) {
  chain_entry();
  const int tid = threadIdx.x;
  if (static_cast<int32_t>(blockIdx.x) < word_ctas) {
    const int lane = tid & 31;
    const uint32_t di = blockIdx.x * kMoveWarps + (tid >> 5);
    if (di >= static_cast<uint32_t>(a.units) * static_cast<uint32_t>(nt)) return;
    const uint32_t u = di / static_cast<uint32_t>(nt);
    const int32_t t = t0 + static_cast<int32_t>(di - u * static_cast<uint32_t>(nt));
    const int32_t src = a.keep_map[int64_t(u) * a.keep_total + t];
    const int32_t dst = a.pinned + t;
    if (src == dst || !source_ok(a, src, dst)) return;
    const int64_t b0 = int64_t(u) * a.cap_blocks;
    if (a.rep_words > 0) {
      const uint32_t* from = a.rep + (b0 + src) * a.rep_words;
      uint32_t* to = a.rep + (b0 + dst) * a.rep_words;
      for (int32_t base = 0; base < a.rep_words; base += 32 * kMoveVecs) {
        uint32_t w[kMoveVecs];
#pragma unroll
        for (int j = 0; j < kMoveVecs; ++j) {
          const int32_t i = base + j * 32 + lane;
          if (i < a.rep_words) w[j] = from[i];
        }
#pragma unroll
        for (int j = 0; j < kMoveVecs; ++j) {
          const int32_t i = base + j * 32 + lane;
          if (i < a.rep_words) to[i] = w[j];
        }
      }
    }
    for (int32_t i = lane; i < a.pos_words; i += 32)
      a.rep_pos[(b0 + dst) * a.pos_words + i] = a.rep_pos[(b0 + src) * a.pos_words + i];
    if (lane == 0) a.counters[b0 + dst] = a.counters[b0 + src];
    return;
  }
  const uint32_t row = (blockIdx.x - static_cast<uint32_t>(word_ctas)) / static_cast<uint32_t>(chunks);
  const uint32_t chunk =
      blockIdx.x - static_cast<uint32_t>(word_ctas) - row * static_cast<uint32_t>(chunks);
  const uint32_t kv = row & 1u;
  const uint32_t r = row >> 1;
  const uint32_t uh = r / static_cast<uint32_t>(a.heads);  // unit * nt + (t - t0)
  const uint32_t h = r - uh * static_cast<uint32_t>(a.heads);
  const uint32_t u = uh / static_cast<uint32_t>(nt);
  const int32_t t = t0 + static_cast<int32_t>(uh - u * static_cast<uint32_t>(nt));
  const int32_t src = a.keep_map[int64_t(u) * a.keep_total + t];
  const int32_t dst = a.pinned + t;
  if (src == dst || !source_ok(a, src, dst)) return;
  uint4* pool = kv ? a.v : a.k;
  const int64_t row0 = (int64_t(u) * a.heads + h) * a.cap_tokens;
  const uint4* from = pool + (row0 + int64_t(src) * a.bs) * a.row_vecs;
  uint4* to = pool + (row0 + int64_t(dst) * a.bs) * a.row_vecs;
  const int32_t blk_vecs = a.bs * a.row_vecs;
  const int32_t e0 = static_cast<int32_t>(chunk) * kChunkVecs + tid;
  uint4 v[kMoveVecs];
#pragma unroll
  for (int j = 0; j < kMoveVecs; ++j) {
    const int32_t e = e0 + j * kMoveThreads;
    if (e < blk_vecs) v[j] = ld_stream(from + e);
  }
#pragma unroll
  for (int j = 0; j < kMoveVecs; ++j) {
    const int32_t e = e0 + j * kMoveThreads;
    if (e < blk_vecs) to[e] = v[j];
  }
}

// The partial tail block's `tail` tokens move from block src_blk to block
// dst_blk (disjoint: dst_blk < src_blk); counters of blocks [clear_from,
// clear_to) are zeroed.
__global__ void __launch_bounds__(kMoveThreads)
    memory_finish_kernel(MoveArgs a, int32_t src_blk, int32_t dst_blk, int32_t tail,
                         int32_t clear_from, int32_t clear_to) {
  chain_entry();
  const int64_t stride = int64_t(gridDim.x) * blockDim.x;
  const int64_t first = int64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t tail_vecs = int64_t(tail) * a.row_vecs;
  const int64_t total = int64_t(a.units) * a.heads * 2 * tail_vecs;
  for (int64_t i = first; i < total; i += stride) {
    int64_t r = i / tail_vecs;
    const int64_t e = i - r * tail_vecs;
    const int kv = static_cast<int>(r & 1);
    r >>= 1;  // r = unit * heads + head
    uint4* pool = kv ? a.v : a.k;
    const int64_t row0 = r * a.cap_tokens;
    pool[(row0 + int64_t(dst_blk) * a.bs) * a.row_vecs + e] =
        pool[(row0 + int64_t(src_blk) * a.bs) * a.row_vecs + e];
  }
  const int64_t span = int64_t(clear_to) - clear_from;
  for (int64_t i = first; i < int64_t(a.units) * span; i += stride) {
    const int64_t u = i / span;
    a.counters[u * a.cap_blocks + clear_from + (i - u * span)] = 0u;
  }
}

// Launches kernel (kMoveThreads threads) as a programmatic dependent of the
// stream's previous kernel; the kernel begins with chain_entry().
template <typename... KArgs, typename... Args>
cudaError_t launch_chained(void (*kernel)(KArgs...), dim3 grid, cudaStream_t stream,
                           Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kMoveThreads);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

int32_t units_of(const rba_store* st) {
  const rba_store_desc& d = st->d;
  return d.mode == RBA_REP_EMBED_COSINE ? d.batch : d.batch * d.n_kv_heads;
}

}  // namespace
}  // namespace rba

extern "C" rba_status rba_memory_rule(int64_t n_entries, int64_t* keep_newest,
                                      int64_t* drop_oldest, int64_t* keep_total) {
  if (n_entries < 0 || keep_newest == nullptr || drop_oldest == nullptr || keep_total == nullptr)
    return RBA_ERR_INVALID_ARG;
  *keep_newest = n_entries / 10;
  *drop_oldest = n_entries / 10;
  *keep_total = n_entries / 2;
  return RBA_OK;
}

extern "C" int32_t rba_memory_units(const rba_store* st) {
  return st == nullptr ? -1 : rba::units_of(st);
}

extern "C" rba_status rba_count_retrievals(const rba_store* st, const int32_t* idx, int32_t rows,
                                           int32_t k, uint32_t* counters, cudaStream_t stream) {
  using namespace rba;
  if (st == nullptr || counters == nullptr || rows < 0 || k < 0) return RBA_ERR_INVALID_ARG;
  const int32_t units = units_of(st);
  if (rows % units != 0) return RBA_ERR_INVALID_ARG;
  const int64_t n = int64_t(rows) * k;
  if (n == 0) return RBA_OK;
  if (idx == nullptr) return RBA_ERR_INVALID_ARG;
  retrieval_count_kernel<<<grid_cap(n, 256), 256, 0, stream>>>(idx, n, k, units,
                                                               st->cap_blocks, counters,
                                                               st->status);
  RBA_LAUNCH_CHECK();
  return RBA_OK;
}

extern "C" rba_status rba_memory_update(rba_store* st, int64_t T, int32_t pinned_blocks,
                                        int64_t keep_newest, int64_t drop_oldest,
                                        int64_t keep_total, uint32_t* counters,
                                        int32_t* keep_map, int64_t* T_new, cudaStream_t stream) {
  using namespace rba;
  if (st == nullptr || counters == nullptr) return RBA_ERR_INVALID_ARG;
  const rba_store_desc& d = st->d;
  if (T < 0 || T > d.capacity_tokens) return RBA_ERR_INVALID_ARG;
  const int64_t bs = d.block_size;
  const int64_t nb = T / bs;
  const int64_t tail = T - nb * bs;
  if (nb >= (int64_t(1) << 31) - 1) return RBA_ERR_UNSUPPORTED;
  if (pinned_blocks < 0 || pinned_blocks > nb) return RBA_ERR_INVALID_ARG;
  const int64_t n = nb - pinned_blocks;
  if (keep_newest < 0 || drop_oldest < 0 || keep_newest + drop_oldest > n ||
      keep_total < keep_newest || keep_total > n - drop_oldest)
    return RBA_ERR_INVALID_ARG;
  if (keep_total > 0 && keep_map == nullptr) return RBA_ERR_INVALID_ARG;
  const int64_t new_nb = pinned_blocks + keep_total;
  if (T_new != nullptr) *T_new = new_nb * bs + tail;

  const int32_t units = units_of(st);
  const int64_t lo = pinned_blocks + drop_oldest;
  const int64_t hi = nb - keep_newest;
  const int64_t kk = keep_total - keep_newest;

  MoveArgs a;
  a.k = static_cast<uint4*>(st->k);
  a.v = static_cast<uint4*>(st->v);
  a.cap_tokens = d.capacity_tokens;
  a.bs = static_cast<int32_t>(bs);
  a.row_vecs = static_cast<int32_t>(st->pitch * dtype_size(d.dtype) / 16);
  a.heads = d.mode == RBA_REP_EMBED_COSINE ? d.n_kv_heads : 1;
  a.units = units;
  a.rep = static_cast<uint32_t*>(st->rep);
  switch (d.mode) {
    case RBA_REP_MEAN: a.rep_words = st->pitch; break;
    case RBA_REP_TOPR_ATTN:
    case RBA_REP_EXTERNAL:
      a.rep_words = static_cast<int32_t>(d.n_rep * st->pitch * dtype_size(d.dtype) / 4);
      break;
    case RBA_REP_EMBED_COSINE: a.rep_words = d.d_ret; break;
    default: a.rep_words = 0;
  }
  if (a.rep == nullptr) a.rep_words = 0;
  a.rep_pos = d.mode == RBA_REP_TOPR_ATTN ? st->rep_pos : nullptr;
  a.pos_words = a.rep_pos != nullptr ? d.n_rep : 0;
  a.counters = counters;
  a.cap_blocks = st->cap_blocks;
  a.keep_map = keep_map;
  a.keep_total = static_cast<int32_t>(keep_total);
  a.pinned = pinned_blocks;
  a.nb = static_cast<int32_t>(nb);
  a.status = st->status;

  if (keep_total > 0) {
    memory_select_kernel<<<units, kSelThreads, 0, stream>>>(
        counters, st->cap_blocks, static_cast<int32_t>(lo), static_cast<int32_t>(hi - lo),
        static_cast<int32_t>(kk), static_cast<int32_t>(hi), static_cast<int32_t>(keep_newest),
        static_cast<int32_t>(keep_total), keep_map);
    RBA_LAUNCH_CHECK();
    // rounds of at most drop_oldest destinations (every kept entry moves by at
    // least that many blocks), as many as that takes and as even as possible
    // (no short last round).  A round may be cut into several launches: each
    // moves a subset of the round's destinations, whose sources none of them writes.
    const int64_t g_max = drop_oldest > 0 ? drop_oldest : 1;
    const int64_t n_rounds = (keep_total + g_max - 1) / g_max;
    const int64_t g = n_rounds > 0 ? (keep_total + n_rounds - 1) / n_rounds : g_max;
    const int64_t blk_vecs = bs * a.row_vecs;
    if (blk_vecs > INT32_MAX - kChunkVecs) return RBA_ERR_UNSUPPORTED;
    const int64_t chunks = (blk_vecs + kChunkVecs - 1) / kChunkVecs;
    const int64_t ctas_per_dest = int64_t(units) * a.heads * 2 * chunks;
    if (ctas_per_dest > kMaxMoveCtas) return RBA_ERR_UNSUPPORTED;
    const int64_t max_nt = kMaxMoveCtas / ctas_per_dest;
    for (int64_t t0 = 0; t0 < keep_total; t0 += g) {
      const int64_t round_end = t0 + g < keep_total ? t0 + g : keep_total;
      for (int64_t s0 = t0; s0 < round_end; s0 += max_nt) {
        const int64_t nt = round_end - s0 < max_nt ? round_end - s0 : max_nt;
        const int64_t word_ctas = (int64_t(units) * nt + kMoveWarps - 1) / kMoveWarps;
        const int64_t ctas = nt * ctas_per_dest + word_ctas;
        if (ctas > INT32_MAX) return RBA_ERR_UNSUPPORTED;
        RBA_CUDA_TRY(launch_chained(memory_move_kernel, dim3(static_cast<unsigned>(ctas)), stream,
                                    a, static_cast<int32_t>(s0), static_cast<int32_t>(nt),
                                    static_cast<int32_t>(chunks),
                                    static_cast<int32_t>(word_ctas)));
      }
    }
  }
  const int64_t clear_to = nb + 1 < st->cap_blocks ? nb + 1 : st->cap_blocks;
  const bool move_tail = tail > 0 && new_nb < nb;
  if (move_tail || clear_to > new_nb) {
    const int64_t work = units * a.heads * 2 * (move_tail ? tail : 0) * a.row_vecs +
                         units * (clear_to > new_nb ? clear_to - new_nb : 0);
    RBA_CUDA_TRY(launch_chained(
        memory_finish_kernel, dim3(grid_cap(work, kMoveThreads)), stream, a,
        static_cast<int32_t>(nb), static_cast<int32_t>(new_nb),
        static_cast<int32_t>(move_tail ? tail : 0), static_cast<int32_t>(new_nb),
        static_cast<int32_t>(clear_to > new_nb ? clear_to : new_nb)));
  }
  return RBA_OK;
}
