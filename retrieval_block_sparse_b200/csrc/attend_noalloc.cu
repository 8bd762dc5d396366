// rba_attend_noalloc: decode attention whose scratch is a fixed device array
// inside the library, for callers that cannot allocate device memory.
//
// Some hosts own every byte of device memory through their own allocator (a
// serving engine that reserves HBM when it starts), and some call sites cannot
// afford the implicit device-wide synchronisation that cudaMalloc may cause.
// Such callers still pass their inputs and outputs, but cannot provide the
// split-K workspace that rba_attend asks for.  This entry point keeps that
// scratch (split partials and merge tickets) in the file-scope array below.
#include <mutex>

#include "attend_impl.cuh"

namespace rba {
namespace {

constexpr size_t kScratchBytes = RBA_ATTEND_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// Zero-initialised when the module loads; every GPU that loads the library
// holds it until the process exits.  In host code this name is only a
// stand-in: its device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_attend_scratch[kScratchBytes];

std::mutex g_mu;
void* g_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device, looked up once
// per device (with that device current).
rba_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return RBA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_attend_scratch) != cudaSuccess || p == nullptr)
      return RBA_ERR_CUDA;
    g_ptr[dev] = p;
  }
  *out = g_ptr[dev];
  return RBA_OK;
}

}  // namespace
}  // namespace rba

extern "C" rba_status rba_attend_noalloc(const rba_store* st, const void* q, const int32_t* idx,
                                         int32_t k, int64_t T, int32_t sink, int32_t window,
                                         float scale, float* out, float* lse,
                                         cudaStream_t stream) {
  using namespace rba;
  if (st == nullptr || q == nullptr || out == nullptr || k < 0) return RBA_ERR_INVALID_ARG;
  if (st->d.mode == RBA_REP_EMBED_COSINE) return RBA_ERR_INVALID_ARG;
  Geometry g;
  rba_status s = geometry(st, T, sink, window, &g);
  if (s != RBA_OK) return s;
  if (k > g.nc || (k > 0 && idx == nullptr)) return RBA_ERR_INVALID_ARG;
  // reject sizes whose scratch does not fit the fixed array
  const size_t need = splitk_workspace_bytes(st, g, k);
  if (need == 0 || need > kScratchBytes) return RBA_ERR_WORKSPACE;
  void* scratch = nullptr;
  s = scratch_address(&scratch);
  if (s != RBA_OK) return s;
  // the merge tickets (start of the scratch) must be zero; the array keeps
  // whatever the previous call left, so clear them on this stream
  const size_t ticket_bytes =
      align_up(size_t(st->d.batch) * st->d.n_kv_heads * sizeof(uint32_t), 256);
  RBA_CUDA_TRY(cudaMemsetAsync(scratch, 0, ticket_bytes, stream));
  return launch_attend(st, q, idx, k, g, scale, out, lse, scratch, kScratchBytes, stream);
}
