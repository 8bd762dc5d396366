// Tensor-map encoding for the bulk tensor copies (through the driver entry
// point, so the library needs no link-time libcuda).
#include <mutex>

#include "rba_internal.cuh"

namespace rba {
namespace {

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                              const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                              const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(p);
  });
  return fn;
}

}  // namespace

bool make_tmap_bf16(CUtensorMap* m, const void* base, int64_t rows, int cols, int box_rows) {
  EncodeFn fn = encode_fn();
  if (fn == nullptr || base == nullptr || rows <= 0 || cols <= 0 || box_rows <= 0 ||
      box_rows > 256)
    return false;
  const cuuint64_t dims[2] = {cuuint64_t(cols), cuuint64_t(rows)};
  const cuuint64_t strides[1] = {cuuint64_t(cols) * 2};
  const cuuint32_t box[2] = {64, cuuint32_t(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

bool store_tmaps64(const rba_store* st, CUtensorMap* kmap, CUtensorMap* vmap) {
  std::call_once(st->tmap_once, [st] {
    const int64_t rows = int64_t(st->d.batch) * st->d.n_kv_heads * st->d.capacity_tokens;
    st->tmap_ok = make_tmap_bf16(&st->kmap64, st->k, rows, st->pitch, 64) &&
                  make_tmap_bf16(&st->vmap64, st->v, rows, st->pitch, 64);
  });
  if (!st->tmap_ok) return false;
  *kmap = st->kmap64;
  *vmap = st->vmap64;
  return true;
}

}  // namespace rba
