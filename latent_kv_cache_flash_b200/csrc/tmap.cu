// Tensor maps for the TMA loads of the tensor-core kernels.
#include <cudaTypedefs.h>

#include "tc.h"

namespace gqla {

namespace {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// The driver's encoder, looked up once through the runtime (no libcuda link).
EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)f;
  }
  return fn;
}

}  // namespace

bool tmap_bf16_sw128(CUtensorMap* map, const void* base, long long cols, long long rows, long long row_pitch_elems,
                     int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)row_pitch_elems * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), gdim, gstride, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool gqa_pool_maps(const Problem& p, const void* k_pool, const void* v_pool, CUtensorMap* kmap, CUtensorMap* vmap) {
  const long long nrows = p.ly.page_size == 0 ? (long long)p.ly.batch * p.ly.capacity
                                              : (long long)p.ly.num_pages * p.ly.page_size;
  const long long vpitch = (long long)p.d.G * p.d.d_v;
  return tmap_bf16_sw128(kmap, k_pool, p.kr.pitch, nrows, p.kr.pitch, 64) &&
         tmap_bf16_sw128(vmap, v_pool, vpitch, nrows, vpitch, 64);
}

}  // namespace gqla
