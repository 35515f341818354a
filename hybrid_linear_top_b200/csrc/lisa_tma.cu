// Host-side construction of TMA tensor maps (cuTensorMapEncodeTiled, reached
// through the runtime's driver entry point so the library does not link the
// driver API).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <mutex>

#include "lisa_internal.h"

namespace lisa {

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    cudaGetLastError();
  });
  return fn;
}

bool make_tmap(CUtensorMap *map, const void *base, int elem_bytes, int rank, const unsigned long long *dims,
               const unsigned long long *strides_bytes, const unsigned *box, int swizzle_bytes) {
  auto fn = encode_fn();
  if (!fn || rank < 1 || rank > 5) return false;
  const CUtensorMapDataType dt = elem_bytes == 2 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  cuuint64_t d[5], st[4];
  cuuint32_t bx[5], es[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
    es[i] = 1;
  }
  for (int i = 0; i + 1 < rank; ++i) st[i] = strides_bytes[i];
  const CUtensorMapSwizzle sw = swizzle_bytes == 128  ? CU_TENSOR_MAP_SWIZZLE_128B
                                : swizzle_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                : swizzle_bytes == 32 ? CU_TENSOR_MAP_SWIZZLE_32B
                                                      : CU_TENSOR_MAP_SWIZZLE_NONE;
  const CUresult r = fn(map, dt, (cuuint32_t)rank, const_cast<void *>(base), d, st, bx, es,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_2d(CUtensorMap *map, const void *base, int elem_bytes, unsigned long long cols,
                  unsigned long long rows, unsigned long long row_stride_bytes, unsigned box_cols, unsigned box_rows,
                  int swizzle_bytes) {
  const unsigned long long dims[2] = {cols, rows};
  const unsigned long long strides[1] = {row_stride_bytes};
  const unsigned box[2] = {box_cols, box_rows};
  return make_tmap(map, base, elem_bytes, 2, dims, strides, box, swizzle_bytes);
}

}  // namespace lisa
