// Host-side creation of TMA tensor maps.  cuTensorMapEncodeTiled is a driver
// function; it is fetched through the runtime's driver entry-point query so
// that the library does not link libcuda and still loads on a machine
// without a GPU driver.
#include <cudaTypedefs.h>

#include <mutex>

#include "fkv_internal.cuh"
#include "sm100_common.cuh"

namespace fkv {

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

bool make_tmap_bf16(CUtensorMap* map, const void* base, uint64_t rows, uint64_t slabs,
                    uint64_t row_stride_bytes, uint64_t slab_stride_bytes) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (!fn || !base || rows == 0 || slabs == 0) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15u) || (row_stride_bytes & 15u) ||
      (slab_stride_bytes & 15u))
    return false;
  cuuint64_t dims[3] = {128, rows, slabs};
  cuuint64_t strides[2] = {row_stride_bytes, slab_stride_bytes};
  cuuint32_t box[3] = {64, 128, 1};
  cuuint32_t elem_strides[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tmap_u8(CUtensorMap* map, const void* base, uint64_t rows, uint64_t slabs,
                  uint64_t row_stride_bytes, uint64_t slab_stride_bytes) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = encode_fn();
  if (!fn || !base || rows == 0 || slabs == 0) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15u) || (row_stride_bytes & 15u) ||
      (slab_stride_bytes & 15u))
    return false;
  cuuint64_t dims[3] = {128, rows, slabs};
  cuuint64_t strides[2] = {row_stride_bytes, slab_stride_bytes};
  cuuint32_t box[3] = {128, 128, 1};
  cuuint32_t elem_strides[3] = {1, 1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides,
                  box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

int num_sms() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

}  // namespace fkv
