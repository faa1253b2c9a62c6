// Host-side tensor-map encoding.  cuTensorMapEncodeTiled is a driver API function; it is fetched
// through the runtime's driver entry-point query so that libra.so does not link libcuda (it
// must load on machines without a GPU driver, e.g. to validate arguments or size workspaces).
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include "tma.cuh"

namespace ra {

bool encode_rows_tmap(CUtensorMap *out, const void *base, uint64_t cols, uint64_t rows,
                      uint64_t planes, uint32_t box_rows, uint64_t plane_rows) {
  static PFN_cuTensorMapEncodeTiled_v12000 encode = nullptr;
  if (encode == nullptr) {
    void *fn = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess || fn == nullptr)
      return false;
    encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  const cuuint64_t dims[3] = {cols, rows, planes};
  const cuuint64_t strides[2] = {cols * 2, cols * 2 * plane_rows};   // bytes, dims 1 and 2
  const cuuint32_t box[3] = {64, box_rows, 1};                 // 64 bf16 = one 128-byte row
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = encode(out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void *>(base),
                            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace ra
