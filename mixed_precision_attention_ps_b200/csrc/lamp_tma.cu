// Host side of the TMA tile loads: tensor maps of the attention inputs.
//
// The encoder (cuTensorMapEncodeTiled) is a CUDA driver function; the library
// links the runtime only, so its address is looked up once through the runtime's
// driver entry-point query.
#include <cudaTypedefs.h>

#include <mutex>

#include "lamp_kernels.h"

namespace lamp {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
cudaError_t g_encode_err = cudaSuccess;
std::once_flag g_encode_once;

cudaError_t encoder(PFN_cuTensorMapEncodeTiled_v12000& fn) {
  std::call_once(g_encode_once, []() {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    g_encode_err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q);
    if (g_encode_err == cudaSuccess && (q != cudaDriverEntryPointSuccess || !f)) g_encode_err = cudaErrorNotSupported;
    if (g_encode_err != cudaSuccess) (void)cudaGetLastError();  // keep the failed query out of the caller's state
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  fn = g_encode;
  return g_encode_err;
}

}  // namespace

cudaError_t make_tmap_bf16(CUtensorMap* map, const void* base, int d, int n, int bh, int box_x, int box_y,
                           int swizzle) {
  PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  cudaError_t e = encoder(fn);
  if (e != cudaSuccess) return e;
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)n, (cuuint64_t)bh};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)n * d * 2};  // bytes, dimensions 1 and 2
  const cuuint32_t box[3] = {(cuuint32_t)box_x, (cuuint32_t)box_y, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE,
                        swizzle == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                       : (swizzle == 32 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_NONE),
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace lamp
