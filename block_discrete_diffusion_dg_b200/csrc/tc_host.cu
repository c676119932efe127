// Host helpers of the tensor-core kernels: TMA tensor-map encoding through the driver entry
// point (no link-time dependency on libcuda) and the device's SM count.
#include <cudaTypedefs.h>

#include <cstdio>
#include <mutex>

#include "dg_common.cuh"
#include "tc_host.h"

namespace dg {

static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
static std::once_flag g_encode_once;

static void load_encode() {
  void *fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
}

int make_tmap_2d(CUtensorMap *out, CUtensorMapDataType dtype, int elem_bytes, const void *base,
                 uint64_t inner, uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner,
                 uint32_t box_rows) {
  std::call_once(g_encode_once, load_encode);
  if (!g_encode) return DG_ERR_CUDA;
  if (((uintptr_t)base & 15) || (row_stride_bytes & 15) || ((box_inner * elem_bytes) & 15))
    return DG_ERR_INVALID_ARG;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {row_stride_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = g_encode(out, dtype, 2, const_cast<void *>(base), dims, strides, box, estr,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DG_OK : DG_ERR_INVALID_ARG;
}

int make_tmap_3d_f32(CUtensorMap *out, const void *base, uint64_t d0, uint64_t d1, uint64_t d2,
                     uint32_t b0, uint32_t b1, uint32_t b2) {
  std::call_once(g_encode_once, load_encode);
  if (!g_encode) return DG_ERR_CUDA;
  if (((uintptr_t)base & 15) || ((d0 * 4) & 15) || ((b0 * 4) & 15)) return DG_ERR_INVALID_ARG;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 4, d0 * d1 * 4};
  cuuint32_t box[3] = {b0, b1, b2};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = g_encode(out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void *>(base),
                              dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? DG_OK : DG_ERR_INVALID_ARG;
}

int num_sms() {
  static int n = 0;
  if (n == 0) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

}  // namespace dg
