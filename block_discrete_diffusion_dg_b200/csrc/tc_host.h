// Host helpers of the tensor-core kernels (tc_host.cu).
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace dg {

// 2-D tensor map over a row-major matrix [rows][inner] with the 128-byte swizzle, box
// [box_rows][box_inner].  Out-of-range boxes read zeros.  Returns DG_OK or an error code.
int make_tmap_2d(CUtensorMap *out, CUtensorMapDataType dtype, int elem_bytes, const void *base,
                 uint64_t inner, uint64_t rows, uint64_t row_stride_bytes, uint32_t box_inner,
                 uint32_t box_rows);

// 3-D tensor map over fp32 [d2][d1][d0] (d0 contiguous), no swizzle, box [b2][b1][b0]; for tiled
// stores from shared memory laid out [b1][b0].
int make_tmap_3d_f32(CUtensorMap *out, const void *base, uint64_t d0, uint64_t d1, uint64_t d2,
                     uint32_t b0, uint32_t b1, uint32_t b2);

// Streaming multiprocessors of the current device.
int num_sms();

}  // namespace dg
