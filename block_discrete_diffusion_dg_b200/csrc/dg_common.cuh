// Shared device helpers of the canvas-step library: element types, the device status word,
// warp/block reductions and the launch bookkeeping used by every kernel file.
#pragma once

#include <utility>

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_fp4.h>
#include <stdint.h>

#include "../../include/dg.h"

namespace dg {

using bf16 = __nv_bfloat16;
using fp8 = __nv_fp8_e4m3;

// ---- element conversion -------------------------------------------------------------------
__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(bf16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float to_f(fp8 v) { return float(v); }

template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float v) { return __float2bfloat16_rn(v); }
template <> __device__ __forceinline__ __half from_f<__half>(float v) { return __float2half_rn(v); }

// Round an fp32 value to the storage type and back (what a store/load round trip yields).
template <typename T> __device__ __forceinline__ float round_to(float v) { return to_f(from_f<T>(v)); }

// NVFP4 elements: two FP4 E2M1 codes of a byte (low nibble first) times their FP8 E4M3 block
// scale, as fp16 (exact: the products have at most 5 significant bits and lie in [2^-10, 2688]).
__device__ __forceinline__ __half2 nvfp4_pair_f16(uint32_t byte, __half2 scale2) {
  const __half2_raw r = __nv_cvt_fp4x2_to_halfraw2((__nv_fp4x2_storage_t)(byte & 0xFFu), __NV_E2M1);
  return __hmul2(*reinterpret_cast<const __half2 *>(&r), scale2);
}
// Four bytes of FP4 E2M1 code pairs (byte k = columns 2k, 2k + 1; low nibble first) to four
// f16x2, each times its scale pair (exact, as nvfp4_pair_f16): the word is split into its bytes
// by one mov, so no shifts per pair.
__device__ __forceinline__ void nvfp4_word_f16(uint32_t w, __half2 scale2, uint32_t (&o)[4]) {
  uint32_t h0, h1, h2, h3;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h0), "=r"(h1), "=r"(h2), "=r"(h3)
      : "r"(w));
  const uint32_t hs[4] = {h0, h1, h2, h3};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const __half2 v = __hmul2(*reinterpret_cast<const __half2 *>(&hs[k]), scale2);
    o[k] = *reinterpret_cast<const uint32_t *>(&v);
  }
}
// Two FP8 E4M3 scales (the low two bytes of `codes`) to f16 (exact), each duplicated into a pair.
__device__ __forceinline__ void e4m3_scales_f16x2(uint32_t codes, __half2 &s0, __half2 &s1) {
  uint32_t h;
  asm("{\n\t.reg .b16 lo, hi;\n\t"
      "mov.b32 {lo, hi}, %1;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, lo;\n\t}"
      : "=r"(h)
      : "r"(codes));
  const __half2 p = *reinterpret_cast<const __half2 *>(&h);
  s0 = __low2half2(p);
  s1 = __high2half2(p);
}
__device__ __forceinline__ __half2 e4m3_scale_f16x2(uint32_t code) {
  const __half_raw r = __nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)(code & 0xFFu), __NV_E4M3);
  const __half h = *reinterpret_cast<const __half *>(&r);
  return __halves2half2(h, h);
}

// ---- device status word ------------------------------------------------------------------
// First error wins; later errors leave the word alone.
__device__ __forceinline__ void set_status(int32_t *st, int code) {
  if (st) atomicCAS(st, 0, code);
}

// ---- reductions ---------------------------------------------------------------------------
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block-wide sum in a fixed order (deterministic); `red` needs blockDim.x/32 floats.
__device__ __forceinline__ float block_sum(float v, float *red) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[w] = v;
  __syncthreads();
  float t = 0.f;
  for (int i = 0; i < nw; ++i) t += red[i];
  return t;
}

// p[0] + p[stride] + ... + p[(n - 1) stride], component-wise, added in slice order
// (deterministic); the loads of up to eight slices are issued before their adds.
__device__ __forceinline__ float4 sum_parts4(const float4 *__restrict__ p, int n, size_t stride) {
  float4 acc = p[0];
  for (int s0 = 1; s0 < n; s0 += 8) {
    float4 t[8];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (s0 + j < n) t[j] = p[(size_t)(s0 + j) * stride];
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (s0 + j < n) {
        acc.x += t[j].x;
        acc.y += t[j].y;
        acc.z += t[j].z;
        acc.w += t[j].w;
      }
  }
  return acc;
}

// Four consecutive values to `dst` in the activation type (one 16- or 8-byte store).
template <typename T>
__device__ __forceinline__ void store4(T *dst, float a, float b, float c, float d);
template <>
__device__ __forceinline__ void store4<float>(float *dst, float a, float b, float c, float d) {
  *reinterpret_cast<float4 *>(dst) = make_float4(a, b, c, d);
}
template <>
__device__ __forceinline__ void store4<bf16>(bf16 *dst, float a, float b, float c, float d) {
  const __nv_bfloat162 lo = __floats2bfloat162_rn(a, b), hi = __floats2bfloat162_rn(c, d);
  uint2 v;
  v.x = *reinterpret_cast<const uint32_t *>(&lo);
  v.y = *reinterpret_cast<const uint32_t *>(&hi);
  *reinterpret_cast<uint2 *>(dst) = v;
}
template <>
__device__ __forceinline__ void store4<__half>(__half *dst, float a, float b, float c, float d) {
  const __half2 lo = __floats2half2_rn(a, b), hi = __floats2half2_rn(c, d);
  uint2 v;
  v.x = *reinterpret_cast<const uint32_t *>(&lo);
  v.y = *reinterpret_cast<const uint32_t *>(&hi);
  *reinterpret_cast<uint2 *>(dst) = v;
}

// acc[j] = p[e_j] + p[stride + e_j] + ... + p[(n - 1) stride + e_j] for the 8 elements
// e_j = e0 + j * step (those < count; the others get 0), added in slice order (deterministic).  The
// slice loop is outermost so the 8 loads of a slice are in flight together.
__device__ __forceinline__ void sum_parts8(const float *__restrict__ p, int n, size_t stride,
                                           int e0, int step, int count, float (&acc)[8]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    const int e = e0 + j * step;
    acc[j] = e < count ? p[e] : 0.f;
  }
  for (int s = 1; s < n; ++s) {
    const float *q = p + (size_t)s * stride;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int e = e0 + j * step;
      if (e < count) acc[j] += q[e];
    }
  }
}

// Programmatic dependent launch.  Every kernel of the library starts with pdl_wait() (nothing is
// read before the preceding kernel of the stream has completed and its writes are visible) and
// pdl_trigger() (the next kernel may be scheduled now, so its launch and block setup overlap this
// kernel's work instead of following it).
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

}  // namespace dg

// ---- host-side launch bookkeeping (defined in dg_api.cu) ----------------------------------
namespace dg {
// Counts a kernel launch on stream `s` (and, while profiling is on in this thread, records a
// timing event on `s` before the launch, labelled `name`).
void note_launch(cudaStream_t s, const char *name);
int check_launch(const char *what);      // DG_OK or DG_ERR_CUDA (records the message)
// Shape and dtype checks of a dg_config that every entry point runs before any launch.
bool cfg_ok(const dg_config *c);
// Whether launches of this thread carry programmatic stream serialisation (on by default; off
// while a step is captured into a graph body that may not take programmatic edges).
bool &pdl_allowed();


// Launches `k` with programmatic stream serialisation allowed (see pdl_wait); errors surface
// through check_launch() like a <<<>>> launch.
template <typename... P, typename... A>
inline void launch_pdl(void (*k)(P...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       A &&...args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = pdl_allowed() ? 1 : 0;
  (void)cudaLaunchKernelEx(&cfg, k, static_cast<P>(args)...);
}

// launch_pdl for a kernel run as clusters of `cluster_x` CTAs along x.
template <typename... P, typename... A>
inline void launch_pdl_cluster(void (*k)(P...), dim3 grid, dim3 block, size_t smem,
                               cudaStream_t s, int cluster_x, A &&...args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  at[1].id = cudaLaunchAttributeClusterDimension;
  at[1].val.clusterDim.x = cluster_x;
  at[1].val.clusterDim.y = 1;
  at[1].val.clusterDim.z = 1;
  const bool pdl = pdl_allowed();
  cfg.attrs = pdl ? at : at + 1;
  cfg.numAttrs = pdl ? 2 : 1;
  (void)cudaLaunchKernelEx(&cfg, k, static_cast<P>(args)...);
}
}  // namespace dg
