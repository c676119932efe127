// Rotary position embedding and head split after the QKV projection.
//
// The pages give no position scheme; the library uses rotate-half RoPE with base theta at
// absolute positions cache_len[b] + i (the canvas continues the cached context, "DiffusionGemma
// Technical Report", Figure 4).  Pairs (j, j + hd/2) rotate by angle pos * theta^(-2j/hd).
// The angle and its cosine/sine are computed in fp64 (positions reach 131k, where an fp32 angle
// would be off by ~1e-2 rad) and stored as fp32.
#include "dg_common.cuh"
#include "dg_kernels.h"

namespace dg {

// cs[(b*n + i)*hd + 2j] = cos, [.. + 2j + 1] = sin
__global__ void rope_table_kernel(int n, int hd, double theta, const int32_t *__restrict__ cache_len,
                                  float *cs) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.y;
  const int half = hd / 2;
  const int total = n * half;
  const double base = cache_len ? (double)cache_len[b] : 0.0;
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < total; t += gridDim.x * blockDim.x) {
    const int i = t / half, j = t % half;
    const double inv = pow(theta, -2.0 * (double)j / (double)hd);
    const double ang = (base + (double)i) * inv;
    double sn, c;
    sincos(ang, &sn, &c);
    float *o = cs + ((size_t)(b * n + i) * hd + 2 * j);
    o[0] = (float)c;
    o[1] = (float)sn;
  }
}

// qkv holds n_parts fp32 partial sums [n_parts][B n][width] (split-K projection), added here in
// slice order; the summed row is staged in shared memory.
template <typename T>
__global__ void qkv_split_kernel(int n, int Hq, int Hkv, int hd, const float *__restrict__ qkv,
                                 int n_parts, size_t part_stride, const float *__restrict__ cs,
                                 T *q, T *k_new, T *v_new, T *k_cache, T *v_cache,
                                 const int32_t *__restrict__ cache_len, int cap, int32_t *st) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ float qkv_row[];
  const int row = blockIdx.x;  // b*n + i
  const int b = row / n, i = row % n;
  const int half = hd / 2;
  const int width = (Hq + 2 * Hkv) * hd;
  for (int e0 = threadIdx.x; e0 < width; e0 += 8 * blockDim.x) {
    float acc[8];
    sum_parts8(qkv + (size_t)row * width, n_parts, part_stride, e0, blockDim.x, width, acc);
#pragma unroll
    for (int j = 0; j < 8; ++j)
      if (e0 + j * (int)blockDim.x < width) qkv_row[e0 + j * blockDim.x] = acc[j];
  }
  __syncthreads();
  const float *src = qkv_row;
  const float *c = cs + (size_t)row * hd;
  int crow = -1;
  if (k_cache) {
    const int r = cache_len[b] + i;
    if (cache_len[b] + n > cap) {
      if (threadIdx.x == 0) set_status(st, DG_ERR_CAPACITY);
    } else {
      crow = r;
    }
  }
  for (int e = threadIdx.x; e < width; e += blockDim.x) {
    const int head = e / hd, dd = e % hd;
    float v = src[e];
    if (head < Hq + Hkv) {  // rotate q and k
      const int j = dd % half;
      const float co = c[2 * j], si = c[2 * j + 1];
      const float x1 = src[head * hd + j], x2 = src[head * hd + j + half];
      v = (dd < half) ? (x1 * co - x2 * si) : (x2 * co + x1 * si);
    }
    const T tv = from_f<T>(v);
    if (head < Hq) {
      q[(size_t)row * Hq * hd + e] = tv;
    } else {
      const bool is_k = head < Hq + Hkv;
      const int g = is_k ? head - Hq : head - Hq - Hkv;
      T *dst = is_k ? k_new : v_new;
      dst[(((size_t)b * Hkv + g) * n + i) * hd + dd] = tv;
      if (crow >= 0) {
        T *cd = is_k ? k_cache : v_cache;
        cd[(((size_t)b * Hkv + g) * cap + crow) * hd + dd] = tv;
      }
    }
  }
}

// qkv_split_kernel with one float4 per thread (blockDim = width / 4 <= 1024): the summed row is
// staged in shared memory, then each thread rotates and stores its four consecutive values.
template <typename T>
__global__ void __launch_bounds__(1024) qkv_split4_kernel(
    int n, int Hq, int Hkv, int hd, const float4 *__restrict__ qkv, int n_parts,
    size_t part_stride4, const float *__restrict__ cs, T *q, T *k_new, T *v_new, T *k_cache,
    T *v_cache, const int32_t *__restrict__ cache_len, int cap, int32_t *st) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ float4 qkv_row4[];
  const int row = blockIdx.x;  // b*n + i
  const int b = row / n, i = row % n;
  const int half = hd / 2;
  const int width4 = (Hq + 2 * Hkv) * hd / 4;
  const int t = threadIdx.x;
  qkv_row4[t] = sum_parts4(qkv + (size_t)row * width4 + t, n_parts, part_stride4);
  int crow = -1;
  if (k_cache) {
    if (cache_len[b] + n > cap) {
      if (t == 0) set_status(st, DG_ERR_CAPACITY);
    } else {
      crow = cache_len[b] + i;
    }
  }
  __syncthreads();
  const float *src = reinterpret_cast<const float *>(qkv_row4);
  const float *c = cs + (size_t)row * hd;
  const int e0 = 4 * t, head = e0 / hd, dd0 = e0 % hd;
  float v[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int dd = dd0 + u;
    v[u] = src[e0 + u];
    if (head < Hq + Hkv) {  // rotate q and k
      const int j = dd % half;
      const float co = c[2 * j], si = c[2 * j + 1];
      const float x1 = src[head * hd + j], x2 = src[head * hd + j + half];
      v[u] = (dd < half) ? (x1 * co - x2 * si) : (x2 * co + x1 * si);
    }
  }
  if (head < Hq) {
    store4<T>(q + (size_t)row * Hq * hd + e0, v[0], v[1], v[2], v[3]);
  } else {
    const bool is_k = head < Hq + Hkv;
    const int g = is_k ? head - Hq : head - Hq - Hkv;
    T *dst = is_k ? k_new : v_new;
    store4<T>(dst + (((size_t)b * Hkv + g) * n + i) * hd + dd0, v[0], v[1], v[2], v[3]);
    if (crow >= 0) {
      T *cd = is_k ? k_cache : v_cache;
      store4<T>(cd + (((size_t)b * Hkv + g) * cap + crow) * hd + dd0, v[0], v[1], v[2], v[3]);
    }
  }
}

__global__ void add_cache_len_kernel(int batch, int n, int cap, int32_t *cache_len) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < batch && cache_len[b] + n <= cap) cache_len[b] += n;
}

int launch_rope_table(int batch, int n, int hd, double theta, const int32_t *cache_len, float *cs,
                      cudaStream_t s) {
  note_launch(s, "rope_table");
  const int total = n * (hd / 2);
  dim3 grid((total + 255) / 256, batch);
  launch_pdl(rope_table_kernel, grid, 256, 0, s, n, hd, theta, cache_len, cs);
  return check_launch("rope_table");
}

int launch_qkv_split(int act, int batch, int n, int Hq, int Hkv, int hd, const float *qkv,
                     int n_parts, const float *cs, void *q, void *k_new, void *v_new,
                     void *k_cache, void *v_cache, const int32_t *cache_len, int cap, int32_t *st,
                     cudaStream_t s) {
  note_launch(s, "qkv_split");
  const int width = (Hq + 2 * Hkv) * hd;
  const size_t smem = (size_t)width * sizeof(float);
  const size_t stride = (size_t)batch * n * width;
  if (smem > 48 * 1024) return DG_ERR_UNSUPPORTED;
  if (width % 4 == 0 && width / 4 <= 1024 && width / 4 >= 32 && hd % 4 == 0) {
    if (act == DG_F32)
      launch_pdl(qkv_split4_kernel<float>, batch * n, width / 4, smem, s, n, Hq, Hkv, hd,
                 (const float4 *)qkv, n_parts, stride / 4, cs, (float *)q, (float *)k_new,
                 (float *)v_new, (float *)k_cache, (float *)v_cache, cache_len, cap, st);
    else
      launch_pdl(qkv_split4_kernel<bf16>, batch * n, width / 4, smem, s, n, Hq, Hkv, hd,
                 (const float4 *)qkv, n_parts, stride / 4, cs, (bf16 *)q, (bf16 *)k_new,
                 (bf16 *)v_new, (bf16 *)k_cache, (bf16 *)v_cache, cache_len, cap, st);
    return check_launch("qkv_split");
  }
  if (act == DG_F32)
    launch_pdl(qkv_split_kernel<float>, batch * n, 256, smem, s, n, Hq, Hkv, hd, qkv, n_parts, stride, cs,
                                                         (float *)q, (float *)k_new,
                                                         (float *)v_new, (float *)k_cache,
                                                         (float *)v_cache, cache_len, cap, st);
  else
    launch_pdl(qkv_split_kernel<bf16>, batch * n, 256, smem, s, n, Hq, Hkv, hd, qkv, n_parts, stride, cs,
                                                        (bf16 *)q, (bf16 *)k_new, (bf16 *)v_new,
                                                        (bf16 *)k_cache, (bf16 *)v_cache,
                                                        cache_len, cap, st);
  return check_launch("qkv_split");
}

int launch_add_cache_len(int batch, int n, int cap, int32_t *cache_len, cudaStream_t s) {
  note_launch(s, "add_cache_len");
  launch_pdl(add_cache_len_kernel, (batch + 127) / 128, 128, 0, s, batch, n, cap, cache_len);
  return check_launch("add_cache_len");
}

}  // namespace dg
