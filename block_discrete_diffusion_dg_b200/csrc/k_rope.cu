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

// RoPE and head split after the QKV projection.  qkv holds n_parts fp32 partial sums
// [n_parts][B n][width] (split-K projection), added here in slice order.  One thread per 8
// outputs, several rows per block, no shared memory.  For a q or k head, item h covers columns 4h .. 4h + 3 of the head's first half and their rotate-half
// partners 4h + hd/2 .. 4h + hd/2 + 3; for a v head, columns 8h .. 8h + 7.  Each thread sums its
// two float4 of the split-K partials (slice order), rotates, and stores.
template <typename T>
__global__ void __launch_bounds__(256) qkv_rope_kernel(
    int rows, int n, int Hq, int Hkv, int hd, const float4 *__restrict__ qkv, int n_parts,
    size_t part_stride4, const float *__restrict__ cs, T *q, T *k_new, T *v_new, T *k_cache,
    T *v_cache, const int32_t *__restrict__ cache_len, int cap, int32_t *st) {
  pdl_wait();
  pdl_trigger();
  const int per_head = hd / 8, items = (Hq + 2 * Hkv) * per_head;
  const long long gid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gid >= (long long)rows * items) return;
  const int row = (int)(gid / items), it = (int)(gid % items);
  const int b = row / n, i = row % n;
  const int half = hd / 2, head = it / per_head, h8 = it % per_head;
  const bool rotate = head < Hq + Hkv;
  const int c0 = rotate ? 4 * h8 : 8 * h8, c1 = rotate ? half + 4 * h8 : 8 * h8 + 4;
  const float4 *src = qkv + (size_t)row * ((Hq + 2 * Hkv) * hd / 4) + head * (hd / 4);
  const float4 a = sum_parts4(src + c0 / 4, n_parts, part_stride4);
  const float4 p = sum_parts4(src + c1 / 4, n_parts, part_stride4);
  float o0[4] = {a.x, a.y, a.z, a.w}, o1[4] = {p.x, p.y, p.z, p.w};
  if (rotate) {
    const float *c = cs + (size_t)row * hd;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = c0 + u;
      const float co = c[2 * j], si = c[2 * j + 1];
      const float x1 = o0[u], x2 = o1[u];
      o0[u] = x1 * co - x2 * si;
      o1[u] = x2 * co + x1 * si;
    }
  }
  int crow = -1;
  if (k_cache && head >= Hq) {
    if (cache_len[b] + n > cap) {
      if (i == 0 && it == Hq * per_head) set_status(st, DG_ERR_CAPACITY);
    } else {
      crow = cache_len[b] + i;
    }
  }
  if (head < Hq) {
    T *dst = q + (size_t)row * Hq * hd + head * hd;
    store4<T>(dst + c0, o0[0], o0[1], o0[2], o0[3]);
    store4<T>(dst + c1, o1[0], o1[1], o1[2], o1[3]);
  } else {
    const bool is_k = head < Hq + Hkv;
    const int g = is_k ? head - Hq : head - Hq - Hkv;
    T *dst = (is_k ? k_new : v_new) + (((size_t)b * Hkv + g) * n + i) * hd;
    store4<T>(dst + c0, o0[0], o0[1], o0[2], o0[3]);
    store4<T>(dst + c1, o1[0], o1[1], o1[2], o1[3]);
    if (crow >= 0) {
      T *cd = (is_k ? k_cache : v_cache) + (((size_t)b * Hkv + g) * cap + crow) * hd;
      store4<T>(cd + c0, o0[0], o0[1], o0[2], o0[3]);
      store4<T>(cd + c1, o1[0], o1[1], o1[2], o1[3]);
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
  const int width = (Hq + 2 * Hkv) * hd;
  const size_t stride = (size_t)batch * n * width;
  if (hd % 8 == 0) {
    note_launch(s, "qkv_split");
    const long long work = (long long)batch * n * (width / 8);
    const int grid = (int)((work + 255) / 256);
    if (act == DG_F32)
      launch_pdl(qkv_rope_kernel<float>, grid, 256, 0, s, batch * n, n, Hq, Hkv, hd,
                 (const float4 *)qkv, n_parts, stride / 4, cs, (float *)q, (float *)k_new,
                 (float *)v_new, (float *)k_cache, (float *)v_cache, cache_len, cap, st);
    else
      launch_pdl(qkv_rope_kernel<bf16>, grid, 256, 0, s, batch * n, n, Hq, Hkv, hd,
                 (const float4 *)qkv, n_parts, stride / 4, cs, (bf16 *)q, (bf16 *)k_new,
                 (bf16 *)v_new, (bf16 *)k_cache, (bf16 *)v_cache, cache_len, cap, st);
    return check_launch("qkv_split");
  }
  return DG_ERR_UNSUPPORTED;  // head_dim is 32, 64 or 128 (cfg_ok)
}

int launch_add_cache_len(int batch, int n, int cap, int32_t *cache_len, cudaStream_t s) {
  note_launch(s, "add_cache_len");
  launch_pdl(add_cache_len_kernel, (batch + 127) / 128, 128, 0, s, batch, n, cap, cache_len);
  return check_launch("add_cache_len");
}

}  // namespace dg
