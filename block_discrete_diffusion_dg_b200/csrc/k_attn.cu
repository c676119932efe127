// Canvas attention on CUDA cores (fp32 math): "DiffusionGemma Technical Report", Figure 4 — the
// decoder attends bidirectionally across the canvas and to the cached context; the causal
// encoder of the append attends causally within the new tokens.  GQA: query head h reads kv
// head h / (Hq / Hkv).  Online (flash-style) softmax over key tiles of 64; keys are the cache
// rows [0, cache_len[b]) followed by the n new rows.
//
// This kernel is the fp32 path and the small-shape path; the bf16 long-key case uses the
// tensor-core kernel.
#include "dg_common.cuh"
#include "dg_kernels.h"

namespace dg {

namespace {
constexpr int QB = 16;   // queries per CTA
constexpr int NT = 128;  // threads

template <typename T, int HD>
__global__ void __launch_bounds__(NT) attn_simt_kernel(int n, int Hq, int Hkv,
                                                       const T *__restrict__ q,
                                                       const T *__restrict__ kc,
                                                       const T *__restrict__ vc,
                                                       const int32_t *__restrict__ cache_len,
                                                       int cap, const T *__restrict__ kn,
                                                       const T *__restrict__ vn, int causal,
                                                       const int32_t *__restrict__ done, T *out) {
  pdl_wait();
  pdl_trigger();
  constexpr int KB = (HD >= 128) ? 32 : 64;  // keys per tile (static smem stays < 48 KB)
  constexpr int G = NT / HD;                  // query groups
  constexpr int QPT = QB / G;                 // queries per thread
  __shared__ float Qs[QB][HD];
  __shared__ float Ks[KB][HD + 1];
  __shared__ float Vs[KB][HD];
  __shared__ float S[QB][KB + 1];
  __shared__ float row_m[QB], row_l[QB], row_scale[QB];

  const int b = blockIdx.z, h = blockIdx.y, i0 = blockIdx.x * QB;
  if (done && done[b]) return;
  const int g = h / (Hq / Hkv);
  const int len = cache_len[b];
  const int tid = threadIdx.x;
  const int dim = tid % HD, qg = tid / HD;
  const float scale = 1.0f / sqrtf((float)HD);

  for (int e = tid; e < QB * HD; e += NT) {
    const int qi = e / HD, dd = e % HD;
    const int i = i0 + qi;
    Qs[qi][dd] = (i < n) ? to_f(q[(((size_t)b * n + i) * Hq + h) * HD + dd]) : 0.f;
  }
  if (tid < QB) { row_m[tid] = -INFINITY; row_l[tid] = 0.f; }
  float acc[QPT];
#pragma unroll
  for (int u = 0; u < QPT; ++u) acc[u] = 0.f;

  const T *kcb = kc + ((size_t)b * Hkv + g) * cap * HD;
  const T *vcb = vc + ((size_t)b * Hkv + g) * cap * HD;
  const T *knb = kn + ((size_t)b * Hkv + g) * n * HD;
  const T *vnb = vn + ((size_t)b * Hkv + g) * n * HD;
  const int total = len + n;
  __syncthreads();

  for (int j0 = 0; j0 < total; j0 += KB) {
    for (int e = tid; e < KB * HD; e += NT) {
      const int jj = e / HD, dd = e % HD;
      const int j = j0 + jj;
      float kv = 0.f, vv = 0.f;
      if (j < len) {
        kv = to_f(kcb[(size_t)j * HD + dd]);
        vv = to_f(vcb[(size_t)j * HD + dd]);
      } else if (j < total) {
        kv = to_f(knb[(size_t)(j - len) * HD + dd]);
        vv = to_f(vnb[(size_t)(j - len) * HD + dd]);
      }
      Ks[jj][dd] = kv;
      Vs[jj][dd] = vv;
    }
    __syncthreads();
    // scores
    for (int e = tid; e < QB * KB; e += NT) {
      const int qi = e / KB, jj = e % KB;
      const int j = j0 + jj;
      float sc = -INFINITY;
      const bool visible = (j < len) || (j < total && (!causal || (j - len) <= i0 + qi));
      if (visible && i0 + qi < n) {
        float a = 0.f;
#pragma unroll 8
        for (int dd = 0; dd < HD; ++dd) a = fmaf(Qs[qi][dd], Ks[jj][dd], a);
        sc = a * scale;
      }
      S[qi][jj] = sc;
    }
    __syncthreads();
    // online softmax: one warp per query row (QB rows, 4 warps)
    for (int qi = tid >> 5; qi < QB; qi += NT / 32) {
      const int lane = tid & 31;
      float mx = -INFINITY;
      for (int jj = lane; jj < KB; jj += 32) mx = fmaxf(mx, S[qi][jj]);
      mx = warp_max(mx);
      const float m_old = row_m[qi];
      const float m_new = fmaxf(m_old, mx);
      float ps = 0.f;
      for (int jj = lane; jj < KB; jj += 32) {
        const float p = (m_new == -INFINITY) ? 0.f : expf(S[qi][jj] - m_new);
        S[qi][jj] = p;
        ps += p;
      }
      ps = warp_sum(ps);
      if (lane == 0) {
        const float sc = (m_new == -INFINITY) ? 1.f : expf(m_old - m_new);
        row_scale[qi] = sc;
        row_l[qi] = row_l[qi] * sc + ps;
        row_m[qi] = m_new;
      }
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < QPT; ++u) {
      const int qi = qg + u * G;
      float a = acc[u] * row_scale[qi];
#pragma unroll 8
      for (int jj = 0; jj < KB; ++jj) a = fmaf(S[qi][jj], Vs[jj][dim], a);
      acc[u] = a;
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < QPT; ++u) {
    const int qi = qg + u * G;
    const int i = i0 + qi;
    if (i < n) {
      const float l = row_l[qi];
      out[(((size_t)b * n + i) * Hq + h) * HD + dim] = from_f<T>(l > 0.f ? acc[u] / l : 0.f);
    }
  }
}

template <typename T>
int run(int hd, dim3 grid, cudaStream_t s, int n, int Hq, int Hkv, const void *q, const void *kc,
        const void *vc, const int32_t *len, int cap, const void *kn, const void *vn, int causal,
        const int32_t *done, void *out) {
  note_launch(s, "attn_simt");
#define DG_ATTN_CASE(HDV)                                                                    \
  case HDV:                                                                                  \
    launch_pdl(attn_simt_kernel<T, HDV>, grid, NT, 0, s, n, Hq, Hkv, (const T *)q, (const T *)kc, \
                                                 (const T *)vc, len, cap, (const T *)kn,     \
                                                 (const T *)vn, causal, done, (T *)out);     \
    break;
  switch (hd) {
    DG_ATTN_CASE(32)
    DG_ATTN_CASE(64)
    DG_ATTN_CASE(128)
    default: return DG_ERR_UNSUPPORTED;
  }
#undef DG_ATTN_CASE
  return check_launch("attn_simt");
}
}  // namespace

size_t attention_ws_bytes(int act, int batch, int n, int Hq, int Hkv, int hd, int cap) {
  return attention_tc_supported(act, Hq, Hkv, hd)
             ? attention_tc_ws_bytes(batch, n, Hq, Hkv, hd, cap)
             : 0;
}

int launch_attention(int act, int batch, int n, int Hq, int Hkv, int hd, const void *q,
                     const void *k_cache, const void *v_cache, const int32_t *cache_len, int cap,
                     const void *k_new, const void *v_new, int causal, const int32_t *done,
                     void *out, void *ws, int32_t *st, cudaStream_t s) {
  if (n <= 0 || batch <= 0) return DG_OK;
  if (attention_tc_supported(act, Hq, Hkv, hd))
    return launch_attention_tc(batch, n, Hq, Hkv, hd, q, k_cache, v_cache, cache_len, cap, k_new,
                               v_new, causal, done, out, ws, st, s);
  dim3 grid((n + QB - 1) / QB, Hq, batch);
  if (act == DG_F32)
    return run<float>(hd, grid, s, n, Hq, Hkv, q, k_cache, v_cache, cache_len, cap, k_new, v_new,
                      causal, done, out);
  return run<bf16>(hd, grid, s, n, Hq, Hkv, q, k_cache, v_cache, cache_len, cap, k_new, v_new,
                   causal, done, out);
}

}  // namespace dg
