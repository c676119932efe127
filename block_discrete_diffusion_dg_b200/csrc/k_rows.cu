// Row kernels: embedding gather + pre-norm, RMSNorm (optionally over a gathered row list), and
// the compaction of the positions that need logits this step.
//
// The residual stream (embedding rows, layer outputs) is fp32; RMSNorm reads it and writes the
// normalised rows in the activation type, the input of the next matrix product.
// RMSNorm(x) = x / sqrt(mean(x^2) + eps), unit gain, computed in fp32 with a fixed-order
// reduction and rounded once to the activation type (the pre-norm of every layer and the
// final norm before the LM head; the pages' model is the Gemma 4 transformer,
// "DiffusionGemma Technical Report", What they did).
#include "dg_common.cuh"
#include "dg_kernels.h"

namespace dg {

template <typename T>
__global__ void __launch_bounds__(256) embed_norm_kernel(const int32_t *__restrict__ tokens,
                                                         const uint8_t *__restrict__ masked,
                                                         const T *__restrict__ emb, int d,
                                                         int vocab, float eps, float *x_out,
                                                         T *a_out, int32_t *st) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[8];
  const int row = blockIdx.x;
  int id = (masked && masked[row]) ? vocab : tokens[row];
  if (id < 0 || id > vocab) {  // out-of-range id: report, embed as MASK
    if (threadIdx.x == 0) set_status(st, DG_ERR_INVALID_ARG);
    id = vocab;
  }
  const T *src = emb + (size_t)id * d;
  float ss = 0.f;
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    float v = to_f(src[j]);
    ss += v * v;
  }
  ss = block_sum(ss, red);
  const float inv = 1.0f / sqrtf(ss / (float)d + eps);
  float *xo = x_out + (size_t)row * d;
  T *ao = a_out + (size_t)row * d;
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    const float v = to_f(src[j]);
    xo[j] = v;
    ao[j] = from_f<T>(v * inv);
  }
}

template <typename T>
__global__ void __launch_bounds__(256) rmsnorm_kernel(const float *__restrict__ in,
                                                      const int32_t *__restrict__ row_idx,
                                                      const int32_t *__restrict__ n_rows_dev,
                                                      int d, float eps, T *out) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[8];
  const int r = blockIdx.x;
  if (n_rows_dev && r >= *n_rows_dev) return;
  const int src_row = row_idx ? row_idx[r] : r;
  const float *src = in + (size_t)src_row * d;
  float ss = 0.f;
  for (int j = threadIdx.x; j < d; j += blockDim.x) {
    const float v = src[j];
    ss += v * v;
  }
  ss = block_sum(ss, red);
  const float inv = 1.0f / sqrtf(ss / (float)d + eps);
  T *o = out + (size_t)r * d;
  for (int j = threadIdx.x; j < d; j += blockDim.x) o[j] = from_f<T>(src[j] * inv);
}

// h = res + sum of n_parts fp32 partials [n_parts][rows][d] (split-K output projection, added in
// slice order), written to h_out; out = RMSNorm(h) in the activation type.  One block per row,
// the row staged in shared memory.
template <typename T>
__global__ void __launch_bounds__(256) resid_norm_kernel(const float *__restrict__ part,
                                                         int n_parts, size_t part_stride,
                                                         const float *__restrict__ res, int d,
                                                         float eps, float *h_out, T *out) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ float hrow[];
  __shared__ float red[8];
  const int r = blockIdx.x;
  float ss = 0.f;
  for (int j0 = threadIdx.x; j0 < d; j0 += 8 * blockDim.x) {
    float acc[8];
    sum_parts8(part + (size_t)r * d, n_parts, part_stride, j0, blockDim.x, d, acc);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int j = j0 + q * blockDim.x;
      if (j < d) {
        const float v = res[(size_t)r * d + j] + acc[q];
        hrow[j] = v;
        h_out[(size_t)r * d + j] = v;
        ss += v * v;
      }
    }
  }
  ss = block_sum(ss, red);
  const float inv = 1.0f / sqrtf(ss / (float)d + eps);
  T *o = out + (size_t)r * d;
  for (int j = threadIdx.x; j < d; j += blockDim.x) o[j] = from_f<T>(hrow[j] * inv);
}

// resid_norm_kernel with one float4 per thread (blockDim = d / 4 <= 1024): the slices of a thread's
// four elements are loaded together, then summed in slice order as above.
template <typename T>
__global__ void __launch_bounds__(1024) resid_norm4_kernel(const float4 *__restrict__ part,
                                                          int n_parts, size_t stride4,
                                                          const float4 *__restrict__ res, int d4,
                                                          float eps, float4 *h_out, T *out) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[32];
  const int r = blockIdx.x, j = threadIdx.x;
  const size_t o = (size_t)r * d4 + j;
  const float4 a = sum_parts4(part + o, n_parts, stride4);
  const float4 x = res[o];
  const float4 h = make_float4(x.x + a.x, x.y + a.y, x.z + a.z, x.w + a.w);
  h_out[o] = h;
  float ss = h.x * h.x;
  ss += h.y * h.y;
  ss += h.z * h.z;
  ss += h.w * h.w;
  ss = block_sum(ss, red);
  const float inv = 1.0f / sqrtf(ss / (float)(4 * d4) + eps);
  store4<T>(out + o * 4, h.x * inv, h.y * inv, h.z * inv, h.w * inv);
}

// One block of 1024 threads scans all B*C positions in chunks (B*C <= 65536).
__global__ void __launch_bounds__(1024) compact_rows_kernel(int batch, int canvas,
                                                            const uint8_t *__restrict__ masked,
                                                            const int32_t *__restrict__ done,
                                                            int32_t *row_idx, int32_t *n_rows,
                                                            uint8_t *token_live) {
  pdl_wait();
  pdl_trigger();
  __shared__ int warp_tot[32];
  __shared__ int base;
  if (threadIdx.x == 0) base = 0;
  __syncthreads();
  const int total = batch * canvas;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (int c0 = 0; c0 < total; c0 += blockDim.x) {
    const int p = c0 + threadIdx.x;
    int live = 0;
    if (p < total) {
      const int b = p / canvas;
      const int alive = done ? (done[b] == 0) : 1;
      if (token_live) token_live[p] = (uint8_t)alive;
      live = alive && (masked == nullptr || masked[p] != 0);
    }
    const unsigned bal = __ballot_sync(0xffffffffu, live);
    if (lane == 0) warp_tot[w] = __popc(bal);
    __syncthreads();
    int before = 0;
    for (int i = 0; i < w; ++i) before += warp_tot[i];
    const int pos = base + before + __popc(bal & ((1u << lane) - 1u));
    if (live) row_idx[pos] = p;
    __syncthreads();
    if (threadIdx.x == 0) {
      int t = 0;
      for (int i = 0; i < 32; ++i) t += warp_tot[i];
      base += t;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) *n_rows = base;
}

// Step prologue in one launch: blocks [0, rows) embed + pre-norm one row each (as
// embed_norm_kernel); the next rope_blocks blocks fill the RoPE table (as rope_table_kernel);
// with compaction requested, the last block lists the rows that need logits (as
// compact_rows_kernel, 256 threads) and the slot of each row in that list (-1 if none).
template <typename T>
__global__ void __launch_bounds__(256) prologue_kernel(
    const int32_t *__restrict__ tokens, const uint8_t *__restrict__ masked, const T *__restrict__ emb,
    int rows, int d, int vocab, float eps, float *x_out, T *a_out, int32_t *st, int rope_blocks,
    int n, int hd, double theta, const int32_t *__restrict__ cache_len, float *cs, int batch,
    int canvas, const int32_t *__restrict__ done, int32_t *row_idx, int32_t *n_rows, int32_t *slot,
    uint8_t *token_live, const uint8_t *__restrict__ emb_q, const uint8_t *__restrict__ emb_s,
    float emb_g, int emb_rows_pad, int drafts) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[8];
  __shared__ int warp_tot[8];
  __shared__ int base;
  const int bid = blockIdx.x;
  if (bid < rows) {  // embedding + pre-norm
    const int row = bid;
    // a masked row is embedded as MASK, or by its revisable draft token (noise canvas)
    int id = (masked && masked[row] && !drafts) ? vocab : tokens[row];
    if (id < 0 || id > vocab) {
      if (threadIdx.x == 0) set_status(st, DG_ERR_INVALID_ARG);
      id = vocab;
    }
    if (emb_q) {
      // NVFP4 rows (d % 256 == 0, d <= 8192): thread t decodes groups of 8 columns j8 = t + 256 u;
      // group j8 lies in k-block j8 / 8 at byte (j8 % 8) * 4 and shares scale (j8 % 8) / 2.
      // e2m1 * e4m3 is exact in fp16; the tensor scale is one fp32 rounding.
      float f[4][8];
      float ss = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j8 = threadIdx.x + u * blockDim.x;
        if (j8 >= d / 8) continue;
        const size_t slab = (size_t)(j8 >> 3) * emb_rows_pad + id;
        const uint32_t w = *reinterpret_cast<const uint32_t *>(emb_q + slab * 32 + (j8 & 7) * 4);
        const __half2 sc = e4m3_scale_f16x2(emb_s[slab * 4 + ((j8 & 7) >> 1)]);
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const float2 v = __half22float2(nvfp4_pair_f16(w >> (8 * b), sc));
          f[u][2 * b] = v.x * emb_g;
          f[u][2 * b + 1] = v.y * emb_g;
          ss += f[u][2 * b] * f[u][2 * b] + f[u][2 * b + 1] * f[u][2 * b + 1];
        }
      }
      ss = block_sum(ss, red);
      const float inv = 1.0f / sqrtf(ss / (float)d + eps);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j8 = threadIdx.x + u * blockDim.x;
        if (j8 >= d / 8) continue;
        float4 *xo = reinterpret_cast<float4 *>(x_out + (size_t)row * d + 8 * j8);
        xo[0] = make_float4(f[u][0], f[u][1], f[u][2], f[u][3]);
        xo[1] = make_float4(f[u][4], f[u][5], f[u][6], f[u][7]);
        store4<T>(a_out + (size_t)row * d + 8 * j8, f[u][0] * inv, f[u][1] * inv, f[u][2] * inv,
                  f[u][3] * inv);
        store4<T>(a_out + (size_t)row * d + 8 * j8 + 4, f[u][4] * inv, f[u][5] * inv,
                  f[u][6] * inv, f[u][7] * inv);
      }
      return;
    }
    const T *src = emb + (size_t)id * d;
    if (sizeof(T) == 2 && d % 8 == 0 && d / 8 <= 4 * (int)blockDim.x) {
      // bf16 rows: eight values per 16-byte load, one pass (the row stays in registers)
      uint4 raw[4];
      float ss = 0.f;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j8 = threadIdx.x + u * blockDim.x;
        if (j8 < d / 8) raw[u] = reinterpret_cast<const uint4 *>(src)[j8];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (threadIdx.x + u * (int)blockDim.x >= d / 8) continue;
        const bf16 *h = reinterpret_cast<const bf16 *>(&raw[u]);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float v = __bfloat162float(h[e]);
          ss += v * v;
        }
      }
      ss = block_sum(ss, red);
      const float inv = 1.0f / sqrtf(ss / (float)d + eps);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j8 = threadIdx.x + u * blockDim.x;
        if (j8 >= d / 8) continue;
        const bf16 *h = reinterpret_cast<const bf16 *>(&raw[u]);
        float f[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) f[e] = __bfloat162float(h[e]);
        float4 *xo = reinterpret_cast<float4 *>(x_out + (size_t)row * d + 8 * j8);
        xo[0] = make_float4(f[0], f[1], f[2], f[3]);
        xo[1] = make_float4(f[4], f[5], f[6], f[7]);
        store4<T>(a_out + (size_t)row * d + 8 * j8, f[0] * inv, f[1] * inv, f[2] * inv, f[3] * inv);
        store4<T>(a_out + (size_t)row * d + 8 * j8 + 4, f[4] * inv, f[5] * inv, f[6] * inv,
                  f[7] * inv);
      }
      return;
    }
    float ss = 0.f;
    for (int j = threadIdx.x; j < d; j += blockDim.x) {
      const float v = to_f(src[j]);
      ss += v * v;
    }
    ss = block_sum(ss, red);
    const float inv = 1.0f / sqrtf(ss / (float)d + eps);
    for (int j = threadIdx.x; j < d; j += blockDim.x) {
      const float v = to_f(src[j]);
      x_out[(size_t)row * d + j] = v;
      a_out[(size_t)row * d + j] = from_f<T>(v * inv);
    }
    return;
  }
  if (bid < rows + rope_blocks) {  // RoPE table: cos/sin of (cache_len[b] + i) * theta^(-2j/hd)
    const int half = hd / 2;
    const int e = (bid - rows) * blockDim.x + threadIdx.x;
    if (e >= batch * n * half) return;
    const int b = e / (n * half), r = e % (n * half);
    const int i = r / half, j = r % half;
    const double inv = pow(theta, -2.0 * (double)j / (double)hd);
    const double ang = ((cache_len ? (double)cache_len[b] : 0.0) + (double)i) * inv;
    double sn, c;
    sincos(ang, &sn, &c);
    float *o = cs + ((size_t)(b * n + i) * hd + 2 * j);
    o[0] = (float)c;
    o[1] = (float)sn;
    return;
  }
  // compaction of the rows that need logits
  if (threadIdx.x == 0) base = 0;
  __syncthreads();
  const int total = batch * canvas;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int c0 = 0; c0 < total; c0 += blockDim.x) {
    const int p = c0 + threadIdx.x;
    int live = 0;
    if (p < total) {
      const int alive = done ? (done[p / canvas] == 0) : 1;
      if (token_live) token_live[p] = (uint8_t)alive;
      live = alive && (masked == nullptr || masked[p] != 0);
    }
    const unsigned bal = __ballot_sync(0xffffffffu, live);
    if (lane == 0) warp_tot[w] = __popc(bal);
    __syncthreads();
    int before = 0;
    for (int i = 0; i < w; ++i) before += warp_tot[i];
    const int pos = base + before + __popc(bal & ((1u << lane) - 1u));
    if (live) row_idx[pos] = p;
    if (p < total && slot) slot[p] = live ? pos : -1;
    __syncthreads();
    if (threadIdx.x == 0) {
      int t = 0;
      for (int i = 0; i < nw; ++i) t += warp_tot[i];
      base += t;
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) *n_rows = base;
}

// e4m3 -> bf16, exact (every e4m3 value is a bf16 value); 16 codes per thread step.  The
// per-output-channel scales stay separate and are applied to the fp32 accumulators.
__global__ void dequant_e4m3_kernel(const uint4 *__restrict__ src, size_t n16, uint4 *dst) {
  pdl_wait();
  pdl_trigger();
  for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n16;
       i += (size_t)gridDim.x * blockDim.x) {
    const uint4 v = src[i];
    const uint8_t *c = reinterpret_cast<const uint8_t *>(&v);
    uint4 o[2];
    bf16 *ob = reinterpret_cast<bf16 *>(o);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      fp8 f;
      f.__x = c[j];
      ob[j] = __float2bfloat16_rn(float(f));
    }
    dst[2 * i] = o[0];
    dst[2 * i + 1] = o[1];
  }
}

int launch_dequant_e4m3(const void *src, size_t n, void *dst, cudaStream_t s) {
  if (n == 0) return DG_OK;
  if (n % 16) return DG_ERR_UNSUPPORTED;
  const size_t n16 = n / 16;
  size_t blocks = (n16 + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  note_launch(s, "dequant_e4m3");
  launch_pdl(dequant_e4m3_kernel, (unsigned)blocks, 256, 0, s, (const uint4 *)src, n16, (uint4 *)dst);
  return check_launch("dequant_e4m3");
}

int launch_prologue(int act, const int32_t *tokens, const uint8_t *masked, const void *emb, int rows,
                    int d, int vocab, double eps, void *x_out, void *a_out, int32_t *st, int batch,
                    int n, int hd, double theta, const int32_t *cache_len, float *cs,
                    const int32_t *done, int32_t *row_idx, int32_t *n_rows, int32_t *slot,
                    uint8_t *token_live, cudaStream_t s, const uint8_t *emb_scale, float emb_g,
                    int drafts) {
  if (rows <= 0) return DG_OK;
  const uint8_t *emb_q = emb_scale ? static_cast<const uint8_t *>(emb) : nullptr;
  const int rows_pad = nvfp4_rows_pad(vocab + 1);
  if (emb_q && (act != DG_BF16 || d % 256 != 0 || d > 8192)) return DG_ERR_UNSUPPORTED;
  const int rope_blocks = (batch * n * (hd / 2) + 255) / 256;
  const int grid = rows + rope_blocks + (row_idx ? 1 : 0);
  note_launch(s, "prologue");
  if (act == DG_F32)
    launch_pdl(prologue_kernel<float>, grid, 256, 0, s, tokens, masked, (const float *)emb, rows, d, vocab, (float)eps, (float *)x_out,
        (float *)a_out, st, rope_blocks, n, hd, theta, cache_len, cs, batch, n, done, row_idx,
        n_rows, slot, token_live, emb_q, emb_scale, emb_g, rows_pad, drafts);
  else
    launch_pdl(prologue_kernel<bf16>, grid, 256, 0, s, tokens, masked, (const bf16 *)emb, rows, d, vocab, (float)eps, (float *)x_out,
        (bf16 *)a_out, st, rope_blocks, n, hd, theta, cache_len, cs, batch, n, done, row_idx,
        n_rows, slot, token_live, emb_q, emb_scale, emb_g, rows_pad, drafts);
  return check_launch("prologue");
}

int launch_embed_norm(int act, const int32_t *tokens, const uint8_t *masked, const void *emb,
                      int rows, int d, int vocab, double eps, void *x_out, void *a_out,
                      int32_t *st, cudaStream_t s) {
  if (rows <= 0) return DG_OK;
  note_launch(s, "embed_norm");
  if (act == DG_F32)
    launch_pdl(embed_norm_kernel<float>, rows, 256, 0, s, tokens, masked, (const float *)emb, d, vocab,
                                                  (float)eps, (float *)x_out, (float *)a_out, st);
  else
    launch_pdl(embed_norm_kernel<bf16>, rows, 256, 0, s, tokens, masked, (const bf16 *)emb, d, vocab,
                                                 (float)eps, (float *)x_out, (bf16 *)a_out, st);
  return check_launch("embed_norm");
}

int launch_rmsnorm(int act, const void *in, const int32_t *row_idx, const int32_t *n_rows_dev,
                   int max_rows, int d, double eps, void *out, cudaStream_t s, int f16_out) {
  if (max_rows <= 0) return DG_OK;
  note_launch(s, "rmsnorm");
  if (f16_out)
    launch_pdl(rmsnorm_kernel<__half>, max_rows, 256, 0, s, (const float *)in, row_idx, n_rows_dev,
               d, (float)eps, (__half *)out);
  else if (act == DG_F32)
    launch_pdl(rmsnorm_kernel<float>, max_rows, 256, 0, s, (const float *)in, row_idx, n_rows_dev, d,
                                                   (float)eps, (float *)out);
  else
    launch_pdl(rmsnorm_kernel<bf16>, max_rows, 256, 0, s, (const float *)in, row_idx, n_rows_dev, d,
                                                  (float)eps, (bf16 *)out);
  return check_launch("rmsnorm");
}

int launch_resid_norm(int act, const float *part, int n_parts, const float *res, int rows, int d,
                      double eps, float *h_out, void *out, cudaStream_t s) {
  if (rows <= 0) return DG_OK;
  const size_t smem = (size_t)d * sizeof(float);
  if (smem > 48 * 1024) return DG_ERR_UNSUPPORTED;
  note_launch(s, "resid_norm");
  const size_t stride = (size_t)rows * d;
  if (d % 4 == 0 && d / 4 <= 1024 && d / 4 >= 32) {
    if (act == DG_F32)
      launch_pdl(resid_norm4_kernel<float>, rows, d / 4, 0, s, (const float4 *)part, n_parts,
                 stride / 4, (const float4 *)res, d / 4, (float)eps, (float4 *)h_out,
                 (float *)out);
    else
      launch_pdl(resid_norm4_kernel<bf16>, rows, d / 4, 0, s, (const float4 *)part, n_parts,
                 stride / 4, (const float4 *)res, d / 4, (float)eps, (float4 *)h_out, (bf16 *)out);
    return check_launch("resid_norm");
  }
  if (act == DG_F32)
    launch_pdl(resid_norm_kernel<float>, rows, 256, smem, s, part, n_parts, stride, res, d, (float)eps,
                                                     h_out, (float *)out);
  else
    launch_pdl(resid_norm_kernel<bf16>, rows, 256, smem, s, part, n_parts, stride, res, d, (float)eps,
                                                    h_out, (bf16 *)out);
  return check_launch("resid_norm");
}

int launch_compact_rows(int batch, int canvas, const uint8_t *masked, const int32_t *done,
                        int32_t *row_idx, int32_t *n_rows, uint8_t *token_live, cudaStream_t s) {
  note_launch(s, "compact_rows");
  launch_pdl(compact_rows_kernel, 1, 1024, 0, s, batch, canvas, masked, done, row_idx, n_rows, token_live);
  return check_launch("compact_rows");
}

}  // namespace dg
