// Canvas attention on tensor cores (bf16 mma.sync m16n8k16, fp32 accumulation) with split-KV.
// "DiffusionGemma Technical Report", Figure 4: the decoder attends bidirectionally across the
// canvas and to the cached context (cross-attention to the KV cache); the causal encoder of the
// append attends causally within the new tokens.  Model card "diffusiongemma", Model Overview.
//
// One CTA = 128 query rows that share one kv head: the rep = Hq / Hkv query heads of that kv head
// times 128 / rep consecutive canvas positions, so every K/V tile is read once per GQA group.
// Keys are split into chunks (split-KV) so that short and 131k-key contexts both fill the GPU;
// each split leaves an unnormalised partial (O, running max m, sum l) that lm-style merging
// combines exactly:  m = max m_s, l = sum l_s 2^(m_s - m), O = sum O_s 2^(m_s - m) / l.
// Scores are kept in the log2 domain: t = q.k / sqrt(hd) * log2(e).
// 8 warps x 16 rows; K/V tiles of 64 keys double-buffered with cp.async (zero-filled past the end)
// in XOR-swizzled shared memory read by ldmatrix.
// Precision: S = Q K^T takes the stored bf16 q and k exactly.  The second product takes P and V
// in fp16: P in [0, 1] keeps 11 significant bits instead of bf16's 8 (the rounding of P is the
// one rounding of this kernel the stored tensors do not have), and every bf16 value of V is
// exact in fp16 for |v| < 65504 (below fp16's normal range the absolute error stays < 3e-8).
// Each thread converts the V chunks it loaded, in place, once they have landed.
#include "dg_common.cuh"
#include "dg_kernels.h"
#include "tc_host.h"

namespace dg {

namespace {

constexpr int ROWS = 128;    // query rows per CTA
constexpr int KT = 64;       // keys per tile
constexpr int NTHR = 256;    // 8 warps x 16 rows
constexpr int MAX_SPLITS = 64;

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async16(void *dst, const void *src, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(dst)), "l"(src),
               "r"(n)
               : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void *p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_addr(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void *p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_addr(p)));
}
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void mma16816_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                             uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  const __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t *>(&v);
}
// 8 bf16 values -> 8 fp16 values, in place (16 bytes).
__device__ __forceinline__ void bf16x8_to_f16x8(uint4 *p) {
  uint4 v = *p;
  uint32_t *w = reinterpret_cast<uint32_t *>(&v);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const __nv_bfloat162 b = *reinterpret_cast<const __nv_bfloat162 *>(&w[i]);
    const __half2 h = __floats2half2_rn(__low2float(b), __high2float(b));
    w[i] = *reinterpret_cast<const uint32_t *>(&h);
  }
  *p = v;
}

// Row r of a [rows][HD] bf16 tile: 16-byte chunk c lives at chunk c ^ (r & 7).
template <int HD>
__device__ __forceinline__ int swz(int r, int col) {
  const int c = col >> 3;
  return r * HD + (((c ^ (r & 7)) << 3) | (col & 7));
}

struct AttnArgs {
  const bf16 *q, *kc, *vc, *kn, *vn;
  const int32_t *cache_len, *done;
  int n, Hq, Hkv, cap, causal, splits, chunk;
  bf16 *out;         // used when splits == 1
  float *part_o;     // [splits][B][Hq][n][HD]
  float2 *part_ml;   // [splits][B][Hq][n]
};

template <int HD>
constexpr size_t attn_smem_bytes() {
  return (size_t)(ROWS + 4 * KT) * HD * sizeof(bf16);
}

template <int HD>
__global__ void __launch_bounds__(NTHR) attn_tc_kernel(AttnArgs a) {
  extern __shared__ __align__(128) uint8_t attn_smem[];
  bf16 *sQ = reinterpret_cast<bf16 *>(attn_smem);
  bf16 *sKb = sQ + ROWS * HD;           // [2][KT * HD]
  bf16 *sVb = sKb + 2 * KT * HD;        // [2][KT * HD]

  const int split = blockIdx.z % a.splits, b = blockIdx.z / a.splits;
  if (a.done && a.done[b]) return;
  const int g = blockIdx.y;
  const int rep = a.Hq / a.Hkv;
  const int qpc = ROWS / rep;            // canvas positions per CTA
  const int i0 = blockIdx.x * qpc;
  const int len = a.cache_len[b];
  const int total = len + a.n;
  const int k_begin = split * a.chunk;
  const int k_end = min(total, k_begin + a.chunk);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const float sl2 = 1.4426950408889634f / sqrtf((float)HD);

  // Q tile: row r = (head h = g*rep + r / qpc, position i0 + r % qpc)
  for (int e = tid; e < ROWS * (HD / 8); e += NTHR) {
    const int r = e / (HD / 8), c = e % (HD / 8);
    const int h = g * rep + r / qpc, i = i0 + r % qpc;
    const bool ok = i < a.n;
    const bf16 *src = a.q + (((size_t)b * a.n + (ok ? i : 0)) * a.Hq + h) * HD + c * 8;
    cp_async16(&sQ[swz<HD>(r, c * 8)], src, ok);
  }
  const bf16 *kcb = a.kc + ((size_t)b * a.Hkv + g) * a.cap * HD;
  const bf16 *vcb = a.vc + ((size_t)b * a.Hkv + g) * a.cap * HD;
  const bf16 *knb = a.kn + ((size_t)b * a.Hkv + g) * a.n * HD;
  const bf16 *vnb = a.vn + ((size_t)b * a.Hkv + g) * a.n * HD;
  auto load_tile = [&](int buf, int j0) {
    for (int e = tid; e < KT * (HD / 8); e += NTHR) {
      const int r = e / (HD / 8), c = e % (HD / 8);
      const int j = j0 + r;
      const bool ok = j < k_end;
      const bf16 *ks, *vs;
      if (j < len) {
        ks = kcb + (size_t)j * HD;
        vs = vcb + (size_t)j * HD;
      } else {
        const int jj = ok ? j - len : 0;
        ks = knb + (size_t)jj * HD;
        vs = vnb + (size_t)jj * HD;
      }
      // a copy of 0 bytes (past the last key) zero-fills; its address is a valid dummy
      cp_async16(&sKb[buf * KT * HD + swz<HD>(r, c * 8)], ok ? ks + c * 8 : (const bf16 *)a.q, ok);
      cp_async16(&sVb[buf * KT * HD + swz<HD>(r, c * 8)], ok ? vs + c * 8 : (const bf16 *)a.q, ok);
    }
  };
  const int ntiles = k_end > k_begin ? (k_end - k_begin + KT - 1) / KT : 0;
  if (ntiles > 0) load_tile(0, k_begin);
  cp_commit();

  // this thread's two rows (within the warp's 16) and their canvas positions
  const int r_lo = warp * 16 + (lane >> 2), r_hi = r_lo + 8;
  const int pos_lo = i0 + r_lo % qpc, pos_hi = i0 + r_hi % qpc;
  float o[HD / 8][4];
#pragma unroll
  for (int j = 0; j < HD / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
  float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;
  uint32_t qf[HD / 16][4];

  for (int t = 0; t < ntiles; ++t) {
    if (t + 1 < ntiles) load_tile((t + 1) & 1, k_begin + (t + 1) * KT);
    cp_commit();
    cp_wait<1>();
    for (int e = tid; e < KT * (HD / 8); e += NTHR) {  // this thread's V chunks of tile t
      const int r = e / (HD / 8), c = e % (HD / 8);
      bf16x8_to_f16x8(reinterpret_cast<uint4 *>(&sVb[(t & 1) * KT * HD + swz<HD>(r, c * 8)]));
    }
    __syncthreads();
    if (t == 0) {
#pragma unroll
      for (int kk = 0; kk < HD / 16; ++kk) {
        const int mi = lane >> 3;
        const int row = warp * 16 + (mi & 1) * 8 + (lane & 7);
        ldsm_x4(qf[kk], &sQ[swz<HD>(row, kk * 16 + (mi >> 1) * 8)]);
      }
    }
    const bf16 *K = sKb + (t & 1) * KT * HD, *V = sVb + (t & 1) * KT * HD;
    const int j0 = k_begin + t * KT;
    float s[KT / 8][4];
#pragma unroll
    for (int j = 0; j < KT / 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk) {
#pragma unroll
      for (int nn = 0; nn < KT / 16; ++nn) {
        uint32_t bb[4];
        const int mi = lane >> 3;
        const int key = nn * 16 + (mi >> 1) * 8 + (lane & 7);
        ldsm_x4(bb, &K[swz<HD>(key, kk * 16 + (mi & 1) * 8)]);
        mma16816(s[2 * nn], qf[kk], bb[0], bb[1]);
        mma16816(s[2 * nn + 1], qf[kk], bb[2], bb[3]);
      }
    }
    // scale, mask, online softmax (rows lo: s[.][0..1], hi: s[.][2..3])
    float tmax_lo = -INFINITY, tmax_hi = -INFINITY;
#pragma unroll
    for (int j = 0; j < KT / 8; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = j0 + j * 8 + (lane & 3) * 2 + (e & 1);
        const int pos = (e < 2) ? pos_lo : pos_hi;
        bool vis = key < k_end;
        if (a.causal && key >= len) vis = vis && (key - len) <= pos;
        const float v = vis ? s[j][e] * sl2 : -INFINITY;
        s[j][e] = v;
        if (e < 2) tmax_lo = fmaxf(tmax_lo, v);
        else tmax_hi = fmaxf(tmax_hi, v);
      }
    }
#pragma unroll
    for (int o_ = 1; o_ <= 2; o_ <<= 1) {
      tmax_lo = fmaxf(tmax_lo, __shfl_xor_sync(0xffffffffu, tmax_lo, o_));
      tmax_hi = fmaxf(tmax_hi, __shfl_xor_sync(0xffffffffu, tmax_hi, o_));
    }
    const float mn_lo = fmaxf(m_lo, tmax_lo), mn_hi = fmaxf(m_hi, tmax_hi);
    const float b_lo = mn_lo == -INFINITY ? 0.f : mn_lo, b_hi = mn_hi == -INFINITY ? 0.f : mn_hi;
    const float sc_lo = exp2f(m_lo - b_lo), sc_hi = exp2f(m_hi - b_hi);
    m_lo = mn_lo;
    m_hi = mn_hi;
    float ps_lo = 0.f, ps_hi = 0.f;
#pragma unroll
    for (int j = 0; j < KT / 8; ++j) {
      s[j][0] = exp2f(s[j][0] - b_lo);
      s[j][1] = exp2f(s[j][1] - b_lo);
      s[j][2] = exp2f(s[j][2] - b_hi);
      s[j][3] = exp2f(s[j][3] - b_hi);
      ps_lo += s[j][0] + s[j][1];
      ps_hi += s[j][2] + s[j][3];
    }
    l_lo = l_lo * sc_lo + ps_lo;
    l_hi = l_hi * sc_hi + ps_hi;
#pragma unroll
    for (int j = 0; j < HD / 8; ++j) {
      o[j][0] *= sc_lo;
      o[j][1] *= sc_lo;
      o[j][2] *= sc_hi;
      o[j][3] *= sc_hi;
    }
    // O += P V
#pragma unroll
    for (int kk = 0; kk < KT / 16; ++kk) {
      uint32_t pa[4];
      pa[0] = pack_f16(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_f16(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_f16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_f16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int nn = 0; nn < HD / 16; ++nn) {
        uint32_t bb[4];
        const int mi = lane >> 3;
        const int key = kk * 16 + (mi & 1) * 8 + (lane & 7);
        ldsm_x4_t(bb, &V[swz<HD>(key, nn * 16 + (mi >> 1) * 8)]);
        mma16816_f16(o[2 * nn], pa, bb[0], bb[1]);
        mma16816_f16(o[2 * nn + 1], pa, bb[2], bb[3]);
      }
    }
    __syncthreads();
  }
  // full row sums over the quad
#pragma unroll
  for (int o_ = 1; o_ <= 2; o_ <<= 1) {
    l_lo += __shfl_xor_sync(0xffffffffu, l_lo, o_);
    l_hi += __shfl_xor_sync(0xffffffffu, l_hi, o_);
  }
  const int h_lo = g * rep + r_lo / qpc, h_hi = g * rep + r_hi / qpc;
  const bool ok_lo = pos_lo < a.n, ok_hi = pos_hi < a.n;
  if (a.splits == 1) {
    const float il = l_lo > 0.f ? 1.f / l_lo : 0.f, ih = l_hi > 0.f ? 1.f / l_hi : 0.f;
#pragma unroll
    for (int j = 0; j < HD / 8; ++j) {
      const int col = j * 8 + (lane & 3) * 2;
      if (ok_lo)
        *reinterpret_cast<__nv_bfloat162 *>(
            &a.out[(((size_t)b * a.n + pos_lo) * a.Hq + h_lo) * HD + col]) =
            __floats2bfloat162_rn(o[j][0] * il, o[j][1] * il);
      if (ok_hi)
        *reinterpret_cast<__nv_bfloat162 *>(
            &a.out[(((size_t)b * a.n + pos_hi) * a.Hq + h_hi) * HD + col]) =
            __floats2bfloat162_rn(o[j][2] * ih, o[j][3] * ih);
    }
  } else {
    const int B = gridDim.z / a.splits;
    const size_t base_lo = (((size_t)split * B + b) * a.Hq + h_lo) * a.n + pos_lo;
    const size_t base_hi = (((size_t)split * B + b) * a.Hq + h_hi) * a.n + pos_hi;
#pragma unroll
    for (int j = 0; j < HD / 8; ++j) {
      const int col = j * 8 + (lane & 3) * 2;
      if (ok_lo) *reinterpret_cast<float2 *>(&a.part_o[base_lo * HD + col]) = make_float2(o[j][0], o[j][1]);
      if (ok_hi) *reinterpret_cast<float2 *>(&a.part_o[base_hi * HD + col]) = make_float2(o[j][2], o[j][3]);
    }
    if ((lane & 3) == 0) {
      if (ok_lo) a.part_ml[base_lo] = make_float2(m_lo, l_lo);
      if (ok_hi) a.part_ml[base_hi] = make_float2(m_hi, l_hi);
    }
  }
}

// One warp per (batch, head, position): merge the splits in order; lanes cover head_dim with
// float4 loads.
template <int HD>
__global__ void attn_merge_kernel(int splits, int B, int Hq, int n, const float *__restrict__ part_o,
                                  const float2 *__restrict__ part_ml,
                                  const int32_t *__restrict__ done, bf16 *out) {
  const int w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= B * Hq * n) return;
  const int i = w % n, h = (w / n) % Hq, b = w / (n * Hq);
  if (done && done[b]) return;
  float m = -INFINITY;
  for (int s = 0; s < splits; ++s) m = fmaxf(m, part_ml[(((size_t)s * B + b) * Hq + h) * n + i].x);
  const float base = m == -INFINITY ? 0.f : m;
  float l = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < splits; ++s) {
    const size_t r = (((size_t)s * B + b) * Hq + h) * n + i;
    const float2 ml = part_ml[r];
    const float c = exp2f(ml.x - base);
    l += ml.y * c;
    if (lane * 4 < HD) {
      const float4 v = reinterpret_cast<const float4 *>(part_o + r * HD)[lane];
      acc.x += v.x * c; acc.y += v.y * c; acc.z += v.z * c; acc.w += v.w * c;
    }
  }
  const float il = l > 0.f ? 1.f / l : 0.f;
  if (lane * 4 < HD) {
    bf16 *o = out + (((size_t)b * n + i) * Hq + h) * HD + lane * 4;
    *reinterpret_cast<__nv_bfloat162 *>(o) = __floats2bfloat162_rn(acc.x * il, acc.y * il);
    *reinterpret_cast<__nv_bfloat162 *>(o + 2) = __floats2bfloat162_rn(acc.z * il, acc.w * il);
  }
}

// Split-KV plan: as many key splits as fill one wave of CTAs (one CTA per SM at this kernel's
// register use), at least one tile of keys per split, at most MAX_SPLITS.
void plan(int batch, int n, int Hq, int Hkv, int cap, int *splits, int *chunk) {
  const int keys = cap + n;
  const int qpc = ROWS / (Hq / Hkv);
  const int base = ((n + qpc - 1) / qpc) * Hkv * batch;
  int s = num_sms() / (base > 0 ? base : 1);
  const int max_by_keys = (keys + KT - 1) / KT;
  if (s > max_by_keys) s = max_by_keys;
  if (s > MAX_SPLITS) s = MAX_SPLITS;
  if (s < 1) s = 1;
  int c = (keys + s - 1) / s;
  c = (c + KT - 1) / KT * KT;
  *splits = s;
  *chunk = c;
}

}  // namespace

bool attention_tc_supported(int act, int Hq, int Hkv, int hd) {
  const int rep = Hq / Hkv;
  return act == DG_BF16 && (hd == 64 || hd == 128) && rep >= 1 && rep <= 64 && (ROWS % rep) == 0;
}

size_t attention_tc_ws_bytes(int batch, int n, int Hq, int Hkv, int hd, int cap) {
  int s, c;
  plan(batch, n, Hq, Hkv, cap, &s, &c);
  if (s == 1) return 0;
  const size_t rows = (size_t)s * batch * Hq * n;
  return rows * hd * 4 + 256 + rows * sizeof(float2);
}

int launch_attention_tc(int batch, int n, int Hq, int Hkv, int hd, const void *q,
                        const void *k_cache, const void *v_cache, const int32_t *cache_len, int cap,
                        const void *k_new, const void *v_new, int causal, const int32_t *done,
                        void *out, void *ws, cudaStream_t s) {
  AttnArgs a;
  a.q = (const bf16 *)q;
  a.kc = (const bf16 *)k_cache;
  a.vc = (const bf16 *)v_cache;
  a.kn = (const bf16 *)k_new;
  a.vn = (const bf16 *)v_new;
  a.cache_len = cache_len;
  a.done = done;
  a.n = n;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.cap = cap;
  a.causal = causal;
  plan(batch, n, Hq, Hkv, cap, &a.splits, &a.chunk);
  a.out = (bf16 *)out;
  const size_t rows = (size_t)a.splits * batch * Hq * n;
  a.part_o = (float *)ws;
  a.part_ml = (float2 *)((char *)ws + ((rows * hd * 4 + 255) & ~(size_t)255));
  const int rep = Hq / Hkv;
  const int qpc = ROWS / rep;
  dim3 grid((n + qpc - 1) / qpc, Hkv, batch * a.splits);
  note_launch(s, "attn_tc");
  if (hd == 128) {
    cudaFuncSetAttribute(attn_tc_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)attn_smem_bytes<128>());
    attn_tc_kernel<128><<<grid, NTHR, attn_smem_bytes<128>(), s>>>(a);
  } else {
    cudaFuncSetAttribute(attn_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)attn_smem_bytes<64>());
    attn_tc_kernel<64><<<grid, NTHR, attn_smem_bytes<64>(), s>>>(a);
  }
  int rc = check_launch("attn_tc");
  if (rc != DG_OK || a.splits == 1) return rc;
  note_launch(s, "attn_merge");
  const int warps = batch * Hq * n;
  const int mgrid = (warps + 7) / 8;
  if (hd == 128)
    attn_merge_kernel<128><<<mgrid, 256, 0, s>>>(a.splits, batch, Hq, n, a.part_o, a.part_ml,
                                                 done, (bf16 *)out);
  else
    attn_merge_kernel<64><<<mgrid, 256, 0, s>>>(a.splits, batch, Hq, n, a.part_o, a.part_ml, done,
                                                (bf16 *)out);
  return check_launch("attn_merge");
}

}  // namespace dg
