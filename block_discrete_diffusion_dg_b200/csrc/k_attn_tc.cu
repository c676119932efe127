// Canvas attention on tensor cores with split-KV: a tcgen05 kernel for head_dim 128 (below) and an
// mma.sync m16n8k16 kernel for head_dim 64.
// "DiffusionGemma Technical Report", Figure 4: the decoder attends bidirectionally across the
// canvas and to the cached context (cross-attention to the KV cache); the causal encoder of the
// append attends causally within the new tokens.  Model card "diffusiongemma", Model Overview.
//
// A tile of 128 query rows shares one kv head: the rep = Hq / Hkv query heads of that kv head
// times 128 / rep consecutive canvas positions, so every K/V tile is read once per GQA group.
// Keys are split into chunks (split-KV) so that short and 131k-key contexts both fill the GPU;
// each split leaves an unnormalised partial (O, running max m, sum l) that lm-style merging
// combines exactly:  m = max m_s, l = sum l_s 2^(m_s - m), O = sum O_s 2^(m_s - m) / l.
// Scores are kept in the log2 domain: t = q.k / sqrt(hd) * log2(e).
// Precision: S = Q K^T takes the stored bf16 q and k exactly (fp32 accumulation).  The second
// product takes V in fp16 (every bf16 value of V is exact in fp16 for |v| < 65504; below fp16's
// normal range the absolute error stays < 3e-8) and P:
//   tcgen05 kernel: P = P_hi + P_lo, two fp16 parts (~22 significant bits).  The output is an
//                   average over many keys with cancelling signs, so a relative error e in each p
//                   reaches O at about e * sqrt(effective keys) of O's own size: with one fp16
//                   part (e ~ 2^-12) about a tenth of the outputs land on the other side of a bf16
//                   rounding boundary, which shows in the logits downstream;
//   mma.sync kernel: P in fp16 (11 significant bits).
// The mma.sync kernel: 8 warps x 16 rows; K/V tiles of 64 keys double-buffered with cp.async
// (zero-filled past the end) in XOR-swizzled shared memory read by ldmatrix; each thread converts
// the V chunks it loaded, in place, once they have landed.
#include "dg_common.cuh"
#include "dg_kernels.h"
#include "tc_common.cuh"
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
// 2^x by the hardware approximation (PTX ex2.approx.ftz: relative error ~2^-22, -inf -> +0).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// max(a, b, c) in one instruction (three-input max.f32, sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
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
  pdl_wait();
  pdl_trigger();
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
  pdl_wait();
  pdl_trigger();
  const int w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= B * Hq * n) return;
  const int i = w % n, h = (w / n) % Hq, b = w / (n * Hq);
  if (done && done[b]) return;
  // the (m, l) of up to eight splits and their O slices are loaded together, then combined in
  // split order
  const size_t sstride = (size_t)B * Hq * n, r0 = ((size_t)b * Hq + h) * n + i;
  if (splits <= 16) {  // one round of loads: every split's (m, l) and O slice at once
    float2 ml[16];
    float4 v[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if (j < splits) {
        const size_t r = j * sstride + r0;
        ml[j] = part_ml[r];
        if (lane * 4 < HD) v[j] = reinterpret_cast<const float4 *>(part_o + r * HD)[lane];
      }
    }
    float m = -INFINITY;
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if (j < splits) m = fmaxf(m, ml[j].x);
    const float base = m == -INFINITY ? 0.f : m;
    float l = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if (j >= splits) continue;
      const float c = exp2f(ml[j].x - base);
      l += ml[j].y * c;
      if (lane * 4 < HD) {
        acc.x += v[j].x * c; acc.y += v[j].y * c; acc.z += v[j].z * c; acc.w += v[j].w * c;
      }
    }
    const float il = l > 0.f ? 1.f / l : 0.f;
    if (lane * 4 < HD) {
      bf16 *o = out + (((size_t)b * n + i) * Hq + h) * HD + lane * 4;
      *reinterpret_cast<__nv_bfloat162 *>(o) = __floats2bfloat162_rn(acc.x * il, acc.y * il);
      *reinterpret_cast<__nv_bfloat162 *>(o + 2) = __floats2bfloat162_rn(acc.z * il, acc.w * il);
    }
    return;
  }
  float m = -INFINITY;
  for (int s0 = 0; s0 < splits; s0 += 8) {
    float mv[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) mv[j] = s0 + j < splits ? part_ml[(s0 + j) * sstride + r0].x : -INFINITY;
#pragma unroll
    for (int j = 0; j < 8; ++j) m = fmaxf(m, mv[j]);
  }
  const float base = m == -INFINITY ? 0.f : m;
  float l = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s0 = 0; s0 < splits; s0 += 8) {
    float2 ml[8];
    float4 v[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (s0 + j < splits) {
        const size_t r = (s0 + j) * sstride + r0;
        ml[j] = part_ml[r];
        if (lane * 4 < HD) v[j] = reinterpret_cast<const float4 *>(part_o + r * HD)[lane];
      }
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (s0 + j >= splits) continue;
      const float c = exp2f(ml[j].x - base);
      l += ml[j].y * c;
      if (lane * 4 < HD) {
        acc.x += v[j].x * c; acc.y += v[j].y * c; acc.z += v[j].z * c; acc.w += v[j].w * c;
      }
    }
  }
  const float il = l > 0.f ? 1.f / l : 0.f;
  if (lane * 4 < HD) {
    bf16 *o = out + (((size_t)b * n + i) * Hq + h) * HD + lane * 4;
    *reinterpret_cast<__nv_bfloat162 *>(o) = __floats2bfloat162_rn(acc.x * il, acc.y * il);
    *reinterpret_cast<__nv_bfloat162 *>(o + 2) = __floats2bfloat162_rn(acc.z * il, acc.w * il);
  }
}

// ================================================================================================
// tcgen05 path (head_dim 128).  One CTA = two tiles of 128 query rows (A and B: the rep query
// heads of one kv head times 2 x 128/rep consecutive canvas positions) x one key split, with both
// products on the 5th-generation tensor cores and the accumulators in tensor memory:
//   S_X = Q_X K_i^T  (M 128 rows, N 128 keys, K 128 = head_dim; bf16 operands from shared memory)
//   O_X += P_X V_i   (M 128 rows, N 128 = head_dim, K 128 keys, twice: P_hi and P_lo fp16 from
//                     tensor memory, V fp16 in shared memory, read MN-major)
// TMEM (512 columns): S_A [0,128), S_B [128,256), O_A [256,384), O_B [384,512).  P_X is written
// over S_X as two fp16 parts, P = P_hi + P_lo (hi pairs in columns [0,64), lo pairs in [64,128)),
// and O_X += P_hi V + P_lo V, so P reaches the product with ~22 significant bits; S_X of the next
// key tile is issued right behind P_X V of this one (in-order MMA execution keeps the read of P
// ahead of the overwrite).  The tensor cores run PV_A(i), S_A(i+1), PV_B(i), S_B(i+1):
// while one softmax warpgroup works on its tile, the MMAs of the other proceed.
// Warp roles (384 threads):
//   warp 0     TMA: both Q tiles once, then K and V tiles of 128 keys (3- and 2-stage rings);
//   warp 1     owns the TMEM columns and issues the MMAs;
//   warps 2-3  convert each landed V tile from bf16 to fp16 in place and zero the rows past the
//              last valid key (so masked keys contribute exactly 0 * 0);
//   warps 4-7  softmax of tile A, warps 8-11 of tile B: one query row per thread (= TMEM lane);
//              the row of S read in one round of TMEM loads, mask, running max in the log2
//              domain, P = 2^(t - m) written back to TMEM as fp16 hi and lo pairs, row sum in
//              fp32 (scale-and-shift, sum and split in packed fp32x2 arithmetic).
// The running maximum is applied lazily: O is rescaled (read, scaled, written back in TMEM) only
// when a row's maximum grows by more than 2^8, so between rescales P can reach 256 (well inside
// fp16's range; the final O / l is unchanged because O and l always share the same base).
// Control flow of the softmax warps is warp-uniform (votes on every exit and on the rescale
// decision): TMEM loads and stores are .sync.aligned and need all 32 lanes.
// Every wait is bounded; on expiry the kernel records DG_ERR_TIMEOUT, lets issued copies and
// MMAs finish, frees TMEM and returns.
#ifndef DG_ATTN_REGS_LO
#define DG_ATTN_REGS_LO 104
#endif
#ifndef DG_ATTN_REGS_HI
#define DG_ATTN_REGS_HI 200
#endif
constexpr int T5_HD = 128, T5_KT = 128, T5_KS = 3, T5_VS = 2, T5_THR = 384;
constexpr int T5_HALF = 128 * 128;       // one box: 128 rows x 64 bf16 (128-byte rows) = 16 KB
constexpr int T5_TILE = 2 * T5_HALF;     // 128 rows x 128 head dims = 32 KB
constexpr uint32_t T5_COL_S = 0, T5_COL_O = 256, T5_TMEM_COLS = 512;
constexpr float T5_RESCALE = 8.f;        // log2 of the largest P between rescales
constexpr size_t T5_SMEM = 1024 + (size_t)T5_TILE * (2 + T5_KS + T5_VS) + 512;
// registers per thread at launch, and after the split for the copy / MMA / converter warpgroup
// (LO) and the two softmax warpgroups (HI)
constexpr int T5_REGS = 168, T5_REGS_LO = DG_ATTN_REGS_LO, T5_REGS_HI = DG_ATTN_REGS_HI;
static_assert(128 * T5_REGS_LO + 256 * T5_REGS_HI <= T5_THR * T5_REGS, "register split");
static_assert(T5_THR * T5_REGS <= 65536, "launch registers");

template <int R>
__device__ __forceinline__ void setmaxnreg_dec() {
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(R));
}
template <int R>
__device__ __forceinline__ void setmaxnreg_inc() {
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(R));
}
constexpr unsigned FULL = 0xffffffffu;

struct T5Args {
  const int32_t *cache_len, *done;
  int n, Hq, Hkv, cap, causal, splits, chunk_tiles;
  bf16 *out;          // splits == 1
  float *part_o;      // [splits][B][Hq][n][HD]
  float2 *part_ml;    // [splits][B][Hq][n]
  int32_t *status;
};

__device__ __forceinline__ void t5_fail(int32_t *st, volatile int *abort_flag) {
  set_status(st, DG_ERR_TIMEOUT);
  *abort_flag = 1;
}

__global__ void __launch_bounds__(T5_THR, 1)
    attn_tc5_kernel(const __grid_constant__ CUtensorMap tmQ,
                    const __grid_constant__ CUtensorMap tmKc,
                    const __grid_constant__ CUtensorMap tmVc,
                    const __grid_constant__ CUtensorMap tmKn,
                    const __grid_constant__ CUtensorMap tmVn, T5Args a) {
  pdl_wait();
  pdl_trigger();
  using namespace tc;
  extern __shared__ uint8_t t5_smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>(((uintptr_t)t5_smem_raw + 1023) & ~(uintptr_t)1023);
  uint8_t *sQ = smem;                       // [2 tiles][TILE]
  uint8_t *sK = sQ + 2 * T5_TILE;
  uint8_t *sV = sK + T5_KS * T5_TILE;
  uint64_t *q_full = reinterpret_cast<uint64_t *>(sV + T5_VS * T5_TILE);
  uint64_t *k_full = q_full + 1, *k_empty = k_full + T5_KS;
  uint64_t *v_full = k_empty + T5_KS, *v_ready = v_full + T5_VS, *v_empty = v_ready + T5_VS;
  uint64_t *s_full = v_empty + T5_VS, *p_full = s_full + 2, *pv_done = p_full + 2;  // [tile]
  uint64_t *mma_fin = pv_done + 2;
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mma_fin + 1);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const int split = blockIdx.z % a.splits, b = blockIdx.z / a.splits;
  if (a.done && a.done[b]) return;  // uniform across the block
  const int g = blockIdx.y, rep = a.Hq / a.Hkv, qpc = ROWS / rep, i0 = blockIdx.x * 2 * qpc;
  const int len = min(max(a.cache_len[b], 0), a.cap);
  const int tcache = (len + T5_KT - 1) / T5_KT;
  int tiles = tcache + (a.n + T5_KT - 1) / T5_KT;
  if (a.causal) tiles = tcache + (min(a.n, i0 + 2 * qpc) - 1) / T5_KT + 1;  // later keys unseen
  const int t_begin = split * a.chunk_tiles;
  const int N = max(0, min(tiles, t_begin + a.chunk_tiles) - t_begin);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slab_c = (b * a.Hkv + g) * a.cap, slab_n = (b * a.Hkv + g) * a.n;

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < T5_KS; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < T5_VS; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_ready[s], 2);
      mbar_init(&v_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&s_full[x], 1);
      mbar_init(&p_full[x], 4);
      mbar_init(&pv_done[x], 1);
    }
    mbar_init(mma_fin, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmKc);
    tma_prefetch_desc(&tmVc);
    tma_prefetch_desc(&tmKn);
    tma_prefetch_desc(&tmVn);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, T5_TMEM_COLS);
    tmem_relinquish();
  }
  fence_before();
  __syncthreads();
  fence_after();
  const uint32_t tmem = *tmem_slot;

  // key tile i of this split: cache rows [j0, j0 + 128) or canvas rows; `valid` keys in it
  auto tile_src = [&](int i, bool &cache, int &row, int &j0, int &valid) {
    const int t = t_begin + i;
    cache = t < tcache;
    j0 = cache ? t * T5_KT : (t - tcache) * T5_KT;
    row = (cache ? slab_c : slab_n) + j0;
    valid = min(T5_KT, (cache ? len : a.n) - j0);
  };

  // Register split: the copy / MMA / converter warpgroup hands registers to the two softmax
  // warpgroups, which hold a whole row of S.  Launch: 384 threads x T5_REGS; after the split:
  // 128 x T5_REGS_LO + 256 x T5_REGS_HI, no more than the launch holds (the host checks the
  // kernel's register count before the first launch).
  if (warp == 0) {
    setmaxnreg_dec<T5_REGS_LO>();
    if (lane == 0) {
      uint32_t armed_k = 0, armed_v = 0;  // tiles whose copies were issued
      bool ok = true;
      mbar_expect_tx(q_full, 2 * T5_TILE);
      for (int x = 0; x < 2; ++x)
        for (int hl = 0; hl < rep; ++hl)
          for (int hf = 0; hf < 2; ++hf)
            tma_load_2d(sQ + x * T5_TILE + hf * T5_HALF + hl * qpc * 128, &tmQ, q_full,
                        (g * rep + hl) * T5_HD + hf * 64, b * a.n + i0 + x * qpc);
      for (int i = 0; i < N && ok && !*abort_flag; ++i) {
        bool cache;
        int row, j0, valid;
        tile_src(i, cache, row, j0, valid);
        const int ks = i % T5_KS, vs = i % T5_VS;
        if (!mbar_wait(&k_empty[ks], ((i / T5_KS) & 1) ^ 1)) { ok = false; break; }
        mbar_expect_tx(&k_full[ks], T5_TILE);
        const CUtensorMap *tk = cache ? &tmKc : &tmKn;
        tma_load_2d(sK + ks * T5_TILE, tk, &k_full[ks], 0, row);
        tma_load_2d(sK + ks * T5_TILE + T5_HALF, tk, &k_full[ks], 64, row);
        armed_k = i + 1;
        if (!mbar_wait(&v_empty[vs], ((i / T5_VS) & 1) ^ 1)) { ok = false; break; }
        mbar_expect_tx(&v_full[vs], T5_TILE);
        const CUtensorMap *tv = cache ? &tmVc : &tmVn;
        tma_load_2d(sV + vs * T5_TILE, tv, &v_full[vs], 0, row);
        tma_load_2d(sV + vs * T5_TILE + T5_HALF, tv, &v_full[vs], 64, row);
        armed_v = i + 1;
      }
      if (!ok) t5_fail(a.status, abort_flag);
      // the copies in flight land before the CTA's shared memory can go away
      (void)mbar_wait(q_full, 0);
      for (uint32_t i = armed_k > T5_KS ? armed_k - T5_KS : 0; i < armed_k; ++i)
        (void)mbar_wait(&k_full[i % T5_KS], (i / T5_KS) & 1);
      for (uint32_t i = armed_v > T5_VS ? armed_v - T5_VS : 0; i < armed_v; ++i)
        (void)mbar_wait(&v_full[i % T5_VS], (i / T5_VS) & 1);
    }
  } else if (warp == 1) {
    setmaxnreg_dec<T5_REGS_LO>();
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16(ROWS, T5_KT);
      const uint32_t id_p = idesc_f16_bmn(ROWS, T5_HD);
      bool ok = mbar_wait(q_full, 0);
      fence_after();
      // Descriptors of the operand buffers, computed once: a descriptor's start-address field is
      // the shared-memory byte address / 16 (all of shared memory fits its 14 bits), so an offset
      // of b bytes is added as b / 16.  Issuing an MMA then costs an add and the instruction;
      // building both descriptors per MMA cost more issue time than an N = 128 MMA takes.
      const uint64_t dq = sdesc_sw128(sQ), dk = sdesc_sw128(sK);
      const uint64_t dv = sdesc_sw128_mn(sV, T5_HALF);
      auto issue_s = [&](int x, int i) {   // S_x(i) = Q_x K_i^T into S_x
        const uint64_t ab = dq + (uint64_t)((x * T5_TILE) >> 4);
        const uint64_t bb = dk + (uint64_t)(((i % T5_KS) * T5_TILE) >> 4);
        const uint32_t d = tmem + T5_COL_S + (uint32_t)x * 128;
#pragma unroll
        for (int kk = 0; kk < T5_HD / 16; ++kk) {
          const uint64_t off = (uint64_t)(((kk >> 2) * T5_HALF) >> 4) + 2 * (kk & 3);
          mma_bf16(d, ab + off, bb + off, id_s, kk > 0 ? 1u : 0u);
        }
        commit(&s_full[x]);
      };
      auto issue_pv = [&](int x, int i) {  // O_x += P_x V_i
        const uint64_t bb = dv + (uint64_t)(((i % T5_VS) * T5_TILE) >> 4);
        const uint32_t pa = tmem + T5_COL_S + (uint32_t)x * 128;
        const uint32_t d = tmem + T5_COL_O + (uint32_t)x * 128;
        const uint32_t acc0 = i != 0 ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < T5_KT / 16; ++kk) {  // P = P_hi + P_lo, both against the same V
          const uint64_t bd = bb + (uint64_t)((kk * 16 * 128) >> 4);
          mma_f16_ts(d, pa + kk * 8, bd, id_p, kk != 0 ? 1u : acc0);
          mma_f16_ts(d, pa + 64 + kk * 8, bd, id_p, 1u);
        }
        commit(&pv_done[x]);
      };
      if (ok && N > 0) {
        ok = mbar_wait(&k_full[0], 0);
        if (ok) {
          fence_after();
          issue_s(0, 0);
          issue_s(1, 0);
          commit(&k_empty[0]);
        }
      }
      for (int i = 0; ok && i < N && !*abort_flag; ++i) {
        const int vs = i % T5_VS;
        const uint32_t ph = i & 1;
        if (!mbar_wait(&v_ready[vs], (i / T5_VS) & 1) || !mbar_wait(&p_full[0], ph)) {
          ok = false;
          break;
        }
        fence_after();
        issue_pv(0, i);
        const bool more = i + 1 < N;
        // S_x(i+1) is written over P_x(i), which PV_x(i) reads.  It is issued right behind it:
        // MMAs issued by one thread execute in issue order (tcgen05.mma -> tcgen05.mma is a
        // pipelined pair), so PV_x(i) has read P_x(i) before S_x(i+1) writes those columns, and the
        // tensor pipe does not drain between the two.
        if (more) {
          if (!mbar_wait(&k_full[(i + 1) % T5_KS], ((i + 1) / T5_KS) & 1)) {
            ok = false;
            break;
          }
          fence_after();
          issue_s(0, i + 1);
        }
        if (!mbar_wait(&p_full[1], ph)) { ok = false; break; }
        fence_after();
        issue_pv(1, i);
        commit(&v_empty[vs]);
        if (more) {
          issue_s(1, i + 1);
          commit(&k_empty[(i + 1) % T5_KS]);
        }
      }
      if (!ok) t5_fail(a.status, abort_flag);
      commit(mma_fin);  // every MMA issued above has completed when this phase does
      (void)mbar_wait(mma_fin, 0);
    }
  } else if (warp < 4) {
    setmaxnreg_dec<T5_REGS_LO>();
    const int ct = threadIdx.x - 64;  // 0..63
    for (int i = 0; i < N; ++i) {
      if (__any_sync(FULL, *abort_flag != 0)) break;
      const int vs = i % T5_VS;
      if (!__all_sync(FULL, mbar_wait(&v_full[vs], (i / T5_VS) & 1))) {
        t5_fail(a.status, abort_flag);
        break;
      }
      bool cache;
      int row, j0, valid;
      tile_src(i, cache, row, j0, valid);
      uint8_t *base = sV + vs * T5_TILE;
      // 16-byte chunk c sits in key row (c mod 1024) / 8 of its half (the swizzle only permutes
      // chunks within a row), so the work is in place and per chunk
#pragma unroll 4
      for (int c = ct; c < T5_TILE / 16; c += 64) {
        uint4 *pc = reinterpret_cast<uint4 *>(base + c * 16);
        if (((c & 1023) >> 3) < valid) bf16x8_to_f16x8(pc);
        else *pc = make_uint4(0u, 0u, 0u, 0u);
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&v_ready[vs]);
    }
  } else {
    setmaxnreg_inc<T5_REGS_HI>();
    const int x = (warp - 4) >> 2;            // query tile (A or B) of this warpgroup
    const int q4 = warp & 3;                  // TMEM lane quarter of this warp
    const int r = q4 * 32 + lane;             // query row of the tile
    const int hl = r / qpc, pos = i0 + x * qpc + r % qpc, h = g * rep + hl;
    const uint32_t lrow = (uint32_t)(q4 * 32) << 16;
    const uint32_t cS = T5_COL_S + (uint32_t)x * 128, cO = T5_COL_O + (uint32_t)x * 128;
    const float sl2 = 1.4426950408889634f / sqrtf((float)T5_HD);
    float m_use = -INFINITY, l = 0.f;
    bool ok = true;
    for (int i = 0; i < N; ++i) {
      if (__any_sync(FULL, *abort_flag != 0)) { ok = false; break; }
      if (!__all_sync(FULL, mbar_wait(&s_full[x], i & 1))) {
        t5_fail(a.status, abort_flag);
        ok = false;
        break;
      }
      fence_after();
      bool cache;
      int row, j0, valid;
      tile_src(i, cache, row, j0, valid);
      int lim = valid;
      if (a.causal && !cache) lim = min(lim, pos - j0 + 1);
      // the row of S in registers: two 64-column TMEM loads (few tcgen05 instructions, since
      // they share the SM's tensor-memory instruction path with the MMAs of the other tile)
      uint32_t sa[64], sb[64];
      tmem_ld64(tmem + lrow + cS, sa);
      tmem_ld64(tmem + lrow + cS + 64, sb);
      tmem_ld_wait64(sa);
      tmem_ld_wait64(sb);
      if (__any_sync(FULL, lim < T5_KT)) {   // a partial or causal tile: mask
#pragma unroll
        for (int j = 0; j < 64; ++j) {
          if (j >= lim) sa[j] = __float_as_uint(-INFINITY);
          if (64 + j >= lim) sb[j] = __float_as_uint(-INFINITY);
        }
      }
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      auto fold_max = [&](const uint32_t (&v)[64]) {
#pragma unroll
        for (int j = 0; j < 64; j += 2)
          m4[(j >> 1) & 3] = fmax3(m4[(j >> 1) & 3], __uint_as_float(v[j]), __uint_as_float(v[j + 1]));
      };
      fold_max(sa);
      fold_max(sb);
      const float mt = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl2;
      const float m_new = fmaxf(m_use, mt);
      // a row whose maximum grew by more than 2^8 needs O rescaled; the whole warp then rescales
      // (factor 1 where nothing changed; a row with nothing accumulated yet only takes m_new)
      if (__any_sync(FULL, m_use != -INFINITY && m_new > m_use + T5_RESCALE)) {
        const float f = m_use == -INFINITY ? 1.f : ex2_approx(m_use - m_new);
        // O must include PV(i-1) before scaling
        if (i >= 1 && !__all_sync(FULL, mbar_wait(&pv_done[x], (i - 1) & 1))) {
          t5_fail(a.status, abort_flag);
          ok = false;
          break;
        }
        fence_after();
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem + lrow + cO + c * 32, o);
          tmem_ld_wait(o);
#pragma unroll
          for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * f);
          tmem_st32(tmem + lrow + cO + c * 32, o);
        }
        tmem_st_wait();
        l *= f;
        m_use = m_new;
      } else if (m_use == -INFINITY) {
        m_use = m_new;  // nothing accumulated yet (O is exactly 0 or not yet written)
      }
      const float nb = m_use == -INFINITY ? 0.f : -m_use;
      const float2 sl2v = make_float2(sl2, sl2), nbv = make_float2(nb, nb);
      float2 s2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      // P of 64 keys (half hf of the row), split into two fp16 parts (P = hi + lo to ~22 bits):
      // hi pairs go to columns [32 hf, 32 hf + 32) of S, lo pairs to [64 + 32 hf, 96 + 32 hf).
      // Every S value of the row is in registers by then, so the order of the writes is free.
      auto emit = [&](const uint32_t (&v)[64], int hf) {
        uint32_t ph[32], pl[32];
#pragma unroll
        for (int j = 0; j < 64; j += 2) {
          const float2 t = __ffma2_rn(make_float2(__uint_as_float(v[j]), __uint_as_float(v[j + 1])),
                                      sl2v, nbv);
          const float2 p = make_float2(ex2_approx(t.x), ex2_approx(t.y));
          s2[(j >> 1) & 1] = __fadd2_rn(s2[(j >> 1) & 1], p);
          const __half2 hi = __floats2half2_rn(p.x, p.y);
          const float2 d = __ffma2_rn(__half22float2(hi), make_float2(-1.f, -1.f), p);  // p - hi
          const __half2 lo = __floats2half2_rn(d.x, d.y);
          ph[j >> 1] = *reinterpret_cast<const uint32_t *>(&hi);
          pl[j >> 1] = *reinterpret_cast<const uint32_t *>(&lo);
        }
        tmem_st32(tmem + lrow + cS + hf * 32, ph);
        tmem_st32(tmem + lrow + cS + 64 + hf * 32, pl);
      };
      emit(sa, 0);
      emit(sb, 1);
      l += (s2[0].x + s2[0].y) + (s2[1].x + s2[1].y);
      tmem_st_wait();
      fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[x]);
    }
    if (ok && N > 0) {
      if (!__all_sync(FULL, mbar_wait(&pv_done[x], (N - 1) & 1))) {
        t5_fail(a.status, abort_flag);
        ok = false;
      }
      fence_after();
    }
    const bool row_ok = pos < a.n;  // guards the stores only; every lane reads TMEM
    if (ok) {
      if (a.splits == 1) {
        const float il = l > 0.f ? 1.f / l : 0.f;
        bf16 *dst = a.out + (((size_t)b * a.n + min(pos, a.n - 1)) * a.Hq + h) * T5_HD;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          tmem_ld32(tmem + lrow + cO + c * 32, o);
          tmem_ld_wait(o);
#pragma unroll
          for (int j = 0; j < 32; j += 8) {
            uint4 v;
            uint32_t *w = reinterpret_cast<uint32_t *>(&v);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const __nv_bfloat162 t = __floats2bfloat162_rn(__uint_as_float(o[j + 2 * e]) * il,
                                                             __uint_as_float(o[j + 2 * e + 1]) * il);
              w[e] = *reinterpret_cast<const uint32_t *>(&t);
            }
            if (row_ok) *reinterpret_cast<uint4 *>(dst + c * 32 + j) = v;
          }
        }
      } else {
        const int B = gridDim.z / a.splits;
        const size_t pr = (((size_t)split * B + b) * a.Hq + h) * a.n + min(pos, a.n - 1);
        float *dst = a.part_o + pr * T5_HD;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t o[32];
          if (N > 0) {
            tmem_ld32(tmem + lrow + cO + c * 32, o);
            tmem_ld_wait(o);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) o[j] = 0u;
          }
          if (row_ok) {
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              *reinterpret_cast<uint4 *>(dst + c * 32 + j) =
                  make_uint4(o[j], o[j + 1], o[j + 2], o[j + 3]);
          }
        }
        if (row_ok) a.part_ml[pr] = make_float2(m_use, l);
      }
    }
  }
  fence_before();
  __syncthreads();
  if (warp == 1) {
    fence_after();
    tmem_dealloc(tmem, T5_TMEM_COLS);
  }
}

// Split plan of the tcgen05 path: tiles of 128 keys; as many splits as fill one wave.
void plan5(int batch, int n, int Hq, int Hkv, int cap, int *splits, int *chunk_tiles) {
  const int tiles = (cap + T5_KT - 1) / T5_KT + (n + T5_KT - 1) / T5_KT;
  const int qpc2 = 2 * (ROWS / (Hq / Hkv));
  const int base = ((n + qpc2 - 1) / qpc2) * Hkv * batch;
  int s = num_sms() / (base > 0 ? base : 1);
  if (s > tiles) s = tiles;
  if (s > MAX_SPLITS) s = MAX_SPLITS;
  if (s < 1) s = 1;
  const int c = (tiles + s - 1) / s;
  *chunk_tiles = c;
  *splits = (tiles + c - 1) / c;
}

bool use_tc5(int batch, int n, int Hq, int Hkv, int hd, int cap) {
  const int rep = Hq / Hkv;
  return hd == T5_HD && rep <= 16 && (size_t)batch * Hkv * (size_t)(cap > n ? cap : n) < (1u << 31) &&
         (size_t)batch * n < (1u << 31);
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
  if (use_tc5(batch, n, Hq, Hkv, hd, cap)) plan5(batch, n, Hq, Hkv, cap, &s, &c);
  else plan(batch, n, Hq, Hkv, cap, &s, &c);
  if (s == 1) return 0;
  const size_t rows = (size_t)s * batch * Hq * n;
  return rows * hd * 4 + 256 + rows * sizeof(float2);
}

namespace {

int launch_tc5(int batch, int n, int Hq, int Hkv, const void *q, const void *k_cache,
               const void *v_cache, const int32_t *cache_len, int cap, const void *k_new,
               const void *v_new, int causal, const int32_t *done, void *out, void *ws,
               int32_t *st, cudaStream_t s) {
  T5Args a;
  a.cache_len = cache_len;
  a.done = done;
  a.n = n;
  a.Hq = Hq;
  a.Hkv = Hkv;
  a.cap = cap;
  a.causal = causal;
  a.status = st;
  plan5(batch, n, Hq, Hkv, cap, &a.splits, &a.chunk_tiles);
  a.out = (bf16 *)out;
  const size_t rows = (size_t)a.splits * batch * Hq * n;
  a.part_o = (float *)ws;
  a.part_ml = (float2 *)((char *)ws + ((rows * T5_HD * 4 + 255) & ~(size_t)255));
  const int qpc = ROWS / (Hq / Hkv);
  CUtensorMap tq, tkc, tvc, tkn, tvn;
  const CUtensorMapDataType bt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  int rc = make_tmap_2d(&tq, bt, 2, q, (uint64_t)Hq * T5_HD, (uint64_t)batch * n,
                        (uint64_t)Hq * T5_HD * 2, 64, qpc);
  if (rc == DG_OK)
    rc = make_tmap_2d(&tkn, bt, 2, k_new, T5_HD, (uint64_t)batch * Hkv * n, T5_HD * 2, 64, T5_KT);
  if (rc == DG_OK)
    rc = make_tmap_2d(&tvn, bt, 2, v_new, T5_HD, (uint64_t)batch * Hkv * n, T5_HD * 2, 64, T5_KT);
  if (rc == DG_OK && cap > 0 && k_cache && v_cache) {
    rc = make_tmap_2d(&tkc, bt, 2, k_cache, T5_HD, (uint64_t)batch * Hkv * cap, T5_HD * 2, 64,
                      T5_KT);
    if (rc == DG_OK)
      rc = make_tmap_2d(&tvc, bt, 2, v_cache, T5_HD, (uint64_t)batch * Hkv * cap, T5_HD * 2, 64,
                        T5_KT);
  } else {
    tkc = tkn;  // no cache rows: never read
    tvc = tvn;
  }
  if (rc != DG_OK) return rc;
  // the in-kernel register split needs the launch to hold T5_REGS registers per thread; a build
  // that allocated fewer would leave setmaxnreg.inc waiting, so it is refused here
  static const int regs = [] {
    cudaFuncAttributes fa{};
    return cudaFuncGetAttributes(&fa, attn_tc5_kernel) == cudaSuccess ? fa.numRegs : -1;
  }();
  if (regs < T5_REGS) return DG_ERR_UNSUPPORTED;
  dim3 grid((n + 2 * qpc - 1) / (2 * qpc), Hkv, batch * a.splits);
  note_launch(s, "attn_tc");
  cudaFuncSetAttribute(attn_tc5_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)T5_SMEM);
  launch_pdl(attn_tc5_kernel, grid, T5_THR, T5_SMEM, s, tq, tkc, tvc, tkn, tvn, a);
  rc = check_launch("attn_tc");
  if (rc != DG_OK || a.splits == 1) return rc;
  note_launch(s, "attn_merge");
  const int warps = batch * Hq * n;
  launch_pdl(attn_merge_kernel<128>, (warps + 7) / 8, 256, 0, s, a.splits, batch, Hq, n, a.part_o,
                                                          a.part_ml, done, (bf16 *)out);
  return check_launch("attn_merge");
}

}  // namespace

int launch_attention_tc(int batch, int n, int Hq, int Hkv, int hd, const void *q,
                        const void *k_cache, const void *v_cache, const int32_t *cache_len, int cap,
                        const void *k_new, const void *v_new, int causal, const int32_t *done,
                        void *out, void *ws, int32_t *st, cudaStream_t s) {
  if (use_tc5(batch, n, Hq, Hkv, hd, cap))
    return launch_tc5(batch, n, Hq, Hkv, q, k_cache, v_cache, cache_len, cap, k_new, v_new, causal,
                      done, out, ws, st, s);
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
    launch_pdl(attn_tc_kernel<128>, grid, NTHR, attn_smem_bytes<128>(), s, a);
  } else {
    cudaFuncSetAttribute(attn_tc_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)attn_smem_bytes<64>());
    launch_pdl(attn_tc_kernel<64>, grid, NTHR, attn_smem_bytes<64>(), s, a);
  }
  int rc = check_launch("attn_tc");
  if (rc != DG_OK || a.splits == 1) return rc;
  note_launch(s, "attn_merge");
  const int warps = batch * Hq * n;
  const int mgrid = (warps + 7) / 8;
  if (hd == 128)
    launch_pdl(attn_merge_kernel<128>, mgrid, 256, 0, s, a.splits, batch, Hq, n, a.part_o,
               a.part_ml, done, (bf16 *)out);
  else
    launch_pdl(attn_merge_kernel<64>, mgrid, 256, 0, s, a.splits, batch, Hq, n, a.part_o,
               a.part_ml, done, (bf16 *)out);
  return check_launch("attn_merge");
}

}  // namespace dg
