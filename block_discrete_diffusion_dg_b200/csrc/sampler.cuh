// Device side of the sampler variants: the counter-based generator, the Gumbel draw and the
// per-row temperature of the annealed schedule.
//
// "DiffusionGemma Technical Report": the canvas starts from random noise (explanatory visual,
// Figure 3) and the sampler's temperature is annealed over the step budget N (Figure 9: a larger N
// anneals more mildly; Figure 10: tau_t = 1 with annealing off).  Readings:
//   tau_s = tau_start + (tau_end - tau_start) * min(s, N - 1) / max(N - 1, 1)   (fp64)
//   a token is drawn from softmax(z / tau) as argmax_v (z_v * (1/tau) + G_v), G = -ln(-ln U)
//   U = ((w >> 9) + 1/2) * 2^-23 for a 32-bit word w of Philox4x32-10 (Salmon, Moraes, Dror and
//   Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC 2011), keyed by the 64-bit seed;
//   counter (v >> 2, a1, a2, (tag << 24) | b), word v & 3, for vocabulary entry v of stream
//   (tag, b, a1, a2).
#pragma once
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "dg_kernels.h"

namespace dg {

constexpr uint32_t PHILOX_M0 = 0xD2511F53u, PHILOX_M1 = 0xCD9E8D57u;
constexpr uint32_t PHILOX_W0 = 0x9E3779B9u, PHILOX_W1 = 0xBB67AE85u;

// Philox4x32 with 10 rounds: (c0, c1, c2, c3) -> (hi(M1 c2) ^ c1 ^ k0, lo(M1 c2),
// hi(M0 c0) ^ c3 ^ k1, lo(M0 c0)), the key growing by (W0, W1) before every round but the first.
__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    if (r) {
      k0 += PHILOX_W0;
      k1 += PHILOX_W1;
    }
    const uint32_t lo0 = PHILOX_M0 * c.x, hi0 = __umulhi(PHILOX_M0, c.x);
    const uint32_t lo1 = PHILOX_M1 * c.z, hi1 = __umulhi(PHILOX_M1, c.z);
    c = make_uint4(hi1 ^ c.y ^ k0, lo1, hi0 ^ c.w ^ k1, lo0);
  }
  return c;
}

// G = -ln(-ln U) for the word w; U is exact in fp32 and lies in [2^-24, 1 - 2^-24], so -ln U is
// positive (the inner logarithm is the accurate one: near U = 1 its result is ~6e-8).
__device__ __forceinline__ float gumbel_of(uint32_t w) {
  const float u = (__uint2float_rn(w >> 9) + 0.5f) * 0x1p-23f;
  return -__logf(-logf(u));
}

// Per-row draw parameters: the fp32 multiplier 1/tau (1 when the row is greedy), whether the row
// draws Gumbel noise, and counter words 1..3 of its stream.
struct RowDraw {
  float inv_tau;
  int on;
  uint32_t c1, c2, c3;
};

__device__ __forceinline__ double anneal_tau(const SampleSpec &sp, int step) {
  const int n1 = sp.max_steps - 1 > 1 ? sp.max_steps - 1 : 1;
  const int s = step < sp.max_steps - 1 ? step : sp.max_steps - 1;
  const double frac = __ddiv_rn((double)(s > 0 ? s : 0), (double)n1);
  return __dadd_rn(sp.tau0, __dmul_rn(__dsub_rn(sp.tau1, sp.tau0), frac));
}

// The draw parameters of source row `src`: mode 1, a canvas position (b = src / canvas,
// i = src % canvas, step s = step[b]; stream (TAG_DENOISE, b, i, s), tau_s annealed); mode 2, the
// last new row of sequence b = src (stream (TAG_AR, b, p, 0) with p = pos[b] + pos_add, the
// position of the token being predicted; tau = tau0).
__device__ __forceinline__ RowDraw row_draw(const SampleSpec &sp, int src) {
  RowDraw rd{1.f, 0, 0u, 0u, 0u};
  double tau = 0.0;
  if (sp.mode == SAMPLE_CANVAS) {
    const int b = src / sp.canvas, i = src - b * sp.canvas;
    const int st = sp.step[b];
    tau = anneal_tau(sp, st);
    rd.c1 = (uint32_t)i;
    rd.c2 = (uint32_t)st;
    rd.c3 = ((uint32_t)SAMPLE_TAG_DENOISE << 24) | (uint32_t)b;
  } else if (sp.mode == SAMPLE_AR) {
    const int b = src;
    tau = sp.tau0;
    rd.c1 = (uint32_t)(sp.pos[b] + sp.pos_add);
    rd.c2 = 0u;
    rd.c3 = ((uint32_t)SAMPLE_TAG_AR << 24) | (uint32_t)b;
  }
  if (tau > 0.0) {
    rd.on = 1;
    rd.inv_tau = __double2float_rn(__ddiv_rn(1.0, tau));
  }
  return rd;
}

// Gumbel draws for the 4 consecutive vocabulary entries 4 q4 .. 4 q4 + 3 of a row's stream.
__device__ __forceinline__ float4 gumbel4(const RowDraw &rd, uint32_t q4, uint32_t k0,
                                          uint32_t k1) {
  const uint4 w = philox4x32_10(make_uint4(q4, rd.c1, rd.c2, rd.c3), k0, k1);
  return make_float4(gumbel_of(w.x), gumbel_of(w.y), gumbel_of(w.z), gumbel_of(w.w));
}

}  // namespace dg
