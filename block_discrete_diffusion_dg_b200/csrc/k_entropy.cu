// Softmax entropy and greedy argmax over materialised fp32 logits (one block per row,
// 128-bit coalesced loads).  "DiffusionGemma Technical Report", explanatory visual: the
// entropy-bounded sampler ranks canvas positions by the entropy of their predictive
// distribution; Table 1: vocabulary 262k.
//
// Streaming state per thread, for the logits z seen so far:
//   m = max z,  s = sum e^(z - m),  u = sum e^(z - m) (z - m)
// so that H = -sum p ln p = ln s - u / s.  Two states merge exactly:
//   m = max(m1, m2),  c_i = e^(m_i - m),  s = s1 c1 + s2 c2,
//   u = c1 (u1 + s1 (m1 - m)) + c2 (u2 + s2 (m2 - m)).
// Argmax keeps the first index of the maximum (lower index wins between equal values).
#include "dg_common.cuh"
#include "dg_kernels.h"
#include "entropy_state.cuh"
#include "sampler.cuh"

namespace dg {

namespace {

// SAMPLE: row r's token is drawn as smp says (see sampler.cuh): the softmax state of z/tau and
// the first argmax of z/tau + G.
template <bool SAMPLE>
__global__ void __launch_bounds__(256) entropy_rows_kernel(const float *__restrict__ logits, int V,
                                                           const int32_t *__restrict__ n_rows,
                                                           const int32_t *__restrict__ row_idx,
                                                           float *entropy, int32_t *argmax,
                                                           int32_t *st, SampleSpec smp) {
  pdl_wait();
  pdl_trigger();
  const int r = blockIdx.x;
  if (n_rows && r >= *n_rows) return;
  const float *z = logits + (size_t)r * V;
  EntState es;
  es.init();
  RowDraw rd{1.f, 0, 0u, 0u, 0u};
  if (SAMPLE) rd = row_draw(smp, row_idx ? row_idx[r] : r);
  if ((V & 3) == 0) {
    const float4 *z4 = reinterpret_cast<const float4 *>(z);
    for (int c = threadIdx.x; c < V / 4; c += blockDim.x) {
      const float4 v = z4[c];
      if (SAMPLE) {
        const float4 g = rd.on ? gumbel4(rd, (uint32_t)c, smp.key0, smp.key1)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
        const float a = v.x * rd.inv_tau, b = v.y * rd.inv_tau;
        const float cc = v.z * rd.inv_tau, d = v.w * rd.inv_tau;
        es.add_keyed(a, a + g.x, 4 * c);
        es.add_keyed(b, b + g.y, 4 * c + 1);
        es.add_keyed(cc, cc + g.z, 4 * c + 2);
        es.add_keyed(d, d + g.w, 4 * c + 3);
      } else {
        es.add(v.x, 4 * c);
        es.add(v.y, 4 * c + 1);
        es.add(v.z, 4 * c + 2);
        es.add(v.w, 4 * c + 3);
      }
    }
  } else {
    for (int c = threadIdx.x; c < V; c += blockDim.x) {
      if (SAMPLE) {
        float g = 0.f;
        if (rd.on) {
          const float4 g4 = gumbel4(rd, (uint32_t)(c >> 2), smp.key0, smp.key1);
          g = (c & 3) == 0 ? g4.x : (c & 3) == 1 ? g4.y : (c & 3) == 2 ? g4.z : g4.w;
        }
        const float a = z[c] * rd.inv_tau;
        es.add_keyed(a, a + g, c);
      } else {
        es.add(z[c], c);
      }
    }
  }
  __shared__ EntState red[8];
  es = es.warp_reduce();
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = es;
  __syncthreads();
  if (threadIdx.x == 0) {
    EntState t = red[0];
    for (int i = 1; i < (int)(blockDim.x >> 5); ++i) t.merge(red[i]);
    const float H = t.entropy();
    const int out = row_idx ? row_idx[r] : r;
    if (!isfinite(H)) set_status(st, DG_ERR_NUMERIC);
    entropy[out] = H;
    argmax[out] = t.am;
  }
}

__global__ void scatter_rows_kernel(const float *__restrict__ src, int width,
                                    const int32_t *__restrict__ n_rows,
                                    const int32_t *__restrict__ row_idx, float *dst) {
  pdl_wait();
  pdl_trigger();
  const int r = blockIdx.y;
  if (n_rows && r >= *n_rows) return;
  const float *sr = src + (size_t)r * width;
  float *dr = dst + (size_t)row_idx[r] * width;
  for (int c = blockIdx.x * blockDim.x + threadIdx.x; c < width; c += gridDim.x * blockDim.x)
    dr[c] = sr[c];
}

}  // namespace

int launch_scatter_rows(const float *src, int width, int max_rows, const int32_t *n_rows,
                        const int32_t *row_idx, float *dst, cudaStream_t s) {
  if (max_rows <= 0) return DG_OK;
  note_launch(s, "scatter_rows");
  dim3 grid((width + 1023) / 1024 < 64 ? (width + 1023) / 1024 : 64, max_rows);
  launch_pdl(scatter_rows_kernel, grid, 256, 0, s, src, width, n_rows, row_idx, dst);
  return check_launch("scatter_rows");
}

int launch_entropy_rows(const float *logits, int V, int max_rows, const int32_t *n_rows,
                        const int32_t *row_idx, float *entropy, int32_t *argmax, int32_t *st,
                        cudaStream_t s, const SampleSpec *smp) {
  if (max_rows <= 0) return DG_OK;
  note_launch(s, "entropy_rows");
  SampleSpec sp{};
  const bool sample = smp && smp->mode != SAMPLE_GREEDY;
  if (sample) sp = *smp;
  launch_pdl(sample ? entropy_rows_kernel<true> : entropy_rows_kernel<false>, max_rows, 256, 0, s,
             logits, V, n_rows, row_idx, entropy, argmax, st, sp);
  return check_launch("entropy_rows");
}

}  // namespace dg
