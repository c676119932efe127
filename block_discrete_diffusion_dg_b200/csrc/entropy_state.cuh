// Streaming softmax-entropy / argmax state shared by the entropy kernels.
//   m = running max, s = sum e^(z - m), u = sum e^(z - m) (z - m), (av, am) = first argmax.
// H = ln s - u / s.  Merging is exact up to rounding; see k_entropy.cu for the algebra.
#pragma once
#include <cuda_runtime.h>
#include <math.h>

namespace dg {

struct EntState {
  float m, s, u, av;
  int am;

  __device__ __forceinline__ void init() {
    m = -INFINITY; s = 0.f; u = 0.f; av = -INFINITY; am = 0x7fffffff;
  }
  // Add one logit z with vocabulary index i (indices of one state arrive in increasing order).
  __device__ __forceinline__ void add(float z, int i) {
    if (z > av) { av = z; am = i; }
    if (z > m) {
      if (s > 0.f) {
        const float c = expf(m - z);
        u = c * (u + s * (m - z));
        s = s * c + 1.f;
      } else {
        s = 1.f; u = 0.f;
      }
      m = z;
    } else {
      const float e = expf(z - m);
      s += e;
      u = fmaf(e, z - m, u);
    }
  }
  // Sampler variants: the softmax state takes the scaled logit v, the argmax the key (v plus a
  // Gumbel draw); indices of one state arrive in increasing order.
  __device__ __forceinline__ void add_keyed(float v, float key, int i) {
    const float av0 = av;
    const int am0 = am;
    add(v, i);
    av = av0;
    am = am0;
    if (key > av) { av = key; am = i; }
  }
  __device__ __forceinline__ void merge(const EntState &o) {
    if (o.av > av || (o.av == av && o.am < am)) { av = o.av; am = o.am; }
    if (o.s <= 0.f) return;
    if (s <= 0.f) { m = o.m; s = o.s; u = o.u; return; }
    const float mn = fmaxf(m, o.m);
    const float c1 = expf(m - mn), c2 = expf(o.m - mn);
    u = c1 * (u + s * (m - mn)) + c2 * (o.u + o.s * (o.m - mn));
    s = s * c1 + o.s * c2;
    m = mn;
  }
  __device__ __forceinline__ EntState warp_reduce() const {
    EntState t = *this;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      EntState x;
      x.m = __shfl_xor_sync(0xffffffffu, t.m, o);
      x.s = __shfl_xor_sync(0xffffffffu, t.s, o);
      x.u = __shfl_xor_sync(0xffffffffu, t.u, o);
      x.av = __shfl_xor_sync(0xffffffffu, t.av, o);
      x.am = __shfl_xor_sync(0xffffffffu, t.am, o);
      t.merge(x);
    }
    return t;
  }
  __device__ __forceinline__ float entropy() const { return logf(s) - u / s; }
};

}  // namespace dg
