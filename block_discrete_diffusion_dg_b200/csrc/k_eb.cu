// Entropy-bounded (EB) selection and commit, one block per canvas.
//
// The pages name the sampler (model card "diffusiongemma", Benchmark Results: the recommended
// Entropy Bound sampler; "DiffusionGemma Technical Report", What they did: entropy-bounded
// sampler with adaptive stopping) but print no rule.  The rule is the published EB sampler
// (Ben-Hamu et al., 2025): take masked positions in ascending entropy and commit the longest
// prefix whose entropy sum minus its largest entropy stays within gamma; at least one position
// per step.  With entropies sorted, that is: commit rank r iff r == 0 or sum_{i<r} H_(i) <= gamma.
//
// Bit-exactness: keys are (fp32 bits of max(H, 0), position) — order-preserving for H >= 0 and
// lower position first on ties, so all keys are distinct; sums run in int64 fixed point with 32
// fraction bits (Q(H) = nearest integer to H * 2^32, exact in fp64), so the prefix test is exact
// and independent of summation order.  The sum over the ranks before r in sorted order is the
// sum of Q over the keys smaller than the rank-r key, which each thread forms directly by one pass
// over the keys in shared memory (every thread reads the same key at a time: a broadcast), so no
// sort is needed.  At step index >= max_steps - 1 every masked position is committed (the canvas
// always finishes within max_steps).
#include "dg_common.cuh"
#include "dg_kernels.h"

namespace dg {

namespace {

__global__ void __launch_bounds__(1024) eb_kernel(int C, const float *__restrict__ H,
                                                  const int32_t *__restrict__ am, long long qg,
                                                  int max_steps, int32_t *tokens, uint8_t *masked,
                                                  uint8_t *selected, int32_t *n_masked,
                                                  int32_t *done, int32_t *step, int32_t *st,
                                                  int revise) {
  pdl_wait();
  pdl_trigger();
  __shared__ unsigned long long keys[1024];
  __shared__ long long qv[1024];
  __shared__ int bad, n_valid, n_commit;
  const int b = blockIdx.x, tid = threadIdx.x;
  if (done[b]) return;
  if (tid == 0) { bad = 0; n_valid = 0; n_commit = 0; }
  __syncthreads();
  const size_t base = (size_t)b * C;
  unsigned long long key = ~0ull;
  long long q = 0;
  const bool mine = tid < C && masked[base + tid];
  if (mine) {
    float h = H[base + tid];
    if (!isfinite(h)) atomicOr(&bad, 1);
    h = (h > 0.f) ? h : 0.f;  // negative rounding residue and -0 count as +0
    key = ((unsigned long long)__float_as_uint(h) << 32) | (unsigned)tid;
    q = __double2ll_rn((double)h * 4294967296.0);
    atomicAdd(&n_valid, 1);
  }
  if (tid < C) {
    keys[tid] = key;
    qv[tid] = q;
  }
  __syncthreads();
  if (bad) {
    if (tid == 0) set_status(st, DG_ERR_NUMERIC);
    return;
  }
  if (tid < C) {
    bool commit = false;
    if (mine) {
      int rank = 0;
      long long excl = 0;  // sum of Q over the smaller keys = the exclusive prefix in sorted order
      for (int j = 0; j < C; ++j) {
        const unsigned long long kj = keys[j];
        if (kj < key) {
          ++rank;
          excl += qv[j];
        }
      }
      commit = step[b] >= max_steps - 1 || rank == 0 || excl <= qg;
      if (commit) {
        tokens[base + tid] = am[base + tid];
        masked[base + tid] = 0;
        atomicAdd(&n_commit, 1);
      } else if (revise) {
        tokens[base + tid] = am[base + tid];  // the draft takes this step's prediction
      }
    }
    if (selected) selected[base + tid] = commit ? 1 : 0;
  }
  __syncthreads();
  if (tid == 0) {
    const int left = n_valid - n_commit;
    n_masked[b] = left;
    step[b] = step[b] + 1;
    done[b] = (left == 0);
  }
}

}  // namespace

int launch_eb_select(int batch, int canvas, const float *entropy, const int32_t *argmax,
                     long long q_gamma, int max_steps, int32_t *tokens, uint8_t *masked,
                     uint8_t *selected, int32_t *n_masked, int32_t *done, int32_t *step,
                     int32_t *st, cudaStream_t s, int revise) {
  if (batch <= 0) return DG_OK;
  int N = 32;
  while (N < canvas) N <<= 1;
  note_launch(s, "eb_select");
  launch_pdl(eb_kernel, batch, N, 0, s, canvas, entropy, argmax, q_gamma, max_steps, tokens, masked,
                                selected, n_masked, done, step, st, revise);
  return check_launch("eb_select");
}

}  // namespace dg
