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
// and independent of summation order.
//
// When the smallest entropy alone exceeds gamma exactly one position commits (rank 1 would need
// Q(H_(0)) <= Q(gamma), and later prefixes only grow), so a block minimum of the keys decides it.
// Otherwise the block sorts the keys (bitonic network: compare-exchange partners closer than a
// warp by shuffles, farther ones through shared memory), so thread r holds the rank-r key; an exclusive
// block scan of Q over the ranks gives each rank its prefix sum, and the committing ranks write
// their positions.  At step index >= max_steps - 1 every masked position is committed (the canvas
// always finishes within max_steps).  With `revise` (the noise canvas's revisable drafts) every
// masked position that does not commit takes argmax as its new draft token.
#include "dg_common.cuh"
#include "dg_kernels.h"

namespace dg {

namespace {

template <int N>
__global__ void __launch_bounds__(N) eb_kernel(int C, const float *__restrict__ H,
                                               const int32_t *__restrict__ am, long long qg,
                                               int max_steps, int32_t *tokens, uint8_t *masked,
                                               uint8_t *selected, int32_t *n_masked,
                                               int32_t *done, int32_t *step, int32_t *st,
                                               int revise) {
  pdl_wait();
  pdl_trigger();
  __shared__ unsigned long long sk[N];
  __shared__ long long wsum[N / 32];
  const int b = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t base = (size_t)b * C;
  // every input of this canvas is loaded at once (one round trip), then the done flag decides
  const int is_done = done[b], stp = step[b];
  const bool mine = tid < C && masked[base + tid];
  const float h_in = tid < C ? H[base + tid] : 0.f;
  const int32_t am_in = tid < C ? am[base + tid] : 0;
  if (is_done) return;  // uniform in the block
  unsigned long long key = ~0ull;  // positions that are not candidates sort last
  bool bad = false;
  if (mine) {
    float h = h_in;
    bad = !isfinite(h);
    h = (h > 0.f) ? h : 0.f;  // negative rounding residue and -0 count as +0
    key = ((unsigned long long)__float_as_uint(h) << 32) | (unsigned)tid;
  }
  if (__syncthreads_or(bad)) {
    if (tid == 0) set_status(st, DG_ERR_NUMERIC);
    return;
  }
  const int n_valid = __syncthreads_count(mine);
  const bool force = stp >= max_steps - 1;
  // Rank 1 commits iff Q(H_(0)) <= Q(gamma), and the prefix sums only grow, so when the smallest
  // entropy alone exceeds the bound exactly one position (the smallest key) commits: a block
  // minimum replaces the sort.
  unsigned long long kmin = key;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long v = __shfl_xor_sync(0xffffffffu, kmin, o);
    kmin = v < kmin ? v : kmin;
  }
  if (lane == 0) sk[warp] = kmin;
  __syncthreads();
  kmin = sk[0];
  for (int w = 1; w < N / 32; ++w) kmin = sk[w] < kmin ? sk[w] : kmin;
  const long long q_min =
      n_valid > 0 ? __double2ll_rn((double)__uint_as_float((uint32_t)(kmin >> 32)) * 4294967296.0)
                  : 0;
  if (!force && n_valid > 0 && q_min > qg) {
    if (tid < C) {
      const bool commit = key == kmin;  // keys are distinct: the one smallest candidate
      if (commit) {
        tokens[base + tid] = am_in;
        masked[base + tid] = 0;
      } else if (revise && mine) {
        tokens[base + tid] = am_in;  // the draft takes this step's prediction
      }
      if (selected) selected[base + tid] = commit ? 1 : 0;
    }
    if (tid == 0) {
      n_masked[b] = n_valid - 1;
      step[b] = stp + 1;
      done[b] = (n_valid - 1 == 0);
    }
    return;
  }
  __syncthreads();  // sk is reused by the sort
  // bitonic sort, ascending over the block
#pragma unroll 1
  for (int k = 2; k <= N; k <<= 1) {
#pragma unroll 1
    for (int j = k >> 1; j > 0; j >>= 1) {
      unsigned long long other;
      if (j >= 32) {
        sk[tid] = key;
        __syncthreads();
        other = sk[tid ^ j];
        __syncthreads();
      } else {
        other = __shfl_xor_sync(0xffffffffu, key, j);
      }
      const bool keep_min = ((tid & k) == 0) == ((tid & j) == 0);
      key = keep_min ? (key < other ? key : other) : (key < other ? other : key);
    }
  }
  // rank tid's fixed-point entropy and the exclusive prefix sum over the ranks before it
  long long q = 0;
  if (tid < n_valid) q = __double2ll_rn((double)__uint_as_float((uint32_t)(key >> 32)) * 4294967296.0);
  long long incl = q;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    long long t = lane < N / 32 ? wsum[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long v = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += v;
    }
    __syncwarp();
    if (lane < N / 32) wsum[lane] = t;  // inclusive warp totals
  }
  __syncthreads();
  const long long excl = incl - q + (warp > 0 ? wsum[warp - 1] : 0);
  const bool commit = tid < n_valid && (force || tid == 0 || excl <= qg);
  if (selected && tid < C) selected[base + tid] = 0;
  __syncthreads();  // the clears land before the committed positions are marked
  if (tid < n_valid) {
    const int pos = (int)(key & 0xffffffffu);
    if (commit) {
      tokens[base + pos] = am[base + pos];
      masked[base + pos] = 0;
      if (selected) selected[base + pos] = 1;
    } else if (revise) {
      tokens[base + pos] = am[base + pos];  // the draft takes this step's prediction
    }
  }
  const int n_commit = __syncthreads_count(commit);
  if (tid == 0) {
    const int left = n_valid - n_commit;
    n_masked[b] = left;
    step[b] = stp + 1;
    done[b] = (left == 0);
  }
}

}  // namespace

int launch_eb_select(int batch, int canvas, const float *entropy, const int32_t *argmax,
                     long long q_gamma, int max_steps, int32_t *tokens, uint8_t *masked,
                     uint8_t *selected, int32_t *n_masked, int32_t *done, int32_t *step,
                     int32_t *st, cudaStream_t s, int revise) {
  if (batch <= 0) return DG_OK;
  if (canvas > 1024) return DG_ERR_UNSUPPORTED;
  int N = 32;
  while (N < canvas) N <<= 1;
  void (*k)(int, const float *, const int32_t *, long long, int, int32_t *, uint8_t *, uint8_t *,
            int32_t *, int32_t *, int32_t *, int32_t *, int) =
      N == 32 ? eb_kernel<32> : N == 64 ? eb_kernel<64> : N == 128 ? eb_kernel<128>
      : N == 256 ? eb_kernel<256> : N == 512 ? eb_kernel<512> : eb_kernel<1024>;
  note_launch(s, "eb_select");
  launch_pdl(k, batch, N, 0, s, canvas, entropy, argmax, q_gamma, max_steps, tokens, masked,
             selected, n_masked, done, step, st, revise);
  return check_launch("eb_select");
}

}  // namespace dg
