// Small kernels of the sampler variants: the uniform-noise canvas, and the row slots of the
// autoregressive step's LM head.
//
// "DiffusionGemma Technical Report", explanatory visual and Figure 3: a canvas starts as uniform
// noise over the vocabulary.  Reading: position i of canvas b holds (w0 * V) >> 32, w0 the first
// word of Philox4x32-10 at counter (i, 0, 0, (TAG_NOISE << 24) | b) keyed by the seed; every
// position starts not final (its token is a revisable draft).
#include "dg_common.cuh"
#include "dg_kernels.h"
#include "sampler.cuh"

namespace dg {

namespace {

__global__ void noise_canvas_kernel(int canvas, int vocab, uint32_t k0, uint32_t k1,
                                    int32_t *tokens, uint8_t *masked, int32_t *n_masked,
                                    int32_t *done, int32_t *step) {
  pdl_wait();
  pdl_trigger();
  const int b = blockIdx.y;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < canvas) {
    const uint4 w = philox4x32_10(
        make_uint4((uint32_t)i, 0u, 0u, ((uint32_t)SAMPLE_TAG_NOISE << 24) | (uint32_t)b), k0, k1);
    const size_t o = (size_t)b * canvas + i;
    tokens[o] = (int32_t)(((uint64_t)w.x * (uint64_t)vocab) >> 32);
    masked[o] = 1;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    n_masked[b] = canvas;
    done[b] = 0;
    step[b] = 0;
  }
}

__global__ void last_row_slots_kernel(int total, int n, int32_t *slot) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t < total) slot[t] = (t % n == n - 1) ? t / n : -1;
}

}  // namespace

int launch_noise_canvas(int batch, int canvas, int vocab, uint32_t key0, uint32_t key1,
                        int32_t *tokens, uint8_t *masked, int32_t *n_masked, int32_t *done,
                        int32_t *step, cudaStream_t s) {
  if (batch <= 0 || canvas <= 0) return DG_OK;
  note_launch(s, "noise_canvas");
  launch_pdl(noise_canvas_kernel, dim3((canvas + 255) / 256, batch), 256, 0, s, canvas, vocab,
             key0, key1, tokens, masked, n_masked, done, step);
  return check_launch("noise_canvas");
}

int launch_last_row_slots(int batch, int n, int32_t *slot, cudaStream_t s) {
  const int total = batch * n;
  if (total <= 0) return DG_OK;
  note_launch(s, "last_row_slots");
  launch_pdl(last_row_slots_kernel, (total + 255) / 256, 256, 0, s, total, n, slot);
  return check_launch("last_row_slots");
}

}  // namespace dg
