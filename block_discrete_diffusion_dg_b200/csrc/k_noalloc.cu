// dg_logits_entropy_static: the final-norm + LM-head + entropy/argmax operation of
// dg_logits_entropy, for callers that cannot hand the library a scratch buffer.
//
// Who needs it: code that runs where device allocation is not available to it — for example a
// serving engine that reserves all device memory for its own pools at start-up (a later
// cudaMalloc fails or fragments the pool), or a plugin whose host application owns every device
// allocation and only lends it the model's tensors.  Such a caller still owns its inputs and
// outputs; the scratch this operation needs lives in a fixed array in the library's device image.
//
// The array is a file-scope __device__ object of DG_STATIC_SCRATCH_BYTES bytes; every GPU that
// loads the library holds it until the process exits.  Its device address belongs to a CUDA
// context (the module is loaded once per context), so it is looked up with cudaGetSymbolAddress
// in the caller's current context on every call made outside stream capture, and remembered per
// context for calls made while the caller's stream is being captured.
#include <cudaTypedefs.h>

#include <mutex>
#include <utility>
#include <vector>

#include "dg_common.cuh"
#include "dg_kernels.h"

namespace dg {
namespace {

constexpr int MAX_ROWS = 256;       // rows per call
constexpr int MAX_D = 2048;         // d_model
constexpr int MAX_VOCAB = 262144;   // vocabulary
constexpr size_t NORM_BYTES = (size_t)MAX_ROWS * MAX_D * 2;   // normalised rows (bf16)

__device__ __align__(256) uint8_t g_static_scratch[DG_STATIC_SCRATCH_BYTES];

std::mutex g_mu;
std::vector<std::pair<CUcontext, void *>> g_scratch_addr;   // per context, most recent lookup
PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
std::once_flag g_ctx_once;

void load_ctx_current() {
  void *fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
}

// Device address of the array in the calling thread's current context.  Outside stream capture it
// is looked up afresh (a context destroyed and re-created, e.g. after cudaDeviceReset, gets the
// new module's address; the lookup also initialises the device's primary context if no context is
// current yet); while `s` is being captured the address remembered for the context is used, so a
// first call on a context must come before any capture there.
int scratch_address(cudaStream_t s, void **out) {
  std::call_once(g_ctx_once, load_ctx_current);
  if (!g_ctx_current) return DG_ERR_CUDA;
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(s, &cs) != cudaSuccess)
    return check_launch("dg_logits_entropy_static: capture status");
  void *p = nullptr;
  if (cs == cudaStreamCaptureStatusNone) {
    const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return check_launch("dg_logits_entropy_static: cudaGetSymbolAddress");
    if (!p) return DG_ERR_CUDA;
  }
  CUcontext ctx = nullptr;
  if (g_ctx_current(&ctx) != CUDA_SUCCESS || !ctx) return DG_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  auto it = g_scratch_addr.begin();
  for (; it != g_scratch_addr.end(); ++it)
    if (it->first == ctx) break;
  if (cs != cudaStreamCaptureStatusNone) {
    if (it == g_scratch_addr.end()) return DG_ERR_CUDA;   // first call inside a capture
    *out = it->second;
    return DG_OK;
  }
  if (it == g_scratch_addr.end())
    g_scratch_addr.emplace_back(ctx, p);
  else
    it->second = p;
  *out = p;
  return DG_OK;
}

}  // namespace
}  // namespace dg

using namespace dg;

extern "C" int dg_logits_entropy_static(const dg_config *cfg, int n_rows,
                                        const int32_t *n_rows_dev, const void *h,
                                        const int32_t *row_idx, const void *w_lm,
                                        float *entropy, int32_t *argmax, int32_t *dev_status,
                                        void *stream) {
  if (!cfg_ok(cfg) || n_rows <= 0 || !h || !w_lm || !entropy || !argmax)
    return DG_ERR_INVALID_ARG;
  if (!lmhead_tc_supported(cfg->act_dtype, cfg->d_model)) return DG_ERR_UNSUPPORTED;
  if (cfg->emb_dtype != cfg->act_dtype) return DG_ERR_UNSUPPORTED;  // NVFP4: not here
  // requests larger than the fixed array: rejected, nothing launched
  if (n_rows > MAX_ROWS || cfg->d_model > MAX_D || cfg->vocab > MAX_VOCAB)
    return DG_ERR_WORKSPACE;
  const int rows128 = (n_rows + 127) / 128 * 128;
  if ((size_t)rows128 * cfg->d_model * 2 > NORM_BYTES ||
      NORM_BYTES + lmhead_tc_ws_bytes(n_rows, cfg->vocab) > (size_t)DG_STATIC_SCRATCH_BYTES)
    return DG_ERR_WORKSPACE;
  const cudaStream_t s = (cudaStream_t)stream;
  void *scratch = nullptr;
  const int rc = scratch_address(s, &scratch);
  if (rc != DG_OK) return rc;
  char *norm_rows = static_cast<char *>(scratch);
  char *partials = norm_rows + NORM_BYTES;
  const int r1 = launch_rmsnorm(cfg->act_dtype, h, row_idx, n_rows_dev, n_rows, cfg->d_model,
                                cfg->rms_eps, norm_rows, s);
  if (r1 != DG_OK) return r1;
  return launch_lmhead_tc(norm_rows, n_rows, n_rows_dev, w_lm, cfg->vocab, cfg->d_model, row_idx,
                          entropy, argmax, nullptr, nullptr, partials, dev_status, s);
}
