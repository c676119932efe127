// Diagnostic: the bounded device-side wait of the tensor-core kernels, run on its own.
//
// Every wait in the library's tcgen05 kernels is bounded (tc::mbar_wait: WAIT_LIMIT_CYCLES, ~2 s);
// on expiry a kernel records DG_ERR_TIMEOUT in the caller's status word, frees the tensor memory
// it holds and returns instead of hanging.  This probe exercises that path without a fault: one
// CTA allocates TMEM the way those kernels do, then waits (with the same primitive and a caller-
// chosen limit) on an mbarrier phase that completes only if the probe itself arrives on it
// (`arrive` != 0).  Nothing else is in flight: no copy and no MMA is ever issued, so giving up
// leaves nothing outstanding.  On expiry it records DG_ERR_TIMEOUT; either way it frees TMEM and
// returns.
#include "dg_common.cuh"
#include "dg_kernels.h"
#include "tc_common.cuh"

namespace dg {

namespace {

using namespace tc;

constexpr uint32_t PROBE_TMEM_COLS = 32;

__global__ void __launch_bounds__(64, 1) wait_probe_kernel(long long limit, int arrive,
                                                           int32_t *st) {
  pdl_wait();
  pdl_trigger();
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_slot;
  __shared__ int timed_out;
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    timed_out = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, PROBE_TMEM_COLS);
    tmem_relinquish();
  }
  fence_before();
  __syncthreads();
  fence_after();
  if (threadIdx.x == 0) {
    if (arrive) mbar_arrive(&bar);
    if (!mbar_wait_limit(&bar, 0, limit)) {
      timed_out = 1;
      set_status(st, DG_ERR_TIMEOUT);
    }
  }
  fence_before();
  __syncthreads();
  if (warp == 1) {
    fence_after();
    tmem_dealloc(tmem_slot, PROBE_TMEM_COLS);
  }
}

}  // namespace

int launch_wait_probe(long long limit_cycles, int arrive, int32_t *st, cudaStream_t s) {
  note_launch(s, "wait_probe");
  launch_pdl(wait_probe_kernel, 1, 64, 0, s, limit_cycles, arrive, st);
  return check_launch("wait_probe");
}

}  // namespace dg
