// selftest.cu — the give-up path of the library's bounded waits, exercised
// on purpose without a hang or a fault.
//
// Every wait inside the kernels (mbarrier phases of the projection's
// pipeline) polls for at most kWaitLimitClocks SM clocks; a wait that runs
// out records TTQ_DEVERR_TIMEOUT in the sticky error word and its kernel
// winds down. This one-thread kernel runs that same wait on a barrier of
// its own: with `arrive` the phase completes at once, without it nothing
// ever arrives and the wait must give up (about 1.5 s at 1965 MHz).
#include "common.cuh"
#include "kernels.h"

namespace ttq {
namespace {

__global__ void __launch_bounds__(32, 1)
    bounded_wait_kernel(int arrive, uint32_t* out, uint32_t* err) {
  __shared__ __align__(8) uint64_t bar;
  griddep_enter();
  if (threadIdx.x != 0) return;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  fence_barrier_init();
  if (arrive) mbar_arrive(b);
  *out = mbar_wait(b, 0, err) ? 1u : 0u;
}

}  // namespace

ttq_status launch_bounded_wait_check(int arrive, uint32_t* out,
                                     cudaStream_t st) {
  LaunchShape ls;
  ls.grid = dim3(1);
  ls.block = dim3(32);
  return launch(ls, st, bounded_wait_kernel, arrive, out,
                device_error_word());
}

}  // namespace ttq
