// Self-check of the bounded-wait path that every waiting kernel of the library
// uses: one warp waits on an mbarrier phase that nothing will ever complete,
// with a short wait limit.  When the limit passes the wait gives up, the kernel
// raises the timeout bit of the device status word and returns, so the caller
// sees SDL_ERR_TIMEOUT from sdl_last_device_status and the context stays
// usable.  Nothing faults, traps or hangs.
#include "internal.cuh"
#include "ptx.cuh"

namespace sdl {
namespace {

__global__ void wait_check_kernel(uint64_t limit_ns, int* status) {
  __shared__ uint64_t bar;
  __shared__ volatile int abort_sh;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
    abort_sh = 0;
  }
  __syncthreads();
  // phase 0 needs one arrival, and none comes
  const bool ok = mbar_wait(&bar, 0, &abort_sh, nullptr, limit_ns);
  if (!ok && threadIdx.x == 0) atomicOr(status, kDevTimeout);
}

}  // namespace

cudaError_t launch_wait_check(uint64_t limit_ns, int* status, cudaStream_t st) {
  wait_check_kernel<<<1, 32, 0, st>>>(limit_ns, status);
  return cudaGetLastError();
}

}  // namespace sdl
