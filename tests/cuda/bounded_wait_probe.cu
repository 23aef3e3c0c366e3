// Test-only kernel: one warp waits on an mbarrier phase that nothing ever
// completes, through the library's bounded wait. The wait must give up after
// `limit_ns` and the kernel must report the timeout and return normally.
#include "ptx.cuh"

__global__ void bounded_wait_probe(int* status, unsigned long long limit_ns, unsigned long long* waited_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    twell::mbar_init(&bar, 1);
    abort_flag = 0;
    twell::fence_mbar_init();
  }
  __syncthreads();
  const uint64_t t0 = twell::global_timer_ns();
  const bool ok = twell::mbar_wait(&bar, 0, &abort_flag, limit_ns);  // no arrival ever comes
  if (threadIdx.x == 0) {
    *waited_ns = twell::global_timer_ns() - t0;
    if (!ok) twell::raise_status(status, twell::kDevTimeout);
  }
}

extern "C" int launch_bounded_wait_probe(int* status, unsigned long long limit_ns, unsigned long long* waited_ns) {
  bounded_wait_probe<<<1, 32>>>(status, limit_ns, waited_ns);
  return static_cast<int>(cudaGetLastError());
}
