// kvb_selftest_timeout: the device-side failure detection of the tcgen05
// kernels, exercised without a fault.
//
// Every mbarrier wait of the Gram and attention kernels goes through mbar_wait
// (sm100.cuh): bounded by %globaltimer, it latches KVB_E_DEVICE_TIMEOUT into the
// status word and raises the CTA's abort flag, and every other role of the CTA
// gives up its own wait as soon as it sees that flag.  This kernel runs the same
// function on two mbarriers that nothing ever arrives on (their phase 0 never
// completes): one role with the caller's limit, the other with a limit 50 times
// longer, so that it can only return early through the abort flag.  Nothing
// hangs: both waits end within their limits whatever happens.
#include "host_util.h"
#include "kvb_device.cuh"
#include "sm100.cuh"

using namespace kvb;
using namespace kvb::sm100;

namespace {

constexpr long long kMinTimeoutNs = 1000;            // 1 us
constexpr long long kMaxTimeoutNs = 100000000LL;     // 100 ms (role 1 then waits at most 5 s)

__global__ void __launch_bounds__(64) selftest_timeout_kernel(int* status, long long* out,
                                                              unsigned long long timeout_ns) {
  __shared__ __align__(8) uint64_t bar[2];
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const int role = threadIdx.x >> 5;
  if ((threadIdx.x & 31) == 0) {  // one lane per role, as the producer and MMA roles wait
    const uint64_t t0 = globaltimer();
    const bool completed = mbar_wait(&bar[role], 0, &abort_flag, status, role == 0 ? timeout_ns : 50 * timeout_ns);
    out[2 * role] = completed ? 1 : 0;
    out[2 * role + 1] = static_cast<long long>(globaltimer() - t0);
  }
}

}  // namespace

extern "C" kvb_status kvb_selftest_timeout(int32_t* status, int64_t* out, int64_t timeout_ns, void* stream) {
  if (!status || !out || timeout_ns < kMinTimeoutNs || timeout_ns > kMaxTimeoutNs) return KVB_E_INVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  LaunchTrace trace("selftest_timeout_kernel", st);
  selftest_timeout_kernel<<<1, 64, 0, st>>>(status, reinterpret_cast<long long*>(out),
                                             static_cast<unsigned long long>(timeout_ns));
  return cuda_status(cudaGetLastError());
}
