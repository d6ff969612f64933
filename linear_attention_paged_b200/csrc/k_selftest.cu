// k_selftest.cu -- failure detection of the bounded waits, exercised without a
// fault: one CTA waits on an mbarrier that no thread ever arrives at, through the
// same bounded wait the tcgen05 kernels use.  The wait has to give up after the
// given limit, record WA_DEVERR_TIMEOUT in the device error word and return, so
// that the context stays usable.  Nothing else is in flight in this kernel (no TMA
// load, no MMA, no TMEM), so giving up leaves nothing behind.
#include <atomic>

#include "sm100.cuh"
#include "wa_internal.h"

namespace wa {

namespace {
std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};

using namespace sm100;

__global__ void __launch_bounds__(32)
k_wait_nobody(uint64_t limit_ns, uint64_t* elapsed_ns, uint32_t* err) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);   // expects one arrival; none will come
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncwarp();
  if (threadIdx.x != 0) return;
  const uint64_t t0 = globaltimer_ns();
  const int r = mbar_wait_bounded(&bar, 0, &abort_flag, limit_ns);
  const uint64_t t1 = globaltimer_ns();
  if (r == kWaitTimeout) atomicOr(err, WA_DEVERR_TIMEOUT);
  if (elapsed_ns) *elapsed_ns = t1 - t0;
}
}  // namespace

uint64_t wait_limit_ns() { return g_wait_limit_ns.load(std::memory_order_relaxed); }

}  // namespace wa

using namespace wa;

extern "C" {

wa_status wa_set_wait_limit_ns(uint64_t limit_ns) {
  if (limit_ns < 1000ull || limit_ns > 60000000000ull)
    return set_error(WA_ERR_INVALID_ARG, "wait limit must be in [1e3, 6e10] ns (got %llu)",
                     static_cast<unsigned long long>(limit_ns));
  g_wait_limit_ns.store(limit_ns, std::memory_order_relaxed);
  return WA_OK;
}

uint64_t wa_get_wait_limit_ns(void) { return wait_limit_ns(); }

wa_status wa_check_bounded_wait(uint64_t limit_ns, uint64_t* elapsed_ns, void* stream) {
  if (limit_ns < 1000ull || limit_ns > 1000000000ull)
    return set_error(WA_ERR_INVALID_ARG, "limit must be in [1e3, 1e9] ns (got %llu)",
                     static_cast<unsigned long long>(limit_ns));
  uint32_t* err = device_error_word();
  if (!err) return set_error(WA_ERR_CUDA, "no CUDA device");
  k_wait_nobody<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(limit_ns, elapsed_ns, err);
  return check_launch("check_bounded_wait");
}

}  // extern "C"
