// selftest.cu - bsa_selftest_bounded_wait: exercises the timeout path that
// every pipeline wait of the library relies on, without any fault.
//
// One thread initialises an mbarrier that nothing will ever arrive on and
// waits for it with the library's bounded wait.  The wait gives up after
// `limit_cycles` SM clocks, records BSA_DEV_WAIT_TIMEOUT in d_err and the
// kernel returns normally, so the CUDA context stays usable.
#include "common.cuh"

namespace bsa {

__global__ void selftest_wait_kernel(int32_t* d_err, long long limit_cycles) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_mbar_init();
  if (!mbar_wait_bounded(&bar, 0, nullptr, limit_cycles)) report(d_err, BSA_DEV_WAIT_TIMEOUT);
}

}  // namespace bsa

extern "C" bsa_status bsa_selftest_bounded_wait(int32_t* d_err, long long limit_cycles,
                                                void* stream) {
  if (d_err == nullptr || limit_cycles <= 0 || limit_cycles > (1LL << 34))
    return BSA_ERR_INVALID_ARG;
  bsa::selftest_wait_kernel<<<1, 32, 0, bsa::as_stream(stream)>>>(d_err, limit_cycles);
  return bsa::launch_status();
}
