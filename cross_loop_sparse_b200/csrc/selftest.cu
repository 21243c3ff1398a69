// flashloop_selftest_bounded_wait: runs the two bounded barrier waits that
// every pipelined kernel of the library relies on against a barrier that
// never completes, and reports the timeout through the error word, as those
// kernels do when a stage they wait for never arrives.  Nothing is loaded or
// copied asynchronously, so a kernel that gives up leaves no transfer in
// flight.
#include "common.cuh"
#include "tc_util.cuh"

namespace fl {

int check_device_arch();

__global__ void __launch_bounds__(32) bounded_wait_selftest_kernel(int kind, int32_t* err) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);  // one arrival expected; none is ever made
  fence_mbar_init();
  const bool done = kind == 0 ? mbar_wait(&bar, 0) : mbar_wait_sleep(&bar, 0);
  if (!done) set_error(err, kDevErrTimeout);
}

}  // namespace fl

extern "C" int flashloop_selftest_bounded_wait(int32_t kind, int32_t* err_word, void* stream) {
  using namespace fl;
  static_assert(kDevErrTimeout == FLASHLOOP_DEVERR_TIMEOUT, "one timeout code");
  if ((kind != 0 && kind != 1) || err_word == nullptr) return FLASHLOOP_ERR_INVALID_ARG;
  const int rc = check_device_arch();
  if (rc != FLASHLOOP_OK) return rc;
  bounded_wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(kind, err_word);
  return launch_status();
}
