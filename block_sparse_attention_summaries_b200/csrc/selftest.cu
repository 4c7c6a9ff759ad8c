// Self-test of the bounded-wait error path: a single thread waits on an mbarrier nothing will
// ever complete, gives up after `polls` tries and records the timeout in the workspace status
// word, exactly as a kernel whose copy never lands would.  No copy is in flight, so the kernel
// ends cleanly and the context stays usable.
#include "bsa_common.cuh"

namespace bsa {
namespace {

__global__ void bounded_wait_kernel(int* status, unsigned polls) {
  __shared__ uint64_t bar;
  mbar_init(&bar, 1);
  fence_mbar_init();
  if (!mbar_wait_bounded(&bar, 0, polls)) report_timeout(status, 99);
}

}  // namespace
}  // namespace bsa

extern "C" bsa_status bsa_selftest_bounded_wait(void* workspace, int polls, void* stream) {
  using namespace bsa;
  BSA_REQUIRE(workspace && polls > 0, BSA_ERR_ARG);
  bounded_wait_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(
      static_cast<int*>(workspace), (unsigned)polls);
  BSA_LAUNCH_CHECK();
  return BSA_OK;
}
