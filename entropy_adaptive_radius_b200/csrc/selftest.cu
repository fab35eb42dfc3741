// Self-test of the bounded waits: a kernel waits, through the same helper
// every kernel of the library uses, on an mbarrier that nothing ever
// completes.  The wait must give up after its limit, record kErrSelfTest in
// the device error word and let the kernel return normally, so the context
// stays usable and tra_get_device_error reports TRA_ERR_TIMEOUT.  No fault,
// trap or unbounded wait is involved.
#include "ptx.cuh"
#include "tra_internal.h"

namespace tra {
namespace {

__global__ void selftest_wait_kernel(int* err, unsigned long long limit_ns, int* completed) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);  // expects one arrival, which never comes
  fence_barrier_init();
  abort_flag = 0;
  const bool done = mbar_wait(b, 0, &abort_flag, err, kErrSelfTest, limit_ns);
  if (completed != nullptr) *completed = done ? 1 : 0;
}

}  // namespace

cudaError_t launch_selftest_wait(unsigned long long limit_ns, int* completed, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(device_error_word(), limit_ns, completed);
  return cudaGetLastError();
}

}  // namespace tra
