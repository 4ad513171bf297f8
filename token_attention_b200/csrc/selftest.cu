// selftest.cu -- a kernel whose wait can never complete, to check on a GPU that
// the library's failure reporting works: the wait gives up after a short limit,
// the kernel records MTA_ERR_TIMEOUT in the caller's workspace and ends, and
// the context stays usable.  Nothing faults and nothing waits without a bound.
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"

namespace mta {
namespace {

constexpr int kSelftestThreads = 128;

// Every thread waits on phase 0 of an mbarrier that expects one arrival which
// never comes (the same bounded wait the attention kernels use, with the limit
// given).  The first thread to give up sets the abort flag and the error bit;
// the others then return at once, and a second wait after the abort returns
// immediately, as the kernels' later waits do.  out[0] counts the threads whose
// wait returned false, out[1] those whose second wait did.
__global__ void __launch_bounds__(kSelftestThreads) wait_timeout_kernel(unsigned long long limit_ns,
                                                                        unsigned *err, unsigned *out) {
  __shared__ uint64_t bar[2];
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int *ab = &abort_flag;
  const bool first = mbar_wait_for(&bar[0], 0, ab, err, limit_ns);
  const bool second = mbar_wait_for(&bar[1], 0, ab, err, limit_ns);
  if (!first) atomicAdd(out, 1u);
  if (!second) atomicAdd(out + 1, 1u);
}

}  // namespace

cudaError_t launch_wait_timeout_selftest(unsigned long long limit_ns, unsigned *err, unsigned *out,
                                         cudaStream_t stream) {
  wait_timeout_kernel<<<1, kSelftestThreads, 0, stream>>>(limit_ns, err, out);
  return cudaGetLastError();
}

}  // namespace mta
