// Test hook for the bounded-wait path that every mbarrier wait of the tensor-core kernels
// uses: one thread waits on an mbarrier that nothing arrives at, with a short limit, so the
// wait gives up, records its code in the status word and the kernel returns normally.  No
// fault, trap or hang is involved; the context stays usable afterwards.
#include "kernels.h"
#include "tc.cuh"

namespace nsa {

namespace {
__global__ void wait_timeout_kernel(int* __restrict__ err, uint64_t limit_ns, int code) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  tc::mbar_init(&bar, 1);
  tc::fence_barrier_init();
  tc::mbar_wait(&bar, 0, err, code, limit_ns);   // nothing arrives: gives up after limit_ns
}
}  // namespace

cudaError_t launch_wait_timeout(int* err, uint64_t limit_ns, int code, cudaStream_t st) {
  wait_timeout_kernel<<<1, 32, 0, st>>>(err, limit_ns, code);
  return cudaGetLastError();
}

}  // namespace nsa
