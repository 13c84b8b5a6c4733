// Bounded device waits: the per-workspace wait limit and a self-test of the
// timeout path.
//
// Every mbarrier wait in the tensor-core kernels gives up after the limit held in
// the workspace header (2 s unless hsa_set_wait_limit changed it), records
// HSA_ERR_TIMEOUT in the status word and lets the kernel drain and exit, so a wait
// that can never complete costs a bounded time and leaves the context usable.
// wait_selftest_kernel exercises exactly that path in isolation: one thread waits on
// an mbarrier that nothing arrives at, with no copy or MMA in flight behind it.
#include "common.cuh"
#include "kernels.h"
#include "sm100.cuh"

namespace hsa {
namespace {

constexpr int kSelftestSite = 0x7E << 24;

__global__ void set_wait_limit_kernel(int* header, uint32_t limit_us) {
  uint32_t* w = reinterpret_cast<uint32_t*>(header);
  w[3] = limit_us;
  w[2] = limit_us ? kWaitTag : 0u;
}

__global__ void wait_selftest_kernel(int* status, unsigned long long* waited_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  sm100::mbar_init(&bar, 1);
  sm100::fence_barrier_init();
  const uint64_t t0 = sm100::global_ns();
  // phase 0 never completes: nothing arrives on the barrier.  The wait's site is
  // kSelftestSite, so that the header's record of it can be checked.
  const bool ok = sm100::mbar_wait(&bar, 0, status, wait_limit_ns(status), kSelftestSite);
  if (waited_ns) *waited_ns = sm100::global_ns() - t0;
  if (ok) set_status(status, HSA_ERR_DEVICE);  // cannot happen: the phase has no arrivals
}

}  // namespace

cudaError_t launch_set_wait_limit(int* header, uint32_t limit_us, cudaStream_t s) {
  set_wait_limit_kernel<<<1, 1, 0, s>>>(header, limit_us);
  return cudaGetLastError();
}

cudaError_t launch_wait_selftest(int* status, unsigned long long* waited_ns, cudaStream_t s) {
  wait_selftest_kernel<<<1, 32, 0, s>>>(status, waited_ns);
  return cudaGetLastError();
}

}  // namespace hsa
