// Self-test of the bounded device-side wait that every kernel of the library
// uses on its mbarriers: a wait on a phase that never completes gives up
// after its cycle limit, ORs MLA_DEVFLAG_TIMEOUT into the device flags and
// returns, so the kernel ends and the context stays usable.  No TMA copy or
// tensor-core operation is in flight in this kernel, so nothing is left
// behind when the wait gives up.
#include "internal.h"
#include "sm100_ptx.cuh"

namespace mla {
namespace {

constexpr uint64_t kSelfTestLimitCycles = 2ull * 1000ull * 1000ull;  // about a millisecond

__global__ void wait_selftest_kernel(int* err, int arrive) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  const uint32_t b = ptx::smem_u32(&bar);
  ptx::mbar_init(b, 1);
  ptx::fence_mbar_init();
  // with an arrival the phase completes and the wait returns at once;
  // without one nothing completes it and the wait gives up
  if (arrive) ptx::mbar_arrive(b);
  ptx::mbar_wait(b, 0, err, MLA_DEVFLAG_TIMEOUT, kSelfTestLimitCycles);
}

}  // namespace

cudaError_t launch_wait_selftest(int* err, bool arrive, cudaStream_t s) {
  wait_selftest_kernel<<<1, 32, 0, s>>>(err, arrive ? 1 : 0);
  return cudaGetLastError();
}

}  // namespace mla
