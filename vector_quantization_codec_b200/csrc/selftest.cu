// selftest.cu -- a check of the bounded waits that every kernel with a
// bulk-copy ring relies on: one CTA waits on an mbarrier that nothing ever
// arrives on, with the same wait the kernels use, and must come back with
// QAMW_STATUS_TIMEOUT instead of hanging.  Nothing faults and nothing spins
// without a limit.
#include "common.cuh"
#include "launch.cuh"

namespace qamw {
namespace {

__global__ void k_wait_selftest(unsigned tries, int32_t* status, long long* cycles) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // one arrival expected, none will come
    fence_mbar_init();
  }
  __syncthreads();
  const long long t0 = clock64();
  const bool ok = mbar_wait_bounded(&bar, 0u, tries);
  const long long t1 = clock64();
  if (threadIdx.x == 0) {
    if (!ok) raise_flag(status, QAMW_STATUS_TIMEOUT);
    if (cycles) *cycles = t1 - t0;
  }
}

}  // namespace
}  // namespace qamw

using namespace qamw;

extern "C" QAMW_API int qamw_selftest_wait_timeout(unsigned tries, int32_t* d_status,
                                                   long long* d_cycles, void* stream) {
  if (tries == 0 || tries > kSpinLimit || !d_status) return QAMW_ERR_INVALID;
  k_wait_selftest<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(tries, d_status, d_cycles);
  return cudaGetLastError() == cudaSuccess ? QAMW_OK : QAMW_ERR_CUDA;
}
