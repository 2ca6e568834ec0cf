// aqua_selftest_wait_timeout: exercises the bounded device wait every kernel
// of the library uses, on a barrier that nothing ever completes, so that the
// time-out path (error status recorded on the device, kernel returns, context
// stays usable) can be checked on a GPU without faulting or hanging it.  The
// pages have no counterpart; it is a diagnostic of this implementation.
#include "aqua_internal.cuh"

namespace aqua {
namespace {

__global__ void wait_timeout_kernel(int32_t* ctrl, unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);   // one expected arrival, which never comes
    fence_barrier_init();
  }
  __syncthreads();
  const bool ok = mbar_wait_bounded(&bar, 0, limit_ns);
  if (__syncthreads_or(!ok) && threadIdx.x == 0) record_status(ctrl, AQUA_ERR_TIMEOUT);
}

}  // namespace
}  // namespace aqua

extern "C" int aqua_selftest_wait_timeout(aqua_cache* cache, unsigned long long limit_ns, aqua_stream_t stream) {
  using aqua::set_error;
  if (cache == nullptr || cache->ctrl == nullptr)
    return set_error(AQUA_ERR_ARG, "aqua_selftest_wait_timeout: cache with a ctrl block required");
  if (limit_ns < 1000ull || limit_ns > 2000000000ull)
    return set_error(AQUA_ERR_ARG, "aqua_selftest_wait_timeout: limit %llu ns outside [1 us, 2 s]", limit_ns);
  aqua::wait_timeout_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(cache->ctrl, limit_ns);
  return aqua::check_launch("wait_timeout_kernel");
}
