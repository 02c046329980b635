// Self-test of the bounded mbarrier wait that every tensor-core kernel in
// this library uses (sm100_primitives.cuh: mbar_wait).  A one-warp kernel
// waits on an mbarrier that nothing ever arrives on; the wait must give up
// after the requested limit and report it, leaving the context usable.  This
// is how the library's failure detection is exercised on a GPU without
// faulting, trapping or hanging it.

#include "sm100_primitives.cuh"
#include "svt_internal.h"

namespace {

using namespace svt::sm100;

__device__ unsigned g_wait_result;   // 0: not run, 1: phase completed, 2: gave up

__global__ void wait_limit_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  const uint32_t b = smem_addr(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    fence_barrier_init();
  }
  __syncthreads();
  const bool completed = mbar_wait(b, 0, nullptr, limit_ns);   // nothing arrives
  if (threadIdx.x == 0) g_wait_result = completed ? 1u : 2u;
}

}  // namespace

extern "C" SVT_API int svt_selftest_wait_limit(int limit_us, svt_stream_t stream) {
  if (limit_us < 1 || limit_us > 10000000)
    return svt::report_error(SVT_EINVAL, "limit_us must be in [1, 10^7]");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const unsigned zero = 0;
  unsigned result = 0;
  cudaError_t e = cudaMemcpyToSymbolAsync(g_wait_result, &zero, sizeof(zero), 0,
                                          cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) {
    wait_limit_kernel<<<1, 32, 0, s>>>((uint64_t)limit_us * 1000ull);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess)
    e = cudaMemcpyFromSymbolAsync(&result, g_wait_result, sizeof(result), 0,
                                  cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return svt::report_error(SVT_ECUDA, cudaGetErrorString(e));
  if (result == 2)
    return svt::report_error(SVT_EDEVICE, "bounded mbarrier wait gave up at its limit");
  if (result == 1) return svt::report_error(SVT_ECUDA, "a barrier nobody arrived on completed");
  return svt::report_error(SVT_ECUDA, "self-test kernel did not run");
}
