// selftest.cu -- exercises the timeout path of the bounded waits that every kernel of the library uses.
//
// One CTA of one thread waits on an mbarrier phase that nothing completes, with the same wait helper
// (polling or back-off) as the GEMM / GEMV kernels.  After the 2 s limit the helper records a timeout in
// the device status word and returns false; the kernel then returns, no copy or MMA being in flight.
#include "common.cuh"
#include "internal.h"

namespace awq {
namespace {

__global__ void wait_timeout_kernel(unsigned* status, int backoff, uint32_t* returned) {
  __shared__ __align__(8) uint64_t bar;
  mbar_init(&bar, 1);  // one arrival expected; none ever comes
  fence_mbar_init();
  const bool ok = backoff ? mbar_wait_backoff(&bar, 0, status) : mbar_wait(&bar, 0, status);
  *returned = ok ? 2u : 1u;  // 1: the wait gave up and returned
}

}  // namespace
}  // namespace awq

extern "C" awq_status awq_selftest_wait_timeout(int backoff, uint32_t* d_returned, awq_stream_t stream) {
  if (d_returned == nullptr) return AWQ_ERR_INVALID_ARG;
  unsigned* status = awq::device_status_ptr();
  if (status == nullptr) return AWQ_ERR_CUDA;
  awq::wait_timeout_kernel<<<1, 1, 0, reinterpret_cast<cudaStream_t>(stream)>>>(status, backoff, d_returned);
  return cudaGetLastError() == cudaSuccess ? AWQ_OK : AWQ_ERR_CUDA;
}
