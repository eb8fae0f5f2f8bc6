// kmip_testing.cu -- test hook for the bounded pipeline wait (kmip_testing.h).
#include "../../include/kmip_testing.h"
#include "kmip_internal.h"
#include "kmip_sm100.cuh"

#if defined(__GNUC__)
#define KMIP_EXPORT extern "C" __attribute__((visibility("default")))
#else
#define KMIP_EXPORT extern "C"
#endif

namespace kmip {
namespace {

__global__ void wait_timeout_kernel(uint64_t timeout_ns, int* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ volatile int abort_flag;
  if (threadIdx.x == 0) {
    sm100::mbar_init(sm100::smem_addr(&bar), 1);
    abort_flag = 0;
    sm100::fence_mbar_init();
  }
  __syncthreads();
  // Nothing ever arrives on `bar`: the wait must give up after timeout_ns.
  const bool ok = sm100::mbar_wait(sm100::smem_addr(&bar), 0, &abort_flag, timeout_ns);
  __syncthreads();
  if (threadIdx.x == 0 && (!ok || abort_flag)) record_status(status, KMIP_ERR_TIMEOUT);
}

}  // namespace
}  // namespace kmip

KMIP_EXPORT kmip_status_t kmip_test_wait_timeout(kmip_stream_t stream, int timeout_us) {
  if (timeout_us < 1 || timeout_us > 1000000) return KMIP_ERR_INVALID_ARG;
  int* status = kmip::status_ptr();
  if (!status) return KMIP_ERR_CUDA;
  kmip::wait_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(
      (uint64_t)timeout_us * 1000ull, status);
  if (cudaGetLastError() != cudaSuccess) return KMIP_ERR_CUDA;
  return KMIP_OK;
}
