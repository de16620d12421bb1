// Self-test of the device-side time-out path used by every bounded wait in
// the tensor-core kernel: one thread initialises an mbarrier that nothing
// will ever complete and waits on it with the same bounded wait; on expiry
// it records CKDA_ERR_DEVICE_TIMEOUT in the status word and returns, leaving
// the context usable.
#include "common.cuh"
#include "sm100.cuh"

namespace ckda {

__global__ void bounded_wait_probe(int* status, unsigned long long limit_ns) {
  __shared__ __align__(8) unsigned long long bar;
  const uint32_t b = sm100::smem_u32(&bar);
  if (threadIdx.x == 0) {
    sm100::mbar_init(b, 1);
    sm100::fence_mbar_init();
    if (!sm100::mbar_wait_bounded(b, 0, limit_ns)) set_status(status, CKDA_ERR_DEVICE_TIMEOUT);
  }
}

cudaError_t launch_bounded_wait_probe(int* status, unsigned long long limit_ns,
                                      cudaStream_t stream) {
  bounded_wait_probe<<<1, 32, 0, stream>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace ckda
