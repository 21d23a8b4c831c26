// Diagnostic kernels: initialisation of mask-probe records, and a kernel
// whose bounded wait is made to run out, so that the device-status path of a
// timeout can be exercised without faulting or hanging the GPU.
#include "common.cuh"
#include "kernels.h"

namespace dory {

namespace {

__global__ void probe_init_kernel(int32_t* probe, size_t n_records) {
  const size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x;
  if (i >= n_records) return;
  reinterpret_cast<int4*>(probe)[i] = make_int4(0x7FFFFFFF, -1, 0, 0);
}

// One warp: lane 0 initialises an mbarrier expecting one arrival, then waits
// for a phase that no thread ever completes.  The wait gives up after
// limit_ns and records kStatusTimeout.  Nothing else is in flight.
__global__ void wait_timeout_kernel(uint32_t* status, uint64_t limit_ns) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_mbarrier_init();
  }
  __syncwarp();
  if (threadIdx.x == 0)
    mbar_wait_bounded_ns(&bar, 0, reinterpret_cast<volatile int*>(&abort_flag), status, limit_ns);
  __syncwarp();
}

}  // namespace

cudaError_t launch_probe_init(int32_t* probe, size_t n_records, cudaStream_t s) {
  if (n_records == 0) return cudaSuccess;
  probe_init_kernel<<<static_cast<unsigned>((n_records + 255) / 256), 256, 0, s>>>(probe, n_records);
  return cudaGetLastError();
}

cudaError_t launch_wait_timeout(uint32_t* status, uint64_t limit_ns, cudaStream_t s) {
  wait_timeout_kernel<<<1, 32, 0, s>>>(status, limit_ns);
  return cudaGetLastError();
}

}  // namespace dory
