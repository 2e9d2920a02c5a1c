// Self-test of the failure path of the scan kernels' bounded waits.
//
// The tensor-core kernels wait for their own MMA completions on mbarriers with mbar_wait,
// which gives up after a poll budget or a wall-time limit, sets a flag and lets the kernel
// finish; the host then reads SRNL_E_TIMEOUT.  This entry point runs that same helper on an
// mbarrier that nothing ever completes (the flag is never set), so the give-up path can be
// exercised without faulting or hanging the device.
#include <cuda_runtime.h>

#include <string>

#include "srnl_internal.h"
#include "srnl_scan.h"
#include "srnl_umma.cuh"

namespace {

__global__ void bounded_wait_probe_kernel(unsigned long long limit_ns, int* status) {
  __shared__ unsigned long long bar;
  __shared__ int failed;
  if (threadIdx.x == 0) {
    failed = 0;
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(srnl::smem_u32(&bar)));
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    srnl::mbar_wait(&bar, 0u, &failed, limit_ns);   // no thread ever arrives on this barrier
    *status = failed ? SRNL_E_TIMEOUT : SRNL_OK;
  }
}

}  // namespace

namespace srnl {
cudaError_t launch_wait_probe(unsigned long long limit_ns, int* status, cudaStream_t s) {
  bounded_wait_probe_kernel<<<1, 32, 0, s>>>(limit_ns, status);
  return cudaGetLastError();
}
}  // namespace srnl

extern "C" srnl_status srnl_selftest_wait_timeout(int wait_ms) {
  if (wait_ms < 1 || wait_ms > 5000) {
    srnl::set_thread_error("wait_ms must lie in [1, 5000]");
    return SRNL_E_INVAL;
  }
  int* dev = nullptr;
  cudaError_t e = cudaMalloc(&dev, sizeof(int));
  int status = SRNL_OK;
  if (e == cudaSuccess) e = cudaMemset(dev, 0xff, sizeof(int));
  if (e == cudaSuccess) {
    bounded_wait_probe_kernel<<<1, 32>>>((unsigned long long)wait_ms * 1000000ull, dev);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(&status, dev, sizeof(int), cudaMemcpyDeviceToHost);
  if (dev != nullptr) cudaFree(dev);
  if (e != cudaSuccess) {
    srnl::set_thread_error(std::string("self-test: ") + cudaGetErrorName(e) + " (" + cudaGetErrorString(e) + ")");
    return SRNL_E_CUDA;
  }
  srnl::set_thread_error(status == SRNL_E_TIMEOUT ? "bounded wait gave up (expected)"
                                                  : "bounded wait completed on a barrier nothing completes");
  return static_cast<srnl_status>(status);
}
