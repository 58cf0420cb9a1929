// Self-check of the device's bounded waits.
//
// Every mbarrier wait of the GEMM roles gives up after a fixed number of SM cycles, records the
// timeout bit in the error word and lets the kernel return, so a wait that can never complete
// costs about two seconds and an error status instead of a hung GPU.  This check runs that same
// wait (afd::mbar_wait) on an mbarrier that no thread arrives on, and reports what the host sees.
#include "afd_ffn.h"

#include <cuda_runtime.h>

#include "common.cuh"
#include "ptx.cuh"

namespace {

// One thread: wait for the first phase of a fresh mbarrier of its CTA (expected count 1, no
// arrival ever), exactly as a consumer role waits for a full stage; on giving up, record the
// timeout the way the roles do.
__global__ void bounded_wait_check_kernel(int* err, long long* cycles) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x != 0) return;
  const uint32_t b = afd::smem_u32(&bar);
  afd::mbar_init(b, 1);
  abort_flag = 0;
  const long long t0 = clock64();
  const bool ok = afd::mbar_wait(b, 0, &abort_flag);
  *cycles = clock64() - t0;
  if (!ok) {
    abort_flag = 1;
    atomicOr(err, afd::kErrTimeout);
  }
}

}  // namespace

extern "C" int afd_ffn_check_bounded_wait(int64_t* waited_cycles) {
  if (waited_cycles) *waited_cycles = 0;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return AFD_ERR_NO_DEVICE;
  int* err = nullptr;
  long long* cycles = nullptr;
  int h_err = 0;
  long long h_cycles = 0;
  cudaError_t e = cudaMalloc(&err, sizeof(int));
  if (e == cudaSuccess) e = cudaMalloc(&cycles, sizeof(long long));
  if (e == cudaSuccess) e = cudaMemset(err, 0, sizeof(int));
  if (e == cudaSuccess) {
    bounded_wait_check_kernel<<<1, 32>>>(err, cycles);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(&h_err, err, sizeof(int), cudaMemcpyDeviceToHost);
  if (e == cudaSuccess) e = cudaMemcpy(&h_cycles, cycles, sizeof(long long), cudaMemcpyDeviceToHost);
  if (err) cudaFree(err);
  if (cycles) cudaFree(cycles);
  if (e != cudaSuccess) return AFD_ERR_CUDA;
  if (waited_cycles) *waited_cycles = h_cycles;
  return (h_err & afd::kErrTimeout) ? AFD_ERR_DEVICE_TIMEOUT : AFD_OK;
}
