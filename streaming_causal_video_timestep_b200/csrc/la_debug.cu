// la_debug_wait_timeout / la_debug_op_wait_timeout: exercise the failure path
// of every pipelined kernel (a bounded mbarrier wait that gives up, raises the
// device error word and returns) without faulting or hanging the GPU; the
// second raises the op-level error word that la_op_status reports.
#include <cuda_runtime.h>

#include "kernels.h"
#include "la_stream.h"
#include "sm100.cuh"

namespace {

// One thread waits on phase 0 of a shared-memory mbarrier of count 1, which it
// completes itself first when `complete` is set and otherwise nothing completes.
__global__ void k_wait_probe(unsigned long long limit_ns, int complete, int* err) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
    if (complete) mbar_arrive(&bar);
    mbar_wait_for(&bar, 0, err, limit_ns);
  }
}

}  // namespace

extern "C" int la_debug_wait_timeout(int64_t limit_ns, int32_t complete, int32_t* device_error) {
  if (limit_ns < 0 || limit_ns > 10000000000LL || !device_error) return LA_EINVAL;
  int* err = nullptr;
  if (cudaMalloc(&err, sizeof(int)) != cudaSuccess) return LA_ENOMEM;
  int code = LA_OK;
  int h = 0;
  if (cudaMemset(err, 0, sizeof(int)) != cudaSuccess) {
    code = LA_ECUDA;
  } else {
    k_wait_probe<<<1, 32>>>(static_cast<unsigned long long>(limit_ns), complete ? 1 : 0, err);
    if (cudaGetLastError() != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess ||
        cudaMemcpy(&h, err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess)
      code = LA_ECUDA;
  }
  cudaFree(err);
  if (code != LA_OK) return code;
  *device_error = h;
  return h ? LA_EDEVICE : LA_OK;
}

extern "C" int la_debug_op_wait_timeout(int64_t limit_ns, void* cuda_stream) {
  if (limit_ns < 0 || limit_ns > 10000000000LL) return LA_EINVAL;
  int* err = nullptr;
  if (op_error_word(&err) != LA_OK) return LA_ECUDA;
  k_wait_probe<<<1, 32, 0, static_cast<cudaStream_t>(cuda_stream)>>>(static_cast<unsigned long long>(limit_ns), 0,
                                                                      err);
  return cudaGetLastError() == cudaSuccess ? LA_OK : LA_ECUDA;
}
