// Per-row e4m3 quantization for the FP8 (kind::f8f6f4) GEMM operands.
//
// Row r of x (fp32 or bf16, cols values) becomes
//   scale[r] = amax_r / 448  (1 for an all-zero row)
//   q[r, c]  = e4m3(x[r, c] / scale[r])
// with IEEE fp32 division and the conversion rounding to nearest even and
// saturating at +-448 (cvt.rn.satfinite), so the codes are a pure function of
// the fp32 inputs.  One CTA per row; cols must be even.
#include <cuda_bf16.h>

#include "kernels.h"
#include "sm100.cuh"

namespace {

__device__ __forceinline__ float load_as_float(const float* p, long long i) { return p[i]; }
__device__ __forceinline__ float load_as_float(const __nv_bfloat16* p, long long i) { return __bfloat162float(p[i]); }

// Two fp32 values to a packed pair of e4m3 codes: lo in the low byte.
__device__ __forceinline__ uint16_t e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

template <typename TI>
__global__ void __launch_bounds__(256) k_quant_rows_e4m3(const TI* __restrict__ x, long long cols,
                                                         uint8_t* __restrict__ q, float* __restrict__ scale) {
  __shared__ float red[8];
  const long long row = blockIdx.x;
  const TI* xr = x + row * cols;
  float m = 0.f;
  for (long long c = threadIdx.x; c < cols; c += blockDim.x) m = fmaxf(m, fabsf(load_as_float(xr, c)));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  float amax = red[0];
  for (int w = 1; w < static_cast<int>(blockDim.x >> 5); ++w) amax = fmaxf(amax, red[w]);
  const float s = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  if (threadIdx.x == 0) scale[row] = s;
  uint16_t* q2 = reinterpret_cast<uint16_t*>(q + row * cols);
  for (long long c = 2 * threadIdx.x; c < cols; c += 2 * blockDim.x)
    q2[c >> 1] = e4m3x2(__fdiv_rn(load_as_float(xr, c), s), __fdiv_rn(load_as_float(xr, c + 1), s));
}

}  // namespace

cudaError_t launch_quant_rows_e4m3(int bf16_in, const void* x, long long rows, long long cols, void* q,
                                   float* scale, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  if (bf16_in)
    k_quant_rows_e4m3<__nv_bfloat16><<<static_cast<unsigned>(rows), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x), cols, static_cast<uint8_t*>(q), scale);
  else
    k_quant_rows_e4m3<float><<<static_cast<unsigned>(rows), 256, 0, st>>>(static_cast<const float*>(x), cols,
                                                                         static_cast<uint8_t*>(q), scale);
  return cudaGetLastError();
}
