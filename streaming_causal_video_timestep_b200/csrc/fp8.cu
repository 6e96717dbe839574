// Per-row e4m3 quantization for the FP8 (kind::f8f6f4) GEMM operands.
//
// Row r of x (fp32 or bf16, cols values) becomes
//   scale[r] = amax_r / 448  (1 for an all-zero row)
//   q[r, c]  = e4m3(x[r, c] / scale[r])
// with IEEE fp32 division and the conversion rounding to nearest even and
// saturating at +-448 (cvt.rn.satfinite), so the codes are a pure function of
// the fp32 inputs.  One CTA per row; cols must be even.
#include <cuda_bf16.h>
#include <cuda_fp16.h>

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

// 8 consecutive values as fp32.
__device__ __forceinline__ void load8(const float* p, float (&v)[8]) {
  const float4 a = reinterpret_cast<const float4*>(p)[0], b = reinterpret_cast<const float4*>(p)[1];
  v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void load8(const __nv_bfloat16* p, float (&v)[8]) {
  const uint4 w = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(h[i]);
    v[2 * i] = f.x;
    v[2 * i + 1] = f.y;
  }
}

// Rows of up to 256 * 8 * QV values, cols % 8 == 0: each thread keeps its
// vectors in registers between the max and the quantization (one read of x).
constexpr int QV = 4;

template <typename TI>
__global__ void __launch_bounds__(256) k_quant_rows_e4m3_vec(const TI* __restrict__ x, long long cols,
                                                             uint8_t* __restrict__ q, float* __restrict__ scale) {
  __shared__ float red[8];
  const long long row = blockIdx.x;
  const int nvec = static_cast<int>(cols / 8);
  const TI* xr = x + row * cols;
  float v[QV][8];
  float m = 0.f;
#pragma unroll
  for (int j = 0; j < QV; ++j) {
    const int idx = threadIdx.x + j * 256;
    if (idx < nvec) {
      load8(xr + static_cast<long long>(idx) * 8, v[j]);
#pragma unroll
      for (int i = 0; i < 8; ++i) m = fmaxf(m, fabsf(v[j][i]));
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  float amax = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) amax = fmaxf(amax, red[w]);
  const float s = amax > 0.f ? __fdiv_rn(amax, 448.0f) : 1.0f;
  if (threadIdx.x == 0) scale[row] = s;
  uint2* q8 = reinterpret_cast<uint2*>(q + row * cols);
#pragma unroll
  for (int j = 0; j < QV; ++j) {
    const int idx = threadIdx.x + j * 256;
    if (idx < nvec) {
      uint32_t lo = e4m3x2(__fdiv_rn(v[j][0], s), __fdiv_rn(v[j][1], s)) |
                    (static_cast<uint32_t>(e4m3x2(__fdiv_rn(v[j][2], s), __fdiv_rn(v[j][3], s))) << 16);
      uint32_t hi = e4m3x2(__fdiv_rn(v[j][4], s), __fdiv_rn(v[j][5], s)) |
                    (static_cast<uint32_t>(e4m3x2(__fdiv_rn(v[j][6], s), __fdiv_rn(v[j][7], s))) << 16);
      q8[idx] = make_uint2(lo, hi);
    }
  }
}

// One e4m3 code to fp32 (exact: every e4m3 value is an fp16 value).
__device__ __forceinline__ float e4m3_to_float(uint8_t c) {
  uint32_t h2;
  const uint16_t c2 = c;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(c2));
  return __half2float(__ushort_as_half(static_cast<unsigned short>(h2 & 0xFFFFu)));
}

// One CTA per (head, part) of one layer's QKV weight: the squared norms of the
// head's d output rows, then the head's power-of-two scale.
__global__ void __launch_bounds__(256) k_attn_fp8_scales(const void* w, int w_fp8, const float* w_rowscale, int D,
                                                         int H, int d, float act_bound, float* scale, float* inv) {
  __shared__ float n2[128];
  const int h = blockIdx.x, part = blockIdx.y;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  for (int r = warp; r < d; r += 8) {
    const long long row = static_cast<long long>(part) * D + static_cast<long long>(h) * d + r;
    float acc = 0.f;
    if (w_fp8) {
      const uint8_t* wr = static_cast<const uint8_t*>(w) + row * D;
      for (int c = lane; c < D; c += 32) {
        const float x = e4m3_to_float(wr[c]);
        acc = fmaf(x, x, acc);
      }
    } else {
      const __nv_bfloat16* wr = static_cast<const __nv_bfloat16*>(w) + row * D;
      for (int c = lane; c < D; c += 32) {
        const float x = __bfloat162float(wr[c]);
        acc = fmaf(x, x, acc);
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      const float rs = w_fp8 ? w_rowscale[row] : 1.0f;
      n2[r] = acc * rs * rs;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float m = 0.f;
    if (part < 2) {
      for (int j = 0; j + 1 < d; j += 2) m = fmaxf(m, n2[j] + n2[j + 1]);
    } else {
      for (int j = 0; j < d; ++j) m = fmaxf(m, n2[j]);
    }
    const float bound = act_bound * sqrtf(m);
    float sc = 1.0f, iv = 1.0f;
    if (bound > 0.f) {
      int ex = 0;
      const float mant = frexpf(bound / 448.0f, &ex);   // bound / 448 = mant * 2^ex, mant in [1/2, 1)
      const int e = mant == 0.5f ? ex - 1 : ex;
      sc = ldexpf(1.0f, e);
      iv = ldexpf(1.0f, -e);
    }
    scale[part * H + h] = sc;
    inv[part * H + h] = iv;
  }
}

}  // namespace

cudaError_t launch_attn_fp8_scales(const void* w, int w_fp8, const float* w_rowscale, int D, int H, int d,
                                   float act_bound, float* scale, float* inv, cudaStream_t st) {
  if (!w || d > 128 || d % 2 != 0 || (w_fp8 && !w_rowscale)) return cudaErrorInvalidValue;
  k_attn_fp8_scales<<<dim3(H, 3), 256, 0, st>>>(w, w_fp8, w_rowscale, D, H, d, act_bound, scale, inv);
  return cudaGetLastError();
}

cudaError_t launch_quant_rows_e4m3(int bf16_in, const void* x, long long rows, long long cols, void* q,
                                   float* scale, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  const uintptr_t align = reinterpret_cast<uintptr_t>(x) | reinterpret_cast<uintptr_t>(q);
  if (cols % 8 == 0 && cols <= 256LL * 8 * QV && align % 16 == 0) {
    if (bf16_in)
      k_quant_rows_e4m3_vec<__nv_bfloat16><<<static_cast<unsigned>(rows), 256, 0, st>>>(
          static_cast<const __nv_bfloat16*>(x), cols, static_cast<uint8_t*>(q), scale);
    else
      k_quant_rows_e4m3_vec<float><<<static_cast<unsigned>(rows), 256, 0, st>>>(
          static_cast<const float*>(x), cols, static_cast<uint8_t*>(q), scale);
    return cudaGetLastError();
  }
  if (bf16_in)
    k_quant_rows_e4m3<__nv_bfloat16><<<static_cast<unsigned>(rows), 256, 0, st>>>(
        static_cast<const __nv_bfloat16*>(x), cols, static_cast<uint8_t*>(q), scale);
  else
    k_quant_rows_e4m3<float><<<static_cast<unsigned>(rows), 256, 0, st>>>(static_cast<const float*>(x), cols,
                                                                         static_cast<uint8_t*>(q), scale);
  return cudaGetLastError();
}
