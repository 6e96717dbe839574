// Bandwidth-bound kernels: RoPE tables, fused Rolling RoPE + ring append +
// sink re-rope, the sink's K/V split, in-projection helpers and the Euler update.
#include <cuda_fp16.h>

#include "kernels.h"
#include "sm100.cuh"

namespace {

template <typename T> struct Vec8;
template <> struct Vec8<__nv_bfloat16> {
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 w = *reinterpret_cast<const uint4*>(p);
    const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float2 f = __bfloat1622float2(b[i]);
      v[2 * i] = f.x;
      v[2 * i + 1] = f.y;
    }
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&v)[8]) {
    uint4 w;
    w.x = pack_bf16x2(v[0], v[1]);
    w.y = pack_bf16x2(v[2], v[3]);
    w.z = pack_bf16x2(v[4], v[5]);
    w.w = pack_bf16x2(v[6], v[7]);
    *reinterpret_cast<uint4*>(p) = w;
  }
};
template <> struct Vec8<float> {
  static __device__ __forceinline__ void load(const float* p, float (&v)[8]) {
    const float4 a = reinterpret_cast<const float4*>(p)[0];
    const float4 b = reinterpret_cast<const float4*>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
  static __device__ __forceinline__ void store(float* p, const float (&v)[8]) {
    reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
};

// Rotate the 4 pairs of an 8-element chunk; pair j = 4*ch + jj.
__device__ __forceinline__ void rotate8(float (&v)[8], int ch, int buf, int trow, int rr, int cc,
                                        const RopeArgs& a) {
#pragma unroll
  for (int jj = 0; jj < 4; ++jj) {
    const int j = 4 * ch + jj;
    float c, s;
    if (j < a.pt) {
      const int idx = (buf * LA_TROWS + trow) * LA_MAX_PT + j;
      c = a.tcos[idx];
      s = a.tsin[idx];
    } else if (j < a.pt + a.ph) {
      const int idx = rr * a.ph + (j - a.pt);
      c = a.rcos[idx];
      s = a.rsin[idx];
    } else {
      const int idx = cc * a.pw + (j - a.pt - a.ph);
      c = a.ccos[idx];
      s = a.csin[idx];
    }
    const float x0 = v[2 * jj], x1 = v[2 * jj + 1];
    v[2 * jj] = x0 * c - x1 * s;
    v[2 * jj + 1] = x0 * s + x1 * c;
  }
}

// One (pair, token) of an active buffer a thread, token fastest (coalesced
// stores); the same three-way table choice as rotate8.
__global__ void k_rope_rows(const __grid_constant__ PassDesc pd, const __grid_constant__ RopeArgs a,
                            float2* __restrict__ out, long long ld) {
  const int half = a.d / 2;
  const long long per_buf = static_cast<long long>(half) * a.T;
  const long long total = pd.nactive * per_buf;
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int ai = static_cast<int>(i / per_buf);
    const long long rem = i - ai * per_buf;
    const int j = static_cast<int>(rem / a.T), n = static_cast<int>(rem - static_cast<long long>(j) * a.T);
    const int buf = pd.active_buf[ai];
    const int f = n / a.F, m = n - f * a.F;
    const int rr = m / a.grid_w, cc = m - rr * a.grid_w;
    float c, s;
    if (j < a.pt) {
      const int idx = (buf * LA_TROWS + f) * LA_MAX_PT + j;
      c = a.tcos[idx];
      s = a.tsin[idx];
    } else if (j < a.pt + a.ph) {
      const int idx = rr * a.ph + (j - a.pt);
      c = a.rcos[idx];
      s = a.rsin[idx];
    } else {
      const int idx = cc * a.pw + (j - a.pt - a.ph);
      c = a.ccos[idx];
      s = a.csin[idx];
    }
    out[static_cast<long long>(j) * ld + static_cast<long long>(buf) * a.T + n] = make_float2(c, s);
  }
}

__global__ void k_rope_ttab(const __grid_constant__ PassDesc pd, int fpb, int pt, const double* __restrict__ omega,
                            float* tcos, float* tsin) {
  const int rows = fpb + 1;
  const int per_buf = rows * pt;
  for (int i = threadIdx.x; i < pd.nactive * per_buf; i += blockDim.x) {
    const int ai = i / per_buf, rem = i % per_buf;
    const int f = rem / pt, j = rem % pt;
    const int buf = pd.active_buf[ai];
    const int pos = f < fpb ? pd.frame_tpos[buf] + f : pd.sink_tpos[buf];
    double s, c;
    sincos(static_cast<double>(pos) * omega[j], &s, &c);
    const int idx = (buf * LA_TROWS + f) * LA_MAX_PT + j;
    tcos[idx] = static_cast<float>(c);
    tsin[idx] = static_cast<float>(s);
  }
}

// Rolling RoPE + ring append from an fp32 [q | k | v] projection (fp32
// streams; bf16 streams do this in the QKV GEMM epilogue).  Outputs are
// rounded once to TO.
template <typename TO>
__global__ void __launch_bounds__(256) k_rope_append(const __grid_constant__ PassDesc pd,
                                                     const __grid_constant__ RopeArgs a, long long n_main) {
  const int chunks = a.d / 8;
  const float* qkv = reinterpret_cast<const float*>(a.qkv);
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < n_main;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    long long rest = idx;
    const int ch = static_cast<int>(rest % chunks); rest /= chunks;
    const int h = static_cast<int>(rest % a.H); rest /= a.H;
    const int part = static_cast<int>(rest % 3); rest /= 3;
    const int n = static_cast<int>(rest % a.T); rest /= a.T;
    const int buf = pd.active_buf[rest];
    const long long row = static_cast<long long>(buf) * a.T + n;
    float v[8];
    Vec8<float>::load(qkv + row * 3 * a.D + part * a.D + h * a.d + ch * 8, v);
    if (part < 2) {
      const int f = n / a.F, rem = n % a.F;
      rotate8(v, ch, buf, f, rem / a.grid_w, rem % a.grid_w, a);
    }
    TO* dst;
    const long long tok = static_cast<long long>(n) * a.d + ch * 8;
    if (part == 0) {
      dst = reinterpret_cast<TO*>(a.q_rope) + (static_cast<long long>(buf) * a.H + h) * a.T * a.d + tok;
    } else {
      const long long slice = a.ring_slice0 + static_cast<long long>(pd.slot[buf]) * a.E + pd.write_entry[buf];
      TO* base = reinterpret_cast<TO*>(part == 1 ? a.ring_k : a.ring_v);
      dst = base + (slice * a.H + h) * a.T * a.d + tok;
    }
    Vec8<TO>::store(dst, v);
  }
}

// Per-block re-rope of the fp32 un-roped sink K of every layer for every active
// buffer, in one launch (the sink positions depend on the buffer's block, not
// on the layer).  The spatial rotation factors depend only on (token, pair) and
// the temporal ones only on (buffer, pair), so one thread takes one (layer,
// token, 8-element chunk) for SINK_HEADS heads: it loads their chunks and the
// factors once and writes each chunk roped, rounded once to TO, for every
// active buffer.  Reads nl*F*H*d*4 bytes once and writes
// nl*nactive*F*H*d*sizeof(TO).
constexpr int SINK_HEADS = 8;

template <typename TO>
__global__ void __launch_bounds__(256) k_sink_rerope(const __grid_constant__ PassDesc pd,
                                                     const __grid_constant__ RopeArgs a, long long n) {
  const int chunks = a.d / 8;
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < n;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int ch = static_cast<int>(idx % chunks);
    long long rest = idx / chunks;
    const int m = static_cast<int>(rest % a.F);
    rest /= a.F;
    const int hgroups = (a.H + SINK_HEADS - 1) / SINK_HEADS;
    const int h0 = static_cast<int>(rest % hgroups) * SINK_HEADS;
    const int l = static_cast<int>(rest / hgroups);
    const int nh = min(SINK_HEADS, a.H - h0);
    const long long plane = static_cast<long long>(a.H) * a.F * a.d;
    float v[SINK_HEADS][8];
#pragma unroll
    for (int k = 0; k < SINK_HEADS; ++k)
      if (k < nh)
        Vec8<float>::load(reinterpret_cast<const float*>(a.sink_k) + l * plane +
                              (static_cast<long long>(h0 + k) * a.F + m) * a.d + ch * 8, v[k]);
    const int rr = m / a.grid_w, cc = m % a.grid_w;
    float c[4], sn[4];
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int j = 4 * ch + jj;
      if (j >= a.pt && j < a.pt + a.ph) {
        c[jj] = a.rcos[rr * a.ph + (j - a.pt)];
        sn[jj] = a.rsin[rr * a.ph + (j - a.pt)];
      } else if (j >= a.pt) {
        c[jj] = a.ccos[cc * a.pw + (j - a.pt - a.ph)];
        sn[jj] = a.csin[cc * a.pw + (j - a.pt - a.ph)];
      } else {
        c[jj] = 1.f;
        sn[jj] = 0.f;
      }
    }
    for (int ai = 0; ai < pd.nactive; ++ai) {
      const int buf = pd.active_buf[ai];
      float cb[4], sb[4];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const int j = 4 * ch + jj;
        if (j < a.pt) {
          const int t = (buf * LA_TROWS + a.fpb) * LA_MAX_PT + j;
          cb[jj] = a.tcos[t];
          sb[jj] = a.tsin[t];
        } else {
          cb[jj] = c[jj];
          sb[jj] = sn[jj];
        }
      }
      TO* out = reinterpret_cast<TO*>(a.sink_k_rope) + (static_cast<long long>(l) * a.nb + buf) * plane;
#pragma unroll
      for (int k = 0; k < SINK_HEADS; ++k) {
        if (k >= nh) break;
        float w[8];
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
          const float x0 = v[k][2 * jj], x1 = v[k][2 * jj + 1];
          w[2 * jj] = x0 * cb[jj] - x1 * sb[jj];
          w[2 * jj + 1] = x0 * sb[jj] + x1 * cb[jj];
        }
        TO* dst = out + (static_cast<long long>(h0 + k) * a.F + m) * a.d + ch * 8;
        if constexpr (sizeof(TO) == 1)
          store_e4m3x8(reinterpret_cast<uint8_t*>(dst), w, a.fp8_inv[l * 3 * a.H + a.H + h0 + k]);
        else
          Vec8<TO>::store(dst, w);
      }
    }
  }
}

// Sink pass: split the fp32 projection [F, 3D] into the layer's un-roped K
// (fp32, kept for re-roping), V (TO), and roped q / k (TO) for the sink's
// self-attention (temporal row 0 of buffer 0 of the table).
template <typename TO>
__global__ void __launch_bounds__(256) k_sink_qkv(const __grid_constant__ RopeArgs a, float qscale, float* sink_k_raw,
                                                  TO* sink_v, TO* q_rope, TO* k_rope, uint8_t* sink_v8) {
  const int chunks = a.d / 8;
  const long long total = static_cast<long long>(a.F) * 3 * a.H * chunks;
  const float* qkv = reinterpret_cast<const float*>(a.qkv);
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < total;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    long long rest = idx;
    const int ch = static_cast<int>(rest % chunks); rest /= chunks;
    const int h = static_cast<int>(rest % a.H); rest /= a.H;
    const int part = static_cast<int>(rest % 3); rest /= 3;
    const int m = static_cast<int>(rest);
    float v[8];
    Vec8<float>::load(qkv + static_cast<long long>(m) * 3 * a.D + part * a.D + h * a.d + ch * 8, v);
    const long long off = (static_cast<long long>(h) * a.F + m) * a.d + ch * 8;
    if (part == 2) {
      Vec8<TO>::store(sink_v + off, v);
      if (sink_v8) store_e4m3x8(sink_v8 + off, v, a.fp8_inv[2 * a.H + h]);
      continue;
    }
    if (part == 1) Vec8<float>::store(sink_k_raw + off, v);
    rotate8(v, ch, 0, 0, m / a.grid_w, m % a.grid_w, a);
    if (part == 0) {
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] *= qscale;
    }
    Vec8<TO>::store(part == 0 ? q_rope + off : k_rope + off, v);
  }
}

template <typename T>
__global__ void k_in_identity(const float* __restrict__ x, float* __restrict__ h32, T* __restrict__ hop, long long n) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float v = x[i];
    h32[i] = v;
    if (hop) hop[i] = static_cast<T>(v);
  }
}

__global__ void k_cvt_bf16(const float* __restrict__ x, __nv_bfloat16* __restrict__ xb, long long n) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
    xb[i] = __float2bfloat16_rn(x[i]);
}

struct EulerArgs {
  float dt[LA_MAX_STEPS];
  int active[LA_MAX_STEPS];
  long long start[LA_MAX_STEPS];   // first float4 index of group g (groups past the last start at n4)
};

// x += dt[g] * v over float4 vectors, g = the timestep group of the row; C % 4 == 0.
// The group is found by comparing the index against the group starts (no division).
__global__ void __launch_bounds__(256) k_euler(float* __restrict__ x, const float* __restrict__ v, long long n4,
                                               const __grid_constant__ EulerArgs e, float* __restrict__ vtap) {
  float4* x4 = reinterpret_cast<float4*>(x);
  const float4* v4 = reinterpret_cast<const float4*>(v);
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
#pragma unroll 4
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n4; i += stride) {
    int g = 0;
#pragma unroll
    for (int k = 1; k < LA_MAX_STEPS; ++k) g += i >= e.start[k] ? 1 : 0;
    if (!e.active[g]) continue;
    const float dt = e.dt[g];
    const float4 vv = __ldcs(v4 + i);
    float4 xx = __ldcs(x4 + i);
    xx.x = __fmaf_rn(dt, vv.x, xx.x);
    xx.y = __fmaf_rn(dt, vv.y, xx.y);
    xx.z = __fmaf_rn(dt, vv.z, xx.z);
    xx.w = __fmaf_rn(dt, vv.w, xx.w);
    __stcs(x4 + i, xx);
    if (vtap) reinterpret_cast<float4*>(vtap)[i] = vv;
  }
}

// Per-token RMS normalisation: out[r, :] = h[r, :] / sqrt(mean(h[r, :]^2) + eps),
// one CTA per row, fp32 sum of squares; writes bf16 and / or fp32.  D % 4 == 0.
__global__ void __launch_bounds__(256) k_rmsnorm(const float* __restrict__ h, long long D, float eps,
                                                 __nv_bfloat16* __restrict__ out_bf16, float* __restrict__ out_f32) {
  const long long row = blockIdx.x;
  const float4* h4 = reinterpret_cast<const float4*>(h + row * D);
  const int n4 = static_cast<int>(D / 4);
  float ss = 0.f;
  for (int i = threadIdx.x; i < n4; i += blockDim.x) {
    const float4 v = h4[i];
    ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss))));
  }
  __shared__ float red[8];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float t = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
#pragma unroll
    for (int off = 4; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
    if (threadIdx.x == 0) red[0] = t;
  }
  __syncthreads();
  const float scale = rsqrtf(red[0] / static_cast<float>(D) + eps);
  for (int i = threadIdx.x; i < n4; i += blockDim.x) {
    const float4 v = h4[i];
    const float4 o = make_float4(v.x * scale, v.y * scale, v.z * scale, v.w * scale);
    if (out_f32) reinterpret_cast<float4*>(out_f32 + row * D)[i] = o;
    if (out_bf16) {
      uint2 w;
      w.x = pack_bf16x2(o.x, o.y);
      w.y = pack_bf16x2(o.z, o.w);
      reinterpret_cast<uint2*>(out_bf16 + row * D)[i] = w;
    }
  }
}

// AdaLN-modulated RMS normalisation: out = n(h) * (1 + scale_g) + shift_g, with
// g = row / rows_per_group selecting the vectors of the row's buffer.
__global__ void __launch_bounds__(256) k_rmsnorm_mod(const float* __restrict__ h, long long D, float eps,
                                                     const __grid_constant__ ModArgs m,
                                                     __nv_bfloat16* __restrict__ out_bf16, float* __restrict__ out_f32) {
  const long long row = blockIdx.x;
  const float4* h4 = reinterpret_cast<const float4*>(h + row * D);
  const int n4 = static_cast<int>(D / 4);
  const int g = static_cast<int>(row / m.rows_per_group);
  const float4* sh4 = reinterpret_cast<const float4*>(m.shift[g]);
  const float4* sc4 = reinterpret_cast<const float4*>(m.scale[g]);
  float ss = 0.f;
  for (int i = threadIdx.x; i < n4; i += blockDim.x) {
    const float4 v = h4[i];
    ss = fmaf(v.x, v.x, fmaf(v.y, v.y, fmaf(v.z, v.z, fmaf(v.w, v.w, ss))));
  }
  __shared__ float red[8];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float t = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
#pragma unroll
    for (int off = 4; off > 0; off >>= 1) t += __shfl_xor_sync(0xffffffffu, t, off);
    if (threadIdx.x == 0) red[0] = t;
  }
  __syncthreads();
  const float scale = rsqrtf(red[0] / static_cast<float>(D) + eps);
  for (int i = threadIdx.x; i < n4; i += blockDim.x) {
    const float4 v = h4[i], sh = sh4[i], sc = sc4[i];
    const float4 o = make_float4(fmaf(v.x * scale, 1.f + sc.x, sh.x), fmaf(v.y * scale, 1.f + sc.y, sh.y),
                                 fmaf(v.z * scale, 1.f + sc.z, sh.z), fmaf(v.w * scale, 1.f + sc.w, sh.w));
    if (out_f32) reinterpret_cast<float4*>(out_f32 + row * D)[i] = o;
    if (out_bf16) {
      uint2 w;
      w.x = pack_bf16x2(o.x, o.y);
      w.y = pack_bf16x2(o.z, o.w);
      reinterpret_cast<uint2*>(out_bf16 + row * D)[i] = w;
    }
  }
}

// Token-major fp32 columns col0 .. col0 + H*d of src [rows, src_ld] to head-major
// planes: dst[((row / rows_per_slice) * H + h) * rows_per_slice + row % rows_per_slice][e],
// times scale, rounded once to TO.  One thread per 8 consecutive values.
template <typename TO>
__global__ void __launch_bounds__(256) k_split_heads(const float* __restrict__ src, long long rows,
                                                     int rows_per_slice, int H, int d, long long src_ld,
                                                     long long col0, TO* __restrict__ dst, float scale) {
  const int chunks = d / 8;
  const long long n = rows * H * chunks;
  for (long long idx = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; idx < n;
       idx += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int ch = static_cast<int>(idx % chunks);
    const long long rest = idx / chunks;
    const int h = static_cast<int>(rest % H);
    const long long row = rest / H;
    float v[8];
    Vec8<float>::load(src + row * src_ld + col0 + static_cast<long long>(h) * d + ch * 8, v);
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] *= scale;
    const long long slice = row / rows_per_slice, r = row - slice * rows_per_slice;
    Vec8<TO>::store(dst + ((slice * H + h) * rows_per_slice + r) * d + ch * 8, v);
  }
}

int grid_for(long long n, int per_block = 256) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  long long blocks = (n + per_block - 1) / per_block;
  const long long cap = static_cast<long long>(sms) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return static_cast<int>(blocks);
}

}  // namespace

cudaError_t launch_rope_rows(const PassDesc& pd, const RopeArgs& a, float2* out, long long ld, cudaStream_t st) {
  if (pd.nactive <= 0) return cudaSuccess;
  if (a.d % 2 != 0 || a.T <= 0 || a.F <= 0 || a.grid_w <= 0) return cudaErrorInvalidValue;
  const long long total = static_cast<long long>(pd.nactive) * (a.d / 2) * a.T;
  k_rope_rows<<<grid_for(total, 256), 256, 0, st>>>(pd, a, out, ld);
  return cudaGetLastError();
}

cudaError_t launch_rope_ttab(const PassDesc& pd, int fpb, int pt, const double* omega_t, float* tcos, float* tsin,
                             cudaStream_t st) {
  if (pt <= 0 || pd.nactive <= 0) return cudaSuccess;
  k_rope_ttab<<<1, 256, 0, st>>>(pd, fpb, pt, omega_t, tcos, tsin);
  return cudaGetLastError();
}

cudaError_t launch_rope_append(int bf16_out, const PassDesc& pd, const RopeArgs& a, cudaStream_t st) {
  const long long n_main = static_cast<long long>(pd.nactive) * a.T * 3 * a.H * (a.d / 8);
  if (n_main == 0) return cudaSuccess;
  const int grid = grid_for(n_main);
  if (bf16_out)
    k_rope_append<__nv_bfloat16><<<grid, 256, 0, st>>>(pd, a, n_main);
  else
    k_rope_append<float><<<grid, 256, 0, st>>>(pd, a, n_main);
  return cudaGetLastError();
}

cudaError_t launch_sink_rerope(int out_kind, const PassDesc& pd, const RopeArgs& a, cudaStream_t st) {
  if (!a.sink_k || pd.nactive == 0) return cudaSuccess;
  if (out_kind == 2 && !a.fp8_inv) return cudaErrorInvalidValue;
  if (a.nl < 1 || a.nb < 1) return cudaErrorInvalidValue;
  for (int ai = 0; ai < pd.nactive; ++ai)
    if (pd.active_buf[ai] < 0 || pd.active_buf[ai] >= a.nb) return cudaErrorInvalidValue;
  const long long n = static_cast<long long>(a.nl) * a.F * ((a.H + SINK_HEADS - 1) / SINK_HEADS) * (a.d / 8);
  const int grid = grid_for(n);
  if (out_kind == 2)
    k_sink_rerope<uint8_t><<<grid, 256, 0, st>>>(pd, a, n);
  else if (out_kind == 1)
    k_sink_rerope<__nv_bfloat16><<<grid, 256, 0, st>>>(pd, a, n);
  else
    k_sink_rerope<float><<<grid, 256, 0, st>>>(pd, a, n);
  return cudaGetLastError();
}

cudaError_t launch_sink_qkv(int bf16_out, const RopeArgs& a, float qscale, float* sink_k_raw, void* sink_v,
                            void* q_rope, void* k_rope, cudaStream_t st, uint8_t* sink_v8) {
  if (sink_v8 && !a.fp8_inv) return cudaErrorInvalidValue;
  const long long n = static_cast<long long>(a.F) * 3 * a.H * (a.d / 8);
  const int grid = grid_for(n);
  if (bf16_out)
    k_sink_qkv<__nv_bfloat16><<<grid, 256, 0, st>>>(a, qscale, sink_k_raw, static_cast<__nv_bfloat16*>(sink_v),
                                                     static_cast<__nv_bfloat16*>(q_rope),
                                                     static_cast<__nv_bfloat16*>(k_rope), sink_v8);
  else
    k_sink_qkv<float><<<grid, 256, 0, st>>>(a, qscale, sink_k_raw, static_cast<float*>(sink_v),
                                            static_cast<float*>(q_rope), static_cast<float*>(k_rope), sink_v8);
  return cudaGetLastError();
}

cudaError_t launch_in_identity(int bf16, const float* x, float* h32, void* hop, long long n, cudaStream_t st) {
  const int grid = grid_for(n);
  if (bf16)
    k_in_identity<__nv_bfloat16><<<grid, 256, 0, st>>>(x, h32, static_cast<__nv_bfloat16*>(hop), n);
  else
    k_in_identity<float><<<grid, 256, 0, st>>>(x, h32, hop == h32 ? nullptr : static_cast<float*>(hop), n);
  return cudaGetLastError();
}

cudaError_t launch_cvt_bf16(const float* x, void* xb, long long n, cudaStream_t st) {
  k_cvt_bf16<<<grid_for(n), 256, 0, st>>>(x, static_cast<__nv_bfloat16*>(xb), n);
  return cudaGetLastError();
}

cudaError_t launch_euler(float* x, const float* v, long long rows, long long C, int rows_per_group, const float* dt,
                         const int* active, float* vtap, cudaStream_t st) {
  EulerArgs e;
  const long long n4 = rows * C / 4;
  for (int i = 0; i < LA_MAX_STEPS; ++i) {
    e.dt[i] = dt ? dt[i] : 0.f;
    e.active[i] = active ? active[i] : 1;
    const long long start = static_cast<long long>(i) * rows_per_group * (C / 4);
    e.start[i] = start < n4 ? start : n4;
  }
  k_euler<<<grid_for(n4), 256, 0, st>>>(x, v, n4, e, vtap);
  return cudaGetLastError();
}

cudaError_t launch_rmsnorm(const float* h, long long rows, long long D, float eps, void* out_bf16, float* out_f32,
                           cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  k_rmsnorm<<<static_cast<unsigned>(rows), 256, 0, st>>>(h, D, eps, static_cast<__nv_bfloat16*>(out_bf16), out_f32);
  return cudaGetLastError();
}

cudaError_t launch_rmsnorm_mod(const float* h, long long rows, long long D, float eps, const ModArgs& m,
                               void* out_bf16, float* out_f32, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  if (m.rows_per_group < 1 || (rows + m.rows_per_group - 1) / m.rows_per_group > LA_MAX_STEPS)
    return cudaErrorInvalidValue;
  k_rmsnorm_mod<<<static_cast<unsigned>(rows), 256, 0, st>>>(h, D, eps, m, static_cast<__nv_bfloat16*>(out_bf16),
                                                             out_f32);
  return cudaGetLastError();
}

cudaError_t launch_split_heads(int bf16_out, const float* src, long long rows, int rows_per_slice, int H, int d,
                               long long src_ld, long long col0, void* dst, float scale, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  if (d % 8 != 0 || src_ld % 4 != 0 || col0 % 4 != 0 || rows_per_slice < 1) return cudaErrorInvalidValue;
  const long long n = rows * H * (d / 8);
  const int grid = grid_for(n);
  if (bf16_out)
    k_split_heads<__nv_bfloat16><<<grid, 256, 0, st>>>(src, rows, rows_per_slice, H, d, src_ld, col0,
                                                        static_cast<__nv_bfloat16*>(dst), scale);
  else
    k_split_heads<float><<<grid, 256, 0, st>>>(src, rows, rows_per_slice, H, d, src_ld, col0,
                                               static_cast<float*>(dst), scale);
  return cudaGetLastError();
}
