// fp32 path on CUDA cores (no TF32), used by fp32 streams: the reference-
// precision configurations are small, so these kernels aim at exactness, not speed.
#include "kernels.h"
#include "sm100.cuh"

namespace {

constexpr int TM = 64, TN = 64, TK = 16;

__device__ __forceinline__ void epi_scalar(const GemmEpiParams& ep, long long row, long long col, float acc) {
  const long long off = row * ep.ld + col;
  float* out = reinterpret_cast<float*>(ep.out);
  switch (ep.kind) {
    case EPI_STORE:
    case EPI_STORE32: out[off] = acc; break;
    case EPI_RESID: {
      const float h = ep.h32[off] + acc;
      ep.h32[off] = h;
      if (out && out != ep.h32) out[off] = h;
      break;
    }
    case EPI_SET32:
      ep.h32[off] = acc;
      if (out && out != ep.h32) out[off] = acc;
      break;
    case EPI_RESID_GATED: {
      const float h = fmaf(ep.gate[row / ep.rows_per_group][col], acc, ep.h32[off]);
      ep.h32[off] = h;
      if (out && out != ep.h32) out[off] = h;
      break;
    }
    case EPI_GELU: out[off] = gelu_tanh(acc); break;
    case EPI_EULER: {
      const int g = static_cast<int>(row / ep.rows_per_group);
      if (!ep.active[g]) break;
      ep.h32[off] += ep.dt[g] * acc;
      if (ep.vtap) ep.vtap[off] = acc;
      break;
    }
  }
}

// C = A W^T: A [M, K], W [N, K] row-major fp32.
__global__ void __launch_bounds__(256) k_gemm_f32(const float* __restrict__ A, const float* __restrict__ W,
                                                  const __grid_constant__ GemmEpiParams ep, int M, int N, int K) {
  __shared__ float As[TK][TM + 4];
  __shared__ float Ws[TK][TN + 4];
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const long long m0 = static_cast<long long>(blockIdx.y) * TM;
  const long long n0 = static_cast<long long>(blockIdx.x) * TN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += TK) {
    for (int i = tid; i < TM * TK; i += 256) {
      const int r = i / TK, kc = i % TK;
      const long long gm = m0 + r, gk = k0 + kc;
      As[kc][r] = (gm < M && gk < K) ? A[gm * K + gk] : 0.f;
      const long long gn = n0 + r;
      Ws[kc][r] = (gn < N && gk < K) ? W[gn * K + gk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Ws[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const long long r = m0 + ty * 4 + i, c = n0 + tx * 4 + j;
      if (r < M && c < N) epi_scalar(ep, r, c, acc[i][j]);
    }
}

// One warp per query row; lanes own keys for the scores and output dims for the sums.
__global__ void __launch_bounds__(128) k_attn_f32(const __grid_constant__ AttnParams p) {
  __shared__ float qs[4][128];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const AttnGroup& g = p.g[blockIdx.z];
  const int h = blockIdx.y;
  const int t = blockIdx.x * 4 + warp;
  const int d = p.d, H = p.H;
  if (t >= p.Tq) return;
  const float* q = reinterpret_cast<const float*>(p.qbase) +
                   ((static_cast<long long>(g.q_slice) * H + h) * p.Tq + t) * d;
  for (int e = lane; e < d; e += 32) qs[warp][e] = q[e];
  __syncwarp();
  float o[4] = {0.f, 0.f, 0.f, 0.f};
  float m = -INFINITY, l = 0.f;
  for (int s = 0; s < g.nseg; ++s) {
    const AttnSeg& sg = g.seg[s];
    const float* kb = reinterpret_cast<const float*>(p.kbase[sg.kmap]) +
                      (static_cast<long long>(sg.kslice) * H + h) * p.krows[sg.kmap] * d;
    const float* vb = reinterpret_cast<const float*>(p.vbase[sg.vmap]) +
                      (static_cast<long long>(sg.vslice) * H + h) * p.vrows[sg.vmap] * d;
    for (int j0 = 0; j0 < sg.len; j0 += 32) {
      const int j = j0 + lane;
      float sj = -INFINITY;
      if (j < sg.len) {
        const float* kr = kb + static_cast<long long>(j) * d;
        float dot = 0.f;
        for (int e = 0; e < d; ++e) dot = fmaf(qs[warp][e], kr[e], dot);
        sj = __fmul_rn(dot, p.scale_log2);   // rounded: the row max then gives exactly 2^0
      }
      float mx = sj;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_new = fmaxf(m, mx);
      const float alpha = exp2f(m - m_new);
      const float pj = j < sg.len ? exp2f(sj - m_new) : 0.f;
      float ps = pj;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
      l = l * alpha + ps;
#pragma unroll
      for (int i = 0; i < 4; ++i) o[i] *= alpha;
      const int cnt = min(32, sg.len - j0);
      for (int jj = 0; jj < cnt; ++jj) {
        const float w = __shfl_sync(0xffffffffu, pj, jj);
        const float* vr = vb + static_cast<long long>(j0 + jj) * d;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int e = lane + 32 * i;
          if (e < d) o[i] = fmaf(w, vr[e], o[i]);
        }
      }
      m = m_new;
    }
  }
  float* out = reinterpret_cast<float*>(p.out) + (static_cast<long long>(g.out_row0) + t) * p.out_ld +
               static_cast<long long>(h) * d;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int e = lane + 32 * i;
    if (e < d) out[e] = o[i] / l;
  }
}

}  // namespace

cudaError_t launch_gemm_f32(const float* A, const float* W, const GemmEpiParams& ep, int M, int N, int K,
                            cudaStream_t st) {
  dim3 grid((N + TN - 1) / TN, (M + TM - 1) / TM);
  k_gemm_f32<<<grid, 256, 0, st>>>(A, W, ep, M, N, K);
  return cudaGetLastError();
}

cudaError_t launch_attn_f32(const AttnParams& p, cudaStream_t st) {
  dim3 grid((p.Tq + 3) / 4, p.H, p.ngroups);
  k_attn_f32<<<grid, 128, 0, st>>>(p);
  return cudaGetLastError();
}
