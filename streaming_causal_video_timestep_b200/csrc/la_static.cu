// la_op_attention_static: the block attention op for callers that cannot
// allocate device memory.
//
// Some callers cannot call cudaMalloc: plugins loaded into a host application
// that owns all device memory (custom allocators, memory pools with fixed
// budgets), or real-time paths where an allocation (and the implicit
// synchronisation it can cause) is not allowed.  This entry point needs one scratch buffer -- the
// queries pre-multiplied by the softmax scale, which the attention kernel reads
// -- and keeps it in a file-scope device array instead of allocating it.
//
// The array is a static __device__ object of LA_STATIC_Q_ELEMS bf16 values
// (16 MiB): every GPU that loads this library holds it until the process exits.
// Host code may not use its name as an address: the name is a host-side stand-in.
// The device address is obtained once per device with cudaGetSymbolAddress (with
// that device current) on the first call made on it, so make the first call on
// each device before any stream capture.  All calls share the array and
// overwrite the part they use; calls that overlap on the GPU (different
// streams, or concurrent host threads) race on it.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <mutex>
#include <string>

#include "kernels.h"
#include "la_stream.h"
#include "sm100.cuh"
#include "tmap.h"

namespace {

static __device__ __align__(256) __nv_bfloat16 g_q_scaled[LA_STATIC_Q_ELEMS];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch[kMaxDevices] = {};

// q (bf16) times the softmax scale log2(e)/sqrt(d), rounded once to bf16.
__global__ void k_prescale_q(const __nv_bfloat16* __restrict__ q, __nv_bfloat16* __restrict__ out, long long n,
                             float scale) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
    out[i] = __float2bfloat16_rn(__fmul_rn(__bfloat162float(q[i]), scale));
}

// Device address of the scratch array on the current device (set-up on first use).
int scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LA_ECUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_q_scaled);
    if (e != cudaSuccess || !p) {
      std::fprintf(stderr, "la_op_attention_static: cudaGetSymbolAddress failed: %s\n", cudaGetErrorString(e));
      return LA_ECUDA;
    }
    g_scratch[dev] = p;
  }
  *out = g_scratch[dev];
  return LA_OK;
}

}  // namespace

extern "C" int la_op_attention_static(const void* q, int64_t Tq, int32_t H, int32_t d, int32_t nseg,
                                      const void* const* k_seg, const void* const* v_seg, const int64_t* seg_len,
                                      void* out, float* out32, void* cuda_stream) {
  if (!q || !out || !k_seg || !v_seg || !seg_len || Tq < 1 || H < 1 || H > 65535 || d != 128) return LA_EINVAL;
  if (nseg < 1 || nseg > LA_MAX_SEG) return LA_EINVAL;
  for (int s = 0; s < nseg; ++s)
    if (!k_seg[s] || !v_seg[s] || seg_len[s] < 1 || seg_len[s] > (1 << 30)) return LA_EINVAL;
  const long long n = static_cast<long long>(H) * Tq * d;
  if (n > static_cast<long long>(LA_STATIC_Q_ELEMS)) {
    std::fprintf(stderr,
                 "la_op_attention_static: H*Tq*d = %lld exceeds the static scratch of %lld elements "
                 "(LA_STATIC_Q_ELEMS); use la_op_attention\n",
                 n, static_cast<long long>(LA_STATIC_Q_ELEMS));
    return LA_EINVAL;
  }
  void* scratch = nullptr;
  int r = scratch_for_current_device(&scratch);
  if (r != LA_OK) return r;
  std::string err;
  if (!tmap_init(err)) return LA_ECUDA;

  AttnParams p{};
  p.ngroups = 1;
  p.Tq = static_cast<int>(Tq);
  p.H = H;
  p.d = d;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(d)));
  p.q_prescaled = 1;
  p.out = out;
  p.out32 = out32;
  p.out_ld = static_cast<long long>(H) * d;
  p.err = nullptr;
  p.qbase = scratch;
  AttnGroup& g = p.g[0];
  g.nseg = nseg;
  AttnMaps maps;
  if (!tmap_planes_bf16(&maps.q, scratch, d, Tq, H, 1, err)) return LA_ECUDA;
  for (int s = 0; s < nseg; ++s) {
    g.seg[s] = AttnSeg{s, s, 0, 0, static_cast<int>(seg_len[s])};
    if (!tmap_planes_bf16(&maps.k[s], k_seg[s], d, seg_len[s], H, 1, err)) return LA_ECUDA;
    if (!tmap_planes_bf16(&maps.v[s], v_seg[s], d, seg_len[s], H, 1, err)) return LA_ECUDA;
  }
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  int blocks = static_cast<int>((n + 255) / 256);
  if (blocks > 148 * 8) blocks = 148 * 8;
  k_prescale_q<<<blocks, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(q), static_cast<__nv_bfloat16*>(scratch),
                                       n, p.scale_log2);
  if (cudaGetLastError() != cudaSuccess) return LA_ECUDA;
  return launch_attention_tc(maps, p, st) == cudaSuccess ? LA_OK : LA_ECUDA;
}
