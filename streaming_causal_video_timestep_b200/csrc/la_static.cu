// la_op_attention_static: the block attention op for callers that cannot
// allocate device memory; la_op_status: the error report of the op-level
// entry points.
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
// The device address is looked up with cudaGetSymbolAddress (with the device
// current) on the first call made on a device, and again whenever the device's
// context has changed since (after a cudaDeviceReset, for instance, the module
// is loaded anew at another address).  Under CUDA's lazy module loading that
// first call also loads the module and reserves the array, so it can fail with
// LA_ECUDA when the device's memory is already taken: make the first call (or
// load with CUDA_MODULE_LOADING=EAGER) before the application's allocator takes
// its budget, and before any stream capture.  All calls share the array and
// overwrite the part they use; calls that overlap on the GPU (different
// streams, or concurrent host threads) race on it.
//
// The op-level entry points (la_op_*) report a bounded wait that gave up in
// their kernels through one more file-scope word, g_op_err, which la_op_status
// reads and clears.
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

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
// First device error raised by an op-level kernel since la_op_status last read it.
static __device__ int g_op_err;

constexpr int kMaxDevices = 64;

struct DeviceSymbols {
  unsigned long long ctx_id = 0;   // context the addresses belong to (0: not set up)
  void* q_scaled = nullptr;
  int* op_err = nullptr;
};
std::mutex g_mu;
DeviceSymbols g_sym[kMaxDevices];

PFN_cuCtxGetCurrent_v4000 g_ctx_current = nullptr;
PFN_cuCtxGetId_v12000 g_ctx_id = nullptr;
std::once_flag g_ctx_once;

void resolve_ctx_api() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
  if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_ctx_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
  fn = nullptr;
  if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_ctx_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(fn);
}

// Unique id of the calling thread's current context, 0 if it cannot be told.
unsigned long long current_ctx_id() {
  std::call_once(g_ctx_once, resolve_ctx_api);
  if (!g_ctx_current || !g_ctx_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (g_ctx_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  if (g_ctx_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// q (bf16) times the softmax scale log2(e)/sqrt(d), rounded once to bf16.
__global__ void k_prescale_q(const __nv_bfloat16* __restrict__ q, __nv_bfloat16* __restrict__ out, long long n,
                             float scale) {
  for (long long i = blockIdx.x * static_cast<long long>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
    out[i] = __float2bfloat16_rn(__fmul_rn(__bfloat162float(q[i]), scale));
}

// Device addresses of the file-scope arrays on the current device: set up on
// the first use in a context, looked up again when the context changes.
int symbols_for_current_device(DeviceSymbols* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return LA_ECUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceSymbols& s = g_sym[dev];
  const unsigned long long id = current_ctx_id();
  if (!s.q_scaled || id == 0 || id != s.ctx_id) {
    void* p = nullptr;
    void* e = nullptr;
    cudaError_t r = cudaGetSymbolAddress(&p, g_q_scaled);
    if (r == cudaSuccess) r = cudaGetSymbolAddress(&e, g_op_err);
    if (r != cudaSuccess || !p || !e) {
      std::fprintf(stderr, "la_op: cudaGetSymbolAddress failed: %s\n", cudaGetErrorString(r));
      s = DeviceSymbols{};
      return LA_ECUDA;
    }
    s.q_scaled = p;
    s.op_err = static_cast<int*>(e);
    s.ctx_id = current_ctx_id();        // the lookup may have created the context
  }
  *out = s;
  return LA_OK;
}

}  // namespace

int op_error_word(int** out) {
  DeviceSymbols s;
  const int r = symbols_for_current_device(&s);
  *out = r == LA_OK ? s.op_err : nullptr;
  return r;
}

extern "C" int la_op_status(void* cuda_stream) {
  int* word = nullptr;
  int r = op_error_word(&word);
  if (r != LA_OK) return r;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(cuda_stream)) != cudaSuccess) return LA_ECUDA;
  int h = 0;
  if (cudaMemcpy(&h, word, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return LA_ECUDA;
  if (h == 0) return LA_OK;
  const int zero = 0;
  if (cudaMemcpy(word, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return LA_ECUDA;
  std::fprintf(stderr, "la_op: a kernel reported device error %d (%s)\n", h,
               h == LA_DEVERR_WAIT_TIMEOUT ? "a bounded wait gave up" : "bad descriptor");
  return LA_EDEVICE;
}

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
  DeviceSymbols sym;
  int r = symbols_for_current_device(&sym);
  if (r != LA_OK) return r;
  void* scratch = sym.q_scaled;
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
  p.err = sym.op_err;
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
