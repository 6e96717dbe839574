// Op-level C entry points: one kernel per call on a caller-given stream.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <string>

#include "kernels.h"
#include "la_stream.h"
#include "tmap.h"

namespace {
int num_sms_current() {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}
int ret(cudaError_t e) { return e == cudaSuccess ? LA_OK : LA_ECUDA; }
}  // namespace

extern "C" {

int la_op_gemm(int32_t dtype, int32_t epilogue, const void* A, const void* W, void* out, float* h32, int64_t M,
               int64_t N, int64_t K, const float* dt, int64_t rows_per_group, void* cuda_stream) {
  if (!A || !W || M < 1 || N < 1 || K < 1 || M > (1LL << 30) || N > (1LL << 30) || K > (1LL << 30)) return LA_EINVAL;
  if (epilogue < LA_EPI_STORE || epilogue > LA_EPI_STORE32) return LA_EINVAL;
  if ((epilogue == LA_EPI_STORE || epilogue == LA_EPI_STORE32) && !out) return LA_EINVAL;
  if (epilogue == LA_EPI_RESID && (!out || !h32)) return LA_EINVAL;
  if ((epilogue == LA_EPI_SET32 || epilogue == LA_EPI_EULER) && !h32) return LA_EINVAL;
  GemmEpiParams ep{};
  ep.kind = epilogue;
  ep.out = out;
  ep.h32 = h32;
  ep.ld = N;
  ep.rows_per_group = 1 << 30;
  for (int i = 0; i < LA_MAX_STEPS; ++i) ep.active[i] = 1;
  if (epilogue == LA_EPI_EULER) {
    if (!dt || rows_per_group < 1 || (M + rows_per_group - 1) / rows_per_group > LA_MAX_STEPS) return LA_EINVAL;
    ep.rows_per_group = static_cast<int>(rows_per_group);
    for (int i = 0; i < (M + rows_per_group - 1) / rows_per_group; ++i) ep.dt[i] = dt[i];
  }
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  if (dtype == LA_BF16) {
    if (N % 32 != 0 || K % 8 != 0) return LA_EINVAL;
    std::string err;
    if (!tmap_init(err)) return LA_ECUDA;
    const int bn = gemm_tc_pick_bn(static_cast<int>(N));
    CUtensorMap ta, tb;
    if (!tmap_2d_bf16(&ta, A, M, K, K, 128, err) || !tmap_2d_bf16(&tb, W, N, K, K, gemm_tc_b_box_rows(bn), err)) return LA_ECUDA;
    int* dev_err = nullptr;
    if (op_error_word(&dev_err) != LA_OK) return LA_ECUDA;
    return ret(launch_gemm_tc(ta, tb, ep, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), bn, dev_err,
                              num_sms_current(), st));
  }
  if (dtype != LA_FP32) return LA_EINVAL;
  return ret(launch_gemm_f32(static_cast<const float*>(A), static_cast<const float*>(W), ep, static_cast<int>(M),
                             static_cast<int>(N), static_cast<int>(K), st));
}

int la_op_attention(int32_t dtype, const void* q, int64_t Tq, int32_t H, int32_t d, int32_t nseg,
                    const void* const* k_seg, const void* const* v_seg, const int64_t* seg_len, void* out,
                    float* out32, int32_t q_scaled, void* cuda_stream) {
  if (!q || !out || !k_seg || !v_seg || !seg_len || Tq < 1 || Tq > (1 << 30) || H < 1 || H > 65535) return LA_EINVAL;
  if (nseg < 1 || nseg > LA_MAX_SEG || d < 8 || d > 128 || d % 8 != 0) return LA_EINVAL;
  for (int s = 0; s < nseg; ++s)
    if (!k_seg[s] || !v_seg[s] || seg_len[s] < 1 || seg_len[s] > (1 << 30)) return LA_EINVAL;
  AttnParams p{};
  p.ngroups = 1;
  p.Tq = static_cast<int>(Tq);
  p.H = H;
  p.d = d;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(d)));
  p.out = out;
  p.out32 = dtype == LA_BF16 ? out32 : nullptr;
  p.q_prescaled = (dtype == LA_BF16 && q_scaled) ? 1 : 0;
  p.out_ld = static_cast<long long>(H) * d;
  if (op_error_word(&p.err) != LA_OK) return LA_ECUDA;
  p.qbase = q;
  AttnGroup& g = p.g[0];
  g.nseg = nseg;
  g.q_slice = 0;
  g.out_row0 = 0;
  for (int s = 0; s < nseg; ++s) {
    g.seg[s] = AttnSeg{s, s, 0, 0, static_cast<int>(seg_len[s])};
    p.kbase[s] = k_seg[s];
    p.vbase[s] = v_seg[s];
    p.krows[s] = static_cast<int>(seg_len[s]);
    p.vrows[s] = static_cast<int>(seg_len[s]);
  }
  cudaStream_t st = static_cast<cudaStream_t>(cuda_stream);
  if (dtype == LA_BF16) {
    if (d != 128) return LA_EINVAL;
    std::string err;
    if (!tmap_init(err)) return LA_ECUDA;
    AttnMaps maps;
    if (!tmap_planes_bf16(&maps.q, q, d, Tq, H, 1, err)) return LA_ECUDA;
    for (int s = 0; s < nseg; ++s) {
      if (!tmap_planes_bf16(&maps.k[s], k_seg[s], d, seg_len[s], H, 1, err)) return LA_ECUDA;
      if (!tmap_planes_bf16(&maps.v[s], v_seg[s], d, seg_len[s], H, 1, err)) return LA_ECUDA;
    }
    return ret(launch_attention_tc(maps, p, st));
  }
  if (dtype != LA_FP32) return LA_EINVAL;
  return ret(launch_attn_f32(p, st));
}

int la_op_attention_fp8(const void* q_codes, int64_t Tq, int32_t H, int32_t d, int32_t nseg,
                        const void* const* k_seg, const void* const* v_seg, const int64_t* seg_len,
                        const float* q_scale, const float* k_scale, const float* v_scale, void* out, float* out32,
                        void* cuda_stream) {
  if (!q_codes || !out || !k_seg || !v_seg || !seg_len || !q_scale || !k_scale || !v_scale) return LA_EINVAL;
  if (Tq < 1 || Tq > (1 << 30) || H < 1 || H > 65535 || d != 128 || nseg < 1 || nseg > LA_MAX_SEG) return LA_EINVAL;
  for (int s = 0; s < nseg; ++s)
    if (!k_seg[s] || !v_seg[s] || seg_len[s] < 1 || seg_len[s] > (1 << 30)) return LA_EINVAL;
  AttnParams p{};
  p.ngroups = 1;
  p.Tq = static_cast<int>(Tq);
  p.H = H;
  p.d = d;
  p.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(d)));
  p.fp8 = 1;
  p.sq = q_scale;
  p.sk = k_scale;
  p.sv = v_scale;
  p.out = out;
  p.out32 = out32;
  p.out_ld = static_cast<long long>(H) * d;
  if (op_error_word(&p.err) != LA_OK) return LA_ECUDA;
  AttnGroup& g = p.g[0];
  g.nseg = nseg;
  for (int s = 0; s < nseg; ++s) g.seg[s] = AttnSeg{s, s, 0, 0, static_cast<int>(seg_len[s])};
  std::string err;
  if (!tmap_init(err)) return LA_ECUDA;
  AttnMaps maps;
  if (!tmap_planes_u8(&maps.q, q_codes, d, Tq, H, 1, err)) return LA_ECUDA;
  for (int s = 0; s < nseg; ++s) {
    if (!tmap_planes_u8(&maps.k[s], k_seg[s], d, seg_len[s], H, 1, err)) return LA_ECUDA;
    if (!tmap_planes_u8(&maps.v[s], v_seg[s], d, seg_len[s], H, 1, err)) return LA_ECUDA;
  }
  return ret(launch_attention_tc(maps, p, static_cast<cudaStream_t>(cuda_stream)));
}

int la_op_quantize_e4m3(int32_t in_dtype, const void* x, int64_t rows, int64_t cols, void* codes, float* scales,
                        void* cuda_stream) {
  if (!x || !codes || !scales || rows < 1 || rows > (1LL << 31) - 1 || cols < 2 || cols % 2 != 0) return LA_EINVAL;
  if (in_dtype != LA_BF16 && in_dtype != LA_FP32) return LA_EINVAL;
  return ret(launch_quant_rows_e4m3(in_dtype == LA_BF16, x, rows, cols, codes, scales,
                                    static_cast<cudaStream_t>(cuda_stream)));
}

int la_op_gemm_fp8(const void* a_codes, const float* a_scales, const void* w_codes, const float* w_scales, void* out,
                   int32_t out_dtype, int64_t M, int64_t N, int64_t K, void* cuda_stream) {
  if (!a_codes || !a_scales || !w_codes || !w_scales || !out) return LA_EINVAL;
  if (M < 1 || N < 32 || K < 16 || M > (1LL << 30) || N > (1LL << 30) || K > (1LL << 30)) return LA_EINVAL;
  if (N % 32 != 0 || K % 16 != 0) return LA_EINVAL;
  if (out_dtype != LA_BF16 && out_dtype != LA_FP32) return LA_EINVAL;
  std::string err;
  if (!tmap_init(err)) return LA_ECUDA;
  const int bn = gemm_tc_pick_bn(static_cast<int>(N));
  CUtensorMap ta, tb;
  if (!tmap_2d_u8(&ta, a_codes, M, K, K, 128, err) || !tmap_2d_u8(&tb, w_codes, N, K, K, bn, err)) return LA_ECUDA;
  GemmEpiParams ep{};
  ep.kind = out_dtype == LA_BF16 ? LA_EPI_STORE : LA_EPI_STORE32;
  ep.out = out;
  ep.ld = N;
  ep.rows_per_group = 1 << 30;
  for (int i = 0; i < LA_MAX_STEPS; ++i) ep.active[i] = 1;
  ep.row_scale = a_scales;
  ep.col_scale = w_scales;
  int* dev_err = nullptr;
  if (op_error_word(&dev_err) != LA_OK) return LA_ECUDA;
  return ret(launch_gemm_tc_fp8(ta, tb, ep, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), bn,
                                dev_err, num_sms_current(), static_cast<cudaStream_t>(cuda_stream)));
}

int la_op_euler(float* x, const float* v, int64_t rows, int64_t C, const float* dt, int64_t rows_per_group,
                void* cuda_stream) {
  if (!x || !v || !dt || rows < 1 || C < 4 || C % 4 != 0 || rows_per_group < 1) return LA_EINVAL;
  const int64_t groups = (rows + rows_per_group - 1) / rows_per_group;
  if (groups > LA_MAX_STEPS) return LA_EINVAL;
  float dts[LA_MAX_STEPS] = {};
  int act[LA_MAX_STEPS];
  for (int i = 0; i < LA_MAX_STEPS; ++i) act[i] = 1;
  for (int i = 0; i < groups; ++i) dts[i] = dt[i];
  return ret(launch_euler(x, v, rows, C, static_cast<int>(std::min<int64_t>(rows_per_group, 1 << 30)), dts, act,
                          nullptr, static_cast<cudaStream_t>(cuda_stream)));
}

}  // extern "C"
