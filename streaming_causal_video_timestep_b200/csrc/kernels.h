// Host-side launchers of the library's kernels (internal).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"

// Device address of the op-level error word on the current device (la_static.cu;
// read and cleared by la_op_status).  Returns LA_OK or LA_ECUDA.
int op_error_word(int** out);

// ---- tcgen05 (bf16) ----------------------------------------------------------------
int gemm_tc_pick_bn(int N);
// Rows of the W box of a bf16 tensor map for launch_gemm_tc with that bn: the
// bn = 256 tiles run on CTA pairs, each CTA loading half of the tile's W rows.
int gemm_tc_b_box_rows(int bn);
// qp: parameters of the EPI_QKV_ROPE epilogue (NULL for the others).
cudaError_t launch_gemm_tc(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmEpiParams& ep, int M, int N,
                           int K, int bn, int* err, int num_sms, cudaStream_t st, const QkvRopeParams* qp = nullptr);

// The same GEMM on e4m3 operands (kind::f8f6f4; tmA / tmB from tmap_2d_u8 with
// box rows 128 / bn); ep.row_scale / ep.col_scale are required and multiply the
// fp32 accumulator before the epilogue.
cudaError_t launch_gemm_tc_fp8(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmEpiParams& ep, int M,
                               int N, int K, int bn, int* err, int num_sms, cudaStream_t st,
                               const QkvRopeParams* qp = nullptr);
// Per-row e4m3 quantization of x (bf16 if bf16_in, else fp32) [rows, cols]:
// q uint8 [rows, cols], scale fp32 [rows] = amax / 448 (1 for a zero row).
cudaError_t launch_quant_rows_e4m3(int bf16_in, const void* x, long long rows, long long cols, void* q,
                                   float* scale, cudaStream_t st);
// Per-head power-of-two scales of the e4m3 attention operands of one layer.
// For output row j of the QKV weight w ([3D, D], bf16, or e4m3 codes with
// per-row scales w_rowscale when w_fp8) the bound on |value| is
//   act_bound * ||w_j||              (V rows),
//   act_bound * ||(w_2m, w_2m+1)||   (q / K rows of rotary pair m: RoPE mixes the pair),
// and scale[part][h] = 2^ceil(log2(max over the head's rows of the bound / 448))
// (1 when the bound is 0); inv = 1 / scale.  Row norms are fp32 sums.
cudaError_t launch_attn_fp8_scales(const void* w, int w_fp8, const float* w_rowscale, int D, int H, int d,
                                   float act_bound, float* scale, float* inv, cudaStream_t st);

// Tensor maps of an attention launch: q (d, Tq, H, q slices) and k[m]/v[m]
// (d, rows_m, H, slices), 128-byte swizzle: bf16 with box (64, 128, 1, 1), or
// e4m3 codes (p.fp8) with box (128, 128, 1, 1).
struct AttnMaps {
  CUtensorMap q;
  CUtensorMap k[LA_MAX_SEG];
  CUtensorMap v[LA_MAX_SEG];
};
// Block-causal attention over the segments of each group (two 128-query tiles
// per CTA).  LA_ATTN_EMU=k in the environment (k in {0, 2, 3, 4}; default 0)
// computes k of every 8 exponential pairs of full key tiles on the FMA pipe.
// p.fp8: e4m3 q/K/V with per-head scales p.sq / p.sk / p.sv (kind::f8f6f4).
cudaError_t launch_attention_tc(const AttnMaps& maps, const AttnParams& p, cudaStream_t st);

// ---- SIMT fp32 -----------------------------------------------------------------------
cudaError_t launch_gemm_f32(const float* A, const float* W, const GemmEpiParams& ep, int M, int N, int K,
                            cudaStream_t st);
cudaError_t launch_attn_f32(const AttnParams& p, cudaStream_t st);

// ---- bandwidth kernels (templated on the activation type) -----------------------------
// Temporal RoPE table of a pass: cos/sin of (pos * omega_t[j]) for every active
// buffer and each of frames_per_block frames plus the sink row (index fpb).
cudaError_t launch_rope_ttab(const PassDesc& pd, int fpb, int pt, const double* omega_t, float* tcos, float* tsin,
                             cudaStream_t st);

struct RopeArgs;
// The per-token RoPE table of a pass for the QKV epilogue: (cos, sin) of every
// pair j < d/2 of every token of every active buffer into out[j * ld + buf * T +
// token], gathered from the pass's temporal table and the height / width tables.
cudaError_t launch_rope_rows(const PassDesc& pd, const RopeArgs& a, float2* out, long long ld, cudaStream_t st);

struct RopeArgs {
  int T, F, H, d, D, grid_w, fpb;
  int pt, ph, pw;
  const float* tcos;  const float* tsin;       // [LA_MAX_STEPS][LA_TROWS][LA_MAX_PT]
  const float* rcos;  const float* rsin;       // [grid_h][ph]
  const float* ccos;  const float* csin;       // [grid_w][pw]
  const void* qkv;                             // fp32 [nbuf*T, 3D]
  void* q_rope;                                // [nbuf][H][T][d]
  void* ring_k; void* ring_v;                  // [L][S][E][H][T][d]
  long long ring_slice0;                       // (layer*S) * E: slice of (layer, slot 0, entry 0)
  int E;
  const void* sink_k;                          // fp32 un-roped [nl][H][F][d] from the first layer (NULL: no sink part)
  void* sink_k_rope;                           // [nl][nb][H][F][d]
  const float* fp8_inv;                        // [nl][3][H] inverse e4m3 scales of q, K, V (e4m3 outputs)
  int nl = 1;                                  // layers of one sink re-rope launch
  int nb = 1;                                  // buffers of sink_k_rope a layer
};
// Rolling RoPE + ring append of every active buffer's block from the fp32 qkv
// (fp32 streams; bf16 streams do it in the QKV GEMM epilogue).  Outputs are
// bf16 (bf16_out) or fp32.
cudaError_t launch_rope_append(int bf16_out, const PassDesc& pd, const RopeArgs& a, cudaStream_t st);
// Re-rope of the fp32 un-roped sink K of a.nl layers at every active buffer's
// sink position (a.sink_k[l] -> a.sink_k_rope[l][buf]), one launch.  out_kind:
// 0 fp32, 1 bf16, 2 e4m3 codes of value * a.fp8_inv[l][H + head].
cudaError_t launch_sink_rerope(int out_kind, const PassDesc& pd, const RopeArgs& a, cudaStream_t st);

// Sink pass: split the fp32 qkv [F, 3D] into the layer's fp32 un-roped K, its
// V, and roped q / k (temporal row 0 of buffer 0 of the table); q is
// multiplied by qscale (the softmax scale on the bf16 path, 1 on fp32).
// sink_v8 (optional, [H][F][d] uint8): e4m3 codes of V * a.fp8_inv[2H + head]
// from the fp32 projection, for e4m3 attention.
cudaError_t launch_sink_qkv(int bf16_out, const RopeArgs& a, float qscale, float* sink_k_raw, void* sink_v,
                            void* q_rope, void* k_rope, cudaStream_t st, uint8_t* sink_v8 = nullptr);

// x (fp32 [rows, C]) -> h32 (fp32) and hop (dtype) when C == D (identity in-proj),
// or -> xop (bf16) for the in-projection GEMM.
cudaError_t launch_in_identity(int bf16, const float* x, float* h32, void* hop, long long n, cudaStream_t st);
cudaError_t launch_cvt_bf16(const float* x, void* xb, long long n, cudaStream_t st);
// x[r, :] += dt[g] * v[r, :], g = r / rows_per_group, for active groups.
cudaError_t launch_euler(float* x, const float* v, long long rows, long long C, int rows_per_group,
                         const float* dt, const int* active, float* vtap, cudaStream_t st);

// out = h / sqrt(mean(h^2) + eps) per row of D fp32 values (D % 4 == 0), written
// as bf16 (out_bf16) and / or fp32 (out_f32).
cudaError_t launch_rmsnorm(const float* h, long long rows, long long D, float eps, void* out_bf16, float* out_f32,
                           cudaStream_t st);

// Token-major fp32 src [rows, src_ld], columns col0 + h*d + e, to head-major
// planes dst [rows / rows_per_slice][H][rows_per_slice][d] times scale, bf16
// (bf16_out) or fp32.  d % 8 == 0, src_ld and col0 multiples of 4.
cudaError_t launch_split_heads(int bf16_out, const float* src, long long rows, int rows_per_slice, int H, int d,
                               long long src_ld, long long col0, void* dst, float scale, cudaStream_t st);

// AdaLN vectors of each row group (buffer) for the modulated norm.
struct ModArgs {
  int rows_per_group;
  const float* shift[LA_MAX_STEPS];   // [D] each
  const float* scale[LA_MAX_STEPS];
};
// out = rms-normalised h * (1 + scale[row / rows_per_group]) + shift[...], bf16 and / or fp32.
cudaError_t launch_rmsnorm_mod(const float* h, long long rows, long long D, float eps, const ModArgs& m,
                               void* out_bf16, float* out_f32, cudaStream_t st);
