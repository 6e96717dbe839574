// Internal definitions shared by the kernels and the host library.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "la_stream.h"

#define LA_MAX_SEG (LA_MAX_WINDOW + 2)
#define LA_MAX_PT 64          // temporal rotary pairs (head_dim <= 128)
#define LA_TROWS (LA_MAX_FPB + 1)

// Device error word codes (first error wins).
#define LA_DEVERR_WAIT_TIMEOUT 1
#define LA_DEVERR_BAD_DESC     2

// Per-pass description of the buffers: which blocks the grouped launch
// processes, in which timestep slot, and where their cache entries live.
struct PassDesc {
  int nbuf;                          // buffers covered by the row range (rows = nbuf*T)
  int nactive;                       // active buffers, listed in active_buf
  int active_buf[LA_MAX_STEPS];
  int active[LA_MAX_STEPS];          // per buffer: 1 if it runs a step this pass
  int slot[LA_MAX_STEPS];            // cache (ring slice) the buffer's block writes and reads itself from
  int win_slot[LA_MAX_STEPS];        // cache the buffer's prior (window) blocks are read from
  int step[LA_MAX_STEPS];            // denoising step of the pass (num_steps: a clean-cache refresh)
  int block[LA_MAX_STEPS];
  int write_entry[LA_MAX_STEPS];     // ring entry the block's K/V go to
  int nwin[LA_MAX_STEPS];            // prior blocks read, oldest first
  int win_entry[LA_MAX_STEPS][LA_MAX_WINDOW];
  int frame_tpos[LA_MAX_STEPS];      // RoPE time of the block's frame 0
  int sink_tpos[LA_MAX_STEPS];       // RoPE time of the sink for this block
  float dt[LA_MAX_STEPS];            // t_{i+1} - t_i of the buffer's slot
};

// One KV segment for attention: K from map kmap, V from map vmap (indices into
// the kernel's map arrays), each a stack of [H, rows, d] planes.
struct AttnSeg {
  int kmap, vmap;
  int kslice, vslice;   // outermost coordinate in the map (which [H, rows, d] plane)
  int len;              // keys
};

struct AttnGroup {
  int nseg;
  AttnSeg seg[LA_MAX_SEG];
  int q_slice;          // slice of the q map
  int out_row0;         // first output row of this group
};

#define LA_MAX_GROUPS LA_MAX_STEPS

struct AttnParams {
  int ngroups;
  AttnGroup g[LA_MAX_GROUPS];
  int Tq;               // queries per group
  int H, d;
  float scale_log2;     // log2(e) / sqrt(d)
  int q_prescaled;      // q already multiplied by scale_log2 (tcgen05 path)
  int fp8;              // q/K/V are e4m3 codes (tcgen05 path): value = code * scale of its head
  const float* sq;      // fp8: DEVICE [H] scales of q, K, V
  const float* sk;
  const float* sv;
  void* out;            // [rows, H*d] bf16 (tcgen05 path) / fp32 (SIMT path)
  float* out32;         // optional fp32 copy of the output (tcgen05 path)
  long long out_ld;     // elements per output row
  int* err;
  // raw pointers for the SIMT path: element offset of (slice, h, n, e) is
  // ((slice*H + h)*rows + n)*d + e, rows = krows/vrows[m] (q: Tq)
  const void* qbase;
  const void* kbase[LA_MAX_SEG];
  const void* vbase[LA_MAX_SEG];
  int krows[LA_MAX_SEG];
  int vrows[LA_MAX_SEG];
};

enum GemmEpi {
  EPI_STORE = 0, EPI_RESID = 1, EPI_SET32 = 2, EPI_EULER = 3, EPI_STORE32 = 4, EPI_QKV_ROPE = 5,
  EPI_RESID_GATED = 6,   // h32 += gate[row / rows_per_group][col] * acc; out (optional) = h32
  EPI_GELU = 7           // out = gelu_tanh(acc)
};

// QKV projection epilogue: rotate q and k (Rolling 3D RoPE) on the fp32
// accumulators, pre-multiply q by the softmax scale log2(e)/sqrt(d), and append
// K/V to the ring, rounding once to bf16.  Rows of inactive buffers are not written.
struct QkvRopeParams {
  int T, F, H, d, D, E, grid_w;
  int pt, ph;
  float qscale;              // log2(e)/sqrt(d)
  int active[LA_MAX_STEPS];
  int slot[LA_MAX_STEPS];
  int write_entry[LA_MAX_STEPS];
  long long ring_slice0;     // slice of (layer, slot 0, entry 0)
  const float* tcos; const float* tsin;   // [LA_MAX_STEPS][LA_TROWS][LA_MAX_PT]
  const float* rcos; const float* rsin;   // [grid_h][ph]
  const float* ccos; const float* csin;   // [grid_w][pw]
  // (cos, sin) of every pair of every token of the pass, [d/2][rowtab_ld] with
  // the grouped row (buffer * T + token) fastest, gathered once a pass from the
  // three tables above; NULL: the epilogue gathers from them itself
  const float2* rowtab;
  long long rowtab_ld;
  void* q_rope;              // [nbuf][H][T][d]
  void* ring_k; void* ring_v;// [L][S][E][H][T][d]
  const float* fp8_inv;      // NULL, or [3][H] inverse scales of q, K, V: write e4m3 codes of
                             // (roped) value * inverse scale instead of bf16 (q not pre-scaled)
};

struct GemmEpiParams {
  int kind;
  void* out;            // dtype [M, N]
  float* h32;           // fp32 [M, N]
  long long ld;         // N
  int rows_per_group;   // EULER: rows of one buffer
  float dt[LA_MAX_STEPS];
  int active[LA_MAX_STEPS];   // EULER: only active groups update
  float* vtap;          // optional fp32 [M, N] copy of acc (velocity capture)
  const float* row_scale;   // optional [M]: acc *= row_scale[row] * col_scale[col] first (FP8 operands)
  const float* col_scale;   // [N], set together with row_scale
  const float* gate[LA_MAX_STEPS];   // RESID_GATED: per row group, [N]
  // The per-token RMS norm folded into the GEMMs (n(h) W^T = diag(1 / rms(h)) (h W^T)):
  float* ssq_out;        // optional [M][ssq_ld]: each row's sum of squares of the new values over this
                         // tile's BN columns, at column-tile index (SET32 / RESID kinds)
  const float* ssq_in;   // optional [M][ssq_ld]: acc *= 1 / sqrt(sum_j ssq_in[row][j] / ssq_n + 1e-6) first
  int ssq_ld;            // partial sums a row (column tiles of the producing GEMM)
  float ssq_n;           // values a row the mean is over
};

// tanh-approximated GELU: u/2 (1 + tanh(sqrt(2/pi) (u + 0.044715 u^3))).
__device__ __forceinline__ float gelu_tanh(float u) {
  return 0.5f * u * (1.0f + tanhf(0.7978845608028654f * fmaf(0.044715f * u, u * u, u)));
}


static inline int ceil_div_i(long long a, long long b) { return (int)((a + b - 1) / b); }
