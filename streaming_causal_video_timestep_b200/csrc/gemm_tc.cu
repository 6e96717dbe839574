// C = A W^T on the 5th-generation tensor cores (tcgen05, accumulators in TMEM).
//
// Persistent kernel, one CTA per SM, 6 warps:
//   warp 0      TMA producer: A [128 x 128 B] and W [BN x 128 B] tiles per k-block
//               (64 bf16 or 128 e4m3 values a row), 128-byte swizzle, into a
//               STAGES-deep shared-memory ring;
//   warp 1      allocates TMEM (2 accumulators of BN fp32 columns) and, with one
//               thread, issues tcgen05.mma into the accumulator: kind::f16
//               128 x BN x 16 (bf16) or kind::f8f6f4 128 x BN x 32 (e4m3), four
//               per k-block (32 bytes of K each);
//   warps 2..5  epilogue: tcgen05.ld of the accumulator (warp w reads TMEM lanes
//               32*(w%4) .. +31 = tile rows), fused epilogue, global stores.
//               The residual and set epilogues move each 32 x 32 chunk of the
//               fp32 residual through a per-warp shared-memory stage, so that the
//               global loads and stores cover whole 128-byte row segments.  The
//               epilogues also carry the per-token RMS norm folded into the
//               GEMMs: the residual writers leave each row's sum of squares per
//               column tile, the QKV and head GEMMs scale rows by 1 / rms.
// The two accumulators let the epilogue of tile n overlap the main loop of n+1.
// 256-column bf16 tiles run on CTA pairs instead (k_gemm_pair below).
// Tiles are visited in bands of GROUP_M row-blocks so the A band and the W
// tiles in flight stay L2-resident.
#include <cuda_fp16.h>

#include "kernels.h"
#include "sm100.cuh"

namespace {

constexpr int BM = 128;
constexpr int BK_BYTES = 128;   // K bytes per k-block: one 128-byte swizzle row
constexpr int GROUP_M = 16;

// Per epilogue warp: a 32 x 32 fp32 chunk (4 KB) and its bf16 copy (2 KB).
constexpr uint32_t EPI_F32_BYTES = 32 * 32 * 4;
constexpr uint32_t EPI_WARP_BYTES = EPI_F32_BYTES + 32 * 32 * 2;

template <int BN>
struct GemmCfg {
  static constexpr int STAGES = BN == 256 ? 4 : (BN == 128 ? 6 : 8);
  static constexpr uint32_t A_BYTES = BM * BK_BYTES;
  static constexpr uint32_t B_BYTES = BN * BK_BYTES;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr uint32_t TMEM_COLS = 2 * BN;
  static constexpr size_t SMEM = 1024 /*align slack*/ + STAGES * STAGE_BYTES + 256 /*barriers*/ + 4 * EPI_WARP_BYTES;
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

__device__ __forceinline__ void tile_coords(int tile, int num_m, int num_n, int& m_blk, int& n_blk) {
  const int per_group = GROUP_M * num_n;
  const int group = tile / per_group;
  const int first_m = group * GROUP_M;
  const int gm = min(GROUP_M, num_m - first_m);
  const int local = tile - group * per_group;
  m_blk = first_m + local % gm;
  n_blk = local / gm;
}

__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const float* v) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 w;
    w.x = pack_bf16x2(v[8 * i + 0], v[8 * i + 1]);
    w.y = pack_bf16x2(v[8 * i + 2], v[8 * i + 3]);
    w.z = pack_bf16x2(v[8 * i + 4], v[8 * i + 5]);
    w.w = pack_bf16x2(v[8 * i + 6], v[8 * i + 7]);
    d4[i] = w;
  }
}

// Where one token (row) of the grouped QKV projection goes: its buffer, index in
// the block, frame and grid position.  Computed once per tile for each lane's
// row; the 32-column chunks of the row reuse it.
struct QkvRow {
  int buf, n, f, rr, ccol;
  bool active;
};

__device__ __forceinline__ QkvRow qkv_row_info(const QkvRopeParams& qp, long long row) {
  QkvRow q;
  const int r32 = static_cast<int>(row);   // rows of one grouped launch fit in int
  q.buf = r32 / qp.T;
  q.n = r32 - q.buf * qp.T;
  q.active = qp.active[q.buf] != 0;
  q.f = q.n / qp.F;
  const int rem = q.n - q.f * qp.F;
  q.rr = rem / qp.grid_w;
  q.ccol = rem - q.rr * qp.grid_w;
  return q;
}

// 32 consecutive columns of one head of the [q | k | v] projection of one token:
// rotate the pairs of q and k, scale q by log2(e)/sqrt(d), then pack bf16 for
// q_rope / the ring entry (or, with qp.fp8_inv, e4m3 codes of the unscaled
// values over the head's scale).  Returns the destination of the packed words
// (64 bytes of bf16 or 32 of e4m3), nullptr when the row's buffer is inactive.
__device__ __forceinline__ void* qkv_rope_words(const QkvRopeParams& qp, const QkvRow& qr, long long col,
                                                float (&acc)[32], uint32_t (&w)[16]) {
  if (!qr.active) return nullptr;
  const int c32 = static_cast<int>(col);
  const int part = c32 / qp.D;
  const int cc = c32 - part * qp.D;
  const int h = cc / qp.d, e0 = cc - h * qp.d;
  if (part < 2 && qp.rowtab) {
    // lanes are consecutive tokens: each pair's load is one contiguous run of (cos, sin)
    const float2* tab = qp.rowtab + static_cast<long long>(e0 >> 1) * qp.rowtab_ld +
                        (static_cast<long long>(qr.buf) * qp.T + qr.n);
#pragma unroll
    for (int jj = 0; jj < 16; ++jj) {
      const float2 cs = __ldg(tab + jj * qp.rowtab_ld);
      const float x0 = acc[2 * jj], x1 = acc[2 * jj + 1];
      acc[2 * jj] = x0 * cs.x - x1 * cs.y;
      acc[2 * jj + 1] = x0 * cs.y + x1 * cs.x;
    }
  } else if (part < 2) {
    const int pw_base = qp.pt + qp.ph;
#pragma unroll
    for (int jj = 0; jj < 16; ++jj) {
      const int j = (e0 >> 1) + jj;
      float c, sn;
      if (j < qp.pt) {
        const int idx = (qr.buf * LA_TROWS + qr.f) * LA_MAX_PT + j;
        c = qp.tcos[idx]; sn = qp.tsin[idx];
      } else if (j < pw_base) {
        const int idx = qr.rr * qp.ph + (j - qp.pt);
        c = qp.rcos[idx]; sn = qp.rsin[idx];
      } else {
        const int pw = qp.d / 2 - pw_base;
        const int idx = qr.ccol * pw + (j - pw_base);
        c = qp.ccos[idx]; sn = qp.csin[idx];
      }
      const float x0 = acc[2 * jj], x1 = acc[2 * jj + 1];
      acc[2 * jj] = x0 * c - x1 * sn;
      acc[2 * jj + 1] = x0 * sn + x1 * c;
    }
  }
  const long long tok = static_cast<long long>(qr.n) * qp.d + e0;
  long long base;
  if (part == 0) {
    base = (static_cast<long long>(qr.buf) * qp.H + h) * qp.T * qp.d;
  } else {
    const long long slice = qp.ring_slice0 + static_cast<long long>(qp.slot[qr.buf]) * qp.E + qp.write_entry[qr.buf];
    base = (slice * qp.H + h) * qp.T * qp.d;
  }
  void* plane = part == 0 ? qp.q_rope : (part == 1 ? qp.ring_k : qp.ring_v);
  if (qp.fp8_inv) {
    // e4m3 attention operands: codes of value / (the head's power-of-two scale)
    const float inv = qp.fp8_inv[part * qp.H + h];
#pragma unroll
    for (int k = 0; k < 8; ++k)
      w[k] = pack_e4m3x4(make_float2(acc[4 * k] * inv, acc[4 * k + 1] * inv),
                         make_float2(acc[4 * k + 2] * inv, acc[4 * k + 3] * inv));
    return static_cast<uint8_t*>(plane) + base + tok;
  }
  if (part == 0) {
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] *= qp.qscale;
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(acc[2 * i], acc[2 * i + 1]);
  return static_cast<__nv_bfloat16*>(plane) + base + tok;
}

// One row segment of WORDS 32-bit words per lane (16: 64 bytes, 8: 32 bytes) to
// dst (16-byte aligned; nullptr: this lane's row stores nothing).
__device__ __forceinline__ void store_row_words_direct(void* dst, const uint32_t* w, int words) {
  if (!dst) return;
  uint4* d4 = reinterpret_cast<uint4*>(dst);
  for (int q = 0; q < words / 4; ++q) d4[q] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
}

// The same for the whole warp through its shared-memory stage: lane t holds row
// t's words; the segments go out Q = WORDS / 4 lanes to a row (16 bytes each), so
// one store instruction covers 32 / Q rows with whole 32-byte sectors.  Each
// row's destination comes from its owner lane by shuffle.  The 16-byte slots are
// XOR-swizzled by row, so neither the row-wise writes nor the lane-group reads
// conflict on banks.
template <int WORDS>
__device__ __forceinline__ void store_row_words_staged(void* dst, const uint32_t* w, uint8_t* stage, int lane) {
  constexpr int Q = WORDS / 4;
  static_assert(Q == 4 || Q == 2, "64- or 32-byte row segments");
  uint4* sq = reinterpret_cast<uint4*>(stage);
  auto swz = [](int r) { return Q == 4 ? ((r >> 1) & 3) : ((r >> 2) & 1); };
  const int sw = swz(lane);
#pragma unroll
  for (int q = 0; q < Q; ++q) sq[lane * Q + (q ^ sw)] = make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
  __syncwarp();
  const unsigned long long d = reinterpret_cast<unsigned long long>(dst);
#pragma unroll
  for (int k = 0; k < Q; ++k) {
    const int r = k * (32 / Q) + lane / Q, q = lane % Q;
    const unsigned long long dr = __shfl_sync(0xffffffffu, d, r);
    if (dr) *reinterpret_cast<uint4*>(dr + 16ull * q) = sq[r * Q + (q ^ swz(r))];
  }
  __syncwarp();   // the next chunk rewrites the stage
}

// The epilogues that end in one packed row segment a row (bf16 store, GELU, the
// QKV RoPE/append): the destination and words of this lane's row, nullptr when
// it stores nothing.
__device__ __forceinline__ void* segment_words(const GemmEpiParams& ep, const QkvRopeParams& qp, const QkvRow& qr,
                                               long long row, long long col, float (&acc)[32], uint32_t (&w)[16]) {
  if (ep.kind == EPI_QKV_ROPE) return qkv_rope_words(qp, qr, col, acc, w);
  if (ep.kind == EPI_GELU) {
#pragma unroll
    for (int i = 0; i < 32; ++i) acc[i] = gelu_tanh(acc[i]);
  }
#pragma unroll
  for (int i = 0; i < 16; ++i) w[i] = pack_bf16x2(acc[2 * i], acc[2 * i + 1]);
  return reinterpret_cast<__nv_bfloat16*>(ep.out) + row * ep.ld + col;
}

// h32 (+)= [gate *] acc (SET: h32 = acc) for the 32 rows row0 .. row0+31 of one epilogue warp and
// the 32 columns col .. col+31 (all in range), plus the bf16 copy to ep.out.
// Lane t holds row t's values in acc.  The chunk passes through the warp's
// shared-memory stage: loaded and stored by lanes 8 to a 128-byte row segment
// (bf16: 4 to a 64-byte segment), combined by lanes one row each.  16-byte
// slots in the stage are XOR-swizzled by row, so neither access pattern has
// bank conflicts beyond the 4 wavefronts that 512 bytes take.
template <bool GATED, bool SET = false>
__device__ __forceinline__ void epilogue_resid_warp(const GemmEpiParams& ep, long long row0, long long col,
                                                   float (&acc)[32], uint8_t* stage, int lane) {
  float4* sf = reinterpret_cast<float4*>(stage);
  uint4* sb = reinterpret_cast<uint4*>(stage + EPI_F32_BYTES);
  const int sub = lane >> 3, ch = lane & 7;
  float4 gvs[8];
  if (GATED) {
    const float4* g4 = reinterpret_cast<const float4*>(ep.gate[(row0 + lane) / ep.rows_per_group] + col);
#pragma unroll
    for (int i = 0; i < 8; ++i) gvs[i] = __ldg(g4 + i);
  }
  if (!SET) {
    float4 hv[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int r = 4 * k + sub;
      hv[k] = *reinterpret_cast<const float4*>(ep.h32 + (row0 + r) * ep.ld + col + 4 * ch);
    }
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const int r = 4 * k + sub;
      sf[r * 8 + (ch ^ (r & 7))] = hv[k];
    }
    __syncwarp();
  }
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float4& slot = sf[lane * 8 + (c ^ (lane & 7))];
    float4 h;
    if (SET) {
      // the chunk is the new value itself (h32 = acc), staged only for the coalesced stores
      h = make_float4(acc[4 * c + 0], acc[4 * c + 1], acc[4 * c + 2], acc[4 * c + 3]);
    } else if (GATED) {
      h = slot;
      h.x = fmaf(gvs[c].x, acc[4 * c + 0], h.x);
      h.y = fmaf(gvs[c].y, acc[4 * c + 1], h.y);
      h.z = fmaf(gvs[c].z, acc[4 * c + 2], h.z);
      h.w = fmaf(gvs[c].w, acc[4 * c + 3], h.w);
    } else {
      h = slot;
      h.x += acc[4 * c + 0];
      h.y += acc[4 * c + 1];
      h.z += acc[4 * c + 2];
      h.w += acc[4 * c + 3];
    }
    slot = h;
    acc[4 * c + 0] = h.x;
    acc[4 * c + 1] = h.y;
    acc[4 * c + 2] = h.z;
    acc[4 * c + 3] = h.w;
  }
  if (ep.out) {
    const int sw = (lane >> 1) & 3;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint4 w;
      w.x = pack_bf16x2(acc[8 * c + 0], acc[8 * c + 1]);
      w.y = pack_bf16x2(acc[8 * c + 2], acc[8 * c + 3]);
      w.z = pack_bf16x2(acc[8 * c + 4], acc[8 * c + 5]);
      w.w = pack_bf16x2(acc[8 * c + 6], acc[8 * c + 7]);
      sb[lane * 4 + (c ^ sw)] = w;
    }
  }
  __syncwarp();
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int r = 4 * k + sub;
    *reinterpret_cast<float4*>(ep.h32 + (row0 + r) * ep.ld + col + 4 * ch) = sf[r * 8 + (ch ^ (r & 7))];
  }
  if (ep.out) {
    const int sub2 = lane >> 2, c2 = lane & 3;
    __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(ep.out);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int r = 8 * k + sub2;
      *reinterpret_cast<uint4*>(out + (row0 + r) * ep.ld + col + 8 * c2) = sb[r * 4 + (c2 ^ ((r >> 1) & 3))];
    }
  }
  __syncwarp();   // the next chunk rewrites the stage
}

// e4m3 operands: acc *= row_scale[row] * col_scale[col + i].  The 32 column
// scales of the chunk (the same for every lane) are read as 8 float4 through
// the read-only path when the array is 16-byte aligned (col is a multiple of
// 32), else one by one.
__device__ __forceinline__ void apply_operand_scales(const GemmEpiParams& ep, long long row, long long col,
                                                     float (&v)[32]) {
  const float rs = ep.row_scale[row];
  if ((reinterpret_cast<uintptr_t>(ep.col_scale) & 15) != 0) {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] *= rs * ep.col_scale[col + i];
    return;
  }
  const float4* c4 = reinterpret_cast<const float4*>(ep.col_scale + col);
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 c = __ldg(c4 + q);
    v[4 * q + 0] *= rs * c.x;
    v[4 * q + 1] *= rs * c.y;
    v[4 * q + 2] *= rs * c.z;
    v[4 * q + 3] *= rs * c.w;
  }
}

// The remaining epilogues, one lane per row (residual kinds on partial warps,
// fp32 stores, set, Euler update).
__device__ __forceinline__ void epilogue_row32(const GemmEpiParams& ep, long long row, long long col,
                                               float (&acc)[32]) {
  const long long off = row * ep.ld + col;
  switch (ep.kind) {
    case EPI_STORE32: {
      float4* o4 = reinterpret_cast<float4*>(reinterpret_cast<float*>(ep.out) + off);
#pragma unroll
      for (int i = 0; i < 8; ++i) o4[i] = make_float4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]);
      break;
    }
    case EPI_RESID: {
      float4* h4 = reinterpret_cast<float4*>(ep.h32 + off);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float4 h = h4[i];
        h.x += acc[4 * i + 0];
        h.y += acc[4 * i + 1];
        h.z += acc[4 * i + 2];
        h.w += acc[4 * i + 3];
        h4[i] = h;
        acc[4 * i + 0] = h.x;
        acc[4 * i + 1] = h.y;
        acc[4 * i + 2] = h.z;
        acc[4 * i + 3] = h.w;
      }
      if (ep.out) store_bf16x32(reinterpret_cast<__nv_bfloat16*>(ep.out) + off, acc);
      break;
    }
    case EPI_RESID_GATED: {
      // the gate chunk is read first, through the read-only path: loaded between the
      // stores to h32 (which the compiler cannot prove disjoint from it) each load
      // would wait on the store before it, about 9x slower
      const float4* g4 = reinterpret_cast<const float4*>(ep.gate[row / ep.rows_per_group] + col);
      float4 gvs[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) gvs[i] = __ldg(g4 + i);
      float4* h4 = reinterpret_cast<float4*>(ep.h32 + off);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 gv = gvs[i];
        float4 h = h4[i];
        h.x = fmaf(gv.x, acc[4 * i + 0], h.x);
        h.y = fmaf(gv.y, acc[4 * i + 1], h.y);
        h.z = fmaf(gv.z, acc[4 * i + 2], h.z);
        h.w = fmaf(gv.w, acc[4 * i + 3], h.w);
        h4[i] = h;
        acc[4 * i + 0] = h.x;
        acc[4 * i + 1] = h.y;
        acc[4 * i + 2] = h.z;
        acc[4 * i + 3] = h.w;
      }
      if (ep.out) store_bf16x32(reinterpret_cast<__nv_bfloat16*>(ep.out) + off, acc);
      break;
    }
    case EPI_SET32: {
      float4* h4 = reinterpret_cast<float4*>(ep.h32 + off);
#pragma unroll
      for (int i = 0; i < 8; ++i) h4[i] = make_float4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]);
      if (ep.out) store_bf16x32(reinterpret_cast<__nv_bfloat16*>(ep.out) + off, acc);
      break;
    }
    case EPI_EULER: {
      const int g = static_cast<int>(row / ep.rows_per_group);
      if (!ep.active[g]) break;
      const float dt = ep.dt[g];
      float4* x4 = reinterpret_cast<float4*>(ep.h32 + off);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float4 x = x4[i];
        x.x += dt * acc[4 * i + 0];
        x.y += dt * acc[4 * i + 1];
        x.z += dt * acc[4 * i + 2];
        x.w += dt * acc[4 * i + 3];
        x4[i] = x;
      }
      if (ep.vtap) {
        float4* v4 = reinterpret_cast<float4*>(ep.vtap + off);
#pragma unroll
        for (int i = 0; i < 8; ++i) v4[i] = make_float4(acc[4 * i], acc[4 * i + 1], acc[4 * i + 2], acc[4 * i + 3]);
      }
      break;
    }
  }
}

// Tensor-memory address of an epilogue warp's lane quarter in accumulator column col0.
__device__ __forceinline__ uint32_t tbase_of(uint32_t tmem, int quarter, int col0) {
  return tmem + (static_cast<uint32_t>(quarter * 32) << 16) + static_cast<uint32_t>(col0);
}

// The epilogue of one 128 x BN accumulator tile in tensor memory (tbase: this
// warp's lane quarter, column 0 of the tile) for rows row_base .. row_base+127
// and column block nb: one epilogue warp takes rows 32*quarter .. +31.
template <int BN>
__device__ __forceinline__ void epilogue_tile(const GemmEpiParams& ep, const QkvRopeParams& qp, int M, int N,
                                              uint32_t tbase, long long row_base, int nb, int quarter, int lane,
                                              uint8_t* epi_stage, bool staged_kind, bool segment_kind,
                                              bool seg_e4m3) {
  const int rit = quarter * 32 + lane;
  const long long row = row_base + rit;
  const long long row0 = row_base + quarter * 32;
  const bool staged = staged_kind && row0 + 32 <= M;
  QkvRow qr{};
  if (ep.kind == EPI_QKV_ROPE && row < M) qr = qkv_row_info(qp, row);
  // the row's RMS norm from the partial sums the producing GEMM left (folded norm)
  float inv_rms = 1.0f;
  if (ep.ssq_in && row < M) {
    float t = 0.f;
    for (int j = 0; j < ep.ssq_ld; ++j) t += ep.ssq_in[row * ep.ssq_ld + j];
    inv_rms = rsqrtf(t / ep.ssq_n + 1e-6f);
  }
  float ss = 0.f;              // sum of squares of the row's new values over this tile
#pragma unroll 1
  for (int c0 = 0; c0 < BN; c0 += 32) {
    uint32_t r[32];
    tmem_ld32(tbase + c0, r);
    tmem_ld_wait();
    const long long col = static_cast<long long>(nb) * BN + c0;
    if (segment_kind && col + 32 <= N) {
      float v[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]) * inv_rms;
      uint32_t w[16];
      void* dst = nullptr;
      if (row < M) {
        if (ep.row_scale) {
          apply_operand_scales(ep, row, col, v);
        }
        dst = segment_words(ep, qp, qr, row, col, v, w);
      }
      if (seg_e4m3)
        store_row_words_staged<8>(dst, w, epi_stage, lane);
      else
        store_row_words_staged<16>(dst, w, epi_stage, lane);
    } else if (staged && col + 32 <= N) {
      float v[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]) * inv_rms;
      if (ep.row_scale) {
        apply_operand_scales(ep, row, col, v);
      }
      if (ep.kind == EPI_RESID_GATED)
        epilogue_resid_warp<true>(ep, row0, col, v, epi_stage, lane);
      else if (ep.kind == EPI_SET32)
        epilogue_resid_warp<false, true>(ep, row0, col, v, epi_stage, lane);
      else
        epilogue_resid_warp<false>(ep, row0, col, v, epi_stage, lane);
      if (ep.ssq_out) {
#pragma unroll
        for (int i = 0; i < 32; ++i) ss = fmaf(v[i], v[i], ss);   // v now holds the row's new values
      }
    } else if (row < M && col < N) {
      float v[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]) * inv_rms;
      if (ep.row_scale) {
        apply_operand_scales(ep, row, col, v);
      }
      if (segment_kind) {
        uint32_t w[16];
        store_row_words_direct(segment_words(ep, qp, qr, row, col, v, w), w, seg_e4m3 ? 8 : 16);
      } else {
        epilogue_row32(ep, row, col, v);
        if (ep.ssq_out) {
#pragma unroll
          for (int i = 0; i < 32; ++i) ss = fmaf(v[i], v[i], ss);   // SET32 / RESID leave the new values in v
        }
      }
    }
  }
  if (ep.ssq_out && row < M) ep.ssq_out[row * ep.ssq_ld + nb] = ss;
}

template <int BN, bool FP8>
__global__ void __launch_bounds__(192, 1)
k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
          const __grid_constant__ GemmEpiParams ep, const __grid_constant__ QkvRopeParams qp, int M, int N, int K,
          int* err) {
  using C = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  __shared__ volatile int abort_flag;

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 4);   // one arrive per epilogue warp
    }
    mbar_init(drain, 1);
    fence_mbar_init();
    tma_prefetch_map(&tmA);
    tma_prefetch_map(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int num_m = (M + BM - 1) / BM;
  const int num_n = (N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;
  constexpr int BK = FP8 ? 128 : 64;   // K elements per k-block
  const int kblocks = (K + BK - 1) / BK;
  constexpr uint32_t idesc = FP8 ? idesc_e4m3(BM, BN) : idesc_bf16(BM, BN, false, false);

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int last_parity[C::STAGES];
      for (int i = 0; i < C::STAGES; ++i) last_parity[i] = -1;
      for (int tile = blockIdx.x; tile < num_tiles && !abort_flag; tile += gridDim.x) {
        int mb, nb;
        tile_coords(tile, num_m, num_n, mb, nb);
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, err)) { abort_flag = 1; break; }
          mbar_expect_tx(&full[stage], C::STAGE_BYTES);
          tma_load_2d(sA + stage * C::A_BYTES, &tmA, &full[stage], kb * BK, mb * BM);
          tma_load_2d(sB + stage * C::B_BYTES, &tmB, &full[stage], kb * BK, nb * BN);
          last_parity[stage] = static_cast<int>(phase);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
      }
      // Every issued load must have landed before the CTA exits: the phase a
      // load completes has already been observed by the MMA thread on the
      // normal path (this returns at once); after an abort it bounds the wait.
      for (int i = 0; i < C::STAGES; ++i)
        if (last_parity[i] >= 0) mbar_wait(&full[i], static_cast<uint32_t>(last_parity[i]), err);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
        if (abort_flag) break;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1, err)) { abort_flag = 1; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(acc * BN);
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&full[stage], phase, err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK_BYTES / 32; ++kk) {
            if (FP8)
              umma_e4m3_ss(d_tmem, sdesc_kmajor(a0 + kk * 32), sdesc_kmajor(b0 + kk * 32), idesc,
                           (kb | kk) != 0 ? 1u : 0u);
            else
              umma_bf16_ss(d_tmem, sdesc_kmajor(a0 + kk * 32), sdesc_kmajor(b0 + kk * 32), idesc,
                           (kb | kk) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
          if (++stage == C::STAGES) { stage = 0; phase ^= 1; }
        }
        if (!ok) { abort_flag = 1; break; }
        umma_commit(&tfull[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
      // all issued MMAs complete before TMEM is released
      umma_commit(drain);
      mbar_wait(drain, 0, err);
    }
  } else {
    const int quarter = warp & 3;
    uint8_t* epi_stage = smem + C::STAGES * C::STAGE_BYTES + 256 + (warp - 2) * EPI_WARP_BYTES;
    // the residual kinds and SET32 take the staged path when the warp's 32 rows are all in
    // range and h32 / out rows start on 16-byte boundaries
    const bool staged_kind = (ep.kind == EPI_RESID || ep.kind == EPI_RESID_GATED || ep.kind == EPI_SET32) &&
                             (ep.ld % 8) == 0 &&
                             (reinterpret_cast<uintptr_t>(ep.h32) & 15) == 0 &&
                             (reinterpret_cast<uintptr_t>(ep.out) & 15) == 0;
    // the kinds that end in one packed segment a row (64 bytes of bf16, or 32 of
    // e4m3 for the QKV epilogue of e4m3 attention) store through the stage
    const bool segment_kind = ep.kind == EPI_STORE || ep.kind == EPI_GELU || ep.kind == EPI_QKV_ROPE;
    const bool seg_e4m3 = ep.kind == EPI_QKV_ROPE && qp.fp8_inv != nullptr;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      if (abort_flag) break;
      int mb, nb;
      tile_coords(tile, num_m, num_n, mb, nb);
      if (!mbar_wait(&tfull[acc], acc_phase, err)) { abort_flag = 1; break; }
      tc_fence_after();
      epilogue_tile<BN>(ep, qp, M, N, tbase_of(tmem, quarter, acc * BN), static_cast<long long>(mb) * BM, nb,
                        quarter, lane, epi_stage, staged_kind, segment_kind, seg_e4m3);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// The same GEMM on CTA pairs (bf16, BN = 256): a cluster of two CTAs computes a
// 256 x BN tile with tcgen05.mma.cta_group::2 (M = 256), CTA r holding rows
// 128r .. 128r+127 of A and columns BN/2 r .. of W in its shared memory (the
// tensor cores exchange the W halves), so each CTA stages 16 KB of A and 16 KB
// of W a k-block and the ring is PAIR_STAGES deep in the same shared memory.
// Each CTA's tensor memory holds its 128 rows of the two BN-column
// accumulators, and its epilogue warps run epilogue_tile on them as above.
//   warp 0 (both CTAs)   TMA producer; the copies complete on the leader's
//                        (even CTA's) full[] barriers, which expect both CTAs'
//                        bytes (the cta_group::2 copy form, no multicast);
//   warp 1 (leader)      issues the MMAs; its commits release empty[] and
//                        tfull[] in both CTAs;
//   warps 2-5 (both)     epilogue; each warp hands its accumulator back on the
//                        leader's tempty[] (8 arrivals).
// Every wait is bounded; a wait that gives up raises the device error word and
// sets both CTAs' abort flags, and both CTAs meet at the final cluster barrier.
constexpr int PAIR_STAGES = 6;

template <int BN>
struct PairCfg {
  static constexpr uint32_t A_BYTES = BM * BK_BYTES;            // this CTA's 128 rows
  static constexpr uint32_t B_BYTES = (BN / 2) * BK_BYTES;      // this CTA's BN/2 columns
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr uint32_t TMEM_COLS = 2 * BN;
  static constexpr size_t SMEM = 1024 + PAIR_STAGES * STAGE_BYTES + 256 + 4 * EPI_WARP_BYTES;
  static_assert(SMEM <= 227 * 1024, "shared memory per CTA");
};

template <int BN>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(192, 1)
k_gemm_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
            const __grid_constant__ GemmEpiParams ep, const __grid_constant__ QkvRopeParams qp, int M, int N, int K,
            int* err) {
  using C = PairCfg<BN>;
  constexpr int ST = PAIR_STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + ST * C::A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + ST * C::STAGE_BYTES);
  uint64_t* empty = full + ST;
  uint64_t* tfull = empty + ST;
  uint64_t* tempty = tfull + 2;
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  __shared__ volatile int abort_flag;

  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = static_cast<int>(blockIdx.x >> 1), npairs = static_cast<int>(gridDim.x >> 1);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    abort_flag = 0;
    for (int i = 0; i < ST; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&tfull[i], 1);
      mbar_init(&tempty[i], 8);   // one arrive per epilogue warp of each CTA
    }
    mbar_init(drain, 1);
    fence_mbar_init();
    tma_prefetch_map(&tmA);
    tma_prefetch_map(&tmB);
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t abort_peer = smem_peer(const_cast<int*>(&abort_flag), rank ^ 1u);
  auto set_abort = [&]() {
    abort_flag = 1;
    st_cluster_u32(abort_peer, 1u);
  };

  const int num_m = (M + 2 * BM - 1) / (2 * BM);
  const int num_n = (N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;
  constexpr int BK = 64;
  const int kblocks = (K + BK - 1) / BK;
  constexpr uint32_t idesc = idesc_bf16(2 * BM, BN, false, false);

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int last_parity[ST];
      for (int i = 0; i < ST; ++i) last_parity[i] = -1;
      for (int tile = pair; tile < num_tiles && !abort_flag; tile += npairs) {
        int mb, nb;
        tile_coords(tile, num_m, num_n, mb, nb);
        const int arow = mb * 2 * BM + static_cast<int>(rank) * BM;
        const int brow = nb * BN + static_cast<int>(rank) * (BN / 2);
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, err)) { ok = false; break; }
          const uint32_t bar = smem_peer(&full[stage], 0);
          if (leader) mbar_expect_tx(&full[stage], 2 * C::STAGE_BYTES);
          tma_load_2d_pair(sA + stage * C::A_BYTES, &tmA, bar, kb * BK, arow);
          tma_load_2d_pair(sB + stage * C::B_BYTES, &tmB, bar, kb * BK, brow);
          last_parity[stage] = static_cast<int>(phase);
          if (++stage == ST) { stage = 0; phase ^= 1; }
        }
        if (!ok) { set_abort(); break; }
      }
      // the leader's full[] phases count both CTAs' bytes: every issued copy has
      // landed once they complete (at once on the normal path)
      if (leader)
        for (int i = 0; i < ST; ++i)
          if (last_parity[i] >= 0) mbar_wait(&full[i], static_cast<uint32_t>(last_parity[i]), err);
    }
  } else if (warp == 1) {
    if (leader && lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      for (int tile = pair; tile < num_tiles; tile += npairs) {
        if (abort_flag) break;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1, err)) { set_abort(); break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem + static_cast<uint32_t>(acc * BN);
        bool ok = true;
        for (int kb = 0; kb < kblocks; ++kb) {
          if (!mbar_wait(&full[stage], phase, err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a0 = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b0 = smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK_BYTES / 32; ++kk)
            umma_bf16_ss_pair(d_tmem, sdesc_kmajor(a0 + kk * 32), sdesc_kmajor(b0 + kk * 32), idesc,
                              (kb | kk) != 0 ? 1u : 0u);
          umma_commit_pair_mc(&empty[stage], 0x3);
          if (++stage == ST) { stage = 0; phase ^= 1; }
        }
        if (!ok) { set_abort(); break; }
        umma_commit_pair_mc(&tfull[acc], 0x3);
        if (++acc == 2) { acc = 0; acc_phase ^= 1; }
      }
      // all issued MMAs complete before either CTA releases its tensor memory
      umma_commit_pair(drain);
      mbar_wait(drain, 0, err);
    }
  } else {
    const int quarter = warp & 3;
    uint8_t* epi_stage = smem + ST * C::STAGE_BYTES + 256 + (warp - 2) * EPI_WARP_BYTES;
    const bool staged_kind = (ep.kind == EPI_RESID || ep.kind == EPI_RESID_GATED || ep.kind == EPI_SET32) &&
                             (ep.ld % 8) == 0 &&
                             (reinterpret_cast<uintptr_t>(ep.h32) & 15) == 0 &&
                             (reinterpret_cast<uintptr_t>(ep.out) & 15) == 0;
    const bool segment_kind = ep.kind == EPI_STORE || ep.kind == EPI_GELU || ep.kind == EPI_QKV_ROPE;
    const bool seg_e4m3 = ep.kind == EPI_QKV_ROPE && qp.fp8_inv != nullptr;
    const uint32_t tempty_leader = smem_peer(&tempty[0], 0);
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = pair; tile < num_tiles; tile += npairs) {
      if (abort_flag) break;
      int mb, nb;
      tile_coords(tile, num_m, num_n, mb, nb);
      if (!mbar_wait(&tfull[acc], acc_phase, err)) { set_abort(); break; }
      tc_fence_after();
      epilogue_tile<BN>(ep, qp, M, N, tbase_of(tmem, quarter, acc * BN),
                        static_cast<long long>(mb) * 2 * BM + static_cast<long long>(rank) * BM, nb, quarter, lane,
                        epi_stage, staged_kind, segment_kind, seg_e4m3);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (leader)
          mbar_arrive(&tempty[acc]);
        else
          mbar_arrive_remote(tempty_leader + acc * 8);
      }
      if (++acc == 2) { acc = 0; acc_phase ^= 1; }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync_all();          // the leader's MMAs into the follower's tensor memory are done
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, C::TMEM_COLS);
  }
}

template <int BN>
cudaError_t launch_pair(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmEpiParams& ep,
                        const QkvRopeParams& qp, int M, int N, int K, int* err, int num_sms, cudaStream_t st) {
  using C = PairCfg<BN>;
  auto kern = k_gemm_pair<BN>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(C::SMEM));
  if (e != cudaSuccess) return e;
  // persistent: as many pairs as can be resident at once (one CTA an SM), at most one a tile
  static int max_pairs = -1;
  if (max_pairs < 0) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3(2 * (num_sms / 2));
    cfg.blockDim = dim3(192);
    cfg.dynamicSmemBytes = C::SMEM;
    cudaLaunchAttribute attr{};
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    max_pairs = (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) == cudaSuccess && n > 0) ? n : num_sms / 2;
    cudaGetLastError();
  }
  const int tiles = ((M + 2 * BM - 1) / (2 * BM)) * ((N + BN - 1) / BN);
  const int pairs = tiles < max_pairs ? tiles : max_pairs;
  kern<<<2 * pairs, 192, C::SMEM, st>>>(tmA, tmB, ep, qp, M, N, K, err);
  return cudaGetLastError();
}

template <int BN, bool FP8>
cudaError_t launch_bn(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmEpiParams& ep,
                      const QkvRopeParams& qp, int M, int N, int K, int* err, int num_sms, cudaStream_t st) {
  using C = GemmCfg<BN>;
  cudaError_t e = cudaFuncSetAttribute(k_gemm_tc<BN, FP8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(C::SMEM));
  if (e != cudaSuccess) return e;
  const int tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const int grid = tiles < num_sms ? tiles : num_sms;
  k_gemm_tc<BN, FP8><<<grid, 192, C::SMEM, st>>>(tmA, tmB, ep, qp, M, N, K, err);
  return cudaGetLastError();
}

}  // namespace

int gemm_tc_b_box_rows(int bn) { return bn == 256 ? bn / 2 : bn; }

int gemm_tc_pick_bn(int N) {
  if (N % 256 == 0 && N >= 1024) return 256;
  if (N % 128 == 0) return 128;
  return 64;
}

cudaError_t launch_gemm_tc(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmEpiParams& ep, int M, int N,
                           int K, int bn, int* err, int num_sms, cudaStream_t st, const QkvRopeParams* qp) {
  QkvRopeParams none{};
  const QkvRopeParams& q = qp ? *qp : none;
  switch (bn) {
    case 256: return launch_pair<256>(tmA, tmB, ep, q, M, N, K, err, num_sms, st);
    case 128: return launch_bn<128, false>(tmA, tmB, ep, q, M, N, K, err, num_sms, st);
    default: return launch_bn<64, false>(tmA, tmB, ep, q, M, N, K, err, num_sms, st);
  }
}

cudaError_t launch_gemm_tc_fp8(const CUtensorMap& tmA, const CUtensorMap& tmB, const GemmEpiParams& ep, int M,
                               int N, int K, int bn, int* err, int num_sms, cudaStream_t st, const QkvRopeParams* qp) {
  if (!ep.row_scale || !ep.col_scale) return cudaErrorInvalidValue;
  QkvRopeParams none{};
  const QkvRopeParams& q = qp ? *qp : none;
  switch (bn) {
    case 256: return launch_bn<256, true>(tmA, tmB, ep, q, M, N, K, err, num_sms, st);
    case 128: return launch_bn<128, true>(tmA, tmB, ep, q, M, N, K, err, num_sms, st);
    default: return launch_bn<64, true>(tmA, tmB, ep, q, M, N, K, err, num_sms, st);
  }
}
