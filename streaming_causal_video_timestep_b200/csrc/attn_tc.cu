// Block-causal attention, tcgen05, head_dim 128, two query tiles per CTA,
// softmax with the scores of a row held in registers.
//
// One CTA = up to 256 queries (two 128-row tiles A and B) of one (group, head),
// sharing every K/V tile of the group's segments [sink | window | block].
// 12 warps in three warpgroups:
//   warpgroup 0  warp 0: TMA producer (Q_A, Q_B once, then one ring stage
//                [V(p-1) | K(p)] per key-tile step p, each tile as two
//                64-column 128-byte-swizzled boxes: a 2-stage ring for bf16,
//                4 stages for e4m3, see kv_stages());
//                warp 1: TMEM owner (512 columns: S_A | S_B | O_A | O_B) and
//                MMA issuer (the whole warp waits, one elected lane issues);
//                warps 2-3 idle.  Drops to 56 registers a thread.
//   warpgroup 1  softmax of tile A, warpgroup 2 softmax of tile B: one thread
//                per query row (= TMEM lane).  Raised to 224 registers a thread
//                so that a row's 128 scores of a key tile stay in registers
//                (one tensor-memory read per tile).
// Per key tile t the tensor core runs, in issue order,
//   ... PV_A(t-1), S_A(t), PV_B(t-1), S_B(t) ...
// so while one softmax warpgroup turns S into P the tensor core works on the
// other tile.  P is written as bf16 into the first 64 columns of its own S
// tile (tcgen05.st) and read from there as the A operand of O += P V
// (tcgen05.mma with A in tensor memory); V is read MN-major from its [keys, d]
// tile.
// Scores are in the log2 domain (q pre-multiplied by log2(e)/sqrt(d) when
// PRESCALED, else scaled here first), so the row maximum contributes exactly
// 2^0 = 1.  The running max is updated lazily: O is rescaled in TMEM only when
// the max grows by more than 2^8.
//
// The exponentials: at 16 ex2 per clock per SM the special-function unit needs
// as many cycles for the 128 x 128 exponentials of a tile pair as the tensor
// core needs for its two 128 x 128 x 128 products, so on full key tiles EMU of
// every 8 column pairs are computed on the FMA pipe instead (exp2_poly2 below:
// Cody-Waite split into integer and fraction, as in the FlashAttention-4
// softmax, with a polynomial of our own fit).  Partial tiles (a segment's
// ragged tail) use ex2 only, so masked keys get exactly 0.
//
// FP8 variant (the FP8 template argument): q, K and V are e4m3 codes with one
// scale per head each, S = Q K^T and O += P V run as kind::f8f6f4 (32 keys or
// dims a tensor-core step; one 128-byte box per 128 x 128 tile), and P is
// written to tensor memory as e4m3 (32 columns).  The scores enter the softmax
// as acc * (sq * sk * log2(e)/sqrt(d)); the running max M is kept as a whole
// number (the tile max rounded up) and P = 2^(s - M + FP8_P_BIAS), so a row's
// largest P lies in (16, 32] when M is set and P stays below 2^(FP8_TAU +
// FP8_P_BIAS) = 256 < 448 until the max grows by more than FP8_TAU.  With M a
// whole number, a later rescale of O multiplies earlier P codes by an exact
// power of two, so the codes are those of P formed against the final row max
// wherever they are normal e4m3 values.  The normaliser sums the unrounded P.
#include <cstdio>
#include <cstdlib>

#include "kernels.h"
#include "sm100.cuh"

namespace {

constexpr int BQ = 128;
constexpr int BKV = 128;
constexpr int THREADS = 384;
constexpr int LAUNCH_REGS = 168;            // 65536 / 384 rounded down to the allocation unit of 8
constexpr int REGS_LOW = 56;                // warpgroup 0 after setmaxnreg.dec
constexpr int REGS_HIGH = 224;              // warpgroups 1-2 after setmaxnreg.inc
static_assert(128 * REGS_LOW + 256 * REGS_HIGH <= THREADS * LAUNCH_REGS, "register split exceeds the launch");
constexpr uint32_t HALF = 16384;            // 128 rows x 128 bytes, one swizzle-128B box
constexpr uint32_t TMEM_COLS = 512;
constexpr float FP8_P_BIAS = 5.0f;
constexpr float FP8_TAU = 3.0f;

// A 128 x 128 tile: two boxes of 64 bf16 columns, or one box of 128 e4m3 columns.
template <bool FP8> __host__ __device__ constexpr uint32_t tile_bytes() { return FP8 ? HALF : 2 * HALF; }
// The K/V ring holds one key-tile step per stage: stage of step p = [V(p-1) | K(p)]
// (step 0: K(0) only; step nt: V(nt-1) only), under one full and one empty barrier.
template <bool FP8> __host__ __device__ constexpr int kv_stages() { return FP8 ? 4 : 2; }
template <bool FP8> __host__ __device__ constexpr size_t smem_bytes() {
  return 1024 + 2 * tile_bytes<FP8>() /*Q_A, Q_B*/ + kv_stages<FP8>() * 2 * tile_bytes<FP8>() /*ring*/ + 256;
}

__device__ __forceinline__ uint32_t s_col(int w) { return static_cast<uint32_t>(w * 128); }
__device__ __forceinline__ uint32_t o_col(int w) { return static_cast<uint32_t>(256 + w * 128); }

struct SegCursor {
  int seg = 0, start = 0;
  __device__ void next(const AttnGroup& g) {
    start += BKV;
    if (start >= g.seg[seg].len) { ++seg; start = 0; }
  }
};

__device__ __forceinline__ int group_tiles(const AttnGroup& g) {
  int n = 0;
  for (int s = 0; s < g.nseg; ++s) n += (g.seg[s].len + BKV - 1) / BKV;
  return n;
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

template <int N>
__device__ __forceinline__ void regs_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N)); }
template <int N>
__device__ __forceinline__ void regs_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N)); }

// 2^x for a pair, x in (-inf, 9): clamp at -125 (2^-125 ~ 2e-38, so the result
// is a normal float), split x = j + f with j = round(x) by adding and removing
// 1.5 * 2^23 (|f| <= 1/2, exact), approximate 2^f by
//   p(f) = 1 + f (c1 + f (c2 + f c3)),
// the degree-3 polynomial with p(0) = 1 of least maximum relative error on
// [-1/2, 1/2] (fit by iteratively reweighted least squares; max relative error
// 1.0e-4 in fp32, 19x below half a bf16 ulp), and add j to its exponent field:
// the low bits of (x + 1.5 * 2^23) hold j, so (bits << 23) is j << 23 mod 2^32.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  constexpr float kShift = 12582912.0f;   // 1.5 * 2^23
  constexpr float c1 = 0.6932829022407532f, c2 = 0.2422107458114624f, c3 = 0.055008791387081146f;
  x.x = fmaxf(x.x, -125.0f);
  x.y = fmaxf(x.y, -125.0f);
  const float2 t = __fadd2_rn(x, make_float2(kShift, kShift));
  const float2 j = __fadd2_rn(t, make_float2(-kShift, -kShift));
  const float2 f = __ffma2_rn(j, make_float2(-1.0f, -1.0f), x);
  float2 p = __ffma2_rn(f, make_float2(c3, c3), make_float2(c2, c2));
  p = __ffma2_rn(p, f, make_float2(c1, c1));
  p = __ffma2_rn(p, f, make_float2(1.0f, 1.0f));
  return make_float2(__int_as_float(__float_as_int(p.x) + (__float_as_int(t.x) << 23)),
                     __int_as_float(__float_as_int(p.y) + (__float_as_int(t.y) << 23)));
}

// One row's pass over the 128 scores of a key tile held in s[]: row max (masked
// beyond `valid` when MASKED), lazy max update, P = 2^(s - m) into P[] (bf16
// pairs), returns the tile's row sum of the unrounded P; m_ref / alpha / need
// are updated for the caller.
template <bool MASKED, int EMU>
__device__ __forceinline__ float softmax_tile(float (&s)[128], uint32_t (&P)[64], int valid, float& m_ref,
                                              float& alpha, bool& need) {
  if (MASKED) {
#pragma unroll
    for (int i = 0; i < 128; ++i)
      if (i >= valid) s[i] = -INFINITY;
  }
  float mx[4];
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    float a = fmax3(s[32 * c], s[32 * c + 1], s[32 * c + 2]);
#pragma unroll
    for (int i = 3; i + 1 < 32; i += 2) a = fmax3(a, s[32 * c + i], s[32 * c + i + 1]);
    mx[c] = fmaxf(a, s[32 * c + 31]);
  }
  const float m_tile = fmaxf(fmax3(mx[0], mx[1], mx[2]), mx[3]);
  need = m_tile > m_ref + 8.0f;
  const float m_new = need ? m_tile : m_ref;
  alpha = need ? fast_exp2(m_ref - m_new) : 1.0f;
  m_ref = m_new;
  const float2 negm = make_float2(-m_new, -m_new);
  float2 acc[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) acc[u] = make_float2(0.f, 0.f);
#pragma unroll
  for (int i = 0; i < 64; ++i) {
    const float2 x = __fadd2_rn(make_float2(s[2 * i], s[2 * i + 1]), negm);
    float2 p;
    if (!MASKED && (i & 7) >= 8 - EMU) {
      p = exp2_poly2(x);
    } else {
      p.x = fast_exp2(x.x);
      p.y = fast_exp2(x.y);
    }
    acc[i & 3] = __fadd2_rn(acc[i & 3], p);
    P[i] = pack_bf16x2(p.x, p.y);
  }
  const float2 a01 = __fadd2_rn(acc[0], acc[1]), a23 = __fadd2_rn(acc[2], acc[3]);
  const float2 a = __fadd2_rn(a01, a23);
  return a.x + a.y;
}

// The FP8 form: s[] holds the raw accumulators q_code . k_code; c = sq * sk *
// log2(e)/sqrt(d) maps them to the log2 domain.  M (m_ref) is a whole number;
// P = 2^(s c - M + FP8_P_BIAS) as e4m3 codes, four to a 32-bit word (key 4i+b
// in byte b of P[i]); returns the tile's row sum of the unrounded P.  On full
// tiles EMU of every 8 pairs take the polynomial exp2 on the FMA pipe.
template <bool MASKED, int EMU>
__device__ __forceinline__ float softmax_tile_fp8(float (&s)[128], uint32_t (&P)[32], int valid, float c,
                                                  float& m_ref, float& alpha, bool& need) {
  if (MASKED) {
#pragma unroll
    for (int i = 0; i < 128; ++i)
      if (i >= valid) s[i] = -INFINITY;
  }
  float mx[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float a = fmax3(s[32 * q], s[32 * q + 1], s[32 * q + 2]);
#pragma unroll
    for (int i = 3; i + 1 < 32; i += 2) a = fmax3(a, s[32 * q + i], s[32 * q + i + 1]);
    mx[q] = fmaxf(a, s[32 * q + 31]);
  }
  const float m_tile = fmaxf(fmax3(mx[0], mx[1], mx[2]), mx[3]) * c;
  need = m_tile > m_ref + FP8_TAU;
  const float m_new = need ? ceilf(m_tile) : m_ref;
  alpha = need ? fast_exp2(m_ref - m_new) : 1.0f;
  m_ref = m_new;
  const float2 cc = make_float2(c, c);
  const float2 off = make_float2(FP8_P_BIAS - m_new, FP8_P_BIAS - m_new);
  float2 acc[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) acc[u] = make_float2(0.f, 0.f);
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    float2 pp[2];
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const int j = 2 * i + h2;              // pair index 0..63
      const float2 x = __ffma2_rn(make_float2(s[2 * j], s[2 * j + 1]), cc, off);
      if (!MASKED && (j & 7) >= 8 - EMU) {
        pp[h2] = exp2_poly2(x);
      } else {
        pp[h2] = make_float2(fast_exp2(x.x), fast_exp2(x.y));
      }
      acc[j & 3] = __fadd2_rn(acc[j & 3], pp[h2]);
    }
    P[i] = pack_e4m3x4(pp[0], pp[1]);
  }
  const float2 a01 = __fadd2_rn(acc[0], acc[1]), a23 = __fadd2_rn(acc[2], acc[3]);
  const float2 a = __fadd2_rn(a01, a23);
  return a.x + a.y;
}

template <bool PRESCALED, int EMU, bool FP8>
__global__ void __launch_bounds__(THREADS, 1)
k_attn_tc(const __grid_constant__ AttnMaps maps, const __grid_constant__ AttnParams p) {
  constexpr uint32_t TILE = tile_bytes<FP8>();
  constexpr int NS = kv_stages<FP8>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                       // Q_A at 0, Q_B at TILE
  uint8_t* sKV = smem + 2 * TILE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + NS * 2 * TILE);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + NS;
  uint64_t* s_full = kv_empty + NS;         // [2]
  uint64_t* p_full = s_full + 2;            // [2]
  uint64_t* pv_done = p_full + 2;           // [2]
  uint64_t* drain = pv_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  __shared__ volatile int abort_flag;

  const AttnGroup& g = p.g[blockIdx.z];
  const int h = blockIdx.y;
  const int q0 = blockIdx.x * 2 * BQ;
  const int nq = (q0 + BQ < p.Tq) ? 2 : 1;  // query tiles of this CTA
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  int* err = p.err;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(q_full, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(&s_full[w], 1);
      mbar_init(&p_full[w], 4);
      mbar_init(&pv_done[w], 1);
    }
    mbar_init(drain, 1);
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nt = group_tiles(g);

  if (warp < 4) {
    regs_dec<REGS_LOW>();
    if (warp == 0 && lane == 0) {
      // -------------------------------------------------------------- producer
      int last_parity[NS];
      for (int i = 0; i < NS; ++i) last_parity[i] = -1;
      mbar_expect_tx(q_full, 2 * TILE);
      for (int w = 0; w < 2; ++w) {
        tma_load_4d(sQ + w * TILE, &maps.q, q_full, 0, q0 + w * BQ, h, g.q_slice);
        if (!FP8) tma_load_4d(sQ + w * TILE + HALF, &maps.q, q_full, 64, q0 + w * BQ, h, g.q_slice);
      }
      // step p of the ring: V(p-1) at the stage's start, K(p) one tile further
      SegCursor ck, cv;
      for (int p = 0; p <= nt && !abort_flag; ++p) {
        const int stage = p % NS;
        const uint32_t par = static_cast<uint32_t>((p / NS) & 1);
        if (!mbar_wait(&kv_empty[stage], par ^ 1, err)) { abort_flag = 1; break; }
        const bool has_v = p >= 1, has_k = p < nt;
        uint8_t* dst = sKV + stage * 2 * TILE;
        mbar_expect_tx(&kv_full[stage], (has_v ? TILE : 0u) + (has_k ? TILE : 0u));
        if (has_v) {
          const AttnSeg& sg = g.seg[cv.seg];
          tma_load_4d(dst, &maps.v[sg.vmap], &kv_full[stage], 0, cv.start, h, sg.vslice);
          if (!FP8) tma_load_4d(dst + HALF, &maps.v[sg.vmap], &kv_full[stage], 64, cv.start, h, sg.vslice);
          cv.next(g);
        }
        if (has_k) {
          const AttnSeg& sg = g.seg[ck.seg];
          tma_load_4d(dst + TILE, &maps.k[sg.kmap], &kv_full[stage], 0, ck.start, h, sg.kslice);
          if (!FP8) tma_load_4d(dst + TILE + HALF, &maps.k[sg.kmap], &kv_full[stage], 64, ck.start, h, sg.kslice);
          ck.next(g);
        }
        last_parity[stage] = static_cast<int>(par);
      }
      mbar_wait(q_full, 0, err);
      for (int i = 0; i < NS; ++i)
        if (last_parity[i] >= 0) mbar_wait(&kv_full[i], static_cast<uint32_t>(last_parity[i]), err);
    } else if (warp == 1) {
      // -------------------------------------------------------------- MMA issuer
      // The whole warp runs the loop and waits (one outcome for all lanes), and
      // one elected lane issues the MMAs and commits: measured 9-12 % faster per
      // clock than the same loop run by a single thread.
      auto wwait = [&](uint64_t* bar, uint32_t par) { return __all_sync(0xffffffffu, mbar_wait(bar, par, err)); };
      // The tensor core queues only a few MMAs, so the issue loop is kept lean:
      // descriptors are precomputed and advanced by adding offsets, pv_done is
      // committed only for the last key tile (the commit of S(t) already covers
      // PV(t-1), issued before it), and the loop polls no flags.
      constexpr uint32_t idS = FP8 ? idesc_e4m3(BQ, BKV) : idesc_bf16(BQ, BKV, false, false);
      constexpr uint32_t idPV = FP8 ? idesc_e4m3(BQ, 128, true) : idesc_bf16(BQ, 128, false, true);
      // The start-address field of a descriptor is (address >> 4) in its low 14
      // bits; every shared address here is below 256 KB, so adding (offset >> 4)
      // moves a descriptor by `offset` bytes without a carry out of the field.
      const uint64_t dQ = sdesc_kmajor(smem_u32(sQ));
      const uint64_t dK = sdesc_kmajor(smem_u32(sKV + TILE));
      const uint64_t dV = sdesc_mnmajor(smem_u32(sKV), HALF);
      // One K step is 32 bytes of a 128-byte row: 16 bf16 or 32 e4m3 head dims.
      auto issue_s = [&](int w, uint32_t stage) {
        if (FP8) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t off = kk * 32;
            umma_e4m3_ss(tmem + s_col(w), dQ + ((w * TILE + off) >> 4), dK + ((stage * 2 * TILE + off) >> 4), idS,
                         kk > 0 ? 1u : 0u);
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < 128 / 16; ++kk) {
            const uint32_t off = (kk >> 2) * HALF + (kk & 3) * 32;
            umma_bf16_ss(tmem + s_col(w), dQ + ((w * TILE + off) >> 4), dK + ((stage * 2 * TILE + off) >> 4), idS,
                         kk > 0 ? 1u : 0u);
          }
        }
        umma_commit(&s_full[w]);
      };
      bool ok = wwait(q_full, 0) && (nt == 0 || wwait(&kv_full[0], 0));
      if (ok && nt > 0) {
        tc_fence_after();
        if (elect_one()) {
          for (int w = 0; w < nq; ++w) issue_s(w, 0);
          umma_commit(&kv_empty[0]);
        }
        __syncwarp();
      }
      // step t reads ring step t+1 = [V(t) | K(t+1)]: stage (t+1) % NS, phase ((t+1) / NS) & 1
      uint32_t vs = 1 % NS, vpar = (1 / NS) & 1;
      for (int t = 0; t < nt && ok; ++t) {
        const bool more = t + 1 < nt;
        ok = wwait(&kv_full[vs], vpar);
        if (!ok) break;
        for (int w = 0; w < nq; ++w) {
          if (!wwait(&p_full[w], static_cast<uint32_t>(t & 1))) { ok = false; break; }
          tc_fence_after();
          if (elect_one()) {
          // One K step is 8 tensor-memory columns of P (16 bf16 or 32 e4m3 keys)
          // and 16 or 32 key rows of the V tile (128 bytes each).
          if (FP8) {
#pragma unroll
            for (int kk = 0; kk < BKV / 32; ++kk)
              umma_e4m3_ts(tmem + o_col(w), tmem + s_col(w) + kk * 8, dV + ((vs * 2 * TILE + kk * 4096) >> 4), idPV,
                           (t > 0 || kk > 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int kk = 0; kk < BKV / 16; ++kk)
              umma_bf16_ts(tmem + o_col(w), tmem + s_col(w) + kk * 8, dV + ((vs * 2 * TILE + kk * 2048) >> 4), idPV,
                           (t > 0 || kk > 0) ? 1u : 0u);
          }
          if (more)
            issue_s(w, vs);
          else
            umma_commit(&pv_done[w]);
          }
          __syncwarp();
        }
        if (!ok) break;
        if (elect_one()) umma_commit(&kv_empty[vs]);
        __syncwarp();
        if (++vs == NS) { vs = 0; vpar ^= 1u; }
      }
      if (!ok) abort_flag = 1;
      if (elect_one()) umma_commit(drain);
      __syncwarp();
      wwait(drain, 0);
    }
  } else {
    regs_inc<REGS_HIGH>();
    // ---------------------------------------------------------------- softmax
    const int w = (warp >> 2) - 1;          // 0: tile A (warps 4..7), 1: tile B (warps 8..11)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_base = tmem + lane_off + s_col(w);
    const uint32_t o_base = tmem + lane_off + o_col(w);
    if (w < nq) {
      float m_ref = -INFINITY, l = 0.f;
      const float c8 = FP8 ? p.sq[h] * p.sk[h] * p.scale_log2 : 0.f;
      SegCursor cur;
      bool ok = true;
      for (int t = 0; t < nt; ++t) {
        const int valid = min(BKV, g.seg[cur.seg].len - cur.start);
        cur.next(g);
        if (abort_flag || !mbar_wait(&s_full[w], static_cast<uint32_t>(t & 1), err)) { ok = false; break; }
        tc_fence_after();
        float s[128];
        {
          uint32_t u[4][32];
#pragma unroll
          for (int c = 0; c < 4; ++c) tmem_ld32(s_base + c * 32, u[c]);
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 4; ++c)
#pragma unroll
            for (int i = 0; i < 32; ++i) s[32 * c + i] = __uint_as_float(u[c][i]);
        }
        if (!PRESCALED && !FP8) {
          const float2 sc = make_float2(p.scale_log2, p.scale_log2);
#pragma unroll
          for (int i = 0; i < 64; ++i) {
            const float2 v = __fmul2_rn(make_float2(s[2 * i], s[2 * i + 1]), sc);
            s[2 * i] = v.x;
            s[2 * i + 1] = v.y;
          }
        }
        uint32_t P[FP8 ? 32 : 64];
        float alpha;
        bool need;
        float rs;
        if constexpr (FP8)
          rs = valid == BKV ? softmax_tile_fp8<false, EMU>(s, P, valid, c8, m_ref, alpha, need)
                            : softmax_tile_fp8<true, EMU>(s, P, valid, c8, m_ref, alpha, need);
        else
          rs = valid == BKV ? softmax_tile<false, EMU>(s, P, valid, m_ref, alpha, need)
                            : softmax_tile<true, EMU>(s, P, valid, m_ref, alpha, need);
        if (t >= 1 && __any_sync(0xffffffffu, need)) {
          // O is stable: the commit that signalled S(t) also covers PV(t-1), issued before it
#pragma unroll 1
          for (int c4 = 0; c4 < 4; ++c4) {
            uint32_t o[32];
            tmem_ld32(o_base + c4 * 32, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(o_base + c4 * 32, o);
          }
        }
        tmem_st32(s_base, *reinterpret_cast<uint32_t(*)[32]>(P));
        if constexpr (!FP8) tmem_st32(s_base + 32, *reinterpret_cast<uint32_t(*)[32]>(P + 32));
        tmem_st_wait();
        l = l * alpha + rs;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[w]);
      }
      if (!ok) abort_flag = 1;
      if (ok && nt > 0 && mbar_wait(&pv_done[w], 0, err)) {   // committed once, after the last PV
        tc_fence_after();
        const float inv = FP8 ? p.sv[h] / l : 1.0f / l;
        const int qrow = q0 + w * BQ + r;
        const bool store = qrow < p.Tq;
        const long long orow_idx = static_cast<long long>(g.out_row0) + qrow;
        __nv_bfloat16* orow =
            reinterpret_cast<__nv_bfloat16*>(p.out) + orow_idx * p.out_ld + static_cast<long long>(h) * 128;
        float* orow32 = p.out32 ? p.out32 + orow_idx * p.out_ld + static_cast<long long>(h) * 128 : nullptr;
#pragma unroll 1
        for (int c4 = 0; c4 < 4; ++c4) {
          uint32_t o[32];
          tmem_ld32(o_base + c4 * 32, o);
          tmem_ld_wait();
          if (store) {
            float v[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(o[i]) * inv;
            uint4* dst = reinterpret_cast<uint4*>(orow + c4 * 32);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              uint4 wv;
              wv.x = pack_bf16x2(v[8 * i + 0], v[8 * i + 1]);
              wv.y = pack_bf16x2(v[8 * i + 2], v[8 * i + 3]);
              wv.z = pack_bf16x2(v[8 * i + 4], v[8 * i + 5]);
              wv.w = pack_bf16x2(v[8 * i + 6], v[8 * i + 7]);
              dst[i] = wv;
            }
            if (orow32) {
              float4* d32 = reinterpret_cast<float4*>(orow32 + c4 * 32);
#pragma unroll
              for (int i = 0; i < 8; ++i) d32[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <bool PRESCALED, int EMU, bool FP8 = false>
cudaError_t launch_variant(const AttnMaps& maps, const AttnParams& p, cudaStream_t st) {
  auto kern = k_attn_tc<PRESCALED, EMU, FP8>;
  constexpr size_t SMEM = smem_bytes<FP8>();
  // The register split above assumes the kernel launches with exactly
  // LAUNCH_REGS registers a thread; with fewer, setmaxnreg.inc could not be
  // satisfied, so refuse to launch.
  static const int regs = [&] {
    cudaFuncAttributes fa{};
    return cudaFuncGetAttributes(&fa, kern) == cudaSuccess ? fa.numRegs : -1;
  }();
  if (regs != LAUNCH_REGS) {
    std::fprintf(stderr, "k_attn_tc: compiled with %d registers a thread, the register split needs %d\n", regs,
                 LAUNCH_REGS);
    return cudaErrorInvalidConfiguration;
  }
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(SMEM));
  if (e != cudaSuccess) return e;
  const int qtiles = (p.Tq + BQ - 1) / BQ;
  dim3 grid((qtiles + 1) / 2, p.H, p.ngroups);
  kern<<<grid, THREADS, SMEM, st>>>(maps, p);
  return cudaGetLastError();
}

// Pairs of every 8 on full key tiles that take the polynomial exp2: LA_ATTN_EMU
// when set (0, 2, 3 or 4), else 2 for bf16 and 0 for e4m3.  With two of eight
// pairs on the FMA pipe the bf16 kernel ran 1.2 % faster under the power cap
// (3.9 % per clock) at the one-slot 14B-like shape, and 0.7 % in the 8-layer
// stream, where the clock drops with it and the tick time stays the same; e4m3
// keeps ex2 alone for parity.
int emu_setting(bool fp8) {
  static const int v = [] {
    const char* e = std::getenv("LA_ATTN_EMU");
    return e ? std::atoi(e) : -1;
  }();
  return v >= 0 ? v : (fp8 ? 0 : 2);
}

}  // namespace

cudaError_t launch_attention_tc(const AttnMaps& maps, const AttnParams& p, cudaStream_t st) {
  if (p.fp8) {
    if (!p.sq || !p.sk || !p.sv) return cudaErrorInvalidValue;
    switch (emu_setting(true)) {
      case 0: return launch_variant<false, 0, true>(maps, p, st);
      case 2: return launch_variant<false, 2, true>(maps, p, st);
      case 4: return launch_variant<false, 4, true>(maps, p, st);
      default: return launch_variant<false, 3, true>(maps, p, st);
    }
  }
  const bool pre = p.q_prescaled != 0;
  switch (emu_setting(false)) {
    case 0: return pre ? launch_variant<true, 0>(maps, p, st) : launch_variant<false, 0>(maps, p, st);
    case 2: return pre ? launch_variant<true, 2>(maps, p, st) : launch_variant<false, 2>(maps, p, st);
    case 4: return pre ? launch_variant<true, 4>(maps, p, st) : launch_variant<false, 4>(maps, p, st);
    default: return pre ? launch_variant<true, 3>(maps, p, st) : launch_variant<false, 3>(maps, p, st);
  }
}
