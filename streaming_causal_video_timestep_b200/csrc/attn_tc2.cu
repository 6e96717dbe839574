// Block-causal attention, tcgen05, head_dim 128, two query tiles per CTA.
//
// One CTA = up to 256 queries (two 128-row tiles A and B) of one (group, head),
// sharing every K/V tile of the group's segments [sink | window | block].
// 10 warps:
//   warp 0      TMA producer: Q_A, Q_B once, then K_t / V_t (two 64-column
//               128-byte-swizzled boxes each) into a 5-stage ring;
//   warp 1      TMEM owner (512 columns: S_A | S_B | O_A | O_B) and MMA issuer;
//   warps 2..5  softmax of tile A, warps 6..9 softmax of tile B: one thread per
//               query row (= TMEM lane).
// Per key tile t the tensor core runs, in issue order,
//   ... PV_A(t-1), S_A(t), PV_B(t-1), S_B(t) ...
// so while one softmax warpgroup turns S into P the tensor core works on the
// other tile.  P is written as bf16 into the first 64 columns of its own S
// tile (tcgen05.st) and read from there as the A operand of O += P V
// (tcgen05.mma with A in tensor memory), so P never touches shared memory;
// V is read MN-major straight from its [keys, d] tile.
// Scores are in the log2 domain (q pre-multiplied by log2(e)/sqrt(d) when
// PRESCALED, else scaled and rounded first), so the row maximum contributes
// exactly 2^0 = 1 and the row sum is >= 1.  The running max is updated lazily:
// O is rescaled in TMEM only when the max grows by more than 2^8.
#include <cstdio>
#include <cstdlib>

#include "kernels.h"
#include "sm100.cuh"

namespace {

constexpr int BQ = 128;
constexpr int BKV = 128;
constexpr int NS = 5;
constexpr uint32_t HALF = 16384;            // 128 rows x 128 bytes, one swizzle-128B box
constexpr uint32_t TILE = 2 * HALF;         // 128 rows x 128 bf16
constexpr uint32_t TMEM_COLS = 512;
constexpr size_t SMEM = 1024 + 2 * TILE /*Q_A, Q_B*/ + NS * TILE /*K, V ring*/ + 256;

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

template <bool PRESCALED>
__global__ void __launch_bounds__(320, 1)
k_attn_tc2(const __grid_constant__ AttnMaps maps, const __grid_constant__ AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;                       // Q_A at 0, Q_B at TILE
  uint8_t* sKV = smem + 2 * TILE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sKV + NS * TILE);
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

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int last_parity[NS];
      for (int i = 0; i < NS; ++i) last_parity[i] = -1;
      mbar_expect_tx(q_full, 2 * TILE);
      for (int w = 0; w < 2; ++w) {
        tma_load_4d(sQ + w * TILE, &maps.q, q_full, 0, q0 + w * BQ, h, g.q_slice);
        tma_load_4d(sQ + w * TILE + HALF, &maps.q, q_full, 64, q0 + w * BQ, h, g.q_slice);
      }
      SegCursor cur;
      int n = 0;
      for (int t = 0; t < nt && !abort_flag; ++t) {
        const AttnSeg& sg = g.seg[cur.seg];
#pragma unroll
        for (int kv = 0; kv < 2; ++kv) {
          const int stage = n % NS;
          const uint32_t par = static_cast<uint32_t>((n / NS) & 1);
          if (!mbar_wait(&kv_empty[stage], par ^ 1, err)) { abort_flag = 1; break; }
          const CUtensorMap* m = kv == 0 ? &maps.k[sg.kmap] : &maps.v[sg.vmap];
          const int slice = kv == 0 ? sg.kslice : sg.vslice;
          uint8_t* dst = sKV + stage * TILE;
          mbar_expect_tx(&kv_full[stage], TILE);
          tma_load_4d(dst, m, &kv_full[stage], 0, cur.start, h, slice);
          tma_load_4d(dst + HALF, m, &kv_full[stage], 64, cur.start, h, slice);
          last_parity[stage] = static_cast<int>(par);
          ++n;
        }
        cur.next(g);
      }
      mbar_wait(q_full, 0, err);
      for (int i = 0; i < NS; ++i)
        if (last_parity[i] >= 0) mbar_wait(&kv_full[i], static_cast<uint32_t>(last_parity[i]), err);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(BQ, BKV, false, false);
      constexpr uint32_t idPV = idesc_bf16(BQ, 128, false, true);
      const uint32_t q_addr = smem_u32(sQ);
      auto issue_s = [&](int w, int stage) {
        const uint32_t k_addr = smem_u32(sKV + stage * TILE);
        const uint32_t qa = q_addr + w * TILE;
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk) {
          const uint32_t off = (kk >> 2) * HALF + (kk & 3) * 32;
          umma_bf16_ss(tmem + s_col(w), sdesc_kmajor(qa + off), sdesc_kmajor(k_addr + off), idS, kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[w]);
      };
      bool ok = mbar_wait(q_full, 0, err);
      // S(0) for every tile
      if (ok && nt > 0) {
        ok = mbar_wait(&kv_full[0], 0, err);
        if (ok) {
          tc_fence_after();
          for (int w = 0; w < nq; ++w) issue_s(w, 0);
          umma_commit(&kv_empty[0]);
        }
      }
      for (int t = 0; t < nt && ok; ++t) {
        if (abort_flag) { ok = false; break; }
        const int nv = 2 * t + 1, vs = nv % NS;
        const int nk = 2 * t + 2, ks = nk % NS;
        if (!mbar_wait(&kv_full[vs], static_cast<uint32_t>((nv / NS) & 1), err)) { ok = false; break; }
        const bool more = t + 1 < nt;
        for (int w = 0; w < nq && ok; ++w) {
          if (!mbar_wait(&p_full[w], static_cast<uint32_t>(t & 1), err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t v_addr = smem_u32(sKV + vs * TILE);
#pragma unroll
          for (int kk = 0; kk < BKV / 16; ++kk) {
            umma_bf16_ts(tmem + o_col(w), tmem + s_col(w) + kk * 8, sdesc_mnmajor(v_addr + kk * 2048, HALF), idPV,
                         (t > 0 || kk > 0) ? 1u : 0u);
          }
          umma_commit(&pv_done[w]);
          if (more) {
            if (w == 0 && !mbar_wait(&kv_full[ks], static_cast<uint32_t>((nk / NS) & 1), err)) { ok = false; break; }
            tc_fence_after();
            issue_s(w, ks);
          }
        }
        if (!ok) break;
        umma_commit(&kv_empty[vs]);
        if (more) umma_commit(&kv_empty[ks]);
      }
      if (!ok) abort_flag = 1;
      umma_commit(drain);
      mbar_wait(drain, 0, err);
    }
  } else {
    // ---------------------------------------------------------------- softmax
    const int w = (warp - 2) >> 2;          // 0: tile A (warps 2..5), 1: tile B (warps 6..9)
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t s_base = tmem + lane_off + s_col(w);
    const uint32_t o_base = tmem + lane_off + o_col(w);
    const float sc = p.scale_log2;
    if (w < nq) {
      float m_ref = -INFINITY, l = 0.f;
      SegCursor cur;
      bool ok = true;
      for (int t = 0; t < nt; ++t) {
        const int valid = min(BKV, g.seg[cur.seg].len - cur.start);
        cur.next(g);
        if (abort_flag || !mbar_wait(&s_full[w], static_cast<uint32_t>(t & 1), err)) { ok = false; break; }
        tc_fence_after();
        // pass 1: row max of the scaled scores, 64 columns at a time
        float mx8[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) mx8[u] = -INFINITY;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t a[32], b[32];
          tmem_ld32(s_base + hf * 64, a);
          tmem_ld32(s_base + hf * 64 + 32, b);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            float xa = __uint_as_float(a[i]), xb = __uint_as_float(b[i]);
            if (!PRESCALED) { xa = __fmul_rn(xa, sc); xb = __fmul_rn(xb, sc); }
            if (hf * 64 + i >= valid) xa = -INFINITY;
            if (hf * 64 + 32 + i >= valid) xb = -INFINITY;
            mx8[i & 7] = fmaxf(mx8[i & 7], fmaxf(xa, xb));
          }
        }
        const float m_tile = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                   fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
        const bool need = m_tile > m_ref + 8.0f;
        const float m_new = need ? m_tile : m_ref;
        const float alpha = need ? fast_exp2(m_ref - m_new) : 1.0f;
        if (t >= 1) {
          // PV(t-1) has completed (it precedes S(t) on the tensor core): O is stable
          if (!mbar_wait(&pv_done[w], static_cast<uint32_t>((t - 1) & 1), err)) { ok = false; break; }
          tc_fence_after();
          if (__any_sync(0xffffffffu, need)) {
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
        }
        // pass 2: P = 2^(x - m) as bf16 over the consumed S columns: S columns
        // [64h, 64h+64) become P columns [32h, 32h+32) (written only after read)
        float rs8[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) rs8[u] = 0.f;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t a[32], b[32];
          tmem_ld32(s_base + hf * 64, a);
          tmem_ld32(s_base + hf * 64 + 32, b);
          tmem_ld_wait();
          uint32_t pa[16], pb[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float x0 = __uint_as_float(a[2 * i]), x1 = __uint_as_float(a[2 * i + 1]);
            float y0 = __uint_as_float(b[2 * i]), y1 = __uint_as_float(b[2 * i + 1]);
            if (!PRESCALED) { x0 = __fmul_rn(x0, sc); x1 = __fmul_rn(x1, sc); y0 = __fmul_rn(y0, sc); y1 = __fmul_rn(y1, sc); }
            const int c = hf * 64 + 2 * i;
            const float p0 = c < valid ? fast_exp2(x0 - m_new) : 0.f;
            const float p1 = c + 1 < valid ? fast_exp2(x1 - m_new) : 0.f;
            const float p2 = c + 32 < valid ? fast_exp2(y0 - m_new) : 0.f;
            const float p3 = c + 33 < valid ? fast_exp2(y1 - m_new) : 0.f;
            rs8[i & 7] += (p0 + p1) + (p2 + p3);
            pa[i] = pack_bf16x2(p0, p1);
            pb[i] = pack_bf16x2(p2, p3);
          }
          tmem_st16(s_base + hf * 32, pa);
          tmem_st16(s_base + hf * 32 + 16, pb);
        }
        tmem_st_wait();
        l = l * alpha + (((rs8[0] + rs8[1]) + (rs8[2] + rs8[3])) + ((rs8[4] + rs8[5]) + (rs8[6] + rs8[7])));
        m_ref = m_new;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[w]);
      }
      if (!ok) abort_flag = 1;
      if (ok && nt > 0 && mbar_wait(&pv_done[w], static_cast<uint32_t>((nt - 1) & 1), err)) {
        tc_fence_after();
        const float inv = 1.0f / l;
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

}  // namespace

cudaError_t launch_attn_tc2(const AttnMaps& maps, const AttnParams& p, cudaStream_t st) {
  auto kern = p.q_prescaled ? k_attn_tc2<true> : k_attn_tc2<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(SMEM));
  if (e != cudaSuccess) return e;
  const int qtiles = (p.Tq + BQ - 1) / BQ;
  dim3 grid((qtiles + 1) / 2, p.H, p.ngroups);
  kern<<<grid, 320, SMEM, st>>>(maps, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) {
    cudaFuncAttributes fa{};
    cudaFuncGetAttributes(&fa, kern);
    std::fprintf(stderr,
                 "k_attn_tc2 launch refused (%s): regs %d, maxThreadsPerBlock %d, static smem %zu, "
                 "max dynamic smem %d, requested dynamic smem %zu, local %zu, param bytes %zu\n",
                 cudaGetErrorString(e), fa.numRegs, fa.maxThreadsPerBlock, fa.sharedSizeBytes,
                 fa.maxDynamicSharedSizeBytes, SMEM, fa.localSizeBytes, sizeof(AttnMaps) + sizeof(AttnParams));
  }
  return e;
}

cudaError_t launch_attention_tc(const AttnMaps& maps, const AttnParams& p, cudaStream_t st) {
  static const int v = [] {
    const char* e = std::getenv("LA_ATTN_VERSION");
    return e ? std::atoi(e) : 3;
  }();
  if (v == 1) return launch_attn_tc(maps, p, st);
  if (v == 2) return launch_attn_tc2(maps, p, st);
  return launch_attn_tc3(maps, p, st);
}
