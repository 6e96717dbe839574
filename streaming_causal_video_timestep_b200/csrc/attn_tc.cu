// Block-causal attention on tcgen05 tensor cores, head_dim 128: bf16 q/K/V/P
// operands, fp32 scores, softmax and accumulation, bf16 output.
//
// One CTA = 128 queries of one (group, head); the keys are the group's list of
// segments [sink | window blocks oldest first | the block itself], walked in
// tiles of 128 keys (the last tile of a segment is ragged and masked).
// 6 warps:
//   warp 0      TMA producer: Q once, then K_t and V_t tiles (two 64-column
//               boxes each, 128-byte swizzle) into a 4-deep ring;
//   warp 1      TMEM owner (512 columns: S0 | S1 | O) and MMA issuer:
//               S_t = Q K_t^T into S[t%2] (K-major A and B), then
//               O += P_{t-1} V_{t-1} (P K-major from shared memory, V read
//               MN-major straight from its [keys, d] tile);
//   warps 2..5  softmax: thread = query row = TMEM lane.  tcgen05.ld of the S
//               row, masked row max, exp2, row sum, lazy rescale of O in TMEM
//               (only when the running max grows by more than 2^8), P written
//               to shared memory as bf16 in the swizzled K-major layout, then
//               the final 1/l normalisation and bf16 store (plus an optional
//               fp32 copy).
// Scores are formed in the log2 domain: with q pre-multiplied by log2(e)/sqrt(d)
// (PRESCALED, the stream's QKV epilogue does it) p = 2^(s - max s); otherwise the
// scaled score x = s * scale is rounded first.  Either way the row maximum gives
// exactly 2^0 = 1, so the row sum is >= 1 whatever the magnitude of the logits.
// S_{t+1} is computed on the tensor cores while the softmax warps work on S_t.
#include "kernels.h"
#include "sm100.cuh"

namespace {

constexpr int BQ = 128;
constexpr int BKV = 128;
constexpr int NS = 4;
constexpr uint32_t HALF = 16384;            // one 128-row x 128-byte swizzled box
constexpr uint32_t TILE = 2 * HALF;         // 128 rows x 128 bf16
constexpr uint32_t TMEM_COLS = 512;
constexpr uint32_t O_COL = 256;
constexpr size_t SMEM = 1024 + TILE /*Q*/ + NS * TILE /*K,V ring*/ + TILE /*P*/ + 256;

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
__global__ void __launch_bounds__(192, 1)
k_attn_tc(const __grid_constant__ AttnMaps maps, const __grid_constant__ AttnParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sKV = smem + TILE;
  uint8_t* sP = sKV + NS * TILE;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sP + TILE);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + NS;
  uint64_t* s_full = kv_empty + NS;
  uint64_t* s_free = s_full + 2;
  uint64_t* p_full = s_free + 2;
  uint64_t* pv_done = p_full + 1;
  uint64_t* drain = pv_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  __shared__ volatile int abort_flag;

  const AttnGroup& g = p.g[blockIdx.z];
  const int h = blockIdx.y;
  const int q0 = blockIdx.x * BQ;
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  int* err = p.err;

  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(q_full, 1);
    for (int i = 0; i < NS; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
    }
    mbar_init(p_full, 4);
    mbar_init(pv_done, 1);
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
    if (lane == 0) {
      int last_parity[NS];
      for (int i = 0; i < NS; ++i) last_parity[i] = -1;
      mbar_expect_tx(q_full, TILE);
      tma_load_4d(sQ, &maps.q, q_full, 0, q0, h, g.q_slice);
      tma_load_4d(sQ + HALF, &maps.q, q_full, 64, q0, h, g.q_slice);
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
    if (lane == 0) {
      constexpr uint32_t idS = idesc_bf16(BQ, BKV, false, false);
      constexpr uint32_t idPV = idesc_bf16(BQ, 128, false, true);
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t p_addr = smem_u32(sP);
      bool ok = mbar_wait(q_full, 0, err);
      auto issue_pv = [&](int u) -> bool {
        const int n = 2 * u + 1;
        const int vs = n % NS;
        if (!mbar_wait(p_full, static_cast<uint32_t>(u & 1), err)) return false;
        if (!mbar_wait(&kv_full[vs], static_cast<uint32_t>((n / NS) & 1), err)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(sKV + vs * TILE);
#pragma unroll
        for (int kk = 0; kk < BKV / 16; ++kk) {
          const uint64_t a = sdesc_kmajor(p_addr + (kk >> 2) * HALF + (kk & 3) * 32);
          const uint64_t b = sdesc_mnmajor(v_addr + kk * 2048, HALF);
          umma_bf16_ss(tmem + O_COL, a, b, idPV, (u > 0 || kk > 0) ? 1u : 0u);
        }
        umma_commit(&kv_empty[vs]);
        umma_commit(pv_done);
        return true;
      };
      for (int t = 0; t < nt && ok; ++t) {
        if (abort_flag) { ok = false; break; }
        const int n = 2 * t;
        const int ks = n % NS;
        const int sb = t & 1;
        if (!mbar_wait(&kv_full[ks], static_cast<uint32_t>((n / NS) & 1), err)) { ok = false; break; }
        if (!mbar_wait(&s_free[sb], static_cast<uint32_t>(((t >> 1) & 1) ^ 1), err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t k_addr = smem_u32(sKV + ks * TILE);
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk) {
          const uint32_t off = (kk >> 2) * HALF + (kk & 3) * 32;
          umma_bf16_ss(tmem + sb * 128, sdesc_kmajor(q_addr + off), sdesc_kmajor(k_addr + off), idS,
                       kk > 0 ? 1u : 0u);
        }
        umma_commit(&s_full[sb]);
        umma_commit(&kv_empty[ks]);
        if (t >= 1 && !issue_pv(t - 1)) { ok = false; break; }
      }
      if (ok && nt > 0) ok = issue_pv(nt - 1);
      if (!ok) abort_flag = 1;
      umma_commit(drain);
      mbar_wait(drain, 0, err);
    }
  } else {
    // softmax warps
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const float sc = p.scale_log2;
    float m_ref = -INFINITY, l = 0.f;
    SegCursor cur;
    bool ok = true;
    for (int t = 0; t < nt; ++t) {
      const int sb = t & 1;
      const int valid = min(BKV, g.seg[cur.seg].len - cur.start);
      cur.next(g);
      if (abort_flag || !mbar_wait(&s_full[sb], static_cast<uint32_t>((t >> 1) & 1), err)) { ok = false; break; }
      tc_fence_after();
      uint32_t s[128];
      {
        uint32_t (&s0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[0]);
        uint32_t (&s1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[32]);
        uint32_t (&s2)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[64]);
        uint32_t (&s3)[32] = *reinterpret_cast<uint32_t(*)[32]>(&s[96]);
        const uint32_t base = tmem + lane_off + static_cast<uint32_t>(sb * 128);
        tmem_ld32(base + 0, s0);
        tmem_ld32(base + 32, s1);
        tmem_ld32(base + 64, s2);
        tmem_ld32(base + 96, s3);
        tmem_ld_wait();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[sb]);

      // scores in the log2 domain (rounded once), row max and sum with 8
      // independent partial accumulators (one warp per scheduler: latency is
      // hidden by ILP, not by other warps)
      float x[128];
#pragma unroll
      for (int c = 0; c < 128; ++c) x[c] = PRESCALED ? __uint_as_float(s[c]) : __fmul_rn(__uint_as_float(s[c]), sc);
      float mx8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mx8[u] = -INFINITY;
      if (valid == BKV) {
#pragma unroll
        for (int c = 0; c < 128; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], x[c]);
      } else {
#pragma unroll
        for (int c = 0; c < 128; ++c) mx8[c & 7] = fmaxf(mx8[c & 7], c < valid ? x[c] : -INFINITY);
      }
      const float m_tile = fmaxf(fmaxf(fmaxf(mx8[0], mx8[1]), fmaxf(mx8[2], mx8[3])),
                                 fmaxf(fmaxf(mx8[4], mx8[5]), fmaxf(mx8[6], mx8[7])));
      const bool need = m_tile > m_ref + 8.0f;
      const float m_new = need ? m_tile : m_ref;
      const float alpha = need ? fast_exp2(m_ref - m_new) : 1.0f;
      float rs8[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) rs8[u] = 0.f;
      uint32_t pk[64];
      if (valid == BKV) {
#pragma unroll
        for (int c = 0; c < 128; c += 2) {
          const float p0 = fast_exp2(x[c] - m_new);
          const float p1 = fast_exp2(x[c + 1] - m_new);
          rs8[(c >> 1) & 7] += p0 + p1;
          pk[c / 2] = pack_bf16x2(p0, p1);
        }
      } else {
#pragma unroll
        for (int c = 0; c < 128; c += 2) {
          const float p0 = c < valid ? fast_exp2(x[c] - m_new) : 0.f;
          const float p1 = c + 1 < valid ? fast_exp2(x[c + 1] - m_new) : 0.f;
          rs8[(c >> 1) & 7] += p0 + p1;
          pk[c / 2] = pack_bf16x2(p0, p1);
        }
      }
      const float rs = ((rs8[0] + rs8[1]) + (rs8[2] + rs8[3])) + ((rs8[4] + rs8[5]) + (rs8[6] + rs8[7]));
      l = l * alpha + rs;
      m_ref = m_new;

      if (t >= 1) {
        if (!mbar_wait(pv_done, static_cast<uint32_t>((t - 1) & 1), err)) { ok = false; break; }
        tc_fence_after();
        if (__any_sync(0xffffffffu, need)) {
#pragma unroll 1
          for (int c4 = 0; c4 < 4; ++c4) {
            uint32_t o[32];
            const uint32_t addr = tmem + lane_off + O_COL + c4 * 32;
            tmem_ld32(addr, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(addr, o);
          }
          tmem_st_wait();
        }
      }
      // P row r, swizzled K-major: 16-byte chunk c of 64-key atom a at
      // a*HALF + r*128 + ((c ^ (r & 7)) * 16)
      uint8_t* prow = sP + r * 128;
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        const int atom = ch >> 3, c = ch & 7;
        uint4 w = make_uint4(pk[4 * ch], pk[4 * ch + 1], pk[4 * ch + 2], pk[4 * ch + 3]);
        *reinterpret_cast<uint4*>(prow + atom * HALF + ((c ^ (r & 7)) << 4)) = w;
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (!ok) abort_flag = 1;
    if (ok && nt > 0 && mbar_wait(pv_done, static_cast<uint32_t>((nt - 1) & 1), err)) {
      tc_fence_after();
      const float inv = 1.0f / l;
      const bool store = q0 + r < p.Tq;
      const long long orow_idx = static_cast<long long>(g.out_row0) + q0 + r;
      __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.out) + orow_idx * p.out_ld + static_cast<long long>(h) * 128;
      float* orow32 = p.out32 ? p.out32 + orow_idx * p.out_ld + static_cast<long long>(h) * 128 : nullptr;
#pragma unroll 1
      for (int c4 = 0; c4 < 4; ++c4) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_off + O_COL + c4 * 32, o);
        tmem_ld_wait();
        if (store) {
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(o[i]) * inv;
          uint4* dst = reinterpret_cast<uint4*>(orow + c4 * 32);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            uint4 w;
            w.x = pack_bf16x2(v[8 * i + 0], v[8 * i + 1]);
            w.y = pack_bf16x2(v[8 * i + 2], v[8 * i + 3]);
            w.z = pack_bf16x2(v[8 * i + 4], v[8 * i + 5]);
            w.w = pack_bf16x2(v[8 * i + 6], v[8 * i + 7]);
            dst[i] = w;
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

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace

cudaError_t launch_attn_tc(const AttnMaps& maps, const AttnParams& p, cudaStream_t st) {
  auto kern = p.q_prescaled ? k_attn_tc<true> : k_attn_tc<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(SMEM));
  if (e != cudaSuccess) return e;
  dim3 grid((p.Tq + BQ - 1) / BQ, p.H, p.ngroups);
  kern<<<grid, 192, SMEM, st>>>(maps, p);
  return cudaGetLastError();
}
