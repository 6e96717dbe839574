// Host side of the streaming step: configuration checks, device buffers, the
// tick state machine, kernel sequencing and the C ABI declared in la_stream.h.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <functional>
#include <new>
#include <string>
#include <vector>

#include "kernels.h"
#include "la_stream.h"
#include "tmap.h"

namespace {

// ---------------------------------------------------------------------------
// Tick state machine.
//
// Pipelined schedule (the timestep-forcing pipeline of the pages): slot i holds
// the block slot i-1 held in the previous call; slot 0 takes the new block.
// Ring of each (layer, slot): window+1 entries; block b writes entry b mod
// (window+1), evicting block b - window - 1; block b reads b-window .. b-1.
// ---------------------------------------------------------------------------
struct SlotRecord {
  int active_block = -1, write_entry = -1, evicted = -1, sink_tpos = 0, frame_tpos = 0, sink_gen = 0;
};

struct Scheduler {
  int S = 0, E = 0, W = 0, fpb = 0, offset = 0, rolling = 1, pipelined = 1, aas = 0, clean = 0;
  int slot_only = -1;       // LA_SCHED_SLOT: the one step this stream runs
  int fixed_step = -1;      // LA_CACHE_FIXED_STEP: the step whose cache every step reads the window from
  long long tick = -1, blocks_in = 0, blocks_out = 0;
  int sink_gen = 0;
  std::vector<long long> held;                  // block held by each slot after the last call
  std::vector<std::vector<long long>> tag_blk;  // [S][E]
  std::vector<std::vector<int>> tag_step;       // [S][E]
  std::vector<SlotRecord> rec;

  void init(const la_config& c) {
    S = c.num_steps;
    E = c.window_blocks + 1;
    W = c.window_blocks;
    fpb = c.frames_per_block;
    offset = c.sink_offset_frames;
    rolling = c.rolling_rope;
    pipelined = c.schedule == LA_SCHED_PIPELINED;
    slot_only = c.schedule == LA_SCHED_SLOT ? c.slot_index : -1;
    aas = c.sink_mode == LA_SINK_AAS && slot_only < 0;   // a slot stream's sink is replaced by the caller
    clean = c.cache_mode == LA_CACHE_CLEAN_REFRESH;
    fixed_step = c.cache_mode == LA_CACHE_FIXED_STEP ? c.cache_step : -1;
    held.assign(S, -1);
    tag_blk.assign(S, std::vector<long long>(E, -1));
    tag_step.assign(S, std::vector<int>(E, -1));
    rec.assign(S, SlotRecord());
  }
  // The cache step i writes (and reads its own block from): its own, or the one clean cache.
  int ring_of(int i) const { return clean ? 0 : i; }
  // The cache step i reads the prior blocks from: its own, the clean one, or step fixed_step's.
  int window_ring(int i) const { return fixed_step >= 0 ? fixed_step : ring_of(i); }
  int sink_tpos_of(long long b) const {
    return rolling ? static_cast<int>(fpb * b - offset) : -offset;
  }
  // Which (slot, block) pairs run in the next call, and which block finishes.
  void plan(bool has_new, std::vector<std::pair<int, long long>>& run, long long& finished,
            std::vector<long long>& next_held) const {
    run.clear();
    if (pipelined) {
      next_held.assign(S, -1);
      next_held[0] = has_new ? blocks_in : -1;
      for (int i = 1; i < S; ++i) next_held[i] = held[i - 1];
      for (int i = 0; i < S; ++i)
        if (next_held[i] >= 0) run.emplace_back(i, next_held[i]);
      finished = next_held[S - 1];
    } else if (slot_only >= 0) {
      next_held.assign(S, -1);
      run.emplace_back(slot_only, blocks_in);
      finished = blocks_in;
    } else {
      next_held.assign(S, -1);
      for (int i = 0; i < S; ++i) run.emplace_back(i, blocks_in);
      finished = blocks_in;
    }
  }
  void begin(bool has_new, const std::vector<long long>& next_held) {
    ++tick;
    if (has_new) ++blocks_in;
    if (pipelined) held = next_held;
    for (auto& r : rec) r = SlotRecord();
  }
  int append(int i, long long b) {
    const int e = static_cast<int>(b % E);
    const int ring = ring_of(i);
    SlotRecord& r = rec[i];
    r.active_block = static_cast<int>(b);
    r.write_entry = e;
    r.evicted = static_cast<int>(tag_blk[ring][e]);
    r.sink_tpos = sink_tpos_of(b);
    r.frame_tpos = static_cast<int>(fpb * b);
    r.sink_gen = sink_gen;
    tag_blk[ring][e] = b;
    tag_step[ring][e] = i;
    return e;
  }
  // The clean-cache refresh of finished block b rewrites its entry, tagged (b, S).
  int append_refresh(long long b) {
    const int e = static_cast<int>(b % E);
    tag_blk[0][e] = b;
    tag_step[0][e] = S;
    return e;
  }
  bool finish(long long finished) {
    if (finished >= 0) ++blocks_out;
    if (finished == 0 && aas && sink_gen == 0) {
      sink_gen = 1;
      return true;
    }
    return false;
  }
  long long state_size() const { return 4 + static_cast<long long>(S) * (8 + 3 * E); }
  void export_state(int32_t* out) const {
    out[0] = static_cast<int32_t>(tick);
    out[1] = static_cast<int32_t>(blocks_in);
    out[2] = static_cast<int32_t>(blocks_out);
    out[3] = sink_gen;
    int32_t* p = out + 4;
    for (int i = 0; i < S; ++i) {
      const SlotRecord& r = rec[i];
      const int ring = ring_of(i);
      std::vector<long long> res;
      for (int e = 0; e < E; ++e)
        if (tag_blk[ring][e] >= 0) res.push_back(tag_blk[ring][e]);
      std::sort(res.begin(), res.end());
      *p++ = r.active_block;
      *p++ = r.write_entry;
      *p++ = r.evicted;
      *p++ = r.active_block >= 0 ? r.sink_tpos : 0;
      *p++ = r.active_block >= 0 ? r.frame_tpos : 0;
      *p++ = r.active_block >= 0 ? r.sink_gen : 0;
      *p++ = i;
      *p++ = static_cast<int32_t>(res.size());
      for (int e = 0; e < E; ++e) *p++ = e < static_cast<int>(res.size()) ? static_cast<int32_t>(res[e]) : -1;
      for (int e = 0; e < E; ++e) {
        *p++ = static_cast<int32_t>(tag_blk[ring][e]);
        *p++ = tag_step[ring][e];
      }
    }
  }
};

struct ProfEvent {
  int kind;
  cudaEvent_t a, b;
};

}  // namespace

struct la_stream {
  la_config cfg{};
  float ts[LA_MAX_STEPS + 1] = {};
  int S = 0, E = 0, F = 0, T = 0, D = 0, C = 0, H = 0, d = 0, L = 0, fpb = 0, nbuf = 0;
  int pt = 0, ph = 0, pw = 0;
  bool bf16 = true, id_in = true, id_head = true;
  bool fp8 = false;         // e4m3 QKV / output projections (bf16 streams)
  bool afp8 = false;        // e4m3 attention operands in the denoising passes (bf16 streams)
  bool dit = false;         // LA_BLOCK_DIT: each layer a full DiT block
  int Fffn = 0;             // its FFN width
  bool cross = false;       // LA_BLOCK_DIT with audio: the audio cross-attention sub-block
  int A = 0, Da = 0;        // audio tokens per block, their width
  size_t eq = 2;            // element of q_rope / sk_rope / the rings (1 with afp8, else ea)
  size_t es = 2;            // activation / weight element (bf16 or fp32)
  size_t ea = 2;            // attention operand element (bf16 or fp32)
  int device = 0, num_sms = 148;
  cudaStream_t st = nullptr;

  const void* w_in = nullptr;
  const void* w_head = nullptr;
  std::vector<const void*> w_qkv, w_out;
  std::vector<const void*> w_ffn1, w_ffn2;   // LA_BLOCK_DIT
  const float* ada = nullptr;                // LA_BLOCK_DIT: [L][S+1][6][D]
  void* ffn_u = nullptr;                     // LA_BLOCK_DIT: GELU output [max(nbuf*T, F)][Fffn], dtype
  CUtensorMap tm_u{}, tm_s_u{};
  std::vector<CUtensorMap> tm_w1, tm_w2;
  std::vector<const void*> w_qc, w_kvc, w_oc;   // audio cross-attention
  void* audio_op = nullptr;  // bf16 [A][Da]: the GEMM operand of an entering block's audio
  float* kv32 = nullptr;     // fp32 [A][2D]: one layer's audio K | V before the head split
  void* audio_k = nullptr;   // attn [L][nbuf][H][A][d]: each in-flight block's audio K
  void* audio_v = nullptr;
  float* qc32 = nullptr;     // fp32 [nbuf*T][D]: cross-attention q before the head split
  void* qc_heads = nullptr;  // attn [nbuf][H][T][d]
  void* xo_buf = nullptr;    // dtype [nbuf*T][D]: cross-attention output (the self-attention's stays in attn_o)
  CUtensorMap tm_audio_op{}, tm_xo{};
  std::vector<CUtensorMap> tm_wqc, tm_wkvc, tm_woc;
  AttnMaps maps_cross{};     // q = qc_heads; k[0] / v[0] = audio K / V

  std::vector<void*> allocs;
  float* xs = nullptr;      // [nbuf][T][C]
  float* h32 = nullptr;     // [nbuf*T][D] residual stream
  void* hop = nullptr;      // [nbuf*T][D] normalised GEMM operand, dtype (fp32: == hn32); with the folded
                            // norm, the residual itself rounded to bf16
  // The per-token RMS norm folded into the GEMMs (bf16 attention sublayers with an in-projection and a
  // head): the in- and output projections' epilogues leave each row's sum of squares per column tile in
  // ssq, and the QKV and head epilogues scale their rows by 1 / rms from it (with e4m3 projections, on
  // top of the operand's per-row scale: per-row scaling makes the codes of h those of h / rms).
  bool fold = false;
  float* ssq = nullptr;     // [nbuf*T][ssq_ld]
  int ssq_ld = 0;
  float* hn32 = nullptr;    // [nbuf*T][D] fp32 normalised residual (fp32 streams, identity head)
  void* xop = nullptr;      // [nbuf*T][C] bf16 (bf16 with an in-projection)
  float* qkv = nullptr;     // fp32 [nbuf*T][3D] (fp32 streams; bf16 fuses it into the GEMM)
  void* q_rope = nullptr;   // attn type [nbuf][H][T][d]
  void* sk_rope = nullptr;  // attn type [L][nbuf][H][F][d]
  void* attn_o = nullptr;   // dtype [nbuf*T][D]
  void* ring_k = nullptr;   // attn type [L][S][E][H][T][d]
  void* ring_v = nullptr;
  float* sink_k = nullptr;  // fp32 [L][H][F][d] un-roped
  void* sink_v = nullptr;   // attn type [L][H][F][d]
  uint8_t* sink_v8 = nullptr;  // afp8: e4m3 codes of the sink V [L][H][F][d]
  float* attn_sc = nullptr;    // afp8: [L][3][H] power-of-two scales of q, K, V
  float* attn_inv = nullptr;   // afp8: their inverses
  float* sink_x = nullptr;  // [F][C]
  float* s_h32 = nullptr;   // [F][D]
  void* s_hop = nullptr;    // normalised operand (fp32 streams: == s_hn32)
  float* s_hn32 = nullptr;
  void* s_xop = nullptr;
  float* s_qkv = nullptr;   // fp32 [F][3D]
  void* s_q = nullptr;      // attn type [H][F][d]
  void* s_k = nullptr;
  void* s_o = nullptr;      // [F][D]
  double* omega_t = nullptr;
  float* tcos = nullptr;
  float* tsin = nullptr;
  float *rcos = nullptr, *rsin = nullptr, *ccos = nullptr, *csin = nullptr;
  float2* rope_rows = nullptr;   // [d/2][nbuf*T] (cos, sin) of the pass (bf16 QKV epilogue)
  int* dev_err = nullptr;

  CUtensorMap tm_hop{}, tm_xop{}, tm_o{}, tm_win{}, tm_whead{};
  std::vector<CUtensorMap> tm_wqkv, tm_wout;
  CUtensorMap tm_s_hop{}, tm_s_xop{}, tm_s_o{};
  // e4m3 projections: weight codes [rows, D] with per-row scales, and the
  // codes / scales of the operand quantized before each projection
  std::vector<void*> wq8, wo8;
  std::vector<float*> wq8s, wo8s;
  void* a8 = nullptr;       // uint8 [max(nbuf*T, F)][D]
  float* a8s = nullptr;     // [max(nbuf*T, F)]
  CUtensorMap tm_a8{}, tm_s_a8{};
  std::vector<CUtensorMap> tm_wq8, tm_wo8;
  AttnMaps maps_stream{};   // q = q_rope; k[0]/v[0] = ring; k[1] = sink K roped per buffer; v[1] = sink V
  AttnMaps maps_sink{};     // q = s_q; k[0] = s_k; v[0] = sink V

  Scheduler sched;
  bool sink_set = false;
  bool started = false;
  long long launches = 0;
  std::string err;

  // debug capture (per slot)
  bool capture = false;
  float* cap_xin = nullptr;   // [S][T][C]
  float* cap_xout = nullptr;  // [S][T][C]
  float* cap_v = nullptr;     // [S][T][C]
  float* cap_vall = nullptr;  // [nbuf*T][C]
  float* cap_oall = nullptr;  // fp32 [nbuf*T][D] (attention output before rounding)
  float* cap_h = nullptr;     // [S][L+1][T][D]
  void* cap_q = nullptr;      // attn type [S][L][H][T][d]
  float* cap_o = nullptr;     // fp32 [S][L][T][D]
  void* cap_sk = nullptr;     // attn type [S][L][H][F][d]
  float* cap_sink_h = nullptr;  // fp32 [L][F][D] sink residual entering each layer
  void* cap_hop = nullptr;      // bf16 [S][L][T][D] normalised residual entering each QKV projection
  void* cap_sink_hop = nullptr; // bf16 [L][F][D] the same in the last sink pass
  float* cap_hmid = nullptr;    // LA_BLOCK_DIT: fp32 [S][L][T][D] residual after the attention sub-block
  float* cap_hx = nullptr;      // audio: fp32 [S][L][T][D] residual after the cross-attention
  void* cap_xq = nullptr;       // audio: attn [S][L][H][T][d] cross-attention q
  void* cap_xk = nullptr;       // audio: attn [S][L][H][A][d] the block's audio K / V
  void* cap_xv = nullptr;
  float* cap_xo = nullptr;      // audio: fp32 [S][L][T][D] cross-attention output
  float* cap_xoall = nullptr;   // audio, bf16 streams: fp32 [nbuf*T][D] cross-attention output of a pass
  void* cap_u = nullptr;        // LA_BLOCK_DIT: dtype [S][L][T][Fffn] GELU output
  bool cap_sink_valid = false;
  std::vector<int> cap_valid;  // per slot: captured in the last call

  bool prof = false;
  std::vector<ProfEvent> prof_events;
  std::vector<cudaEvent_t> ev_pool;
  size_t ev_next = 0;
};

namespace {

const char* kStatus[] = {"ok", "invalid argument", "invalid state", "out of device memory", "CUDA error",
                         "device error"};

int fail(la_stream* s, int code, const std::string& msg) {
  if (s) s->err = msg;
  return code;
}

#define CU(call)                                                                                \
  do {                                                                                          \
    cudaError_t e_ = (call);                                                                    \
    if (e_ != cudaSuccess)                                                                      \
      return fail(s, LA_ECUDA, std::string(#call) + ": " + cudaGetErrorString(e_));            \
  } while (0)

cudaEvent_t next_event(la_stream* s) {
  if (s->ev_next >= s->ev_pool.size()) {
    cudaEvent_t e;
    cudaEventCreate(&e);
    s->ev_pool.push_back(e);
  }
  return s->ev_pool[s->ev_next++];
}

// Launch wrapper: counts launches and, when profiling, brackets with events.
template <typename Fn>
int launch(la_stream* s, int kind, Fn&& fn) {
  cudaEvent_t a = nullptr, b = nullptr;
  if (s->prof) {
    a = next_event(s);
    b = next_event(s);
    cudaEventRecord(a, s->st);
  }
  const cudaError_t e = fn();
  if (e != cudaSuccess) return fail(s, LA_ECUDA, std::string("kernel launch: ") + cudaGetErrorString(e));
  ++s->launches;
  if (s->prof) {
    cudaEventRecord(b, s->st);
    s->prof_events.push_back({kind, a, b});
  }
  return LA_OK;
}

int dalloc(la_stream* s, void** p, size_t bytes) {
  if (bytes == 0) bytes = 16;
  const cudaError_t e = cudaMalloc(p, bytes);
  if (e != cudaSuccess) return fail(s, LA_ENOMEM, std::string("cudaMalloc: ") + cudaGetErrorString(e));
  s->allocs.push_back(*p);
  const cudaError_t z = cudaMemsetAsync(*p, 0, bytes, s->st);
  if (z != cudaSuccess) return fail(s, LA_ECUDA, std::string("cudaMemsetAsync: ") + cudaGetErrorString(z));
  return LA_OK;
}

#define DALLOC(ptr, bytes)                                                              \
  do {                                                                                  \
    void* p_ = nullptr;                                                                 \
    int r_ = dalloc(s, &p_, (bytes));                                                   \
    if (r_ != LA_OK) return r_;                                                         \
    ptr = reinterpret_cast<decltype(ptr)>(p_);                                          \
  } while (0)

// The fields the tick scheduler reads (shared by stream creation and la_sched_trace).
int validate_schedule(const la_config* c, std::string& msg) {
  if (c->frames_per_block < 1 || c->frames_per_block > LA_MAX_FPB) { msg = "frames_per_block out of range"; return LA_EINVAL; }
  if (c->window_blocks < 0 || c->window_blocks > LA_MAX_WINDOW) { msg = "window_blocks out of range"; return LA_EINVAL; }
  if (c->num_steps < 1 || c->num_steps > LA_MAX_STEPS) { msg = "num_steps out of range"; return LA_EINVAL; }
  if (c->sink_mode != LA_SINK_FIXED && c->sink_mode != LA_SINK_AAS) { msg = "bad sink_mode"; return LA_EINVAL; }
  if (c->schedule != LA_SCHED_PIPELINED && c->schedule != LA_SCHED_SEQUENTIAL && c->schedule != LA_SCHED_SLOT) {
    msg = "bad schedule";
    return LA_EINVAL;
  }
  if (c->schedule == LA_SCHED_SLOT) {
    if (c->slot_index < 0 || c->slot_index >= c->num_steps) { msg = "slot_index must name one of the steps"; return LA_EINVAL; }
    if (c->cache_mode != LA_CACHE_TIMESTEP) { msg = "a slot stream keeps its own step's cache (timestep forcing)"; return LA_EINVAL; }
  }
  if (c->cache_mode != LA_CACHE_TIMESTEP && c->cache_mode != LA_CACHE_CLEAN_REFRESH &&
      c->cache_mode != LA_CACHE_FIXED_STEP) {
    msg = "bad cache_mode";
    return LA_EINVAL;
  }
  if (c->cache_mode == LA_CACHE_FIXED_STEP) {
    if (c->schedule != LA_SCHED_SEQUENTIAL) { msg = "the fixed-noise cache runs in the sequential schedule"; return LA_EINVAL; }
    if (c->cache_step < 0 || c->cache_step >= c->num_steps) { msg = "cache_step must name one of the steps"; return LA_EINVAL; }
  }
  if (c->cache_mode == LA_CACHE_CLEAN_REFRESH && c->schedule != LA_SCHED_SEQUENTIAL) {
    msg = "the clean-cache refresh needs the sequential schedule";
    return LA_EINVAL;
  }
  if (c->rolling_rope != 0 && c->rolling_rope != 1) { msg = "rolling_rope must be 0 or 1"; return LA_EINVAL; }
  if (c->sink_offset_frames < 0) { msg = "sink_offset_frames must be >= 0"; return LA_EINVAL; }
  return LA_OK;
}

int validate(const la_config* c, const la_weights* w, std::string& msg) {
  if (!c || !w) { msg = "NULL config or weights"; return LA_EINVAL; }
  if (c->num_layers < 1 || c->hidden < 1 || c->heads < 1 || c->head_dim < 2 || c->latent_ch < 1 ||
      c->grid_h < 1 || c->grid_w < 1) { msg = "sizes must be positive"; return LA_EINVAL; }
  if (static_cast<long long>(c->heads) * c->head_dim != c->hidden) { msg = "hidden != heads*head_dim"; return LA_EINVAL; }
  if (c->head_dim % 8 != 0 || c->head_dim > 128) { msg = "head_dim must be a multiple of 8 and <= 128"; return LA_EINVAL; }
  if (c->dtype == LA_BF16 && c->head_dim != 128) { msg = "the bf16 path needs head_dim == 128"; return LA_EINVAL; }
  if (c->dtype != LA_BF16 && c->dtype != LA_FP32) { msg = "dtype must be LA_BF16 or LA_FP32"; return LA_EINVAL; }
  if (c->sink_frames != 1) { msg = "sink_frames must be 1"; return LA_EINVAL; }
  if (const int r = validate_schedule(c, msg); r != LA_OK) return r;
  if (!c->timesteps) { msg = "NULL timesteps"; return LA_EINVAL; }
  for (int i = 0; i <= c->num_steps; ++i)
    if (!std::isfinite(c->timesteps[i])) { msg = "timesteps must be finite"; return LA_EINVAL; }
  for (int i = 0; i < c->num_steps; ++i)
    if (!(c->timesteps[i + 1] < c->timesteps[i])) { msg = "timesteps must be strictly descending"; return LA_EINVAL; }
  const int P = c->head_dim / 2;
  if (c->rope_split[0] < 0 || c->rope_split[1] < 0 || c->rope_split[2] < 0 ||
      c->rope_split[0] + c->rope_split[1] + c->rope_split[2] != P) { msg = "rope_split must sum to head_dim/2"; return LA_EINVAL; }
  if (c->rope_split[0] > LA_MAX_PT) { msg = "too many temporal rotary pairs"; return LA_EINVAL; }
  if (!(c->rope_theta > 0.0) || !std::isfinite(c->rope_theta)) { msg = "rope_theta must be positive"; return LA_EINVAL; }
  if (c->proj_fp8 != 0 && c->proj_fp8 != 1) { msg = "proj_fp8 must be 0 or 1"; return LA_EINVAL; }
  if (c->proj_fp8 && c->dtype != LA_BF16) { msg = "e4m3 projections need the bf16 stream"; return LA_EINVAL; }
  if (c->attn_fp8 != 0 && c->attn_fp8 != 1) { msg = "attn_fp8 must be 0 or 1"; return LA_EINVAL; }
  if (c->block_kind != LA_BLOCK_ATTN && c->block_kind != LA_BLOCK_DIT) { msg = "bad block_kind"; return LA_EINVAL; }
  if (c->block_kind == LA_BLOCK_DIT) {
    if (c->ffn_dim < 32 || c->ffn_dim % 32 != 0 || c->ffn_dim > (1 << 20)) { msg = "ffn_dim must be a multiple of 32"; return LA_EINVAL; }
    if (c->proj_fp8 || c->attn_fp8) { msg = "the DiT block runs without the e4m3 modes"; return LA_EINVAL; }
  }
  if (c->audio_tokens != 0) {
    if (c->block_kind != LA_BLOCK_DIT) { msg = "the audio cross-attention needs the DiT block"; return LA_EINVAL; }
    if (c->audio_tokens < 0 || c->audio_tokens > 65536) { msg = "bad audio_tokens"; return LA_EINVAL; }
    if (c->audio_dim < 8 || c->audio_dim % 8 != 0 || c->audio_dim > 65536) { msg = "audio_dim must be a multiple of 8"; return LA_EINVAL; }
  }
  if (c->attn_fp8 && (c->dtype != LA_BF16 || c->head_dim != 128)) {
    msg = "e4m3 attention needs the bf16 stream and head_dim 128";
    return LA_EINVAL;
  }
  if ((w->w_in == nullptr) != (w->w_head == nullptr)) { msg = "w_in and w_head must both be set or both NULL"; return LA_EINVAL; }
  if (w->w_in == nullptr && c->latent_ch != c->hidden) { msg = "identity projections need latent_ch == hidden"; return LA_EINVAL; }
  if (!w->w_qkv || !w->w_out) { msg = "NULL layer weight arrays"; return LA_EINVAL; }
  for (int l = 0; l < c->num_layers; ++l)
    if (!w->w_qkv[l] || !w->w_out[l]) { msg = "NULL layer weight"; return LA_EINVAL; }
  if (c->block_kind == LA_BLOCK_DIT) {
    if (!w->w_ffn1 || !w->w_ffn2 || !w->ada) { msg = "the DiT block needs w_ffn1, w_ffn2 and ada"; return LA_EINVAL; }
    for (int l = 0; l < c->num_layers; ++l)
      if (!w->w_ffn1[l] || !w->w_ffn2[l]) { msg = "NULL FFN weight"; return LA_EINVAL; }
  }
  if (c->block_kind == LA_BLOCK_DIT && c->audio_tokens > 0) {
    if (!w->w_qc || !w->w_kvc || !w->w_oc) { msg = "the audio cross-attention needs w_qc, w_kvc and w_oc"; return LA_EINVAL; }
    for (int l = 0; l < c->num_layers; ++l)
      if (!w->w_qc[l] || !w->w_kvc[l] || !w->w_oc[l]) { msg = "NULL cross-attention weight"; return LA_EINVAL; }
  }
  if (c->dtype == LA_BF16) {
    if (c->hidden % 64 != 0) { msg = "bf16 path needs hidden % 64 == 0"; return LA_EINVAL; }
    if (w->w_in && (c->latent_ch % 32 != 0)) { msg = "bf16 path needs latent_ch % 32 == 0"; return LA_EINVAL; }
  }
  if (c->latent_ch % 4 != 0) { msg = "latent_ch must be a multiple of 4"; return LA_EINVAL; }
  const long long T = static_cast<long long>(c->frames_per_block) * c->grid_h * c->grid_w;
  if (T * c->num_steps > (1LL << 30)) { msg = "block too large"; return LA_EINVAL; }
  return LA_OK;
}

// ---------------------------------------------------------------------------
// Pass execution
// ---------------------------------------------------------------------------
RopeArgs rope_args(la_stream* s) {
  RopeArgs a{};
  a.T = s->T; a.F = s->F; a.H = s->H; a.d = s->d; a.D = s->D; a.grid_w = s->cfg.grid_w; a.fpb = s->fpb;
  a.pt = s->pt; a.ph = s->ph; a.pw = s->pw;
  a.tcos = s->tcos; a.tsin = s->tsin; a.rcos = s->rcos; a.rsin = s->rsin; a.ccos = s->ccos; a.csin = s->csin;
  a.E = s->E;
  return a;
}

int gemm(la_stream* s, int kind, const CUtensorMap* tmA, const CUtensorMap* tmB, const void* A32, const void* W32,
         const GemmEpiParams& ep, int M, int N, int K) {
  if (s->bf16) {
    const int bn = gemm_tc_pick_bn(N);
    return launch(s, kind, [&] { return launch_gemm_tc(*tmA, *tmB, ep, M, N, K, bn, s->dev_err, s->num_sms, s->st); });
  }
  return launch(s, kind, [&] {
    return launch_gemm_f32(static_cast<const float*>(A32), static_cast<const float*>(W32), ep, M, N, K, s->st);
  });
}

// The folded norm: a GEMM whose epilogue produces the residual leaves each row's
// partial sums of squares; one that consumes its operand scales rows by 1 / rms.
void fold_out(la_stream* s, GemmEpiParams& e) {
  if (!s->fold) return;
  e.ssq_out = s->ssq;
  e.ssq_ld = s->ssq_ld;
}
void fold_in(la_stream* s, GemmEpiParams& e) {
  if (!s->fold) return;
  e.ssq_in = s->ssq;
  e.ssq_ld = s->ssq_ld;
  e.ssq_n = static_cast<float>(s->D);
}

GemmEpiParams epi(int kind, void* out, float* h32, long long ld) {
  GemmEpiParams e{};
  e.kind = kind;
  e.out = out;
  e.h32 = h32;
  e.ld = ld;
  e.rows_per_group = 1 << 30;
  for (int i = 0; i < LA_MAX_STEPS; ++i) e.active[i] = 1;
  return e;
}

// A projection on e4m3 operands: the bf16 operand a [M, K] is quantized per
// row into a8 / a8s, then the GEMM runs on its codes and the layer's weight
// codes (tmW, per-row scales wscale) with the scales ahead of the epilogue.
int proj_fp8(la_stream* s, int kind, const void* a, const CUtensorMap& tmA8, const CUtensorMap& tmW,
             const float* wscale, GemmEpiParams ep, int M, int N, int K, const QkvRopeParams* qp = nullptr) {
  int r = launch(s, LA_KIND_OTHER, [&] { return launch_quant_rows_e4m3(1, a, M, K, s->a8, s->a8s, s->st); });
  if (r != LA_OK) return r;
  ep.row_scale = s->a8s;
  ep.col_scale = wscale;
  const int bn = gemm_tc_pick_bn(N);
  return launch(s, kind, [&] {
    return launch_gemm_tc_fp8(tmA8, tmW, ep, M, N, K, bn, s->dev_err, s->num_sms, s->st, qp);
  });
}

char* elem(void* base, long long idx, size_t es) { return static_cast<char*>(base) + idx * static_cast<long long>(es); }

int capture_pass(la_stream* s, const PassDesc& pd, int layer) {
  // copy the intermediates of every active buffer into its slot's capture area
  const size_t eq = s->eq;
  const long long T = s->T, D = s->D, H = s->H, d = s->d, F = s->F, L = s->L;
  const float* o32 = s->bf16 ? s->cap_oall : static_cast<const float*>(s->attn_o);
  for (int ai = 0; ai < pd.nactive; ++ai) {
    const int buf = pd.active_buf[ai];
    const int slot = pd.step[buf];   // capture areas are per denoising step
    if (slot >= s->S) continue;      // the clean-cache refresh is not captured
    if (layer < 0) {
      CU(cudaMemcpyAsync(s->cap_h + (static_cast<long long>(slot) * (L + 1)) * T * D, s->h32 + buf * T * D,
                         T * D * 4, cudaMemcpyDeviceToDevice, s->st));
      continue;
    }
    CU(cudaMemcpyAsync(s->cap_h + (static_cast<long long>(slot) * (L + 1) + layer + 1) * T * D, s->h32 + buf * T * D,
                       T * D * 4, cudaMemcpyDeviceToDevice, s->st));
    CU(cudaMemcpyAsync(elem(s->cap_q, (static_cast<long long>(slot) * L + layer) * H * T * d, eq),
                       elem(s->q_rope, buf * H * T * d, eq), H * T * d * eq, cudaMemcpyDeviceToDevice, s->st));
    CU(cudaMemcpyAsync(s->cap_o + (static_cast<long long>(slot) * L + layer) * T * D, o32 + buf * T * D, T * D * 4,
                       cudaMemcpyDeviceToDevice, s->st));
    CU(cudaMemcpyAsync(elem(s->cap_sk, (static_cast<long long>(slot) * L + layer) * H * F * d, eq),
                       elem(s->sk_rope, (static_cast<long long>(layer) * s->nbuf + buf) * H * F * d, eq), H * F * d * eq,
                       cudaMemcpyDeviceToDevice, s->st));
  }
  return LA_OK;
}

constexpr float kRmsEps = 1e-6f;
// |value| of an e4m3 attention operand <= kAttnActBound * sqrt(D) * the norm of its
// weight row (or rotary pair of rows): an RMS-normalised row has norm <= sqrt(D),
// and rounding it to the GEMM operand (bf16, or per-row e4m3) grows each element by
// at most a factor 1 + 2^-4 plus e4m3's subnormal floor; 1.07 covers both.
constexpr double kAttnActBound = 1.07;

// Per-token RMS normalisation of the residual into the next GEMM's operand.
int normalise(la_stream* s, const float* h, long long rows, void* op_bf16, float* op_f32) {
  return launch(s, LA_KIND_OTHER, [&] {
    return launch_rmsnorm(h, rows, s->D, kRmsEps, s->bf16 ? op_bf16 : nullptr, op_f32, s->st);
  });
}

// LA_BLOCK_DIT: AdaLN vector k (0 shift1, 1 scale1, 2 gate1, 3 shift2, 4 scale2,
// 5 gate2) of layer l at timestep index t (num_steps: the t = 0 set).
const float* ada_vec(const la_stream* s, int l, int t, int k) {
  return s->ada + ((static_cast<long long>(l) * (s->S + 1) + t) * 6 + k) * s->D;
}

// The AdaLN-modulated norm of each row group g with the vectors (k_shift, k_shift+1)
// of timestep index tidx[g].
int normalise_mod(la_stream* s, const float* h, long long rows, int rows_per_group, const int* tidx, int ngroups,
                  int l, int k_shift, void* op_bf16, float* op_f32) {
  ModArgs m{};
  m.rows_per_group = rows_per_group;
  for (int g = 0; g < LA_MAX_STEPS; ++g) {
    const int t = g < ngroups ? tidx[g] : 0;
    m.shift[g] = ada_vec(s, l, t, k_shift);
    m.scale[g] = ada_vec(s, l, t, k_shift + 1);
  }
  return launch(s, LA_KIND_OTHER, [&] {
    return launch_rmsnorm_mod(h, rows, s->D, kRmsEps, m, s->bf16 ? op_bf16 : nullptr, op_f32, s->st);
  });
}

// Turn a residual epilogue into the gated one with AdaLN vector k per row group.
void set_gates(const la_stream* s, GemmEpiParams& e, int rows_per_group, const int* tidx, int ngroups, int l, int k) {
  e.kind = EPI_RESID_GATED;
  e.rows_per_group = rows_per_group;
  for (int g = 0; g < LA_MAX_STEPS; ++g) e.gate[g] = ada_vec(s, l, g < ngroups ? tidx[g] : 0, k);
}

// The DiT block's FFN sub-block on h (rows of `rows_per_group` per group):
// m = modulated norm (shift2, scale2) into the operand buffer, u = gelu(m W1^T),
// h += gate2 * (u W2^T).  tm_op / op32 / tm_u describe the operand and u buffers.
int ffn_block(la_stream* s, float* h, long long rows, int rows_per_group, const int* tidx, int ngroups, int l,
              void* op_bf16, float* op32, const CUtensorMap* tm_op, const CUtensorMap* tm_u,
              const std::function<void()>& after_gelu) {
  const int D = s->D, F = s->Fffn;
  int r;
  if ((r = normalise_mod(s, h, rows, rows_per_group, tidx, ngroups, l, 3, op_bf16, s->bf16 ? nullptr : op32)) != LA_OK)
    return r;
  GemmEpiParams e1 = epi(EPI_GELU, s->ffn_u, nullptr, F);
  if ((r = gemm(s, LA_KIND_FFN, tm_op, &s->tm_w1[l], op32, s->w_ffn1[l], e1, static_cast<int>(rows), F, D)) != LA_OK)
    return r;
  if (after_gelu) after_gelu();
  GemmEpiParams e2 = epi(EPI_RESID, nullptr, h, D);
  set_gates(s, e2, rows_per_group, tidx, ngroups, l, 5);
  return gemm(s, LA_KIND_FFN, tm_u, &s->tm_w2[l], s->ffn_u, s->w_ffn2[l], e2, static_cast<int>(rows), D, F);
}

// The audio K / V of every layer for the block entering buffer buf: [k | v] =
// audio W_kvc^T (fp32), split into the buffer's head-major planes.
int audio_kv(la_stream* s, const float* audio, int buf) {
  const int D = s->D, H = s->H, d = s->d, A = s->A;
  int r;
  if (s->bf16 && (r = launch(s, LA_KIND_CROSS, [&] {
                    return launch_cvt_bf16(audio, s->audio_op, static_cast<long long>(A) * s->Da, s->st);
                  })) != LA_OK)
    return r;
  for (int l = 0; l < s->L; ++l) {
    GemmEpiParams e = epi(s->bf16 ? EPI_STORE32 : EPI_STORE, s->kv32, nullptr, 2LL * D);
    if ((r = gemm(s, LA_KIND_CROSS, &s->tm_audio_op, &s->tm_wkvc[l], audio, s->w_kvc[l], e, A, 2 * D, s->Da)) !=
        LA_OK)
      return r;
    const long long plane = (static_cast<long long>(l) * s->nbuf + buf) * H * A * d;
    for (int part = 0; part < 2; ++part)
      if ((r = launch(s, LA_KIND_CROSS, [&] {
             return launch_split_heads(s->bf16, s->kv32, A, A, H, d, 2LL * D, static_cast<long long>(part) * D,
                                       elem(part ? s->audio_v : s->audio_k, plane, s->ea), 1.0f, s->st);
           })) != LA_OK)
        return r;
  }
  return LA_OK;
}

// The DiT block's audio cross-attention sub-block of layer l on the pass's rows:
// q = n(h) W_qc^T (split into heads; bf16 streams times log2(e)/sqrt(d)),
// attention over each active buffer's audio K / V, h += O W_oc^T.
int cross_block(la_stream* s, const PassDesc& pd, int l, int rows) {
  const int T = s->T, D = s->D, H = s->H, d = s->d, S = s->S;
  int r;
  if ((r = normalise(s, s->h32, rows, s->hop, s->bf16 ? nullptr : s->hn32)) != LA_OK) return r;
  GemmEpiParams eq = epi(s->bf16 ? EPI_STORE32 : EPI_STORE, s->qc32, nullptr, D);
  if ((r = gemm(s, LA_KIND_CROSS, &s->tm_hop, &s->tm_wqc[l], s->hn32, s->w_qc[l], eq, rows, D, D)) != LA_OK) return r;
  const float scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(d)));
  if ((r = launch(s, LA_KIND_CROSS, [&] {
         return launch_split_heads(s->bf16, s->qc32, rows, T, H, d, D, 0, s->qc_heads, s->bf16 ? scale_log2 : 1.0f,
                                   s->st);
       })) != LA_OK)
    return r;
  AttnParams ap{};
  ap.Tq = T; ap.H = H; ap.d = d;
  ap.scale_log2 = scale_log2;
  ap.q_prescaled = s->bf16 ? 1 : 0;
  ap.out = s->xo_buf; ap.out_ld = D; ap.err = s->dev_err;
  ap.out32 = (s->bf16 && s->capture) ? s->cap_xoall : nullptr;
  ap.qbase = s->qc_heads;
  ap.kbase[0] = s->audio_k; ap.vbase[0] = s->audio_v; ap.krows[0] = s->A; ap.vrows[0] = s->A;
  ap.ngroups = pd.nactive;
  for (int ai = 0; ai < pd.nactive; ++ai) {
    const int buf = pd.active_buf[ai];
    AttnGroup& g = ap.g[ai];
    g.q_slice = buf;
    g.out_row0 = buf * T;
    g.nseg = 1;
    const int plane = l * s->nbuf + buf;
    g.seg[0] = AttnSeg{0, 0, plane, plane, s->A};
  }
  if (s->bf16) {
    if ((r = launch(s, LA_KIND_CROSS, [&] { return launch_attention_tc(s->maps_cross, ap, s->st); })) != LA_OK) return r;
  } else if ((r = launch(s, LA_KIND_CROSS, [&] { return launch_attn_f32(ap, s->st); })) != LA_OK) {
    return r;
  }
  GemmEpiParams eo = epi(EPI_RESID, nullptr, s->h32, D);
  if ((r = gemm(s, LA_KIND_CROSS, &s->tm_xo, &s->tm_woc[l], s->xo_buf, s->w_oc[l], eo, rows, D, D)) != LA_OK) return r;
  if (s->capture) {
    const float* o32 = s->bf16 ? s->cap_xoall : static_cast<const float*>(s->xo_buf);
    const long long HTd = static_cast<long long>(H) * T * d, HAd = static_cast<long long>(H) * s->A * d;
    for (int ai = 0; ai < pd.nactive; ++ai) {
      const int buf = pd.active_buf[ai];
      if (pd.step[buf] >= S) continue;
      const long long at = static_cast<long long>(pd.step[buf]) * s->L + l;
      const long long plane = static_cast<long long>(l) * s->nbuf + buf;
      CU(cudaMemcpyAsync(s->cap_hx + at * T * D, s->h32 + static_cast<long long>(buf) * T * D,
                         static_cast<size_t>(T) * D * 4, cudaMemcpyDeviceToDevice, s->st));
      CU(cudaMemcpyAsync(s->cap_xo + at * T * D, o32 + static_cast<long long>(buf) * T * D,
                         static_cast<size_t>(T) * D * 4, cudaMemcpyDeviceToDevice, s->st));
      CU(cudaMemcpyAsync(elem(s->cap_xq, at * HTd, s->ea), elem(s->qc_heads, buf * HTd, s->ea), HTd * s->ea,
                         cudaMemcpyDeviceToDevice, s->st));
      CU(cudaMemcpyAsync(elem(s->cap_xk, at * HAd, s->ea), elem(s->audio_k, plane * HAd, s->ea), HAd * s->ea,
                         cudaMemcpyDeviceToDevice, s->st));
      CU(cudaMemcpyAsync(elem(s->cap_xv, at * HAd, s->ea), elem(s->audio_v, plane * HAd, s->ea), HAd * s->ea,
                         cudaMemcpyDeviceToDevice, s->st));
    }
  }
  return LA_OK;
}

// One grouped pass over nbuf buffers (rows = nbuf*T) with the active ones in pd.
int run_pass(la_stream* s, const PassDesc& pd) {
  const int T = s->T, D = s->D, C = s->C, H = s->H, d = s->d, F = s->F, S = s->S, E = s->E;
  const int rows = pd.nbuf * T;
  int r;
  if (s->capture) {
    for (int ai = 0; ai < pd.nactive; ++ai) {
      const int buf = pd.active_buf[ai];
      if (pd.step[buf] >= S) continue;
      CU(cudaMemcpyAsync(s->cap_xin + static_cast<long long>(pd.step[buf]) * T * C,
                         s->xs + static_cast<long long>(buf) * T * C, static_cast<size_t>(T) * C * 4,
                         cudaMemcpyDeviceToDevice, s->st));
    }
  }
  if ((r = launch(s, LA_KIND_OTHER, [&] {
         return launch_rope_ttab(pd, s->fpb, s->pt, s->omega_t, s->tcos, s->tsin, s->st);
       })) != LA_OK)
    return r;
  if (s->bf16 && (r = launch(s, LA_KIND_OTHER, [&] {
                    return launch_rope_rows(pd, rope_args(s), s->rope_rows, static_cast<long long>(s->nbuf) * T,
                                            s->st);
                  })) != LA_OK)
    return r;

  // in-projection into the fp32 residual stream, then its normalised operand
  if (s->id_in) {
    if ((r = launch(s, LA_KIND_IN_PROJ, [&] {
           return launch_in_identity(s->bf16, s->xs, s->h32, nullptr, static_cast<long long>(rows) * D, s->st);
         })) != LA_OK)
      return r;
  } else {
    if (s->bf16 &&
        (r = launch(s, LA_KIND_IN_PROJ, [&] {
           return launch_cvt_bf16(s->xs, s->xop, static_cast<long long>(rows) * C, s->st);
         })) != LA_OK)
      return r;
    GemmEpiParams e = epi(EPI_SET32, s->fold ? s->hop : nullptr, s->h32, D);
    fold_out(s, e);
    if ((r = gemm(s, LA_KIND_IN_PROJ, &s->tm_xop, &s->tm_win, s->xs, s->w_in, e, rows, D, C)) != LA_OK) return r;
  }
  if (s->capture && (r = capture_pass(s, pd, -1)) != LA_OK) return r;
  // timestep index of each buffer's AdaLN vectors (the DiT block)
  int tidx[LA_MAX_STEPS] = {};
  for (int b = 0; b < pd.nbuf; ++b) tidx[b] = pd.active[b] ? std::min(pd.step[b], S) : 0;
  if (!s->dit && !s->fold && (r = normalise(s, s->h32, rows, s->hop, s->bf16 ? nullptr : s->hn32)) != LA_OK)
    return r;

  RopeArgs ra = rope_args(s);
  AttnParams ap{};
  ap.Tq = T; ap.H = H; ap.d = d;
  ap.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(d)));
  ap.out = s->attn_o; ap.out_ld = D; ap.err = s->dev_err;
  ap.qbase = s->q_rope;
  ap.kbase[0] = s->ring_k; ap.vbase[0] = s->ring_v; ap.krows[0] = T; ap.vrows[0] = T;
  ap.kbase[1] = s->sk_rope; ap.vbase[1] = s->sink_v; ap.krows[1] = F; ap.vrows[1] = F;
  ap.ngroups = pd.nactive;

  // per-block re-rope of every layer's sink K (fp32 -> bf16, e4m3 or fp32), once
  // per active buffer: the sink's positions depend on the buffer's block only
  ra.sink_k = s->sink_k;
  ra.sink_k_rope = s->sk_rope;
  ra.nl = s->L;
  ra.nb = s->nbuf;
  ra.fp8_inv = s->afp8 ? s->attn_inv : nullptr;
  if ((r = launch(s, LA_KIND_ROPE, [&] {
         return launch_sink_rerope(s->bf16 ? (s->afp8 ? 2 : 1) : 0, pd, ra, s->st);
       })) != LA_OK)
    return r;

  QkvRopeParams qp{};
  qp.T = T; qp.F = F; qp.H = H; qp.d = d; qp.D = D; qp.E = E; qp.grid_w = s->cfg.grid_w;
  qp.pt = s->pt; qp.ph = s->ph;
  qp.qscale = ap.scale_log2;
  for (int i = 0; i < LA_MAX_STEPS; ++i) {
    qp.active[i] = pd.active[i];
    qp.slot[i] = pd.slot[i];
    qp.write_entry[i] = pd.write_entry[i];
  }
  qp.tcos = s->tcos; qp.tsin = s->tsin; qp.rcos = s->rcos; qp.rsin = s->rsin; qp.ccos = s->ccos; qp.csin = s->csin;
  qp.q_rope = s->q_rope; qp.ring_k = s->ring_k; qp.ring_v = s->ring_v;
  qp.rowtab = s->rope_rows;
  qp.rowtab_ld = static_cast<long long>(s->nbuf) * T;
  ap.out32 = (s->bf16 && s->capture) ? s->cap_oall : nullptr;
  ap.q_prescaled = s->bf16 ? 1 : 0;

  for (int l = 0; l < s->L; ++l) {
    if (s->dit &&
        (r = normalise_mod(s, s->h32, rows, T, tidx, pd.nbuf, l, 0, s->hop, s->bf16 ? nullptr : s->hn32)) != LA_OK)
      return r;
    if (s->capture && s->bf16) {
      // the normalised residual as the QKV projection consumes it (bf16)
      for (int ai = 0; ai < pd.nactive; ++ai) {
        const int buf = pd.active_buf[ai];
        if (pd.step[buf] >= S) continue;
        CU(cudaMemcpyAsync(elem(s->cap_hop, (static_cast<long long>(pd.step[buf]) * s->L + l) * T * D, s->es),
                           elem(s->hop, static_cast<long long>(buf) * T * D, s->es), static_cast<size_t>(T) * D * s->es,
                           cudaMemcpyDeviceToDevice, s->st));
      }
    }
    ra.qkv = s->qkv; ra.q_rope = s->q_rope; ra.ring_k = s->ring_k; ra.ring_v = s->ring_v;
    ra.ring_slice0 = static_cast<long long>(l) * S * E;
    if (s->afp8) {
      const long long so = static_cast<long long>(l) * 3 * H;
      ra.fp8_inv = qp.fp8_inv = s->attn_inv + so;
      ap.fp8 = 1;
      ap.sq = s->attn_sc + so;
      ap.sk = s->attn_sc + so + H;
      ap.sv = s->attn_sc + so + 2 * H;
    }
    if (s->bf16) {
      // QKV projection with Rolling RoPE + ring append fused into the epilogue
      qp.ring_slice0 = ra.ring_slice0;
      GemmEpiParams eq = epi(EPI_QKV_ROPE, nullptr, nullptr, 3LL * D);
      fold_in(s, eq);
      const int bn = gemm_tc_pick_bn(3 * D);
      if (s->fp8) {
        if ((r = proj_fp8(s, LA_KIND_QKV_GEMM, s->hop, s->tm_a8, s->tm_wq8[l], s->wq8s[l], eq, rows, 3 * D, D, &qp)) !=
            LA_OK)
          return r;
      } else if ((r = launch(s, LA_KIND_QKV_GEMM, [&] {
                    return launch_gemm_tc(s->tm_hop, s->tm_wqkv[l], eq, rows, 3 * D, D, bn, s->dev_err, s->num_sms,
                                          s->st, &qp);
                  })) != LA_OK) {
        return r;
      }
    } else {
      GemmEpiParams eq = epi(EPI_STORE, s->qkv, nullptr, 3LL * D);
      if ((r = gemm(s, LA_KIND_QKV_GEMM, &s->tm_hop, &s->tm_wqkv[l], s->hn32, s->w_qkv[l], eq, rows, 3 * D, D)) !=
          LA_OK)
        return r;
      if ((r = launch(s, LA_KIND_ROPE, [&] { return launch_rope_append(0, pd, ra, s->st); })) != LA_OK) return r;
    }
    // block-causal attention: [sink | window oldest first | self]
    for (int ai = 0; ai < pd.nactive; ++ai) {
      const int buf = pd.active_buf[ai];
      AttnGroup& g = ap.g[ai];
      g.q_slice = buf;
      g.out_row0 = buf * T;
      int ns = 0;
      g.seg[ns++] = AttnSeg{1, 1, l * s->nbuf + buf, l, F};
      const long long base = static_cast<long long>(l) * S * E + static_cast<long long>(pd.slot[buf]) * E;
      const long long wbase = static_cast<long long>(l) * S * E + static_cast<long long>(pd.win_slot[buf]) * E;
      for (int w = 0; w < pd.nwin[buf]; ++w)
        g.seg[ns++] = AttnSeg{0, 0, static_cast<int>(wbase + pd.win_entry[buf][w]),
                              static_cast<int>(wbase + pd.win_entry[buf][w]), T};
      g.seg[ns++] = AttnSeg{0, 0, static_cast<int>(base + pd.write_entry[buf]),
                            static_cast<int>(base + pd.write_entry[buf]), T};
      g.nseg = ns;
    }
    if (s->bf16) {
      if ((r = launch(s, LA_KIND_ATTN, [&] { return launch_attention_tc(s->maps_stream, ap, s->st); })) != LA_OK) return r;
    } else {
      if ((r = launch(s, LA_KIND_ATTN, [&] { return launch_attn_f32(ap, s->st); })) != LA_OK) return r;
    }
    // output projection + residual, then the next operand (next layer or head)
    GemmEpiParams eo = epi(EPI_RESID, s->fold ? s->hop : nullptr, s->h32, D);
    fold_out(s, eo);
    if (s->dit) set_gates(s, eo, T, tidx, pd.nbuf, l, 2);
    if (s->fp8) {
      if ((r = proj_fp8(s, LA_KIND_OUT_GEMM, s->attn_o, s->tm_a8, s->tm_wo8[l], s->wo8s[l], eo, rows, D, D)) != LA_OK)
        return r;
    } else if ((r = gemm(s, LA_KIND_OUT_GEMM, &s->tm_o, &s->tm_wout[l], s->attn_o, s->w_out[l], eo, rows, D, D)) !=
               LA_OK)
      return r;
    if (s->dit) {
      // the FFN sub-block (captures: the residual entering it, the GELU output)
      int cerr = LA_OK;
      auto cap = [&](bool gelu) {
        for (int ai = 0; ai < pd.nactive && s->capture; ++ai) {
          const int buf = pd.active_buf[ai];
          if (pd.step[buf] >= S) continue;
          const long long at = static_cast<long long>(pd.step[buf]) * s->L + l;
          cudaError_t ce = gelu ? cudaMemcpyAsync(elem(s->cap_u, at * T * s->Fffn, s->es),
                                                  elem(s->ffn_u, static_cast<long long>(buf) * T * s->Fffn, s->es),
                                                  static_cast<size_t>(T) * s->Fffn * s->es, cudaMemcpyDeviceToDevice, s->st)
                                : cudaMemcpyAsync(s->cap_hmid + at * T * D, s->h32 + static_cast<long long>(buf) * T * D,
                                                  static_cast<size_t>(T) * D * 4, cudaMemcpyDeviceToDevice, s->st);
          if (ce != cudaSuccess) cerr = fail(s, LA_ECUDA, cudaGetErrorString(ce));
        }
      };
      cap(false);
      if (s->cross && (r = cross_block(s, pd, l, rows)) != LA_OK) return r;
      if ((r = ffn_block(s, s->h32, rows, T, tidx, pd.nbuf, l, s->hop, s->hn32, &s->tm_hop, &s->tm_u,
                         [&] { cap(true); })) != LA_OK)
        return r;
      if (cerr != LA_OK) return cerr;
    }
    if (s->capture && (r = capture_pass(s, pd, l)) != LA_OK) return r;
    const bool last = l == s->L - 1;
    const bool want_f32 = !s->bf16 || (last && s->id_head);
    if ((!s->dit || last) && !s->fold &&
        (r = normalise(s, s->h32, rows, (s->bf16 && !(last && s->id_head)) ? s->hop : nullptr,
                       want_f32 ? s->hn32 : nullptr)) != LA_OK)
      return r;
  }

  // velocity head + Euler update x += (t_{i+1} - t_i) v, per buffer
  float* vtap = s->capture ? s->cap_vall : nullptr;
  if (s->id_head) {
    if ((r = launch(s, LA_KIND_HEAD, [&] {
           return launch_euler(s->xs, s->hn32, rows, C, T, pd.dt, pd.active, vtap, s->st);
         })) != LA_OK)
      return r;
  } else {
    GemmEpiParams e = epi(EPI_EULER, nullptr, s->xs, C);
    e.rows_per_group = T;
    for (int i = 0; i < LA_MAX_STEPS; ++i) {
      e.dt[i] = pd.dt[i];
      e.active[i] = pd.active[i];
    }
    e.vtap = vtap;
    fold_in(s, e);
    if ((r = gemm(s, LA_KIND_HEAD, &s->tm_hop, &s->tm_whead, s->hn32, s->w_head, e, rows, C, D)) != LA_OK)
      return r;
  }
  if (s->capture) {
    for (int ai = 0; ai < pd.nactive; ++ai) {
      const int buf = pd.active_buf[ai];
      if (pd.step[buf] >= S) continue;
      const long long so = static_cast<long long>(pd.step[buf]) * T * C, bo = static_cast<long long>(buf) * T * C;
      CU(cudaMemcpyAsync(s->cap_xout + so, s->xs + bo, static_cast<size_t>(T) * C * 4, cudaMemcpyDeviceToDevice, s->st));
      CU(cudaMemcpyAsync(s->cap_v + so, s->cap_vall + bo, static_cast<size_t>(T) * C * 4, cudaMemcpyDeviceToDevice, s->st));
      s->cap_valid[pd.step[buf]] = 1;
    }
  }
  return LA_OK;
}

// The sink frame through the layers: stores per-layer un-roped K and V.
int run_sink(la_stream* s) {
  const int F = s->F, D = s->D, C = s->C, H = s->H, d = s->d;
  int r;
  PassDesc pd{};
  pd.nbuf = 1;
  pd.nactive = 1;
  pd.active_buf[0] = 0;
  pd.active[0] = 1;
  pd.frame_tpos[0] = -s->cfg.sink_offset_frames;
  pd.sink_tpos[0] = -s->cfg.sink_offset_frames;
  if ((r = launch(s, LA_KIND_OTHER, [&] {
         return launch_rope_ttab(pd, s->fpb, s->pt, s->omega_t, s->tcos, s->tsin, s->st);
       })) != LA_OK)
    return r;
  if (s->id_in) {
    if ((r = launch(s, LA_KIND_IN_PROJ, [&] {
           return launch_in_identity(s->bf16, s->sink_x, s->s_h32, nullptr, static_cast<long long>(F) * D, s->st);
         })) != LA_OK)
      return r;
  } else {
    if (s->bf16 && (r = launch(s, LA_KIND_IN_PROJ, [&] {
                      return launch_cvt_bf16(s->sink_x, s->s_xop, static_cast<long long>(F) * C, s->st);
                    })) != LA_OK)
      return r;
    GemmEpiParams e = epi(EPI_SET32, nullptr, s->s_h32, D);
    if ((r = gemm(s, LA_KIND_IN_PROJ, &s->tm_s_xop, &s->tm_win, s->sink_x, s->w_in, e, F, D, C)) != LA_OK) return r;
  }
  RopeArgs ra = rope_args(s);
  ra.T = F;
  AttnParams ap{};
  ap.Tq = F; ap.H = H; ap.d = d;
  ap.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(d)));
  ap.out = s->s_o; ap.out_ld = D; ap.err = s->dev_err;
  ap.qbase = s->s_q;
  ap.q_prescaled = s->bf16 ? 1 : 0;
  ap.kbase[0] = s->s_k; ap.krows[0] = F;
  ap.vbase[0] = s->sink_v; ap.vrows[0] = F;
  ap.ngroups = 1;
  for (int l = 0; l < s->L; ++l) {
    if (s->capture) {
      CU(cudaMemcpyAsync(s->cap_sink_h + static_cast<long long>(l) * F * D, s->s_h32,
                         static_cast<size_t>(F) * D * 4, cudaMemcpyDeviceToDevice, s->st));
      s->cap_sink_valid = true;
    }
    const int tS[1] = {s->S};   // the sink is a clean frame: the DiT block's t = 0 AdaLN set
    if (s->dit) {
      if ((r = normalise_mod(s, s->s_h32, F, F, tS, 1, l, 0, s->s_hop, s->bf16 ? nullptr : s->s_hn32)) != LA_OK)
        return r;
    } else if ((r = normalise(s, s->s_h32, F, s->s_hop, s->bf16 ? nullptr : s->s_hn32)) != LA_OK) {
      return r;
    }
    if (s->capture && s->bf16)
      CU(cudaMemcpyAsync(elem(s->cap_sink_hop, static_cast<long long>(l) * F * D, s->es), s->s_hop,
                         static_cast<size_t>(F) * D * s->es, cudaMemcpyDeviceToDevice, s->st));
    GemmEpiParams eq = epi(s->bf16 ? EPI_STORE32 : EPI_STORE, s->s_qkv, nullptr, 3LL * D);
    if (s->fp8) {
      if ((r = proj_fp8(s, LA_KIND_QKV_GEMM, s->s_hop, s->tm_s_a8, s->tm_wq8[l], s->wq8s[l], eq, F, 3 * D, D)) !=
          LA_OK)
        return r;
    } else if ((r = gemm(s, LA_KIND_QKV_GEMM, &s->tm_s_hop, &s->tm_wqkv[l], s->s_hn32, s->w_qkv[l], eq, F, 3 * D,
                         D)) != LA_OK) {
      return r;
    }
    ra.qkv = s->s_qkv;
    float* kraw = s->sink_k + static_cast<long long>(l) * H * F * d;
    void* vraw = elem(s->sink_v, static_cast<long long>(l) * H * F * d, s->ea);
    uint8_t* v8 = s->afp8 ? s->sink_v8 + static_cast<long long>(l) * H * F * d : nullptr;
    ra.fp8_inv = s->afp8 ? s->attn_inv + static_cast<long long>(l) * 3 * H : nullptr;
    if ((r = launch(s, LA_KIND_ROPE, [&] {
           return launch_sink_qkv(s->bf16, ra, s->bf16 ? ap.scale_log2 : 1.0f, kraw, vraw, s->s_q, s->s_k, s->st,
                                  v8);
         })) != LA_OK)
      return r;
    if (l == s->L - 1) break;   // the last layer's sink output feeds nothing
    AttnGroup& g = ap.g[0];
    g.q_slice = 0;
    g.out_row0 = 0;
    g.nseg = 1;
    g.seg[0] = AttnSeg{0, 0, 0, l, F};
    if (s->bf16) {
      if ((r = launch(s, LA_KIND_ATTN, [&] { return launch_attention_tc(s->maps_sink, ap, s->st); })) != LA_OK) return r;
    } else {
      if ((r = launch(s, LA_KIND_ATTN, [&] { return launch_attn_f32(ap, s->st); })) != LA_OK) return r;
    }
    GemmEpiParams eo = epi(EPI_RESID, nullptr, s->s_h32, D);
    if (s->dit) set_gates(s, eo, F, tS, 1, l, 2);
    if (s->fp8) {
      if ((r = proj_fp8(s, LA_KIND_OUT_GEMM, s->s_o, s->tm_s_a8, s->tm_wo8[l], s->wo8s[l], eo, F, D, D)) != LA_OK)
        return r;
    } else if ((r = gemm(s, LA_KIND_OUT_GEMM, &s->tm_s_o, &s->tm_wout[l], s->s_o, s->w_out[l], eo, F, D, D)) !=
               LA_OK) {
      return r;
    }
    if (s->dit && (r = ffn_block(s, s->s_h32, F, F, tS, 1, l, s->s_hop, s->s_hn32, &s->tm_s_hop, &s->tm_s_u,
                                 nullptr)) != LA_OK)
      return r;
  }
  return LA_OK;
}

// Buffer buf runs block b at step `step` (num_steps: a clean-cache refresh, dt 0)
// reading and writing ring `ring`.
void fill_pass_slot(la_stream* s, PassDesc& pd, int buf, int ring, int step, long long b, int write_entry) {
  const int W = s->cfg.window_blocks;
  pd.active[buf] = 1;
  pd.active_buf[pd.nactive++] = buf;
  pd.slot[buf] = ring;
  pd.win_slot[buf] = step < s->S ? s->sched.window_ring(step) : ring;
  pd.step[buf] = step;
  pd.block[buf] = static_cast<int>(b);
  pd.write_entry[buf] = write_entry;
  const int nw = static_cast<int>(std::min<long long>(b, W));
  pd.nwin[buf] = nw;
  for (int w = 0; w < nw; ++w) pd.win_entry[buf][w] = static_cast<int>((b - nw + w) % s->E);
  pd.frame_tpos[buf] = static_cast<int>(s->fpb * b);
  pd.sink_tpos[buf] = s->sched.sink_tpos_of(b);
  pd.dt[buf] = step < s->S ? s->ts[step + 1] - s->ts[step] : 0.0f;
}

int step_impl(la_stream* s, const float* x_new, float* x_out, int64_t* finished_block, cudaMemcpyKind in_kind,
              cudaMemcpyKind out_kind, const float* audio_new = nullptr) {
  if (!s) return LA_EINVAL;
  if (!finished_block || !x_out) return fail(s, LA_EINVAL, "NULL x_out or finished_block");
  if (s->cross && x_new && !audio_new)
    return fail(s, LA_EINVAL, "this stream has the audio cross-attention: la_denoise_step_av with the block's audio");
  if (!s->cross && audio_new) return fail(s, LA_EINVAL, "this stream has no audio cross-attention");
  if (!s->sink_set) return fail(s, LA_ESTATE, "la_set_sink must be called first");
  const bool has_new = x_new != nullptr;
  const bool pipelined = s->cfg.schedule == LA_SCHED_PIPELINED;
  if (!pipelined && !has_new) return fail(s, LA_EINVAL, "the sequential schedule needs x_new");
  if (has_new && (s->sched.blocks_in + 1) * static_cast<long long>(s->fpb) > 0x7FFFFFF0LL)
    return fail(s, LA_ESTATE, "block index exceeds the int32 RoPE position range");
  std::vector<std::pair<int, long long>> run;
  std::vector<long long> next_held;
  long long finished = -1;
  s->sched.plan(has_new, run, finished, next_held);
  const long long TC = static_cast<long long>(s->T) * s->C;
  const long long new_block = s->sched.blocks_in;
  s->sched.begin(has_new, next_held);
  s->started = true;
  if (s->capture) std::fill(s->cap_valid.begin(), s->cap_valid.end(), 0);
  int r;
  if (pipelined) {
    if (has_new)
      CU(cudaMemcpyAsync(s->xs + (new_block % s->S) * TC, x_new, TC * 4, in_kind, s->st));
    if (has_new && s->cross && (r = audio_kv(s, audio_new, static_cast<int>(new_block % s->S))) != LA_OK) return r;
    PassDesc pd{};
    pd.nbuf = s->S;
    for (auto& [slot, b] : run) {
      const int e = s->sched.append(slot, b);
      fill_pass_slot(s, pd, static_cast<int>(b % s->S), slot, slot, b, e);
    }
    if (pd.nactive > 0 && (r = run_pass(s, pd)) != LA_OK) return r;
    if (finished >= 0)
      CU(cudaMemcpyAsync(x_out, s->xs + (finished % s->S) * TC, TC * 4, out_kind, s->st));
  } else {
    CU(cudaMemcpyAsync(s->xs, x_new, TC * 4, in_kind, s->st));
    if (s->cross && (r = audio_kv(s, audio_new, 0)) != LA_OK) return r;
    for (auto& [slot, b] : run) {
      PassDesc pd{};
      pd.nbuf = 1;
      const int e = s->sched.append(slot, b);
      fill_pass_slot(s, pd, 0, s->sched.ring_of(slot), slot, b, e);
      if ((r = run_pass(s, pd)) != LA_OK) return r;
    }
    if (s->sched.clean) {
      // clean-cache refresh: the finished latent through the stack once more
      // (dt 0 leaves it unchanged); its K/V replace the block's cache entry
      PassDesc pd{};
      pd.nbuf = 1;
      const int e = s->sched.append_refresh(finished);
      fill_pass_slot(s, pd, 0, 0, s->S, finished, e);
      if ((r = run_pass(s, pd)) != LA_OK) return r;
    }
    CU(cudaMemcpyAsync(x_out, s->xs, TC * 4, out_kind, s->st));
  }
  if (s->sched.finish(finished)) {
    // Adaptive Attention Sink: frame 0 of finished block 0 becomes the sink
    const float* src = s->xs + (pipelined ? (finished % s->S) * TC : 0);
    CU(cudaMemcpyAsync(s->sink_x, src, static_cast<size_t>(s->F) * s->C * 4, cudaMemcpyDeviceToDevice, s->st));
    if ((r = run_sink(s)) != LA_OK) return r;
  }
  *finished_block = finished;
  return LA_OK;
}

int alloc_capture(la_stream* s) {
  if (s->cap_xin) return LA_OK;
  const long long S = s->S, T = s->T, C = s->C, D = s->D, L = s->L, H = s->H, d = s->d, F = s->F;
  DALLOC(s->cap_xin, S * T * C * 4);
  DALLOC(s->cap_xout, S * T * C * 4);
  DALLOC(s->cap_v, S * T * C * 4);
  DALLOC(s->cap_vall, static_cast<long long>(s->nbuf) * T * C * 4);
  DALLOC(s->cap_oall, static_cast<long long>(s->nbuf) * T * D * 4);
  DALLOC(s->cap_h, S * (L + 1) * T * D * 4);
  DALLOC(s->cap_q, S * L * H * T * d * s->eq);
  DALLOC(s->cap_o, S * L * T * D * 4);
  DALLOC(s->cap_sk, S * L * H * F * d * s->eq);
  DALLOC(s->cap_sink_h, L * F * D * 4);
  if (s->bf16) {
    DALLOC(s->cap_hop, S * L * T * D * s->es);
    DALLOC(s->cap_sink_hop, L * F * D * s->es);
  }
  if (s->dit) {
    DALLOC(s->cap_hmid, S * L * T * D * 4);
    DALLOC(s->cap_u, S * L * T * s->Fffn * static_cast<long long>(s->es));
  }
  if (s->cross) {
    DALLOC(s->cap_hx, S * L * T * D * 4);
    DALLOC(s->cap_xo, S * L * T * D * 4);
    DALLOC(s->cap_xq, S * L * H * T * d * s->ea);
    DALLOC(s->cap_xk, S * L * H * s->A * d * s->ea);
    DALLOC(s->cap_xv, S * L * H * s->A * d * s->ea);
    if (s->bf16) DALLOC(s->cap_xoall, static_cast<long long>(s->nbuf) * T * D * 4);
  }
  s->cap_valid.assign(s->S, 0);
  return LA_OK;
}

void free_all(la_stream* s) {
  for (void* p : s->allocs) cudaFree(p);
  s->allocs.clear();
  for (auto e : s->ev_pool) cudaEventDestroy(e);
  s->ev_pool.clear();
}

}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

const char* la_status_string(int status) {
  if (status > 0 || status < -5) return "unknown status";
  return kStatus[-status];
}

const char* la_last_error(const la_stream* s) {
  if (!s) return "no stream";
  return s->err.c_str();
}

int la_stream_create(const la_config* cfg, const la_weights* w, void* cuda_stream, la_stream** out) {
  if (!out) return LA_EINVAL;
  *out = nullptr;
  std::string msg;
  int v = validate(cfg, w, msg);
  if (v != LA_OK) {
    std::fprintf(stderr, "la_stream_create: %s\n", msg.c_str());
    return v;
  }
  la_stream* s = new (std::nothrow) la_stream();
  if (!s) return LA_ENOMEM;
  auto bail = [&](int code) {
    if (!s->err.empty()) std::fprintf(stderr, "la_stream_create: %s\n", s->err.c_str());
    free_all(s);
    delete s;
    return code;
  };
  s->cfg = *cfg;
  for (int i = 0; i <= cfg->num_steps; ++i) s->ts[i] = cfg->timesteps[i];
  s->cfg.timesteps = s->ts;
  s->S = cfg->num_steps; s->E = cfg->window_blocks + 1; s->F = cfg->grid_h * cfg->grid_w;
  s->fpb = cfg->frames_per_block; s->T = s->fpb * s->F; s->D = cfg->hidden; s->C = cfg->latent_ch;
  s->H = cfg->heads; s->d = cfg->head_dim; s->L = cfg->num_layers;
  s->pt = cfg->rope_split[0]; s->ph = cfg->rope_split[1]; s->pw = cfg->rope_split[2];
  s->bf16 = cfg->dtype == LA_BF16; s->es = s->bf16 ? 2 : 4; s->ea = s->es;
  s->fp8 = s->bf16 && cfg->proj_fp8;
  s->afp8 = s->bf16 && cfg->attn_fp8;
  s->dit = cfg->block_kind == LA_BLOCK_DIT;
  s->Fffn = s->dit ? cfg->ffn_dim : 0;
  s->cross = s->dit && cfg->audio_tokens > 0;
  s->A = s->cross ? cfg->audio_tokens : 0;
  s->Da = s->cross ? cfg->audio_dim : 0;
  s->eq = s->afp8 ? 1 : s->ea;
  s->id_in = w->w_in == nullptr; s->id_head = w->w_head == nullptr;
  s->fold = s->bf16 && !s->dit && !s->id_in && !s->id_head;
  s->ssq_ld = s->fold ? ceil_div_i(s->D, gemm_tc_pick_bn(s->D)) : 0;
  s->nbuf = cfg->schedule == LA_SCHED_PIPELINED ? s->S : 1;
  s->st = static_cast<cudaStream_t>(cuda_stream);
  s->w_in = w->w_in; s->w_head = w->w_head;
  s->w_qkv.assign(w->w_qkv, w->w_qkv + s->L);
  s->w_out.assign(w->w_out, w->w_out + s->L);
  if (s->dit) {
    s->w_ffn1.assign(w->w_ffn1, w->w_ffn1 + s->L);
    s->w_ffn2.assign(w->w_ffn2, w->w_ffn2 + s->L);
    s->ada = w->ada;
  }
  if (s->cross) {
    s->w_qc.assign(w->w_qc, w->w_qc + s->L);
    s->w_kvc.assign(w->w_kvc, w->w_kvc + s->L);
    s->w_oc.assign(w->w_oc, w->w_oc + s->L);
  }
  s->sched.init(s->cfg);

  cudaError_t e = cudaGetDevice(&s->device);
  if (e != cudaSuccess) { s->err = cudaGetErrorString(e); return bail(LA_ECUDA); }
  cudaDeviceProp prop{};
  e = cudaGetDeviceProperties(&prop, s->device);
  if (e != cudaSuccess) { s->err = cudaGetErrorString(e); return bail(LA_ECUDA); }
  if (prop.major != 10) { s->err = "this library is built for sm_100 (B200) devices"; return bail(LA_ECUDA); }
  s->num_sms = prop.multiProcessorCount;
  if (s->bf16 && !tmap_init(s->err)) return bail(LA_ECUDA);

  // memory plan, checked before allocating
  const long long T = s->T, D = s->D, C = s->C, F = s->F, H = s->H, d = s->d, L = s->L, S = s->S, E = s->E;
  const long long NB = s->nbuf;
  const size_t es = s->es, ea = s->ea, eq = s->eq;
  const long long need = NB * T * C * 4 + NB * T * D * 4 + (s->bf16 ? NB * T * D * es : 0) +
                         ((!s->bf16 || s->id_head) ? NB * T * D * 4 : 0) + F * D * 4 +
                         (s->bf16 && !s->id_in ? NB * T * C * 2 : 0) + (s->bf16 ? 0 : NB * T * 3 * D * 4) +
                         NB * T * D * eq + NB * T * D * es + L * NB * H * F * d * eq + 2 * L * S * E * H * T * d * eq +
                         L * H * F * d * (4 + ea) + F * C * 4 + F * D * 4 + F * D * es * 2 + F * C * 2 +
                         F * 3 * D * 4 + 2 * H * F * d * ea + (s->afp8 ? L * H * F * d + L * 3 * H * 8 : 0) +
                         (s->dit ? std::max(NB * T, F) * s->Fffn * static_cast<long long>(es) : 0) +
                         (s->cross ? static_cast<long long>(s->A) * (s->Da * 2 + 2 * D * 4) + 2 * L * NB * s->A * D * ea +
                                         NB * T * D * (4 + ea + es)
                                   : 0) +
                         (64 << 20);
  size_t free_b = 0, total_b = 0;
  e = cudaMemGetInfo(&free_b, &total_b);
  if (e != cudaSuccess) { s->err = cudaGetErrorString(e); return bail(LA_ECUDA); }
  if (static_cast<long long>(free_b) < need) {
    s->err = "stream needs " + std::to_string(need >> 20) + " MiB, " + std::to_string(free_b >> 20) + " MiB free";
    return bail(LA_ENOMEM);
  }
  int r;
#define ALLOC_OR_BAIL(ptr, bytes)                  \
  do {                                             \
    void* p_ = nullptr;                            \
    r = dalloc(s, &p_, (bytes));                   \
    if (r != LA_OK) return bail(r);                \
    ptr = reinterpret_cast<decltype(ptr)>(p_);     \
  } while (0)
  ALLOC_OR_BAIL(s->xs, NB * T * C * 4);
  ALLOC_OR_BAIL(s->h32, NB * T * D * 4);
  if (!s->bf16 || s->id_head) ALLOC_OR_BAIL(s->hn32, NB * T * D * 4);
  if (s->bf16) ALLOC_OR_BAIL(s->hop, NB * T * D * es); else s->hop = s->hn32;
  if (s->bf16 && !s->id_in) ALLOC_OR_BAIL(s->xop, NB * T * C * 2);
  if (!s->bf16) ALLOC_OR_BAIL(s->qkv, NB * T * 3 * D * 4);
  ALLOC_OR_BAIL(s->q_rope, NB * T * D * eq);
  ALLOC_OR_BAIL(s->attn_o, NB * T * D * es);
  if (s->fold) ALLOC_OR_BAIL(s->ssq, NB * T * s->ssq_ld * 4);
  ALLOC_OR_BAIL(s->sk_rope, L * NB * H * F * d * eq);
  ALLOC_OR_BAIL(s->ring_k, L * S * E * H * T * d * eq);
  ALLOC_OR_BAIL(s->ring_v, L * S * E * H * T * d * eq);
  ALLOC_OR_BAIL(s->sink_k, L * H * F * d * 4);
  ALLOC_OR_BAIL(s->sink_v, L * H * F * d * ea);
  if (s->dit) ALLOC_OR_BAIL(s->ffn_u, std::max(NB * T, F) * s->Fffn * static_cast<long long>(es));
  if (s->cross) {
    const long long Aa = s->A;
    if (s->bf16) ALLOC_OR_BAIL(s->audio_op, Aa * s->Da * 2);
    ALLOC_OR_BAIL(s->kv32, Aa * 2 * D * 4);
    ALLOC_OR_BAIL(s->audio_k, L * NB * Aa * D * ea);
    ALLOC_OR_BAIL(s->audio_v, L * NB * Aa * D * ea);
    ALLOC_OR_BAIL(s->qc32, NB * T * D * 4);
    ALLOC_OR_BAIL(s->qc_heads, NB * T * D * ea);
    ALLOC_OR_BAIL(s->xo_buf, NB * T * D * es);
  }
  if (s->afp8) {
    ALLOC_OR_BAIL(s->sink_v8, L * H * F * d);
    ALLOC_OR_BAIL(s->attn_sc, L * 3 * H * 4);
    ALLOC_OR_BAIL(s->attn_inv, L * 3 * H * 4);
  }
  ALLOC_OR_BAIL(s->sink_x, F * C * 4);
  ALLOC_OR_BAIL(s->s_h32, F * D * 4);
  if (s->bf16) ALLOC_OR_BAIL(s->s_hop, F * D * es);
  else { ALLOC_OR_BAIL(s->s_hn32, F * D * 4); s->s_hop = s->s_hn32; }
  if (s->bf16 && !s->id_in) ALLOC_OR_BAIL(s->s_xop, F * C * 2);
  ALLOC_OR_BAIL(s->s_qkv, F * 3 * D * 4);
  ALLOC_OR_BAIL(s->s_q, H * F * d * ea);
  ALLOC_OR_BAIL(s->s_k, H * F * d * ea);
  ALLOC_OR_BAIL(s->s_o, F * D * es);
  ALLOC_OR_BAIL(s->omega_t, std::max(1, s->pt) * 8);
  ALLOC_OR_BAIL(s->tcos, LA_MAX_STEPS * LA_TROWS * LA_MAX_PT * 4);
  ALLOC_OR_BAIL(s->tsin, LA_MAX_STEPS * LA_TROWS * LA_MAX_PT * 4);
  ALLOC_OR_BAIL(s->rcos, std::max(1, cfg->grid_h * s->ph) * 4);
  ALLOC_OR_BAIL(s->rsin, std::max(1, cfg->grid_h * s->ph) * 4);
  ALLOC_OR_BAIL(s->ccos, std::max(1, cfg->grid_w * s->pw) * 4);
  if (s->bf16) ALLOC_OR_BAIL(s->rope_rows, static_cast<long long>(d / 2) * NB * T * 8);
  ALLOC_OR_BAIL(s->csin, std::max(1, cfg->grid_w * s->pw) * 4);
  ALLOC_OR_BAIL(s->dev_err, 64);

  // RoPE frequencies and spatial tables, fp64 on the host
  {
    const double theta = cfg->rope_theta;
    std::vector<double> om(std::max(1, s->pt));
    for (int j = 0; j < s->pt; ++j) om[j] = std::pow(theta, -static_cast<double>(j) / s->pt);
    std::vector<float> rc(std::max(1, cfg->grid_h * s->ph)), rs(rc.size()), cc(std::max(1, cfg->grid_w * s->pw)),
        cs(cc.size());
    for (int rr = 0; rr < cfg->grid_h; ++rr)
      for (int j = 0; j < s->ph; ++j) {
        const double a = rr * std::pow(theta, -static_cast<double>(j) / s->ph);
        rc[rr * s->ph + j] = static_cast<float>(std::cos(a));
        rs[rr * s->ph + j] = static_cast<float>(std::sin(a));
      }
    for (int c = 0; c < cfg->grid_w; ++c)
      for (int j = 0; j < s->pw; ++j) {
        const double a = c * std::pow(theta, -static_cast<double>(j) / s->pw);
        cc[c * s->pw + j] = static_cast<float>(std::cos(a));
        cs[c * s->pw + j] = static_cast<float>(std::sin(a));
      }
    e = cudaMemcpy(s->omega_t, om.data(), om.size() * 8, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(s->rcos, rc.data(), rc.size() * 4, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(s->rsin, rs.data(), rs.size() * 4, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(s->ccos, cc.data(), cc.size() * 4, cudaMemcpyHostToDevice);
    if (e == cudaSuccess) e = cudaMemcpy(s->csin, cs.data(), cs.size() * 4, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) { s->err = cudaGetErrorString(e); return bail(LA_ECUDA); }
  }

  if (s->bf16) {
    bool ok = true;
    const int bn_qkv = gemm_tc_pick_bn(3 * s->D), bn_d = gemm_tc_pick_bn(s->D), bn_c = gemm_tc_pick_bn(s->C);
    ok = ok && tmap_2d_bf16(&s->tm_hop, s->hop, NB * T, D, D, 128, s->err);
    ok = ok && tmap_2d_bf16(&s->tm_o, s->attn_o, NB * T, D, D, 128, s->err);
    ok = ok && tmap_2d_bf16(&s->tm_s_hop, s->s_hop, F, D, D, 128, s->err);
    ok = ok && tmap_2d_bf16(&s->tm_s_o, s->s_o, F, D, D, 128, s->err);
    s->tm_wqkv.resize(L);
    s->tm_wout.resize(L);
    for (int l = 0; l < L && ok; ++l) {
      ok = ok && tmap_2d_bf16(&s->tm_wqkv[l], s->w_qkv[l], 3 * D, D, D, gemm_tc_b_box_rows(bn_qkv), s->err);
      ok = ok && tmap_2d_bf16(&s->tm_wout[l], s->w_out[l], D, D, D, gemm_tc_b_box_rows(bn_d), s->err);
    }
    if (s->dit) {
      const long long Ff = s->Fffn;
      ok = ok && tmap_2d_bf16(&s->tm_u, s->ffn_u, NB * T, Ff, Ff, 128, s->err);
      ok = ok && tmap_2d_bf16(&s->tm_s_u, s->ffn_u, F, Ff, Ff, 128, s->err);
      s->tm_w1.resize(L);
      s->tm_w2.resize(L);
      for (int l = 0; l < L && ok; ++l) {
        ok = ok && tmap_2d_bf16(&s->tm_w1[l], s->w_ffn1[l], Ff, D, D, gemm_tc_b_box_rows(gemm_tc_pick_bn(s->Fffn)), s->err);
        ok = ok && tmap_2d_bf16(&s->tm_w2[l], s->w_ffn2[l], D, Ff, Ff, gemm_tc_b_box_rows(bn_d), s->err);
      }
    }
    if (s->cross) {
      const long long Aa = s->A;
      ok = ok && tmap_2d_bf16(&s->tm_audio_op, s->audio_op, Aa, s->Da, s->Da, 128, s->err);
      ok = ok && tmap_2d_bf16(&s->tm_xo, s->xo_buf, NB * T, D, D, 128, s->err);
      s->tm_wqc.resize(L);
      s->tm_wkvc.resize(L);
      s->tm_woc.resize(L);
      for (int l = 0; l < L && ok; ++l) {
        ok = ok && tmap_2d_bf16(&s->tm_wqc[l], s->w_qc[l], D, D, D, gemm_tc_b_box_rows(bn_d), s->err);
        ok = ok && tmap_2d_bf16(&s->tm_wkvc[l], s->w_kvc[l], 2 * D, s->Da, s->Da, gemm_tc_b_box_rows(gemm_tc_pick_bn(2 * s->D)), s->err);
        ok = ok && tmap_2d_bf16(&s->tm_woc[l], s->w_oc[l], D, D, D, gemm_tc_b_box_rows(bn_d), s->err);
      }
      ok = ok && tmap_planes_bf16(&s->maps_cross.q, s->qc_heads, d, T, H, NB, s->err);
      ok = ok && tmap_planes_bf16(&s->maps_cross.k[0], s->audio_k, d, Aa, H, L * NB, s->err);
      ok = ok && tmap_planes_bf16(&s->maps_cross.v[0], s->audio_v, d, Aa, H, L * NB, s->err);
    }
    if (!s->id_in) {
      ok = ok && tmap_2d_bf16(&s->tm_xop, s->xop, NB * T, C, C, 128, s->err);
      ok = ok && tmap_2d_bf16(&s->tm_s_xop, s->s_xop, F, C, C, 128, s->err);
      ok = ok && tmap_2d_bf16(&s->tm_win, s->w_in, D, C, C, gemm_tc_b_box_rows(bn_d), s->err);
      ok = ok && tmap_2d_bf16(&s->tm_whead, s->w_head, C, D, D, gemm_tc_b_box_rows(bn_c), s->err);
    }
    if (s->afp8) {
      ok = ok && tmap_planes_u8(&s->maps_stream.q, s->q_rope, d, T, H, NB, s->err);
      ok = ok && tmap_planes_u8(&s->maps_stream.k[0], s->ring_k, d, T, H, L * S * E, s->err);
      ok = ok && tmap_planes_u8(&s->maps_stream.v[0], s->ring_v, d, T, H, L * S * E, s->err);
      ok = ok && tmap_planes_u8(&s->maps_stream.k[1], s->sk_rope, d, F, H, L * NB, s->err);
      ok = ok && tmap_planes_u8(&s->maps_stream.v[1], s->sink_v8, d, F, H, L, s->err);
    } else {
      ok = ok && tmap_planes_bf16(&s->maps_stream.q, s->q_rope, d, T, H, NB, s->err);
      ok = ok && tmap_planes_bf16(&s->maps_stream.k[0], s->ring_k, d, T, H, L * S * E, s->err);
      ok = ok && tmap_planes_bf16(&s->maps_stream.v[0], s->ring_v, d, T, H, L * S * E, s->err);
      ok = ok && tmap_planes_bf16(&s->maps_stream.k[1], s->sk_rope, d, F, H, L * NB, s->err);
      ok = ok && tmap_planes_bf16(&s->maps_stream.v[1], s->sink_v, d, F, H, L, s->err);
    }
    ok = ok && tmap_planes_bf16(&s->maps_sink.q, s->s_q, d, F, H, 1, s->err);
    ok = ok && tmap_planes_bf16(&s->maps_sink.k[0], s->s_k, d, F, H, 1, s->err);
    ok = ok && tmap_planes_bf16(&s->maps_sink.v[0], s->sink_v, d, F, H, L, s->err);
    if (!ok) return bail(LA_ECUDA);
  }
  if (s->fp8) {
    // weights quantized once per output row; operand buffers for the projections
    const long long rows_max = std::max(NB * T, F);
    ALLOC_OR_BAIL(s->a8, rows_max * D);
    ALLOC_OR_BAIL(s->a8s, rows_max * 4);
    s->wq8.resize(L); s->wo8.resize(L); s->wq8s.resize(L); s->wo8s.resize(L);
    s->tm_wq8.resize(L); s->tm_wo8.resize(L);
    const int bn_qkv = gemm_tc_pick_bn(3 * s->D), bn_d = gemm_tc_pick_bn(s->D);
    bool ok = tmap_2d_u8(&s->tm_a8, s->a8, NB * T, D, D, 128, s->err) &&
              tmap_2d_u8(&s->tm_s_a8, s->a8, F, D, D, 128, s->err);
    for (int l = 0; l < L && ok; ++l) {
      ALLOC_OR_BAIL(s->wq8[l], 3 * D * D);
      ALLOC_OR_BAIL(s->wq8s[l], 3 * D * 4);
      ALLOC_OR_BAIL(s->wo8[l], D * D);
      ALLOC_OR_BAIL(s->wo8s[l], D * 4);
      e = launch_quant_rows_e4m3(1, s->w_qkv[l], 3 * D, D, s->wq8[l], s->wq8s[l], s->st);
      if (e == cudaSuccess) e = launch_quant_rows_e4m3(1, s->w_out[l], D, D, s->wo8[l], s->wo8s[l], s->st);
      if (e != cudaSuccess) { s->err = cudaGetErrorString(e); return bail(LA_ECUDA); }
      ok = tmap_2d_u8(&s->tm_wq8[l], s->wq8[l], 3 * D, D, D, bn_qkv, s->err) &&
           tmap_2d_u8(&s->tm_wo8[l], s->wo8[l], D, D, D, bn_d, s->err);
    }
    if (!ok) return bail(LA_ECUDA);
  }
  if (s->afp8) {
    // per-head e4m3 scales from the QKV weights as the projection uses them
    const float act_bound = static_cast<float>(kAttnActBound * std::sqrt(static_cast<double>(D)));
    for (int l = 0; l < L; ++l) {
      e = launch_attn_fp8_scales(s->fp8 ? s->wq8[l] : s->w_qkv[l], s->fp8 ? 1 : 0, s->fp8 ? s->wq8s[l] : nullptr,
                                 s->D, s->H, s->d, act_bound, s->attn_sc + static_cast<long long>(l) * 3 * H,
                                 s->attn_inv + static_cast<long long>(l) * 3 * H, s->st);
      if (e != cudaSuccess) { s->err = cudaGetErrorString(e); return bail(LA_ECUDA); }
    }
  }
  e = cudaStreamSynchronize(s->st);
  if (e != cudaSuccess) { s->err = cudaGetErrorString(e); return bail(LA_ECUDA); }
  *out = s;
  return LA_OK;
}

int la_set_sink(la_stream* s, const float* sink_latent) {
  if (!s) return LA_EINVAL;
  if (!sink_latent) return fail(s, LA_EINVAL, "NULL sink latent");
  if (s->started) return fail(s, LA_ESTATE, "the sink can only be set before the first step");
  CU(cudaMemcpyAsync(s->sink_x, sink_latent, static_cast<size_t>(s->F) * s->C * 4, cudaMemcpyDeviceToDevice, s->st));
  int r = run_sink(s);
  if (r != LA_OK) return r;
  s->sink_set = true;
  return LA_OK;
}

int la_replace_sink(la_stream* s, const float* sink_latent) {
  if (!s) return LA_EINVAL;
  if (!sink_latent) return fail(s, LA_EINVAL, "NULL sink latent");
  if (s->cfg.schedule != LA_SCHED_SLOT)
    return fail(s, LA_ESTATE, "la_replace_sink is for slot streams (the others replace the sink themselves)");
  if (!s->sink_set) return fail(s, LA_ESTATE, "la_set_sink must be called first");
  if (s->sched.sink_gen != 0) return fail(s, LA_ESTATE, "the sink is replaced once");
  CU(cudaMemcpyAsync(s->sink_x, sink_latent, static_cast<size_t>(s->F) * s->C * 4, cudaMemcpyDeviceToDevice, s->st));
  int r = run_sink(s);
  if (r != LA_OK) return r;
  s->sched.sink_gen = 1;
  return LA_OK;
}

int la_denoise_step(la_stream* s, const float* x_new, float* x_out, int64_t* finished_block) {
  return step_impl(s, x_new, x_out, finished_block, cudaMemcpyDeviceToDevice, cudaMemcpyDeviceToDevice);
}

int la_denoise_step_host(la_stream* s, const float* x_new_host, float* x_out_host, int64_t* finished_block) {
  return step_impl(s, x_new_host, x_out_host, finished_block, cudaMemcpyHostToDevice, cudaMemcpyDeviceToHost);
}

int la_denoise_step_av(la_stream* s, const float* x_new, const float* audio_new, float* x_out,
                       int64_t* finished_block) {
  if (s && (x_new == nullptr) != (audio_new == nullptr))
    return fail(s, LA_EINVAL, "x_new and audio_new must both be set or both NULL");
  return step_impl(s, x_new, x_out, finished_block, cudaMemcpyDeviceToDevice, cudaMemcpyDeviceToDevice, audio_new);
}

int la_synchronize(la_stream* s) {
  if (!s) return LA_EINVAL;
  CU(cudaStreamSynchronize(s->st));
  int code = 0;
  CU(cudaMemcpy(&code, s->dev_err, sizeof(int), cudaMemcpyDeviceToHost));
  if (code != 0) {
    cudaMemset(s->dev_err, 0, sizeof(int));
    return fail(s, LA_EDEVICE, "kernel raised device error " + std::to_string(code) +
                                   (code == LA_DEVERR_WAIT_TIMEOUT ? " (bounded wait timed out)" : ""));
  }
  return LA_OK;
}

int la_stream_destroy(la_stream* s) {
  if (!s) return LA_OK;
  cudaStreamSynchronize(s->st);
  free_all(s);
  delete s;
  return LA_OK;
}

int64_t la_index_state_size(const la_stream* s) { return s ? s->sched.state_size() : 0; }

int la_get_index_state(const la_stream* s, int32_t* host_buf, int64_t n) {
  if (!s || !host_buf || n < s->sched.state_size()) return LA_EINVAL;
  s->sched.export_state(host_buf);
  return LA_OK;
}

int64_t la_sched_state_size(const la_config* cfg) {
  std::string msg;
  if (!cfg || validate_schedule(cfg, msg) != LA_OK) return -1;
  return 4 + static_cast<int64_t>(cfg->num_steps) * (8 + 3 * (cfg->window_blocks + 1));
}

int la_sched_trace(const la_config* cfg, int32_t nticks, const uint8_t* has_new, int32_t* out, int64_t out_len) {
  std::string msg;
  if (!cfg || nticks < 0 || (nticks > 0 && (!has_new || !out))) return LA_EINVAL;
  if (validate_schedule(cfg, msg) != LA_OK) {
    std::fprintf(stderr, "la_sched_trace: %s\n", msg.c_str());
    return LA_EINVAL;
  }
  Scheduler sc;
  sc.init(*cfg);
  const long long n = sc.state_size();
  if (out_len < n * nticks) return LA_EINVAL;
  std::vector<std::pair<int, long long>> run;
  std::vector<long long> next_held;
  for (int k = 0; k < nticks; ++k) {
    // the scheduling calls of one la_denoise_step, in its order, without the passes
    const bool nw = has_new[k] != 0;
    if (!sc.pipelined && !nw) return LA_ESTATE;
    if (nw && (sc.blocks_in + 1) * static_cast<long long>(sc.fpb) > 0x7FFFFFF0LL) return LA_ESTATE;
    long long finished = -1;
    sc.plan(nw, run, finished, next_held);
    sc.begin(nw, next_held);
    for (auto& [slot, b] : run) sc.append(slot, b);
    if (!sc.pipelined && sc.clean) sc.append_refresh(finished);
    sc.finish(finished);
    sc.export_state(out + n * k);
  }
  return LA_OK;
}

int la_debug_capture(la_stream* s, int32_t enable) {
  if (!s) return LA_EINVAL;
  if (enable) {
    int r = alloc_capture(s);
    if (r != LA_OK) return r;
  }
  s->capture = enable != 0;
  return LA_OK;
}

int la_debug_tap(la_stream* s, int32_t what, int32_t layer, int32_t slot, void* dst, int64_t dst_bytes) {
  if (!s || !dst) return LA_EINVAL;
  const long long T = s->T, C = s->C, D = s->D, H = s->H, d = s->d, F = s->F, L = s->L, E = s->E, S = s->S;
  const size_t ea = s->ea, eq = s->eq;
  const bool per_layer = what == LA_TAP_H || what == LA_TAP_Q || what == LA_TAP_O || what == LA_TAP_RING_K ||
                         what == LA_TAP_RING_V || what == LA_TAP_SINK_K || what == LA_TAP_SINK_V ||
                         what == LA_TAP_SINK_KROPE || what == LA_TAP_SINK_H || what == LA_TAP_HOP ||
                         what == LA_TAP_SINK_HOP || what == LA_TAP_SINK_V8 || what == LA_TAP_ATTN_SCALES ||
                         what == LA_TAP_H_MID || what == LA_TAP_FFN_U || (what >= LA_TAP_H_CROSS && what <= LA_TAP_XO);
  if (per_layer && (layer < (what == LA_TAP_H ? -1 : 0) || layer >= L)) return fail(s, LA_EINVAL, "bad layer");
  if (slot < 0 || slot >= S) return fail(s, LA_EINVAL, "bad slot");
  const void* src = nullptr;
  long long bytes = 0;
  const bool xtap = what >= LA_TAP_H_CROSS && what <= LA_TAP_XO;
  const bool needs_capture = what <= LA_TAP_V || what == LA_TAP_SINK_KROPE || what == LA_TAP_HOP ||
                             what == LA_TAP_H_MID || what == LA_TAP_FFN_U || xtap;
  if (xtap && !s->cross) return fail(s, LA_EINVAL, "the cross-attention taps exist with audio only");
  if ((what == LA_TAP_H_MID || what == LA_TAP_FFN_U) && !s->dit)
    return fail(s, LA_EINVAL, "the FFN taps exist with the DiT block only");
  if ((what == LA_TAP_HOP || what == LA_TAP_SINK_HOP) && !s->bf16)
    return fail(s, LA_EINVAL, "the GEMM-operand taps exist in bf16 streams only");
  if ((what == LA_TAP_SINK_V8 || what == LA_TAP_ATTN_SCALES) && !s->afp8)
    return fail(s, LA_EINVAL, "the e4m3 attention taps exist with attn_fp8 only");
  if (needs_capture && (!s->cap_xin || s->cap_valid.empty() || !s->cap_valid[slot]))
    return fail(s, LA_ESTATE, "no capture of that slot in the last call");
  switch (what) {
    case LA_TAP_X_IN: src = s->cap_xin + slot * T * C; bytes = T * C * 4; break;
    case LA_TAP_X_OUT: src = s->cap_xout + slot * T * C; bytes = T * C * 4; break;
    case LA_TAP_V: src = s->cap_v + slot * T * C; bytes = T * C * 4; break;
    case LA_TAP_H: src = s->cap_h + (slot * (L + 1) + layer + 1) * T * D; bytes = T * D * 4; break;
    case LA_TAP_Q: src = elem(s->cap_q, (slot * L + layer) * H * T * d, eq); bytes = H * T * d * eq; break;
    case LA_TAP_O: src = s->cap_o + (slot * L + layer) * T * D; bytes = T * D * 4; break;
    case LA_TAP_SINK_KROPE: src = elem(s->cap_sk, (slot * L + layer) * H * F * d, eq); bytes = H * F * d * eq; break;
    case LA_TAP_RING_K:
    case LA_TAP_RING_V:
      src = elem(what == LA_TAP_RING_K ? s->ring_k : s->ring_v,
                 (static_cast<long long>(layer) * S + s->sched.ring_of(slot)) * E * H * T * d, eq);
      bytes = E * H * T * d * eq;
      break;
    case LA_TAP_SINK_K: src = s->sink_k + static_cast<long long>(layer) * H * F * d; bytes = H * F * d * 4; break;
    case LA_TAP_SINK_V: src = elem(s->sink_v, static_cast<long long>(layer) * H * F * d, ea); bytes = H * F * d * ea; break;
    case LA_TAP_SINK_V8: src = s->sink_v8 + static_cast<long long>(layer) * H * F * d; bytes = H * F * d; break;
    case LA_TAP_H_MID: src = s->cap_hmid + (slot * L + layer) * T * D; bytes = T * D * 4; break;
    case LA_TAP_H_CROSS: src = s->cap_hx + (slot * L + layer) * T * D; bytes = T * D * 4; break;
    case LA_TAP_XO: src = s->cap_xo + (slot * L + layer) * T * D; bytes = T * D * 4; break;
    case LA_TAP_XQ: src = elem(s->cap_xq, (slot * L + layer) * H * T * d, ea); bytes = H * T * d * ea; break;
    case LA_TAP_XK:
    case LA_TAP_XV:
      src = elem(what == LA_TAP_XK ? s->cap_xk : s->cap_xv, (slot * L + layer) * H * s->A * d, ea);
      bytes = H * s->A * d * ea;
      break;
    case LA_TAP_FFN_U:
      src = elem(s->cap_u, (slot * L + layer) * T * s->Fffn, s->es);
      bytes = T * s->Fffn * static_cast<long long>(s->es);
      break;
    case LA_TAP_ATTN_SCALES: src = s->attn_sc + static_cast<long long>(layer) * 3 * H; bytes = 3 * H * 4; break;
    case LA_TAP_SINK_H:
      if (!s->cap_sink_valid) return fail(s, LA_ESTATE, "no capture of a sink pass");
      src = s->cap_sink_h + static_cast<long long>(layer) * F * D;
      bytes = F * D * 4;
      break;
    case LA_TAP_HOP:
      src = elem(s->cap_hop, (static_cast<long long>(slot) * L + layer) * T * D, s->es);
      bytes = T * D * s->es;
      break;
    case LA_TAP_SINK_HOP:
      if (!s->cap_sink_valid) return fail(s, LA_ESTATE, "no capture of a sink pass");
      src = elem(s->cap_sink_hop, static_cast<long long>(layer) * F * D, s->es);
      bytes = F * D * s->es;
      break;
    default: return fail(s, LA_EINVAL, "bad tap");
  }
  if (dst_bytes < bytes) return fail(s, LA_EINVAL, "tap destination too small");
  CU(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, s->st));
  return LA_OK;
}

int la_debug_set_slot_input(la_stream* s, int32_t slot, const float* x) {
  if (!s || !x) return LA_EINVAL;
  if (slot < 0 || slot >= s->S) return fail(s, LA_EINVAL, "bad slot");
  if (s->cfg.schedule != LA_SCHED_PIPELINED) return fail(s, LA_ESTATE, "only the pipelined schedule has slot inputs");
  if (slot == 0) return fail(s, LA_ESTATE, "slot 0 is fed by x_new");
  const long long b = s->sched.held[slot - 1];
  if (b < 0) return fail(s, LA_ESTATE, "slot will be idle in the next tick");
  const long long TC = static_cast<long long>(s->T) * s->C;
  CU(cudaMemcpyAsync(s->xs + (b % s->S) * TC, x, TC * 4, cudaMemcpyDeviceToDevice, s->st));
  return LA_OK;
}

int la_profile_enable(la_stream* s, int32_t enable) {
  if (!s) return LA_EINVAL;
  CU(cudaStreamSynchronize(s->st));
  s->prof_events.clear();
  s->ev_next = 0;
  s->prof = enable != 0;
  return LA_OK;
}

int la_profile_read(la_stream* s, int32_t kind, int64_t* launches, double* total_ms) {
  if (!s || kind < 0 || kind >= LA_NUM_KINDS) return LA_EINVAL;
  CU(cudaStreamSynchronize(s->st));
  int64_t n = 0;
  double ms = 0.0;
  for (const ProfEvent& pe : s->prof_events) {
    if (pe.kind != kind) continue;
    float t = 0.f;
    CU(cudaEventElapsedTime(&t, pe.a, pe.b));
    ms += t;
    ++n;
  }
  if (launches) *launches = n;
  if (total_ms) *total_ms = ms;
  return LA_OK;
}

int64_t la_launch_count(const la_stream* s) { return s ? s->launches : 0; }

}  // extern "C"
