/*
 * la_stream.h -- C ABI of the timestep-forced streaming denoising step.
 *
 * The operation is the streaming generator step of Live Avatar (arXiv
 * 2512.04677) as the pages describe it:
 *   - blocks of 3 latent frames advance autoregressively under a block-causal
 *     mask (papernotes.org ECCV2026 note, 整体框架; 10100.com article,
 *     training-framework caption);
 *   - the KV cache keeps the noisy K/V of the step that produced them and is
 *     never refreshed by a clean forward (papernotes note, 关键设计 2 "History
 *     Corrupt"; gitcode blog, question 4);
 *   - every denoising step t_i has its own cache (timestep forcing) and the 4
 *     steps of 4 consecutive blocks run as a pipeline (papernotes note,
 *     关键设计 4 "TPP"; 10100.com article, TPP caption).  On one GPU the 4
 *     pipeline stages run as one grouped launch per tick;
 *   - the sink frame is re-offset in RoPE time each block so its distance to
 *     the active block stays constant (Rolling RoPE, papernotes note 关键设计 3)
 *     and is replaced once by the first generated latent (Adaptive Attention
 *     Sink, papernotes note 关键设计 3; gitcode blog question 5);
 *   - each step ends with the flow-matching Euler update
 *     x_{t_{i+1}} = x_{t_i} + (t_{i+1} - t_i) v (papernotes note, 损失函数).
 *
 * The synthetic stack per step: h = x W_in^T; per sublayer
 * [q|k|v] = n(h) W_qkv^T, Rolling RoPE on q/k, ring append, block-causal
 * attention, h += O W_out^T; v = n(h) W_head^T; with n the per-token RMS
 * normalisation n(h) = h / sqrt(mean(h^2) + LA_RMS_EPS) (the pages give no
 * layer internals; without it the stacked residual map expands).
 *
 * Conventions for every function:
 *   - Return value: LA_OK (0) or a negative LA_E* status.  No C++ exception
 *     crosses this boundary.  la_last_error() gives a text for the last
 *     failure of a stream.
 *   - "device" pointers are CUDA device memory of the stream's device;
 *     "host" pointers are CPU memory (pinned memory makes copies asynchronous).
 *   - Work is enqueued asynchronously on the CUDA stream given at creation;
 *     host-side state (tick counter, ring indices, finished block id) is
 *     updated synchronously.  la_synchronize() waits and reports device-side
 *     errors (LA_EDEVICE) raised by bounded waits inside the kernels.
 *   - The caller owns inputs, outputs and weights; the library owns the ring
 *     caches, the sink buffers, scratch and the tick state.
 *   - There is no CPU fallback: without a usable sm_100 device creation fails
 *     with LA_ECUDA.
 */
#ifndef LA_STREAM_H
#define LA_STREAM_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
#define LA_OK        0
#define LA_EINVAL   -1   /* bad argument or configuration                   */
#define LA_ESTATE   -2   /* call not valid in the stream's current state    */
#define LA_ENOMEM   -3   /* device memory would not fit (checked up front)  */
#define LA_ECUDA    -4   /* a CUDA runtime / driver call failed             */
#define LA_EDEVICE  -5   /* a kernel raised the device error word           */

/* ---- enums ------------------------------------------------------------- */
#define LA_SINK_FIXED        0  /* reference sink kept for the whole stream           */
#define LA_SINK_AAS          1  /* sink replaced once by frame 0 of finished block 0  */
#define LA_SCHED_PIPELINED   0  /* one call = one tick: slot i runs step i of block k-i */
#define LA_SCHED_SEQUENTIAL  1  /* one call = one block through all steps in order     */
#define LA_SCHED_SLOT        2  /* one rank of the timestep pipeline across GPUs (TPP):
                                   one call = step slot_index of the next block, with
                                   that step's own cache; the caller moves the latent
                                   from rank to rank and replaces the sink on every
                                   rank (la_replace_sink) when block 0 finishes       */
#define LA_BF16              0  /* bf16 GEMM operands and attention operands, fp32
                                   accumulation, fp32 residual stream and latent x    */
#define LA_FP32              1  /* fp32 everywhere (SIMT path, no TF32)                */
#define LA_CACHE_TIMESTEP    0  /* each step keeps the noisy K/V it computed in its own
                                   cache (timestep forcing; papernotes note, key design
                                   4; gitcode blog, question 6)                         */
#define LA_CACHE_CLEAN_REFRESH 1 /* the ablation the method removes: one cache of clean
                                   K/V; after a block's last step one more pass of the
                                   finished latent rewrites its entry (NFE num_steps+1;
                                   papernotes note, key design 2 and the paper's Table 3; gitcode
                                   blog, question 4).  Sequential schedule only.       */
#define LA_CACHE_FIXED_STEP  2  /* the other alternative the pages compare ("fixed noise or
                                   clean cache", papernotes note, key findings = the
                                   paper's Table 6): every step reads the prior blocks'
                                   K/V written at one fixed step (cache_step); each step
                                   still writes its own cache and attends to its own
                                   block's current K/V.  NFE num_steps.  Sequential
                                   schedule only.                                      */

#define LA_RMS_EPS 1e-6

/* Compile-time limits of the library (larger configurations return LA_EINVAL). */
#define LA_MAX_STEPS     8
#define LA_MAX_WINDOW   14
#define LA_MAX_FPB       7

/*
 * Stream configuration.  D = heads*head_dim, F = grid_h*grid_w tokens per
 * latent frame, T_b = frames_per_block*F tokens per block.
 */
typedef struct la_config {
  int32_t num_layers;          /* >= 1 attention sublayers                               */
  int32_t hidden;              /* D; must equal heads*head_dim                           */
  int32_t heads;               /* H                                                      */
  int32_t head_dim;            /* d; bf16 path: 128; fp32 path: even, <= 128             */
  int32_t latent_ch;           /* C; C == D with NULL w_in/w_head means identity maps   */
  int32_t grid_h, grid_w;      /* latent frame token grid                                */
  int32_t frames_per_block;    /* 3 on the pages; 1..LA_MAX_FPB                          */
  int32_t sink_frames;         /* 1 (only value supported)                               */
  int32_t window_blocks;       /* N_w: prior blocks each timestep slot keeps, 0..LA_MAX_WINDOW */
  int32_t num_steps;           /* S: timestep slots, 1..LA_MAX_STEPS                      */
  const float* timesteps;      /* HOST, num_steps+1 values, strictly descending, finite;
                                  step i integrates from timesteps[i] to timesteps[i+1].
                                  Copied at creation.                                    */
  int32_t rope_split[3];       /* rotary PAIRS for (t, h, w); sum == head_dim/2         */
  double  rope_theta;          /* > 0, e.g. 10000                                        */
  int32_t sink_mode;           /* LA_SINK_FIXED | LA_SINK_AAS                            */
  int32_t rolling_rope;        /* 1: sink t-pos = frames_per_block*b - sink_offset_frames;
                                  0: fixed at -sink_offset_frames                         */
  int32_t sink_offset_frames;  /* 3                                                      */
  int32_t schedule;            /* LA_SCHED_PIPELINED | LA_SCHED_SEQUENTIAL | LA_SCHED_SLOT */
  int32_t dtype;               /* LA_BF16 | LA_FP32                                      */
  int32_t cache_mode;          /* LA_CACHE_TIMESTEP | LA_CACHE_CLEAN_REFRESH | LA_CACHE_FIXED_STEP */
  int32_t proj_fp8;            /* 1 (LA_BF16 only): the QKV and output projections run on
                                  e4m3 operands: weights quantized per output row at
                                  creation, the bf16 GEMM operand per token before each
                                  projection (la_op_quantize_e4m3's definition), fp32
                                  accumulate, scales applied before the epilogue.  The
                                  pages' FP8 row (papernotes note, the paper's Table 3).
                                  0: bf16 projections.                                   */
  int32_t attn_fp8;            /* 1 (LA_BF16, head_dim 128 only): the denoising passes'
                                  attention runs on e4m3 q / K / V (la_op_attention_fp8's
                                  definition): the QKV epilogue, the sink re-rope and the
                                  sink V store e4m3 codes of value / scale, with one
                                  power-of-two scale per (layer, q|K|V, head) fixed at
                                  creation: the smallest 2^k >= bound / 448, where bound =
                                  1.07 sqrt(hidden) times the largest norm of the head's
                                  QKV weight rows (of a rotary pair of rows for q and K),
                                  a bound on |value| for any RMS-normalised input (the
                                  1.07 covers the rounding of the GEMM operand).  The
                                  sink's own pass keeps bf16 attention.  Same row as
                                  proj_fp8.  0: bf16 attention.                          */
  int32_t cache_step;          /* LA_CACHE_FIXED_STEP: the step (0 .. num_steps-1) whose
                                  K/V of the prior blocks every step reads; ignored by
                                  the other cache modes.                                */
  int32_t block_kind;          /* LA_BLOCK_ATTN | LA_BLOCK_DIT                           */
  int32_t ffn_dim;             /* LA_BLOCK_DIT: FFN hidden width F (multiple of 32)       */
  int32_t audio_tokens;        /* LA_BLOCK_DIT: audio tokens A per block for the audio
                                  cross-attention (0: none; then la_denoise_step_av)     */
  int32_t audio_dim;           /* their feature width D_a (multiple of 8)               */
  int32_t slot_index;          /* LA_SCHED_SLOT: the step this stream runs (0 .. num_steps-1) */
} la_config;

/* Layer kinds.  The pages give the model's base (a 14B DiT with timestep
 * conditioning; papernotes note, overall framework and FM loss) but no layer
 * internals; LA_BLOCK_DIT is the Wan-style block the model is built on:
 *   h += gate1 * Attn(n(h) * (1 + scale1) + shift1)
 *   h += gate2 * (gelu_tanh(m W_ffn1^T) W_ffn2^T),  m = n(h) * (1 + scale2) + shift2
 * with n the per-token RMS norm, Attn the attention sublayer (QKV, Rolling
 * RoPE, cache, block-causal attention, output projection) and the AdaLN
 * vectors of the layer at the step's timestep (la_weights.ada).  Needs
 * proj_fp8 = attn_fp8 = 0.  The FFN runs on the same GEMM kernels.
 * With audio_tokens > 0 the block also has the audio cross-attention (the
 * model is audio-driven; reading: Wan's cross-attention sub-block), between
 * the attention and the FFN sub-blocks:
 *   h += (softmax(q k^T / sqrt(d)) v) W_oc^T,  q = n(h) W_qc^T,  [k | v] = audio_b W_kvc^T
 * over the A audio tokens of the block (no RoPE, no mask).  A block's audio
 * K/V are computed once, when the block enters the stream; the sink pass
 * has no audio and skips the sub-block. */
#define LA_BLOCK_ATTN        0  /* each layer: the attention sublayer               */
#define LA_BLOCK_DIT         1  /* each layer: the full DiT block                   */

/*
 * Weights: DEVICE pointers, BORROWED (they must outlive the stream and must
 * not change while it exists).  Element type = config dtype (bf16 or fp32).
 * Layout [out_features, in_features], row-major, i.e. y = x W^T.
 */
typedef struct la_weights {
  const void* w_in;              /* [D, C] or NULL (identity; needs C == D)     */
  const void* w_head;            /* [C, D] or NULL (identity; needs C == D)     */
  const void* const* w_qkv;      /* HOST array of num_layers DEVICE pointers, each [3D, D];
                                    rows 0..D-1 give q, D..2D-1 k, 2D..3D-1 v; head h
                                    owns rows h*d .. h*d+d-1 of each part        */
  const void* const* w_out;      /* HOST array of num_layers DEVICE pointers, each [D, D] */
  /* LA_BLOCK_DIT only (ignored otherwise): */
  const void* const* w_ffn1;     /* HOST array of num_layers DEVICE pointers, each [F, D] */
  const void* const* w_ffn2;     /* HOST array of num_layers DEVICE pointers, each [D, F] */
  const float* ada;              /* DEVICE fp32 [num_layers][num_steps + 1][6][D]: the AdaLN
                                    vectors shift1, scale1, gate1, shift2, scale2, gate2 of
                                    each layer at timesteps[0 .. num_steps-1], and at t = 0
                                    (index num_steps: the sink pass and the clean refresh) */
  /* LA_BLOCK_DIT with audio_tokens > 0 only: */
  const void* const* w_qc;       /* HOST array of num_layers DEVICE pointers, each [D, D] */
  const void* const* w_kvc;      /* ... each [2D, D_a]: rows 0..D-1 K, D..2D-1 V          */
  const void* const* w_oc;       /* ... each [D, D]                                      */
} la_weights;

typedef struct la_stream la_stream;

/*
 * Create a stream on the current CUDA device.  cuda_stream is a cudaStream_t
 * (NULL = legacy default stream).  Allocates every buffer up front after a
 * cudaMemGetInfo check (LA_ENOMEM if it would not fit).  *out is set to NULL
 * on failure.  LA_EINVAL: invalid config (sizes <= 0, hidden != heads*head_dim,
 * head_dim unsupported for the dtype, timesteps not strictly descending,
 * window out of range, rope_split not summing to head_dim/2, NULL weights).
 */
int la_stream_create(const la_config* cfg, const la_weights* w, void* cuda_stream,
                     la_stream** out);

/*
 * Set the reference sink: DEVICE fp32 [sink_frames*F, C].  Runs the sink
 * frame through the layers (self-attention over the sink only, RoPE time
 * -sink_offset_frames) and stores, per layer, the un-roped sink K and the
 * sink V shared by all slots.  Must precede the first la_denoise_step; may
 * only be called before it (LA_ESTATE afterwards).
 */
int la_set_sink(la_stream* s, const float* sink_latent);

/*
 * One call.  Pipelined schedule: one tick.  x_new (DEVICE fp32 [T_b, C]) is
 * the noise of the next block at timesteps[0]; it enters slot 0.  NULL drains
 * the pipeline (no new block).  Every in-flight block advances one step in
 * its slot.  If the block in the last slot finishes, its latent is copied to
 * x_out (DEVICE fp32 [T_b, C]) and its id is written to *finished_block
 * (HOST), else *finished_block = -1 and x_out is untouched.
 * Sequential schedule: x_new must be non-NULL; the block runs all steps in
 * order and always finishes.
 * When the sink mode is LA_SINK_AAS and block 0 finishes, frame 0 of its
 * latent becomes the sink for every later step (once per stream).
 * LA_ESTATE before la_set_sink; LA_EINVAL for NULL x_out / finished_block or
 * a NULL x_new in the sequential schedule.
 */
int la_denoise_step(la_stream* s, const float* x_new, float* x_out, int64_t* finished_block);

/* Same as la_denoise_step with HOST x_new / x_out: the host->device copy of
 * the new block and the device->host copy of the finished block are enqueued
 * on the stream (asynchronous if the host memory is pinned); the call returns
 * after enqueueing, so read x_out only after la_synchronize(). */
int la_denoise_step_host(la_stream* s, const float* x_new_host, float* x_out_host,
                         int64_t* finished_block);

/* la_denoise_step for streams with the audio cross-attention (audio_tokens >
 * 0): audio_new (DEVICE fp32 [audio_tokens, audio_dim]) is the audio of the
 * new block x_new (both NULL to drain).  Its K/V for every layer are
 * computed in this call and kept while the block is in flight, so audio_new
 * may be reused after the call is enqueued.  la_denoise_step and
 * la_denoise_step_host return LA_EINVAL for a new block of such a stream. */
int la_denoise_step_av(la_stream* s, const float* x_new, const float* audio_new, float* x_out,
                       int64_t* finished_block);

/* LA_SCHED_SLOT streams (one rank of the timestep pipeline; the papernotes
 * note's TPP: each GPU pinned to one denoising step with its own cache, the
 * latent passed on): each call runs step slot_index of the next block (ids
 * 0, 1, ... in call order).  x_new (DEVICE fp32 [T_b, C], required) is the
 * block's latent at timesteps[slot_index] (noise for slot 0, the previous
 * rank's x_out otherwise); x_out receives it after the step and
 * *finished_block the block's id.  Such a stream never replaces its sink on
 * its own: with LA_SINK_AAS the caller calls la_replace_sink on every rank
 * with frame 0 of block 0's finished latent (the last rank's output) before
 * any rank runs a step of a later tick, which gives the single-GPU pipeline's
 * timing (the new sink from tick num_steps on).
 * la_replace_sink: sink_latent DEVICE fp32 [F * sink_frames, C]; reruns the
 * sink pass and marks the sink generation 1.  LA_ESTATE for other schedules
 * or a second replacement. */
int la_replace_sink(la_stream* s, const float* sink_latent);

/* Wait for all work of the stream; LA_EDEVICE if a kernel raised the device
 * error word (the word is cleared after being reported). */
int la_synchronize(la_stream* s);

/* Free everything.  NULL is a no-op.  The pointer is invalid afterwards. */
int la_stream_destroy(la_stream* s);

/* Text of the last error on s (never NULL; "" if none); static text if s is NULL. */
const char* la_last_error(const la_stream* s);
const char* la_status_string(int status);

/* ---- debug / test exports ------------------------------------------------ */

/* Number of int32 values of the index state (see la_get_index_state). */
int64_t la_index_state_size(const la_stream* s);

/*
 * Integer state after the last call, HOST buffer of n >= la_index_state_size
 * int32: header [tick, blocks_in, blocks_out, sink_generation] then, for each
 * slot i < num_steps, E = window_blocks+1 and R = 8 + 3E values:
 *   [active_block, write_entry, evicted_block, sink_tpos, frame_tpos,
 *    sink_generation_used, step_index, n_resident,
 *    resident[E] (oldest -> newest, -1 padded), tags[E] x (block, step)].
 * active_block/write_entry/evicted_block are -1 and sink_tpos/frame_tpos/
 * sink_generation_used are 0 for a slot that was idle in the last call.
 */
int la_get_index_state(const la_stream* s, int32_t* host_buf, int64_t n);

/* The tick scheduler on the host alone: no stream, no GPU, no device memory.
 * la_sched_trace runs the scheduling of `nticks` la_denoise_step calls on a
 * fresh stream of configuration cfg (has_new[k] != 0: call k brings a new
 * block; the sequential and slot schedules need one on every call), in the
 * order a call makes them (plan the tick, append each running (slot, block) to
 * its ring, the clean-cache refresh, finish), and writes the index state after
 * each call (the layout of la_get_index_state, la_sched_state_size(cfg) int32
 * values each) to out[k * size ...].  Only the scheduling fields of cfg are read
 * (frames_per_block, window_blocks, num_steps, sink_mode, schedule, slot_index,
 * cache_mode, cache_step, rolling_rope, sink_offset_frames).
 * Returns LA_EINVAL for a bad configuration, NULL pointers or out_len below
 * nticks * size; LA_ESTATE at a call the schedule does not allow (then out holds
 * the states of the calls before it).  la_sched_state_size returns -1 for a bad
 * configuration.  A stream's AAS sink replacement by the caller
 * (la_replace_sink, slot schedule) is not modelled. */
int64_t la_sched_state_size(const la_config* cfg);
int la_sched_trace(const la_config* cfg, int32_t nticks, const uint8_t* has_new, int32_t* out, int64_t out_len);

/* Enable (1) / disable (0) capture of per-slot intermediates for la_debug_tap.
 * Allocates capture buffers on enable. */
int la_debug_capture(la_stream* s, int32_t enable);

#define LA_TAP_X_IN      0  /* fp32 [T_b, C]   latent the slot's last step started from        */
#define LA_TAP_X_OUT     1  /* fp32 [T_b, C]   latent after the slot's last step               */
#define LA_TAP_H         2  /* fp32 [T_b, D]   residual after layer `layer` (-1: after in-proj) */
/* "attn" = the attention operand type: bf16 for LA_BF16 streams, fp32 for LA_FP32. */
#define LA_TAP_Q         3  /* attn [H, T_b, d] roped queries of layer; LA_BF16 streams store
                               them pre-multiplied by the softmax scale log2(e)/sqrt(d)         */
#define LA_TAP_O         4  /* fp32 [T_b, D]   attention output of layer, before rounding        */
#define LA_TAP_V         5  /* fp32 [T_b, C]    velocity of the slot's last step                 */
#define LA_TAP_RING_K    6  /* attn [E, H, T_b, d] ring K of (layer, slot), by entry (the one
                               clean cache for every slot under LA_CACHE_CLEAN_REFRESH)          */
#define LA_TAP_RING_V    7  /* attn [E, H, T_b, d] ring V of (layer, slot)                       */
#define LA_TAP_SINK_K    8  /* fp32 [H, F, d] un-roped sink K of layer (slot ignored)            */
#define LA_TAP_SINK_V    9  /* attn [H, F, d] sink V of layer (slot ignored)                     */
#define LA_TAP_SINK_KROPE 10 /* attn [H, F, d] sink K as roped for the slot's last step          */
#define LA_TAP_SINK_H    11 /* fp32 [F, D] sink residual entering layer `layer` in the last sink
                               pass (la_set_sink or the AAS replacement; slot ignored)           */
#define LA_TAP_HOP       12 /* bf16 [T_b, D] the QKV projection's operand of layer `layer` at the
                               slot's step (bf16 streams): the normalised residual, or, where
                               the stream folds the norm into its GEMMs (bf16 attention
                               sublayers with w_in and w_head), the residual itself rounded
                               to bf16 (the GEMM scales its rows by 1 / rms)                 */
#define LA_TAP_SINK_HOP  13 /* bf16 [F, D] the same in the last sink pass (slot ignored)         */
/* With attn_fp8 the Q, RING_K, RING_V and SINK_KROPE taps hold uint8 e4m3 codes
 * (value = code * scale of its layer, part and head; Q not pre-scaled), and: */
#define LA_TAP_SINK_V8   14 /* uint8 [H, F, d] e4m3 codes of the sink V of layer (slot ignored) */
#define LA_TAP_ATTN_SCALES 15 /* fp32 [3, H] scales of q, K, V of layer (slot ignored)          */
/* LA_BLOCK_DIT only: */
#define LA_TAP_H_MID     16 /* fp32 [T_b, D] residual of layer after the attention sub-block   */
#define LA_TAP_FFN_U     17 /* dtype [T_b, F] GELU output of layer's FFN (the second GEMM's
                               operand)                                                       */
/* LA_BLOCK_DIT with audio only: */
#define LA_TAP_H_CROSS   18 /* fp32 [T_b, D] residual of layer after the cross-attention      */
#define LA_TAP_XQ        19 /* attn [H, T_b, d] cross-attention q (bf16 streams: times
                               log2(e)/sqrt(d), like LA_TAP_Q)                                */
#define LA_TAP_XK        20 /* attn [H, A, d] the block's audio K of layer                    */
#define LA_TAP_XV        21 /* attn [H, A, d] the block's audio V of layer                    */
#define LA_TAP_XO        22 /* fp32 [T_b, D] cross-attention output of layer, before rounding */

/* Copy one tapped tensor into dst (DEVICE, dst_bytes >= the tensor's size),
 * ordered on the stream.  Taps other than ring / sink need capture enabled
 * before the call being inspected.  LA_EINVAL on bad what/layer/slot/size. */
int la_debug_tap(la_stream* s, int32_t what, int32_t layer, int32_t slot, void* dst,
                 int64_t dst_bytes);

/* Overwrite the latent that `slot` will start its next step from (DEVICE fp32
 * [T_b, C]).  Slot 0 of the pipelined schedule is fed by x_new instead.
 * Used to inject fresh per-step inputs in soak tests.  LA_ESTATE if the slot
 * will be idle in the next tick. */
int la_debug_set_slot_input(la_stream* s, int32_t slot, const float* x);

/* Kernel timing with CUDA events on the stream.  kind: LA_KIND_*. */
#define LA_KIND_IN_PROJ   0
#define LA_KIND_QKV_GEMM  1
#define LA_KIND_ROPE      2
#define LA_KIND_ATTN      3
#define LA_KIND_OUT_GEMM  4
#define LA_KIND_HEAD      5
#define LA_KIND_OTHER     6
#define LA_KIND_FFN       7  /* LA_BLOCK_DIT: the two FFN GEMMs                   */
#define LA_KIND_CROSS     8  /* LA_BLOCK_DIT with audio: the cross-attention's q and
                                output GEMMs, head split and attention, and the
                                audio K/V of each entering block                 */
#define LA_NUM_KINDS      9
int la_profile_enable(la_stream* s, int32_t enable);   /* resets the counters */
int la_profile_read(la_stream* s, int32_t kind, int64_t* launches, double* total_ms);
/* Kernels launched by this stream since creation. */
int64_t la_launch_count(const la_stream* s);

/*
 * Failure-detection check (the pages have no counterpart; it tests the
 * library's own error path without faulting the GPU).  Launches one CTA on the
 * current device whose thread waits on an mbarrier phase with a limit of
 * limit_ns nanoseconds (0 <= limit_ns <= 1e10), as every pipelined kernel of
 * the library waits.  complete != 0: the phase is completed before the wait;
 * 0: nothing completes it, the wait gives up after the limit, raises the
 * device error word and the kernel returns.  Synchronises the device.
 * *device_error receives the word (0, or LA_DEVERR_WAIT_TIMEOUT = 1).
 * Returns LA_OK, LA_EDEVICE when the word was raised, LA_EINVAL, LA_ENOMEM
 * (the 4-byte word could not be allocated) or LA_ECUDA.  The CUDA context
 * stays usable after LA_EDEVICE.
 */
int la_debug_wait_timeout(int64_t limit_ns, int32_t complete, int32_t* device_error);

/*
 * The same check for the op-level entry points: enqueues on cuda_stream one
 * CTA whose wait nothing completes, so that after limit_ns (0..1e10) it raises
 * the op-level error word (see la_op_status) and returns.  Asynchronous;
 * allocates nothing.  LA_OK, LA_EINVAL or LA_ECUDA.
 */
int la_debug_op_wait_timeout(int64_t limit_ns, void* cuda_stream);

/* ---- op-level entry points (unit tests, microbenchmarks) ------------------
 * Each enqueues one kernel on cuda_stream (a cudaStream_t, NULL = default).
 * They allocate nothing except where stated.  Their tensor-core kernels wait
 * on mbarriers with a limit, like the stream's; a wait that gives up raises a
 * per-device op-level error word (a file-scope device int of the library,
 * first error wins) and the kernel returns with its output unfinished.
 */

/*
 * Reports and clears the op-level error word of the current device:
 * synchronises cuda_stream, then returns LA_EDEVICE (message on stderr) if a
 * kernel of an la_op_* call raised the word since the last la_op_status on
 * this device, else LA_OK; LA_ECUDA if the word cannot be read.  Allocates
 * nothing.  The word is shared by every op-level call on the device, so an
 * error raised by a call on another stream is reported here too.
 */
int la_op_status(void* cuda_stream);

/*
 * C = A W^T with an epilogue.  A: DEVICE [M, K] row-major, W: DEVICE [N, K]
 * row-major, both of `dtype` (LA_BF16: tcgen05 tensor cores, fp32
 * accumulate, N % 32 == 0, K % 8 == 0; LA_FP32: SIMT fp32).
 *   LA_EPI_STORE:   out (dtype [M, N]) = acc
 *   LA_EPI_STORE32: out (fp32 [M, N]) = acc
 *   LA_EPI_RESID:   h32 (fp32 [M, N]) += acc; out (dtype [M, N]) = h32
 *   LA_EPI_SET32:   h32 = acc; out (dtype [M, N]) = acc   (out may be NULL)
 *   LA_EPI_EULER:   h32[m, n] += dt[m / rows_per_group] * acc (the Euler update;
 *                   dt: HOST array of ceil(M/rows_per_group) floats, <= LA_MAX_STEPS)
 * For LA_FP32 "out" of RESID/SET32 may alias h32.
 */
#define LA_EPI_STORE    0
#define LA_EPI_RESID    1
#define LA_EPI_SET32    2
#define LA_EPI_EULER    3
#define LA_EPI_STORE32  4
int la_op_gemm(int32_t dtype, int32_t epilogue, const void* A, const void* W, void* out,
               float* h32, int64_t M, int64_t N, int64_t K, const float* dt,
               int64_t rows_per_group, void* cuda_stream);

/*
 * Block attention over a list of KV segments for one group of Tq queries:
 * O[t, h*d + e] = sum_j softmax_j(q_h[t] . k_h[j] / sqrt(d)) v_h[j][e] over the
 * concatenation of the segments (every key visible; the block-causal mask is
 * expressed by which segments are passed).  q: DEVICE [H, Tq, d]; segment s:
 * k_seg[s], v_seg[s] DEVICE [H, seg_len[s], d] (HOST arrays of nseg pointers /
 * lengths, 1 <= nseg <= LA_MAX_WINDOW + 2, seg_len >= 1).
 * dtype LA_BF16: q/K/V bf16, d == 128, tcgen05; out DEVICE bf16 [Tq, H*d] and,
 *   if out32 != NULL, an fp32 copy [Tq, H*d] (the value before rounding).
 *   q_scaled != 0: q is already multiplied by log2(e)/sqrt(d) (the stream's
 *   layout); 0: plain q.
 * dtype LA_FP32: q/K/V/out fp32, d % 8 == 0, d <= 128, SIMT; out32 and
 *   q_scaled ignored.
 */
int la_op_attention(int32_t dtype, const void* q, int64_t Tq, int32_t H, int32_t d,
                    int32_t nseg, const void* const* k_seg, const void* const* v_seg,
                    const int64_t* seg_len, void* out, float* out32, int32_t q_scaled,
                    void* cuda_stream);

/*
 * Standalone Euler update x[r, :] += dt[r / rows_per_group] * v[r, :] over
 * `rows` rows of C fp32 values (DEVICE x, v); dt HOST, <= LA_MAX_STEPS groups.
 */
int la_op_euler(float* x, const float* v, int64_t rows, int64_t C, const float* dt,
                int64_t rows_per_group, void* cuda_stream);

/*
 * FP8 (e4m3) operands for the projections: the pages' operator-level
 * optimisation row (papernotes note, inference-efficiency ablation = the
 * paper's Table 3: FP8 quantisation + FlashAttention-3 + fused kernels; the
 * pages give no scheme, per-row scaling is the reading taken).
 *
 * la_op_quantize_e4m3: per-row quantization of x (DEVICE, in_dtype LA_BF16 or
 * LA_FP32, [rows, cols] dense, cols even): scales[r] = amax_r / 448 (fp32;
 * 1 for an all-zero row), codes[r, c] = e4m3(x[r, c] / scales[r]) with IEEE
 * fp32 division, rounding to nearest even and saturation at +-448 (OCP E4M3,
 * no infinities).  codes: DEVICE uint8 [rows, cols]; scales: DEVICE fp32 [rows].
 *
 * la_op_gemm_fp8: out[m, n] = (sum_k a[m, k] w[n, k]) * a_scales[m] *
 * w_scales[n] on the tensor cores (tcgen05 kind::f8f6f4, fp32 accumulate):
 * a_codes DEVICE uint8 [M, K], w_codes [N, K] (both dense, K % 16 == 0),
 * scales DEVICE fp32 [M] / [N]; out DEVICE [M, N], out_dtype LA_BF16 (rounded
 * once) or LA_FP32.  N % 32 == 0.  LA_EINVAL on bad sizes or NULL pointers.
 */
int la_op_quantize_e4m3(int32_t in_dtype, const void* x, int64_t rows, int64_t cols,
                        void* codes, float* scales, void* cuda_stream);
int la_op_gemm_fp8(const void* a_codes, const float* a_scales, const void* w_codes,
                   const float* w_scales, void* out, int32_t out_dtype, int64_t M, int64_t N,
                   int64_t K, void* cuda_stream);

/*
 * FP8 (e4m3) attention, the attention half of the same operator-optimisation
 * row ("FP8 quantisation + FlashAttention-3"; the pages give no scheme).  The
 * reading taken is FlashAttention-3's FP8 form: e4m3 q, K, V with one fp32
 * scale per head each, and an e4m3 probability matrix in P V:
 *   s[t, j] = (q_code[t] . k_code[j]) * q_scale[h] * k_scale[h] * log2(e)/sqrt(d)
 *   M[t]    = ceil(max_j s[t, j])            (a whole number)
 *   p[t, j] = 2^(s[t, j] - M[t] + 5)         (fp32; the row max lies in (16, 32])
 *   O[t, h*d + e] = v_scale[h] * sum_j e4m3(p[t, j]) v_code[j][e] / sum_j p[t, j]
 * over the concatenation of the segments (every key visible).  The kernel
 * keeps M as a running whole number that is raised only when a key tile's
 * max exceeds it by more than 3; a raise rescales O by an exact power of two,
 * so the codes of P equal those formed against the final M wherever they are
 * normal e4m3 values (keys weighing >= 2^-11 of the row's largest).
 *   q_codes DEVICE uint8 [H, Tq, d]; segment s: k_seg[s], v_seg[s] DEVICE uint8
 *   [H, seg_len[s], d] (HOST arrays of nseg pointers / lengths, 1 <= nseg <=
 *   LA_MAX_WINDOW + 2, seg_len >= 1), 16-byte aligned; d == 128.
 *   q_scale, k_scale, v_scale: DEVICE fp32 [H], positive.
 *   out DEVICE bf16 [Tq, H*d] (rounded once) and, if out32 != NULL, the fp32
 *   value [Tq, H*d].
 * Codes are the caller's (no NaN codes expected).  LA_EINVAL on bad sizes or
 * NULL pointers; LA_ECUDA if the launch fails.
 */
int la_op_attention_fp8(const void* q_codes, int64_t Tq, int32_t H, int32_t d, int32_t nseg,
                        const void* const* k_seg, const void* const* v_seg,
                        const int64_t* seg_len, const float* q_scale, const float* k_scale,
                        const float* v_scale, void* out, float* out32, void* cuda_stream);

/*
 * Block attention for callers that cannot allocate device memory (a plugin
 * whose host application owns all device memory through its own allocator or
 * a fixed budget, or a real-time path where an allocation and its implicit
 * synchronisation are not allowed).  No
 * counterpart on the pages.  It takes a plain bf16 q, writes q times the
 * softmax scale log2(e)/sqrt(d) (fp32 product, rounded once to bf16: the form
 * the stream's QKV epilogue writes) to its one scratch buffer, and runs the
 * la_op_attention kernel with q_scaled = 1 on it; the result equals
 * la_op_attention(LA_BF16, that scaled q, ..., q_scaled = 1) bit for bit.  The
 * scratch is a file-scope device array of LA_STATIC_Q_ELEMS bf16 values
 * (16 MiB) instead of an allocation.  Every GPU that loads the library holds
 * that array until the process exits.
 *   - Arguments as la_op_attention with dtype LA_BF16 (q, segments, out, out32),
 *     d == 128.  H*Tq*d must be <= LA_STATIC_Q_ELEMS, else LA_EINVAL with a
 *     message on stderr. *   - Calls no cudaMalloc, cudaFree or allocating library routine.  The first
 *     call on a device (and the first after the device's context changed, as
 *     after cudaDeviceReset) looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current); make that first call
 *     before any stream capture.  Under CUDA's default lazy module loading the
 *     first call also loads the library's device code and so reserves the
 *     array then: it can fail with LA_ECUDA if the device's memory is already
 *     taken.  Callers with a fixed memory budget make one call (or set
 *     CUDA_MODULE_LOADING=EAGER) before their allocator takes the budget.
 *   - All calls share the array and overwrite the part they use (nothing needs
 *     to start at zero); calls that overlap on the GPU race on it.
 *   - A bounded wait that gives up in the kernel raises the op-level error
 *     word: la_op_status reports it (LA_EDEVICE) and clears it.
 */
#define LA_STATIC_Q_ELEMS (8LL * 1024 * 1024)
int la_op_attention_static(const void* q, int64_t Tq, int32_t H, int32_t d, int32_t nseg,
                           const void* const* k_seg, const void* const* v_seg,
                           const int64_t* seg_len, void* out, float* out32, void* cuda_stream);

#ifdef __cplusplus
}
#endif
#endif /* LA_STREAM_H */
