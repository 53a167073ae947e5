/*
 * dg.h - C ABI of the DiffusionGemma denoising-step library for NVIDIA B200
 * (sm_100a).
 *
 * The method (DiffusionGemma technical report; arXiv abstract page
 * "DiffusionGemma 技术报告" and the laozijiushiniubi.cn article
 * "谷歌DeepMind如何将一台'逐字打稿机'改造成'整段喷墨机'", §一, §二, §四):
 * a prompt is encoded with causal attention; text is produced in blocks of
 * 256 tokens, each block starting from uniformly random tokens and refined
 * in rounds in which every position is predicted in parallel by a
 * 128-expert top-8 mixture-of-experts transformer that attends
 * bidirectionally over the block and into the encoded context; each round
 * locks the confident positions, re-randomises the others, feeds its
 * prediction back as a self-conditioning input, and stops adaptively on the
 * mean entropy.  A finished block is appended to the context causally.
 *
 * Conventions
 *  - The caller owns all device memory (weights, KV cache, canvas state,
 *    outputs, workspace) and passes raw device pointers; sizes come from the
 *    *_bytes queries.  The library never allocates device memory.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *  - dg_encode_context and dg_denoise_step only enqueue work on `stream`;
 *    dg_decode_block synchronises `stream` once per round to read the stop flags.
 *  - Argument and shape errors are reported before anything is launched
 *    (DG_ERR_INVALID_ARG).  CUDA launch errors give DG_ERR_CUDA.  Errors found
 *    on the device (a token id outside [0, V), a bounded wait that ran out)
 *    are latched in a device error word of the context and reported by
 *    dg_check_device_error and by dg_decode_block.
 *  - No C++ exception crosses this interface.  dg_last_error() returns a
 *    thread-local message for the last failing call on that thread.
 *  - Canvas length is fixed at DG_CANVAS (256) tokens per canvas.
 */
#ifndef DG_H
#define DG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DG_CANVAS 256

typedef enum dg_status {
  DG_OK = 0,
  DG_ERR_INVALID_ARG = 1,  /* bad pointer, size or configuration; nothing was launched */
  DG_ERR_CUDA = 2,         /* a CUDA call or launch failed (message in dg_last_error) */
  DG_ERR_WORKSPACE = 3,    /* the workspace passed to dg_context_create is too small */
  DG_ERR_TIMEOUT = 4,      /* a bounded device-side wait ran out (device error word) */
  DG_ERR_UNSUPPORTED = 5,  /* a configuration this build does not implement */
  DG_ERR_BAD_TOKEN = 6     /* a token id outside [0, vocab) reached the device */
} dg_status;

/* Model dimensions.  The pages fix 128 experts with 8 active per token
   (laozijiushiniubi.cn article §二); the other dimensions are the caller's.
   Limits of this build: d_model % 64 == 0 and 256 <= d_model <= 4096,
   head_dim in {32, 64, 128, 176}, n_q_heads % n_kv_heads == 0,
   d_ff % 64 == 0, vocab % 256 == 0, top_k <= 8, n_experts <= 256. */
typedef struct dg_model_config {
  int32_t n_layers;
  int32_t d_model;
  int32_t n_q_heads;
  int32_t n_kv_heads;
  int32_t head_dim;
  int32_t n_experts;
  int32_t top_k;
  int32_t d_ff;        /* expert hidden width (SwiGLU) */
  int32_t vocab;
  int32_t self_cond;   /* 1: add bf16(e_prev) W_sc^T to the canvas embedding */
  float rope_theta;    /* rotary base (1e4) */
  float rms_eps;       /* RMSNorm epsilon (1e-6) */
} dg_model_config;

/* Lock rules (laozijiushiniubi.cn article §四: lowest-entropy positions are
   locked until the cumulative entropy would exceed 0.1; the benchmark
   configuration locks positions whose max probability exceeds 0.9). */
typedef enum dg_lock_policy {
  DG_LOCK_PROB = 0,            /* lock iff pmax > lock_threshold */
  DG_LOCK_ENTROPY_CUMSUM = 1   /* lock the longest (H, position)-ascending prefix
                                  whose cumulative entropy is <= lock_threshold */
} dg_lock_policy;

/* Sampler parameters (laozijiushiniubi.cn article §四: temperature 0.8 -> 0.4
   linearly; stop on low mean entropy and an unchanged argmax sequence; 48
   rounds budget). */
typedef struct dg_sampler_config {
  int32_t lock_policy;                 /* dg_lock_policy */
  float lock_threshold;                /* 0.9 (PROB) or 0.1 (ENTROPY_CUMSUM) */
  float t_start;                       /* 0.8 */
  float t_end;                         /* 0.4 */
  int32_t max_steps;                   /* round budget, 1..256 */
  float stop_entropy;                  /* stop when mean entropy < this (nats) */
  int32_t stop_require_stable_argmax;  /* also require argmax == previous round's */
  uint64_t seed;                       /* Philox4x32-10 key of the method's draws */
  int32_t persistent_lock;             /* 0: the lock mask is recomputed every round and locked
                                          tokens may change later (the method: laozijiushiniubi.cn
                                          article §一); 1: the masked-style variant, a position once
                                          locked keeps its token for the rest of the block (needs
                                          dg_canvas.locked) */
  int32_t selfcond_topk;               /* 0: the expected embedding over the whole vocabulary (the
                                          method); K in [1, min(1024, vocab)]: the high-batch variant
                                          (laozijiushiniubi.cn article §九, top-k vocabulary
                                          truncation): over each position's K largest bf16 logits
                                          (ties to the lower id), renormalised over them */
} dg_sampler_config;

/* Causally encoded context, one K and one V buffer of dg_kv_bytes() each:
   K bf16 [n_layers][batch][n_kv_heads][c_max][head_dim] (keys after RoPE),
   V transposed, [n_layers][batch][n_kv_heads][head_dim][c_max], in fp16:
   the bf16-rounded values (exact in fp16 for magnitudes >= 2^-14), the
   operand type of the attention's P V product.
   c_max must be a multiple of 8 (16-byte row pitch of the transposed V).
   Positions [0, length) hold the context; a denoising round uses positions
   [length, length + 256) as scratch for the canvas keys, so
   c_max >= length + 256 is required. */
typedef struct dg_kv {
  void* k;
  void* v;
  int32_t batch;
  int32_t c_max;
  int32_t length;   /* in/out: dg_encode_context advances it */
} dg_kv;

/* Per-canvas decoding state, device memory, [batch] canvases. */
typedef struct dg_canvas {
  int32_t* tokens;       /* [B, 256] current canvas; after the final round the block */
  uint16_t* sc_state;    /* [B, 256, d_model] bf16 self-conditioning input (expected
                            embedding of the previous round; zero before round 0) */
  int32_t* prev_argmax;  /* [B, 256] argmax of the previous round */
  uint8_t* done;         /* [B] 1 once the canvas has stopped (frozen) */
  int32_t batch;
  uint8_t* locked;       /* [B, 256] positions committed so far (persistent_lock only; may be
                            NULL otherwise); dg_canvas_init clears it */
} dg_canvas;

typedef struct dg_step_args {
  int32_t block;              /* block index (random stream), >= 0 */
  int32_t step;               /* round index within the block, 0..max_steps-1 */
  dg_sampler_config sampler;
} dg_step_args;

/* Outputs of one round, device memory; NULL members are not written. */
typedef struct dg_step_out {
  int32_t* argmax;        /* [B, 256] most likely token (ties to the lower id) */
  int32_t* sample;        /* [B, 256] Gumbel-max draw from softmax(logits / T_step) */
  float* entropy;         /* [B, 256] untempered entropy, nats */
  float* pmax;            /* [B, 256] untempered max probability */
  uint8_t* lock;          /* [B, 256] lock mask of this round */
  float* mean_entropy;    /* [B] */
  uint8_t* stop;          /* [B] 1 if the adaptive stop fired this round */
  uint8_t* final_round;   /* [B] 1 if this round ended the canvas (stop or budget) */
  float* logits;          /* optional [B, 256, vocab] fp32 LM-head logits */
  int32_t* route_idx;     /* optional [n_layers, B*256, top_k] expert ids */
  float* route_w;         /* optional [n_layers, B*256, top_k] renormalised weights */
  float* route_logits;    /* optional [n_layers, B*256, n_experts] fp32 router logits */
  float* hidden;          /* optional [n_layers + 1, B*256, d_model] fp32 residual stream after
                             the embedding (a1) and after each layer */
  float* hidden_attn;     /* optional [n_layers, B*256, d_model] fp32 residual stream after each
                             layer's attention block (the input of its router and experts) */
} dg_step_out;

/* Host-side statistics of one dg_decode_block call. */
typedef struct dg_block_stats {
  int32_t* steps_taken;      /* host [B]: rounds run for each canvas (may be NULL) */
  int32_t rounds;            /* rounds launched for the batch */
  float tokens_per_pass;     /* tokens finished per round launched: B * 256 / rounds (the pages'
                                tokens per forward pass, laozijiushiniubi.cn article §四, §五) */
  float* distinct_experts;   /* host [n_layers] (may be NULL): per layer, the number of distinct
                                experts the router gave at least one of the batch's canvas tokens,
                                averaged over the block's canvas rounds (a round that also
                                appends a pending block is not counted); the article's "about 84
                                of 128 experts per 256 tokens" (§五) */
} dg_block_stats;

typedef struct dg_ctx dg_ctx;

/* Thread-local text of the last error on this thread ("" if none). */
const char* dg_last_error(void);

/* Bytes of the weight buffer (bf16; layout private to the library). 0 on a
   bad configuration. */
size_t dg_weights_bytes(const dg_model_config* cfg);
/* Bytes of ONE of the two KV buffers (K or V) for `batch` canvases; 0 when
   c_max is not a positive multiple of 8. */
size_t dg_kv_bytes(const dg_model_config* cfg, int32_t batch, int32_t c_max);
/* Bytes of the scratch workspace for up to `batch` canvases. */
size_t dg_workspace_bytes(const dg_model_config* cfg, int32_t batch);
/* The same for a context whose causal encodes (dg_encode_context) run passes
   of up to prefill_tokens tokens (all canvases together; 0 or anything up to
   batch * 256 gives dg_workspace_bytes).  Larger passes read every layer's
   weights once per pass instead of once per 256 tokens: the prompt's
   prefill becomes compute-bound (laozijiushiniubi.cn article §二: the prompt
   is encoded causally, in one go). */
size_t dg_workspace_bytes_ex(const dg_model_config* cfg, int32_t batch, int32_t prefill_tokens);

/* Fill the weight buffer with seeded random-init weights: every matrix from
   the seeded generator of synth/synth.h (approximately N(0, std^2), bf16)
   with std = kind_std[kind] if kind_std is non-NULL and that entry is > 0,
   else 0.02; RMSNorm gains = 1.  Asynchronous on `stream`. */
dg_status dg_model_init_random(const dg_model_config* cfg, uint64_t seed, const float* kind_std,
                               void* d_weights, void* stream);

/* Create a host handle bound to one weight buffer and one workspace.  The
   workspace must hold dg_workspace_bytes(cfg, batch) bytes, 256-byte aligned;
   it is used by every call on this handle, so calls on one handle must not
   overlap on the GPU.  *out is NULL on failure. */
dg_status dg_context_create(const dg_model_config* cfg, const void* d_weights, void* d_workspace,
                            size_t ws_bytes, int32_t batch, dg_ctx** out);
/* dg_context_create for a workspace of dg_workspace_bytes_ex(cfg, batch,
   prefill_tokens) bytes. */
dg_status dg_context_create_ex(const dg_model_config* cfg, const void* d_weights, void* d_workspace,
                               size_t ws_bytes, int32_t batch, int32_t prefill_tokens, dg_ctx** out);
void dg_context_destroy(dg_ctx* ctx);

/* Causal encoding (laozijiushiniubi.cn article §二: the prompt is encoded with
   causal attention): tokens [kv->batch, n] (device int32) are appended at
   positions kv->length .. kv->length + n - 1 of every layer's K/V, then
   kv->length += n.  Processed in passes of up to max(256, prefill_tokens /
   batch) tokens per canvas (prefill_tokens of dg_context_create_ex; the
   canvas batch of the context). */
dg_status dg_encode_context(dg_ctx* ctx, dg_kv* kv, const int32_t* d_tokens, int32_t n,
                            void* stream);

/* Initialise a canvas for block `block`: uniform random tokens (Philox draw
   purpose 1), zero self-conditioning state, prev_argmax = -1, done = 0,
   locked = 0 (when given). */
dg_status dg_canvas_init(dg_ctx* ctx, dg_canvas* cv, int32_t block, uint64_t seed, void* stream);

/* One denoising round over every canvas (the steps a1-a9: embedding plus
   self-conditioning, the transformer layers with bidirectional canvas
   attention into the context, LM head with per-position entropy, max
   probability, argmax and Gumbel-max sample at the annealed temperature,
   the expected embedding for the next round, then mean entropy, stop, lock
   and the next canvas: locked positions keep their sample, the others are
   re-noised uniformly; on stop or at the last budgeted round the canvas
   becomes the argmax sequence and is frozen).  Canvases already done are
   left unchanged.  With sampler.persistent_lock a position locked in an
   earlier round keeps its token (and counts as locked) in every later round,
   the final round included; the other positions follow the rules above. */
dg_status dg_denoise_step(dg_ctx* ctx, const dg_kv* kv, dg_canvas* cv, const dg_step_args* args,
                          const dg_step_out* out, void* stream);

/* A round that first appends a finished block to the context, in the same
   pass (one read of every layer's weights for both): d_append [kv->batch,
   256] (device int32) are appended causally at positions kv->length ..
   kv->length + 255 of each canvas's context, exactly as dg_encode_context
   would (laozijiushiniubi.cn article §二, §四: a finished block becomes
   context), while the canvas round of dg_denoise_step runs on the positions
   after them, seeing the appended block; then kv->length += 256.  Needs
   c_max >= length + 512 and a workspace for layer passes of 512 tokens per
   canvas (dg_workspace_bytes_ex, prefill_tokens >= batch * 512, else
   DG_ERR_WORKSPACE).  The routing outputs hold the canvas rows' routing
   ([n_layers, B*256, ...], as in dg_denoise_step); the hidden-state outputs
   are not available (must be NULL, else DG_ERR_INVALID_ARG).  Asynchronous. */
dg_status dg_denoise_step_append(dg_ctx* ctx, dg_kv* kv, dg_canvas* cv, const dg_step_args* args,
                                 const int32_t* d_append, const dg_step_out* out, void* stream);

/* The same round as dg_denoise_step, replayed from a CUDA graph that the
   context captures on first use and keeps while the KV cache (pointers and
   length), canvas and output pointers stay the same (a change re-captures
   it).  Results are bit-identical to dg_denoise_step.  Falls back to direct
   launches while profiling is on.  The graph belongs to the context: do not
   call this concurrently on one context. */
dg_status dg_denoise_step_graph(dg_ctx* ctx, const dg_kv* kv, dg_canvas* cv, const dg_step_args* args,
                                const dg_step_out* out, void* stream);

/* Decode one block per canvas: dg_canvas_init, rounds until every canvas has
   stopped or the budget is spent (one 8-byte device-to-host read per round),
   copy the blocks to d_out [B, 256] and append them to the context with
   dg_encode_context.  `args->step` is ignored.  h_stats may be NULL. */
dg_status dg_decode_block(dg_ctx* ctx, dg_kv* kv, dg_canvas* cv, const dg_step_args* args,
                          int32_t* d_out, dg_block_stats* h_stats, void* stream);

/* dg_decode_block with the block append fused into the next block's first
   round: d_pending (device [batch, 256], may be NULL) is a finished block
   not yet in the context; this block's round 0 appends it
   (dg_denoise_step_append).  With DG_DECODE_DEFER_APPEND in `flags` the
   block decoded here is not appended at the end (the caller passes d_out as
   the next call's d_pending, a different buffer from that call's d_out).
   Needs a context created with dg_context_create_ex(prefill_tokens >=
   batch * 512) when d_pending is given. */
#define DG_DECODE_DEFER_APPEND 1
dg_status dg_decode_block_ex(dg_ctx* ctx, dg_kv* kv, dg_canvas* cv, const dg_step_args* args,
                             const int32_t* d_pending, int32_t flags, int32_t* d_out,
                             dg_block_stats* h_stats, void* stream);

/* Retained autoregressive mode (laozijiushiniubi.cn article §七: the same
   weights still generate one token at a time), the comparison workload of
   the method: d_tokens [kv->batch] (device int32) are appended at position
   P = kv->length of each canvas's context with causal attention (the causal
   encode of one token), then that position's final RMSNorm, LM head and
   vocabulary statistics give the next token: its argmax (ties to the lower
   id) to d_argmax [batch] and its Gumbel-max draw from softmax(l /
   temperature) to d_sample [batch] (Philox4x32-10 with key = seed, counter
   (c0 = v / 4, c1 = 0, c2 = P, c3 = 5 << 24 | canvas), word v % 4).
   d_logits (optional, NULL for none) [batch, vocab] fp32.  kv->length += 1.
   Asynchronous on `stream`; uses the context's workspace. */
dg_status dg_ar_step(dg_ctx* ctx, dg_kv* kv, const int32_t* d_tokens, float temperature, uint64_t seed,
                     int32_t* d_argmax, int32_t* d_sample, float* d_logits, void* stream);

/* Synchronise `stream` and report (then clear) the device error word:
   DG_OK, DG_ERR_BAD_TOKEN or DG_ERR_TIMEOUT. */
dg_status dg_check_device_error(dg_ctx* ctx, void* stream);

/* ---- measurement hooks (not part of the method) --------------------------
   While profiling is on, every launch made through the context is counted
   and the launches of the classes below are bracketed by CUDA events on
   their own stream; dg_profile_stop synchronises those events and returns the
   summed device time per class. */
enum {
  DG_PROF_EXPERT_GATE_UP = 0,  /* grouped gate/up projection + SwiGLU (one launch per layer) */
  DG_PROF_EXPERT_DOWN = 1,     /* grouped down projection (one launch per layer) */
  DG_PROF_LM_HEAD = 2,         /* LM head + online vocabulary statistics + Gumbel keys */
  DG_PROF_ATTENTION = 3,       /* attention (+ split merge) */
  DG_PROF_DENSE = 4,           /* QKV, output, router and self-conditioning projections */
  DG_PROF_EXPECTED_EMB = 5,    /* softmax probabilities + expected-embedding product + reduce */
  DG_PROF_KINDS = 6
};
typedef struct dg_profile {
  double ms[DG_PROF_KINDS];        /* summed device milliseconds per class */
  int32_t launches[DG_PROF_KINDS]; /* profiled launches per class */
  int64_t launches_total;          /* every kernel launched while profiling was on */
} dg_profile;
/* Start counting (clears previous totals).  Events are created on first use
   and reused; at most 65536 profiled launches are kept per start/stop. */
dg_status dg_profile_start(dg_ctx* ctx);
/* Stop, synchronise the recorded events and fill *out. */
dg_status dg_profile_stop(dg_ctx* ctx, dg_profile* out);

/* Router-load probe (measurement hook): layer `layer`'s RMSNorm, router
   product and top-k routing on T (1 <= T <= the context's batch * 256) given
   hidden states d_x [T, d_model] fp32 (device), exactly as that layer routes
   its residual stream in a round; d_idx [T, top_k] int32 (device) receives
   each token's experts (selection order).  It uses the context's workspace,
   so it must not overlap other calls on the context.  Asynchronous. */
dg_status dg_router_probe(dg_ctx* ctx, int32_t layer, const float* d_x, int32_t T, int32_t* d_idx,
                          void* stream);

/* ---- attention without caller-provided scratch ---------------------------
   The pages have no counterpart for this call.  It is for callers that cannot
   allocate device memory when they call in: code that runs inside a memory
   pool sized once at start-up, a host program whose allocator is closed after
   initialisation, or a caller that has no CUDA allocator of its own.

   Computes the same attention as dg_test_attention (dg_testing.h), with the
   same argument meaning and layout: q bf16 packed by kv head
   [B][Hkv][nq][Hq / Hkv][hd], K cache bf16 [B][Hkv][c_max][hd], V cache
   transposed fp16 [B][Hkv][hd][c_max], both holding keys [0, L0 + nq),
   c_max a multiple of 8; out bf16 [B * nq, Hq * hd]; causal as there;
   splits 1..8 key splits (0 means 1).  All four pointers are device memory
   owned by the caller.  The split-KV partial
   results, which dg_test_attention takes from the caller, live here in one
   fixed array inside the library, DG_ATTN_STATIC_SCRATCH_BYTES long (16 MiB);
   every GPU the library runs on holds its own copy for the life of the
   process.  No cudaMalloc, cudaFree or other allocating routine is called.

   Limit: splits * B * Hq * nq * (hd + 2) * 4 bytes (plus up to 256 bytes of
   alignment) must fit the array; a larger request returns DG_ERR_INVALID_ARG
   and launches nothing.  splits 0 or 1 uses no scratch.
   Set-up: the first call on each GPU (that GPU current) looks up the array's
   address (cudaGetSymbolAddress; nothing is allocated); make that first call
   before any stream capture begins.
   Nothing has to start at zero: each call writes every partial it reads.
   One array per GPU: calls on the same GPU that may run at the same time
   (several host threads, or streams with no ordering between them) race on
   it, so the caller serialises them.  Every call synchronises `stream` (it
   waits for its work there to finish) before it returns. */
#define DG_ATTN_STATIC_SCRATCH_BYTES (16u << 20)
dg_status dg_attention_static_scratch(const uint16_t* d_q, const uint16_t* d_k, const uint16_t* d_v,
                                      uint16_t* d_out, int32_t B, int32_t nq, int32_t L0, int32_t c_max,
                                      int32_t Hq, int32_t Hkv, int32_t hd, int32_t causal, int32_t splits,
                                      void* stream);

#ifdef __cplusplus
}
#endif
#endif /* DG_H */
