/*
 * rlt.h -- C ABI of the B200 (sm_100a) Recurrent Looped Transformer decoder.
 *
 * Page key used in the citations below:
 *   [RLT-96] "RLT Runs 96 Blocks Per Token With Recurrent State, No Resets"
 *            (aimastery.page)
 *   [RLT-TC] "Recurrent Looped Transformer (RLT): prompts in parallel, depth in
 *            sequence" (thakicloud.com)
 *   [RLT-FT] "Recurrent Looped Transformer debunked" (flowtivity.ai)
 *   [RLT-PV] "Per-token recurrence, no quality gain" (news.promtvault.app)
 *
 * The model: a causal encoder turns every known token into e_t and projects
 * the prefix-restricted key/value memory M<=t, shared by all decoder layers
 * (G = 1) or one per decoder layer (G = L_D) ([RLT-96] "Architecture: encoder
 * memory meets recurrent decoder"). A recurrent decoder carries the state
 * H_t = (s_t, C_t^D): s_t the final decoder output vector, C_t^D the retained
 * sliding-window keys/values of every decoder layer, W - 1 of them since the
 * window W includes the current token. Each transition H_{t-1} -> H_t runs a
 * gated merge of e_t with s_{t-1} (feedback scale alpha), then per decoder
 * block causal SWA, cross-attention to M<=t and an FFN (same section). The
 * state starts from the learned s* and an empty cache and is never reset at
 * the prompt/response boundary ([RLT-TC] "What is this technology").
 * Independent sequences share one batched step ([RLT-96] "Three design
 * principles and their caveats", model-hardware co-design).
 *
 * Conventions for every call:
 *   - Every call returns an rlt_status (RLT_OK = 0) unless stated otherwise.
 *   - Arguments are validated completely on the host before anything is
 *     enqueued: a call that returns an error changed no state.
 *   - Device work is enqueued asynchronously on `stream` (a cudaStream_t;
 *     NULL = the legacy default stream). Host pointers named h_* are read
 *     before the call returns.
 *   - The library allocates no device memory: all device state lives in the
 *     caller's arena (rlt_arena_bytes), owned by the caller.
 *   - One model is driven from one host thread at a time.
 *   - Matrices are row-major [out][in] (y = W x). The q/k/v projection stacks
 *     rows q | k | v; head h owns entries h*dh .. h*dh + dh - 1 of each.
 */
#ifndef RLT_H
#define RLT_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define RLT_API __attribute__((visibility("default")))
#define RLT_MAX_LAYERS 64

typedef struct CUstream_st *rlt_stream; /* the same type as cudaStream_t */
typedef struct rlt_model rlt_model;     /* opaque; host memory only */

typedef enum rlt_status {
  RLT_OK = 0,
  RLT_ERR_INVALID_ARG = 1,  /* null pointer, bad size, id out of range */
  RLT_ERR_UNSUPPORTED = 2,  /* shape the kernels do not cover */
  RLT_ERR_NOT_READY = 3,    /* t_dec >= t_enc: e_t / M<=t not produced yet */
  RLT_ERR_CAPACITY = 4,     /* position or arena capacity exceeded */
  RLT_ERR_DUPLICATE_ID = 5, /* a sequence listed twice in one batch */
  RLT_ERR_CUDA = 6,         /* a CUDA runtime call failed */
  RLT_ERR_TIMEOUT = 7,      /* a bounded device wait gave up */
  RLT_ERR_DEVICE = 8,       /* a kernel's own bounds check fired */
  RLT_ERR_STALE = 9         /* snapshot of another configuration or other weights */
} rlt_status;

enum { RLT_GELU = 0, RLT_SWIGLU = 1 }; /* FFN form */
enum { RLT_F32 = 0, RLT_BF16 = 1 };    /* storage of matrices, K/V, e, M */

/* Model shape and capacity. [RLT-96] "Architecture" names d-independent
 * quantities W (window, includes the current token) and G (memory groups). */
typedef struct rlt_config {
  int d;            /* model width; d = n_heads * head_dim */
  int n_heads;      /* heads of self- and cross-attention */
  int head_dim;     /* 16, 32, 64 or 128 */
  int n_enc_layers; /* L_E */
  int n_dec_layers; /* L_D */
  int ffn_dim;      /* F */
  int ffn_kind;     /* RLT_GELU: W2 GELU(W1 u); RLT_SWIGLU: W2 (SiLU(Wa u) * Wb u) */
  int vocab;        /* V */
  int window;       /* W >= 1, at most RLT_ATTEND_CHUNK (1024) */
  int mem_groups;   /* G: 1 or n_dec_layers */
  int tied;         /* 1: decoder layer l uses encoder layer l's q/k/v, o and
                       FFN matrices ([RLT-96] "Architecture", tied config) */
  int dtype;        /* RLT_F32 or RLT_BF16 */
  int max_seqs;     /* sequence slots in the arena */
  int max_len;      /* positions per sequence (encoder memory capacity) */
  int max_prefill_tokens; /* encoder work buffer, tokens; 0 = automatic */
  int enc_cache;    /* 1: keep every encoder layer's rotary keys and values of
                       every position, so tokens can be appended one at a time
                       (rlt_append_encoder, rlt_serve_step) and snapshots carry
                       the encoder cache; 0: whole-sequence prefill only */
  float alpha;      /* feedback scale of the gated merge; 0 turns feedback off */
  float rms_eps;    /* RMSNorm epsilon (1e-6) */
  float rope_theta; /* rotary base (1e4) */
} rlt_config;

/* Borrowed device pointers, alive until rlt_destroy. Matrices are in the
 * model dtype; norm gains, gate bias and s* are always float32.
 *   embed [V][d]
 *   enc_ln1/enc_ln2 [d], enc_wqkv [3d][d], enc_wo [d][d],
 *   enc_w1 [F][d] (GELU W1, or SwiGLU Wa), enc_wb [F][d] (SwiGLU Wb, else
 *   unused), enc_w2 [d][F], enc_lnf [d]
 *   mem_wk/mem_wv [d][d] per group
 *   gate_w [d][2d] (columns 0..d-1 multiply e_t, d..2d-1 multiply s_{t-1}),
 *   gate_b [d], sstar [d]
 *   dec_ln1/ln2/ln3 [d], dec_wqkv, dec_wo, dec_wqx [d][d], dec_wox [d][d],
 *   dec_w1, dec_wb, dec_w2 as in the encoder (ignored when tied), dec_lnf [d]
 */
typedef struct rlt_weights {
  const void *embed;
  const void *enc_ln1[RLT_MAX_LAYERS], *enc_wqkv[RLT_MAX_LAYERS],
      *enc_wo[RLT_MAX_LAYERS], *enc_ln2[RLT_MAX_LAYERS],
      *enc_w1[RLT_MAX_LAYERS], *enc_wb[RLT_MAX_LAYERS], *enc_w2[RLT_MAX_LAYERS];
  const void *enc_lnf;
  const void *mem_wk[RLT_MAX_LAYERS], *mem_wv[RLT_MAX_LAYERS];
  const void *gate_w, *gate_b, *sstar;
  const void *dec_ln1[RLT_MAX_LAYERS], *dec_wqkv[RLT_MAX_LAYERS],
      *dec_wo[RLT_MAX_LAYERS], *dec_ln2[RLT_MAX_LAYERS],
      *dec_wqx[RLT_MAX_LAYERS], *dec_wox[RLT_MAX_LAYERS],
      *dec_ln3[RLT_MAX_LAYERS], *dec_w1[RLT_MAX_LAYERS],
      *dec_wb[RLT_MAX_LAYERS], *dec_w2[RLT_MAX_LAYERS];
  const void *dec_lnf;
} rlt_weights;

/* Host only. RLT_OK if the kernels cover `cfg`; else why not. */
RLT_API int rlt_check_config(const rlt_config *cfg);

/* Host only. Bytes of device arena rlt_create needs for `cfg` (0 if the
 * config is invalid). The arena holds s, the ring KV cache, e, M, positions
 * and all work buffers. */
RLT_API size_t rlt_arena_bytes(const rlt_config *cfg);

/* Bind a model to weights and an arena (>= rlt_arena_bytes, 256-byte
 * aligned device memory owned by the caller). Runs set-up kernels on the
 * legacy default stream and waits for them; every sequence slot starts reset.
 * *out receives a host handle released by rlt_destroy. */
RLT_API int rlt_create(const rlt_config *cfg, const rlt_weights *weights,
                       void *d_arena, size_t arena_bytes, rlt_model **out);

/* Release the host handle (not the arena, not the weights). NULL is a no-op. */
RLT_API void rlt_destroy(rlt_model *model);

/* Slot `seq`: s <- s*, empty cache, t_dec = t_enc = 0 ([RLT-96]
 * "Architecture": start state and empty cache before the first token). */
RLT_API int rlt_reset_seq(rlt_model *model, int seq, rlt_stream stream);

/* Causal encoder + memory projection over whole sequences from position 0
 * ([RLT-96] "Architecture"; [RLT-TC] "What is this technology": token-
 * parallel prefill). Sequence h_seq_ids[i] gets tokens
 * tokens[h_offsets[i] .. h_offsets[i] + h_lengths[i]) (int32; `tokens` may be
 * a device pointer or pinned host memory). Sets t_enc = length and resets the
 * decoder state of those slots (s*, empty cache, t_dec = 0).
 * Errors: INVALID_ARG (ids, offsets, token values are not checked on the host
 * but out-of-range tokens set RLT_ERR_DEVICE), DUPLICATE_ID, CAPACITY
 * (length > max_len). */
RLT_API int rlt_prefill_encoder(rlt_model *model, const int32_t *tokens,
                                const int32_t *h_seq_ids,
                                const int32_t *h_offsets,
                                const int32_t *h_lengths, int n,
                                rlt_stream stream);

/* One transition H_{t-1} -> H_t for each listed sequence, batched into one
 * step (t = that sequence's own t_dec). Errors: INVALID_ARG, DUPLICATE_ID,
 * NOT_READY (t_dec >= t_enc), CAPACITY (t_dec >= max_len). */
RLT_API int rlt_decoder_step(rlt_model *model, const int32_t *h_ready_ids,
                             int n_ready, rlt_stream stream);

/* n_steps lock-step transitions of the listed sequences (every sequence must
 * have n_steps positions ready). Equivalent to n_steps rlt_decoder_step calls
 * with the same list. On a non-NULL stream every step after the first of its
 * shape replays a captured CUDA graph (the graphs are cached in the model and
 * keyed by the batch bound and the cross-attention split count), so the first
 * call on such a stream must not itself be inside a stream capture. */
RLT_API int rlt_run_sequence(rlt_model *model, const int32_t *h_seq_ids, int n,
                             int n_steps, rlt_stream stream);

/* Token-parallel decoder pass for feedback off (alpha = 0). With alpha = 0
 * the transition at t never reads s_{t-1} (x_t = e_t), so every decoder
 * quantity at t depends only on e_0..e_t: the n_steps transitions of a fresh
 * sequence can run for all positions at once, block by block, as a
 * window-masked causal prefill (the feedback-off ablation of [RLT-PV]
 * "Per-token recurrence, no quality gain" and the parallel-training argument
 * of [RLT-FT] "How slow is per-token recurrence to train?"). The result is
 * the recurrent state after n_steps transitions: s = s_{n_steps-1}, each
 * layer's window of rotary k and v, t_dec = n_steps, so rlt_decoder_step
 * continues from there. s_all (optional, device memory, fp32
 * [n][n_steps][d], row i of sequence h_seq_ids[i]) receives every s_t.
 * Sequences are processed in chunks of whole sequences that fit the prefill
 * buffers (max_prefill_tokens).
 * Errors: INVALID_ARG (bad ids, n_steps < 0, or a sequence that has already
 * taken a decoder step), DUPLICATE_ID, NOT_READY (t_enc < n_steps),
 * CAPACITY (n_steps > max_len), UNSUPPORTED (alpha != 0). */
RLT_API int rlt_decoder_parallel(rlt_model *model, const int32_t *h_seq_ids, int n,
                                 int n_steps, float *s_all, rlt_stream stream);

/* How a bf16 model's decoder step runs.
 *   RLT_STEP_FUSED: one launch of a persistent kernel per step. Thread-block
 *     clusters, as many as can be resident, walk the step's work -- GEMM
 *     tiles of every projection on the tensor cores, attention units, the
 *     gather and the final norm -- in one global order (layer, sublayer
 *     phase, 128-row tile), each waiting on dependency counters in the arena
 *     instead of on kernel boundaries ([RLT-96] "Three design principles and
 *     their caveats": kernel fusion and batched ready updates). Available
 *     for the bf16 models it covers (up to 8192 slots, 64 decoder layers).
 *   RLT_STEP_CHAIN: a captured chain of about eight kernels per decoder
 *     block; the default (measured faster), and the only form for fp32
 *     models.
 * Both compute the same transition; results agree within the bf16
 * tolerance, not bit for bit (different split-K partitions). */
enum { RLT_STEP_CHAIN = 0, RLT_STEP_FUSED = 1 };

/* Select the step kernel for later steps. Errors: INVALID_ARG (unknown
 * kind), UNSUPPORTED (RLT_STEP_FUSED for a model it does not cover). */
RLT_API int rlt_set_step_kernel(rlt_model *model, int kind);

/* The step kernel later steps use (RLT_STEP_CHAIN or RLT_STEP_FUSED); -1 for
 * a NULL model. */
RLT_API int rlt_get_step_kernel(rlt_model *model);

/* CTAs of one persistent-step launch (0 if the model does not have it). */
RLT_API int rlt_step_kernel_ctas(rlt_model *model);

/* Measurement hook of the persistent step (no counterpart in the method).
 * d_buf (device, 8-byte aligned, NULL = off) receives, for every CTA c and
 * work item k it runs in a step, 4 uint64 words at
 * ((c * cap + k) * 4): item id, start, dependency met, end, in device
 * globaltimer nanoseconds; cap = bytes / (32 * rlt_step_kernel_ctas()).
 * Item id = (layer + 1) << 16 | phase << 8 | row tile, where phase bit 7
 * marks an attention sublayer (phases: 0 q/k/v GEMM, 1 SWA, 2 W_o, 3 W_qx,
 * 4 cross-attention, 5 W_ox, 6 FFN up, 7 SwiGLU value half, 8 FFN down;
 * layer slot L_D: 1 gate GEMM, 0x20 gather, 0x21 final norm). Slots a step
 * does not use keep their contents: clear the buffer between steps.
 * Synchronises the model's last stream and drops its captured step graphs.
 * Errors: INVALID_ARG (misaligned or smaller than one record per CTA),
 * UNSUPPORTED (no persistent step for this model). */
RLT_API int rlt_set_step_trace(rlt_model *model, void *d_buf, size_t bytes);

/* Ready-set scheduler: sequence h_seq_ids[i] still needs h_steps[i]
 * transitions. Each tick batches every sequence with a pending step into one
 * decoder step, until none is left (ragged batches: sequences drop out as
 * they finish). Same errors as rlt_decoder_step, checked for every tick
 * before any is enqueued. */
RLT_API int rlt_run_ragged(rlt_model *model, const int32_t *h_seq_ids,
                           const int32_t *h_steps, int n, rlt_stream stream);

/* Host only: the scheduler's plan. h_tick_sizes[k] = number of sequences in
 * tick k (k < *n_ticks <= max_ticks); h_order lists the n sequence indices in
 * the order ticks batch them (ids that finish last first). */
RLT_API int rlt_plan_ragged(const int32_t *h_steps, int n, int32_t *h_order,
                            int32_t *h_tick_sizes, int max_ticks, int *n_ticks);

/* Export H_t of slot `seq`: s_out [d] float32; cache_out [L_D][2][W-1][d]
 * in the model dtype, K rows then V rows, positions t-(W-1) .. t-1 oldest
 * first with slots of negative positions zero; *t_out = t (number of
 * transitions taken). Any output may be NULL; outputs may be device or
 * pinned host memory and are complete when `stream` reaches this point.
 * K entries are stored with their rotary encoding applied. */
RLT_API int rlt_get_state(rlt_model *model, int seq, float *s_out,
                          void *cache_out, int64_t *t_out, rlt_stream stream);

/* Import H_t into slot `seq` (same layouts as rlt_get_state). t must be
 * <= max_len. Inputs may be device or pinned host memory. */
RLT_API int rlt_set_state(rlt_model *model, int seq, const float *s_in,
                          const void *cache_in, int64_t t, rlt_stream stream);

/* ------------------------------------------------------------ serving loop
 * Once tokens are no longer given, each generated token goes back into the
 * encoder, so the encoder cache and memory are part of the serving state
 * ([RLT-96] "Training and serving implications"). These calls need a model
 * created with enc_cache = 1. */

/* Append one token to the encoder of each listed sequence (tokens[i] for
 * h_seq_ids[i]; device or pinned host int32): the causal encoder runs at
 * position t = t_enc over the encoder cache of positions 0..t-1 (the
 * encoder is causal, [RLT-TC] "What is this technology", so this equals a
 * whole-sequence prefill of the longer prompt at that position), writes e_t
 * and the memory rows M_t of every group, and t_enc += 1.
 * Errors: INVALID_ARG, DUPLICATE_ID, UNSUPPORTED (enc_cache = 0), CAPACITY
 * (t_enc = max_len); out-of-range tokens set RLT_ERR_DEVICE. */
RLT_API int rlt_append_encoder(rlt_model *model, const int32_t *tokens,
                               const int32_t *h_seq_ids, int n, rlt_stream stream);

/* Next-token logits from each listed sequence's current s_t ([RLT-96]
 * "Architecture": the next-token distribution is read from s_t), with the
 * embedding matrix as the output head: logits[i][v] = embed[v] . s (device
 * float32 [n][vocab]). bf16 models round s to bf16 for the tensor cores.
 * Errors: INVALID_ARG, DUPLICATE_ID, UNSUPPORTED (bf16 with vocab % 64). */
RLT_API int rlt_lm_head(rlt_model *model, const int32_t *h_seq_ids, int n, float *logits,
                        rlt_stream stream);

/* One token per row from logits (device float32 [n][vocab]) into tokens_out
 * (device int32 [n]). temperature 0: the argmax (lowest index among equal
 * maxima). temperature > 0: the inverse CDF of softmax(logits /
 * temperature) at uniforms[i] (device float32 [n] in [0, 1), drawn by the
 * caller): the smallest v whose cumulative weight exceeds uniforms[i] times
 * the total, summed in a fixed order in fp32 (reproducible).
 * Errors: INVALID_ARG (negative or non-finite temperature, null pointers). */
RLT_API int rlt_sample(rlt_model *model, const float *logits, int n, float temperature,
                       const float *uniforms, int32_t *tokens_out, rlt_stream stream);

/* One autoregressive step for each listed sequence, whose decoder stands at
 * its last known token (t_dec = t_enc - 1): the transition at t = t_dec,
 * logits from the new s_t (rlt_lm_head; `logits` is caller workspace,
 * device float32 [n][vocab], left holding them), a token drawn as
 * rlt_sample does into tokens_out (device int32 [n]), and that token
 * appended to the encoder (rlt_append_encoder), so the next call continues.
 * Errors: as the calls it runs; NOT_READY when t_dec != t_enc - 1. */
RLT_API int rlt_serve_step(rlt_model *model, const int32_t *h_seq_ids, int n,
                           float temperature, const float *uniforms, float *logits,
                           int32_t *tokens_out, rlt_stream stream);

/* ------------------------------------------------------------ snapshots
 * An exact prefix snapshot of one slot: everything a later transition of
 * that sequence reads, so restoring it into any slot of a model with the
 * same configuration and the same weight values continues bit for bit as
 * if nothing had happened ([RLT-96] "Training and serving implications":
 * encoder cache and memory, the full decoder state, position metadata, the
 * window convention and a model version; "RLT carries decoder state between
 * tokens..." (lub-systems.com), "How to prepare systems for state storage
 * and transfer": a weight update invalidates stored states).
 * Layout: this header, then the sections at the header's byte offsets
 * (256-byte aligned), in the model dtype unless noted:
 *   s        [d] float32                      decoder output s_{t_dec - 1}
 *   window   [L_D][2][W-1][d]                 as rlt_get_state
 *   e        [t_enc][d]                       encoder outputs
 *   mem      [G][t_enc][2][d]                 memory rows (K row, V row)
 *   enc_kv   [L_E][t_enc][2][d]               encoder cache (enc_cache only)
 * The fingerprint is a 64-bit hash of the configuration and of every weight
 * value the model reads, computed on the device when the snapshot is taken
 * and again when it is restored. */
#define RLT_SNAPSHOT_MAGIC 0x3150414E53544C52ull /* "RLTSNAP1", little-endian */
typedef struct rlt_snapshot_header {
  uint64_t magic;       /* RLT_SNAPSHOT_MAGIC */
  uint64_t fingerprint; /* configuration and weight values */
  uint64_t bytes;       /* the whole snapshot, header included */
  uint64_t off_s, off_window, off_e, off_mem, off_enc_kv; /* section offsets */
  int64_t t_dec, t_enc; /* transitions taken, encoder positions known */
  int32_t version;      /* 1 */
  int32_t d, n_heads, head_dim, n_enc_layers, n_dec_layers, ffn_dim, ffn_kind, vocab;
  int32_t window, mem_groups, tied, dtype, enc_cache;
  float alpha, rms_eps, rope_theta;
} rlt_snapshot_header;

/* Host only. Bytes of slot `seq`'s snapshot as it stands (0 if invalid). */
RLT_API size_t rlt_snapshot_bytes(rlt_model *model, int seq);

/* Write slot `seq`'s snapshot to buf (device or pinned host memory, >=
 * rlt_snapshot_bytes); complete when `stream` reaches this point.
 * Errors: INVALID_ARG, CAPACITY (bytes too small). */
RLT_API int rlt_get_snapshot(rlt_model *model, int seq, void *buf, size_t bytes,
                             rlt_stream stream);

/* Restore a snapshot (device or pinned host memory) into slot `seq`. Reads
 * and checks the header and recomputes the weight fingerprint before
 * returning (synchronising `stream`), then enqueues the copies. Errors:
 * INVALID_ARG (not a snapshot, sizes), STALE (another configuration or other
 * weight values), CAPACITY (positions beyond max_len). */
RLT_API int rlt_set_snapshot(rlt_model *model, int seq, const void *buf, size_t bytes,
                             rlt_stream stream);

/* Host only (synchronous): the fingerprint snapshots carry for this model's
 * configuration and current weight values. */
RLT_API int rlt_model_fingerprint(rlt_model *model, uint64_t *out);

/* ---------------------------------------------------------------- training
 * Backpropagation through time of the decoder recurrence. The decoder is
 * trained by full backpropagation through time ([RLT-PV] "Per-token
 * recurrence, no quality gain", body: a custom reverse-traversal backward
 * pass), and both parts of the carried state H_t = (s_t, C_t^D) carry
 * gradient: the state-to-state Jacobian has cross-terms through the decoder
 * cache, so a truncation that detaches s alone leaves paths open through it
 * ([RLT-96] "Training and serving implications").
 *
 * Gradients of the decoder's parameters and of the memory projection:
 * float32 device buffers the caller owns, each shaped like its weight
 * (rlt_weights), ADDED into (zero them before the first call; successive
 * calls accumulate, as chunks and batches of one optimizer step should). For
 * a tied model dec_wqkv, dec_wo, dec_w1, dec_wb, dec_w2 receive the decoder's
 * use of the shared encoder matrices. dec_wb only for SwiGLU; mem_wk/mem_wv
 * for g < G. */
typedef struct rlt_grads {
  float *gate_w, *gate_b, *sstar, *dec_lnf;
  float *dec_ln1[RLT_MAX_LAYERS], *dec_wqkv[RLT_MAX_LAYERS], *dec_wo[RLT_MAX_LAYERS],
      *dec_ln2[RLT_MAX_LAYERS], *dec_wqx[RLT_MAX_LAYERS], *dec_wox[RLT_MAX_LAYERS],
      *dec_ln3[RLT_MAX_LAYERS], *dec_w1[RLT_MAX_LAYERS], *dec_wb[RLT_MAX_LAYERS],
      *dec_w2[RLT_MAX_LAYERS];
  float *mem_wk[RLT_MAX_LAYERS], *mem_wv[RLT_MAX_LAYERS];
} rlt_grads;

/* Floats per row of a carried state gradient: [s: d] then the cache
 * [L_D][2][W-1][d] in the rlt_get_state layout (positions tb-(W-1) .. tb-1,
 * oldest first; entries of negative positions are zero). */
#define RLT_CARRY_FLOATS(d, n_dec_layers, window) \
  ((size_t)(d) * (1 + 2 * (size_t)(n_dec_layers) * ((window) - 1)))

/* Host only. Device workspace bytes of rlt_backward for n rows and n_steps
 * positions (0 if the configuration is invalid). It holds the recorded s_t
 * and keys/values of the chunk, the activations of a batch of up to eight
 * recomputed steps, the saved cross-attention terms, the saved SWA terms of
 * the last 8 + W steps and the memory-row gradients: about
 * n * n_steps * L_D * d * 8 + G * n * max_len * d * 8 bytes plus a term
 * independent of n_steps. */
RLT_API size_t rlt_backward_workspace_bytes(const rlt_config *cfg, int n, int n_steps);

/* One chunk of backpropagation through time for the listed sequences, all
 * at the same position t0 = t_dec (e.g. 0 after rlt_reset_seq).
 *   1. The forward of positions t0 .. t1-1 (t1 = t0 + n_steps) runs on the
 *      model's own step kernels, exactly as rlt_run_sequence, recording s_t
 *      and every layer's (k_t, v_t) in the workspace; the sequences end at
 *      t_dec = t1 as after rlt_run_sequence.
 *   2. Reverse traversal t = t1-1 .. t0: the forward is recomputed from
 *      the recorded state (up to eight steps at once) and each step is
 *      differentiated layer by layer; a key or value entry's gradient
 *      accumulates over the steps that read it.
 *   3. The gradient of the memory rows M<=t1-1 is pushed through the memory
 *      projection into e and the mem_wk / mem_wv gradients.
 * The loss is L = sum_t <d_sgrad[i][t-t0], s_t> (+ <d_carry_in, H_{t1-1}>):
 *   d_sgrad     device float32 [n][n_steps][d]: dL/ds_t (e.g. from an LM head)
 *   d_carry_in  device float32 [n][RLT_CARRY_FLOATS] or NULL: the gradient of
 *               the state leaving the chunk (from the chunk after it)
 *   d_carry_out device float32 [n][RLT_CARRY_FLOATS] or NULL: written with the
 *               gradient of the state entering the chunk, H_{t0-1}
 *   d_egrad     device float32 [n][max_len][d], ADDED into: dL/de_j for rows
 *               j < t1 (the encoder's gradient, for the encoder's backward)
 *   grads       accumulated parameter gradients; when t0 = 0 the gradient of
 *               s_{-1} = s* is also added into grads->sstar.
 * Exact chunked backpropagation: run the forward over all chunks keeping the
 * state at each chunk start (rlt_get_state), then for the chunks in reverse
 * restore that state (rlt_set_state) and call this with the previous call's
 * d_carry_out as d_carry_in. Arithmetic is fp32 with the weights in the model
 * dtype; the recorded keys and values are the forward's own.
 * Errors: INVALID_ARG (null pointers, n < 1, n_steps < 1, sequences at
 * different t_dec, workspace too small or not 256-byte aligned, a needed
 * gradient buffer missing), DUPLICATE_ID, CAPACITY, NOT_READY (t1 > t_enc). */
RLT_API int rlt_backward(rlt_model *model, const int32_t *h_seq_ids, int n, int n_steps,
                         const float *d_sgrad, const float *d_carry_in, float *d_carry_out,
                         float *d_egrad, const rlt_grads *grads, void *d_work,
                         size_t work_bytes, rlt_stream stream);

/* Export the encoder output of slot `seq`: e_out [t_enc][d] and mem_out
 * [G][t_enc][2][d] (K row then V row per position) in the model dtype.
 * Either may be NULL. */
RLT_API int rlt_get_encoder_output(rlt_model *model, int seq, void *e_out,
                                   void *mem_out, int64_t *t_enc_out,
                                   rlt_stream stream);

/* Memory positions per split of rlt_attend (and of the decoder's
 * cross-attention for models with max_seqs * n_heads >= 2048; 256 below
 * that): rows longer than this are split into chunks of
 * this many positions and merged in chunk order. */
#define RLT_ATTEND_CHUNK 1024

/* Bytes of device workspace rlt_attend needs (0 if the shape is invalid). */
RLT_API size_t rlt_attend_workspace_bytes(int n, int n_heads, int head_dim, int cap);

/* The decoder's cross-attention kernel as a standalone operation: for every
 * row i < n and head h, out[i][h] = softmax(q[i][h] . K_j / sqrt(dh)) V_j
 * over the first h_lengths[i] rows j of that (row, head)'s key and value
 * blocks -- one query against a prefix-restricted memory M<=t ([RLT-96]
 * "Architecture": cross-attention to encoder memory; [RLT-TC] "What is this
 * technology": the prefix-restricted global KV memory).
 *   q       device, float32 [n][n_heads][head_dim]
 *   kv      device, dtype, [n][n_heads][2][cap][head_dim]: a key block of
 *           cap rows, then a value block of cap rows, per (row, head)
 *   h_lengths host, int32 [n], each in [1, cap]; read before return
 *   out     device, dtype, [n][n_heads][head_dim]
 *   workspace device, >= rlt_attend_workspace_bytes(n, n_heads, head_dim,
 *           cap) bytes, 256-byte aligned, owned by the caller; its first
 *           int32 is a device error word (0 = ok, RLT_ERR_TIMEOUT if a
 *           bounded wait gave up). Calls sharing a workspace must not overlap.
 * Rows are split into chunks of RLT_ATTEND_CHUNK (1024) positions (the
 * decoder's own cross-attention uses shorter chunks for models with few
 * (slot, head) pairs, so that few long rows still occupy every SM), each
 * chunk attended by one warp; the chunks of a row are merged in chunk order,
 * so a row's result does not depend on the other rows or on timing.
 * The call copies the per-row positions from pageable host memory on
 * `stream`, so it must not be made while `stream` is being captured into a
 * CUDA graph. Errors: INVALID_ARG, UNSUPPORTED (head_dim not
 * 16/32/64/128), CAPACITY (workspace too small). */
RLT_API int rlt_attend(const float *q, const void *kv, const int32_t *h_lengths, int n,
                       int n_heads, int head_dim, int cap, int dtype, void *out,
                       void *workspace, size_t workspace_bytes, rlt_stream stream);

/* Scratch bytes compiled into the library for rlt_attend_noalloc (8 MiB). */
#define RLT_ATTEND_NOALLOC_BYTES (8u << 20)

/* rlt_attend for callers that cannot allocate device memory (no counterpart
 * in the paper: a deployment convenience). Same arguments, layouts and
 * results as rlt_attend, minus the workspace: the scratch lives in a
 * file-scope device array of RLT_ATTEND_NOALLOC_BYTES that every GPU loading
 * the library holds until exit. Allocates nothing (no cudaMalloc / cudaFree).
 *   - Returns RLT_ERR_CAPACITY when rlt_attend_workspace_bytes(n, n_heads,
 *     head_dim, cap) exceeds RLT_ATTEND_NOALLOC_BYTES.
 *   - The first call on a device (with that device current) looks up the
 *     array's device address once; make that first call before any stream
 *     capture.
 *   - All calls on a device share its one array; each call clears what must
 *     start at zero, but calls that overlap on the GPU (for example on two
 *     streams) race on the array: serialise them.
 *   - Like rlt_attend, it must not be called while `stream` is being
 *     captured into a CUDA graph.
 *   - The device error word of rlt_attend is not reported. If a bounded
 *     device wait gives up (RLT_ERR_TIMEOUT in rlt_attend's error word), the
 *     call still returns RLT_OK and the contents of `out` are unspecified. */
RLT_API int rlt_attend_noalloc(const float *q, const void *kv, const int32_t *h_lengths, int n,
                               int n_heads, int head_dim, int cap, int dtype, void *out,
                               rlt_stream stream);

/* Kernel classes reported by rlt_get_stats. */
enum {
  RLT_K_XATTN = 0, /* decoder cross-attention over M<=t (split-KV + merge) */
  RLT_K_SWA = 1,   /* decoder sliding-window self-attention over the ring */
  RLT_K_GEMM = 2,  /* decoder projections / FFN / gate GEMMs */
  RLT_K_OTHER = 3, /* decoder norms, rotary/ring writes, gather, final norm */
  RLT_K_ENC = 4,   /* every encoder prefill kernel */
  RLT_K_STEP = 5,  /* the persistent decoder-step kernel (a whole step, one launch) */
  RLT_K_COUNT = 6
};

typedef struct rlt_stats {
  int64_t launches;                    /* kernels enqueued since rlt_create */
  int64_t kernel_launches[RLT_K_COUNT]; /* profiled launches per class */
  double kernel_ms[RLT_K_COUNT];       /* summed CUDA-event time per class */
  double kernel_bytes[RLT_K_COUNT];    /* algorithmic HBM bytes of those launches */
  double kernel_flops[RLT_K_COUNT];    /* algorithmic FLOPs of those launches */
} rlt_stats;

/* Measurement hook (no counterpart in the method). enable = k > 0: every
 * k-th decoder step (and every encoder prefill) runs with each kernel launch
 * bracketed by a pair of CUDA events on its own stream and attributed to a
 * class with the bytes/FLOPs the algorithm must move for it (weights once per
 * launch; K/V rows actually attended; activations). The other steps replay
 * unprofiled. enable = 0 turns it off. Either call clears the per-class sums
 * (the launch counter keeps running). Synchronises the model's last stream. */
RLT_API int rlt_profile(rlt_model *model, int enable);

/* Synchronises the model's last stream, folds every completed event pair
 * into the per-class sums and copies the counters into *out. */
RLT_API int rlt_get_stats(rlt_model *model, rlt_stats *out);

/* Faults rlt_set_fault can plant (failure detection, tested without
 * faulting the GPU). */
enum {
  RLT_FAULT_NONE = 0,
  /* the decoder attention's producer fills no stage: every consumer's
   * bounded wait runs out, records RLT_ERR_TIMEOUT and the kernel returns */
  RLT_FAULT_SKIP_ATTN_PRODUCER = 1
};

/* Failure-detection hook (no counterpart in the method). Synchronises the
 * model's last stream, then makes every later decoder-attention launch of
 * this model run with `fault` planted and its bounded device waits limited
 * to wait_limit_ns of device time (0 = the default bound, 2 s). The
 * attention output of a faulted step is unspecified; rlt_poll_device_error
 * reports RLT_ERR_TIMEOUT. Captured step graphs read the controls at run
 * time. Errors: INVALID_ARG (unknown fault, negative limit), CUDA. */
RLT_API int rlt_set_fault(rlt_model *model, int fault, int64_t wait_limit_ns);

/* Synchronises the model's last stream and returns the first device-side
 * error recorded since the previous poll (RLT_OK if none), then clears it. */
RLT_API int rlt_poll_device_error(rlt_model *model);

/* Static description of a status code (never NULL). */
RLT_API const char *rlt_status_string(int status);

/* Host only. The first CUDA error the calling thread met inside the library
 * since the previous call (after an RLT_ERR_CUDA): returns its cudaError_t
 * value (0 if none) and writes its name and the library source line that saw
 * it into buf (len bytes, may be NULL). Reading it clears it. */
RLT_API int rlt_last_cuda_error(char *buf, size_t len);

#ifdef __cplusplus
}
#endif
#endif /* RLT_H */
