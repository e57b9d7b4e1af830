/*
 * rlt.h -- C ABI of librlt.so, the B200 (sm_100a) implementation of the
 * Recurrent Looped Transformer (RLT) hot path: the batched recurrent decoder
 * state transition, the token-parallel causal encoder and the encoder KV
 * memory that feeds it.
 *
 * Definitions follow "Recurrent Looped Transformer" (Y. Zhang, technical
 * report, Sept. 2026) and its project page:
 *   §2.1      sequence, state H_t = (s_t, C^D_t), window W includes the current
 *             token, at most W-1 retained positions per layer
 *   §2.2      eq. 2.1 causal encoder, eq. 2.2 memory groups (G = 1 or L_D)
 *   §2.3      eqs. 2.3-2.7 H_0 = (s_*, empty), Merge, D_phi, readout
 *   §2.4      eq. 2.8 encoder step form, prefix-restricted memory
 *   §2.5      eqs. 2.9-2.11 gated merge, eqs. 2.12-2.16 decoder block
 *   §2.6      tied configuration
 *   §5.3      behaviour log-probabilities under the actual sampler
 *   App. A    execution schedules (A.1 prefill, A.2 generation, A.4 replay)
 * Readings where the pages leave a step open: FFN = SwiGLU; rotate-half RoPE
 * (base rope_base) at position p = t-1 on every query and key; one pre-norm
 * RMSNorm per sublayer; multi-head attention scaled by 1/sqrt(d/n_heads); no
 * final encoder norm; BOS id bos_id.
 *
 * Conventions for every entry point
 *  - Every function returns an int32 status: RLT_OK (0) or a negative code.
 *    Nothing throws across the ABI.  rlt_last_error() returns the text of the
 *    calling thread's last error.
 *  - Arguments and capacities are validated synchronously before any work is
 *    enqueued; a rejected call leaves model and state unchanged.
 *  - "_dev" pointers are device pointers owned by the caller, ordered on the
 *    CUDA stream passed as `stream` (a cudaStream_t; NULL = legacy default
 *    stream).  Host pointers are read/written synchronously.
 *  - The library owns all model and state device memory.  Kernel errors are
 *    asynchronous: they surface as RLT_E_CUDA on a later call.
 *  - A state remembers the model version it was built under.  Loading weights
 *    bumps the version; using an older state then fails with RLT_E_STALE
 *    (report §5.4 and App. C: caches built under other weights are invalid).
 *  - Every sequence of a state has its own positions n_enc[b] and n_dec[b]
 *    (report §4.1: the batch gathers ready transitions of independent
 *    sequences, each with its own memory, cache, s and position).  A
 *    transition advances every sequence of the batch by one, each at its own
 *    position; rlt_append_spans appends spans of different lengths and lets
 *    each sequence sit out the transitions its span does not need.
 *  - A model and its states are used from one host thread at a time: calls
 *    on one model, or on its states, must not overlap across threads (the
 *    model holds the state of rlt_replay_logprobs and the profiling record).
 *    Different models may be used from different threads.
 */
#ifndef RLT_H_
#define RLT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define RLT_OK 0
#define RLT_E_INVAL (-1)       /* bad argument or unsupported shape */
#define RLT_E_CAPACITY (-2)    /* position would pass max_len, or batch > capacity */
#define RLT_E_OOM (-3)         /* device allocation failed */
#define RLT_E_CUDA (-4)        /* a CUDA call or kernel failed */
#define RLT_E_STALE (-5)       /* state built under older weights */
#define RLT_E_STATE (-6)       /* call not valid in the state's current phase */

#define RLT_MERGE_PAPER 0      /* eqs. 2.9-2.11: u = e + alpha g*(W_s r), g = sig(W_g[e;r]+b_g), r = RMSNorm_s(s) */
#define RLT_MERGE_CONVEX 1     /* u = g*e + (1-g)*s, g = sig(W_g[e;s]) */

#define RLT_DTYPE_F32 0        /* fp32 weights, caches and arithmetic */
#define RLT_DTYPE_BF16 1       /* bf16 weights/caches/GEMM inputs, fp32 accumulation and residual stream */

typedef struct rlt_config {
  int32_t d_model;     /* residual width d */
  int32_t n_heads;     /* heads; head size d/n_heads is 16, 32, 64 or 128 */
  int32_t n_layers;    /* L_E = L_D = L */
  int32_t window;      /* SWA window W >= 1, includes the current token */
  int32_t groups;      /* memory groups G: 1 (shared) or n_layers (per layer) */
  int32_t ffn;         /* SwiGLU hidden width F */
  int32_t vocab;       /* V */
  int32_t tied;        /* 1: decoder SWA/FFN reuse encoder layer weights (§2.6); 0: untied */
  int32_t merge_kind;  /* RLT_MERGE_* */
  int32_t dtype;       /* RLT_DTYPE_* */
  float alpha;         /* feedback scale of eq. 2.11 */
  float rms_eps;       /* epsilon inside every RMSNorm */
  float rope_base;     /* rotary base */
  float init_std;      /* std of random initialisation */
  int32_t bos_id;      /* token id of BOS */
} rlt_config;

typedef struct rlt_model rlt_model;
typedef struct rlt_state rlt_state;

/* Behaviour sampler (report §5.3): the top_k largest raw logits, ordered by
 * (value desc, id asc), tempered by 1/temperature and renormalised; the
 * uniform is (Philox4x32-10(counter = (t, b, 0, 0), key = seed).x0 >> 8) *
 * 2^-24 where t is the position of the state s_t that predicts the token and
 * b the sequence's batch index.  1 <= top_k <= 256, temperature > 0. */
typedef struct rlt_sampling {
  float temperature;
  int32_t top_k;
  uint64_t seed;
} rlt_sampling;

/* Outputs of one readout.  Every pointer is a caller-owned device array or
 * NULL (not wanted). */
typedef struct rlt_readout_out {
  float* logp;          /* [B] log p(next[b] | x_1..t), needs next_dev */
  int32_t* sampled;     /* [B] sampled x_{t+1}, needs a sampler */
  float* logp_sampled;  /* [B] raw log p of the sampled token */
  float* logmu;         /* [B] behaviour log-prob of the sampled token (tempered, truncated) */
  float* logits;        /* [B, V] raw logits */
} rlt_readout_out;

/* State inspection (test hooks, report §6 snapshot contents).  The position
 * fields are those of the furthest sequence; rlt_state_positions gives every
 * sequence's own. */
typedef struct rlt_state_info {
  int32_t batch, max_len;
  int32_t n_enc;        /* tokens encoded: e_1..e_n_enc and M_<=n_enc exist (maximum over sequences) */
  int32_t n_dec;        /* decoder transitions applied: the state is H_n_dec (maximum over sequences) */
  int32_t ring_valid;   /* retained SWA entries per layer: min(n_dec, W-1) */
  int32_t ring_head;    /* slot the next transition writes: n_dec mod (W-1), 0 if W = 1 */
  int32_t has_encoder_cache;
  uint64_t model_version;
  int32_t has_pending;  /* a sampled x_{t+1} awaits its transition (App. A, pending token) */
  int32_t uniform;      /* 1: every sequence stands at the same n_enc and n_dec */
} rlt_state_info;

#define RLT_STATE_ENCODER_CACHE 1   /* keep C^E (needed for incremental encoding, eq. 2.8) */
#define RLT_STATE_GRAPHS 2          /* replay rlt_decoder_step's kernels as CUDA graphs, one per step shape */

/* what for rlt_state_read: */
#define RLT_READ_S 0        /* [B][d] fp32 recurrent output s_t */
#define RLT_READ_E 1        /* [B][max_len][d] fp32 encoder outputs */
#define RLT_READ_RING_K 2   /* layer `index`: [B][H][W-1][hd] keys (model dtype), slot of position j = (j-1) mod (W-1) */
#define RLT_READ_RING_V 3   /* layer `index`: values, same layout */
#define RLT_READ_MEM_K 4    /* group `index`: [B][H][max_len][hd] memory keys (rotated) */
#define RLT_READ_MEM_V 5    /* group `index`: memory values */
#define RLT_READ_ENC_K 6    /* layer `index`: [B][H][max_len][hd] encoder cache keys (needs the encoder cache) */
#define RLT_READ_ENC_V 7

/* ---------------------------------------------------------------- model */

/* Allocates a model on the current device and fills every weight from the
 * counter-based generator: element i of the tensor with stream id s is
 * init_std * (sum of the twelve 32-bit words of Philox4x32-10 with counters
 * (i_lo, i_hi, s, j), j = 0..2, key = seed, times 2^-32, minus 6), rounded to
 * fp32 and then (bf16 models) to bf16 by round-to-nearest-even.  Gains are 1
 * and b_gate is 0.  Tensor names, shapes and stream ids: see rlt_tensor_info.
 * Errors: RLT_E_INVAL (config), RLT_E_OOM, RLT_E_CUDA. */
int32_t rlt_init_weights(const rlt_config* cfg, uint64_t seed, rlt_model** out);

/* Copies a whole tensor from host memory in the model's storage format (fp32,
 * or bf16 bit patterns) and bumps the model version.  bytes must equal
 * rows*cols*element size.  Waits for the device first, so work enqueued
 * before the call (on any stream) reads the old values.  Errors:
 * RLT_E_INVAL (unknown name, size), RLT_E_CUDA. */
int32_t rlt_load_weights(rlt_model* m, const char* name, const void* host, size_t bytes);

/* Copies a whole tensor to host memory (storage format). */
int32_t rlt_get_weights(const rlt_model* m, const char* name, void* host, size_t bytes);

/* Shape and generator stream id of a tensor: names are emb [V,d], s_star [d],
 * g_mem [d], g_merge [d], w_gate [d,2d], b_gate [d], w_state [d,d], g_out [d],
 * w_out [V,d], wk_mem.g / wv_mem.g [d,d], and per layer l: wq.l wk.l wv.l
 * wo.l [d,d], w1.l w3.l [F,d], w2.l [d,F], g_ea.l g_ef.l g_dsa.l g_dmem.l
 * g_dffn.l [d], wq_mem.l wo_mem.l [d,d], and when untied dwq.l dwk.l dwv.l
 * dwo.l dw1.l dw2.l dw3.l.  Stream ids: emb 0, s_star 1, g_mem 2, g_merge 3,
 * w_gate 4, b_gate 5, w_state 6, g_out 7, w_out 8, wk_mem.g 16+2g,
 * wv_mem.g 17+2g, layer slot k of layer l 1024+32l+k in the order listed. */
int32_t rlt_tensor_info(const rlt_model* m, const char* name, int64_t* rows, int64_t* cols, int32_t* stream_id);

/* Frees the model's device memory, after a device synchronisation.  Every
 * state made by rlt_state_create on it must be freed first; otherwise the
 * call frees nothing and returns RLT_E_STATE. */
int32_t rlt_model_free(rlt_model* m);

/* ---------------------------------------------------------------- state */

/* Creates the state of `batch` independent sequences of up to max_len tokens,
 * at H_0 = (s_*, empty) with empty encoder caches (eq. 2.3).  Device memory:
 * encoder outputs [B][max_len][d] fp32, memory 2*G*B*max_len*d elements, SWA
 * ring 2*L*B*(W-1)*d elements, plus (flag RLT_STATE_ENCODER_CACHE) the encoder
 * cache 2*L*B*max_len*d elements, plus step workspace: the GEMM operands and
 * bf16 folded-norm operand of one step, the split-K exchange area of the
 * decode GEMMs (at most a few tens of MB), the attention chunk partials, the
 * logits [B][V] fp32 and the pending-token record.  The token-parallel
 * encoder adds its own workspace on first use (at most 4 GB).
 * Errors: RLT_E_INVAL, RLT_E_OOM. */
int32_t rlt_state_create(rlt_model* m, int32_t batch, int32_t max_len, int32_t flags, rlt_state** out);
int32_t rlt_state_free(rlt_state* s);

/* Returns the state to H_0 with empty caches (positions 0) under the model's
 * current weights. */
int32_t rlt_state_reset(rlt_state* s, void* stream);

int32_t rlt_state_info_get(const rlt_state* s, rlt_state_info* out);

/* Per-sequence positions (report §2.1, §4.1) into caller-owned host arrays
 * of `batch` entries, each of which may be NULL: n_enc[b], n_dec[b], the
 * retained SWA entries ring_valid[b] = min(n_dec[b], W-1) and the slot the
 * next transition of sequence b writes, ring_head[b] = n_dec[b] mod (W-1)
 * (0 if W = 1).  Errors: RLT_E_INVAL. */
int32_t rlt_state_positions(const rlt_state* s, int32_t* n_enc, int32_t* n_dec, int32_t* ring_valid,
                            int32_t* ring_head);

/* Copies one state component to host memory (synchronous); layouts above. */
int32_t rlt_state_read(const rlt_state* s, int32_t what, int32_t index, void* host, size_t bytes);

/* Exact prefix snapshot (report §6, "Multi-turn Serving and Cache
 * Semantics"): writes to host memory everything the continuation depends on
 * -- the encoder cache C^E (when the state keeps it) and the memory M for
 * positions 1..n_enc, the encoder outputs e_1..e_n_enc, the decoder state
 * H_t = (s_t, C^D_t) with the whole SWA ring, the positions n_enc and n_dec,
 * the pending sampled token (App. A) if any, the model configuration
 * (window convention included) and the identity of the weights (generator
 * seed and model version).  The header holds the furthest sequence's
 * positions and the rows up to them are stored for every sequence; when the
 * sequences stand at different positions a last section holds n_enc[B] and
 * n_dec[B] (int32).  bf16 models also store the readout operand the
 * last transition left (gamma_o * s_t in bf16 and its sums of squares), so
 * that a restored state reads out bit-identically.  Layout: a 120-byte
 * little-endian header ("RLTSNAP1") followed by the sections in that order.
 * *used receives the size; with host == NULL nothing is copied and the call
 * only reports the size.  Ordered on `stream`, and synchronises it.
 * Errors: RLT_E_CAPACITY (cap < size), RLT_E_INVAL. */
int32_t rlt_state_export(const rlt_state* s, void* host, size_t cap, size_t* used, void* stream);

/* Restores a snapshot into a state of the same batch size created under the
 * same model configuration, replacing its contents; max_len may differ as
 * long as it covers the snapshot's positions.  A state without the encoder
 * cache drops the snapshot's cache (it can then decode up to n_enc but not
 * encode further); a state with the cache needs a snapshot that has one.
 * Weight updates invalidate snapshots (report §6): the model's generator
 * seed and version must equal the snapshot's, else RLT_E_STALE.
 * Synchronises `stream` (host may be freed on return).
 * Errors: RLT_E_INVAL (format, configuration, batch, size), RLT_E_STALE,
 * RLT_E_CAPACITY (positions > max_len), RLT_E_STATE (cache missing). */
int32_t rlt_state_import(rlt_state* s, const void* host, size_t bytes, void* stream);

/* ---------------------------------------------------------------- schedules */

/* Token-parallel causal encoder (eq. 2.1) and memory projection (eq. 2.2) for
 * T tokens per sequence, tok_dev [B][T] int32 (row-major), placed at positions
 * n_enc+1..n_enc+T (every sequence must stand at the same n_enc, else
 * RLT_E_STATE: rlt_append_spans takes spans at different positions).  With n_enc > 0 the tokens attend to the encoded prefix
 * through the encoder cache: the chunked schedule of App. A.2 (an appended
 * span -- a user turn or a tool result -- is encoded in one pass; every
 * token still receives its decoder transition through rlt_decoder_step).
 * Does not advance the decoder.  Errors: RLT_E_CAPACITY (n_enc+T >
 * max_len), RLT_E_STATE (n_enc > 0 without the encoder cache), RLT_E_STALE,
 * RLT_E_INVAL. */
int32_t rlt_encode_prefix(rlt_model* m, rlt_state* s, const int32_t* tok_dev, int32_t T, void* stream);

/* Appends a span of lens[b] tokens to every sequence b (report §6 multi-turn
 * serving: a user turn or tool result; App. A.1 prefill when the state is
 * fresh): span b is tok_dev[b * ld_tok + 0 .. lens[b]-1] (int32, device),
 * lens is a host array of B entries >= 0 (0: the sequence takes no part).
 * Each span is encoded token-parallel over its sequence's cached prefix
 * (eq. 2.1, the chunked schedule of App. A.2; runs of consecutive sequences
 * with the same position and length share one pass), then every span token
 * receives its decoder transition: max(lens) transitions in lock step, in
 * which sequence b takes part only while its span lasts (its state is
 * otherwise left unchanged).  If logp_dev != NULL, logp_dev[b * ld_logp + i]
 * receives log p(span_b[i+1] | history) for i = 0..lens[b]-2 (other entries
 * are not written).  Afterwards n_enc[b] = n_dec[b] = old + lens[b].
 * Requires every encoded token to be consumed (n_enc[b] = n_dec[b]) and no
 * pending sampled token; a non-empty span after an encoded prefix needs the
 * encoder cache.  Copies lens to the device with an ordinary host copy, so
 * the call waits for `stream` once.  Errors: RLT_E_INVAL, RLT_E_CAPACITY
 * (n_enc[b] + lens[b] > max_len), RLT_E_STATE, RLT_E_STALE. */
int32_t rlt_append_spans(rlt_model* m, rlt_state* s, const int32_t* tok_dev, int64_t ld_tok, const int32_t* lens,
                         float* logp_dev, int64_t ld_logp, void* stream);

/* Readout of the current s_t (eq. 2.6): log p of next_dev [B] (may be NULL),
 * and/or a sample from the behaviour sampler (samp may be NULL; its counter
 * position t is each sequence's own n_dec).  A sample is also recorded in
 * the state as the pending token x_{t+1} (App. A): the state represents the
 * consumed prefix only, and the next rlt_decoder_step consumes the pending
 * token when it is given no tokens.  Requires n_dec[b] >= 1 for every
 * sequence. */
int32_t rlt_readout(rlt_model* m, rlt_state* s, const int32_t* next_dev, const rlt_sampling* samp,
                    const rlt_readout_out* out, void* stream);

/* Consumes x_t for every sequence b, at its own t = n_dec[b]+1 (App. A.2).
 * With RLT_STATE_GRAPHS the step's kernels (encoder step and transition,
 * not the readout) run as a CUDA graph: one graph per step shape (which
 * sequences run the encoder step, the token source, and the number of
 * 256-key attention chunks), captured the second time a shape occurs and
 * launched on a stream private to the state, ordered after `stream` by
 * events.  Results are bit-identical to plain launches; if a capture fails
 * the state falls back to plain launches for good.  Graphs are not used
 * while profiling is enabled.
 */
/* Consumes x_t for every sequence b, at its own t = n_dec[b]+1 (App. A.2):
 * for the sequences whose x_t is not yet encoded (n_enc[b] < t), runs the
 * encoder step (eq. 2.8, needs the encoder cache) and the memory append;
 * then the merge and the L_D decoder blocks
 * (eqs. 2.4, 2.5, 2.12-2.16) with one SWA insert per layer; then the readout
 * as rlt_readout does (skipped when next_dev, samp and out are all NULL).
 * tok_dev [B] int32 is read only when the token is encoded here; NULL takes
 * the pending sampled token.  Every transition clears the pending record.
 * Errors: RLT_E_CAPACITY (t > max_len), RLT_E_STATE (no encoder cache and x_t
 * not encoded, or no token given and none pending), RLT_E_STALE,
 * RLT_E_INVAL. */
int32_t rlt_decoder_step(rlt_model* m, rlt_state* s, const int32_t* tok_dev, const int32_t* next_dev,
                         const rlt_sampling* samp, const rlt_readout_out* out, void* stream);

/* Prompt prefill (App. A.1): rlt_encode_prefix over tok_dev [B][T], then T
 * decoder transitions.  If logp_dev != NULL it receives [B][T-1] teacher
 * log-probs log p(x_{t+1} | x_1..t), t = 1..T-1.  The state ends at H_T; call
 * rlt_readout to sample the first response token. */
int32_t rlt_prefill(rlt_model* m, rlt_state* s, const int32_t* tok_dev, int32_t T, float* logp_dev, void* stream);

/* Current-policy replay (App. A.4): from a fresh H_0 under the current
 * weights, encode tok_dev [B][S] token-parallel, run the S-1 transitions and
 * write logp_dev [B][S-1] = log p(x_{t+1} | x_1..t).  Uses a state the model
 * keeps for replay (allocated on first use or growth).  S >= 2. */
int32_t rlt_replay_logprobs(rlt_model* m, const int32_t* tok_dev, int32_t B, int32_t S, float* logp_dev,
                            void* stream);

/* RL replay with importance ratios (report §5.3, eq. 5.5, and App. A.4):
 * rlt_replay_logprobs under the current weights, then for every scored
 * token t = 1..S-1 (row-major [B][S-1], the same indexing as logp_dev)
 *   ratio_dev[b][t]      = exp(logp - logmu_dev)  where action_mask_dev != 0,
 *                        = 1                      elsewhere (user/tool/prompt
 *                          tokens get no action factor, report §6),
 *   seq_logratio_dev[b]  = sum over action tokens of (logp - logmu_dev), the
 *                          log of the trajectory ratio prod_i r_i,
 * summed in double in a fixed order.  logmu_dev holds the behaviour
 * log-probabilities the sampler recorded (temperature, truncation and
 * renormalisation included, as rlt_readout's logmu); action_mask_dev is
 * uint8.  logp_dev [B][S-1] receives the current-policy log-probs.  Either
 * ratio output may be NULL (not both).  Errors: as rlt_replay_logprobs,
 * RLT_E_INVAL. */
int32_t rlt_replay_ratios(rlt_model* m, const int32_t* tok_dev, int32_t B, int32_t S, const float* logmu_dev,
                          const uint8_t* action_mask_dev, float* logp_dev, float* ratio_dev,
                          float* seq_logratio_dev, void* stream);

/* ---------------------------------------------------------------- gradients */

/* Full back-propagation through time of the replay (report §5.1-§5.4 and
 * App. C): for tok_dev [B][S] int32 and target weights w_dev [B][S-1] fp32,
 *   L_w = - sum_{b,t} w[b][t] log p(x_{b,t+1} | x_{b,1..t}),
 * and its gradient with respect to every stored tensor.  The gradient runs
 * through the causal encoder, the memory projections, the merge, every
 * decoder SWA key/value and the recurrent output over all positions.
 * Nothing is detached: evicting an entry from the SWA window is not a
 * stop-gradient.  The objectives of report §5 are choices of w: eq. 5.1
 * (1/(S-1) on every target), eq. 5.2 (the assistant mask over its count),
 * eq. 5.4 (R - b on the response targets, 0 on the prompt).
 * The decoder is reversed one step at a time in segments of `segment`
 * steps.  Each segment is recomputed from the recurrent output at its
 * start, with the same parameters (activation checkpointing, §4.3).  The
 * arithmetic is fp32 on fp32 copies of the weights.  Gradients are
 * accumulated into fp32 buffers the model owns, one per stored tensor, read
 * with rlt_grad_read and cleared with rlt_grad_zero.  logp_dev [B][S-1]
 * (may be NULL) receives the log-probs the pass computed.
 * Device memory, in fp32: about 4 * B * S * (L * (12d + 3F) + 4 G d + 13d +
 * 3F) bytes for the encoder activations, the decoder key/value history and
 * their adjoints, plus 4 * segment * B * (L * (11d + 3F) + 6d + V) bytes for
 * one segment's recomputed steps, plus the fp32 weight copies.  It is
 * allocated by the first call for a (B, S, segment) and kept by the model
 * for the next calls of the same sizes (another size frees it first;
 * rlt_backward_release and rlt_model_free free it).  The first call of a
 * size launches its kernels one by one; the second captures the whole pass
 * (weight copies included, so weights loaded between calls are used) as a
 * CUDA graph, which later calls replay.  A pass of more than 400,000 kernels
 * is never captured.  The work runs on a stream of the model's own, ordered
 * after the work already on `stream`, and `stream` waits for it; the call
 * returns once it is enqueued.  Head size at most 128.  The token ids are
 * copied to the host and checked against the vocabulary before any work is
 * enqueued (this waits for `stream`).  Errors: RLT_E_INVAL (arguments, a
 * token id out of range), RLT_E_OOM, RLT_E_CUDA (the kept buffers are freed
 * after an error). */
int32_t rlt_replay_backward(rlt_model* m, const int32_t* tok_dev, int32_t B, int32_t S, const float* w_dev,
                            int32_t segment, float* logp_dev, void* stream);

/* Frees the device memory and the graph rlt_replay_backward keeps between
 * calls (after the device has finished its work).  Errors: RLT_E_INVAL. */
int32_t rlt_backward_release(rlt_model* m);

/* Copies the accumulated fp32 gradient of a stored tensor (rlt_tensor_info
 * names and shapes, [rows][cols] row-major) to host.  Before any
 * rlt_replay_backward the gradient is zero.  Errors: RLT_E_INVAL (name or
 * size). */
int32_t rlt_grad_read(const rlt_model* m, const char* name, float* host, size_t bytes);

/* Sets every accumulated gradient of the model to zero. */
int32_t rlt_grad_zero(rlt_model* m, void* stream);

/* ---------------------------------------------------------------- ops */

/* Kernel-level check of the step's contraction: y_dev [N][M] fp32 =
 * x_dev [N][K] . w_dev [M][K]^T, both operands row-major in `dtype`
 * (RLT_DTYPE_BF16: bf16, RLT_DTYPE_F32: fp32).  use_tensor_cores = 1 runs the
 * tcgen05 kernel (bf16 only; M % 128 == 0, K % 64 == 0), 0 the CUDA-core
 * kernel.  Split-K workspace is allocated and freed inside the call.
 * Errors: RLT_E_INVAL (shape/dtype), RLT_E_OOM, RLT_E_CUDA. */
int32_t rlt_op_linear(const void* w_dev, const void* x_dev, float* y_dev, int32_t M, int32_t N, int32_t K,
                      int32_t dtype, int32_t use_tensor_cores, void* stream);

/* Kernel-level check of the decode attention of eq. 2.15 / eq. 2.8: for
 * every sequence b and head h, softmax over keys j < n of
 * (q_b,h . k_b,h,j) / sqrt(hd), weighting v_b,h,j.  q_dev [B][H*hd] fp32 (a
 * query row per sequence, heads concatenated); k_dev, v_dev [B][H][ld_t][hd]
 * in `dtype` (rows 0..n-1 are read); out_dev [B][H*hd] in `dtype`.  When
 * rope_cs_dev is not NULL the query is first rotated at position qpos with
 * the rotate-half map, using the table rope_cs_dev[p][i][0..1] =
 * (cos, sin)(p * base^(-2i/hd)) (fp32, rows 0..qpos).  Keys are taken as
 * given.  n > 256 splits the keys into 256-key chunks whose partial results
 * need scratch of B*H*ceil(n/256)*(hd+2) floats, allocated and freed inside
 * the call (the call synchronises the stream in that case).
 * Errors: RLT_E_INVAL (shape/dtype), RLT_E_OOM, RLT_E_CUDA. */
int32_t rlt_op_prefix_attention(const float* q_dev, const void* k_dev, const void* v_dev, int64_t ld_t, int32_t B,
                                int32_t H, int32_t hd, int32_t n, int32_t dtype, const float* rope_cs_dev,
                                int32_t qpos, void* out_dev, void* stream);

/* The same attention as rlt_op_prefix_attention, for callers that cannot
 * allocate device memory: serving engines that reserve all of the GPU's
 * memory for their own pool up front, and latency-critical paths that cannot
 * afford the device-wide synchronisation that cudaMalloc/cudaFree imply.  It
 * calls no allocating routine.  The chunk partials of the split-key attention
 * go to a scratch array of at most 16 MiB (4,194,304 floats) that the library
 * places in device memory as a static array; every GPU that loads the library
 * holds it until the process exits.  A call needs B*H*ceil(n/256)*(hd+2)
 * floats of it (none when n <= 256); larger calls are rejected with
 * RLT_E_CAPACITY and nothing is launched.  The first call on a device looks
 * up the array's device address (once per device, with that device current);
 * make that first call before any stream capture.  All calls share the one
 * array and it keeps the last call's contents; nothing in it needs to start
 * at zero, since every partial a call reads is written earlier in that call.
 * Calls that overlap on the GPU (other streams, other threads) race on the
 * array: order them.  The report has no counterpart to this entry point; it
 * exists for the callers above.
 * Errors: RLT_E_INVAL, RLT_E_CAPACITY, RLT_E_CUDA. */
int32_t rlt_op_prefix_attention_noalloc(const float* q_dev, const void* k_dev, const void* v_dev, int64_t ld_t,
                                        int32_t B, int32_t H, int32_t hd, int32_t n, int32_t dtype,
                                        const float* rope_cs_dev, int32_t qpos, void* out_dev, void* stream);

/* Behaviour sampler (see rlt_sampling) on caller-given logits_dev [B][V]
 * fp32, as position t: writes token_dev [B] int32, logp_dev [B] (raw
 * log-softmax of the token, may be NULL) and logmu_dev [B] (tempered and
 * truncated log-prob, may be NULL).  Errors: RLT_E_INVAL. */
int32_t rlt_op_sample(const float* logits_dev, int32_t B, int32_t V, const rlt_sampling* samp, uint32_t t,
                      int32_t* token_dev, float* logp_dev, float* logmu_dev, void* stream);

/* ---------------------------------------------------------------- misc */

/* Copies the calling thread's last error text (NUL-terminated, truncated to
 * n) and returns its status code. */
int32_t rlt_last_error(char* buf, size_t n);

/* Checks the device-side error word that bounded waits inside the kernels
 * set when a wait runs out (never expected); returns RLT_E_CUDA and clears it
 * if set.  Synchronises the device. */
int32_t rlt_check_device(void);

/* Kernel timing hook for measurement: when enabled, the library records CUDA
 * events on the launching stream around the decode-attention launches of
 * every 4th position (t = 0 mod 4), and wraps the token-parallel encoder and
 * the transitions with t = 64 (mod 128) in an NVTX range "rlt_sample" (a
 * stratified sample a kernel profiler can select).  Enabling (or disabling)
 * clears the record.  rlt_profile_read
 * synchronises the device and, for kind 0 (prefix attention: cross-attention
 * to the memory and the encoder step) or kind 1 (SWA attention), returns the
 * summed event intervals in milliseconds, the launch count and the
 * algorithmic KV bytes those launches read and wrote (keys and values of
 * every attended position, plus the SWA insert). */
int32_t rlt_profile_enable(rlt_model* m, int32_t on);

/* Test hook of the failure detection above (the report has no counterpart):
 * launches one block whose thread waits, through the same bounded mbarrier
 * wait the tensor-core kernels use, on a barrier that no thread ever arrives
 * at, with a limit of limit_us microseconds (1..1000000) instead of the
 * kernels' 2 s.  The wait runs out, the kernel returns and the device error
 * word is set: the next rlt_check_device() reports RLT_E_CUDA ("a bounded
 * device wait ran out") and clears it; the context stays usable.
 * Synchronises `stream`; *waited_ns receives how long the wait lasted.
 * Errors: RLT_E_INVAL, RLT_E_CUDA. */
int32_t rlt_test_bounded_wait(uint32_t limit_us, uint64_t* waited_ns, void* stream);

/* Number of kernel launches the library has issued since it was loaded
 * (host-side counter, all devices and threads). */
int32_t rlt_kernel_launches(int64_t* count);
int32_t rlt_profile_read(rlt_model* m, int32_t kind, double* ms, int64_t* launches, double* bytes);

#ifdef __cplusplus
}
#endif
#endif /* RLT_H_ */
