// internal.h -- launchers of librlt's kernels (host side, not exported).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "bptt_core.h"
#include "common.cuh"
#include "epilogue.cuh"

namespace rlt {

constexpr int kSmCount = 148;  // B200 streaming multiprocessors

// Host-side count of kernel launches issued by the library (every launcher
// calls note_launch once per <<<>>>).
void note_launch();
int64_t launch_count();

// Launches a kernel with programmatic stream serialisation (see
// griddep_wait in common.cuh) and counts it.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
  note_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

// ---------------------------------------------------------------- GEMMs
// C[n][m] = sum_k X[n][k] W[m][k] with a fused epilogue (epilogue.cuh).
// bf16 on tcgen05: M % 128 == 0, K % 64 == 0, ld* % 8 == 0, 16-byte aligned
// bases.  split_mode 1 (decode steps) splits K inside a thread-block cluster
// by a rule that depends only on M and K, exchanging the fp32 partials
// through `ws` (gemm_tc_workspace_floats; the caller keeps it private to the
// stream); split_mode 0 (token-parallel encoder) never splits and needs none.
cudaError_t gemm_tc(const bf16* W, int64_t ldw, const bf16* X, int64_t ldx, int M, int N, int K, int epi,
                    const EpiParams& ep, int split_mode, float* ws, size_t ws_floats, cudaStream_t st);
// Exchange area (floats) a split_mode launch of this shape needs (0 when it
// is not split over a cluster).
size_t gemm_tc_workspace_floats(int M, int N, int K, int split_mode);
int gemm_tc_cluster(int M, int K, int split_mode);
int gemm_tc_bn(int M, int N, int K, int split_mode);

// CUDA-core GEMM (fp32 models; also a cross-check for the tensor-core path).
template <typename WT, typename XT>
cudaError_t gemm_simt(const WT* W, int64_t ldw, const XT* X, int64_t ldx, int M, int N, int K, int epi,
                      const EpiParams& ep, cudaStream_t st);

// ---------------------------------------------------------------- attention
// SWA decode attention of one decoder layer (eq. 2.14) over the ring of
// retained entries plus the current key/value, then the ring insert; at
// position t, or at each sequence's own position when sp is on.
template <typename KT>
cudaError_t swa_attn(const float* qkv, int64_t ld_qkv, KT* ring_k, KT* ring_v, int B, int H, int hd, int t,
                     const SeqPos& sp, int W, const float* rope_cs, KT* out, int64_t ld_out, cudaStream_t st);

// Decode attention of one query per (sequence, head) over key/value rows
// 0..n-1 of a [B][H][ld_t][hd] cache; the query is rotated at position
// qpos (0-based) first unless rope_cs is null.  With sp on, sequence b reads
// its own sp.n_keys(b) rows (query at n_keys - 1) and n only bounds them.
// Split over fixed chunks of keys when n is large; the chunk partials go to
// `ws` (prefix_attn_workspace_floats).  With `counters` (B*H ints, zero
// between launches) the last chunk block of each (sequence, head) combines
// them; without, a second kernel does.
template <typename KT>
cudaError_t prefix_attn(const float* q, int64_t ld_q, const KT* k, const KT* v, int64_t ld_t, int B, int H, int hd,
                        int n, int qpos, const SeqPos& sp, const float* rope_cs, KT* out, int64_t ld_out, float* ws,
                        size_t ws_floats, int* counters, cudaStream_t st);
size_t prefix_attn_workspace_floats(int B, int H, int hd, int n);
constexpr int kPrefixChunk = 256;

// Token-parallel causal attention for the encoder (eq. 2.1): query rows
// 0..T-1 of Q ([B][H][ld_tq][hd]) are positions q_off..q_off+T-1 and attend
// to key/value rows 0..q_off+i of K, V ([B][H][ld_tkv][hd]); out row b*T+i,
// columns h*hd.  q_off > 0 continues an encoded prefix held in the cache.
template <typename KT>
cudaError_t causal_attn(const KT* q, const KT* k, const KT* v, int64_t ld_tq, int64_t ld_tkv, int B, int H, int hd,
                        int T, int q_off, KT* out, int64_t ld_out, cudaStream_t st);

// The same on the tensor cores (bf16, hd 64 or 128): two-pass softmax with
// S and O in tensor memory.
cudaError_t causal_attn_tc(const bf16* q, const bf16* k, const bf16* v, int64_t ld_tq, int64_t ld_tkv, int B, int H,
                           int hd, int T, int q_off, bf16* out, int64_t ld_out, cudaStream_t st);

// ---------------------------------------------------------------- elementwise
// Generator fill of a [rows][cols] view (rows `pitch` elements apart).
template <typename WT>
cudaError_t init_normal(WT* dst, int64_t rows, int64_t cols, int64_t pitch, uint64_t seed, uint32_t stream_id,
                        float std, cudaStream_t st);
template <typename WT>
cudaError_t init_const(WT* dst, int64_t rows, int64_t cols, int64_t pitch, float value, cudaStream_t st);

// e rows (RowMap) = Emb[tok]
template <typename WT>
cudaError_t embed(const int32_t* tok, int64_t n_rows, int tok_per_seq, int64_t tok_seq_stride, const WT* emb, int d,
                  int vocab, float* out, RowMap out_map, cudaStream_t st);

// out[r] = gamma * x[r] / sqrt(mean(x[r]^2) + eps), x fp32 rows via RowMap
template <typename WT, typename OT>
cudaError_t rmsnorm(const float* x, RowMap x_map, const WT* gamma, int64_t rows, int d, float eps, OT* out,
                    int64_t ld_out, cudaStream_t st);

// Merge operand: xb[b] = [e_t ; RMSNorm_s(s)] (kind 0) or [e_t ; s] (kind 1)
template <typename WT, typename OT>
cudaError_t merge_prep(const float* e, RowMap e_map, const float* s, const WT* gamma, int B, int d, float eps,
                       int kind, OT* out, cudaStream_t st);

// RL replay ratios over [B][n] log-probs: ratio = exp(logp - logmu) where
// mask != 0, else 1; seq_logratio[b] = sum over masked tokens of
// (logp - logmu).  Either output may be null.
cudaError_t replay_ratios(const float* logp, const float* logmu, const uint8_t* mask, int B, int n, float* ratio,
                          float* seq_logratio, cudaStream_t st);

// Scatter head-split rows into a [B][H][ld_t][hd] store: row i = r %
// rows_per_seq of a sequence goes to store row dst_row0 + i, rotated (rope
// != 0) at position pos0 + i.
template <typename XT, typename KT>
cudaError_t head_scatter(const XT* x, int64_t ld_x, int64_t col0, int64_t rows, int rows_per_seq, int pos0,
                         int dst_row0, int H, int hd, int rope, const float* rope_cs, KT* dst, int64_t ld_t,
                         cudaStream_t st);
// The encoder step's insert of one row per sequence at its own position:
// row b goes to store row t_b - 1 (rotated at t_b - 1) for the sequences
// whose transition encodes its token (sp.encodes(b)); the others are left.
template <typename XT, typename KT>
cudaError_t head_insert(const XT* x, int64_t ld_x, int64_t col0, int B, const SeqPos& sp, int H, int hd, int rope,
                        const float* rope_cs, KT* dst, int64_t ld_t, cudaStream_t st);

// et[b] = e[b][t_b - 1] ([B][max_len][d] -> [B][d]; idle sequences copy a
// row they hold), and its inverse for the sequences whose transition encoded
// their token.
cudaError_t erow_gather(const float* e, int max_len, int d, int B, const SeqPos& sp, float* et, cudaStream_t st);
cudaError_t erow_scatter(const float* et, int max_len, int d, int B, const SeqPos& sp, float* e, cudaStream_t st);

// Position bookkeeping after a transition (report §2.1): every active
// sequence b moves to n_dec = t_b (and n_enc = max(n_enc, t_b)).  In a
// masked phase, the idle sequences get back the recurrent output and the
// folded-norm operand saved by save_rows before the transition, so that a
// transition they took no part in leaves them unchanged.
cudaError_t advance_positions(int32_t* dec, int32_t* enc, const int32_t* lim, int B, int d, float* s,
                              const float* s_save, bf16* zb, const bf16* zb_save, float* ss, const float* ss_save,
                              int n_ss, cudaStream_t st);
cudaError_t save_rows(const float* s, float* s_save, const bf16* zb, bf16* zb_save, const float* ss, float* ss_save,
                      int B, int d, int n_ss, cudaStream_t st);
// n[b] = value for b in [b0, b1)
cudaError_t set_positions(int32_t* n, int b0, int b1, int32_t value, cudaStream_t st);

// logp[b*ld_logp] = logits[b][next[b*next_stride]] - logsumexp(logits[b]);
// with `lim`, only for the sequences whose (advanced) dec[b] < lim[b], i.e.
// whose masked phase has a next token left.
cudaError_t logp_gather(const float* logits, int B, int V, const int32_t* next, int64_t next_stride, float* logp,
                        int64_t ld_logp, const int32_t* dec, const int32_t* lim, cudaStream_t st);

// Top-k / temperature behaviour sampler (report §5.3); the Philox counter's
// position is t, or t_rows[b] per sequence when t_rows is not null.
cudaError_t sample_topk(const float* logits, int B, int V, float temperature, int top_k, uint64_t seed, uint32_t t,
                        const int32_t* t_rows, int32_t* token, float* logp_tok, float* logmu, cudaStream_t st);

cudaError_t copy_f32(float* dst, const float* src, int64_t n, cudaStream_t st);

// Failure-detection probe: one bounded mbarrier wait that can never complete
// runs out after limit_ns and raises the device error word; synchronises
// `st` and returns how long the wait lasted.
cudaError_t bounded_wait_probe(uint64_t limit_ns, uint64_t* waited_ns, cudaStream_t st);

// dst[b][:] = src[:] (fp32) for b < B
template <typename WT>
cudaError_t broadcast_row(const WT* src, int d, float* dst, int B, cudaStream_t st);

// ---------------------------------------------------------------- gradients
namespace bptt {
// dst [rows][cols] fp32 = src (dtype 0 fp32, 1 bf16; rows `pitch` elements apart)
cudaError_t widen_to_f32(const void* src, int dtype, int64_t rows, int64_t cols, int64_t pitch, float* dst,
                         cudaStream_t st);
// Full-BPTT gradient of the weighted replay loss (bptt_core.h) on fp32
// weights W32 into G32 (per catalogue index; null where a tensor is absent),
// held for repeated calls of one size: the runner owns the engine's buffers,
// staging copies of the inputs, its own stream and, from its second pass on,
// a CUDA graph of the whole pass (prologue included) that later passes
// replay.  The W32 and G32 arrays and the buffers they point to must outlive
// the runner.  tensor_cores: run the contractions whose shapes allow it on
// tcgen05 with bf16 operands (bf16 models).
struct Runner;
cudaError_t runner_create(const Dims& D, int seg, bool tensor_cores, const float* const* W32, float* const* G32,
                          Runner** out);
// One pass: waits for `st`, copies tok [B][S] and wts [B][S-1] to staging,
// runs prologue(stream) (it fills W32) and the engine on the runner's
// stream, copies the log-probs to logp (may be null), and makes `st` wait for
// the pass.  Does not block the host.
cudaError_t runner_run(Runner* r, cudaError_t (*prologue)(void* ctx, cudaStream_t s), void* ctx, const int32_t* tok,
                       const float* wts, float* logp, cudaStream_t st);
// Drains the runner's stream and frees everything it holds.
void runner_free(Runner* r);
}  // namespace bptt

}  // namespace rlt
