// rlt_api.cu -- host engine and C ABI of librlt (include/rlt.h).
//
// Owns model weights and per-batch state in device memory and schedules the
// kernels of one lock-step transition for B independent sequences
// ("Recurrent Looped Transformer" §4.1: ready decoder transitions of
// independent sequences are batched).  Schedules follow App. A: encoder
// prefill (A.1, eq. 2.1), incremental generation (A.2, eq. 2.8), replay
// (A.4).
//
// Weight storage.  Every tensor is kept in the model dtype.  Matrices that
// feed one contraction are stored together so one GEMM covers them:
//   wq/wk/wv of a layer  -> rows [0,d), [d,2d), [2d,3d) of a [3d][d] block
//   w1/w3 of a layer     -> interleaved rows of a [2F][d] block (row 2i = w1
//                           row i, row 2i+1 = w3 row i; SwiGLU pairs meet in
//                           adjacent accumulator lanes)
//   wk_mem.g/wv_mem.g    -> rows [2dg, 2dg+d) and [2dg+d, 2d(g+1)) of [2dG][d]
// The named tensors of rlt.h are views into these blocks.
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <algorithm>
#include <cmath>
#include <type_traits>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <set>
#include <string>
#include <tuple>
#include <vector>

#include "internal.h"
#include "rlt.h"

using namespace rlt;

// ------------------------------------------------------------------ errors
namespace {
thread_local std::string t_err = "";
thread_local int32_t t_err_code = RLT_OK;

int32_t fail(int32_t code, const std::string& msg) {
  t_err = msg;
  t_err_code = code;
  return code;
}
int32_t ok() { return RLT_OK; }
}  // namespace

#define RLT_CUDA(...)                                                                                          \
  do {                                                                                                         \
    cudaError_t e_ = (__VA_ARGS__);                                                                            \
    if (e_ != cudaSuccess) return fail(RLT_E_CUDA, std::string(#__VA_ARGS__) + ": " + cudaGetErrorString(e_)); \
  } while (0)
#define RLT_TRY(...)                 \
  do {                               \
    int32_t r_ = (__VA_ARGS__);      \
    if (r_ != RLT_OK) return r_;     \
  } while (0)

// ------------------------------------------------------------------ model
struct View {
  void* base;       // first element
  int64_t rows, cols, pitch;  // pitch in elements between logical rows
  int32_t sid;      // generator stream id
  int32_t kind;     // 0 random, 1 ones, 2 zeros
};

struct LayerW {
  void* qkv;   // [3d][d]
  void* wo;    // [d][d]
  void* w13;   // [2F][d] interleaved
  void* w2;    // [d][F]
  void* wq_mem;
  void* wo_mem;
  void* g_ea; void* g_ef; void* g_dsa; void* g_dmem; void* g_dffn;
  void* dqkv; void* dwo; void* dw13; void* dw2;  // decoder weights (== encoder ones when tied)
};

struct ProfileRec {
  bool on = false;
  bool sample_now = false;  // current transition is one of the sampled ones
  std::vector<cudaEvent_t> ev;
  size_t used = 0;
  double bytes[2] = {0, 0};
  int64_t launches[2] = {0, 0};
  std::vector<int> kind;  // per event pair
};

struct rlt_model {
  rlt_config cfg;
  uint64_t seed = 0;  // generator seed of rlt_init_weights (part of the weights' identity)
  int hd = 0;
  size_t esz = 0;
  int device = 0;
  uint64_t version = 1;
  std::vector<void*> allocs;
  void* emb = nullptr; void* s_star = nullptr; void* g_mem = nullptr; void* g_merge = nullptr;
  void* w_gate = nullptr; void* b_gate = nullptr; void* w_state = nullptr; void* g_out = nullptr;
  void* w_out = nullptr; void* w_kvm = nullptr;
  std::vector<LayerW> layers;
  std::map<std::string, View> views;
  float* rope_cs = nullptr;
  int rope_len = 0;
  rlt_state* replay = nullptr;  // model-owned state of rlt_replay_logprobs
  int64_t live_states = 0;      // states made by rlt_state_create and not yet freed
  std::vector<float*> grad;     // fp32 gradient per catalogue index of bptt_core.h (rlt_replay_backward)
  struct BackwardHold* bwd = nullptr;  // buffers of rlt_replay_backward, kept for calls of the same sizes
  ProfileRec prof;
};

// What rlt_replay_backward keeps between calls with the same (B, S, segment):
// fp32 copies of the weights (refilled by every pass) and the runner
// (engine buffers, staging inputs, its stream and its graph).
struct BackwardHold {
  int B = 0, S = 0, seg = 0, dtype = 0;
  std::vector<float*> w32;
  std::vector<const View*> views;
  std::vector<void*> allocs;
  bptt::Runner* runner = nullptr;
};

namespace {
void release_backward(rlt_model* m);
}  // namespace

struct rlt_state {
  rlt_model* m = nullptr;
  int32_t B = 0, max_len = 0, flags = 0;
  uint64_t version = 0;
  // Per-sequence positions (report §4.1: each sequence of a batch has its
  // own position): n_enc[b] tokens encoded, n_dec[b] transitions applied.
  // The host copies decide shapes and validate calls; the device copy `pos`
  // ([3][B]: n_enc, n_dec, lim) is what the kernels read and advance, so
  // no host-to-device copy is needed per transition.  lim is the end of a
  // masked phase (rlt_append_spans).
  std::vector<int32_t> enc_h, dec_h, lim_h;
  int32_t* pos = nullptr;
  std::vector<void*> allocs;
  float* e = nullptr;          // [B][max_len][d]
  float* et = nullptr;         // [B][d] encoder output of each sequence's position in flight
  float* s_save = nullptr;     // [B][d] masked phases: rows of idle sequences, restored after a transition
  void* zb_save = nullptr;     // [B][d] bf16
  float* ss_save = nullptr;    // [d/128][B]
  void* mem_k = nullptr; void* mem_v = nullptr;  // [G][B][H][max_len][hd]
  void* ce_k = nullptr; void* ce_v = nullptr;    // [L][B][H][max_len][hd]
  void* ring_k = nullptr; void* ring_v = nullptr;  // [L][B][H][W-1][hd]
  float* s = nullptr;          // [B][d]
  void* xb = nullptr;          // [B][2d] GEMM operand (model dtype)
  void* zb = nullptr;          // [B][d] bf16 gamma*z operand of the folded RMSNorm (bf16 models)
  float* ss = nullptr;         // [d/128][B] partial sums of z^2 for the folded RMSNorm
  float* qkv = nullptr;        // [B][max(3d, 2dG)]
  int64_t ld_qkv = 0;
  void* attn = nullptr;        // [B][d]
  void* hbuf = nullptr;        // [B][F]
  float* gate = nullptr;       // [B][d]
  float* logits = nullptr;     // [B][V]
  float* attn_ws = nullptr; size_t attn_ws_floats = 0;
  int* attn_cnt = nullptr;     // [B][H] chunk counters of the decode attention (zero between launches)
  float* gemm_ws = nullptr; size_t gemm_ws_floats = 0;  // split-K exchange of the decode GEMMs (bf16)
  int32_t* pending = nullptr;  // [B] last sampled x_{t+1}, not yet consumed (report App. A, pending token)
  bool has_pending = false;
  // CUDA-graph replay of decoder steps (flag RLT_STATE_GRAPHS): one
  // executable graph per step shape -- (encoder step: none / some / all
  // sequences, its token source, decode-attention chunks) -- captured the
  // second time the shape occurs and launched on a private stream that is
  // ordered after the caller's stream by events.  A failed capture turns
  // graphs off for the state (every step then launches its kernels).
  using GraphKey = std::tuple<int, const void*, int>;
  struct StepGraph {
    cudaGraphExec_t exec;
    int64_t kernels;
  };
  std::map<GraphKey, StepGraph> graphs;
  std::set<GraphKey> graph_seen;
  bool graph_ok = true;
  cudaStream_t gstream = nullptr;
  cudaEvent_t ev_in = nullptr, ev_out = nullptr;
  // encoder-prefill workspace, rows = sequences x tokens of one chunk
  int64_t pf_rows = 0;
  void* pf_x = nullptr; void* pf_big = nullptr; void* pf_q = nullptr; void* pf_k = nullptr; void* pf_v = nullptr;
  void* pf_attn = nullptr;
  int64_t pf_big_cols = 0;
};

namespace {

int32_t dev_alloc(std::vector<void*>& list, void** p, size_t bytes) {
  *p = nullptr;
  if (bytes == 0) return RLT_OK;
  cudaError_t e = cudaMalloc(p, bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    *p = nullptr;
    return fail(RLT_E_OOM, "cudaMalloc of " + std::to_string(bytes) + " bytes failed: " + cudaGetErrorString(e));
  }
  list.push_back(*p);
  return RLT_OK;
}

void free_all(std::vector<void*>& list) {
  for (void* p : list) cudaFree(p);
  list.clear();
}

char* off(void* base, int64_t elems, size_t esz) { return static_cast<char*>(base) + elems * (int64_t)esz; }

int32_t validate(const rlt_config* c) {
  if (!c) return fail(RLT_E_INVAL, "null config");
  if (c->d_model <= 0 || c->n_heads <= 0 || c->d_model % c->n_heads) return fail(RLT_E_INVAL, "d_model % n_heads != 0");
  const int hd = c->d_model / c->n_heads;
  if (!(hd == 16 || hd == 32 || hd == 64 || hd == 128)) return fail(RLT_E_INVAL, "head size must be 16, 32, 64 or 128");
  if (c->n_layers <= 0 || c->window < 1 || c->ffn <= 0 || c->vocab <= 1) return fail(RLT_E_INVAL, "bad sizes");
  if (!(c->groups == 1 || c->groups == c->n_layers)) return fail(RLT_E_INVAL, "groups must be 1 or n_layers");
  if (c->tied != 0 && c->tied != 1) return fail(RLT_E_INVAL, "tied must be 0 or 1");
  if (c->merge_kind != RLT_MERGE_PAPER && c->merge_kind != RLT_MERGE_CONVEX) return fail(RLT_E_INVAL, "merge_kind");
  if (c->dtype != RLT_DTYPE_F32 && c->dtype != RLT_DTYPE_BF16) return fail(RLT_E_INVAL, "dtype");
  if (c->bos_id < 0 || c->bos_id >= c->vocab) return fail(RLT_E_INVAL, "bos_id");
  if (!(c->rms_eps >= 0.f) || !(c->rope_base > 1.f) || !(c->init_std >= 0.f)) return fail(RLT_E_INVAL, "eps/base/std");
  if (c->dtype == RLT_DTYPE_BF16) {
    // tensor-core contraction shapes: 128-row weight tiles, 64-deep K steps
    if (c->d_model % 128 || c->ffn % 64 || c->vocab % 128)
      return fail(RLT_E_INVAL, "bf16 models need d_model % 128 == 0, ffn % 64 == 0, vocab % 128 == 0");
  }
  return RLT_OK;
}

int32_t ensure_rope(rlt_model* m, int len) {
  if (len <= m->rope_len) return RLT_OK;
  int n = m->rope_len > 0 ? m->rope_len : 4096;
  while (n < len) n *= 2;
  const int half = m->hd / 2;
  std::vector<float> h((size_t)n * half * 2);
  for (int p = 0; p < n; ++p)
    for (int i = 0; i < half; ++i) {
      const double th = (double)p * std::pow((double)m->cfg.rope_base, -2.0 * i / m->hd);
      h[((size_t)p * half + i) * 2] = (float)std::cos(th);
      h[((size_t)p * half + i) * 2 + 1] = (float)std::sin(th);
    }
  void* p = nullptr;
  RLT_TRY(dev_alloc(m->allocs, &p, h.size() * sizeof(float)));
  RLT_CUDA(cudaMemcpy(p, h.data(), h.size() * sizeof(float), cudaMemcpyHostToDevice));
  m->rope_cs = static_cast<float*>(p);
  m->rope_len = n;
  return RLT_OK;
}

void add_view(rlt_model* m, const std::string& name, void* base, int64_t rows, int64_t cols, int64_t pitch, int sid,
              int kind) {
  m->views[name] = View{base, rows, cols, pitch, sid, kind};
}

int32_t build_model(rlt_model* m) {
  const rlt_config& c = m->cfg;
  const int64_t d = c.d_model, F = c.ffn, V = c.vocab, L = c.n_layers, G = c.groups;
  const size_t es = m->esz;
  auto A = [&](void** p, int64_t elems) { return dev_alloc(m->allocs, p, (size_t)elems * es); };
  RLT_TRY(A(&m->emb, V * d));
  RLT_TRY(A(&m->s_star, d));
  RLT_TRY(A(&m->g_mem, d));
  RLT_TRY(A(&m->g_merge, d));
  RLT_TRY(A(&m->w_gate, d * 2 * d));
  RLT_TRY(A(&m->b_gate, d));
  RLT_TRY(A(&m->w_state, d * d));
  RLT_TRY(A(&m->g_out, d));
  RLT_TRY(A(&m->w_out, V * d));
  RLT_TRY(A(&m->w_kvm, G * 2 * d * d));
  add_view(m, "emb", m->emb, V, d, d, 0, 0);
  add_view(m, "s_star", m->s_star, 1, d, d, 1, 0);
  add_view(m, "g_mem", m->g_mem, 1, d, d, 2, 1);
  add_view(m, "g_merge", m->g_merge, 1, d, d, 3, 1);
  add_view(m, "w_gate", m->w_gate, d, 2 * d, 2 * d, 4, 0);
  add_view(m, "b_gate", m->b_gate, 1, d, d, 5, 2);
  add_view(m, "w_state", m->w_state, d, d, d, 6, 0);
  add_view(m, "g_out", m->g_out, 1, d, d, 7, 1);
  add_view(m, "w_out", m->w_out, V, d, d, 8, 0);
  for (int g = 0; g < G; ++g) {
    add_view(m, "wk_mem." + std::to_string(g), off(m->w_kvm, (int64_t)g * 2 * d * d, es), d, d, d, 16 + 2 * g, 0);
    add_view(m, "wv_mem." + std::to_string(g), off(m->w_kvm, ((int64_t)g * 2 + 1) * d * d, es), d, d, d, 17 + 2 * g, 0);
  }
  m->layers.resize(L);
  for (int l = 0; l < L; ++l) {
    LayerW& w = m->layers[l];
    const std::string sfx = "." + std::to_string(l);
    const int sid0 = 1024 + 32 * l;
    RLT_TRY(A(&w.qkv, 3 * d * d));
    RLT_TRY(A(&w.wo, d * d));
    RLT_TRY(A(&w.w13, 2 * F * d));
    RLT_TRY(A(&w.w2, d * F));
    RLT_TRY(A(&w.wq_mem, d * d));
    RLT_TRY(A(&w.wo_mem, d * d));
    RLT_TRY(A(&w.g_ea, d));
    RLT_TRY(A(&w.g_ef, d));
    RLT_TRY(A(&w.g_dsa, d));
    RLT_TRY(A(&w.g_dmem, d));
    RLT_TRY(A(&w.g_dffn, d));
    add_view(m, "wq" + sfx, w.qkv, d, d, d, sid0 + 0, 0);
    add_view(m, "wk" + sfx, off(w.qkv, d * d, es), d, d, d, sid0 + 1, 0);
    add_view(m, "wv" + sfx, off(w.qkv, 2 * d * d, es), d, d, d, sid0 + 2, 0);
    add_view(m, "wo" + sfx, w.wo, d, d, d, sid0 + 3, 0);
    add_view(m, "w1" + sfx, w.w13, F, d, 2 * d, sid0 + 4, 0);
    add_view(m, "w2" + sfx, w.w2, d, F, F, sid0 + 5, 0);
    add_view(m, "w3" + sfx, off(w.w13, d, es), F, d, 2 * d, sid0 + 6, 0);
    add_view(m, "g_ea" + sfx, w.g_ea, 1, d, d, sid0 + 7, 1);
    add_view(m, "g_ef" + sfx, w.g_ef, 1, d, d, sid0 + 8, 1);
    add_view(m, "g_dsa" + sfx, w.g_dsa, 1, d, d, sid0 + 9, 1);
    add_view(m, "g_dmem" + sfx, w.g_dmem, 1, d, d, sid0 + 10, 1);
    add_view(m, "g_dffn" + sfx, w.g_dffn, 1, d, d, sid0 + 11, 1);
    add_view(m, "wq_mem" + sfx, w.wq_mem, d, d, d, sid0 + 12, 0);
    add_view(m, "wo_mem" + sfx, w.wo_mem, d, d, d, sid0 + 13, 0);
    if (c.tied) {
      w.dqkv = w.qkv; w.dwo = w.wo; w.dw13 = w.w13; w.dw2 = w.w2;
    } else {
      RLT_TRY(A(&w.dqkv, 3 * d * d));
      RLT_TRY(A(&w.dwo, d * d));
      RLT_TRY(A(&w.dw13, 2 * F * d));
      RLT_TRY(A(&w.dw2, d * F));
      add_view(m, "dwq" + sfx, w.dqkv, d, d, d, sid0 + 14, 0);
      add_view(m, "dwk" + sfx, off(w.dqkv, d * d, es), d, d, d, sid0 + 15, 0);
      add_view(m, "dwv" + sfx, off(w.dqkv, 2 * d * d, es), d, d, d, sid0 + 16, 0);
      add_view(m, "dwo" + sfx, w.dwo, d, d, d, sid0 + 17, 0);
      add_view(m, "dw1" + sfx, w.dw13, F, d, 2 * d, sid0 + 18, 0);
      add_view(m, "dw2" + sfx, w.dw2, d, F, F, sid0 + 19, 0);
      add_view(m, "dw3" + sfx, off(w.dw13, d, es), F, d, 2 * d, sid0 + 20, 0);
    }
  }
  return RLT_OK;
}

template <typename T>
int32_t init_views(rlt_model* m, uint64_t seed) {
  for (auto& kv : m->views) {
    const View& v = kv.second;
    cudaError_t e;
    if (v.kind == 0)
      e = init_normal<T>(static_cast<T*>(v.base), v.rows, v.cols, v.pitch, seed, (uint32_t)v.sid, m->cfg.init_std, 0);
    else
      e = init_const<T>(static_cast<T*>(v.base), v.rows, v.cols, v.pitch, v.kind == 1 ? 1.0f : 0.0f, 0);
    if (e != cudaSuccess) return fail(RLT_E_CUDA, "init " + kv.first + ": " + cudaGetErrorString(e));
  }
  RLT_CUDA(cudaDeviceSynchronize());
  return RLT_OK;
}

// ------------------------------------------------------------------ GEMM dispatch
// Decode-step contractions (split = true) may split K inside a cluster and
// exchange partials through the state's exchange area; token-parallel
// encoder contractions never split.  The split depends on the weight shape
// only, so no reduction order depends on how many rows share a GEMM.
template <typename T>
int32_t gemm(rlt_state* S, const void* W, int64_t ldw, const void* X, int64_t ldx, int M, int N, int K, int epi,
             const EpiParams& ep, bool split, cudaStream_t st);

template <>
int32_t gemm<bf16>(rlt_state* S, const void* W, int64_t ldw, const void* X, int64_t ldx, int M, int N, int K, int epi,
                   const EpiParams& ep, bool split, cudaStream_t st) {
  RLT_CUDA(gemm_tc(static_cast<const bf16*>(W), ldw, static_cast<const bf16*>(X), ldx, M, N, K, epi, ep,
                   split ? 1 : 0, split ? S->gemm_ws : nullptr, split ? S->gemm_ws_floats : 0, st));
  return RLT_OK;
}

template <>
int32_t gemm<float>(rlt_state*, const void* W, int64_t ldw, const void* X, int64_t ldx, int M, int N, int K, int epi,
                    const EpiParams& ep, bool, cudaStream_t st) {
  RLT_CUDA(gemm_simt<float, float>(static_cast<const float*>(W), ldw, static_cast<const float*>(X), ldx, M, N, K, epi,
                                   ep, st));
  return RLT_OK;
}

EpiParams epi_out(void* out, RowMap map, int out_bf16) {
  EpiParams p{};
  p.out = out;
  p.out_map = map;
  p.out_bf16 = out_bf16;
  p.aux0_map = plain_rows(0);
  return p;
}

// Folded RMSNorm (bf16 models): a producer epilogue writes gamma_next * z as
// the next GEMM's bf16 operand plus per-weight-tile sums of z^2; the
// consumer GEMM scales its accumulators by 1/rms(z).  The layer norms of the
// decoder therefore need no kernel of their own.
EpiParams norm_out(EpiParams p, rlt_state* S, const void* gamma) {
  p.zb = static_cast<bf16*>(S->zb);
  p.ld_zb = S->m->cfg.d_model;
  p.gamma_next = gamma;
  p.gamma_bf16 = 1;
  p.ss_out = S->ss;
  p.ss_ld = S->B;
  return p;
}
EpiParams norm_in(EpiParams p, rlt_state* S) {
  p.ss_in = S->ss;
  p.n_ss = S->m->cfg.d_model / 128;
  p.ss_ld = S->B;
  p.norm_scale = 1.0f / (float)S->m->cfg.d_model;
  p.norm_eps = S->m->cfg.rms_eps;
  return p;
}

// ------------------------------------------------------------------ profiling
// Records an event before (prof_begin) and after (prof_end) one kernel launch
// on the launching stream; kind 0 = prefix attention, 1 = SWA attention.
void prof_begin(rlt_model* m, cudaStream_t st) {
  ProfileRec& p = m->prof;
  if (!p.on || !p.sample_now) return;
  if (p.used + 2 > p.ev.size()) {
    for (int i = 0; i < 1024; ++i) {
      cudaEvent_t e;
      if (cudaEventCreate(&e) != cudaSuccess) break;
      p.ev.push_back(e);
    }
  }
  if (p.used + 2 <= p.ev.size()) cudaEventRecord(p.ev[p.used], st);
}
void prof_end(rlt_model* m, cudaStream_t st, int kind, double bytes) {
  ProfileRec& p = m->prof;
  if (!p.on || !p.sample_now || p.used + 2 > p.ev.size()) return;
  cudaEventRecord(p.ev[p.used + 1], st);
  p.kind.push_back(kind);
  p.bytes[kind] += bytes;
  p.launches[kind] += 1;
  p.used += 2;
}

// ------------------------------------------------------------------ state
int32_t make_state(rlt_model* m, int32_t B, int32_t max_len, int32_t flags, rlt_state** out) {
  const rlt_config& c = m->cfg;
  if (B <= 0 || max_len <= 0) return fail(RLT_E_INVAL, "batch and max_len must be positive");
  RLT_TRY(ensure_rope(m, max_len + 1));
  rlt_state* S = new rlt_state();
  S->m = m;
  S->B = B;
  S->max_len = max_len;
  S->flags = flags;
  S->version = m->version;
  const int64_t d = c.d_model, L = c.n_layers, G = c.groups, F = c.ffn, V = c.vocab, Wm1 = c.window - 1;
  const size_t es = m->esz;
  auto A = [&](void** p, int64_t bytes) { return dev_alloc(S->allocs, p, (size_t)bytes); };
  int32_t r = RLT_OK;
  void* p = nullptr;
  if ((r = A(&p, (int64_t)B * max_len * d * 4))) goto fail_;
  S->e = static_cast<float*>(p);
  if ((r = A(&S->mem_k, G * B * max_len * d * (int64_t)es))) goto fail_;
  if ((r = A(&S->mem_v, G * B * max_len * d * (int64_t)es))) goto fail_;
  if (flags & RLT_STATE_ENCODER_CACHE) {
    if ((r = A(&S->ce_k, L * B * max_len * d * (int64_t)es))) goto fail_;
    if ((r = A(&S->ce_v, L * B * max_len * d * (int64_t)es))) goto fail_;
  }
  if (Wm1 > 0) {
    if ((r = A(&S->ring_k, L * B * Wm1 * d * (int64_t)es))) goto fail_;
    if ((r = A(&S->ring_v, L * B * Wm1 * d * (int64_t)es))) goto fail_;
  }
  if ((r = A(&p, (int64_t)B * d * 4))) goto fail_;
  S->s = static_cast<float*>(p);
  if ((r = A(&p, (int64_t)B * d * 4))) goto fail_;
  S->et = static_cast<float*>(p);
  if ((r = A(&p, (int64_t)B * d * 4))) goto fail_;
  S->s_save = static_cast<float*>(p);
  if ((r = A(&p, (int64_t)3 * B * 4))) goto fail_;
  S->pos = static_cast<int32_t*>(p);
  if ((r = A(&S->xb, (int64_t)B * 2 * d * es))) goto fail_;
  if (c.dtype == RLT_DTYPE_BF16) {
    if ((r = A(&S->zb, (int64_t)B * d * 2))) goto fail_;
    if ((r = A(&S->zb_save, (int64_t)B * d * 2))) goto fail_;
    if ((r = A(&p, (int64_t)(d / 128) * B * 4))) goto fail_;
    S->ss = static_cast<float*>(p);
    if ((r = A(&p, (int64_t)(d / 128) * B * 4))) goto fail_;
    S->ss_save = static_cast<float*>(p);
  }
  S->enc_h.assign(B, 0);
  S->dec_h.assign(B, 0);
  S->lim_h.assign(B, 0);
  S->ld_qkv = std::max<int64_t>(3 * d, 2 * d * G);
  if ((r = A(&p, (int64_t)B * S->ld_qkv * 4))) goto fail_;
  S->qkv = static_cast<float*>(p);
  if ((r = A(&S->attn, (int64_t)B * d * es))) goto fail_;
  if ((r = A(&S->hbuf, (int64_t)B * F * es))) goto fail_;
  if ((r = A(&p, (int64_t)B * d * 4))) goto fail_;
  S->gate = static_cast<float*>(p);
  if ((r = A(&p, (int64_t)B * V * 4))) goto fail_;
  S->logits = static_cast<float*>(p);
  S->attn_ws_floats = prefix_attn_workspace_floats(B, c.n_heads, (int)(d / c.n_heads), max_len);
  if ((r = A(&p, (int64_t)S->attn_ws_floats * 4))) goto fail_;
  S->attn_ws = static_cast<float*>(p);
  if ((r = A(&p, (int64_t)B * c.n_heads * 4))) goto fail_;
  S->attn_cnt = static_cast<int*>(p);  // zeroed by reset_state
  if ((r = A(&p, (int64_t)B * 4))) goto fail_;
  S->pending = static_cast<int32_t*>(p);
  if (c.dtype == RLT_DTYPE_BF16) {
    // every weight shape a step contracts with B rows
    const int64_t shapes[][2] = {{d, 2 * d}, {d, d}, {3 * d, d}, {2 * (int64_t)F, d}, {d, F}, {V, d}, {2 * d * G, d}};
    for (const auto& mk : shapes)
      S->gemm_ws_floats = std::max(S->gemm_ws_floats, gemm_tc_workspace_floats((int)mk[0], B, (int)mk[1], 1));
    if ((r = A(&p, (int64_t)S->gemm_ws_floats * 4))) goto fail_;
    S->gemm_ws = static_cast<float*>(p);
  }
  *out = S;
  return RLT_OK;
fail_:
  free_all(S->allocs);
  delete S;
  return r;
}

template <typename T>
int32_t reset_state(rlt_state* S, cudaStream_t st) {
  RLT_CUDA(broadcast_row<T>(static_cast<const T*>(S->m->s_star), S->m->cfg.d_model, S->s, S->B, st));
  RLT_CUDA(cudaMemsetAsync(S->pos, 0, (size_t)3 * S->B * 4, st));
  RLT_CUDA(cudaMemsetAsync(S->attn_cnt, 0, (size_t)S->B * S->m->cfg.n_heads * 4, st));
  std::fill(S->enc_h.begin(), S->enc_h.end(), 0);
  std::fill(S->dec_h.begin(), S->dec_h.end(), 0);
  S->has_pending = false;
  S->version = S->m->version;
  return RLT_OK;
}

int32_t ensure_prefill_ws(rlt_state* S, int T) {
  const rlt_config& c = S->m->cfg;
  const int64_t d = c.d_model, G = c.groups, F = c.ffn;
  const size_t es = S->m->esz;
  const int64_t big_cols = std::max<int64_t>(std::max<int64_t>(3 * d, F), 2 * d * G);
  const bool cache = (S->flags & RLT_STATE_ENCODER_CACHE) != 0;
  // bytes per token row of the prefill workspace
  const int64_t per_row = (int64_t)es * (d /*x*/ + big_cols + d /*q*/ + d /*attn*/ + (cache ? 0 : 2 * d));
  const int64_t budget = (int64_t)4 << 30;
  int64_t seqs = std::max<int64_t>(1, std::min<int64_t>(S->B, budget / (per_row * T)));
  const int64_t rows = seqs * T;
  if (rows <= S->pf_rows && S->pf_big_cols == big_cols) return RLT_OK;
  for (void* p : {S->pf_x, S->pf_big, S->pf_q, S->pf_k, S->pf_v, S->pf_attn}) {
    if (!p) continue;
    cudaFree(p);
    for (auto it = S->allocs.begin(); it != S->allocs.end(); ++it)
      if (*it == p) { S->allocs.erase(it); break; }
  }
  S->pf_x = S->pf_big = S->pf_q = S->pf_k = S->pf_v = S->pf_attn = nullptr;
  S->pf_rows = 0;
  auto A = [&](void** p, int64_t bytes) { return dev_alloc(S->allocs, p, (size_t)bytes); };
  RLT_TRY(A(&S->pf_x, rows * d * (int64_t)es));
  RLT_TRY(A(&S->pf_big, rows * big_cols * (int64_t)es));
  RLT_TRY(A(&S->pf_q, rows * d * (int64_t)es));
  RLT_TRY(A(&S->pf_attn, rows * d * (int64_t)es));
  if (!cache) {
    RLT_TRY(A(&S->pf_k, rows * d * (int64_t)es));
    RLT_TRY(A(&S->pf_v, rows * d * (int64_t)es));
  }
  S->pf_rows = rows;
  S->pf_big_cols = big_cols;
  return RLT_OK;
}

int32_t check_state(rlt_model* m, rlt_state* S) {
  if (!m || !S) return fail(RLT_E_INVAL, "null model or state");
  if (S->m != m) return fail(RLT_E_INVAL, "state belongs to another model");
  if (S->version != m->version) return fail(RLT_E_STALE, "state was built under older weights");
  RLT_CUDA(cudaSetDevice(m->device));
  return RLT_OK;
}

// ------------------------------------------------------------------ schedules
// Device views of a state's per-sequence positions.
SeqPos seq_pos(const rlt_state* S, bool masked) {
  return SeqPos{S->pos + S->B, S->pos, masked ? S->pos + 2 * S->B : nullptr};
}
bool active_h(const rlt_state* S, bool masked, int b) { return !masked || S->dec_h[b] < S->lim_h[b]; }
// Keys an attention query of sequence b reads in the transition in flight
// (the host image of SeqPos::n_keys).
int n_keys_h(const rlt_state* S, bool masked, int b) {
  return active_h(S, masked, b) ? S->dec_h[b] + 1 : std::max(1, S->dec_h[b]);
}
int max_of(const std::vector<int32_t>& v) { return v.empty() ? 0 : *std::max_element(v.begin(), v.end()); }
bool uniform(const std::vector<int32_t>& v) {
  return std::all_of(v.begin(), v.end(), [&](int32_t x) { return x == v[0]; });
}

// Token-parallel encoder (eq. 2.1) and the memory projection of eq. 2.2 over
// Tn tokens of sequences [b_begin, b_end), which all stand at n_enc = p0;
// sequence b's tokens are tok[b * ld_tok + 0..Tn-1].  Chunked over
// sequences.  With p0 > 0 (keys and values of the prefix in the encoder
// cache) the tokens are positions p0+1..p0+Tn and attend to the cached
// prefix too: the chunked schedule of the same causal computation (App. A.2).
template <typename T>
int32_t encode_prefix_impl(rlt_model* m, rlt_state* S, const int32_t* tok, int64_t ld_tok, int32_t Tn, int b_begin,
                           int b_end, int p0, cudaStream_t st) {
  struct Range {
    bool on;
    explicit Range(bool o) : on(o) { if (on) nvtxRangePushA("rlt_sample"); }
    ~Range() { if (on) nvtxRangePop(); }
  } range(m->prof.on);
  const rlt_config& c = m->cfg;
  const int d = c.d_model, H = c.n_heads, hd = m->hd, F = c.ffn, G = c.groups, L = c.n_layers;
  const int is_bf16 = c.dtype == RLT_DTYPE_BF16;
  const bool cache = (S->flags & RLT_STATE_ENCODER_CACHE) != 0;
  RLT_TRY(ensure_prefill_ws(S, Tn));
  const int64_t seqs_per_chunk = S->pf_rows / Tn;
  for (int64_t b0 = b_begin; b0 < b_end; b0 += seqs_per_chunk) {
    const int Bc = (int)std::min<int64_t>(seqs_per_chunk, b_end - b0);
    const int64_t rows = (int64_t)Bc * Tn;
    float* e0 = S->e + b0 * S->max_len * d + (int64_t)p0 * d;
    const RowMap emap{d, Tn, (int64_t)S->max_len * d};
    RLT_CUDA(embed<T>(tok + b0 * ld_tok, rows, Tn, ld_tok, static_cast<const T*>(m->emb), d, c.vocab, e0, emap, st));
    for (int l = 0; l < L; ++l) {
      const LayerW& w = m->layers[l];
      RLT_CUDA(rmsnorm<T, T>(e0, emap, static_cast<const T*>(w.g_ea), rows, d, c.rms_eps, static_cast<T*>(S->pf_x), d, st));
      RLT_TRY(gemm<T>(S, w.qkv, d, S->pf_x, d, 3 * d, (int)rows, d, EPI_STORE, epi_out(S->pf_big, plain_rows(3 * d), is_bf16),
                      false, st));
      T* kdst;
      T* vdst;
      int64_t ld_tk;
      if (cache) {
        const int64_t lay = (int64_t)l * S->B * H * S->max_len * hd;
        kdst = static_cast<T*>(S->ce_k) + lay + b0 * H * S->max_len * hd;
        vdst = static_cast<T*>(S->ce_v) + lay + b0 * H * S->max_len * hd;
        ld_tk = S->max_len;
      } else {
        kdst = static_cast<T*>(S->pf_k);
        vdst = static_cast<T*>(S->pf_v);
        ld_tk = Tn;
      }
      const T* qkv = static_cast<const T*>(S->pf_big);
      const int kv_row0 = cache ? p0 : 0;
      RLT_CUDA((head_scatter<T, T>(qkv, 3 * d, 0, rows, Tn, p0, 0, H, hd, 1, m->rope_cs, static_cast<T*>(S->pf_q), Tn,
                                   st)));
      RLT_CUDA((head_scatter<T, T>(qkv, 3 * d, d, rows, Tn, p0, kv_row0, H, hd, 1, m->rope_cs, kdst, ld_tk, st)));
      RLT_CUDA((head_scatter<T, T>(qkv, 3 * d, 2 * d, rows, Tn, p0, kv_row0, H, hd, 0, m->rope_cs, vdst, ld_tk, st)));
      if constexpr (std::is_same<T, bf16>::value) {
        if (hd == 64 || hd == 128)
          RLT_CUDA(causal_attn_tc(static_cast<const bf16*>(S->pf_q), kdst, vdst, Tn, ld_tk, Bc, H, hd, Tn, p0,
                                  static_cast<bf16*>(S->pf_attn), d, st));
        else
          RLT_CUDA(causal_attn<T>(static_cast<const T*>(S->pf_q), kdst, vdst, Tn, ld_tk, Bc, H, hd, Tn, p0,
                                  static_cast<T*>(S->pf_attn), d, st));
      } else {
        RLT_CUDA(causal_attn<T>(static_cast<const T*>(S->pf_q), kdst, vdst, Tn, ld_tk, Bc, H, hd, Tn, p0,
                                static_cast<T*>(S->pf_attn), d, st));
      }
      RLT_TRY(gemm<T>(S, w.wo, d, S->pf_attn, d, d, (int)rows, d, EPI_RESID, epi_out(e0, emap, 0), false, st));
      RLT_CUDA(rmsnorm<T, T>(e0, emap, static_cast<const T*>(w.g_ef), rows, d, c.rms_eps, static_cast<T*>(S->pf_x), d, st));
      RLT_TRY(gemm<T>(S, w.w13, d, S->pf_x, d, 2 * F, (int)rows, d, EPI_SWIGLU, epi_out(S->pf_big, plain_rows(F), is_bf16),
                      false, st));
      RLT_TRY(gemm<T>(S, w.w2, F, S->pf_big, F, d, (int)rows, F, EPI_RESID, epi_out(e0, emap, 0), false, st));
    }
    // memory projection (eq. 2.2): n = RMSNorm_E(e); k^g = RoPE(W_K^g n), v^g = W_V^g n
    RLT_CUDA(rmsnorm<T, T>(e0, emap, static_cast<const T*>(m->g_mem), rows, d, c.rms_eps, static_cast<T*>(S->pf_x), d, st));
    RLT_TRY(gemm<T>(S, m->w_kvm, d, S->pf_x, d, 2 * d * G, (int)rows, d, EPI_STORE,
                    epi_out(S->pf_big, plain_rows(2 * d * G), is_bf16), false, st));
    for (int g = 0; g < G; ++g) {
      const int64_t grp = ((int64_t)g * S->B + b0) * H * S->max_len * hd;
      const T* kv = static_cast<const T*>(S->pf_big);
      RLT_CUDA((head_scatter<T, T>(kv, 2 * d * G, (int64_t)2 * d * g, rows, Tn, p0, p0, H, hd, 1, m->rope_cs,
                                   static_cast<T*>(S->mem_k) + grp, S->max_len, st)));
      RLT_CUDA((head_scatter<T, T>(kv, 2 * d * G, (int64_t)2 * d * g + d, rows, Tn, p0, p0, H, hd, 0, m->rope_cs,
                                   static_cast<T*>(S->mem_v) + grp, S->max_len, st)));
    }
  }
  RLT_CUDA(set_positions(S->pos, b_begin, b_end, p0 + Tn, st));
  for (int b = b_begin; b < b_end; ++b) S->enc_h[b] = p0 + Tn;
  return RLT_OK;
}

// Encoder step (eq. 2.8) and memory append for the token x_t of every
// sequence whose position t = n_dec + 1 is not yet encoded (n_enc < t); the
// other sequences' rows are computed but written nowhere.  The step works on
// S->et (one row per sequence) and then stores the encoded rows into e.
template <typename T>
int32_t encode_step_impl(rlt_model* m, rlt_state* S, const int32_t* tok, bool masked, cudaStream_t st) {
  const rlt_config& c = m->cfg;
  const int d = c.d_model, H = c.n_heads, hd = m->hd, F = c.ffn, G = c.groups, L = c.n_layers, B = S->B;
  const int is_bf16 = c.dtype == RLT_DTYPE_BF16;
  const SeqPos sp = seq_pos(S, masked);
  int n_max = 1;
  double key_rows = 0;
  for (int b = 0; b < B; ++b) {
    n_max = std::max(n_max, n_keys_h(S, masked, b));
    key_rows += n_keys_h(S, masked, b);
  }
  m->prof.sample_now = ((max_of(S->dec_h) + 1) % 4) == 0;
  float* et = S->et;
  const RowMap erow = plain_rows(d);
  // bf16 models fold the pre-norms after the first into the GEMMs, as the
  // decoder does: each residual epilogue leaves gamma_next * e and the sums of
  // squares, and the next GEMM scales its accumulators by 1/rms.  The folded
  // operand lives in the state's zb/ss, which the transition that follows
  // overwrites.
  constexpr bool fused = std::is_same<T, bf16>::value;
  auto normed_in = [&](const void* gamma, bool first) -> int32_t {
    if (fused && !first) return RLT_OK;
    RLT_CUDA(rmsnorm<T, T>(et, erow, static_cast<const T*>(gamma), B, d, c.rms_eps, static_cast<T*>(S->xb), d, st));
    return RLT_OK;
  };
  auto xin = [&](bool first) -> const void* { return (fused && !first) ? S->zb : S->xb; };
  auto cin = [&](EpiParams p, bool first) { return (fused && !first) ? norm_in(p, S) : p; };
  auto cout_ = [&](EpiParams p, const void* gamma_next) { return fused ? norm_out(p, S, gamma_next) : p; };
  RLT_CUDA(embed<T>(tok, B, 1, 1, static_cast<const T*>(m->emb), d, c.vocab, et, erow, st));
  for (int l = 0; l < L; ++l) {
    const LayerW& w = m->layers[l];
    const int64_t lay = (int64_t)l * B * H * S->max_len * hd;
    T* ck = static_cast<T*>(S->ce_k) + lay;
    T* cv = static_cast<T*>(S->ce_v) + lay;
    const void* g_next = l + 1 < L ? m->layers[l + 1].g_ea : m->g_mem;
    RLT_TRY(normed_in(w.g_ea, l == 0));
    RLT_TRY(gemm<T>(S, w.qkv, d, xin(l == 0), d, 3 * d, B, d, EPI_STORE,
                    cin(epi_out(S->qkv, plain_rows(S->ld_qkv), 0), l == 0), true, st));
    RLT_CUDA((head_insert<float, T>(S->qkv, S->ld_qkv, d, B, sp, H, hd, 1, m->rope_cs, ck, S->max_len, st)));
    RLT_CUDA((head_insert<float, T>(S->qkv, S->ld_qkv, 2 * d, B, sp, H, hd, 0, m->rope_cs, cv, S->max_len, st)));
    prof_begin(m, st);
    RLT_CUDA(prefix_attn<T>(S->qkv, S->ld_qkv, ck, cv, S->max_len, B, H, hd, n_max, n_max - 1, sp, m->rope_cs,
                            static_cast<T*>(S->attn), d, S->attn_ws, S->attn_ws_floats, S->attn_cnt, st));
    prof_end(m, st, 0, key_rows * H * hd * 2 * m->esz);
    RLT_TRY(gemm<T>(S, w.wo, d, S->attn, d, d, B, d, EPI_RESID, cout_(epi_out(et, erow, 0), w.g_ef), true, st));
    RLT_TRY(normed_in(w.g_ef, false));
    RLT_TRY(gemm<T>(S, w.w13, d, xin(false), d, 2 * F, B, d, EPI_SWIGLU,
                    cin(epi_out(S->hbuf, plain_rows(F), is_bf16), false), true, st));
    RLT_TRY(gemm<T>(S, w.w2, F, S->hbuf, F, d, B, F, EPI_RESID, cout_(epi_out(et, erow, 0), g_next), true, st));
  }
  RLT_TRY(normed_in(m->g_mem, false));
  RLT_TRY(gemm<T>(S, m->w_kvm, d, xin(false), d, 2 * d * G, B, d, EPI_STORE,
                  cin(epi_out(S->qkv, plain_rows(S->ld_qkv), 0), false), true, st));
  for (int g = 0; g < G; ++g) {
    const int64_t grp = (int64_t)g * B * H * S->max_len * hd;
    RLT_CUDA((head_insert<float, T>(S->qkv, S->ld_qkv, (int64_t)2 * d * g, B, sp, H, hd, 1, m->rope_cs,
                                    static_cast<T*>(S->mem_k) + grp, S->max_len, st)));
    RLT_CUDA((head_insert<float, T>(S->qkv, S->ld_qkv, (int64_t)2 * d * g + d, B, sp, H, hd, 0, m->rope_cs,
                                    static_cast<T*>(S->mem_v) + grp, S->max_len, st)));
  }
  RLT_CUDA(erow_scatter(et, S->max_len, d, B, sp, S->e, st));
  return RLT_OK;
}

// One decoder transition H_t = D_phi(Merge(e_t, s_{t-1}); M_<=t, C^D_{t-1}, t)
// (eqs. 2.4-2.5, 2.9-2.16) for every sequence b at its own t_b = n_dec[b] + 1.
// s is updated in place: it holds u_t after the merge, then z^l after every
// block, and s_t at the end.  In a masked phase only the sequences with
// n_dec < lim take part: the others' rows are computed, their ring and
// positions left as they were, and their s restored at the end.  `et_ready`:
// S->et already holds e_t of every sequence (the encoder step ran for all).
// While profiling is on, every 4th transition records kernel events
// (prof_begin/prof_end), and each position with t = 64 (mod 128) -- its
// encoder step, transition and readout -- is wrapped in an NVTX range named
// "rlt_sample", so a kernel profiler can capture a stratified sample of a
// long schedule instead of every launch.
struct StepRange {
  bool nvtx = false;
  StepRange(rlt_model* m, int t) {
    if (m->prof.on && (t % 128) == 64) {
      nvtxRangePushA("rlt_sample");
      nvtx = true;
    }
  }
  ~StepRange() {
    if (nvtx) nvtxRangePop();
  }
};

template <typename T>
int32_t transition_impl(rlt_model* m, rlt_state* S, bool masked, bool et_ready, cudaStream_t st) {
  const rlt_config& c = m->cfg;
  const int d = c.d_model, H = c.n_heads, hd = m->hd, F = c.ffn, L = c.n_layers, B = S->B, W = c.window;
  const int is_bf16 = c.dtype == RLT_DTYPE_BF16;
  const SeqPos sp = seq_pos(S, masked);
  int n_max = 1;
  double key_rows = 0, ring_rows = 0;
  for (int b = 0; b < B; ++b) {
    const int n = n_keys_h(S, masked, b);
    n_max = std::max(n_max, n);
    key_rows += n;
    ring_rows += std::min(S->dec_h[b], W - 1) + ((W > 1 && active_h(S, masked, b)) ? 1 : 0);
  }
  m->prof.sample_now = ((max_of(S->dec_h) + 1) % 4) == 0;
  const RowMap srow = plain_rows(d);
  constexpr bool fused = std::is_same<T, bf16>::value;  // folded RMSNorm on the tensor-core path
  const int n_ss = fused ? d / 128 : 0;
  if (masked)
    RLT_CUDA(save_rows(S->s, S->s_save, static_cast<const bf16*>(S->zb), static_cast<bf16*>(S->zb_save), S->ss,
                       S->ss_save, B, d, n_ss, st));
  if (!et_ready) RLT_CUDA(erow_gather(S->e, S->max_len, d, B, sp, S->et, st));
  const float* et = S->et;
  // merge
  RLT_CUDA((merge_prep<T, T>(et, srow, S->s, static_cast<const T*>(m->g_merge), B, d, c.rms_eps, c.merge_kind,
                             static_cast<T*>(S->xb), st)));
  if (c.merge_kind == RLT_MERGE_PAPER) {
    EpiParams g = epi_out(S->gate, srow, 0);
    g.bias = m->b_gate;
    g.bias_bf16 = is_bf16;
    RLT_TRY(gemm<T>(S, m->w_gate, 2 * d, S->xb, 2 * d, d, B, 2 * d, EPI_GATE, g, true, st));
    EpiParams u = epi_out(S->s, srow, 0);
    u.aux0 = et;
    u.aux0_map = srow;
    u.aux1 = S->gate;
    u.ld_aux1 = d;
    u.alpha = c.alpha;
    if (fused) u = norm_out(u, S, m->layers[0].g_dsa);
    RLT_TRY(gemm<T>(S, m->w_state, d, off(S->xb, d, m->esz), 2 * d, d, B, d, EPI_MERGE, u, true, st));
  } else {
    EpiParams u = epi_out(S->s, srow, 0);
    u.aux0 = et;
    u.aux0_map = srow;
    if (fused) u = norm_out(u, S, m->layers[0].g_dsa);
    RLT_TRY(gemm<T>(S, m->w_gate, 2 * d, S->xb, 2 * d, d, B, 2 * d, EPI_CONVEX, u, true, st));
  }
  // operand of a normalised sublayer: gamma*z from the previous epilogue
  // (fused), or a separate RMSNorm of the residual stream
  auto normed = [&](const void* gamma) -> int32_t {
    if (fused) return RLT_OK;
    RLT_CUDA(rmsnorm<T, T>(S->s, srow, static_cast<const T*>(gamma), B, d, c.rms_eps, static_cast<T*>(S->xb), d, st));
    return RLT_OK;
  };
  const void* xin = fused ? S->zb : S->xb;
  auto cin = [&](EpiParams p) { return fused ? norm_in(p, S) : p; };
  auto cout_ = [&](EpiParams p, const void* gamma_next) { return fused ? norm_out(p, S, gamma_next) : p; };
  for (int l = 0; l < L; ++l) {
    const LayerW& w = m->layers[l];
    const int grp = c.groups == 1 ? 0 : l;
    const void* g_next = l + 1 < L ? m->layers[l + 1].g_dsa : m->g_out;
    // SWA sublayer (eqs. 2.12-2.14)
    RLT_TRY(normed(w.g_dsa));
    RLT_TRY(gemm<T>(S, w.dqkv, d, xin, d, 3 * d, B, d, EPI_STORE, cin(epi_out(S->qkv, plain_rows(3 * d), 0)), true, st));
    const int64_t rlay = (int64_t)l * B * H * (W > 1 ? W - 1 : 0) * hd;
    T* rk = W > 1 ? static_cast<T*>(S->ring_k) + rlay : nullptr;
    T* rv = W > 1 ? static_cast<T*>(S->ring_v) + rlay : nullptr;
    prof_begin(m, st);
    RLT_CUDA(swa_attn<T>(S->qkv, 3 * d, rk, rv, B, H, hd, 0, sp, W, m->rope_cs, static_cast<T*>(S->attn), d, st));
    prof_end(m, st, 1, ring_rows * H * hd * m->esz * 2.0);
    RLT_TRY(gemm<T>(S, w.dwo, d, S->attn, d, d, B, d, EPI_RESID, cout_(epi_out(S->s, srow, 0), w.g_dmem), true, st));
    // cross-attention to M^{g(l)}_{<=t} (eq. 2.15)
    RLT_TRY(normed(w.g_dmem));
    RLT_TRY(gemm<T>(S, w.wq_mem, d, xin, d, d, B, d, EPI_STORE, cin(epi_out(S->qkv, plain_rows(d), 0)), true, st));
    const int64_t mg = (int64_t)grp * B * H * S->max_len * hd;
    prof_begin(m, st);
    RLT_CUDA(prefix_attn<T>(S->qkv, d, static_cast<const T*>(S->mem_k) + mg, static_cast<const T*>(S->mem_v) + mg,
                            S->max_len, B, H, hd, n_max, n_max - 1, sp, m->rope_cs, static_cast<T*>(S->attn), d,
                            S->attn_ws, S->attn_ws_floats, S->attn_cnt, st));
    prof_end(m, st, 0, key_rows * H * hd * 2 * m->esz);
    RLT_TRY(gemm<T>(S, w.wo_mem, d, S->attn, d, d, B, d, EPI_RESID, cout_(epi_out(S->s, srow, 0), w.g_dffn), true, st));
    // FFN (eq. 2.16)
    RLT_TRY(normed(w.g_dffn));
    RLT_TRY(gemm<T>(S, w.dw13, d, xin, d, 2 * F, B, d, EPI_SWIGLU, cin(epi_out(S->hbuf, plain_rows(F), is_bf16)), true,
                    st));
    RLT_TRY(gemm<T>(S, w.dw2, F, S->hbuf, F, d, B, F, EPI_RESID, cout_(epi_out(S->s, srow, 0), g_next), true, st));
  }
  // positions (and, for idle sequences of a masked phase, their saved rows);
  // the caller moves the host copies with advance_host
  RLT_CUDA(advance_positions(S->pos + B, S->pos, masked ? S->pos + 2 * B : nullptr, B, d, S->s,
                             masked ? S->s_save : nullptr, static_cast<bf16*>(S->zb),
                             static_cast<const bf16*>(S->zb_save), S->ss, S->ss_save, n_ss, st));
  return RLT_OK;
}

// Host copies of the positions after a transition, as advance_kernel moves
// the device copy.
void advance_host(rlt_state* S, bool masked) {
  for (int b = 0; b < S->B; ++b) {
    if (!active_h(S, masked, b)) continue;
    S->dec_h[b] += 1;
    S->enc_h[b] = std::max(S->enc_h[b], S->dec_h[b]);
  }
}

// Readout (eq. 2.6) of s_t: logits = W_o RMSNorm_o(s_t), then the teacher
// log-prob and/or the behaviour sample (the sampler's position is each
// sequence's own n_dec).  In a masked phase the log-prob is written only for
// the sequences whose phase has a next token left.
template <typename T>
int32_t readout_impl(rlt_model* m, rlt_state* S, const int32_t* next, int64_t next_stride, float* logp, int64_t ld_logp,
                     const rlt_sampling* samp, const rlt_readout_out* out, bool masked, cudaStream_t st) {
  const rlt_config& c = m->cfg;
  const int d = c.d_model, V = c.vocab, B = S->B;
  if constexpr (std::is_same<T, bf16>::value) {
    // the last transition's final epilogue left gamma_o * s_t and its sums of squares
    RLT_TRY(gemm<T>(S, m->w_out, d, S->zb, d, V, B, d, EPI_STORE, norm_in(epi_out(S->logits, plain_rows(V), 0), S),
                    true, st));
  } else {
    RLT_CUDA(rmsnorm<T, T>(S->s, plain_rows(d), static_cast<const T*>(m->g_out), B, d, c.rms_eps,
                           static_cast<T*>(S->xb), d, st));
    RLT_TRY(gemm<T>(S, m->w_out, d, S->xb, d, V, B, d, EPI_STORE, epi_out(S->logits, plain_rows(V), 0), true, st));
  }
  if (next && logp)
    RLT_CUDA(logp_gather(S->logits, B, V, next, next_stride, logp, ld_logp, S->pos + B,
                         masked ? S->pos + 2 * B : nullptr, st));
  if (samp) {
    int32_t* tok_out = out && out->sampled ? out->sampled : S->pending;
    RLT_CUDA(sample_topk(S->logits, B, V, samp->temperature, samp->top_k, samp->seed, 0, S->pos + B, tok_out,
                         out ? out->logp_sampled : nullptr, out ? out->logmu : nullptr, st));
    if (tok_out != S->pending)
      RLT_CUDA(cudaMemcpyAsync(S->pending, tok_out, (size_t)B * 4, cudaMemcpyDeviceToDevice, st));
    S->has_pending = true;  // the sampled token is owed to the next transition
  }
  if (out && out->logits) RLT_CUDA(copy_f32(out->logits, S->logits, (int64_t)B * V, st));
  return RLT_OK;
}

#define RLT_DISPATCH(m, fn, ...) \
  ((m)->cfg.dtype == RLT_DTYPE_BF16 ? fn<bf16>(__VA_ARGS__) : fn<float>(__VA_ARGS__))

// The kernels of one decoder step (encoder step where needed, then the
// transition), launched directly or, for states made with RLT_STATE_GRAPHS,
// through the step graph of their shape.
int32_t step_kernels(rlt_model* m, rlt_state* s, const int32_t* tok_src, bool any_enc, bool all_enc, cudaStream_t st) {
  if (any_enc) RLT_TRY(RLT_DISPATCH(m, encode_step_impl, m, s, tok_src, false, st));
  RLT_TRY(RLT_DISPATCH(m, transition_impl, m, s, false, any_enc && all_enc, st));
  return RLT_OK;
}

int32_t step_launch(rlt_model* m, rlt_state* s, const int32_t* tok_src, bool any_enc, bool all_enc, cudaStream_t st) {
  if (!(s->flags & RLT_STATE_GRAPHS) || !s->graph_ok || m->prof.on)
    return step_kernels(m, s, tok_src, any_enc, all_enc, st);
  int n_max = 1;
  for (int b = 0; b < s->B; ++b) n_max = std::max(n_max, n_keys_h(s, false, b));
  const rlt_state::GraphKey key{(any_enc ? 1 : 0) + (all_enc ? 2 : 0), tok_src, (n_max + kPrefixChunk - 1) / kPrefixChunk};
  auto it = s->graphs.find(key);
  if (it == s->graphs.end()) {
    if (!s->graph_seen.count(key)) {  // first time: plain launches (one-time kernel setup happens outside a capture)
      s->graph_seen.insert(key);
      return step_kernels(m, s, tok_src, any_enc, all_enc, st);
    }
    if (!s->gstream) {
      RLT_CUDA(cudaStreamCreateWithFlags(&s->gstream, cudaStreamNonBlocking));
      RLT_CUDA(cudaEventCreateWithFlags(&s->ev_in, cudaEventDisableTiming));
      RLT_CUDA(cudaEventCreateWithFlags(&s->ev_out, cudaEventDisableTiming));
    }
    cudaGraph_t g = nullptr;
    const int64_t n0 = launch_count();
    bool captured = cudaStreamBeginCapture(s->gstream, cudaStreamCaptureModeThreadLocal) == cudaSuccess;
    const int32_t r = captured ? step_kernels(m, s, tok_src, any_enc, all_enc, s->gstream) : RLT_OK;
    if (captured) captured = cudaStreamEndCapture(s->gstream, &g) == cudaSuccess && r == RLT_OK;
    cudaGraphExec_t exec = nullptr;
    if (captured) captured = cudaGraphInstantiate(&exec, g, 0) == cudaSuccess;
    if (g) cudaGraphDestroy(g);
    if (!captured) {  // graphs off for this state; this step launches its kernels
      cudaGetLastError();
      s->graph_ok = false;
      return step_kernels(m, s, tok_src, any_enc, all_enc, st);
    }
    it = s->graphs.emplace(key, rlt_state::StepGraph{exec, launch_count() - n0}).first;
  } else {
    for (int64_t i = 0; i < it->second.kernels; ++i) note_launch();
  }
  RLT_CUDA(cudaEventRecord(s->ev_in, st));
  RLT_CUDA(cudaStreamWaitEvent(s->gstream, s->ev_in, 0));
  RLT_CUDA(cudaGraphLaunch(it->second.exec, s->gstream));
  RLT_CUDA(cudaEventRecord(s->ev_out, s->gstream));
  RLT_CUDA(cudaStreamWaitEvent(st, s->ev_out, 0));
  return RLT_OK;
}

int32_t check_sampling(const rlt_sampling* samp, const rlt_readout_out* out) {
  if (!samp) return RLT_OK;
  if (!(samp->temperature > 0.f) || samp->top_k < 1 || samp->top_k > 256)
    return fail(RLT_E_INVAL, "sampler needs temperature > 0 and 1 <= top_k <= 256");
  if (!out || !(out->sampled || out->logmu || out->logp_sampled)) return fail(RLT_E_INVAL, "sampler without outputs");
  return RLT_OK;
}

}  // namespace

// ====================================================================== C ABI
extern "C" {

int32_t rlt_init_weights(const rlt_config* cfg, uint64_t seed, rlt_model** out) {
  if (!out) return fail(RLT_E_INVAL, "null output");
  *out = nullptr;
  RLT_TRY(validate(cfg));
  rlt_model* m = new rlt_model();
  m->cfg = *cfg;
  m->seed = seed;
  m->hd = cfg->d_model / cfg->n_heads;
  m->esz = cfg->dtype == RLT_DTYPE_BF16 ? 2 : 4;
  cudaGetDevice(&m->device);
  int32_t r = build_model(m);
  if (r == RLT_OK) r = ensure_rope(m, 4096);
  if (r == RLT_OK) r = RLT_DISPATCH(m, init_views, m, seed);
  if (r != RLT_OK) {
    free_all(m->allocs);
    delete m;
    return r;
  }
  *out = m;
  return ok();
}

int32_t rlt_tensor_info(const rlt_model* m, const char* name, int64_t* rows, int64_t* cols, int32_t* sid) {
  if (!m || !name) return fail(RLT_E_INVAL, "null argument");
  auto it = m->views.find(name);
  if (it == m->views.end()) return fail(RLT_E_INVAL, std::string("unknown tensor ") + name);
  if (rows) *rows = it->second.rows;
  if (cols) *cols = it->second.cols;
  if (sid) *sid = it->second.sid;
  return ok();
}

int32_t rlt_load_weights(rlt_model* m, const char* name, const void* host, size_t bytes) {
  if (!m || !name || !host) return fail(RLT_E_INVAL, "null argument");
  auto it = m->views.find(name);
  if (it == m->views.end()) return fail(RLT_E_INVAL, std::string("unknown tensor ") + name);
  const View& v = it->second;
  if (bytes != (size_t)(v.rows * v.cols) * m->esz) return fail(RLT_E_INVAL, "size mismatch for " + std::string(name));
  RLT_CUDA(cudaSetDevice(m->device));
  // work still reading the weights may run on streams that do not order
  // with this copy (the backward's own stream, a caller's non-blocking one)
  RLT_CUDA(cudaDeviceSynchronize());
  RLT_CUDA(cudaMemcpy2D(v.base, v.pitch * m->esz, host, v.cols * m->esz, v.cols * m->esz, v.rows, cudaMemcpyHostToDevice));
  m->version += 1;
  return ok();
}

int32_t rlt_get_weights(const rlt_model* m, const char* name, void* host, size_t bytes) {
  if (!m || !name || !host) return fail(RLT_E_INVAL, "null argument");
  auto it = m->views.find(name);
  if (it == m->views.end()) return fail(RLT_E_INVAL, std::string("unknown tensor ") + name);
  const View& v = it->second;
  if (bytes != (size_t)(v.rows * v.cols) * m->esz) return fail(RLT_E_INVAL, "size mismatch for " + std::string(name));
  RLT_CUDA(cudaSetDevice(m->device));
  RLT_CUDA(cudaMemcpy2D(host, v.cols * m->esz, v.base, v.pitch * m->esz, v.cols * m->esz, v.rows, cudaMemcpyDeviceToHost));
  return ok();
}

int32_t rlt_state_free(rlt_state* s);

int32_t rlt_model_free(rlt_model* m) {
  if (!m) return ok();
  if (m->live_states > 0)
    return fail(RLT_E_STATE, std::to_string(m->live_states) + " state(s) of this model are still alive; free them first");
  cudaSetDevice(m->device);
  cudaDeviceSynchronize();
  if (m->replay) rlt_state_free(m->replay);
  release_backward(m);
  for (cudaEvent_t e : m->prof.ev) cudaEventDestroy(e);
  free_all(m->allocs);
  delete m;
  return ok();
}

int32_t rlt_state_create(rlt_model* m, int32_t batch, int32_t max_len, int32_t flags, rlt_state** out) {
  if (!m || !out) return fail(RLT_E_INVAL, "null argument");
  *out = nullptr;
  if (flags & ~(RLT_STATE_ENCODER_CACHE | RLT_STATE_GRAPHS)) return fail(RLT_E_INVAL, "unknown flags");
  RLT_CUDA(cudaSetDevice(m->device));
  rlt_state* S = nullptr;
  RLT_TRY(make_state(m, batch, max_len, flags, &S));
  int32_t r = RLT_DISPATCH(m, reset_state, S, (cudaStream_t)0);
  if (r == RLT_OK) {
    cudaError_t e = cudaStreamSynchronize(0);
    if (e != cudaSuccess) r = fail(RLT_E_CUDA, cudaGetErrorString(e));
  }
  if (r != RLT_OK) {
    free_all(S->allocs);
    delete S;
    return r;
  }
  m->live_states += 1;
  *out = S;
  return ok();
}

int32_t rlt_state_free(rlt_state* s) {
  if (!s) return ok();
  if (s != s->m->replay) s->m->live_states -= 1;
  cudaSetDevice(s->m->device);
  cudaDeviceSynchronize();
  for (auto& g : s->graphs) cudaGraphExecDestroy(g.second.exec);
  if (s->gstream) cudaStreamDestroy(s->gstream);
  if (s->ev_in) cudaEventDestroy(s->ev_in);
  if (s->ev_out) cudaEventDestroy(s->ev_out);
  free_all(s->allocs);
  delete s;
  return ok();
}

int32_t rlt_state_reset(rlt_state* s, void* stream) {
  if (!s) return fail(RLT_E_INVAL, "null state");
  RLT_CUDA(cudaSetDevice(s->m->device));
  return RLT_DISPATCH(s->m, reset_state, s, (cudaStream_t)stream);
}

int32_t rlt_state_info_get(const rlt_state* s, rlt_state_info* out) {
  if (!s || !out) return fail(RLT_E_INVAL, "null argument");
  const int Wm1 = s->m->cfg.window - 1;
  out->batch = s->B;
  out->max_len = s->max_len;
  const int n_enc = max_of(s->enc_h), n_dec = max_of(s->dec_h);
  out->n_enc = n_enc;
  out->n_dec = n_dec;
  out->ring_valid = std::min(n_dec, Wm1);
  out->ring_head = Wm1 > 0 ? n_dec % Wm1 : 0;
  out->has_encoder_cache = (s->flags & RLT_STATE_ENCODER_CACHE) ? 1 : 0;
  out->model_version = s->version;
  out->has_pending = s->has_pending ? 1 : 0;
  out->uniform = (uniform(s->enc_h) && uniform(s->dec_h)) ? 1 : 0;
  return ok();
}

int32_t rlt_state_positions(const rlt_state* s, int32_t* n_enc, int32_t* n_dec, int32_t* ring_valid,
                            int32_t* ring_head) {
  if (!s) return fail(RLT_E_INVAL, "null state");
  const int Wm1 = s->m->cfg.window - 1;
  for (int b = 0; b < s->B; ++b) {
    if (n_enc) n_enc[b] = s->enc_h[b];
    if (n_dec) n_dec[b] = s->dec_h[b];
    if (ring_valid) ring_valid[b] = std::min(s->dec_h[b], Wm1);
    if (ring_head) ring_head[b] = Wm1 > 0 ? s->dec_h[b] % Wm1 : 0;
  }
  return ok();
}

// ------------------------------------------------------------------ snapshots
namespace {

// Exact prefix snapshot (report §6): encoder cache, memory M_<=t, H_t =
// (s_t, C^D_t), positions, window and model identity.  Little-endian; the
// payload follows the header in the order of snapshot_sections().
struct SnapHeader {
  char magic[8];  // "RLTSNAP1"
  uint32_t header_bytes, flags;
  int32_t d_model, n_heads, n_layers, window, groups, ffn, vocab, tied, merge_kind, dtype, bos_id, batch;
  float alpha, rms_eps, rope_base, reserved_f;
  int32_t n_enc, n_dec, reserved0, reserved1;
  uint64_t weight_seed, model_version, payload_bytes;
};
constexpr uint32_t kSnapCache = 1, kSnapPending = 2, kSnapFold = 4, kSnapRagged = 8;

struct SnapSection {
  void* dev;      // first byte on the device
  size_t width;   // bytes per row in the snapshot
  size_t pitch;   // bytes between rows on the device
  size_t rows;
};

std::vector<SnapSection> snapshot_sections(rlt_state* S, int n_enc, uint32_t flags) {
  const rlt_model* m = S->m;
  const rlt_config& c = m->cfg;
  const size_t es = m->esz, d = c.d_model, hd = m->hd, B = S->B, H = c.n_heads, L = c.n_layers, G = c.groups;
  const size_t ml = S->max_len, Wm1 = c.window - 1;
  std::vector<SnapSection> v;
  v.push_back({S->s, B * d * 4, B * d * 4, 1});
  if (n_enc > 0) {
    v.push_back({S->e, (size_t)n_enc * d * 4, ml * d * 4, B});
    v.push_back({S->mem_k, (size_t)n_enc * hd * es, ml * hd * es, G * B * H});
    v.push_back({S->mem_v, (size_t)n_enc * hd * es, ml * hd * es, G * B * H});
    if (flags & kSnapCache) {
      v.push_back({S->ce_k, (size_t)n_enc * hd * es, ml * hd * es, L * B * H});
      v.push_back({S->ce_v, (size_t)n_enc * hd * es, ml * hd * es, L * B * H});
    }
  }
  if (Wm1 > 0) {
    v.push_back({S->ring_k, L * B * H * Wm1 * hd * es, L * B * H * Wm1 * hd * es, 1});
    v.push_back({S->ring_v, L * B * H * Wm1 * hd * es, L * B * H * Wm1 * hd * es, 1});
  }
  if (flags & kSnapPending) v.push_back({S->pending, B * 4, B * 4, 1});
  if (flags & kSnapFold) {
    v.push_back({S->zb, B * d * 2, B * d * 2, 1});
    v.push_back({S->ss, (d / 128) * B * 4, (d / 128) * B * 4, 1});
  }
  // per-sequence positions n_enc[B], n_dec[B] (the first 2B entries of pos)
  if (flags & kSnapRagged) v.push_back({S->pos, 2 * B * 4, 2 * B * 4, 1});
  return v;
}

size_t payload_bytes(const std::vector<SnapSection>& v) {
  size_t n = 0;
  for (const auto& x : v) n += x.width * x.rows;
  return n;
}

uint32_t snapshot_flags(const rlt_state* S) {
  uint32_t f = 0;
  if ((S->flags & RLT_STATE_ENCODER_CACHE) && max_of(S->enc_h) > 0) f |= kSnapCache;
  if (S->has_pending) f |= kSnapPending;
  if (S->m->cfg.dtype == RLT_DTYPE_BF16 && max_of(S->dec_h) > 0) f |= kSnapFold;
  if (!uniform(S->enc_h) || !uniform(S->dec_h)) f |= kSnapRagged;
  return f;
}

}  // namespace

int32_t rlt_state_read(const rlt_state* s, int32_t what, int32_t index, void* host, size_t bytes) {
  if (!s || !host) return fail(RLT_E_INVAL, "null argument");
  const rlt_model* m = s->m;
  const rlt_config& c = m->cfg;
  const int64_t d = c.d_model, B = s->B, Wm1 = c.window - 1;
  const void* src = nullptr;
  size_t n = 0;
  switch (what) {
    case RLT_READ_S: src = s->s; n = (size_t)(B * d) * 4; break;
    case RLT_READ_E: src = s->e; n = (size_t)(B * s->max_len * d) * 4; break;
    case RLT_READ_RING_K:
    case RLT_READ_RING_V:
      if (index < 0 || index >= c.n_layers || Wm1 == 0) return fail(RLT_E_INVAL, "bad layer or empty ring");
      n = (size_t)(B * Wm1 * d) * m->esz;
      src = off(what == RLT_READ_RING_K ? s->ring_k : s->ring_v, (int64_t)index * B * Wm1 * d, m->esz);
      break;
    case RLT_READ_MEM_K:
    case RLT_READ_MEM_V:
      if (index < 0 || index >= c.groups) return fail(RLT_E_INVAL, "bad group");
      n = (size_t)(B * s->max_len * d) * m->esz;
      src = off(what == RLT_READ_MEM_K ? s->mem_k : s->mem_v, (int64_t)index * B * s->max_len * d, m->esz);
      break;
    case RLT_READ_ENC_K:
    case RLT_READ_ENC_V:
      if (!(s->flags & RLT_STATE_ENCODER_CACHE) || index < 0 || index >= c.n_layers)
        return fail(RLT_E_INVAL, "no encoder cache or bad layer");
      n = (size_t)(B * s->max_len * d) * m->esz;
      src = off(what == RLT_READ_ENC_K ? s->ce_k : s->ce_v, (int64_t)index * B * s->max_len * d, m->esz);
      break;
    default: return fail(RLT_E_INVAL, "unknown component");
  }
  if (bytes != n) return fail(RLT_E_INVAL, "size mismatch: need " + std::to_string(n));
  RLT_CUDA(cudaSetDevice(m->device));
  RLT_CUDA(cudaDeviceSynchronize());
  RLT_CUDA(cudaMemcpy(host, src, n, cudaMemcpyDeviceToHost));
  return ok();
}

int32_t rlt_state_export(const rlt_state* s_const, void* host, size_t cap, size_t* used, void* stream) {
  if (!s_const || !used) return fail(RLT_E_INVAL, "null argument");
  rlt_state* S = const_cast<rlt_state*>(s_const);
  const rlt_model* m = S->m;
  const uint32_t flags = snapshot_flags(S);
  const std::vector<SnapSection> secs = snapshot_sections(S, max_of(S->enc_h), flags);
  const size_t total = sizeof(SnapHeader) + payload_bytes(secs);
  *used = total;
  if (!host) return ok();
  if (cap < total) return fail(RLT_E_CAPACITY, "snapshot needs " + std::to_string(total) + " bytes");
  const rlt_config& c = m->cfg;
  SnapHeader h{};
  std::memcpy(h.magic, "RLTSNAP1", 8);
  h.header_bytes = sizeof(SnapHeader);
  h.flags = flags;
  h.d_model = c.d_model; h.n_heads = c.n_heads; h.n_layers = c.n_layers; h.window = c.window; h.groups = c.groups;
  h.ffn = c.ffn; h.vocab = c.vocab; h.tied = c.tied; h.merge_kind = c.merge_kind; h.dtype = c.dtype;
  h.bos_id = c.bos_id; h.batch = S->B;
  h.alpha = c.alpha; h.rms_eps = c.rms_eps; h.rope_base = c.rope_base;
  h.n_enc = max_of(S->enc_h); h.n_dec = max_of(S->dec_h);
  h.weight_seed = m->seed; h.model_version = S->version;
  h.payload_bytes = total - sizeof(SnapHeader);
  std::memcpy(host, &h, sizeof h);
  RLT_CUDA(cudaSetDevice(m->device));
  cudaStream_t st = (cudaStream_t)stream;
  uint8_t* dst = static_cast<uint8_t*>(host) + sizeof h;
  for (const auto& x : secs) {
    RLT_CUDA(cudaMemcpy2DAsync(dst, x.width, x.dev, x.pitch, x.width, x.rows, cudaMemcpyDeviceToHost, st));
    dst += x.width * x.rows;
  }
  RLT_CUDA(cudaStreamSynchronize(st));
  if (flags & kSnapRagged) {
    // The per-position sections hold the furthest sequence's rows for every
    // sequence; the rows a shorter sequence has not reached were never
    // written, so the snapshot carries zeros there (its contents then depend
    // only on the state's history).
    const size_t d = c.d_model, hd = m->hd, es = m->esz, B = S->B, H = c.n_heads;
    dst = static_cast<uint8_t*>(host) + sizeof h;
    for (const auto& x : secs) {
      const bool e_sec = x.dev == S->e;
      const bool kv_sec = x.dev == S->mem_k || x.dev == S->mem_v || x.dev == S->ce_k || x.dev == S->ce_v;
      if (e_sec || kv_sec) {
        const size_t row_bytes = e_sec ? d * 4 : hd * es;
        for (size_t r = 0; r < x.rows; ++r) {
          const size_t b = e_sec ? r : (r / H) % B;
          const size_t keep = (size_t)S->enc_h[b] * row_bytes;
          if (keep < x.width) std::memset(dst + r * x.width + keep, 0, x.width - keep);
        }
      }
      dst += x.width * x.rows;
    }
  }
  return ok();
}

int32_t rlt_state_import(rlt_state* S, const void* host, size_t bytes, void* stream) {
  if (!S || !host) return fail(RLT_E_INVAL, "null argument");
  if (bytes < sizeof(SnapHeader)) return fail(RLT_E_INVAL, "not a snapshot (too short)");
  SnapHeader h;
  std::memcpy(&h, host, sizeof h);
  if (std::memcmp(h.magic, "RLTSNAP1", 8) != 0 || h.header_bytes != sizeof(SnapHeader))
    return fail(RLT_E_INVAL, "not a snapshot of this format");
  rlt_model* m = S->m;
  const rlt_config& c = m->cfg;
  if (h.d_model != c.d_model || h.n_heads != c.n_heads || h.n_layers != c.n_layers || h.window != c.window ||
      h.groups != c.groups || h.ffn != c.ffn || h.vocab != c.vocab || h.tied != c.tied ||
      h.merge_kind != c.merge_kind || h.dtype != c.dtype || h.bos_id != c.bos_id || h.alpha != c.alpha ||
      h.rms_eps != c.rms_eps || h.rope_base != c.rope_base)
    return fail(RLT_E_INVAL, "snapshot of a model with another configuration");
  if (h.weight_seed != m->seed || h.model_version != m->version)
    return fail(RLT_E_STALE, "snapshot was taken under other weights");
  if (h.batch != S->B) return fail(RLT_E_INVAL, "snapshot batch differs from the state's");
  if (h.n_enc < 0 || h.n_dec < 0 || h.n_dec > h.n_enc) return fail(RLT_E_INVAL, "bad positions in snapshot");
  if (h.n_enc > S->max_len) return fail(RLT_E_CAPACITY, "snapshot positions exceed the state's max_len");
  const bool want_cache = (S->flags & RLT_STATE_ENCODER_CACHE) && h.n_enc > 0;
  if (want_cache && !(h.flags & kSnapCache))
    return fail(RLT_E_STATE, "the state keeps an encoder cache but the snapshot has none");
  if (c.dtype == RLT_DTYPE_BF16 && h.n_dec > 0 && !(h.flags & kSnapFold))
    return fail(RLT_E_INVAL, "snapshot lacks the readout operand");
  const std::vector<SnapSection> secs = snapshot_sections(S, h.n_enc, h.flags);
  if (h.payload_bytes != payload_bytes(secs) || bytes < sizeof(SnapHeader) + h.payload_bytes)
    return fail(RLT_E_INVAL, "snapshot payload size mismatch");
  // per-sequence positions: the ragged section (the payload's last), else
  // every sequence at the header's positions
  std::vector<int32_t> enc(S->B, h.n_enc), dec(S->B, h.n_dec);
  if (h.flags & kSnapRagged) {
    const uint8_t* pp = static_cast<const uint8_t*>(host) + sizeof h + h.payload_bytes - (size_t)2 * S->B * 4;
    std::memcpy(enc.data(), pp, (size_t)S->B * 4);
    std::memcpy(dec.data(), pp + (size_t)S->B * 4, (size_t)S->B * 4);
    for (int b = 0; b < S->B; ++b)
      if (dec[b] < 0 || dec[b] > enc[b] || enc[b] > h.n_enc) return fail(RLT_E_INVAL, "bad positions in snapshot");
  }
  RLT_CUDA(cudaSetDevice(m->device));
  cudaStream_t st = (cudaStream_t)stream;
  const uint8_t* src = static_cast<const uint8_t*>(host) + sizeof h;
  const bool has_cache_here = (S->flags & RLT_STATE_ENCODER_CACHE) != 0;
  for (const auto& x : secs) {
    const bool cache_sec = x.dev == S->ce_k || x.dev == S->ce_v;
    if (!(cache_sec && !has_cache_here))  // a state without the cache drops those sections
      RLT_CUDA(cudaMemcpy2DAsync(x.dev, x.pitch, src, x.width, x.width, x.rows, cudaMemcpyHostToDevice, st));
    src += x.width * x.rows;
  }
  if (!(h.flags & kSnapRagged)) {
    RLT_CUDA(set_positions(S->pos, 0, S->B, h.n_enc, st));
    RLT_CUDA(set_positions(S->pos + S->B, 0, S->B, h.n_dec, st));
  }
  RLT_CUDA(cudaStreamSynchronize(st));
  S->enc_h = enc;
  S->dec_h = dec;
  S->has_pending = (h.flags & kSnapPending) != 0;
  S->version = m->version;
  return ok();
}

int32_t rlt_encode_prefix(rlt_model* m, rlt_state* s, const int32_t* tok_dev, int32_t T, void* stream) {
  RLT_TRY(check_state(m, s));
  if (!tok_dev || T <= 0) return fail(RLT_E_INVAL, "need tokens and T > 0");
  if (!uniform(s->enc_h))
    return fail(RLT_E_STATE, "the sequences have encoded different numbers of tokens: use rlt_append_spans");
  const int p0 = s->enc_h[0];
  if (p0 != 0 && !(s->flags & RLT_STATE_ENCODER_CACHE))
    return fail(RLT_E_STATE, "continuing an encoded prefix needs the encoder cache");
  if ((int64_t)p0 + T > s->max_len) return fail(RLT_E_CAPACITY, "n_enc + T exceeds max_len");
  return RLT_DISPATCH(m, encode_prefix_impl, m, s, tok_dev, (int64_t)T, T, 0, s->B, p0, (cudaStream_t)stream);
}

int32_t rlt_append_spans(rlt_model* m, rlt_state* s, const int32_t* tok_dev, int64_t ld_tok, const int32_t* lens,
                         float* logp_dev, int64_t ld_logp, void* stream) {
  RLT_TRY(check_state(m, s));
  if (!tok_dev || !lens) return fail(RLT_E_INVAL, "null tokens or lengths");
  int max_len_span = 0;
  for (int b = 0; b < s->B; ++b) {
    if (lens[b] < 0) return fail(RLT_E_INVAL, "negative span length");
    max_len_span = std::max(max_len_span, (int)lens[b]);
  }
  if (max_len_span == 0) return fail(RLT_E_INVAL, "every span is empty");
  if (ld_tok < max_len_span) return fail(RLT_E_INVAL, "ld_tok is shorter than the longest span");
  if (logp_dev && ld_logp < max_len_span - 1) return fail(RLT_E_INVAL, "ld_logp is shorter than the longest span - 1");
  if (s->has_pending) return fail(RLT_E_STATE, "a sampled token is pending: consume it with rlt_decoder_step first");
  for (int b = 0; b < s->B; ++b) {
    if (s->enc_h[b] != s->dec_h[b])
      return fail(RLT_E_STATE, "sequence " + std::to_string(b) + " has encoded tokens not yet consumed");
    if ((int64_t)s->enc_h[b] + lens[b] > s->max_len)
      return fail(RLT_E_CAPACITY, "sequence " + std::to_string(b) + ": n_enc + span exceeds max_len");
    if (lens[b] > 0 && s->enc_h[b] > 0 && !(s->flags & RLT_STATE_ENCODER_CACHE))
      return fail(RLT_E_STATE, "appending to an encoded prefix needs the encoder cache");
  }
  cudaStream_t st = (cudaStream_t)stream;
  // token-parallel encoding of each run of consecutive sequences with the
  // same position and span length (App. A.2, chunked encoder)
  for (int b0 = 0; b0 < s->B;) {
    int b1 = b0 + 1;
    while (b1 < s->B && lens[b1] == lens[b0] && s->enc_h[b1] == s->enc_h[b0]) ++b1;
    if (lens[b0] > 0)
      RLT_TRY(RLT_DISPATCH(m, encode_prefix_impl, m, s, tok_dev, ld_tok, (int32_t)lens[b0], b0, b1, s->enc_h[b0], st));
    b0 = b1;
  }
  // then every span token gets its transition, in lock step; a sequence
  // whose span is over sits out the remaining transitions (masked phase)
  for (int b = 0; b < s->B; ++b) s->lim_h[b] = s->dec_h[b] + lens[b];
  RLT_CUDA(cudaMemcpyAsync(s->pos + 2 * s->B, s->lim_h.data(), (size_t)s->B * 4, cudaMemcpyHostToDevice, st));
  for (int k = 1; k <= max_len_span; ++k) {
    StepRange range(m, max_of(s->dec_h) + 1);
    RLT_TRY(RLT_DISPATCH(m, transition_impl, m, s, true, false, st));
    advance_host(s, true);
    if (logp_dev && k < max_len_span)
      RLT_TRY(RLT_DISPATCH(m, readout_impl, m, s, tok_dev + k, ld_tok, logp_dev + (k - 1), ld_logp,
                           (const rlt_sampling*)nullptr, (const rlt_readout_out*)nullptr, true, st));
  }
  return ok();
}

int32_t rlt_readout(rlt_model* m, rlt_state* s, const int32_t* next_dev, const rlt_sampling* samp,
                    const rlt_readout_out* out, void* stream) {
  RLT_TRY(check_state(m, s));
  if (*std::min_element(s->dec_h.begin(), s->dec_h.end()) < 1)
    return fail(RLT_E_STATE, "readout needs at least one transition of every sequence");
  RLT_TRY(check_sampling(samp, out));
  return RLT_DISPATCH(m, readout_impl, m, s, next_dev, (int64_t)1, out ? out->logp : nullptr, (int64_t)1, samp, out,
                      false, (cudaStream_t)stream);
}

int32_t rlt_decoder_step(rlt_model* m, rlt_state* s, const int32_t* tok_dev, const int32_t* next_dev,
                         const rlt_sampling* samp, const rlt_readout_out* out, void* stream) {
  RLT_TRY(check_state(m, s));
  RLT_TRY(check_sampling(samp, out));
  // every sequence takes its transition at its own t_b = n_dec[b] + 1; the
  // ones whose x_t is not yet encoded run the encoder step first
  int t_max = 0;
  bool any_enc = false, all_enc = true;
  for (int b = 0; b < s->B; ++b) {
    const int t = s->dec_h[b] + 1;
    t_max = std::max(t_max, t);
    if (s->enc_h[b] < t) any_enc = true;
    else all_enc = false;
  }
  if (t_max > s->max_len) return fail(RLT_E_CAPACITY, "position would pass max_len");
  cudaStream_t st = (cudaStream_t)stream;
  StepRange range(m, t_max);
  if (any_enc) {
    if (!(s->flags & RLT_STATE_ENCODER_CACHE)) return fail(RLT_E_STATE, "x_t not encoded and the state has no encoder cache");
    if (!tok_dev && !s->has_pending)
      return fail(RLT_E_STATE, "x_t must be given: it is not yet encoded and no sampled token is pending");
  }
  const int32_t* tok_src = any_enc ? (tok_dev ? tok_dev : s->pending) : nullptr;
  RLT_TRY(step_launch(m, s, tok_src, any_enc, all_enc, st));
  advance_host(s, false);
  s->has_pending = false;
  if (next_dev || samp || (out && out->logits))
    RLT_TRY(RLT_DISPATCH(m, readout_impl, m, s, next_dev, (int64_t)1, out ? out->logp : nullptr, (int64_t)1, samp, out,
                         false, st));
  return ok();
}

int32_t rlt_prefill(rlt_model* m, rlt_state* s, const int32_t* tok_dev, int32_t T, float* logp_dev, void* stream) {
  RLT_TRY(check_state(m, s));
  if (!tok_dev || T <= 0) return fail(RLT_E_INVAL, "need tokens and T > 0");
  if (max_of(s->enc_h) != 0 || max_of(s->dec_h) != 0) return fail(RLT_E_STATE, "prefill starts from H_0");
  if (T > s->max_len) return fail(RLT_E_CAPACITY, "T exceeds max_len");
  cudaStream_t st = (cudaStream_t)stream;
  RLT_TRY(RLT_DISPATCH(m, encode_prefix_impl, m, s, tok_dev, (int64_t)T, T, 0, s->B, 0, st));
  for (int t = 1; t <= T; ++t) {
    StepRange range(m, t);
    RLT_TRY(step_launch(m, s, nullptr, false, false, st));
    advance_host(s, false);
    if (logp_dev && t < T)
      RLT_TRY(RLT_DISPATCH(m, readout_impl, m, s, tok_dev + t, (int64_t)T, logp_dev + (t - 1), (int64_t)(T - 1),
                           (const rlt_sampling*)nullptr, (const rlt_readout_out*)nullptr, false, st));
  }
  return ok();
}

int32_t rlt_replay_logprobs(rlt_model* m, const int32_t* tok_dev, int32_t B, int32_t S, float* logp_dev, void* stream) {
  if (!m || !tok_dev || !logp_dev) return fail(RLT_E_INVAL, "null argument");
  if (B <= 0 || S < 2) return fail(RLT_E_INVAL, "need B > 0 and S >= 2");
  RLT_CUDA(cudaSetDevice(m->device));
  if (m->replay && (m->replay->B != B || m->replay->max_len < S)) {
    rlt_state_free(m->replay);
    m->replay = nullptr;
  }
  if (!m->replay) RLT_TRY(make_state(m, B, S, RLT_STATE_GRAPHS, &m->replay));
  rlt_state* st_ = m->replay;
  cudaStream_t st = (cudaStream_t)stream;
  RLT_TRY(RLT_DISPATCH(m, reset_state, st_, st));
  RLT_TRY(RLT_DISPATCH(m, encode_prefix_impl, m, st_, tok_dev, (int64_t)S, S, 0, B, 0, st));
  for (int t = 1; t <= S - 1; ++t) {
    StepRange range(m, t);
    RLT_TRY(step_launch(m, st_, nullptr, false, false, st));
    advance_host(st_, false);
    RLT_TRY(RLT_DISPATCH(m, readout_impl, m, st_, tok_dev + t, (int64_t)S, logp_dev + (t - 1), (int64_t)(S - 1),
                         (const rlt_sampling*)nullptr, (const rlt_readout_out*)nullptr, false, st));
  }
  return ok();
}

int32_t rlt_replay_ratios(rlt_model* m, const int32_t* tok_dev, int32_t B, int32_t S, const float* logmu_dev,
                          const uint8_t* action_mask_dev, float* logp_dev, float* ratio_dev, float* seq_logratio_dev,
                          void* stream) {
  if (!logmu_dev || !action_mask_dev) return fail(RLT_E_INVAL, "null behaviour log-probs or action mask");
  if (!ratio_dev && !seq_logratio_dev) return fail(RLT_E_INVAL, "no ratio output requested");
  RLT_TRY(rlt_replay_logprobs(m, tok_dev, B, S, logp_dev, stream));
  RLT_CUDA(replay_ratios(logp_dev, logmu_dev, action_mask_dev, B, S - 1, ratio_dev, seq_logratio_dev,
                         (cudaStream_t)stream));
  return ok();
}

int32_t rlt_op_linear(const void* w_dev, const void* x_dev, float* y_dev, int32_t M, int32_t N, int32_t K,
                      int32_t dtype, int32_t use_tensor_cores, void* stream) {
  if (!w_dev || !x_dev || !y_dev || M <= 0 || N <= 0 || K <= 0) return fail(RLT_E_INVAL, "bad linear arguments");
  cudaStream_t st = (cudaStream_t)stream;
  const EpiParams ep = epi_out(y_dev, plain_rows(M), 0);
  if (dtype == RLT_DTYPE_F32) {
    if (use_tensor_cores) return fail(RLT_E_INVAL, "the tensor-core path takes bf16 operands");
    RLT_CUDA(gemm_simt<float, float>(static_cast<const float*>(w_dev), K, static_cast<const float*>(x_dev), K, M, N, K,
                                     EPI_STORE, ep, st));
    return ok();
  }
  if (dtype != RLT_DTYPE_BF16) return fail(RLT_E_INVAL, "dtype");
  if (!use_tensor_cores) {
    RLT_CUDA(gemm_simt<bf16, bf16>(static_cast<const bf16*>(w_dev), K, static_cast<const bf16*>(x_dev), K, M, N, K,
                                   EPI_STORE, ep, st));
    return ok();
  }
  if (M % 128 || K % 64) return fail(RLT_E_INVAL, "tensor-core path needs M % 128 == 0 and K % 64 == 0");
  const size_t ws_floats = gemm_tc_workspace_floats(M, N, K, 1);
  float* ws = nullptr;
  if (ws_floats > 0) {
    RLT_CUDA(cudaMallocAsync(reinterpret_cast<void**>(&ws), ws_floats * 4, st));
  }
  cudaError_t e = gemm_tc(static_cast<const bf16*>(w_dev), K, static_cast<const bf16*>(x_dev), K, M, N, K, EPI_STORE,
                          ep, 1, ws, ws_floats, st);
  if (ws) cudaFreeAsync(ws, st);
  if (e != cudaSuccess) return fail(RLT_E_CUDA, std::string("gemm_tc: ") + cudaGetErrorString(e));
  return ok();
}

int32_t rlt_op_prefix_attention(const float* q_dev, const void* k_dev, const void* v_dev, int64_t ld_t, int32_t B,
                                int32_t H, int32_t hd, int32_t n, int32_t dtype, const float* rope_cs_dev,
                                int32_t qpos, void* out_dev, void* stream) {
  if (!q_dev || !k_dev || !v_dev || !out_dev || B <= 0 || H <= 0 || n <= 0 || ld_t < n || qpos < 0)
    return fail(RLT_E_INVAL, "bad prefix attention arguments");
  if (!(hd == 16 || hd == 32 || hd == 64 || hd == 128 || hd == 256)) return fail(RLT_E_INVAL, "head size");
  if (dtype != RLT_DTYPE_F32 && dtype != RLT_DTYPE_BF16) return fail(RLT_E_INVAL, "dtype");
  cudaStream_t st = (cudaStream_t)stream;
  const size_t wsf = prefix_attn_workspace_floats(B, H, hd, n);
  float* ws = nullptr;
  if (wsf && cudaMalloc(&ws, wsf * sizeof(float)) != cudaSuccess) {
    cudaGetLastError();
    return fail(RLT_E_OOM, "prefix attention scratch");
  }
  cudaError_t e;
  if (dtype == RLT_DTYPE_BF16)
    e = prefix_attn<bf16>(q_dev, (int64_t)H * hd, static_cast<const bf16*>(k_dev), static_cast<const bf16*>(v_dev), ld_t,
                          B, H, hd, n, qpos, no_pos(), rope_cs_dev, static_cast<bf16*>(out_dev), (int64_t)H * hd, ws,
                          wsf, nullptr, st);
  else
    e = prefix_attn<float>(q_dev, (int64_t)H * hd, static_cast<const float*>(k_dev), static_cast<const float*>(v_dev),
                           ld_t, B, H, hd, n, qpos, no_pos(), rope_cs_dev, static_cast<float*>(out_dev),
                           (int64_t)H * hd, ws, wsf, nullptr, st);
  if (ws) {
    cudaStreamSynchronize(st);
    cudaFree(ws);
  }
  if (e != cudaSuccess) return fail(RLT_E_CUDA, std::string("prefix attention: ") + cudaGetErrorString(e));
  return ok();
}

int32_t rlt_op_sample(const float* logits_dev, int32_t B, int32_t V, const rlt_sampling* samp, uint32_t t,
                      int32_t* token_dev, float* logp_dev, float* logmu_dev, void* stream) {
  if (!logits_dev || !samp || !token_dev || B <= 0 || V <= 0) return fail(RLT_E_INVAL, "bad sample arguments");
  if (!(samp->temperature > 0.f) || samp->top_k < 1 || samp->top_k > 256)
    return fail(RLT_E_INVAL, "sampler needs temperature > 0 and 1 <= top_k <= 256");
  RLT_CUDA(sample_topk(logits_dev, B, V, samp->temperature, samp->top_k, samp->seed, t, nullptr, token_dev, logp_dev,
                       logmu_dev, (cudaStream_t)stream));
  return ok();
}

// ------------------------------------------------------------------ gradients
}  // extern "C"

namespace {

bptt::Dims bptt_dims(const rlt_model* m, int B, int S) {
  const rlt_config& c = m->cfg;
  bptt::Dims D{};
  D.B = B; D.S = S; D.d = c.d_model; D.H = c.n_heads; D.L = c.n_layers; D.W = c.window; D.G = c.groups;
  D.F = c.ffn; D.V = c.vocab; D.tied = c.tied; D.merge_kind = c.merge_kind;
  D.alpha = c.alpha; D.eps = c.rms_eps; D.rope_base = c.rope_base;
  return D;
}

// The model's view of catalogue index i (null when the model does not store it).
const View* bptt_view(const rlt_model* m, const bptt::Dims& D, int i) {
  if (!bptt::tensor_exists(D, i)) return nullptr;
  auto it = m->views.find(bptt::tensor_name(D, i));
  return it == m->views.end() ? nullptr : &it->second;
}

// Frees what rlt_replay_backward keeps (after its work has drained).
void release_backward(rlt_model* m) {
  BackwardHold* h = m->bwd;
  if (!h) return;
  m->bwd = nullptr;
  if (h->runner) bptt::runner_free(h->runner);
  cudaDeviceSynchronize();
  free_all(h->allocs);
  delete h;
}

// The prologue of every backward pass: the fp32 copies of the current weights.
cudaError_t widen_weights(void* ctx, cudaStream_t st) {
  const BackwardHold* h = static_cast<const BackwardHold*>(ctx);
  for (size_t i = 0; i < h->w32.size(); ++i) {
    const View* v = h->views[i];
    if (!v) continue;
    const cudaError_t e = bptt::widen_to_f32(v->base, h->dtype, v->rows, v->cols, v->pitch, h->w32[i], st);
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

// Allocates the model's gradient buffers on first use and zeroes them on the
// caller's stream `st`, so the zeroing is ordered before the backward that
// accumulates into them on the same stream.  The buffers join the model's
// allocations only once all exist; a failure part-way frees those already
// made, so a retry starts clean.
int32_t ensure_grads(rlt_model* m, const bptt::Dims& D, cudaStream_t st) {
  if (!m->grad.empty()) return RLT_OK;
  const int n = bptt::n_tensors(D);
  std::vector<float*> g(n, nullptr);
  std::vector<void*> made;
  int32_t r = RLT_OK;
  for (int i = 0; i < n && r == RLT_OK; ++i) {
    const View* v = bptt_view(m, D, i);
    if (!v) continue;
    void* p = nullptr;
    r = dev_alloc(made, &p, (size_t)(v->rows * v->cols) * 4);
    if (r != RLT_OK) break;
    const cudaError_t e = cudaMemsetAsync(p, 0, (size_t)(v->rows * v->cols) * 4, st);
    if (e != cudaSuccess) r = fail(RLT_E_CUDA, std::string("zeroing a gradient: ") + cudaGetErrorString(e));
    g[i] = static_cast<float*>(p);
  }
  if (r != RLT_OK) {
    cudaStreamSynchronize(st);
    free_all(made);
    return r;
  }
  m->allocs.insert(m->allocs.end(), made.begin(), made.end());
  m->grad = g;
  return RLT_OK;
}

}  // namespace

extern "C" {

int32_t rlt_replay_backward(rlt_model* m, const int32_t* tok_dev, int32_t B, int32_t S, const float* w_dev,
                            int32_t segment, float* logp_dev, void* stream) {
  if (!m || !tok_dev || !w_dev) return fail(RLT_E_INVAL, "null argument");
  if (B <= 0 || S < 2) return fail(RLT_E_INVAL, "need B > 0 and S >= 2");
  if (segment < 1) return fail(RLT_E_INVAL, "segment must be at least 1");
  if (m->hd > bptt::kMaxHead) return fail(RLT_E_INVAL, "the backward pass takes head sizes up to 128");
  RLT_CUDA(cudaSetDevice(m->device));
  cudaStream_t st = (cudaStream_t)stream;
  {  // the engine indexes the embedding and the targets by these ids: check them first
    std::vector<int32_t> ids((size_t)B * S);
    RLT_CUDA(cudaMemcpyAsync(ids.data(), tok_dev, ids.size() * 4, cudaMemcpyDeviceToHost, st));
    RLT_CUDA(cudaStreamSynchronize(st));
    for (int32_t v : ids)
      if (v < 0 || v >= m->cfg.vocab) return fail(RLT_E_INVAL, "token id " + std::to_string(v) + " out of range");
  }
  const bptt::Dims D = bptt_dims(m, B, S);
  const int seg = std::min(segment, S - 1);
  RLT_TRY(ensure_grads(m, D, st));
  if (m->bwd && (m->bwd->B != B || m->bwd->S != S || m->bwd->seg != seg)) release_backward(m);
  if (!m->bwd) {
    BackwardHold* h = new BackwardHold();
    h->B = B;
    h->S = S;
    h->seg = seg;
    h->dtype = m->cfg.dtype;
    const int n = bptt::n_tensors(D);
    h->w32.assign(n, nullptr);
    h->views.assign(n, nullptr);
    int32_t r = RLT_OK;
    for (int i = 0; i < n && r == RLT_OK; ++i) {
      const View* v = bptt_view(m, D, i);
      if (!v) continue;
      void* p = nullptr;
      r = dev_alloc(h->allocs, &p, (size_t)(v->rows * v->cols) * 4);
      h->views[i] = v;
      h->w32[i] = static_cast<float*>(p);
    }
    if (r == RLT_OK) {
      const cudaError_t e = bptt::runner_create(D, seg, m->cfg.dtype == RLT_DTYPE_BF16, h->w32.data(),
                                                m->grad.data(), &h->runner);
      if (e == cudaErrorMemoryAllocation) r = fail(RLT_E_OOM, "backward buffers: out of device memory");
      else if (e != cudaSuccess) r = fail(RLT_E_CUDA, std::string("backward setup: ") + cudaGetErrorString(e));
    }
    if (r != RLT_OK) {
      free_all(h->allocs);
      delete h;
      return r;
    }
    m->bwd = h;
  }
  const cudaError_t e = bptt::runner_run(m->bwd->runner, widen_weights, m->bwd, tok_dev, w_dev, logp_dev, st);
  if (e != cudaSuccess) {
    cudaGetLastError();
    release_backward(m);
    if (e == cudaErrorMemoryAllocation) return fail(RLT_E_OOM, "backward buffers: out of device memory");
    return fail(RLT_E_CUDA, std::string("backward: ") + cudaGetErrorString(e));
  }
  return ok();
}

int32_t rlt_backward_release(rlt_model* m) {
  if (!m) return fail(RLT_E_INVAL, "null argument");
  RLT_CUDA(cudaSetDevice(m->device));
  release_backward(m);
  return ok();
}

int32_t rlt_grad_read(const rlt_model* m, const char* name, float* host, size_t bytes) {
  if (!m || !name || !host) return fail(RLT_E_INVAL, "null argument");
  auto it = m->views.find(name);
  if (it == m->views.end()) return fail(RLT_E_INVAL, std::string("unknown tensor ") + name);
  const View& v = it->second;
  const size_t need = (size_t)(v.rows * v.cols) * 4;
  if (bytes != need) return fail(RLT_E_INVAL, "size mismatch: need " + std::to_string(need));
  if (m->grad.empty()) {
    std::memset(host, 0, bytes);
    return ok();
  }
  const bptt::Dims D = bptt_dims(m, 1, 2);
  for (int i = 0; i < bptt::n_tensors(D); ++i) {
    if (!bptt::tensor_exists(D, i) || bptt::tensor_name(D, i) != name) continue;
    RLT_CUDA(cudaSetDevice(m->device));
    RLT_CUDA(cudaDeviceSynchronize());
    RLT_CUDA(cudaMemcpy(host, m->grad[i], bytes, cudaMemcpyDeviceToHost));
    return ok();
  }
  return fail(RLT_E_INVAL, std::string("no gradient for ") + name);
}

int32_t rlt_grad_zero(rlt_model* m, void* stream) {
  if (!m) return fail(RLT_E_INVAL, "null model");
  if (m->grad.empty()) return ok();
  RLT_CUDA(cudaSetDevice(m->device));
  const bptt::Dims D = bptt_dims(m, 1, 2);
  for (int i = 0; i < bptt::n_tensors(D); ++i) {
    const View* v = bptt_view(m, D, i);
    if (v && m->grad[i])
      RLT_CUDA(cudaMemsetAsync(m->grad[i], 0, (size_t)(v->rows * v->cols) * 4, (cudaStream_t)stream));
  }
  return ok();
}

int32_t rlt_last_error(char* buf, size_t n) {
  if (buf && n) {
    std::strncpy(buf, t_err.c_str(), n - 1);
    buf[n - 1] = 0;
  }
  return t_err_code;
}

int32_t rlt_check_device(void) {
  RLT_CUDA(cudaDeviceSynchronize());
  int v = 0;
  RLT_CUDA(cudaMemcpyFromSymbol(&v, rlt::g_device_error, sizeof(int)));
  if (v) {
    int z = 0;
    RLT_CUDA(cudaMemcpyToSymbol(rlt::g_device_error, &z, sizeof(int)));
    return fail(RLT_E_CUDA, v == 1 ? "a bounded device wait ran out" : "a token id was out of range");
  }
  return ok();
}

int32_t rlt_test_bounded_wait(uint32_t limit_us, uint64_t* waited_ns, void* stream) {
  if (!waited_ns || limit_us < 1 || limit_us > 1000000u) return fail(RLT_E_INVAL, "limit_us must be in 1..1000000");
  RLT_CUDA(bounded_wait_probe((uint64_t)limit_us * 1000ull, waited_ns, (cudaStream_t)stream));
  return ok();
}

int32_t rlt_kernel_launches(int64_t* count) {
  if (!count) return fail(RLT_E_INVAL, "null argument");
  *count = launch_count();
  return ok();
}

int32_t rlt_profile_enable(rlt_model* m, int32_t on) {
  if (!m) return fail(RLT_E_INVAL, "null model");
  m->prof.on = on != 0;
  m->prof.used = 0;
  m->prof.kind.clear();
  m->prof.bytes[0] = m->prof.bytes[1] = 0;
  m->prof.launches[0] = m->prof.launches[1] = 0;
  return ok();
}

int32_t rlt_profile_read(rlt_model* m, int32_t kind, double* ms, int64_t* launches, double* bytes) {
  if (!m || kind < 0 || kind > 1) return fail(RLT_E_INVAL, "bad argument");
  RLT_CUDA(cudaSetDevice(m->device));
  RLT_CUDA(cudaDeviceSynchronize());
  double total = 0;
  for (size_t i = 0; i + 1 < m->prof.used; i += 2) {
    if (m->prof.kind[i / 2] != kind) continue;
    float x = 0;
    RLT_CUDA(cudaEventElapsedTime(&x, m->prof.ev[i], m->prof.ev[i + 1]));
    total += x;
  }
  if (ms) *ms = total;
  if (launches) *launches = m->prof.launches[kind];
  if (bytes) *bytes = m->prof.bytes[kind];
  return ok();
}

}  // extern "C"

// ====================================================================== no-alloc variant
// rlt_op_prefix_attention_noalloc: the split-key attention with its chunk
// partials in a static device array instead of memory allocated per call (for
// callers that own all device memory or cannot take an allocation's implicit
// synchronisation).  The array is 16 MiB; host code must not use its name as
// a device pointer (in host code it is only a stand-in), so the device
// address is looked up per device with cudaGetSymbolAddress.
namespace {
constexpr size_t kNoallocScratchFloats = (size_t)4 << 20;  // 16 MiB
static __device__ __align__(256) float g_noalloc_scratch[kNoallocScratchFloats];

std::mutex g_noalloc_mu;
std::map<int, float*> g_noalloc_ptr;  // device ordinal -> device address of the array

int32_t noalloc_scratch(float** out) {
  int dev = 0;
  RLT_CUDA(cudaGetDevice(&dev));
  std::lock_guard<std::mutex> g(g_noalloc_mu);
  auto it = g_noalloc_ptr.find(dev);
  if (it == g_noalloc_ptr.end()) {
    void* p = nullptr;
    RLT_CUDA(cudaGetSymbolAddress(&p, g_noalloc_scratch));
    it = g_noalloc_ptr.emplace(dev, static_cast<float*>(p)).first;
  }
  *out = it->second;
  return RLT_OK;
}
}  // namespace

extern "C" int32_t rlt_op_prefix_attention_noalloc(const float* q_dev, const void* k_dev, const void* v_dev,
                                                   int64_t ld_t, int32_t B, int32_t H, int32_t hd, int32_t n,
                                                   int32_t dtype, const float* rope_cs_dev, int32_t qpos,
                                                   void* out_dev, void* stream) {
  if (!q_dev || !k_dev || !v_dev || !out_dev || B <= 0 || H <= 0 || n <= 0 || ld_t < n || qpos < 0)
    return fail(RLT_E_INVAL, "bad prefix attention arguments");
  if (!(hd == 16 || hd == 32 || hd == 64 || hd == 128 || hd == 256)) return fail(RLT_E_INVAL, "head size");
  if (dtype != RLT_DTYPE_F32 && dtype != RLT_DTYPE_BF16) return fail(RLT_E_INVAL, "dtype");
  const size_t need = prefix_attn_workspace_floats(B, H, hd, n);
  if (need > kNoallocScratchFloats)
    return fail(RLT_E_CAPACITY, "prefix attention needs " + std::to_string(need) +
                                    " floats of scratch; the static scratch array holds " +
                                    std::to_string(kNoallocScratchFloats));
  float* ws = nullptr;
  if (need) RLT_TRY(noalloc_scratch(&ws));
  cudaStream_t st = (cudaStream_t)stream;
  cudaError_t e;
  if (dtype == RLT_DTYPE_BF16)
    e = prefix_attn<bf16>(q_dev, (int64_t)H * hd, static_cast<const bf16*>(k_dev), static_cast<const bf16*>(v_dev), ld_t,
                          B, H, hd, n, qpos, no_pos(), rope_cs_dev, static_cast<bf16*>(out_dev), (int64_t)H * hd, ws,
                          kNoallocScratchFloats, nullptr, st);
  else
    e = prefix_attn<float>(q_dev, (int64_t)H * hd, static_cast<const float*>(k_dev), static_cast<const float*>(v_dev),
                           ld_t, B, H, hd, n, qpos, no_pos(), rope_cs_dev, static_cast<float*>(out_dev),
                           (int64_t)H * hd, ws, kNoallocScratchFloats, nullptr, st);
  if (e != cudaSuccess) return fail(RLT_E_CUDA, std::string("prefix attention: ") + cudaGetErrorString(e));
  return ok();
}
