/*
 * rlt_oracle.c -- plain fp64 CPU oracle for the Recurrent Looped Transformer
 * (RLT) hot path: causal encoder, encoder KV memory, gated merge, recurrent
 * decoder transition with a sliding-window (SWA) cache, readout and the
 * behaviour sampler.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may load, link or
 * call this file: only the tests, the smoke check and the CPU-baseline leg of
 * the benchmark use it.  It shares no code, header or table with the CUDA
 * library; the only thing both sides consume is the seeded input generator
 * (tokens) and the published Philox4x32-10 definition, which each side
 * implements on its own.
 *
 * Sources (all from "Recurrent Looped Transformer", Y. Zhang, technical
 * report, Sept. 2026, and its project page):
 *   report §2.1  sequence/state definitions, window W includes current token
 *   report §2.2  eq. 2.1 causal encoder, eq. 2.2 memory groups
 *   report §2.3  eqs. 2.3-2.7 H_0, Merge, D_phi, readout
 *   report §2.4  eq. 2.8 encoder step form; prefix-restricted memory
 *   report §2.5  eqs. 2.9-2.11 gated merge; eqs. 2.12-2.16 decoder block;
 *                cache retention max(1,t-W+2)..t
 *   report §2.6  tied configuration
 *   report §5.3  behaviour log-probabilities under the actual sampler;
 *                eq. 5.5 replay ratios
 *   report App. A.1/A.2/A.4 execution schedules (prefill, generation, replay)
 *   project page, "The complete state matters" (clean forms of 2.3/2.5/2.6)
 *
 * Readings taken where the pages leave a step open (each listed in the
 * design notes): FFN = SwiGLU; positional map = rotate-half RoPE at
 * p = t-1, base 10000, on queries/keys only; one pre-norm RMSNorm per
 * sublayer; no final encoder norm; MHA with 1/sqrt(hd) scaling; no biases
 * except b_g; merge either the report's eqs. 2.9-2.11 (kind 0) or the convex
 * form g*e+(1-g)*s with g = sigmoid(W_g[e;s]) (kind 1).
 *
 * Everything is evaluated in double precision.  Weights are stored in the
 * precision the model is configured for (fp32 or bf16 bit patterns) and
 * converted exactly to double when read, so the oracle sees exactly the
 * weights the device sees and parity measures compute error only.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* ------------------------------------------------------------------------ */
/* configuration                                                             */
/* ------------------------------------------------------------------------ */

typedef struct {
  int32_t d, n_heads, n_layers, window, groups, ffn, vocab;
  int32_t tied;       /* 1: decoder reuses encoder attention+FFN weights (§2.6) */
  int32_t merge_kind; /* 0: eqs. 2.9-2.11; 1: convex gate */
  int32_t dtype;      /* storage of weights: 0 fp32, 1 bf16 */
  double alpha, rms_eps, rope_base, init_std;
  int32_t bos_id;
} orc_config;

/* ------------------------------------------------------------------------ */
/* Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as   */
/* easy as 1, 2, 3", SC'11): 10 rounds of the 4x32 Philox S-box with the     */
/* Weyl key schedule.                                                         */
/* ------------------------------------------------------------------------ */

void orc_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4]) {
  const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
  const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
  uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
  uint32_t k0 = key_in[0], k1 = key_in[1];
  for (int r = 0; r < 10; ++r) {
    if (r > 0) { k0 += W0; k1 += W1; }
    uint64_t p0 = (uint64_t)M0 * c0;
    uint64_t p1 = (uint64_t)M1 * c2;
    uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    uint32_t n0 = hi1 ^ c1 ^ k0;
    uint32_t n1 = lo1;
    uint32_t n2 = hi0 ^ c3 ^ k1;
    uint32_t n3 = lo0;
    c0 = n0; c1 = n1; c2 = n2; c3 = n3;
  }
  out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* Standard-normal draw used for weight initialisation: the Irwin-Hall sum of
 * twelve uniforms on [0,1) minus 6 (mean 0, variance 1).  The twelve 32-bit
 * words come from three Philox blocks with counter (idx_lo, idx_hi, tensor,
 * j), j = 0,1,2, and key = seed.  The sum is an exact integer, so the value
 * is reproducible bit for bit without any transcendental function. */
double orc_normal_ih12(uint64_t seed, uint32_t tensor_id, uint64_t idx) {
  uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
  uint64_t sum = 0;
  for (uint32_t j = 0; j < 3; ++j) {
    uint32_t ctr[4] = {(uint32_t)idx, (uint32_t)(idx >> 32), tensor_id, j};
    uint32_t o[4];
    orc_philox4x32_10(ctr, key, o);
    sum += (uint64_t)o[0] + o[1] + o[2] + o[3];
  }
  return (double)sum * (1.0 / 4294967296.0) - 6.0;
}

/* ------------------------------------------------------------------------ */
/* weight storage                                                            */
/* ------------------------------------------------------------------------ */

static float bf16_bits_to_float(uint16_t b) {
  uint32_t u = (uint32_t)b << 16;
  float f;
  memcpy(&f, &u, 4);
  return f;
}

/* round-to-nearest-even float -> bf16 (NaN is not produced by the generator) */
static uint16_t float_to_bf16_bits(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7FFFu + lsb;
  return (uint16_t)(u >> 16);
}

typedef struct {
  char name[32];
  int32_t id;      /* generator stream id */
  int32_t kind;    /* 0 random matrix/vector, 1 gain (ones), 2 zeros */
  int64_t rows, cols;
  void *data;      /* float or uint16 (bf16 bits) */
} orc_tensor;

typedef struct {
  orc_config cfg;
  int32_t n_tensors;
  orc_tensor *t;
} orc_model;

static inline double tw(const orc_model *m, const orc_tensor *t, int64_t i) {
  if (m->cfg.dtype == 0) return (double)((const float *)t->data)[i];
  return (double)bf16_bits_to_float(((const uint16_t *)t->data)[i]);
}

/* Tensor catalogue: names, shapes and generator ids.  Global tensors use ids
 * 0..8, memory-group tensors 16+2g (+1), layer tensors 1024+32*l+slot. */
enum { L_WQ, L_WK, L_WV, L_WO, L_W1, L_W2, L_W3, L_GEA, L_GEF, L_GDSA, L_GDMEM,
       L_GDFFN, L_WQM, L_WOM, L_DWQ, L_DWK, L_DWV, L_DWO, L_DW1, L_DW2, L_DW3, L_NSLOT };

static const char *layer_names[L_NSLOT] = {
    "wq", "wk", "wv", "wo", "w1", "w2", "w3", "g_ea", "g_ef", "g_dsa", "g_dmem",
    "g_dffn", "wq_mem", "wo_mem", "dwq", "dwk", "dwv", "dwo", "dw1", "dw2", "dw3"};

enum { G_EMB, G_SSTAR, G_GMEM, G_GMERGE, G_WGATE, G_BGATE, G_WSTATE, G_GOUT, G_WOUT, G_NGLOB };

static void set_tensor(orc_tensor *t, const char *name, int32_t id, int32_t kind, int64_t rows, int64_t cols) {
  snprintf(t->name, sizeof t->name, "%s", name);
  t->id = id; t->kind = kind; t->rows = rows; t->cols = cols; t->data = NULL;
}

static int n_layer_slots(const orc_config *c) { return c->tied ? L_DWQ : L_NSLOT; }

static orc_tensor *glob(const orc_model *m, int slot) { return &m->t[slot]; }
static orc_tensor *memt(const orc_model *m, int g, int kv) { return &m->t[G_NGLOB + 2 * g + kv]; }
static orc_tensor *lay(const orc_model *m, int l, int slot) {
  return &m->t[G_NGLOB + 2 * m->cfg.groups + l * L_NSLOT + slot];
}

/* weight of the decoder: with tying the encoder's matrices are reused (§2.6) */
static const orc_tensor *dec_w(const orc_model *m, int l, int enc_slot) {
  if (m->cfg.tied) return lay(m, l, enc_slot);
  return lay(m, l, enc_slot - L_WQ + L_DWQ);
}

orc_model *orc_model_new(const orc_config *cfg) {
  if (cfg->d <= 0 || cfg->n_heads <= 0 || cfg->d % cfg->n_heads) return NULL;
  if ((cfg->d / cfg->n_heads) % 2) return NULL;
  if (cfg->n_layers <= 0 || cfg->window < 1 || cfg->ffn <= 0 || cfg->vocab <= 0) return NULL;
  if (!(cfg->groups == 1 || cfg->groups == cfg->n_layers)) return NULL;
  if (cfg->dtype != 0 && cfg->dtype != 1) return NULL;
  orc_model *m = (orc_model *)calloc(1, sizeof *m);
  m->cfg = *cfg;
  const int64_t d = cfg->d, F = cfg->ffn, V = cfg->vocab;
  m->n_tensors = G_NGLOB + 2 * cfg->groups + cfg->n_layers * L_NSLOT;
  m->t = (orc_tensor *)calloc((size_t)m->n_tensors, sizeof(orc_tensor));
  set_tensor(glob(m, G_EMB), "emb", 0, 0, V, d);
  set_tensor(glob(m, G_SSTAR), "s_star", 1, 0, 1, d);
  set_tensor(glob(m, G_GMEM), "g_mem", 2, 1, 1, d);
  set_tensor(glob(m, G_GMERGE), "g_merge", 3, 1, 1, d);
  set_tensor(glob(m, G_WGATE), "w_gate", 4, 0, d, 2 * d);
  set_tensor(glob(m, G_BGATE), "b_gate", 5, 2, 1, d);
  set_tensor(glob(m, G_WSTATE), "w_state", 6, 0, d, d);
  set_tensor(glob(m, G_GOUT), "g_out", 7, 1, 1, d);
  set_tensor(glob(m, G_WOUT), "w_out", 8, 0, V, d);
  char nm[32];
  for (int g = 0; g < cfg->groups; ++g) {
    snprintf(nm, sizeof nm, "wk_mem.%d", g);
    set_tensor(memt(m, g, 0), nm, 16 + 2 * g, 0, d, d);
    snprintf(nm, sizeof nm, "wv_mem.%d", g);
    set_tensor(memt(m, g, 1), nm, 16 + 2 * g + 1, 0, d, d);
  }
  for (int l = 0; l < cfg->n_layers; ++l) {
    for (int s = 0; s < L_NSLOT; ++s) {
      int64_t r = d, c = d;
      int kind = 0;
      if (s == L_W1 || s == L_W3 || s == L_DW1 || s == L_DW3) { r = F; c = d; }
      if (s == L_W2 || s == L_DW2) { r = d; c = F; }
      if (s >= L_GEA && s <= L_GDFFN) { r = 1; c = d; kind = 1; }
      snprintf(nm, sizeof nm, "%s.%d", layer_names[s], l);
      set_tensor(lay(m, l, s), nm, 1024 + 32 * l + s, kind, r, c);
    }
  }
  const size_t esz = cfg->dtype == 0 ? 4 : 2;
  for (int i = 0; i < m->n_tensors; ++i) {
    orc_tensor *t = &m->t[i];
    /* untied decoder slots only exist when the stacks are untied */
    int is_dec_slot = 0;
    if (i >= G_NGLOB + 2 * cfg->groups) {
      int s = (i - G_NGLOB - 2 * cfg->groups) % L_NSLOT;
      is_dec_slot = s >= L_DWQ;
    }
    if (is_dec_slot && cfg->tied) continue;
    t->data = calloc((size_t)(t->rows * t->cols), esz);
    if (t->kind == 1) {
      for (int64_t j = 0; j < t->rows * t->cols; ++j) {
        if (cfg->dtype == 0) ((float *)t->data)[j] = 1.0f;
        else ((uint16_t *)t->data)[j] = float_to_bf16_bits(1.0f);
      }
    }
  }
  (void)n_layer_slots;
  return m;
}

void orc_model_free(orc_model *m) {
  if (!m) return;
  for (int i = 0; i < m->n_tensors; ++i) free(m->t[i].data);
  free(m->t);
  free(m);
}

/* Random initialisation: every random tensor element is
 * init_std * N01 (Irwin-Hall), rounded to the storage precision. */
void orc_model_init(orc_model *m, uint64_t seed) {
  const double sd = (double)(float)m->cfg.init_std;
  for (int i = 0; i < m->n_tensors; ++i) {
    orc_tensor *t = &m->t[i];
    if (!t->data || t->kind != 0) continue;
    const int64_t n = t->rows * t->cols;
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < n; ++j) {
      double w = sd * orc_normal_ih12(seed, (uint32_t)t->id, (uint64_t)j);
      float f = (float)w;
      if (m->cfg.dtype == 0) ((float *)t->data)[j] = f;
      else ((uint16_t *)t->data)[j] = float_to_bf16_bits(f);
    }
  }
}

static orc_tensor *find(const orc_model *m, const char *name) {
  for (int i = 0; i < m->n_tensors; ++i)
    if (m->t[i].data && strcmp(m->t[i].name, name) == 0) return &m->t[i];
  return NULL;
}

/* raw copy in the model's storage format; returns 0 or -1 */
int orc_tensor_set(orc_model *m, const char *name, const void *raw, int64_t bytes) {
  orc_tensor *t = find(m, name);
  const int64_t esz = m->cfg.dtype == 0 ? 4 : 2;
  if (!t || bytes != t->rows * t->cols * esz) return -1;
  memcpy(t->data, raw, (size_t)bytes);
  return 0;
}

int orc_tensor_get(const orc_model *m, const char *name, void *raw, int64_t bytes) {
  orc_tensor *t = find(m, name);
  const int64_t esz = m->cfg.dtype == 0 ? 4 : 2;
  if (!t || bytes != t->rows * t->cols * esz) return -1;
  memcpy(raw, t->data, (size_t)bytes);
  return 0;
}

/* ------------------------------------------------------------------------ */
/* building blocks                                                           */
/* ------------------------------------------------------------------------ */

/* y = W x, W stored row-major [rows, cols]; x may be a concatenation handled
 * by the caller. */
static void matvec(const orc_model *m, const orc_tensor *W, const double *x, double *y) {
  const int64_t R = W->rows, C = W->cols;
#pragma omp parallel for schedule(static) if (R * C > 65536)
  for (int64_t r = 0; r < R; ++r) {
    double acc = 0.0;
    for (int64_t c = 0; c < C; ++c) acc += tw(m, W, r * C + c) * x[c];
    y[r] = acc;
  }
}

/* RMSNorm(x; gamma) = gamma * x / sqrt(mean(x^2) + eps) */
void orc_rmsnorm(const double *x, const double *gamma, int n, double eps, double *out) {
  double ss = 0.0;
  for (int i = 0; i < n; ++i) ss += x[i] * x[i];
  const double inv = 1.0 / sqrt(ss / n + eps);
  for (int i = 0; i < n; ++i) out[i] = gamma[i] * x[i] * inv;
}

static void rmsnorm_w(const orc_model *m, const orc_tensor *g, const double *x, double *out) {
  const int n = m->cfg.d;
  double *gm = (double *)malloc(sizeof(double) * n);
  for (int i = 0; i < n; ++i) gm[i] = tw(m, g, i);
  orc_rmsnorm(x, gm, n, m->cfg.rms_eps, out);
  free(gm);
}

/* Rotate-half rotary position map on one head of size hd at position p:
 * pairs (i, i+hd/2) are rotated by angle p * base^(-2i/hd). */
void orc_rope(double *x, int hd, double p, double base) {
  const int h = hd / 2;
  for (int i = 0; i < h; ++i) {
    const double th = p * pow(base, -2.0 * i / hd);
    const double c = cos(th), s = sin(th);
    const double a = x[i], b = x[i + h];
    x[i] = a * c - b * s;
    x[i + h] = a * s + b * c;
  }
}

static void rope_all_heads(const orc_model *m, double *x, int64_t pos1) {
  const int H = m->cfg.n_heads, hd = m->cfg.d / H;
  for (int h = 0; h < H; ++h) orc_rope(x + h * hd, hd, (double)(pos1 - 1), m->cfg.rope_base);
}

/* Single-head attention of query q over n (key, value) rows:
 * softmax_j(q.k_j / sqrt(hd)) weighted sum of v_j.  Keys and values are
 * addressed through row pointers so callers can pass any index set. */
void orc_attend(const double *q, const double *const *k, const double *const *v, int n, int hd, double *out) {
  double *sc = (double *)malloc(sizeof(double) * (n > 0 ? n : 1));
  const double scale = 1.0 / sqrt((double)hd);
  double mx = -INFINITY;
  for (int j = 0; j < n; ++j) {
    double s = 0.0;
    for (int i = 0; i < hd; ++i) s += q[i] * k[j][i];
    sc[j] = s * scale;
    if (sc[j] > mx) mx = sc[j];
  }
  double den = 0.0;
  for (int j = 0; j < n; ++j) { sc[j] = exp(sc[j] - mx); den += sc[j]; }
  for (int i = 0; i < hd; ++i) out[i] = 0.0;
  for (int j = 0; j < n; ++j) {
    const double p = sc[j] / den;
    for (int i = 0; i < hd; ++i) out[i] += p * v[j][i];
  }
  free(sc);
}

/* Multi-head attention for one query row against rows k[j], v[j] (each of
 * width d, heads concatenated). */
static void mha(const orc_model *m, const double *q, const double *const *k, const double *const *v, int n, double *out) {
  const int H = m->cfg.n_heads, hd = m->cfg.d / H;
  const double **kh = (const double **)malloc(sizeof(double *) * (n > 0 ? n : 1));
  const double **vh = (const double **)malloc(sizeof(double *) * (n > 0 ? n : 1));
  for (int h = 0; h < H; ++h) {
    for (int j = 0; j < n; ++j) { kh[j] = k[j] + h * hd; vh[j] = v[j] + h * hd; }
    orc_attend(q + h * hd, kh, vh, n, hd, out + h * hd);
  }
  free(kh);
  free(vh);
}

static double silu(double x) { return x / (1.0 + exp(-x)); }
static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }

/* SwiGLU FFN: W2 (silu(W1 y) * (W3 y)) */
static void ffn(const orc_model *m, const orc_tensor *w1, const orc_tensor *w2, const orc_tensor *w3,
                const double *y, double *out) {
  const int F = m->cfg.ffn;
  double *a = (double *)malloc(sizeof(double) * F);
  double *b = (double *)malloc(sizeof(double) * F);
  matvec(m, w1, y, a);
  matvec(m, w3, y, b);
  for (int i = 0; i < F; ++i) a[i] = silu(a[i]) * b[i];
  matvec(m, w2, a, out);
  free(a);
  free(b);
}

/* log-softmax over n logits */
void orc_log_softmax(const double *x, int n, double *out) {
  double mx = -INFINITY;
  for (int i = 0; i < n; ++i) if (x[i] > mx) mx = x[i];
  double s = 0.0;
  for (int i = 0; i < n; ++i) s += exp(x[i] - mx);
  const double lse = mx + log(s);
  for (int i = 0; i < n; ++i) out[i] = x[i] - lse;
}

/* ------------------------------------------------------------------------ */
/* per-sequence state                                                        */
/* ------------------------------------------------------------------------ */

typedef struct {
  const orc_model *m;
  int32_t max_len;
  int32_t n_enc;        /* tokens encoded so far: e_1..e_n_enc, memory rows */
  int32_t n_dec;        /* decoder transitions applied: state is H_{n_dec} */
  int32_t keep_enc_cache; /* keep per-layer encoder K/V for the step form (eq. 2.8) */
  int32_t *tok;         /* tokens consumed by the encoder */
  double *e;            /* [max_len][d] encoder outputs */
  double *ce_k, *ce_v;  /* [L][max_len][d] encoder continuation cache C^E */
  double *mk, *mv;      /* [G][max_len][d] memory M^g (keys already rotated) */
  double *s;            /* [d] recurrent output s_t */
  /* decoder SWA cache C^D: per layer up to W-1 entries tagged by position */
  int32_t *win_pos;     /* [L][W-1], 0 = empty */
  double *win_k, *win_v;/* [L][W-1][d] */
} orc_seq;

orc_seq *orc_seq_new(const orc_model *m, int32_t max_len, int32_t keep_enc_cache) {
  const orc_config *c = &m->cfg;
  if (max_len <= 0) return NULL;
  orc_seq *q = (orc_seq *)calloc(1, sizeof *q);
  const int64_t d = c->d, L = c->n_layers, G = c->groups, Wm1 = c->window - 1;
  q->m = m;
  q->max_len = max_len;
  q->keep_enc_cache = keep_enc_cache;
  q->tok = (int32_t *)calloc((size_t)max_len, sizeof(int32_t));
  q->e = (double *)calloc((size_t)(max_len * d), sizeof(double));
  if (keep_enc_cache) {
    q->ce_k = (double *)calloc((size_t)(L * max_len * d), sizeof(double));
    q->ce_v = (double *)calloc((size_t)(L * max_len * d), sizeof(double));
  }
  q->mk = (double *)calloc((size_t)(G * max_len * d), sizeof(double));
  q->mv = (double *)calloc((size_t)(G * max_len * d), sizeof(double));
  q->s = (double *)calloc((size_t)d, sizeof(double));
  q->win_pos = (int32_t *)calloc((size_t)(L * (Wm1 > 0 ? Wm1 : 1)), sizeof(int32_t));
  q->win_k = (double *)calloc((size_t)(L * (Wm1 > 0 ? Wm1 : 1) * d), sizeof(double));
  q->win_v = (double *)calloc((size_t)(L * (Wm1 > 0 ? Wm1 : 1) * d), sizeof(double));
  /* H_0 = (s_star, empty), eq. 2.3 */
  for (int64_t i = 0; i < d; ++i) q->s[i] = tw(m, glob(m, G_SSTAR), i);
  return q;
}

void orc_seq_free(orc_seq *q) {
  if (!q) return;
  free(q->tok); free(q->e); free(q->ce_k); free(q->ce_v); free(q->mk); free(q->mv);
  free(q->s); free(q->win_pos); free(q->win_k); free(q->win_v);
  free(q);
}

/* memory rows for position j (1-based) from e_j, eq. 2.2:
 * k^g_j = RoPE(W^g_K RMSNorm_E(e_j), j-1), v^g_j = W^g_V RMSNorm_E(e_j) */
static void memory_append(orc_seq *q, int32_t j) {
  const orc_model *m = q->m;
  const int d = m->cfg.d;
  double *n = (double *)malloc(sizeof(double) * d);
  rmsnorm_w(m, glob(m, G_GMEM), q->e + (int64_t)(j - 1) * d, n);
  for (int g = 0; g < m->cfg.groups; ++g) {
    double *k = q->mk + ((int64_t)g * q->max_len + (j - 1)) * d;
    double *v = q->mv + ((int64_t)g * q->max_len + (j - 1)) * d;
    matvec(m, memt(m, g, 0), n, k);
    matvec(m, memt(m, g, 1), n, v);
    rope_all_heads(m, k, j);
  }
  free(n);
}

/* Token-parallel causal encoder, eq. 2.1: positions n_enc+1..n_enc+T are
 * processed together inside each layer (layers in sequence) under a causal
 * mask.  This schedule starts from an empty prefix (n_enc == 0). */
int orc_encode_prefill(orc_seq *q, const int32_t *tok, int32_t T) {
  const orc_model *m = q->m;
  const orc_config *c = &m->cfg;
  if (q->n_enc != 0 || T <= 0 || T > q->max_len) return -1;
  const int64_t d = c->d;
  for (int i = 0; i < T; ++i) {
    if (tok[i] < 0 || tok[i] >= c->vocab) return -1;
    q->tok[i] = tok[i];
  }
  double *h = q->e; /* residual stream lives in e */
  for (int i = 0; i < T; ++i)
    for (int64_t a = 0; a < d; ++a) h[i * d + a] = tw(m, glob(m, G_EMB), (int64_t)tok[i] * d + a);
  double *x = (double *)malloc(sizeof(double) * T * d);
  double *Q = (double *)malloc(sizeof(double) * T * d);
  double *K = (double *)malloc(sizeof(double) * T * d);
  double *Vv = (double *)malloc(sizeof(double) * T * d);
  double *o = (double *)malloc(sizeof(double) * T * d);
  for (int l = 0; l < c->n_layers; ++l) {
    for (int i = 0; i < T; ++i) {
      rmsnorm_w(m, lay(m, l, L_GEA), h + i * d, x + i * d);
      matvec(m, lay(m, l, L_WQ), x + i * d, Q + i * d);
      matvec(m, lay(m, l, L_WK), x + i * d, K + i * d);
      matvec(m, lay(m, l, L_WV), x + i * d, Vv + i * d);
      rope_all_heads(m, Q + i * d, i + 1);
      rope_all_heads(m, K + i * d, i + 1);
    }
    if (q->keep_enc_cache) {
      memcpy(q->ce_k + (int64_t)l * q->max_len * d, K, sizeof(double) * T * d);
      memcpy(q->ce_v + (int64_t)l * q->max_len * d, Vv, sizeof(double) * T * d);
    }
#pragma omp parallel for schedule(dynamic, 4)
    for (int i = 0; i < T; ++i) {
      const double **kr = (const double **)malloc(sizeof(double *) * (i + 1));
      const double **vr = (const double **)malloc(sizeof(double *) * (i + 1));
      for (int j = 0; j <= i; ++j) { kr[j] = K + j * d; vr[j] = Vv + j * d; } /* causal: j <= i */
      mha(m, Q + i * d, kr, vr, i + 1, o + i * d);
      free(kr);
      free(vr);
    }
    double *tmp = (double *)malloc(sizeof(double) * d);
    for (int i = 0; i < T; ++i) {
      matvec(m, lay(m, l, L_WO), o + i * d, tmp);
      for (int64_t a = 0; a < d; ++a) h[i * d + a] += tmp[a];
      rmsnorm_w(m, lay(m, l, L_GEF), h + i * d, x + i * d);
      ffn(m, lay(m, l, L_W1), lay(m, l, L_W2), lay(m, l, L_W3), x + i * d, tmp);
      for (int64_t a = 0; a < d; ++a) h[i * d + a] += tmp[a];
    }
    free(tmp);
  }
  free(x); free(Q); free(K); free(Vv); free(o);
  q->n_enc = T;
  for (int j = 1; j <= T; ++j) memory_append(q, j);
  return 0;
}

/* Incremental encoder step, eq. 2.8: (e_t, C^E_t) = E^step(x_t, C^E_{t-1}),
 * followed by the memory append for position t. */
int orc_encode_step(orc_seq *q, int32_t token) {
  const orc_model *m = q->m;
  const orc_config *c = &m->cfg;
  if (!q->keep_enc_cache || q->n_enc >= q->max_len) return -1;
  if (token < 0 || token >= c->vocab) return -1;
  const int64_t d = c->d;
  const int32_t t = q->n_enc + 1;
  q->tok[t - 1] = token;
  double *h = q->e + (int64_t)(t - 1) * d;
  for (int64_t a = 0; a < d; ++a) h[a] = tw(m, glob(m, G_EMB), (int64_t)token * d + a);
  double *x = (double *)malloc(sizeof(double) * d);
  double *qv = (double *)malloc(sizeof(double) * d);
  double *o = (double *)malloc(sizeof(double) * d);
  double *tmp = (double *)malloc(sizeof(double) * d);
  const double **kr = (const double **)malloc(sizeof(double *) * t);
  const double **vr = (const double **)malloc(sizeof(double *) * t);
  for (int l = 0; l < c->n_layers; ++l) {
    double *CK = q->ce_k + (int64_t)l * q->max_len * d;
    double *CV = q->ce_v + (int64_t)l * q->max_len * d;
    rmsnorm_w(m, lay(m, l, L_GEA), h, x);
    matvec(m, lay(m, l, L_WQ), x, qv);
    matvec(m, lay(m, l, L_WK), x, CK + (int64_t)(t - 1) * d);
    matvec(m, lay(m, l, L_WV), x, CV + (int64_t)(t - 1) * d);
    rope_all_heads(m, qv, t);
    rope_all_heads(m, CK + (int64_t)(t - 1) * d, t);
    for (int j = 0; j < t; ++j) { kr[j] = CK + (int64_t)j * d; vr[j] = CV + (int64_t)j * d; }
    mha(m, qv, kr, vr, t, o);
    matvec(m, lay(m, l, L_WO), o, tmp);
    for (int64_t a = 0; a < d; ++a) h[a] += tmp[a];
    rmsnorm_w(m, lay(m, l, L_GEF), h, x);
    ffn(m, lay(m, l, L_W1), lay(m, l, L_W2), lay(m, l, L_W3), x, tmp);
    for (int64_t a = 0; a < d; ++a) h[a] += tmp[a];
  }
  free(x); free(qv); free(o); free(tmp); free(kr); free(vr);
  q->n_enc = t;
  memory_append(q, t);
  return 0;
}

/* u_t = Merge(e_t, s_{t-1}), eq. 2.4 with the merge of eqs. 2.9-2.11 (kind 0)
 * or the convex gate (kind 1). */
void orc_merge(const orc_model *m, const double *e, const double *s, double *u) {
  const int d = m->cfg.d;
  double *cat = (double *)malloc(sizeof(double) * 2 * d);
  double *g = (double *)malloc(sizeof(double) * d);
  if (m->cfg.merge_kind == 0) {
    double *r = (double *)malloc(sizeof(double) * d);
    double *ws = (double *)malloc(sizeof(double) * d);
    rmsnorm_w(m, glob(m, G_GMERGE), s, r);                     /* eq. 2.9 */
    memcpy(cat, e, sizeof(double) * d);
    memcpy(cat + d, r, sizeof(double) * d);
    matvec(m, glob(m, G_WGATE), cat, g);                       /* eq. 2.10 */
    for (int i = 0; i < d; ++i) g[i] = sigmoid(g[i] + tw(m, glob(m, G_BGATE), i));
    matvec(m, glob(m, G_WSTATE), r, ws);                       /* eq. 2.11 */
    for (int i = 0; i < d; ++i) u[i] = e[i] + m->cfg.alpha * g[i] * ws[i];
    free(r);
    free(ws);
  } else {
    memcpy(cat, e, sizeof(double) * d);
    memcpy(cat + d, s, sizeof(double) * d);
    matvec(m, glob(m, G_WGATE), cat, g);
    for (int i = 0; i < d; ++i) {
      g[i] = sigmoid(g[i]);
      u[i] = g[i] * e[i] + (1.0 - g[i]) * s[i];
    }
  }
  free(cat);
  free(g);
}

/* One decoder transition H_t = D_phi(u_t; M_<=t, C^D_{t-1}, t), eqs. 2.5 and
 * 2.12-2.16, for t = n_dec + 1.  Requires e_t and M_<=t (n_enc >= t).
 * If logits != NULL the readout W_o RMSNorm_o(s_t) (eq. 2.6) is written. */
int orc_decoder_step(orc_seq *q, double *logits) {
  const orc_model *m = q->m;
  const orc_config *c = &m->cfg;
  const int32_t t = q->n_dec + 1;
  if (t > q->n_enc) return -1;
  const int64_t d = c->d;
  const int W = c->window, Wm1 = W - 1;
  double *z = (double *)malloc(sizeof(double) * d);
  double *x = (double *)malloc(sizeof(double) * d);
  double *qv = (double *)malloc(sizeof(double) * d);
  double *kc = (double *)malloc(sizeof(double) * d);
  double *vc = (double *)malloc(sizeof(double) * d);
  double *o = (double *)malloc(sizeof(double) * d);
  double *tmp = (double *)malloc(sizeof(double) * d);
  const double **kr = (const double **)malloc(sizeof(double *) * (t > W ? t : W) + 8);
  const double **vr = (const double **)malloc(sizeof(double *) * (t > W ? t : W) + 8);

  orc_merge(m, q->e + (int64_t)(t - 1) * d, q->s, z); /* z^0 = u_t */
  for (int l = 0; l < c->n_layers; ++l) {
    /* eqs. 2.12-2.13: current q, k, v from the layer input, before SWA */
    rmsnorm_w(m, lay(m, l, L_GDSA), z, x);
    matvec(m, dec_w(m, l, L_WQ), x, qv);
    matvec(m, dec_w(m, l, L_WK), x, kc);
    matvec(m, dec_w(m, l, L_WV), x, vc);
    rope_all_heads(m, qv, t);
    rope_all_heads(m, kc, t);
    /* eq. 2.14: keys at positions max(1, t-W+1) .. t: retained history plus
     * the current entry */
    int n = 0;
    const int32_t lo = t - W + 1 > 1 ? t - W + 1 : 1;
    for (int sidx = 0; sidx < Wm1; ++sidx) {
      const int32_t p = q->win_pos[l * Wm1 + sidx];
      if (p >= lo && p <= t - 1) {
        kr[n] = q->win_k + ((int64_t)l * Wm1 + sidx) * d;
        vr[n] = q->win_v + ((int64_t)l * Wm1 + sidx) * d;
        ++n;
      }
    }
    kr[n] = kc;
    vr[n] = vc;
    ++n;
    mha(m, qv, kr, vr, n, o);
    matvec(m, dec_w(m, l, L_WO), o, tmp);
    for (int64_t a = 0; a < d; ++a) z[a] += tmp[a]; /* z now holds b_t^l */
    /* eq. 2.15: cross-attention to M^{g(l)}_{<=t} */
    const int g = c->groups == 1 ? 0 : l;
    rmsnorm_w(m, lay(m, l, L_GDMEM), z, x);
    matvec(m, lay(m, l, L_WQM), x, qv);
    rope_all_heads(m, qv, t);
    for (int j = 0; j < t; ++j) { /* prefix restriction: positions 1..t only */
      kr[j] = q->mk + ((int64_t)g * q->max_len + j) * d;
      vr[j] = q->mv + ((int64_t)g * q->max_len + j) * d;
    }
    mha(m, qv, kr, vr, t, o);
    matvec(m, lay(m, l, L_WOM), o, tmp);
    for (int64_t a = 0; a < d; ++a) z[a] += tmp[a]; /* a_t^l */
    /* eq. 2.16: FFN with residual */
    rmsnorm_w(m, lay(m, l, L_GDFFN), z, x);
    ffn(m, dec_w(m, l, L_W1), dec_w(m, l, L_W2), dec_w(m, l, L_W3), x, tmp);
    for (int64_t a = 0; a < d; ++a) z[a] += tmp[a]; /* z_t^l */
    /* §2.5 retention: after the update keep positions max(1,t-W+2)..t;
     * the set is empty for W = 1. */
    if (Wm1 > 0) {
      const int32_t keep_lo = t - W + 2;
      int slot = -1;
      for (int sidx = 0; sidx < Wm1; ++sidx) {
        int32_t *p = &q->win_pos[l * Wm1 + sidx];
        if (*p != 0 && *p < keep_lo) *p = 0; /* evict */
      }
      for (int sidx = 0; sidx < Wm1; ++sidx)
        if (q->win_pos[l * Wm1 + sidx] == 0) { slot = sidx; break; }
      if (slot < 0) { slot = 0; } /* unreachable: at most W-2 entries remain */
      q->win_pos[l * Wm1 + slot] = t;
      memcpy(q->win_k + ((int64_t)l * Wm1 + slot) * d, kc, sizeof(double) * d);
      memcpy(q->win_v + ((int64_t)l * Wm1 + slot) * d, vc, sizeof(double) * d);
    }
  }
  memcpy(q->s, z, sizeof(double) * d); /* s_t = z_t^{L_D} */
  q->n_dec = t;
  if (logits) {
    rmsnorm_w(m, glob(m, G_GOUT), q->s, x);
    matvec(m, glob(m, G_WOUT), x, logits);
  }
  free(z); free(x); free(qv); free(kc); free(vc); free(o); free(tmp); free(kr); free(vr);
  return 0;
}

/* ------------------------------------------------------------------------ */
/* sampler (report §5.3: the behaviour log-probability includes temperature, */
/* truncation and renormalisation)                                           */
/* ------------------------------------------------------------------------ */

/* Top-k temperature sampler.  Candidates are the top_k raw logits ordered by
 * (value desc, id asc) (top_k <= 0 or >= V keeps all).  Weights
 * w_i = exp((l_i - l_max)/tau) and their running sums are formed in fp32 in
 * that order (the decision is taken in the device's precision).  The
 * uniform is u = (philox(ctr = (t, b, 0, 0), key = seed).x0 >> 8) * 2^-24;
 * the token is the first candidate whose running sum exceeds u * sum.
 * Outputs: token, log mu (fp64, exact tempered+truncated distribution),
 * log p (fp64 raw log-softmax, from double logits if given else from the
 * fp32 ones) and the decision margin relative to the total weight. */
int orc_sample(const float *logits, const double *logits64, int32_t V, float temperature, int32_t top_k,
               uint64_t seed, uint32_t t, uint32_t b, int32_t *token, double *log_mu, double *log_p,
               double *margin) {
  if (V <= 0 || !(temperature > 0.0f)) return -1;
  int32_t k = (top_k <= 0 || top_k > V) ? V : top_k;
  int32_t *idx = (int32_t *)malloc(sizeof(int32_t) * k);
  char *used = (char *)calloc((size_t)V, 1);
  for (int32_t r = 0; r < k; ++r) { /* selection by (value desc, id asc) */
    int32_t best = -1;
    for (int32_t i = 0; i < V; ++i) {
      if (used[i]) continue;
      if (best < 0 || logits[i] > logits[best]) best = i;
    }
    used[best] = 1;
    idx[r] = best;
  }
  const float inv_mx = logits[idx[0]] / temperature;
  float *w = (float *)malloc(sizeof(float) * k);
  float sum = 0.0f;
  for (int32_t r = 0; r < k; ++r) {
    w[r] = expf(logits[idx[r]] / temperature - inv_mx);
    sum += w[r];
  }
  uint32_t ctr[4] = {t, b, 0u, 0u}, key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)}, o[4];
  orc_philox4x32_10(ctr, key, o);
  const float u = (float)(o[0] >> 8) * (1.0f / 16777216.0f);
  const float target = u * sum;
  float run = 0.0f;
  int32_t pick = k - 1;
  float lo_edge = 0.0f, hi_edge = sum;
  for (int32_t r = 0; r < k; ++r) {
    float prev = run;
    run += w[r];
    if (run > target) { pick = r; lo_edge = prev; hi_edge = run; break; }
  }
  *token = idx[pick];
  if (margin) {
    double m1 = (double)target - lo_edge, m2 = (double)hi_edge - target;
    *margin = (m1 < m2 ? m1 : m2) / (double)sum;
  }
  /* log mu in fp64 from the same tempered, truncated distribution */
  {
    double mx = (double)logits[idx[0]] / temperature, s = 0.0;
    for (int32_t r = 0; r < k; ++r) s += exp((double)logits[idx[r]] / temperature - mx);
    *log_mu = ((double)logits[idx[pick]] / temperature - mx) - log(s);
  }
  if (log_p) {
    double mx = -INFINITY, s = 0.0;
    for (int32_t i = 0; i < V; ++i) {
      double v = logits64 ? logits64[i] : (double)logits[i];
      if (v > mx) mx = v;
    }
    for (int32_t i = 0; i < V; ++i) s += exp((logits64 ? logits64[i] : (double)logits[i]) - mx);
    *log_p = (logits64 ? logits64[*token] : (double)logits[*token]) - mx - log(s);
  }
  free(idx); free(used); free(w);
  return 0;
}

/* ------------------------------------------------------------------------ */
/* schedules (report App. A)                                                 */
/* ------------------------------------------------------------------------ */

/* Current-policy replay (App. A.4) / teacher-forced scoring (App. A.3):
 * from H_0, encode x_{1:S} (schedule 0: token-parallel prefill, eq. 2.1;
 * schedule 1: incremental step form, eq. 2.8), then apply decoder updates
 * t = 1..S-1, each followed by out[t-1] = log p(x_{t+1} | x_{1:t}). */
int orc_replay_logprobs(const orc_model *m, const int32_t *tok, int32_t S, int32_t schedule, double *out) {
  if (S < 2) return -1;
  orc_seq *q = orc_seq_new(m, S, schedule == 1);
  double *lg = (double *)malloc(sizeof(double) * m->cfg.vocab);
  double *lp = (double *)malloc(sizeof(double) * m->cfg.vocab);
  int rc = 0;
  if (schedule == 0) rc = orc_encode_prefill(q, tok, S);
  for (int32_t t = 1; t <= S - 1 && rc == 0; ++t) {
    if (schedule == 1) rc = orc_encode_step(q, tok[t - 1]);
    if (rc) break;
    rc = orc_decoder_step(q, lg);
    if (rc) break;
    orc_log_softmax(lg, m->cfg.vocab, lp);
    out[t - 1] = lp[tok[t]];
  }
  free(lg); free(lp);
  orc_seq_free(q);
  return rc;
}

/* RL replay with importance ratios (report §5.3, eq. 5.5; App. A.4): the
 * current-policy replay of one rollout, then per scored token
 * r = exp(log p - log mu) for sampled actions (mask != 0) and no factor (1)
 * for external tokens (report §6), and the log of the trajectory ratio, the
 * sum of log r over the actions. */
int orc_replay_ratios(const orc_model *m, const int32_t *tok, int32_t S, const double *logmu, const uint8_t *mask,
                      double *out_logp, double *out_ratio, double *out_seq_logratio) {
  const int rc = orc_replay_logprobs(m, tok, S, 0, out_logp);
  if (rc) return rc;
  double sum = 0.0;
  for (int32_t i = 0; i < S - 1; ++i) {
    const double lr = out_logp[i] - logmu[i];
    out_ratio[i] = mask[i] ? exp(lr) : 1.0;
    if (mask[i]) sum += lr;
  }
  *out_seq_logratio = sum;
  return 0;
}

/* Prompt prefill (App. A.1) then sampled generation (App. A.2) for one
 * sequence with batch index b: n_new tokens are sampled; the last sampled
 * token is left pending (not consumed).  Outputs per generated token: id,
 * log p (raw), log mu (behaviour), decision margin. */
int orc_generate(const orc_model *m, const int32_t *prompt, int32_t T, int32_t n_new, float temperature,
                 int32_t top_k, uint64_t seed, uint32_t b, int32_t *out_tok, double *out_logp,
                 double *out_logmu, double *out_margin) {
  if (T < 1 || n_new < 1) return -1;
  orc_seq *q = orc_seq_new(m, T + n_new, 1);
  const int V = m->cfg.vocab;
  double *lg = (double *)malloc(sizeof(double) * V);
  float *lf = (float *)malloc(sizeof(float) * V);
  int rc = orc_encode_prefill(q, prompt, T);
  for (int32_t t = 1; t <= T && rc == 0; ++t) rc = orc_decoder_step(q, t == T ? lg : NULL);
  for (int32_t i = 0; i < n_new && rc == 0; ++i) {
    for (int v = 0; v < V; ++v) lf[v] = (float)lg[v];
    const uint32_t t = (uint32_t)q->n_dec;
    rc = orc_sample(lf, lg, V, temperature, top_k, seed, t, b, &out_tok[i], &out_logmu[i], &out_logp[i],
                    out_margin ? &out_margin[i] : NULL);
    if (rc || i == n_new - 1) break;
    rc = orc_encode_step(q, out_tok[i]);
    if (!rc) rc = orc_decoder_step(q, lg);
  }
  free(lg); free(lf);
  orc_seq_free(q);
  return rc;
}

/* ------------------------------------------------------------------------ */
/* state inspection for tests                                                */
/* ------------------------------------------------------------------------ */

int32_t orc_seq_pos(const orc_seq *q, int32_t which) { return which == 0 ? q->n_enc : q->n_dec; }

void orc_seq_get_s(const orc_seq *q, double *out) { memcpy(out, q->s, sizeof(double) * q->m->cfg.d); }

void orc_seq_get_e(const orc_seq *q, int32_t pos1, double *out) {
  memcpy(out, q->e + (int64_t)(pos1 - 1) * q->m->cfg.d, sizeof(double) * q->m->cfg.d);
}

/* memory row of group g at position pos1: which 0 = key, 1 = value */
void orc_seq_get_mem(const orc_seq *q, int32_t g, int32_t pos1, int32_t which, double *out) {
  const double *src = which == 0 ? q->mk : q->mv;
  memcpy(out, src + ((int64_t)g * q->max_len + pos1 - 1) * q->m->cfg.d, sizeof(double) * q->m->cfg.d);
}

/* Retained SWA entries of layer l: writes their positions (ascending) and
 * returns the count; optionally copies keys/values in that order. */
int32_t orc_seq_window(const orc_seq *q, int32_t l, int32_t *pos, double *k, double *v) {
  const int Wm1 = q->m->cfg.window - 1;
  const int64_t d = q->m->cfg.d;
  int32_t n = 0;
  for (int32_t want = 1; want <= q->n_dec; ++want) {
    for (int s = 0; s < Wm1; ++s) {
      if (q->win_pos[l * Wm1 + s] == want) {
        if (pos) pos[n] = want;
        if (k) memcpy(k + n * d, q->win_k + ((int64_t)l * Wm1 + s) * d, sizeof(double) * d);
        if (v) memcpy(v + n * d, q->win_v + ((int64_t)l * Wm1 + s) * d, sizeof(double) * d);
        ++n;
      }
    }
  }
  return n;
}

/* overwrite s (used by invariance tests that perturb the state) */
void orc_seq_set_s(orc_seq *q, const double *s) { memcpy(q->s, s, sizeof(double) * q->m->cfg.d); }

int32_t orc_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
