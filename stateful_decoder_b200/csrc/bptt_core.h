// bptt_core.h -- full back-propagation through time of the Recurrent Looped
// Transformer replay ("Recurrent Looped Transformer" §5.1-§5.4, App. C).
//
// Computes L_w = -sum_{b,t} w[b][t] log p(x_{b,t+1} | x_{b,1:t}) over a
// lock-step batch of B sequences of S tokens, and its gradient with respect
// to every stored tensor.  The gradient runs through the causal encoder, the
// memory projections, the merge, every decoder SWA key/value and the
// recurrent output over all positions; nothing is detached.
//
// Schedule (reverse time, segment checkpointing, §4.3 and §5.4):
//   forward   encoder and memory token-parallel, activations kept per layer;
//             decoder steps t = 0..S-2 keep every layer's SWA key/value
//             (the whole history, so any window can be rebuilt) and the
//             recurrent output at each segment start;
//   backward  segments in reverse order: recompute the segment's steps from
//             its checkpoint (same parameters, same values), then reverse
//             its steps one at a time -- readout, and per layer FFN, memory
//             cross-attention, SWA -- and the merge, handing ds to the step
//             before and de_t to the encoder.  SWA key/value adjoints are
//             accumulated per position and are complete when their own
//             step is reversed (the later steps that read them come first).
//             Off the serial chain, after the segment's reversal: every
//             weight gradient of the segment as one contraction over its
//             seg*B rows (dW += dY^T X, the adjoints dY of each step kept per
//             step), and the memory key/value adjoints of the segment's
//             queries as one masked token-parallel pass per layer;
//   encoder   the encoder backward runs token-parallel at the end.
//
// Every operation is a functor whose operator()(i) computes output element
// (or row) i from its inputs alone: no shared memory, no ordering between
// threads except the atomic adds of the embedding gradient.  A backend runs
// a functor over i = 0..n-1: the CUDA backend (bptt.cu) as a kernel, one
// thread per i; a host backend runs the same functors in a loop, which lets
// the index arithmetic be checked on the CPU.  Real is the arithmetic type
// (float on the GPU).
//
// Readings: the forward definitions of the library (SwiGLU FFN, rotate-half
// RoPE at 0-based position p, pre-norm RMSNorm per sublayer, 1/sqrt(hd)
// attention scale, merge of eqs. 2.9-2.11 or the convex gate).
#pragma once
#include <math.h>
#include <stdint.h>
#include <stdio.h>

#include <string>
#include <utility>
#include <vector>

#if defined(__CUDACC__)
#define RLT_HD __host__ __device__
#else
#define RLT_HD
#endif

namespace rlt {
namespace bptt {

// ------------------------------------------------------------------ math
RLT_HD inline float r_exp(float x) { return expf(x); }
RLT_HD inline double r_exp(double x) { return exp(x); }
RLT_HD inline float r_log(float x) { return logf(x); }
RLT_HD inline double r_log(double x) { return log(x); }
RLT_HD inline float r_sqrt(float x) { return sqrtf(x); }
RLT_HD inline double r_sqrt(double x) { return sqrt(x); }
template <class Real> RLT_HD inline Real r_sigmoid(Real x) { return Real(1) / (Real(1) + r_exp(-x)); }

RLT_HD inline void r_atomic_add(float* a, float v) {
#if defined(__CUDA_ARCH__)
  atomicAdd(a, v);
#else
  *a += v;
#endif
}
RLT_HD inline void r_atomic_add(double* a, double v) {
#if defined(__CUDA_ARCH__)
  atomicAdd(a, v);
#else
  *a += v;
#endif
}

constexpr int kMaxHead = 128;  // largest head size the attention functors hold in registers

// ------------------------------------------------------------------ tensor catalogue
// The stored tensors of a model, named as in rlt.h.  Indices: the nine
// global tensors, then wk_mem.g / wv_mem.g, then L_NSLOT slots per layer
// (the seven decoder slots exist only for untied stacks).
enum { T_EMB, T_SSTAR, T_GMEM, T_GMERGE, T_WGATE, T_BGATE, T_WSTATE, T_GOUT, T_WOUT, T_NGLOB };
enum { L_WQ, L_WK, L_WV, L_WO, L_W1, L_W2, L_W3, L_GEA, L_GEF, L_GDSA, L_GDMEM, L_GDFFN, L_WQM, L_WOM,
       L_DWQ, L_DWK, L_DWV, L_DWO, L_DW1, L_DW2, L_DW3, L_NSLOT };

struct Dims {
  int B, S;                        // sequences, tokens per sequence
  int d, H, L, W, G, F, V;         // model sizes (hd = d/H)
  int tied, merge_kind;            // merge_kind 0: eqs. 2.9-2.11; 1: convex gate
  double alpha, eps, rope_base;
  int hd() const { return d / H; }
};

inline int n_tensors(const Dims& D) { return T_NGLOB + 2 * D.G + D.L * L_NSLOT; }
inline int idx_mem(const Dims&, int g, int kv) { return T_NGLOB + 2 * g + kv; }
inline int idx_layer(const Dims& D, int l, int slot) { return T_NGLOB + 2 * D.G + l * L_NSLOT + slot; }

// Whether index i names a tensor the model stores (untied decoder slots
// only exist for untied stacks).
inline bool tensor_exists(const Dims& D, int i) {
  if (i < T_NGLOB + 2 * D.G) return true;
  const int s = (i - T_NGLOB - 2 * D.G) % L_NSLOT;
  return s < L_DWQ || !D.tied;
}

inline std::string tensor_name(const Dims& D, int i) {
  static const char* glob[T_NGLOB] = {"emb", "s_star", "g_mem", "g_merge", "w_gate", "b_gate", "w_state", "g_out", "w_out"};
  static const char* lay[L_NSLOT] = {"wq", "wk", "wv", "wo", "w1", "w2", "w3", "g_ea", "g_ef", "g_dsa", "g_dmem",
                                     "g_dffn", "wq_mem", "wo_mem", "dwq", "dwk", "dwv", "dwo", "dw1", "dw2", "dw3"};
  if (i < T_NGLOB) return glob[i];
  if (i < T_NGLOB + 2 * D.G) {
    const int j = i - T_NGLOB;
    return std::string(j % 2 ? "wv_mem." : "wk_mem.") + std::to_string(j / 2);
  }
  const int j = i - T_NGLOB - 2 * D.G;
  return std::string(lay[j % L_NSLOT]) + "." + std::to_string(j / L_NSLOT);
}

inline void tensor_shape(const Dims& D, int i, int64_t* rows, int64_t* cols) {
  const int64_t d = D.d;
  *rows = d;
  *cols = d;
  if (i < T_NGLOB) {
    switch (i) {
      case T_EMB: case T_WOUT: *rows = D.V; break;
      case T_WGATE: *cols = 2 * d; break;
      case T_WSTATE: break;
      default: *rows = 1;  // s_star and the gains/bias
    }
    return;
  }
  if (i < T_NGLOB + 2 * D.G) return;
  const int s = (i - T_NGLOB - 2 * D.G) % L_NSLOT;
  if (s == L_W1 || s == L_W3 || s == L_DW1 || s == L_DW3) *rows = D.F;
  if (s == L_W2 || s == L_DW2) *cols = D.F;
  if (s >= L_GEA && s <= L_GDFFN) *rows = 1;
}

// ------------------------------------------------------------------ functors
// Y[r][m] = (acc ? Y[r][m] : 0) + sum_k X[r][k] W[m][k]; i = r*M + m.
template <class Real> struct MmNT {
  const Real* X; int64_t ldx; const Real* Wm; int64_t ldw; Real* Y; int64_t ldy; int M, K; int acc;
  RLT_HD void operator()(int64_t i) const {
    const int64_t r = i / M;
    const int m = (int)(i % M);
    const Real* x = X + r * ldx;
    const Real* w = Wm + (int64_t)m * ldw;
    Real s = 0;
    for (int k = 0; k < K; ++k) s += x[k] * w[k];
    Real* y = Y + r * ldy + m;
    *y = acc ? *y + s : s;
  }
};

// Y[r][k] = (acc ? Y[r][k] : 0) + sum_m D[r][m] W[m][k]; i = r*K + k.
template <class Real> struct MmNN {
  const Real* Dm; int64_t ldd; const Real* Wm; int64_t ldw; Real* Y; int64_t ldy; int M, K; int acc;
  RLT_HD void operator()(int64_t i) const {
    const int64_t r = i / K;
    const int k = (int)(i % K);
    const Real* dr = Dm + r * ldd;
    Real s = 0;
    for (int m = 0; m < M; ++m) s += dr[m] * Wm[(int64_t)m * ldw + k];
    Real* y = Y + r * ldy + k;
    *y = acc ? *y + s : s;
  }
};

// Gw[m][k] += sum_r D[r][m] X[r][k]; i = m*K + k.
template <class Real> struct MmTN {
  const Real* Dm; int64_t ldd; const Real* X; int64_t ldx; Real* Gw; int64_t ldg; int R, K;
  RLT_HD void operator()(int64_t i) const {
    const int64_t m = i / K;
    const int k = (int)(i % K);
    Real s = 0;
    for (int r = 0; r < R; ++r) s += Dm[(int64_t)r * ldd + m] * X[(int64_t)r * ldx + k];
    Gw[m * ldg + k] += s;
  }
};

// Y = g * X / rms(X) per row, rinv[r] = 1/rms; i = row.
template <class Real> struct RmsF {
  const Real* X; int64_t ldx; const Real* g; Real* Y; int64_t ldy; Real* rinv; int d; Real eps;
  RLT_HD void operator()(int64_t r) const {
    const Real* x = X + r * ldx;
    Real ss = 0;
    for (int j = 0; j < d; ++j) ss += x[j] * x[j];
    const Real ri = Real(1) / r_sqrt(ss / Real(d) + eps);
    rinv[r] = ri;
    Real* y = Y + r * ldy;
    for (int j = 0; j < d; ++j) y[j] = x[j] * ri * g[j];
  }
};

// dX[r] += adjoint of y = g * x / rms(x) for the row adjoint dY[r]; i = row.
template <class Real> struct RmsBX {
  const Real* dY; int64_t ldd; const Real* X; int64_t ldx; const Real* rinv; const Real* g; Real* dX; int64_t lddx;
  int d;
  RLT_HD void operator()(int64_t r) const {
    const Real* dy = dY + r * ldd;
    const Real* x = X + r * ldx;
    const Real ri = rinv[r];
    Real dot = 0;
    for (int j = 0; j < d; ++j) dot += dy[j] * g[j] * x[j] * ri;
    dot /= Real(d);
    Real* dx = dX + r * lddx;
    for (int j = 0; j < d; ++j) dx[j] += ri * (dy[j] * g[j] - x[j] * ri * dot);
  }
};

// dg[j] += sum_r dY[r][j] X[r][j] rinv[r]; i = j.
template <class Real> struct RmsBG {
  const Real* dY; int64_t ldd; const Real* X; int64_t ldx; const Real* rinv; Real* dg; int R;
  RLT_HD void operator()(int64_t j) const {
    Real s = 0;
    for (int r = 0; r < R; ++r) s += dY[(int64_t)r * ldd + j] * X[(int64_t)r * ldx + j] * rinv[r];
    dg[j] += s;
  }
};

// Rotate-half RoPE in place: within each head the pair (x_i, x_{i+hd/2}) of
// row r turns by sign * pos * inv[i], pos = pos0 + r % T; i = (r*H + h)*hd/2 + i.
template <class Real> struct Rope {
  Real* X; int64_t ldx; int T, pos0, H, hd; const double* inv; double sign;
  RLT_HD void operator()(int64_t i) const {
    const int half = hd / 2;
    const int e = (int)(i % half);
    const int64_t rh = i / half;
    const int h = (int)(rh % H);
    const int64_t r = rh / H;
    const double ang = sign * (double)(pos0 + (int)(r % T)) * inv[e];
    const Real c = (Real)cos(ang), s = (Real)sin(ang);
    Real* x = X + r * ldx + (int64_t)h * hd;
    const Real a = x[e], b = x[e + half];
    x[e] = a * c - b * s;
    x[e + half] = a * s + b * c;
  }
};

// Addressing of attention operands.  Query (b, i) sits at Q + b*q_sb + i*q_si
// (head h at +h*hd); key/value position p of sequence b at K + b*k_sb +
// p*k_sp; the per-head log-sum-exp of query (b, i) at lse + b*l_sb + i*l_si
// + h.  Query i has position qpos0 + i and sees the keys p with
// max(0, pos - win + 1) <= p <= pos.
template <class Real> struct AttnGeom {
  int64_t q_sb, q_si, k_sb, k_sp, l_sb, l_si;
  int Tq, H, hd, qpos0, win;
  RLT_HD int lo(int i) const {
    const int p = qpos0 + i - win + 1;
    return p > 0 ? p : 0;
  }
  RLT_HD int hi(int i) const { return qpos0 + i; }
};

// Forward: O and lse of query (b, i, h); i = ((b*Tq) + i)*H + h.
template <class Real> struct AttnF {
  AttnGeom<Real> g; const Real* Q; const Real* K; const Real* Vv; Real* O; Real* lse; Real scale;
  RLT_HD void operator()(int64_t idx) const {
    const int h = (int)(idx % g.H);
    const int64_t bi = idx / g.H;
    const int i = (int)(bi % g.Tq);
    const int64_t b = bi / g.Tq;
    const Real* q = Q + b * g.q_sb + i * g.q_si + (int64_t)h * g.hd;
    const int lo = g.lo(i), hi = g.hi(i);
    Real mx = -1e30f;
    for (int p = lo; p <= hi; ++p) {
      const Real* k = K + b * g.k_sb + p * g.k_sp + (int64_t)h * g.hd;
      Real s = 0;
      for (int e = 0; e < g.hd; ++e) s += q[e] * k[e];
      s *= scale;
      mx = s > mx ? s : mx;
    }
    Real acc[kMaxHead];
    for (int e = 0; e < g.hd; ++e) acc[e] = 0;
    Real den = 0;
    for (int p = lo; p <= hi; ++p) {
      const Real* k = K + b * g.k_sb + p * g.k_sp + (int64_t)h * g.hd;
      const Real* v = Vv + b * g.k_sb + p * g.k_sp + (int64_t)h * g.hd;
      Real s = 0;
      for (int e = 0; e < g.hd; ++e) s += q[e] * k[e];
      const Real w = r_exp(s * scale - mx);
      den += w;
      for (int e = 0; e < g.hd; ++e) acc[e] += w * v[e];
    }
    Real* o = O + b * g.q_sb + i * g.q_si + (int64_t)h * g.hd;
    for (int e = 0; e < g.hd; ++e) o[e] = acc[e] / den;
    lse[b * g.l_sb + i * g.l_si + h] = mx + r_log(den);
  }
};

// dQ of query (b, i, h) (overwritten): dS_p = P_p (dO.v_p - dO.o), dq = scale
// sum_p dS_p k_p.  O, dO and dQ share the query addressing.
template <class Real> struct AttnBQ {
  AttnGeom<Real> g; const Real* Q; const Real* K; const Real* Vv; const Real* O; const Real* dO; const Real* lse;
  Real* dQ; Real scale;
  RLT_HD void operator()(int64_t idx) const {
    const int h = (int)(idx % g.H);
    const int64_t bi = idx / g.H;
    const int i = (int)(bi % g.Tq);
    const int64_t b = bi / g.Tq;
    const int64_t qo = b * g.q_sb + i * g.q_si + (int64_t)h * g.hd;
    const Real* q = Q + qo;
    const Real* o = O + qo;
    const Real* dout = dO + qo;
    const Real L = lse[b * g.l_sb + i * g.l_si + h];
    Real Dv = 0;
    for (int e = 0; e < g.hd; ++e) Dv += dout[e] * o[e];
    Real acc[kMaxHead];
    for (int e = 0; e < g.hd; ++e) acc[e] = 0;
    for (int p = g.lo(i); p <= g.hi(i); ++p) {
      const Real* k = K + b * g.k_sb + p * g.k_sp + (int64_t)h * g.hd;
      const Real* v = Vv + b * g.k_sb + p * g.k_sp + (int64_t)h * g.hd;
      Real s = 0, dp = 0;
      for (int e = 0; e < g.hd; ++e) {
        s += q[e] * k[e];
        dp += dout[e] * v[e];
      }
      const Real P = r_exp(s * scale - L);
      const Real ds = P * (dp - Dv) * scale;
      for (int e = 0; e < g.hd; ++e) acc[e] += ds * k[e];
    }
    Real* dq = dQ + qo;
    for (int e = 0; e < g.hd; ++e) dq[e] = acc[e];
  }
};

// dK, dV of key position p of sequence b, head h (accumulated): the sum over
// the queries i in [0, Tq) that see p.  Positions p0 + (idx / H) % np.
template <class Real> struct AttnBKV {
  AttnGeom<Real> g; const Real* Q; const Real* K; const Real* Vv; const Real* O; const Real* dO; const Real* lse;
  Real* dK; Real* dV; Real scale; int p0, np;
  RLT_HD void operator()(int64_t idx) const {
    const int h = (int)(idx % g.H);
    const int64_t bp = idx / g.H;
    const int p = p0 + (int)(bp % np);
    const int64_t b = bp / np;
    const int64_t ko = b * g.k_sb + p * g.k_sp + (int64_t)h * g.hd;
    const Real* k = K + ko;
    const Real* v = Vv + ko;
    Real* ak = dK + ko;  // this thread owns the (b, p, h) slices of dK and dV
    Real* av = dV + ko;
    for (int i = 0; i < g.Tq; ++i) {
      if (p < g.lo(i) || p > g.hi(i)) continue;
      const int64_t qo = b * g.q_sb + i * g.q_si + (int64_t)h * g.hd;
      const Real* q = Q + qo;
      const Real* o = O + qo;
      const Real* dout = dO + qo;
      Real s = 0, dp = 0, Dv = 0;
      for (int e = 0; e < g.hd; ++e) {
        s += q[e] * k[e];
        dp += dout[e] * v[e];
        Dv += dout[e] * o[e];
      }
      const Real P = r_exp(s * scale - lse[b * g.l_sb + i * g.l_si + h]);
      const Real ds = P * (dp - Dv) * scale;
      for (int e = 0; e < g.hd; ++e) {
        ak[e] += ds * q[e];
        av[e] += P * dout[e];
      }
    }
  }
};

// SwiGLU: Hs = silu(U1) * U3, rows of F; i = element.
template <class Real> struct SwiF {
  const Real* U1; const Real* U3; Real* Hs;
  RLT_HD void operator()(int64_t i) const { Hs[i] = U1[i] * r_sigmoid(U1[i]) * U3[i]; }
};
template <class Real> struct SwiB {
  const Real* dHs; const Real* U1; const Real* U3; Real* dU1; Real* dU3;
  RLT_HD void operator()(int64_t i) const {
    const Real u = U1[i], sg = r_sigmoid(u);
    dU3[i] = dHs[i] * u * sg;
    dU1[i] = dHs[i] * U3[i] * sg * (Real(1) + u * (Real(1) - sg));
  }
};

// Y[r][j] = X[r][j] over rows of n columns (strided copy); i = r*n + j.
template <class Real> struct Copy2 {
  const Real* X; int64_t ldx; Real* Y; int64_t ldy; int n;
  RLT_HD void operator()(int64_t i) const {
    const int64_t r = i / n;
    const int j = (int)(i % n);
    Y[r * ldy + j] = X[r * ldx + j];
  }
};

// Y[r][j] += a * X[r][j]; i = r*n + j.
template <class Real> struct Axpy2 {
  const Real* X; int64_t ldx; Real* Y; int64_t ldy; int n; Real a;
  RLT_HD void operator()(int64_t i) const {
    const int64_t r = i / n;
    const int j = (int)(i % n);
    Y[r * ldy + j] += a * X[r * ldx + j];
  }
};

// out[j] += sum_r X[r][j]; i = j.
template <class Real> struct ColSum {
  const Real* X; int64_t ldx; Real* out; int R;
  RLT_HD void operator()(int64_t j) const {
    Real s = 0;
    for (int r = 0; r < R; ++r) s += X[(int64_t)r * ldx + j];
    out[j] += s;
  }
};

// Embedding rows: Hh[r] = emb[tok[r]]; i = r*d + j.
template <class Real> struct Embed {
  const int32_t* tok; const Real* emb; Real* Hh; int d;
  RLT_HD void operator()(int64_t i) const {
    const int64_t r = i / d;
    const int j = (int)(i % d);
    Hh[i] = emb[(int64_t)tok[r] * d + j];
  }
};
template <class Real> struct EmbedB {
  const int32_t* tok; const Real* dH; Real* gemb; int d;
  RLT_HD void operator()(int64_t i) const {
    const int64_t r = i / d;
    const int j = (int)(i % d);
    r_atomic_add(gemb + (int64_t)tok[r] * d + j, dH[i]);
  }
};

// Merge, eqs. 2.9-2.11 after its contractions: gate = sigmoid(gpre + bias),
// z = e + alpha * gate * ws (kind 0); or gate = sigmoid(gpre),
// z = gate * e + (1 - gate) * s (kind 1).  e rows strided; i = b*d + j.
template <class Real> struct MergeF {
  const Real* E; int64_t lde; const Real* Sv; const Real* bias; const Real* ws; Real* gate; Real* Z; int d, kind;
  Real alpha;
  RLT_HD void operator()(int64_t i) const {
    const int64_t b = i / d;
    const int j = (int)(i % d);
    const Real e = E[b * lde + j];
    if (kind == 0) {
      const Real gt = r_sigmoid(gate[i] + bias[j]);
      gate[i] = gt;
      Z[i] = e + alpha * gt * ws[i];
    } else {
      const Real gt = r_sigmoid(gate[i]);
      gate[i] = gt;
      Z[i] = gt * e + (Real(1) - gt) * Sv[i];
    }
  }
};

// Merge backward, elementwise part.  kind 0: dE += dz; dws = dz*alpha*gate;
// dgp = dz*alpha*ws*gate*(1-gate).  kind 1: dE += dz*gate; dS = dz*(1-gate);
// dgp = dz*(e-s)*gate*(1-gate).  i = b*d + j.
template <class Real> struct MergeB {
  const Real* dZ; const Real* E; int64_t lde; const Real* Sv; const Real* gate; const Real* ws; Real* dE; Real* dws;
  Real* dgp; Real* dS; int d, kind; Real alpha;
  RLT_HD void operator()(int64_t i) const {
    const int64_t b = i / d;
    const int j = (int)(i % d);
    const Real dz = dZ[i], gt = gate[i];
    if (kind == 0) {
      dE[b * lde + j] += dz;
      dws[i] = dz * alpha * gt;
      dgp[i] = dz * alpha * ws[i] * gt * (Real(1) - gt);
    } else {
      const Real e = E[b * lde + j];
      dE[b * lde + j] += dz * gt;
      dS[i] = dz * (Real(1) - gt);
      dgp[i] = dz * (e - Sv[i]) * gt * (Real(1) - gt);
    }
  }
};

// Readout loss of row b: logp = logits[target] - logsumexp(logits); with
// dlogits != null also the adjoint w * (softmax - onehot).  i = b.
template <class Real> struct Xent {
  const Real* logits; int V; const int32_t* tok; int64_t tok_sb; int t; const Real* wts; int64_t w_sb;
  Real* logp; Real* dlogits;
  RLT_HD void operator()(int64_t b) const {
    const Real* l = logits + b * V;
    Real mx = l[0];
    for (int v = 1; v < V; ++v) mx = l[v] > mx ? l[v] : mx;
    Real den = 0;
    for (int v = 0; v < V; ++v) den += r_exp(l[v] - mx);
    const Real lse = mx + r_log(den);
    const int y = tok[b * tok_sb + t + 1];
    if (logp) logp[b * w_sb + t] = l[y] - lse;
    if (dlogits) {
      const Real w = wts[b * w_sb + t];
      Real* dl = dlogits + b * V;
      for (int v = 0; v < V; ++v) dl[v] = w * (r_exp(l[v] - lse) - (v == y ? Real(1) : Real(0)));
    }
  }
};

// ------------------------------------------------------------------ engine
// Backend concept: T* alloc<T>(n) (zeroed; null and ok() != 0 on failure),
// zero(p, n), copy(dst, src, n) on the backend, upload(dst, host_src, n),
// launch(functor, n) running functor(i) for i in [0, n), ok() (0 when every
// operation so far succeeded; after a failure the backend runs nothing),
// range_push(name) / range_pop() marking a phase for a profiler (may do
// nothing).
template <class BK, class Real>
class Engine {
 public:
  // Wt / Gt: per catalogue index, the tensor as Real [rows][cols] (null for
  // absent untied slots).  Gradients are accumulated into Gt.
  Engine(BK& bk, const Dims& D, const Real* const* Wt, Real* const* Gt) : bk_(bk), D_(D), Wt_(Wt), Gt_(Gt) {}

  // tok [B][S] and wts [B][S-1] on the backend; logp [B][S-1] (may be null).
  // An engine may run several passes of the same sizes and segment length:
  // the first allocates its buffers, later ones set every buffer back to
  // zero, the state the first pass starts from (-1: another segment length).
  int run(const int32_t* tok, const Real* wts, int seg, Real* logp) {
    const Dims& D = D_;
    if (seg < 1) seg = 1;
    if (seg > D.S - 1) seg = D.S - 1;
    if (!ready_) {
      seg_ = seg;
      setup();
      ready_ = true;
    } else {
      if (seg != seg_) return -1;
      for (const auto& b : bufs_) bk_.zero(b.first, b.second);
    }
    if (bk_.ok() != 0) return bk_.ok();
    encoder_forward(tok);
    copy2(Wt(T_SSTAR), 0, s_cur_, D.d, D.B, D.d);  // H_0: s_star in every sequence (eq. 2.3)
    // decoder forward: checkpoints at segment starts, logp of every target
    std::vector<int> starts;
    for (int t = 0; t < D.S - 1; t += seg) starts.push_back(t);
    int si = 0;
    for (int t = 0; t < D.S - 1; ++t) {
      if (si < (int)starts.size() && starts[si] == t) {
        bk_.copy(ckpt_ + (size_t)si * D.B * D.d, s_cur_, (size_t)D.B * D.d);
        ++si;
      }
      step_forward(t, s_cur_, t % seg);
      launch(Xent<Real>{rec(t % seg).logits, D.V, tok, D.S, t, wts, D.S - 1, logp, nullptr}, D.B);
      bk_.copy(s_cur_, rec(t % seg).zout, (size_t)D.B * D.d);
    }
    // backward
    bk_.zero(ds_, (size_t)D.B * D.d);
    for (int k = (int)starts.size() - 1; k >= 0; --k) {
      const int t0 = starts[k], t1 = (t0 + seg < D.S - 1) ? t0 + seg : D.S - 1;
      bk_.copy(s_cur_, ckpt_ + (size_t)k * D.B * D.d, (size_t)D.B * D.d);
      for (int t = t0; t < t1; ++t) {
        step_forward(t, s_cur_, t - t0);
        bk_.copy(s_cur_, rec(t - t0).zout, (size_t)D.B * D.d);
      }
      for (int t = t1 - 1; t >= t0; --t) step_backward(t, t - t0, tok, wts);
      bk_.range_push("rlt_weight_grads");  // a profiler can select the segment's dW contractions
      segment_grads(t0, t1);
      bk_.range_pop();
      memory_pass(t0, t1);
    }
    launch(ColSum<Real>{ds_, D.d, G(T_SSTAR), D.B}, D.d);
    encoder_backward(tok);
    return bk_.ok();
  }

 private:
  // Step records of a segment.  Every field is a slice of a [seg][B][width]
  // block, so that the rows of one field over the whole segment are one
  // contiguous matrix (the weight-gradient contractions and the memory pass
  // run over them).  The d* fields are the step's adjoints at the points
  // where a weight gradient needs them.
  struct LayerRec {
    Real *z, *x, *r1, *q, *o, *lse_sa, *b, *xm, *r2, *qm, *om, *lse_m, *dom, *a, *y, *r3, *u1, *u3, *hs;
    Real *dz, *du1, *du3, *da, *dqm, *db, *dq, *dk, *dv;
  };
  struct StepRec {
    Real *sprev, *rm, *rr, *gate, *ws, *zout, *nrm, *rn, *logits, *et;
    Real *dlog, *dgp, *dws;
    std::vector<LayerRec> lay;
  };
  struct EncRec {
    Real *h, *x, *r1, *q, *k, *v, *o, *lse, *h2, *y, *r2, *u1, *u3, *hs;
  };

  BK& bk_;
  Dims D_;
  const Real* const* Wt_;
  Real* const* Gt_;
  int seg_ = 1;
  bool ready_ = false;
  std::vector<std::pair<Real*, size_t>> bufs_;  // every buffer of setup(), zero at the start of a pass
  std::vector<double> inv_host_;
  double* inv_ = nullptr;
  std::vector<EncRec> enc_;
  Real *e_ = nullptr, *nmem_ = nullptr, *rnmem_ = nullptr;
  std::vector<Real*> memk_, memv_, dmemk_, dmemv_, kh_, vh_, dkh_, dvh_;
  std::vector<StepRec> recs_;
  Real *ckpt_ = nullptr, *s_cur_ = nullptr, *ds_ = nullptr, *de_ = nullptr;
  // step scratch
  Real *dz_, *dx_, *dn_, *dxm_, *dhs_, *dy_, *drm_;
  // encoder scratch
  Real *edh_, *edh2_, *edhs_, *edu1_, *edu3_, *edy_, *edq_, *edk_, *edv_, *edo_, *edx_, *edn_, *edk2_;

  template <class K> void launch(const K& k, int64_t n) {
    if (n > 0) bk_.launch(k, n);
  }
  const Real* Wt(int i) const { return Wt_[i]; }
  Real* G(int i) const { return Gt_[i]; }
  // decoder weight slot: the encoder's matrix when the stacks are tied
  int dslot(int slot) const { return D_.tied ? slot : slot - L_WQ + L_DWQ; }
  const Real* Wl(int l, int slot) const { return Wt_[idx_layer(D_, l, slot)]; }
  Real* Gl(int l, int slot) const { return Gt_[idx_layer(D_, l, slot)]; }
  StepRec& rec(int slot) { return recs_[slot]; }
  Real scale() const { return Real(1) / r_sqrt(Real(D_.hd())); }

  Real* A(size_t n) {
    Real* p = bk_.template alloc<Real>(n);
    bufs_.emplace_back(p, n);
    return p;
  }

  void setup() {
    const Dims& D = D_;
    const size_t B = D.B, S = D.S, d = D.d, F = D.F, H = D.H, N = B * S;
    const int half = D.hd() / 2;
    inv_host_.resize(half);
    for (int i = 0; i < half; ++i) inv_host_[i] = pow(D.rope_base, -2.0 * i / D.hd());
    inv_ = bk_.template alloc<double>(half);
    bk_.upload(inv_, inv_host_.data(), (size_t)half);
    enc_.resize(D.L);
    for (auto& r : enc_) {
      r.h = A(N * d); r.x = A(N * d); r.r1 = A(N); r.q = A(N * d); r.k = A(N * d); r.v = A(N * d); r.o = A(N * d);
      r.lse = A(N * H); r.h2 = A(N * d); r.y = A(N * d); r.r2 = A(N); r.u1 = A(N * F); r.u3 = A(N * F);
      r.hs = A(N * F);
    }
    e_ = A(N * d); nmem_ = A(N * d); rnmem_ = A(N); de_ = A(N * d);
    for (int g = 0; g < D.G; ++g) {
      memk_.push_back(A(N * d)); memv_.push_back(A(N * d));
      dmemk_.push_back(A(N * d)); dmemv_.push_back(A(N * d));
    }
    for (int l = 0; l < D.L; ++l) {
      kh_.push_back(A(N * d)); vh_.push_back(A(N * d));
      dkh_.push_back(A(N * d)); dvh_.push_back(A(N * d));
    }
    recs_.resize(seg_);
    // one [seg][B][width] block per field; step `slot` takes rows slot*B..
    auto field = [&](Real* StepRec::*f, size_t w) {
      Real* blk = A((size_t)seg_ * B * w);
      for (int k = 0; k < seg_; ++k) recs_[k].*f = blk + (size_t)k * B * w;
    };
    auto lfield = [&](Real* LayerRec::*f, size_t w) {
      for (int l = 0; l < D.L; ++l) {
        Real* blk = A((size_t)seg_ * B * w);
        for (int k = 0; k < seg_; ++k) recs_[k].lay[l].*f = blk + (size_t)k * B * w;
      }
    };
    for (auto& r : recs_) r.lay.resize(D.L);
    field(&StepRec::sprev, d); field(&StepRec::rm, d); field(&StepRec::rr, 1); field(&StepRec::gate, d);
    field(&StepRec::ws, d); field(&StepRec::zout, d); field(&StepRec::nrm, d); field(&StepRec::rn, 1);
    field(&StepRec::logits, D.V); field(&StepRec::et, d); field(&StepRec::dlog, D.V); field(&StepRec::dgp, d);
    field(&StepRec::dws, d);
    for (Real* LayerRec::*f : {&LayerRec::z, &LayerRec::x, &LayerRec::q, &LayerRec::o, &LayerRec::b, &LayerRec::xm,
                               &LayerRec::qm, &LayerRec::om, &LayerRec::dom, &LayerRec::a, &LayerRec::y,
                               &LayerRec::dz, &LayerRec::da, &LayerRec::dqm, &LayerRec::db, &LayerRec::dq,
                               &LayerRec::dk, &LayerRec::dv})
      lfield(f, d);
    for (Real* LayerRec::*f : {&LayerRec::r1, &LayerRec::r2, &LayerRec::r3}) lfield(f, 1);
    for (Real* LayerRec::*f : {&LayerRec::lse_sa, &LayerRec::lse_m}) lfield(f, H);
    for (Real* LayerRec::*f : {&LayerRec::u1, &LayerRec::u3, &LayerRec::hs, &LayerRec::du1, &LayerRec::du3})
      lfield(f, F);
    const size_t nseg = (S - 1 + seg_ - 1) / seg_;
    ckpt_ = A(nseg * B * d); s_cur_ = A(B * d); ds_ = A(B * d);
    dz_ = A(B * d); dx_ = A(B * d); dn_ = A(B * d); dxm_ = A(B * d); dhs_ = A(B * F); dy_ = A(B * d);
    drm_ = A(B * d);
    edh_ = A(N * d); edh2_ = A(N * d); edhs_ = A(N * F); edu1_ = A(N * F); edu3_ = A(N * F); edy_ = A(N * d);
    edq_ = A(N * d); edk_ = A(N * d); edv_ = A(N * d); edo_ = A(N * d); edx_ = A(N * d); edn_ = A(N * d);
    edk2_ = A(N * d);
  }

  // ---- shorthand launches over R rows
  void mm_nt(const Real* X, int64_t ldx, const Real* W, int64_t ldw, Real* Y, int64_t ldy, int64_t R, int M, int K,
             int acc) {
    launch(MmNT<Real>{X, ldx, W, ldw, Y, ldy, M, K, acc}, R * M);
  }
  void mm_nn(const Real* Dm, int64_t ldd, const Real* W, int64_t ldw, Real* Y, int64_t ldy, int64_t R, int M, int K,
             int acc) {
    launch(MmNN<Real>{Dm, ldd, W, ldw, Y, ldy, M, K, acc}, R * K);
  }
  void mm_tn(const Real* Dm, int64_t ldd, const Real* X, int64_t ldx, Real* Gw, int64_t ldg, int R, int M, int K) {
    launch(MmTN<Real>{Dm, ldd, X, ldx, Gw, ldg, R, K}, (int64_t)M * K);
  }
  void rms_f(const Real* X, int64_t ldx, const Real* g, Real* Y, Real* rinv, int64_t R) {
    launch(RmsF<Real>{X, ldx, g, Y, D_.d, rinv, D_.d, (Real)D_.eps}, R);
  }
  // dX += adjoint; dg += gain adjoint
  void rms_b(const Real* dY, const Real* X, int64_t ldx, const Real* rinv, const Real* g, Real* dX, Real* dg, int R) {
    launch(RmsBX<Real>{dY, D_.d, X, ldx, rinv, g, dX, D_.d, D_.d}, R);
    launch(RmsBG<Real>{dY, D_.d, X, ldx, rinv, dg, R}, D_.d);
  }
  void rope(Real* X, int64_t ldx, int64_t R, int T, int pos0, double sign) {
    const int half = D_.hd() / 2;
    launch(Rope<Real>{X, ldx, T, pos0, D_.H, D_.hd(), inv_, sign}, R * D_.H * half);
  }
  void copy2(const Real* X, int64_t ldx, Real* Y, int64_t ldy, int64_t R, int n) {
    launch(Copy2<Real>{X, ldx, Y, ldy, n}, R * n);
  }
  void axpy2(const Real* X, int64_t ldx, Real* Y, int64_t ldy, int64_t R, int n, Real a) {
    launch(Axpy2<Real>{X, ldx, Y, ldy, n, a}, R * n);
  }
  // geometry of one decoder step's B queries at position t over keys stored
  // [B][S][d]
  AttnGeom<Real> step_geom(int t, int win) const {
    const Dims& D = D_;
    return AttnGeom<Real>{(int64_t)D.d, 0, (int64_t)D.S * D.d, (int64_t)D.d, (int64_t)D.H, 0, 1, D.H, D.hd(), t, win};
  }
  int full_win() const { return D_.S + 1; }

  // ---- encoder (eq. 2.1) and memory (eq. 2.2), token-parallel over N = B*S rows
  void encoder_forward(const int32_t* tok) {
    const Dims& D = D_;
    const int64_t N = (int64_t)D.B * D.S;
    const int d = D.d, F = D.F;
    launch(Embed<Real>{tok, Wt(T_EMB), enc_[0].h, d}, N * d);
    const AttnGeom<Real> gq{(int64_t)D.S * d, d, (int64_t)D.S * d, d, (int64_t)D.S * D.H, D.H, D.S, D.H, D.hd(), 0,
                            full_win()};
    for (int l = 0; l < D.L; ++l) {
      EncRec& r = enc_[l];
      rms_f(r.h, d, Wl(l, L_GEA), r.x, r.r1, N);
      mm_nt(r.x, d, Wl(l, L_WQ), d, r.q, d, N, d, d, 0);
      mm_nt(r.x, d, Wl(l, L_WK), d, r.k, d, N, d, d, 0);
      mm_nt(r.x, d, Wl(l, L_WV), d, r.v, d, N, d, d, 0);
      rope(r.q, d, N, D.S, 0, 1.0);
      rope(r.k, d, N, D.S, 0, 1.0);
      launch(AttnF<Real>{gq, r.q, r.k, r.v, r.o, r.lse, scale()}, N * D.H);
      copy2(r.h, d, r.h2, d, N, d);
      mm_nt(r.o, d, Wl(l, L_WO), d, r.h2, d, N, d, d, 1);
      rms_f(r.h2, d, Wl(l, L_GEF), r.y, r.r2, N);
      mm_nt(r.y, d, Wl(l, L_W1), d, r.u1, F, N, F, d, 0);
      mm_nt(r.y, d, Wl(l, L_W3), d, r.u3, F, N, F, d, 0);
      launch(SwiF<Real>{r.u1, r.u3, r.hs}, N * F);
      Real* out = l + 1 < D.L ? enc_[l + 1].h : e_;
      copy2(r.h2, d, out, d, N, d);
      mm_nt(r.hs, F, Wl(l, L_W2), F, out, d, N, d, F, 1);
    }
    rms_f(e_, d, Wt(T_GMEM), nmem_, rnmem_, N);
    for (int g = 0; g < D.G; ++g) {
      mm_nt(nmem_, d, Wt(idx_mem(D, g, 0)), d, memk_[g], d, N, d, d, 0);
      mm_nt(nmem_, d, Wt(idx_mem(D, g, 1)), d, memv_[g], d, N, d, d, 0);
      rope(memk_[g], d, N, D.S, 0, 1.0);
    }
  }

  // ---- one decoder transition at 0-based position t (eqs. 2.4-2.6, 2.9-2.16)
  void step_forward(int t, const Real* s_in, int slot) {
    const Dims& D = D_;
    const int d = D.d, F = D.F, B = D.B;
    const int64_t lde = (int64_t)D.S * d;
    StepRec& R = rec(slot);
    copy2(e_ + (int64_t)t * d, lde, R.et, d, B, d);  // e_t rows of the step, contiguous
    const Real* et = R.et;
    copy2(s_in, d, R.sprev, d, B, d);
    if (D.merge_kind == 0) {
      rms_f(R.sprev, d, Wt(T_GMERGE), R.rm, R.rr, B);
      mm_nt(et, d, Wt(T_WGATE), 2 * d, R.gate, d, B, d, d, 0);
      mm_nt(R.rm, d, Wt(T_WGATE) + d, 2 * d, R.gate, d, B, d, d, 1);
      mm_nt(R.rm, d, Wt(T_WSTATE), d, R.ws, d, B, d, d, 0);
    } else {
      mm_nt(et, d, Wt(T_WGATE), 2 * d, R.gate, d, B, d, d, 0);
      mm_nt(R.sprev, d, Wt(T_WGATE) + d, 2 * d, R.gate, d, B, d, d, 1);
    }
    launch(MergeF<Real>{et, d, R.sprev, Wt(T_BGATE), R.ws, R.gate, R.lay[0].z, d, D.merge_kind, (Real)D.alpha},
           (int64_t)B * d);
    for (int l = 0; l < D.L; ++l) {
      LayerRec& r = R.lay[l];
      const int grp = D.G == 1 ? 0 : l;
      rms_f(r.z, d, Wl(l, L_GDSA), r.x, r.r1, B);
      mm_nt(r.x, d, Wl(l, dslot(L_WQ)), d, r.q, d, B, d, d, 0);
      Real* kt = kh_[l] + (int64_t)t * d;
      Real* vt = vh_[l] + (int64_t)t * d;
      mm_nt(r.x, d, Wl(l, dslot(L_WK)), d, kt, lde, B, d, d, 0);
      mm_nt(r.x, d, Wl(l, dslot(L_WV)), d, vt, lde, B, d, d, 0);
      rope(r.q, d, B, 1, t, 1.0);
      rope(kt, lde, B, 1, t, 1.0);
      launch(AttnF<Real>{step_geom(t, D.W), r.q, kh_[l], vh_[l], r.o, r.lse_sa, scale()}, (int64_t)B * D.H);
      copy2(r.z, d, r.b, d, B, d);
      mm_nt(r.o, d, Wl(l, dslot(L_WO)), d, r.b, d, B, d, d, 1);
      rms_f(r.b, d, Wl(l, L_GDMEM), r.xm, r.r2, B);
      mm_nt(r.xm, d, Wl(l, L_WQM), d, r.qm, d, B, d, d, 0);
      rope(r.qm, d, B, 1, t, 1.0);
      launch(AttnF<Real>{step_geom(t, full_win()), r.qm, memk_[grp], memv_[grp], r.om, r.lse_m, scale()},
             (int64_t)B * D.H);
      copy2(r.b, d, r.a, d, B, d);
      mm_nt(r.om, d, Wl(l, L_WOM), d, r.a, d, B, d, d, 1);
      rms_f(r.a, d, Wl(l, L_GDFFN), r.y, r.r3, B);
      mm_nt(r.y, d, Wl(l, dslot(L_W1)), d, r.u1, F, B, F, d, 0);
      mm_nt(r.y, d, Wl(l, dslot(L_W3)), d, r.u3, F, B, F, d, 0);
      launch(SwiF<Real>{r.u1, r.u3, r.hs}, (int64_t)B * F);
      Real* out = l + 1 < D.L ? R.lay[l + 1].z : R.zout;
      copy2(r.a, d, out, d, B, d);
      mm_nt(r.hs, F, Wl(l, dslot(L_W2)), F, out, d, B, d, F, 1);
    }
    rms_f(R.zout, d, Wt(T_GOUT), R.nrm, R.rn, B);
    mm_nt(R.nrm, d, Wt(T_WOUT), d, R.logits, D.V, B, D.V, d, 0);
  }

  // ---- reverse of the transition at position t; ds_ holds dL/ds_t on entry
  // and dL/ds_{t-1} on exit.  The adjoints a weight gradient needs are left
  // in the step's record; segment_grads turns them into the gradients.
  void step_backward(int t, int slot, const int32_t* tok, const Real* wts) {
    const Dims& D = D_;
    const int d = D.d, F = D.F, B = D.B;
    const int64_t lde = (int64_t)D.S * d;
    StepRec& R = rec(slot);
    launch(Xent<Real>{R.logits, D.V, tok, D.S, t, wts, D.S - 1, nullptr, R.dlog}, B);
    mm_nn(R.dlog, D.V, Wt(T_WOUT), d, dn_, d, B, D.V, d, 0);
    Real* dz = R.lay[D.L - 1].dz;
    copy2(ds_, d, dz, d, B, d);
    rms_b(dn_, R.zout, d, R.rn, Wt(T_GOUT), dz, G(T_GOUT), B);
    for (int l = D.L - 1; l >= 0; --l) {
      LayerRec& r = R.lay[l];
      const int grp = D.G == 1 ? 0 : l;
      // FFN (eq. 2.16): z_out = a + W2 (silu(W1 y) * W3 y), y = RMSNorm(a)
      mm_nn(r.dz, d, Wl(l, dslot(L_W2)), F, dhs_, F, B, d, F, 0);
      launch(SwiB<Real>{dhs_, r.u1, r.u3, r.du1, r.du3}, (int64_t)B * F);
      mm_nn(r.du1, F, Wl(l, dslot(L_W1)), d, dy_, d, B, F, d, 0);
      mm_nn(r.du3, F, Wl(l, dslot(L_W3)), d, dy_, d, B, F, d, 1);
      copy2(r.dz, d, r.da, d, B, d);
      rms_b(dy_, r.a, d, r.r3, Wl(l, L_GDFFN), r.da, Gl(l, L_GDFFN), B);
      // memory cross-attention (eq. 2.15): a = b + W_om attn(q_m, M_<=t)
      mm_nn(r.da, d, Wl(l, L_WOM), d, r.dom, d, B, d, d, 0);
      launch(AttnBQ<Real>{step_geom(t, full_win()), r.qm, memk_[grp], memv_[grp], r.om, r.dom, r.lse_m, r.dqm,
                          scale()},
             (int64_t)B * D.H);
      rope(r.dqm, d, B, 1, t, -1.0);
      mm_nn(r.dqm, d, Wl(l, L_WQM), d, dxm_, d, B, d, d, 0);
      copy2(r.da, d, r.db, d, B, d);
      rms_b(dxm_, r.b, d, r.r2, Wl(l, L_GDMEM), r.db, Gl(l, L_GDMEM), B);
      // SWA (eqs. 2.12-2.14): b = z + W_o attn(q, window of K/V)
      mm_nn(r.db, d, Wl(l, dslot(L_WO)), d, dx_, d, B, d, d, 0);  // dx_ = adjoint of the attention output
      const AttnGeom<Real> gw = step_geom(t, D.W);
      launch(AttnBQ<Real>{gw, r.q, kh_[l], vh_[l], r.o, dx_, r.lse_sa, r.dq, scale()}, (int64_t)B * D.H);
      const int p0 = gw.lo(0), np = t - p0 + 1;
      launch(AttnBKV<Real>{gw, r.q, kh_[l], vh_[l], r.o, dx_, r.lse_sa, dkh_[l], dvh_[l], scale(), p0, np},
             (int64_t)B * np * D.H);
      // the adjoints of this position's key and value are complete now
      copy2(dkh_[l] + (int64_t)t * d, lde, r.dk, d, B, d);
      copy2(dvh_[l] + (int64_t)t * d, lde, r.dv, d, B, d);
      rope(r.dk, d, B, 1, t, -1.0);
      rope(r.dq, d, B, 1, t, -1.0);
      mm_nn(r.dq, d, Wl(l, dslot(L_WQ)), d, dx_, d, B, d, d, 0);
      mm_nn(r.dk, d, Wl(l, dslot(L_WK)), d, dx_, d, B, d, d, 1);
      mm_nn(r.dv, d, Wl(l, dslot(L_WV)), d, dx_, d, B, d, d, 1);
      Real* dz_in = l > 0 ? R.lay[l - 1].dz : dz_;  // adjoint of this layer's input
      copy2(r.db, d, dz_in, d, B, d);
      rms_b(dx_, r.z, d, r.r1, Wl(l, L_GDSA), dz_in, Gl(l, L_GDSA), B);
    }
    // merge (eqs. 2.9-2.11 or the convex gate); dz_ = dL/du_t
    Real* det = de_ + (int64_t)t * d;
    // (e_t and its adjoint share MergeB's row stride: both in the [B][S][d] layout)
    launch(MergeB<Real>{dz_, e_ + (int64_t)t * d, lde, R.sprev, R.gate, R.ws, det, R.dws, R.dgp, ds_, d, D.merge_kind,
                        (Real)D.alpha},
           (int64_t)B * d);
    mm_nn(R.dgp, d, Wt(T_WGATE), 2 * d, det, lde, B, d, d, 1);
    if (D.merge_kind == 0) {
      mm_nn(R.dws, d, Wt(T_WSTATE), d, drm_, d, B, d, d, 0);
      mm_nn(R.dgp, d, Wt(T_WGATE) + d, 2 * d, drm_, d, B, d, d, 1);
      bk_.zero(ds_, (size_t)B * d);
      rms_b(drm_, R.sprev, d, R.rr, Wt(T_GMERGE), ds_, G(T_GMERGE), B);
    } else {
      mm_nn(R.dgp, d, Wt(T_WGATE) + d, 2 * d, ds_, d, B, d, d, 1);
    }
  }

  // ---- weight gradients of the segment's steps t0..t1-1: dW += dY^T X, one
  // contraction per weight over the (t1-t0)*B rows of the step records
  void segment_grads(int t0, int t1) {
    const Dims& D = D_;
    const int d = D.d, F = D.F;
    const int R = (t1 - t0) * D.B;
    const StepRec& S0 = rec(0);
    mm_tn(S0.dlog, D.V, S0.nrm, d, G(T_WOUT), d, R, D.V, d);
    mm_tn(S0.dgp, d, S0.et, d, G(T_WGATE), 2 * d, R, d, d);
    if (D.merge_kind == 0) {
      launch(ColSum<Real>{S0.dgp, d, G(T_BGATE), R}, d);
      mm_tn(S0.dgp, d, S0.rm, d, G(T_WGATE) + d, 2 * d, R, d, d);
      mm_tn(S0.dws, d, S0.rm, d, G(T_WSTATE), d, R, d, d);
    } else {
      mm_tn(S0.dgp, d, S0.sprev, d, G(T_WGATE) + d, 2 * d, R, d, d);
    }
    for (int l = 0; l < D.L; ++l) {
      const LayerRec& r = S0.lay[l];
      mm_tn(r.dz, d, r.hs, F, Gl(l, dslot(L_W2)), F, R, d, F);
      mm_tn(r.du1, F, r.y, d, Gl(l, dslot(L_W1)), d, R, F, d);
      mm_tn(r.du3, F, r.y, d, Gl(l, dslot(L_W3)), d, R, F, d);
      mm_tn(r.da, d, r.om, d, Gl(l, L_WOM), d, R, d, d);
      mm_tn(r.dqm, d, r.xm, d, Gl(l, L_WQM), d, R, d, d);
      mm_tn(r.db, d, r.o, d, Gl(l, dslot(L_WO)), d, R, d, d);
      mm_tn(r.dq, d, r.x, d, Gl(l, dslot(L_WQ)), d, R, d, d);
      mm_tn(r.dk, d, r.x, d, Gl(l, dslot(L_WK)), d, R, d, d);
      mm_tn(r.dv, d, r.x, d, Gl(l, dslot(L_WV)), d, R, d, d);
    }
  }

  // ---- memory key/value adjoints of the segment's queries t0..t1-1: per
  // layer one token-parallel pass over the memory positions 0..t1-1, each
  // position gathering the queries of the segment that see it (p <= t)
  void memory_pass(int t0, int t1) {
    const Dims& D = D_;
    const int d = D.d, B = D.B;
    for (int l = 0; l < D.L; ++l) {
      const int grp = D.G == 1 ? 0 : l;
      const LayerRec& r = rec(0).lay[l];
      const AttnGeom<Real> g{(int64_t)d, (int64_t)B * d, (int64_t)D.S * d, (int64_t)d, (int64_t)D.H,
                             (int64_t)B * D.H, t1 - t0, D.H, D.hd(), t0, full_win()};
      launch(AttnBKV<Real>{g, r.qm, memk_[grp], memv_[grp], r.om, r.dom, r.lse_m, dmemk_[grp], dmemv_[grp], scale(),
                           0, t1},
             (int64_t)B * t1 * D.H);
    }
  }

  // ---- encoder backward (token-parallel); de_ holds dL/de on entry
  void encoder_backward(const int32_t* tok) {
    const Dims& D = D_;
    const int64_t N = (int64_t)D.B * D.S;
    const int d = D.d, F = D.F;
    // memory projection: k^g = RoPE(W_k^g n), v^g = W_v^g n, n = RMSNorm(e)
    bk_.zero(edn_, (size_t)N * d);
    for (int g = 0; g < D.G; ++g) {
      copy2(dmemk_[g], d, edk2_, d, N, d);
      rope(edk2_, d, N, D.S, 0, -1.0);
      mm_tn(edk2_, d, nmem_, d, G(idx_mem(D, g, 0)), d, (int)N, d, d);
      mm_tn(dmemv_[g], d, nmem_, d, G(idx_mem(D, g, 1)), d, (int)N, d, d);
      mm_nn(edk2_, d, Wt(idx_mem(D, g, 0)), d, edn_, d, N, d, d, 1);
      mm_nn(dmemv_[g], d, Wt(idx_mem(D, g, 1)), d, edn_, d, N, d, d, 1);
    }
    copy2(de_, d, edh_, d, N, d);
    rms_b(edn_, e_, d, rnmem_, Wt(T_GMEM), edh_, G(T_GMEM), (int)N);
    const AttnGeom<Real> gq{(int64_t)D.S * d, d, (int64_t)D.S * d, d, (int64_t)D.S * D.H, D.H, D.S, D.H, D.hd(), 0,
                            full_win()};
    for (int l = D.L - 1; l >= 0; --l) {
      EncRec& r = enc_[l];
      mm_tn(edh_, d, r.hs, F, Gl(l, L_W2), F, (int)N, d, F);
      mm_nn(edh_, d, Wl(l, L_W2), F, edhs_, F, N, d, F, 0);
      launch(SwiB<Real>{edhs_, r.u1, r.u3, edu1_, edu3_}, N * F);
      mm_tn(edu1_, F, r.y, d, Gl(l, L_W1), d, (int)N, F, d);
      mm_tn(edu3_, F, r.y, d, Gl(l, L_W3), d, (int)N, F, d);
      mm_nn(edu1_, F, Wl(l, L_W1), d, edy_, d, N, F, d, 0);
      mm_nn(edu3_, F, Wl(l, L_W3), d, edy_, d, N, F, d, 1);
      copy2(edh_, d, edh2_, d, N, d);
      rms_b(edy_, r.h2, d, r.r2, Wl(l, L_GEF), edh2_, Gl(l, L_GEF), (int)N);
      mm_tn(edh2_, d, r.o, d, Gl(l, L_WO), d, (int)N, d, d);
      mm_nn(edh2_, d, Wl(l, L_WO), d, edo_, d, N, d, d, 0);
      launch(AttnBQ<Real>{gq, r.q, r.k, r.v, r.o, edo_, r.lse, edq_, scale()}, N * D.H);
      bk_.zero(edk_, (size_t)N * d);
      bk_.zero(edv_, (size_t)N * d);
      launch(AttnBKV<Real>{gq, r.q, r.k, r.v, r.o, edo_, r.lse, edk_, edv_, scale(), 0, D.S}, N * D.H);
      rope(edq_, d, N, D.S, 0, -1.0);
      rope(edk_, d, N, D.S, 0, -1.0);
      mm_tn(edq_, d, r.x, d, Gl(l, L_WQ), d, (int)N, d, d);
      mm_tn(edk_, d, r.x, d, Gl(l, L_WK), d, (int)N, d, d);
      mm_tn(edv_, d, r.x, d, Gl(l, L_WV), d, (int)N, d, d);
      mm_nn(edq_, d, Wl(l, L_WQ), d, edx_, d, N, d, d, 0);
      mm_nn(edk_, d, Wl(l, L_WK), d, edx_, d, N, d, d, 1);
      mm_nn(edv_, d, Wl(l, L_WV), d, edx_, d, N, d, d, 1);
      copy2(edh2_, d, edh_, d, N, d);
      rms_b(edx_, r.h, d, r.r1, Wl(l, L_GEA), edh_, Gl(l, L_GEA), (int)N);
    }
    launch(EmbedB<Real>{tok, edh_, G(T_EMB), d}, N * d);
  }
};

}  // namespace bptt
}  // namespace rlt
