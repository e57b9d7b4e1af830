// epilogue.cuh -- fused GEMM epilogues.  Every GEMM here computes
// C[n][m] = sum_k X[n][k] * W[m][k] (W = weight rows, X = activation rows) and
// hands each accumulator to one of these functors, which fold the elementwise
// step that follows the contraction in "Recurrent Looped Transformer":
//   STORE   plain store (fp32 or the activation type)
//   RESID   residual add into the fp32 stream (eqs. 2.14-2.16 and the encoder)
//   SWIGLU  silu(gate) * up on interleaved W1/W3 rows (row 2i = W1 row i,
//           row 2i+1 = W3 row i); writes column i
//   GATE    sigmoid(acc + b_g) (eq. 2.10)
//   MERGE   u = e + alpha * g * acc with acc = W_s r (eq. 2.11)
//   CONVEX  g = sigmoid(acc), u = g*e + (1-g)*s (convex merge, in place on s)
#pragma once
#include "common.cuh"

namespace rlt {

enum EpiKind : int {
  EPI_STORE = 0,
  EPI_RESID = 1,
  EPI_SWIGLU = 2,
  EPI_GATE = 3,
  EPI_MERGE = 4,
  EPI_CONVEX = 5,
};

struct EpiParams {
  void* out;            // output base
  RowMap out_map;       // row addressing of the output
  int out_bf16;         // STORE/SWIGLU: 1 = bf16 output, 0 = fp32
  const float* aux0;    // MERGE/CONVEX: e_t rows
  RowMap aux0_map;
  const float* aux1;    // MERGE: gate rows
  int64_t ld_aux1;
  const void* bias;     // GATE: b_g [M], model storage type
  int bias_bf16;
  float alpha;          // MERGE: feedback scale
  // RMSNorm of the next sublayer folded into the epilogues.  A producer
  // (RESID/MERGE/CONVEX with zb != null) also writes zb[n][m] =
  // bf16(gamma_next[m] * z) and, per 128-row weight tile mt, the partial sum
  // ss_out[mt][n] of z^2 over that tile's rows.  A consumer (STORE/SWIGLU
  // with ss_in != null) reads such a zb as its activation operand and scales
  // each accumulator of row n by 1/sqrt(norm_scale * sum_mt ss_in[mt][n] +
  // norm_eps): gamma * z / rms(z) times a weight row equals 1/rms(z) times
  // the weight row applied to gamma * z.
  bf16* zb;
  int64_t ld_zb;
  const void* gamma_next;
  int gamma_bf16;
  float* ss_out;
  const float* ss_in;
  int n_ss;
  int64_t ss_ld;
  float norm_scale;
  float norm_eps;
};

// The fast division (__fdividef) keeps the epilogue free of the IEEE division
// subroutine and its branches; 1 + exp(-x) lies in [1, inf), where it is
// accurate to a few ulp and returns 0 for an infinite divisor (the correct
// limits sigmoid -> 0, silu -> -0).
__device__ __forceinline__ float sigmoidf_(float x) { return __fdividef(1.0f, 1.0f + __expf(-x)); }
__device__ __forceinline__ float siluf_(float x) { return __fdividef(x, 1.0f + __expf(-x)); }

__device__ __forceinline__ float load_bias(const EpiParams& p, int m) {
  return p.bias_bf16 ? __bfloat162float(reinterpret_cast<const bf16*>(p.bias)[m])
                     : reinterpret_cast<const float*>(p.bias)[m];
}

// Does the epilogue read the aux0 rows (e_t)?
template <int EPI>
__device__ __forceinline__ constexpr bool epi_uses_aux0() {
  return EPI == EPI_MERGE || EPI == EPI_CONVEX;
}

// Non-pair epilogues: one accumulator for output (n, m); `orow` and `arow`
// are the precomputed row offsets out_map.off(n) and aux0_map.off(n).
template <int EPI>
__device__ __forceinline__ void epi_apply_at(const EpiParams& p, int64_t n, int64_t orow, int64_t arow, int m,
                                             float acc) {
  if constexpr (EPI == EPI_STORE) {
    const int64_t o = orow + m;
    if (p.out_bf16) reinterpret_cast<bf16*>(p.out)[o] = __float2bfloat16_rn(acc);
    else reinterpret_cast<float*>(p.out)[o] = acc;
  } else if constexpr (EPI == EPI_RESID) {
    float* o = reinterpret_cast<float*>(p.out) + orow + m;
    *o = *o + acc;
  } else if constexpr (EPI == EPI_GATE) {
    reinterpret_cast<float*>(p.out)[orow + m] = sigmoidf_(acc + load_bias(p, m));
  } else if constexpr (EPI == EPI_MERGE) {
    const float e = p.aux0[arow + m];
    const float g = p.aux1[n * p.ld_aux1 + m];
    reinterpret_cast<float*>(p.out)[orow + m] = e + p.alpha * g * acc;
  } else if constexpr (EPI == EPI_CONVEX) {
    const float e = p.aux0[arow + m];
    float* o = reinterpret_cast<float*>(p.out) + orow + m;
    const float g = sigmoidf_(acc);
    *o = g * e + (1.0f - g) * (*o);
  }
}

template <int EPI>
__device__ __forceinline__ void epi_apply(const EpiParams& p, int64_t n, int m, float acc) {
  epi_apply_at<EPI>(p, n, p.out_map.off(n), epi_uses_aux0<EPI>() ? p.aux0_map.off(n) : 0, m, acc);
}

// Two-phase form of the same epilogues, so that a thread can issue the loads
// of many outputs before any store (read-modify-write epilogues would
// otherwise wait on one load per output): epi_load fetches what the
// epilogue reads (old residual, e_t, gate), epi_store finishes it.  What
// depends on the output feature m alone (bias, next gain) is loaded once per
// thread into EpiRowConst; the output type (OBF: bf16) and the folded-norm
// operand (ZB) are template parameters, so a run of outputs compiles to
// straight-line code.
struct EpiPre {
  float a, b;
};

struct EpiRowConst {
  float bias;   // GATE: b_g[m]
  float gamma;  // producers with zb: gamma_next[m]
};

// Does the epilogue produce a residual-stream value z (and so may feed the
// next sublayer's folded RMSNorm)?
template <int EPI>
__device__ __forceinline__ constexpr bool epi_produces_z() {
  return EPI == EPI_RESID || EPI == EPI_MERGE || EPI == EPI_CONVEX;
}

__device__ __forceinline__ float load_gamma(const EpiParams& p, int m) {
  return p.gamma_bf16 ? __bfloat162float(reinterpret_cast<const bf16*>(p.gamma_next)[m])
                      : reinterpret_cast<const float*>(p.gamma_next)[m];
}

template <int EPI>
__device__ __forceinline__ EpiRowConst epi_row_const(const EpiParams& p, int m) {
  EpiRowConst r{0.f, 0.f};
  if constexpr (EPI == EPI_GATE) r.bias = load_bias(p, m);
  if constexpr (epi_produces_z<EPI>()) {
    if (p.zb != nullptr) r.gamma = load_gamma(p, m);
  }
  return r;
}

template <int EPI>
__device__ __forceinline__ EpiPre epi_load(const EpiParams& p, int64_t n, int64_t orow, int64_t arow, int m) {
  EpiPre r{0.f, 0.f};
  if constexpr (EPI == EPI_RESID) {
    r.a = reinterpret_cast<const float*>(p.out)[orow + m];
  } else if constexpr (EPI == EPI_MERGE) {
    r.a = p.aux0[arow + m];
    r.b = p.aux1[n * p.ld_aux1 + m];
  } else if constexpr (EPI == EPI_CONVEX) {
    r.a = p.aux0[arow + m];
    r.b = reinterpret_cast<const float*>(p.out)[orow + m];
  }
  return r;
}

// Finishes the epilogue of output (n, m); returns z for producers (0 else).
template <int EPI, bool OBF, bool ZB>
__device__ __forceinline__ float epi_store(const EpiParams& p, const EpiRowConst& rc, int64_t n, int64_t orow, int m,
                                           float acc, EpiPre pre) {
  float z = 0.f;
  if constexpr (EPI == EPI_STORE) {
    if constexpr (OBF) reinterpret_cast<bf16*>(p.out)[orow + m] = __float2bfloat16_rn(acc);
    else reinterpret_cast<float*>(p.out)[orow + m] = acc;
  } else if constexpr (EPI == EPI_RESID) {
    z = pre.a + acc;
    reinterpret_cast<float*>(p.out)[orow + m] = z;
  } else if constexpr (EPI == EPI_GATE) {
    reinterpret_cast<float*>(p.out)[orow + m] = sigmoidf_(acc + rc.bias);
  } else if constexpr (EPI == EPI_MERGE) {
    z = pre.a + p.alpha * pre.b * acc;
    reinterpret_cast<float*>(p.out)[orow + m] = z;
  } else if constexpr (EPI == EPI_CONVEX) {
    const float g = sigmoidf_(acc);
    z = g * pre.a + (1.0f - g) * pre.b;
    reinterpret_cast<float*>(p.out)[orow + m] = z;
  }
  if constexpr (ZB && epi_produces_z<EPI>()) p.zb[n * p.ld_zb + m] = __float2bfloat16_rn(rc.gamma * z);
  return z;
}

// SWIGLU pair epilogue: gate accumulator of row 2i and up accumulator of row
// 2i+1 give hidden column i.
__device__ __forceinline__ void epi_swiglu_at(const EpiParams& p, int64_t orow, int i, float gate, float up) {
  const float h = siluf_(gate) * up;
  const int64_t o = orow + i;
  if (p.out_bf16) reinterpret_cast<bf16*>(p.out)[o] = __float2bfloat16_rn(h);
  else reinterpret_cast<float*>(p.out)[o] = h;
}

__device__ __forceinline__ void epi_swiglu(const EpiParams& p, int64_t n, int i, float gate, float up) {
  epi_swiglu_at(p, p.out_map.off(n), i, gate, up);
}

}  // namespace rlt
