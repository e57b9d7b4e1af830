// attn_decode.cu -- one-query-per-(sequence, head) attention of the decoder
// step.  These kernels carry almost all of a step's HBM traffic: every
// decoder layer reads its SWA ring (eq. 2.14) and the prefix of the encoder
// memory M_<=t (eq. 2.15), and the encoder step reads its cache C^E (eq. 2.8).
//
// Layout: keys and values of one (sequence, head) are contiguous rows of hd
// elements ([B][H][rows][hd]), so a block streams them with 16-byte vector
// loads: hd/8 lanes cover one key, a warp covers 32/(hd/8) keys per load, the
// four warps of a block interleave over keys.  Scores go to shared memory,
// the block takes max and sum, then the same lanes stream the values.  Keys
// and values are each read exactly once.  Softmax runs in the log2 domain.
#include "common.cuh"
#include "internal.h"

namespace rlt {

namespace {

constexpr int kThreads = 128;
constexpr int kUnroll = 4;

// Rotate the pair (x[i], x[i+hd/2]) at position p (table rope_cs holds cos and
// sin of p * base^(-2i/hd), interleaved, [pos][hd/2][2]).
__device__ __forceinline__ void rope_pair(float a, float b, const float* cs, float& oa, float& ob) {
  const float c = cs[0], s = cs[1];
  oa = a * c - b * s;
  ob = a * s + b * c;
}

// Scores of keys [j0, j1) (rows of `kb`) against the block's query fragment.
template <typename KT, int HD>
__device__ __forceinline__ void score_keys(const KT* __restrict__ kb, int j0, int j1, const float* qf, float* sc,
                                           int kg, int nkg, int sub) {
  constexpr int LPK = HD / 8;
  // the trip count is uniform across the block (the shuffles below need the
  // whole warp); lanes past the end load zeros and store nothing
  for (int jb = j0; jb < j1; jb += nkg * kUnroll) {
    float kf[kUnroll][8];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int j = jb + u * nkg + kg;
      if (j < j1) load8_stream(kb + (int64_t)j * HD + sub * 8, kf[u]);
      else {
#pragma unroll
        for (int i = 0; i < 8; ++i) kf[u][i] = 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      float dot = 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) dot = fmaf(qf[i], kf[u][i], dot);
#pragma unroll
      for (int o = LPK / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
      const int j = jb + u * nkg + kg;
      if (sub == 0 && j < j1) sc[j - j0] = dot;
    }
  }
}

// Probability-weighted sum of value rows [j0, j1) into o[8] (this lane's
// dimensions).
template <typename KT, int HD>
__device__ __forceinline__ void accumulate_values(const KT* __restrict__ vb, int j0, int j1, const float* p, float* o,
                                                  int kg, int nkg, int sub) {
  for (int jb = j0; jb < j1; jb += nkg * kUnroll) {
    float vf[kUnroll][8];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int j = jb + u * nkg + kg;
      if (j < j1) load8_stream(vb + (int64_t)j * HD + sub * 8, vf[u]);
      else {
#pragma unroll
        for (int i = 0; i < 8; ++i) vf[u][i] = 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int j = jb + u * nkg + kg;
      const float pj = j < j1 ? p[j - j0] : 0.f;
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = fmaf(pj, vf[u][i], o[i]);
    }
  }
}

// softmax over sc[0..n): sc <- exp2(sc - max); returns (max, sum)
__device__ __forceinline__ float2 softmax_inplace(float* sc, int n, float* red) {
  float mx = -INFINITY;
  for (int j = threadIdx.x; j < n; j += blockDim.x) mx = fmaxf(mx, sc[j]);
  mx = block_max(mx, red);
  float l = 0.f;
  for (int j = threadIdx.x; j < n; j += blockDim.x) {
    const float p = exp2f(sc[j] - mx);
    sc[j] = p;
    l += p;
  }
  l = block_sum(l, red);  // contains the barrier that publishes sc
  return make_float2(mx, l);
}

// ------------------------------------------------------------------ SWA
template <typename KT, int HD>
__global__ void __launch_bounds__(kThreads, 9) swa_attn_kernel(const float* __restrict__ qkv, int64_t ld_qkv, KT* ring_k,
                                                            KT* ring_v, int H, int t_all, SeqPos sp, int W,
                                                            const float* __restrict__ rope_cs, KT* out,
                                                            int64_t ld_out, float scale_log2) {
  // Dependents (the next GEMM) are released only once this block has issued
  // all its ring loads: released at the start, their CTAs would take SMs
  // (shared memory, registers) from the blocks of this HBM-bound kernel.
  griddep_wait();
  // position of this sequence's transition; an idle sequence (masked phase)
  // reads its ring but inserts nothing
  const int t = sp.on() ? sp.dec[blockIdx.y] + 1 : t_all;
  const bool insert = !sp.on() || sp.active(blockIdx.y);
  constexpr int LPK = HD / 8, KPW = 32 / LPK, NKG = (kThreads / 32) * KPW, HALF = HD / 2;
  extern __shared__ float sm[];
  float* sq = sm;            // rotated, scaled query
  float* sk = sq + HD;       // rotated current key
  float* sv = sk + HD;       // current value
  float* red_o = sv + HD;    // [NKG][HD]
  float* sc = red_o + NKG * HD;  // scores of ring slots, then the current key
  __shared__ float red[32];

  const int h = blockIdx.x, b = blockIdx.y;
  const int d = H * HD;
  const float* row = qkv + (int64_t)b * ld_qkv;
  const float* cs = rope_cs + (int64_t)(t - 1) * HALF * 2;
  for (int i = threadIdx.x; i < HALF; i += kThreads) {
    float a, c;
    rope_pair(row[h * HD + i], row[h * HD + i + HALF], cs + 2 * i, a, c);
    sq[i] = a * scale_log2;
    sq[i + HALF] = c * scale_log2;
    rope_pair(row[d + h * HD + i], row[d + h * HD + i + HALF], cs + 2 * i, a, c);
    sk[i] = a;
    sk[i + HALF] = c;
  }
  for (int i = threadIdx.x; i < HD; i += kThreads) sv[i] = row[2 * d + h * HD + i];
  __syncthreads();

  const int Wm1 = W - 1;
  const int n_ring = min(t - 1, Wm1);  // retained positions max(1,t-W+1)..t-1, one per slot
  const int64_t base = ((int64_t)b * H + h) * (int64_t)(Wm1 > 0 ? Wm1 : 1) * HD;
  KT* kb = ring_k + base;
  KT* vb = ring_v + base;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kg = warp * KPW + lane / LPK, sub = lane % LPK;
  float qf[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) qf[i] = sq[sub * 8 + i];

  score_keys<KT, HD>(kb, 0, n_ring, qf, sc, kg, NKG, sub);
  if (warp == 0) {  // current key
    float dot = 0.f;
    for (int i = lane; i < HD; i += 32) dot = fmaf(sq[i], sk[i], dot);
    dot = warp_sum(dot);
    if (lane == 0) sc[n_ring] = dot;
  }
  __syncthreads();
  const float2 ml = softmax_inplace(sc, n_ring + 1, red);

  float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  accumulate_values<KT, HD>(vb, 0, n_ring, sc, o, kg, NKG, sub);
  griddep_launch_dependents();
#pragma unroll
  for (int i = 0; i < 8; ++i) red_o[kg * HD + sub * 8 + i] = o[i];
  __syncthreads();
  const float inv = 1.0f / ml.y;
  for (int i = threadIdx.x; i < HD; i += kThreads) {
    float acc = sc[n_ring] * sv[i];
    for (int g = 0; g < NKG; ++g) acc += red_o[g * HD + i];
    out[(int64_t)b * ld_out + h * HD + i] = from_f32<KT>(acc * inv);
  }
  // Ring insert after every read of the ring above: the slot of position t is
  // the one that held t-W+1, which this step still attended to (§2.5).
  if (Wm1 > 0 && insert) {
    const int slot = (t - 1) % Wm1;
    for (int i = threadIdx.x; i < HD; i += kThreads) {
      kb[(int64_t)slot * HD + i] = from_f32<KT>(sk[i]);
      vb[(int64_t)slot * HD + i] = from_f32<KT>(sv[i]);
    }
  }
}

// ------------------------------------------------------------------ prefix
template <typename KT, int HD>
__global__ void __launch_bounds__(kThreads) prefix_attn_kernel(const float* __restrict__ q, int64_t ld_q,
                                                               const KT* __restrict__ kc, const KT* __restrict__ vc,
                                                               int64_t ld_t, int H, int n_all, int qpos_all,
                                                               SeqPos sp, const float* __restrict__ rope_cs, KT* out,
                                                               int64_t ld_out, float* ws, int nchunks, int* counters,
                                                               float scale_log2) {
  griddep_wait();  // dependents are released after the last K/V load, as in swa_attn_kernel
  constexpr int LPK = HD / 8, KPW = 32 / LPK, NKG = (kThreads / 32) * KPW, HALF = HD / 2;
  extern __shared__ float sm[];
  float* sq = sm;
  float* red_o = sq + HD;
  float* sc = red_o + NKG * HD;
  __shared__ float red[32];
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  // keys 0..n-1 of this sequence (its own position when the state has
  // per-sequence positions); the grid covers the longest sequence
  const int n = sp.on() ? sp.n_keys(b) : n_all;
  const int qpos = sp.on() ? n - 1 : qpos_all;
  const int nch = (n + kPrefixChunk - 1) / kPrefixChunk;
  if (c >= nch) return;
  const int j0 = c * kPrefixChunk, j1 = min(n, j0 + kPrefixChunk);
  const float* qrow = q + (int64_t)b * ld_q + h * HD;
  if (rope_cs != nullptr) {
    const float* cs = rope_cs + (int64_t)qpos * HALF * 2;
    for (int i = threadIdx.x; i < HALF; i += kThreads) {
      float a, bb;
      rope_pair(qrow[i], qrow[i + HALF], cs + 2 * i, a, bb);
      sq[i] = a * scale_log2;
      sq[i + HALF] = bb * scale_log2;
    }
  } else {
    for (int i = threadIdx.x; i < HD; i += kThreads) sq[i] = qrow[i] * scale_log2;
  }
  __syncthreads();
  const int64_t base = ((int64_t)b * H + h) * ld_t * HD;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kg = warp * KPW + lane / LPK, sub = lane % LPK;
  float qf[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) qf[i] = sq[sub * 8 + i];
  score_keys<KT, HD>(kc + base, j0, j1, qf, sc, kg, NKG, sub);
  __syncthreads();
  const float2 ml = softmax_inplace(sc, j1 - j0, red);
  float o[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  accumulate_values<KT, HD>(vc + base, j0, j1, sc, o, kg, NKG, sub);
  griddep_launch_dependents();
#pragma unroll
  for (int i = 0; i < 8; ++i) red_o[kg * HD + sub * 8 + i] = o[i];
  __syncthreads();
  if (nch == 1) {
    const float inv = 1.0f / ml.y;
    for (int i = threadIdx.x; i < HD; i += kThreads) {
      float acc = 0.f;
      for (int g = 0; g < NKG; ++g) acc += red_o[g * HD + i];
      out[(int64_t)b * ld_out + h * HD + i] = from_f32<KT>(acc * inv);
    }
  } else {
    const int64_t unit = ((int64_t)b * H + h) * nchunks + c;
    float* po = ws + unit * (HD + 2);
    for (int i = threadIdx.x; i < HD; i += kThreads) {
      float acc = 0.f;
      for (int g = 0; g < NKG; ++g) acc += red_o[g * HD + i];
      po[i] = acc;
    }
    if (threadIdx.x == 0) {
      po[HD] = ml.x;
      po[HD + 1] = ml.y;
    }
    if (counters != nullptr) {
      // The last of this (sequence, head)'s chunk blocks to finish combines
      // the partials in chunk order (the arithmetic of
      // prefix_combine_kernel, so the result does not depend on which block
      // it is) and resets the counter for the next launch.
      __shared__ int s_last;
      __threadfence();
      __syncthreads();
      if (threadIdx.x == 0) {
        const int prev = atomicAdd(&counters[b * H + h], 1);
        s_last = prev == nch - 1;
        if (s_last) counters[b * H + h] = 0;
      }
      __syncthreads();
      if (s_last) {
        __threadfence();
        const float* p = ws + ((int64_t)b * H + h) * nchunks * (HD + 2);
        float mx = -INFINITY;
        for (int cc = 0; cc < nch; ++cc) mx = fmaxf(mx, __ldcg(p + cc * (HD + 2) + HD));
        float l = 0.f;
        for (int cc = 0; cc < nch; ++cc)
          l += __ldcg(p + cc * (HD + 2) + HD + 1) * exp2f(__ldcg(p + cc * (HD + 2) + HD) - mx);
        const float inv = 1.0f / l;
        for (int i = threadIdx.x; i < HD; i += kThreads) {
          float acc = 0.f;
          for (int cc = 0; cc < nch; ++cc)
            acc += __ldcg(p + cc * (HD + 2) + i) * exp2f(__ldcg(p + cc * (HD + 2) + HD) - mx);
          out[(int64_t)b * ld_out + h * HD + i] = from_f32<KT>(acc * inv);
        }
      }
    }
  }
}

// Combines the chunk partials of one (sequence, head) in chunk order; a
// sequence whose keys fit one chunk was finished by prefix_attn_kernel.
template <typename KT, int HD>
__global__ void prefix_combine_kernel(const float* __restrict__ ws, int H, int nchunks, int n_all, SeqPos sp, KT* out,
                                      int64_t ld_out) {
  griddep_enter();
  const int h = blockIdx.x, b = blockIdx.y;
  const int n = sp.on() ? sp.n_keys(b) : n_all;
  const int nch = (n + kPrefixChunk - 1) / kPrefixChunk;
  if (nch <= 1) return;
  const float* p = ws + ((int64_t)b * H + h) * nchunks * (HD + 2);
  float mx = -INFINITY;
  for (int c = 0; c < nch; ++c) mx = fmaxf(mx, p[c * (HD + 2) + HD]);
  float l = 0.f;
  for (int c = 0; c < nch; ++c) l += p[c * (HD + 2) + HD + 1] * exp2f(p[c * (HD + 2) + HD] - mx);
  const float inv = 1.0f / l;
  for (int i = threadIdx.x; i < HD; i += blockDim.x) {
    float acc = 0.f;
    for (int c = 0; c < nch; ++c) acc += p[c * (HD + 2) + i] * exp2f(p[c * (HD + 2) + HD] - mx);
    out[(int64_t)b * ld_out + h * HD + i] = from_f32<KT>(acc * inv);
  }
}

template <int HD>
constexpr int nkg_of() {
  return (kThreads / 32) * (32 / (HD / 8));
}

template <typename KT, int HD>
cudaError_t swa_launch(const float* qkv, int64_t ld_qkv, KT* rk, KT* rv, int B, int H, int t, const SeqPos& sp, int W,
                       const float* rope_cs, KT* out, int64_t ld_out, cudaStream_t st) {
  const size_t smem = sizeof(float) * (3 * HD + nkg_of<HD>() * HD + W + 1);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(swa_attn_kernel<KT, HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)HD);
  {
    const cudaError_t e_l = launch_pdl(swa_attn_kernel<KT, HD>, dim3(dim3(H, B)), dim3(kThreads), smem, st, qkv, ld_qkv, rk, rv, H, t, sp, W, rope_cs, out, ld_out,
                                                               scale_log2);
    if (e_l != cudaSuccess) return e_l;
  }
  return cudaGetLastError();
}

template <typename KT, int HD>
cudaError_t prefix_launch(const float* q, int64_t ld_q, const KT* k, const KT* v, int64_t ld_t, int B, int H, int n,
                          int qpos, const SeqPos& sp, const float* rope_cs, KT* out, int64_t ld_out, float* ws,
                          size_t ws_floats, int* counters, cudaStream_t st) {
  const int nchunks = (n + kPrefixChunk - 1) / kPrefixChunk;
  if (nchunks > 1 && (!ws || ws_floats < (size_t)B * H * nchunks * (HD + 2))) return cudaErrorInvalidValue;
  const size_t smem = sizeof(float) * (HD + nkg_of<HD>() * HD + kPrefixChunk);
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)HD);
  {
    const cudaError_t e_l = launch_pdl(prefix_attn_kernel<KT, HD>, dim3(dim3(nchunks, H, B)), dim3(kThreads), smem, st, q, ld_q, k, v, ld_t, H, n, qpos, sp, rope_cs,
                                                                          out, ld_out, ws, nchunks, counters, scale_log2);
    if (e_l != cudaSuccess) return e_l;
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || nchunks == 1 || counters != nullptr) return e;
  {
    const cudaError_t e_l = launch_pdl(prefix_combine_kernel<KT, HD>, dim3(dim3(H, B)), dim3(HD < 128 ? HD : 128), 0, st, ws, H, nchunks, n, sp, out, ld_out);
    if (e_l != cudaSuccess) return e_l;
  }
  return cudaGetLastError();
}

}  // namespace

template <typename KT>
cudaError_t swa_attn(const float* qkv, int64_t ld_qkv, KT* ring_k, KT* ring_v, int B, int H, int hd, int t,
                     const SeqPos& sp, int W, const float* rope_cs, KT* out, int64_t ld_out, cudaStream_t st) {
  if ((!sp.on() && t < 1) || W < 1 || B <= 0) return cudaErrorInvalidValue;
  switch (hd) {
    case 16: return swa_launch<KT, 16>(qkv, ld_qkv, ring_k, ring_v, B, H, t, sp, W, rope_cs, out, ld_out, st);
    case 32: return swa_launch<KT, 32>(qkv, ld_qkv, ring_k, ring_v, B, H, t, sp, W, rope_cs, out, ld_out, st);
    case 64: return swa_launch<KT, 64>(qkv, ld_qkv, ring_k, ring_v, B, H, t, sp, W, rope_cs, out, ld_out, st);
    case 128: return swa_launch<KT, 128>(qkv, ld_qkv, ring_k, ring_v, B, H, t, sp, W, rope_cs, out, ld_out, st);
    case 256: return swa_launch<KT, 256>(qkv, ld_qkv, ring_k, ring_v, B, H, t, sp, W, rope_cs, out, ld_out, st);
  }
  return cudaErrorInvalidValue;
}

template <typename KT>
cudaError_t prefix_attn(const float* q, int64_t ld_q, const KT* k, const KT* v, int64_t ld_t, int B, int H, int hd,
                        int n, int qpos, const SeqPos& sp, const float* rope_cs, KT* out, int64_t ld_out, float* ws,
                        size_t ws_floats, int* counters, cudaStream_t st) {
  if (n < 1 || B <= 0) return cudaErrorInvalidValue;
#define RLT_PFX(HD) \
  prefix_launch<KT, HD>(q, ld_q, k, v, ld_t, B, H, n, qpos, sp, rope_cs, out, ld_out, ws, ws_floats, counters, st)
  switch (hd) {
    case 16: return RLT_PFX(16);
    case 32: return RLT_PFX(32);
    case 64: return RLT_PFX(64);
    case 128: return RLT_PFX(128);
    case 256: return RLT_PFX(256);
  }
#undef RLT_PFX
  return cudaErrorInvalidValue;
}

size_t prefix_attn_workspace_floats(int B, int H, int hd, int n) {
  const int nchunks = (n + kPrefixChunk - 1) / kPrefixChunk;
  return nchunks > 1 ? (size_t)B * H * nchunks * (hd + 2) : 0;
}

template cudaError_t swa_attn<float>(const float*, int64_t, float*, float*, int, int, int, int, const SeqPos&, int,
                                     const float*, float*, int64_t, cudaStream_t);
template cudaError_t swa_attn<bf16>(const float*, int64_t, bf16*, bf16*, int, int, int, int, const SeqPos&, int,
                                    const float*, bf16*, int64_t, cudaStream_t);
template cudaError_t prefix_attn<float>(const float*, int64_t, const float*, const float*, int64_t, int, int, int, int,
                                        int, const SeqPos&, const float*, float*, int64_t, float*, size_t, int*,
                                        cudaStream_t);
template cudaError_t prefix_attn<bf16>(const float*, int64_t, const bf16*, const bf16*, int64_t, int, int, int, int,
                                       int, const SeqPos&, const float*, bf16*, int64_t, float*, size_t, int*,
                                       cudaStream_t);

}  // namespace rlt
