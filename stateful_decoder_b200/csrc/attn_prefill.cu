// attn_prefill.cu -- token-parallel causal self-attention of the encoder
// ("Recurrent Looped Transformer" §2.2, eq. 2.1: positions of one layer are
// processed together under a causal mask).
//
// Flash-style tiling on CUDA cores: a block owns 64 queries of one (sequence,
// head) and streams 64-key tiles up to the diagonal.  The queries may start
// at position q_off > 0 (a chunk appended to an encoded prefix, whose keys
// and values are rows 0..q_off-1 of the cache).  S = Q K^T is formed as a
// 4x4 register tile per thread from transposed shared-memory copies of Q and
// K, the online softmax keeps a running max and sum per query row, and
// O += P V accumulates 4 rows x (hd/16) columns per thread.
#include "common.cuh"
#include "internal.h"

namespace rlt {

namespace {

constexpr int BQ = 64, BKV = 64, PADQ = BQ + 4, PADK = BKV + 4;

template <int HD>
constexpr size_t causal_smem_floats() {
  return (size_t)HD * PADQ + (size_t)HD * PADK + (size_t)BKV * (HD + 4) + (size_t)BKV * PADQ + 3 * BQ;
}

template <typename KT, int HD>
__global__ void __launch_bounds__(256) causal_attn_kernel(const KT* __restrict__ Q, const KT* __restrict__ K,
                                                          const KT* __restrict__ V, int64_t ld_tq, int64_t ld_tkv,
                                                          int H, int T, int q_off, KT* out, int64_t ld_out,
                                                          float scale_log2) {
  griddep_enter();
  constexpr int DPT = HD / 16;
  extern __shared__ float sm[];
  float* sQt = sm;                      // [HD][PADQ]
  float* sKt = sQt + HD * PADQ;         // [HD][PADK]
  float* sV = sKt + HD * PADK;          // [BKV][HD+4]
  float* sP = sV + BKV * (HD + 4);      // [BKV][PADQ]  probabilities, key-major
  float* sAlpha = sP + BKV * PADQ;      // [BQ]
  float* sL = sAlpha + BQ;              // [BQ]
  float* sM = sL + BQ;                  // [BQ]

  const int q0 = blockIdx.x * BQ, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const KT* Qb = Q + ((int64_t)b * H + h) * ld_tq * HD;
  const KT* Kb = K + ((int64_t)b * H + h) * ld_tkv * HD;
  const KT* Vb = V + ((int64_t)b * H + h) * ld_tkv * HD;

  for (int i = tid; i < BQ * HD; i += 256) {
    const int r = i / HD, c = i % HD;
    const float v = (q0 + r < T) ? to_f32(Qb[(int64_t)(q0 + r) * HD + c]) : 0.f;
    sQt[c * PADQ + r] = v * scale_log2;
  }
  for (int i = tid; i < BQ; i += 256) {
    sM[i] = -INFINITY;
    sL[i] = 0.f;
  }
  float o[4][DPT];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < DPT; ++j) o[i][j] = 0.f;

  // queries are positions q_off + 0..T-1; keys 0..q_off+T-1
  const int Tk = q_off + T;
  const int kv_end = min(Tk, q_off + q0 + BQ);
  for (int k0 = 0; k0 < kv_end; k0 += BKV) {
    __syncthreads();
    for (int i = tid; i < BKV * HD; i += 256) {
      const int r = i / HD, c = i % HD;
      const bool ok = k0 + r < Tk;
      sKt[c * PADK + r] = ok ? to_f32(Kb[(int64_t)(k0 + r) * HD + c]) : 0.f;
      sV[r * (HD + 4) + c] = ok ? to_f32(Vb[(int64_t)(k0 + r) * HD + c]) : 0.f;
    }
    __syncthreads();
    float s[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) s[i][j] = 0.f;
#pragma unroll 8
    for (int c = 0; c < HD; ++c) {
      const float4 qa = *reinterpret_cast<const float4*>(&sQt[c * PADQ + ty * 4]);
      const float4 ka = *reinterpret_cast<const float4*>(&sKt[c * PADK + tx * 4]);
      const float qv[4] = {qa.x, qa.y, qa.z, qa.w}, kv[4] = {ka.x, ka.y, ka.z, ka.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) s[i][j] = fmaf(qv[i], kv[j], s[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int qpos = q_off + q0 + ty * 4 + i, kj = k0 + tx * 4 + j;
        sP[(tx * 4 + j) * PADQ + ty * 4 + i] = (kj <= qpos && kj < Tk) ? s[i][j] : -INFINITY;
      }
    __syncthreads();
    {
      // online softmax: four threads per query row, 16 keys each
      const int row = tid >> 2, part = tid & 3;
      float mx = -INFINITY;
      for (int j = part * 16; j < part * 16 + 16; ++j) mx = fmaxf(mx, sP[j * PADQ + row]);
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      const float m_old = sM[row];
      const float m_new = fmaxf(m_old, mx);
      float sum = 0.f;
      for (int j = part * 16; j < part * 16 + 16; ++j) {
        const float p = exp2f(sP[j * PADQ + row] - m_new);
        sP[j * PADQ + row] = p;
        sum += p;
      }
      sum += __shfl_xor_sync(0xffffffffu, sum, 1);
      sum += __shfl_xor_sync(0xffffffffu, sum, 2);
      __syncwarp();
      if (part == 0) {
        const float a = exp2f(m_old - m_new);
        sAlpha[row] = a;
        sL[row] = sL[row] * a + sum;
        sM[row] = m_new;
      }
    }
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float a = sAlpha[ty * 4 + i];
#pragma unroll
      for (int j = 0; j < DPT; ++j) o[i][j] *= a;
    }
    const int kn = min(BKV, kv_end - k0);
    for (int j = 0; j < kn; ++j) {
      const float4 p4 = *reinterpret_cast<const float4*>(&sP[j * PADQ + ty * 4]);
      const float pv[4] = {p4.x, p4.y, p4.z, p4.w};
      float vv[DPT];
#pragma unroll
      for (int c = 0; c < DPT; ++c) vv[c] = sV[j * (HD + 4) + tx * DPT + c];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int c = 0; c < DPT; ++c) o[i][c] = fmaf(pv[i], vv[c], o[i][c]);
    }
  }
  __syncthreads();
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int qi = q0 + ty * 4 + i;
    if (qi >= T) continue;
    const float inv = 1.0f / sL[ty * 4 + i];
#pragma unroll
    for (int c = 0; c < DPT; ++c)
      out[((int64_t)b * T + qi) * ld_out + h * HD + tx * DPT + c] = from_f32<KT>(o[i][c] * inv);
  }
}

template <typename KT, int HD>
cudaError_t launch(const KT* q, const KT* k, const KT* v, int64_t ld_tq, int64_t ld_tkv, int B, int H, int T, int q_off,
                   KT* out, int64_t ld_out, cudaStream_t st) {
  const size_t smem = causal_smem_floats<HD>() * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(causal_attn_kernel<KT, HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)HD);
  dim3 grid((T + BQ - 1) / BQ, H, B);
  {
    const cudaError_t e_l = launch_pdl(causal_attn_kernel<KT, HD>, dim3(grid), dim3(256), smem, st, q, k, v, ld_tq, ld_tkv, H, T, q_off, out, ld_out, scale_log2);
    if (e_l != cudaSuccess) return e_l;
  }
  return cudaGetLastError();
}

}  // namespace

template <typename KT>
cudaError_t causal_attn(const KT* q, const KT* k, const KT* v, int64_t ld_tq, int64_t ld_tkv, int B, int H, int hd,
                        int T, int q_off, KT* out, int64_t ld_out, cudaStream_t st) {
  if (T <= 0 || B <= 0 || q_off < 0) return cudaErrorInvalidValue;
  switch (hd) {
    case 16: return launch<KT, 16>(q, k, v, ld_tq, ld_tkv, B, H, T, q_off, out, ld_out, st);
    case 32: return launch<KT, 32>(q, k, v, ld_tq, ld_tkv, B, H, T, q_off, out, ld_out, st);
    case 64: return launch<KT, 64>(q, k, v, ld_tq, ld_tkv, B, H, T, q_off, out, ld_out, st);
    case 128: return launch<KT, 128>(q, k, v, ld_tq, ld_tkv, B, H, T, q_off, out, ld_out, st);
  }
  return cudaErrorInvalidValue;
}

template cudaError_t causal_attn<float>(const float*, const float*, const float*, int64_t, int64_t, int, int, int, int,
                                        int, float*, int64_t, cudaStream_t);
template cudaError_t causal_attn<bf16>(const bf16*, const bf16*, const bf16*, int64_t, int64_t, int, int, int, int,
                                       int, bf16*, int64_t, cudaStream_t);

}  // namespace rlt
