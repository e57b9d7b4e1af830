// gemm_simt.cu -- CUDA-core GEMM with the same fused epilogues as the
// tensor-core path.  It is the contraction of fp32 models (where a tf32 or
// bf16 tensor-core pass would not meet fp32 accuracy) and a cross-check of the
// tcgen05 kernel in the tests.  Tile 64 (weights) x 64 (activations) x 16,
// 256 threads, 4 x 4 outputs per thread; weight rows of one thread are
// consecutive so SwiGLU pairs (rows 2i, 2i+1) meet in one thread.
#include "common.cuh"
#include "epilogue.cuh"
#include "internal.h"

namespace rlt {

namespace {

constexpr int TM = 64, TN = 64, TK = 16;

template <typename WT, typename XT, int EPI>
__global__ void __launch_bounds__(256) gemm_simt_kernel(const WT* __restrict__ W, int64_t ldw, const XT* __restrict__ X,
                                                        int64_t ldx, int M, int N, int K, EpiParams ep) {
  griddep_enter();
  __shared__ float sW[TK][TM + 4];
  __shared__ float sX[TK][TN + 4];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int m0 = blockIdx.x * TM, n0 = blockIdx.y * TN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += TK) {
    for (int i = threadIdx.x; i < TM * TK; i += 256) {
      const int r = i / TK, c = i % TK;
      const int m = m0 + r, k = k0 + c;
      sW[c][r] = (m < M && k < K) ? to_f32(W[(int64_t)m * ldw + k]) : 0.f;
    }
    for (int i = threadIdx.x; i < TN * TK; i += 256) {
      const int r = i / TK, c = i % TK;
      const int n = n0 + r, k = k0 + c;
      sX[c][r] = (n < N && k < K) ? to_f32(X[(int64_t)n * ldx + k]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = sW[kk][tx * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = sX[kk][ty * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int64_t n = n0 + ty * 4 + j;
    if (n >= N) continue;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int m = m0 + tx * 4 + i;
      if (m >= M) continue;
      if constexpr (EPI == EPI_SWIGLU) {
        if ((i & 1) == 0 && m + 1 < M) epi_swiglu(ep, n, m >> 1, acc[i][j], acc[i + 1][j]);
      } else {
        epi_apply<EPI>(ep, n, m, acc[i][j]);
      }
    }
  }
}

template <typename WT, typename XT, int EPI>
cudaError_t launch(const WT* W, int64_t ldw, const XT* X, int64_t ldx, int M, int N, int K, const EpiParams& ep,
                   cudaStream_t st) {
  dim3 grid((M + TM - 1) / TM, (N + TN - 1) / TN);
  {
    const cudaError_t e_l = launch_pdl(gemm_simt_kernel<WT, XT, EPI>, dim3(grid), dim3(256), 0, st, W, ldw, X, ldx, M, N, K, ep);
    if (e_l != cudaSuccess) return e_l;
  }
  return cudaGetLastError();
}

}  // namespace

template <typename WT, typename XT>
cudaError_t gemm_simt(const WT* W, int64_t ldw, const XT* X, int64_t ldx, int M, int N, int K, int epi,
                      const EpiParams& ep, cudaStream_t st) {
  if (M <= 0 || N <= 0 || K <= 0) return cudaErrorInvalidValue;
  switch (epi) {
    case EPI_STORE: return launch<WT, XT, EPI_STORE>(W, ldw, X, ldx, M, N, K, ep, st);
    case EPI_RESID: return launch<WT, XT, EPI_RESID>(W, ldw, X, ldx, M, N, K, ep, st);
    case EPI_SWIGLU: return launch<WT, XT, EPI_SWIGLU>(W, ldw, X, ldx, M, N, K, ep, st);
    case EPI_GATE: return launch<WT, XT, EPI_GATE>(W, ldw, X, ldx, M, N, K, ep, st);
    case EPI_MERGE: return launch<WT, XT, EPI_MERGE>(W, ldw, X, ldx, M, N, K, ep, st);
    case EPI_CONVEX: return launch<WT, XT, EPI_CONVEX>(W, ldw, X, ldx, M, N, K, ep, st);
  }
  return cudaErrorInvalidValue;
}

template cudaError_t gemm_simt<float, float>(const float*, int64_t, const float*, int64_t, int, int, int, int,
                                             const EpiParams&, cudaStream_t);
template cudaError_t gemm_simt<bf16, bf16>(const bf16*, int64_t, const bf16*, int64_t, int, int, int, int,
                                           const EpiParams&, cudaStream_t);

}  // namespace rlt
