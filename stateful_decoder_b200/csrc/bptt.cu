// bptt.cu -- CUDA backend of the full-BPTT engine (bptt_core.h).  Every
// functor of the engine runs as a kernel with one thread per output index,
// except the three contractions of a bf16 model: Y = X W^T (MmNT),
// Y = D W (MmNN) and W_grad += D^T X (MmTN) run on the tensor cores through
// the library's tcgen05 GEMM (C[n][m] = sum_k B[n][k] A[m][k], both operands
// K-major bf16, fp32 accumulation), with the operands rounded to bf16 -- the
// precision of the model's forward.  The weights enter as bf16 copies made
// once per call, plain and transposed; activations and adjoints are rounded
// (and, for the weight gradients, transposed) per contraction.  Shapes that
// do not meet the GEMM's tiling (weight rows % 128, reduction % 64) and fp32
// models keep the CUDA-core functors.
// Also the widening of stored weights (fp32 or bf16, possibly pitched views)
// into the fp32 copies the engine differentiates.
#include <map>
#include <tuple>
#include <vector>

#include "bptt_core.h"
#include "internal.h"

namespace rlt {
namespace bptt {
namespace {

template <class K>
__global__ void __launch_bounds__(256) functor_kernel(K k, int64_t n) {
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) k(i);
}

// dst[r][c] = bf16(src[r*ld + c]) for c < cols; i = r*cols + c.
struct ToBf16 {
  const float* src; int64_t ld; bf16* dst; int64_t cols;
  __device__ void operator()(int64_t i) const {
    const int64_t r = i / cols, c = i % cols;
    dst[i] = __float2bfloat16_rn(src[r * ld + c]);
  }
};

// dst[c][r] = bf16(src[r*ld + c]) for r < R (zero for R <= r < Rp): a
// [R][C] fp32 matrix transposed to [C][Rp] bf16 through 32 x 32 shared-memory
// tiles (coalesced on both sides).  Grid (ceil(C/32), Rp/32), block (32, 8).
__global__ void to_bf16_t_kernel(const float* __restrict__ src, int64_t ld, int R, int C, int Rp, bf16* dst) {
  __shared__ float tile[32][33];
  const int c0 = blockIdx.x * 32, r0 = blockIdx.y * 32;
  for (int y = threadIdx.y; y < 32; y += 8) {
    const int r = r0 + y, c = c0 + threadIdx.x;
    tile[y][threadIdx.x] = (r < R && c < C) ? src[(int64_t)r * ld + c] : 0.f;
  }
  __syncthreads();
  for (int y = threadIdx.y; y < 32; y += 8) {
    const int c = c0 + y, r = r0 + threadIdx.x;
    if (c < C && r < Rp) dst[(int64_t)c * Rp + r] = __float2bfloat16_rn(tile[threadIdx.x][y]);
  }
}

// Device backend of Engine: plain stream-ordered launches (no dependent
// launch), buffers from cudaMalloc released after the stream drains.
struct CudaBackend {
  cudaStream_t st;
  bool tc;  // bf16 model: contractions on the tensor cores
  std::vector<void*> allocs;
  cudaError_t err = cudaSuccess;
  // bf16 weight copies (plain [M][K] and transposed [K][M]) by (address, pitch, rows, cols)
  using WKey = std::tuple<const float*, int64_t, int, int>;
  std::map<WKey, bf16*> w_plain, w_trans;
  // per-contraction operand scratch and the split-K exchange area, grown on demand
  bf16* sa = nullptr; size_t sa_n = 0;
  bf16* sb = nullptr; size_t sb_n = 0;
  float* ws = nullptr; size_t ws_n = 0;
  CudaBackend(cudaStream_t s, bool use_tc) : st(s), tc(use_tc) {}
  ~CudaBackend() {
    cudaStreamSynchronize(st);
    for (void* p : allocs) cudaFree(p);
  }
  template <class T> T* alloc(size_t n) {
    if (err != cudaSuccess) return nullptr;
    void* p = nullptr;
    const size_t bytes = (n ? n : 1) * sizeof(T);
    err = cudaMalloc(&p, bytes);
    if (err != cudaSuccess) {
      cudaGetLastError();
      return nullptr;
    }
    allocs.push_back(p);
    err = cudaMemsetAsync(p, 0, bytes, st);
    return static_cast<T*>(p);
  }
  template <class T> void zero(T* p, size_t n) {
    if (err == cudaSuccess && n) err = cudaMemsetAsync(p, 0, n * sizeof(T), st);
  }
  template <class T> void copy(T* dst, const T* src, size_t n) {
    if (err == cudaSuccess && n) err = cudaMemcpyAsync(dst, src, n * sizeof(T), cudaMemcpyDeviceToDevice, st);
  }
  template <class T> void upload(T* dst, const T* src, size_t n) {
    if (err == cudaSuccess && n) err = cudaMemcpyAsync(dst, src, n * sizeof(T), cudaMemcpyHostToDevice, st);
    if (err == cudaSuccess) err = cudaStreamSynchronize(st);  // the host source is the engine's own vector
  }
  template <class K> void launch(const K& k, int64_t n) {
    if (err != cudaSuccess || n <= 0) return;
    const int64_t blocks = (n + 255) / 256;
    functor_kernel<K><<<(unsigned)blocks, 256, 0, st>>>(k, n);
    note_launch();
    err = cudaGetLastError();
  }
  int ok() const { return err == cudaSuccess ? 0 : -1; }

  // ---- tensor-core contractions
  bf16* grow(bf16** p, size_t* cap, size_t n) {
    if (err != cudaSuccess) return nullptr;
    if (n > *cap) {
      void* q = nullptr;
      err = cudaMalloc(&q, n * sizeof(bf16));
      if (err != cudaSuccess) { cudaGetLastError(); return nullptr; }
      allocs.push_back(q);
      *p = static_cast<bf16*>(q);
      *cap = n;
    }
    return *p;
  }
  float* workspace(size_t n) {
    if (err != cudaSuccess) return nullptr;
    if (n > ws_n) {
      void* q = nullptr;
      err = cudaMalloc(&q, n * sizeof(float));
      if (err != cudaSuccess) { cudaGetLastError(); return nullptr; }
      allocs.push_back(q);
      ws = static_cast<float*>(q);
      ws_n = n;
    }
    return ws;
  }
  void to_bf16(const float* src, int64_t ld, int64_t rows, int64_t cols, bf16* dst) {
    launch(ToBf16{src, ld, dst, cols}, rows * cols);
  }
  void to_bf16_t(const float* src, int64_t ld, int R, int C, int Rp, bf16* dst) {
    if (err != cudaSuccess) return;
    to_bf16_t_kernel<<<dim3((unsigned)((C + 31) / 32), (unsigned)(Rp / 32)), dim3(32, 8), 0, st>>>(src, ld, R, C, Rp,
                                                                                                 dst);
    note_launch();
    err = cudaGetLastError();
  }
  // bf16 copy of the weight block W[M][K] (pitch ldw), plain or transposed, once per call
  const bf16* weight(const float* W, int64_t ldw, int M, int K, bool transposed) {
    auto& cache = transposed ? w_trans : w_plain;
    const WKey key{W, ldw, M, K};
    auto it = cache.find(key);
    if (it != cache.end()) return it->second;
    void* q = nullptr;
    if (err != cudaSuccess) return nullptr;
    err = cudaMalloc(&q, (size_t)M * K * sizeof(bf16));
    if (err != cudaSuccess) { cudaGetLastError(); return nullptr; }
    allocs.push_back(q);
    bf16* b = static_cast<bf16*>(q);
    if (transposed) to_bf16_t(W, ldw, M, K, M, b);  // [K][M]; M % 64 == 0 where used
    else to_bf16(W, ldw, M, K, b);
    cache.emplace(key, b);
    return b;
  }
  // C[n][m] (+)= sum_k Bop[n][k] Aop[m][k] into fp32 rows `ldc` apart
  void gemm(const bf16* Aop, int M, const bf16* Bop, int N, int K, float* C, int64_t ldc, bool acc) {
    if (err != cudaSuccess) return;
    EpiParams ep{};
    ep.out = C;
    ep.out_map = plain_rows(ldc);
    ep.aux0_map = plain_rows(0);
    const size_t wsn = gemm_tc_workspace_floats(M, N, K, 1);
    float* w = wsn ? workspace(wsn) : nullptr;
    if (err != cudaSuccess) return;
    err = gemm_tc(Aop, K, Bop, K, M, N, K, acc ? EPI_RESID : EPI_STORE, ep, 1, w, wsn, st);
  }
  static int64_t round64(int64_t x) { return (x + 63) / 64 * 64; }

  // Y[r][m] (+)= sum_k X[r][k] W[m][k]
  void launch(const MmNT<float>& k, int64_t n) {
    const int64_t R = n / k.M;
    if (!tc || k.M % 128 || k.K % 64) return launch<MmNT<float>>(k, n);
    const bf16* Wb = weight(k.Wm, k.ldw, k.M, k.K, false);
    bf16* Xb = grow(&sb, &sb_n, (size_t)R * k.K);
    if (!Wb || !Xb) return;
    to_bf16(k.X, k.ldx, R, k.K, Xb);
    gemm(Wb, k.M, Xb, (int)R, k.K, k.Y, k.ldy, k.acc != 0);
  }
  // Y[r][c] (+)= sum_m D[r][m] W[m][c]   (c < K)
  void launch(const MmNN<float>& k, int64_t n) {
    const int64_t R = n / k.K;
    if (!tc || k.K % 128 || k.M % 64) return launch<MmNN<float>>(k, n);
    const bf16* Wt = weight(k.Wm, k.ldw, k.M, k.K, true);  // [K][M]
    bf16* Db = grow(&sb, &sb_n, (size_t)R * k.M);
    if (!Wt || !Db) return;
    to_bf16(k.Dm, k.ldd, R, k.M, Db);
    gemm(Wt, k.K, Db, (int)R, k.M, k.Y, k.ldy, k.acc != 0);
  }
  // G[m][c] += sum_r D[r][m] X[r][c]   (m < M = n / K, c < K), reduction padded to 64
  void launch(const MmTN<float>& k, int64_t n) {
    const int64_t M = n / k.K;
    if (!tc || k.K % 128) return launch<MmTN<float>>(k, n);
    const int Rp = (int)round64(k.R);
    bf16* Xt = grow(&sa, &sa_n, (size_t)k.K * Rp);
    bf16* Dt = grow(&sb, &sb_n, (size_t)M * Rp);
    if (!Xt || !Dt) return;
    to_bf16_t(k.X, k.ldx, k.R, k.K, Rp, Xt);    // [K][Rp]
    to_bf16_t(k.Dm, k.ldd, k.R, (int)M, Rp, Dt);  // [M][Rp]
    gemm(Xt, k.K, Dt, (int)M, Rp, k.Gw, k.ldg, true);
  }
};

// dst[r][c] = float(src[r*pitch + c]); i = r*cols + c.
template <typename T> struct Widen {
  const T* src; int64_t pitch; float* dst; int64_t cols;
  __device__ void operator()(int64_t i) const {
    const int64_t r = i / cols, c = i % cols;
    dst[i] = to_f32(src[r * pitch + c]);
  }
};

}  // namespace

cudaError_t widen_to_f32(const void* src, int dtype, int64_t rows, int64_t cols, int64_t pitch, float* dst,
                         cudaStream_t st) {
  const int64_t n = rows * cols;
  if (n <= 0) return cudaSuccess;
  const int64_t blocks = (n + 255) / 256;
  if (dtype == 1)
    functor_kernel<<<(unsigned)blocks, 256, 0, st>>>(Widen<bf16>{static_cast<const bf16*>(src), pitch, dst, cols}, n);
  else
    functor_kernel<<<(unsigned)blocks, 256, 0, st>>>(Widen<float>{static_cast<const float*>(src), pitch, dst, cols}, n);
  note_launch();
  return cudaGetLastError();
}

cudaError_t replay_backward_f32(const Dims& D, const float* const* W32, float* const* G32, const int32_t* tok,
                                const float* wts, int seg, float* logp, bool tensor_cores, cudaStream_t st) {
  cudaError_t e;
  {
    CudaBackend bk(st, tensor_cores);
    Engine<CudaBackend, float> eng(bk, D, W32, G32);
    eng.run(tok, wts, seg, logp);
    e = bk.err;
  }  // the backend drains the stream and frees the engine's buffers here
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace bptt
}  // namespace rlt
