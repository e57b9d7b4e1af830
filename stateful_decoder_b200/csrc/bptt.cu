// bptt.cu -- CUDA backend of the full-BPTT engine (bptt_core.h).  Most
// functors of the engine run as a kernel with one thread per output index;
// the readout loss runs one block per row, the RMSNorms and the three
// attention functors one warp per row, query or key; and the three
// contractions of a bf16 model: Y = X W^T (MmNT),
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
#include <nvtx3/nvToolsExt.h>

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
  griddep_enter();
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
  griddep_enter();
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

// ---- row and attention functors with warp- or block-level parallelism: the
// arithmetic of the bptt_core.h functors (up to the order of summation),
// without one thread walking a whole row or key range alone.

// Readout loss of row b (Xent): one block of 1024 threads per row.  One
// pass keeps a running maximum and sum per thread (combined over the block),
// a second writes the adjoint; rows of V % 4 == 0 move as float4.
constexpr int kXentThreads = 1024;
__device__ __forceinline__ void online_add(float x, float& mx, float& den) {
  if (x > mx) {
    den = den * expf(mx - x) + 1.f;
    mx = x;
  } else {
    den += expf(x - mx);
  }
}
__global__ void __launch_bounds__(kXentThreads) xent_kernel(Xent<float> k) {
  griddep_enter();
  __shared__ float red[32];
  const int b = blockIdx.x;
  const float* l = k.logits + (int64_t)b * k.V;
  const bool vec = (k.V & 3) == 0;
  float mx = -INFINITY, den = 0.f;
  if (vec) {
    const float4* l4 = reinterpret_cast<const float4*>(l);
    for (int v = threadIdx.x; v < k.V / 4; v += kXentThreads) {
      const float4 x = l4[v];
      online_add(x.x, mx, den);
      online_add(x.y, mx, den);
      online_add(x.z, mx, den);
      online_add(x.w, mx, den);
    }
  } else {
    for (int v = threadIdx.x; v < k.V; v += kXentThreads) online_add(l[v], mx, den);
  }
  const float M = block_max(mx, red);
  den = block_sum(mx == -INFINITY ? 0.f : den * expf(mx - M), red);
  const float lse = M + logf(den);
  const int y = k.tok[(int64_t)b * k.tok_sb + k.t + 1];
  if (k.logp && threadIdx.x == 0) k.logp[(int64_t)b * k.w_sb + k.t] = l[y] - lse;
  if (k.dlogits) {
    const float w = k.wts[(int64_t)b * k.w_sb + k.t];
    float* dl = k.dlogits + (int64_t)b * k.V;
    if (vec) {
      const float4* l4 = reinterpret_cast<const float4*>(l);
      float4* d4 = reinterpret_cast<float4*>(dl);
      for (int v = threadIdx.x; v < k.V / 4; v += kXentThreads) {
        const float4 x = l4[v];
        float4 o;
        o.x = w * (expf(x.x - lse) - (4 * v == y ? 1.f : 0.f));
        o.y = w * (expf(x.y - lse) - (4 * v + 1 == y ? 1.f : 0.f));
        o.z = w * (expf(x.z - lse) - (4 * v + 2 == y ? 1.f : 0.f));
        o.w = w * (expf(x.w - lse) - (4 * v + 3 == y ? 1.f : 0.f));
        d4[v] = o;
      }
    } else {
      for (int v = threadIdx.x; v < k.V; v += kXentThreads) dl[v] = w * (expf(l[v] - lse) - (v == y ? 1.f : 0.f));
    }
  }
}

// RMSNorm forward (RmsF) and its input adjoint (RmsBX): one warp per row.
__global__ void __launch_bounds__(256) rmsf_kernel(RmsF<float> k, int64_t rows) {
  griddep_enter();
  const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const float* x = k.X + r * k.ldx;
  float ss = 0.f;
#pragma unroll 8
  for (int j = lane; j < k.d; j += 32) ss += x[j] * x[j];
  ss = warp_sum(ss);
  const float ri = 1.0f / sqrtf(ss / (float)k.d + k.eps);
  if (lane == 0) k.rinv[r] = ri;
  float* y = k.Y + r * k.ldy;
#pragma unroll 8
  for (int j = lane; j < k.d; j += 32) y[j] = x[j] * ri * k.g[j];
}
__global__ void __launch_bounds__(256) rmsbx_kernel(RmsBX<float> k, int64_t rows) {
  griddep_enter();
  const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const float* dy = k.dY + r * k.ldd;
  const float* x = k.X + r * k.ldx;
  const float ri = k.rinv[r];
  float dot = 0.f;
#pragma unroll 8
  for (int j = lane; j < k.d; j += 32) dot += dy[j] * k.g[j] * x[j] * ri;
  dot = warp_sum(dot) / (float)k.d;
  float* dx = k.dX + r * k.lddx;
#pragma unroll 8
  for (int j = lane; j < k.d; j += 32) dx[j] += ri * (dy[j] * k.g[j] - x[j] * ri * dot);
}

// Attention functors, one warp per (sequence, query or key, head); lane l
// holds head dimensions l, l+32, ... (at most kMaxHead / 32 of them).
constexpr int kLaneDims = kMaxHead / 32;

__device__ __forceinline__ float lane_dot(const float* a, const float* b, int hd, int lane) {
  float s = 0.f;
#pragma unroll
  for (int j = 0; j < kLaneDims; ++j) {
    const int e = lane + 32 * j;
    if (e < hd) s += a[e] * b[e];
  }
  return warp_sum(s);
}

// Keys per round of the attention loops: the round's key and value loads
// are all issued before any is used, so a warp waits for one load latency per
// round instead of one per key.
constexpr int kKeyRound = 8;

// AttnF: online softmax over the query's keys, kKeyRound keys per update.
__global__ void __launch_bounds__(256) attnf_kernel(AttnF<float> k, int64_t n) {
  griddep_enter();
  const int64_t idx = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (idx >= n) return;
  const AttnGeom<float>& g = k.g;
  const int h = (int)(idx % g.H);
  const int64_t bi = idx / g.H;
  const int i = (int)(bi % g.Tq);
  const int64_t b = bi / g.Tq;
  const float* q = k.Q + b * g.q_sb + i * g.q_si + (int64_t)h * g.hd;
  float qd[kLaneDims];
#pragma unroll
  for (int j = 0; j < kLaneDims; ++j) qd[j] = lane + 32 * j < g.hd ? q[lane + 32 * j] : 0.f;
  float mx = -INFINITY, den = 0.f, acc[kLaneDims];
#pragma unroll
  for (int j = 0; j < kLaneDims; ++j) acc[j] = 0.f;
  const int lo = g.lo(i), hi = g.hi(i);
  const float* kb = k.K + b * g.k_sb + (int64_t)h * g.hd;
  const float* vb = k.Vv + b * g.k_sb + (int64_t)h * g.hd;
  for (int p0 = lo; p0 <= hi; p0 += kKeyRound) {
    float kk[kKeyRound][kLaneDims], vv[kKeyRound][kLaneDims];
#pragma unroll
    for (int u = 0; u < kKeyRound; ++u) {
      const bool ok = p0 + u <= hi;
#pragma unroll
      for (int j = 0; j < kLaneDims; ++j) {
        const int e = lane + 32 * j;
        kk[u][j] = ok && e < g.hd ? kb[(int64_t)(p0 + u) * g.k_sp + e] : 0.f;
        vv[u][j] = ok && e < g.hd ? vb[(int64_t)(p0 + u) * g.k_sp + e] : 0.f;
      }
    }
    float sc[kKeyRound];
#pragma unroll
    for (int u = 0; u < kKeyRound; ++u) {
      sc[u] = 0.f;
#pragma unroll
      for (int j = 0; j < kLaneDims; ++j) sc[u] += qd[j] * kk[u][j];
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
#pragma unroll
      for (int u = 0; u < kKeyRound; ++u) sc[u] += __shfl_xor_sync(0xffffffffu, sc[u], off);
    float bm = -INFINITY;
#pragma unroll
    for (int u = 0; u < kKeyRound; ++u) {
      sc[u] = p0 + u <= hi ? sc[u] * k.scale : -INFINITY;
      bm = fmaxf(bm, sc[u]);
    }
    const float nm = fmaxf(mx, bm);
    const float c = expf(mx - nm);
    den *= c;
#pragma unroll
    for (int j = 0; j < kLaneDims; ++j) acc[j] *= c;
#pragma unroll
    for (int u = 0; u < kKeyRound; ++u) {
      const float w = expf(sc[u] - nm);
      den += w;
#pragma unroll
      for (int j = 0; j < kLaneDims; ++j) acc[j] += w * vv[u][j];
    }
    mx = nm;
  }
  float* o = k.O + b * g.q_sb + i * g.q_si + (int64_t)h * g.hd;
#pragma unroll
  for (int j = 0; j < kLaneDims; ++j) {
    const int e = lane + 32 * j;
    if (e < g.hd) o[e] = acc[j] / den;
  }
  if (lane == 0) k.lse[b * g.l_sb + i * g.l_si + h] = mx + logf(den);
}

// AttnBQ: dq = scale * sum_p P_p (dO.v_p - dO.o) k_p (overwrites dQ),
// kKeyRound keys per round.
__global__ void __launch_bounds__(256) attnbq_kernel(AttnBQ<float> k, int64_t n) {
  griddep_enter();
  const int64_t idx = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (idx >= n) return;
  const AttnGeom<float>& g = k.g;
  const int h = (int)(idx % g.H);
  const int64_t bi = idx / g.H;
  const int i = (int)(bi % g.Tq);
  const int64_t b = bi / g.Tq;
  const int64_t qo = b * g.q_sb + i * g.q_si + (int64_t)h * g.hd;
  const float L = k.lse[b * g.l_sb + i * g.l_si + h];
  const float Dv = lane_dot(k.dO + qo, k.O + qo, g.hd, lane);
  float qd[kLaneDims], dod[kLaneDims], acc[kLaneDims];
#pragma unroll
  for (int j = 0; j < kLaneDims; ++j) {
    const int e = lane + 32 * j;
    qd[j] = e < g.hd ? k.Q[qo + e] : 0.f;
    dod[j] = e < g.hd ? k.dO[qo + e] : 0.f;
    acc[j] = 0.f;
  }
  const int lo = g.lo(i), hi = g.hi(i);
  const float* kb = k.K + b * g.k_sb + (int64_t)h * g.hd;
  const float* vb = k.Vv + b * g.k_sb + (int64_t)h * g.hd;
  for (int p0 = lo; p0 <= hi; p0 += kKeyRound) {
    float kk[kKeyRound][kLaneDims], vv[kKeyRound][kLaneDims];
#pragma unroll
    for (int u = 0; u < kKeyRound; ++u) {
      const bool ok = p0 + u <= hi;
#pragma unroll
      for (int j = 0; j < kLaneDims; ++j) {
        const int e = lane + 32 * j;
        kk[u][j] = ok && e < g.hd ? kb[(int64_t)(p0 + u) * g.k_sp + e] : 0.f;
        vv[u][j] = ok && e < g.hd ? vb[(int64_t)(p0 + u) * g.k_sp + e] : 0.f;
      }
    }
    float sc[kKeyRound], dp[kKeyRound];
#pragma unroll
    for (int u = 0; u < kKeyRound; ++u) {
      sc[u] = dp[u] = 0.f;
#pragma unroll
      for (int j = 0; j < kLaneDims; ++j) {
        sc[u] += qd[j] * kk[u][j];
        dp[u] += dod[j] * vv[u][j];
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
#pragma unroll
      for (int u = 0; u < kKeyRound; ++u) {
        sc[u] += __shfl_xor_sync(0xffffffffu, sc[u], off);
        dp[u] += __shfl_xor_sync(0xffffffffu, dp[u], off);
      }
#pragma unroll
    for (int u = 0; u < kKeyRound; ++u) {
      if (p0 + u > hi) continue;
      const float P = expf(sc[u] * k.scale - L);
      const float ds = P * (dp[u] - Dv) * k.scale;
#pragma unroll
      for (int j = 0; j < kLaneDims; ++j) acc[j] += ds * kk[u][j];
    }
  }
#pragma unroll
  for (int j = 0; j < kLaneDims; ++j) {
    const int e = lane + 32 * j;
    if (e < g.hd) k.dQ[qo + e] = acc[j];
  }
}

// AttnBKV: dK, dV of one key position (accumulated) over the queries that see it.
__global__ void __launch_bounds__(256) attnbkv_kernel(AttnBKV<float> k, int64_t n) {
  griddep_enter();
  const int64_t idx = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (idx >= n) return;
  const AttnGeom<float>& g = k.g;
  const int h = (int)(idx % g.H);
  const int64_t bp = idx / g.H;
  const int p = k.p0 + (int)(bp % k.np);
  const int64_t b = bp / k.np;
  const int64_t ko = b * g.k_sb + p * g.k_sp + (int64_t)h * g.hd;
  float ak[kLaneDims], av[kLaneDims];
#pragma unroll
  for (int j = 0; j < kLaneDims; ++j) ak[j] = av[j] = 0.f;
  for (int i = 0; i < g.Tq; ++i) {
    if (p < g.lo(i) || p > g.hi(i)) continue;
    const int64_t qo = b * g.q_sb + i * g.q_si + (int64_t)h * g.hd;
    const float s = lane_dot(k.Q + qo, k.K + ko, g.hd, lane);
    const float dp = lane_dot(k.dO + qo, k.Vv + ko, g.hd, lane);
    const float Dv = lane_dot(k.dO + qo, k.O + qo, g.hd, lane);
    const float P = expf(s * k.scale - k.lse[b * g.l_sb + i * g.l_si + h]);
    const float ds = P * (dp - Dv) * k.scale;
#pragma unroll
    for (int j = 0; j < kLaneDims; ++j) {
      const int e = lane + 32 * j;
      if (e < g.hd) {
        ak[j] += ds * k.Q[qo + e];
        av[j] += P * k.dO[qo + e];
      }
    }
  }
#pragma unroll
  for (int j = 0; j < kLaneDims; ++j) {
    const int e = lane + 32 * j;
    if (e < g.hd) {
      k.dK[ko + e] += ak[j];
      k.dV[ko + e] += av[j];
    }
  }
}

// Device backend of Engine: stream-ordered launches with programmatic
// dependent launch (every kernel here waits for its predecessor at entry, then
// releases its own dependents, so the next launch overlaps this one's tail;
// the GEMM's pre-wait weight loads read operands made two or more kernels
// back, which are complete by then), buffers from cudaMalloc released after
// the stream drains.
struct CudaBackend {
  cudaStream_t st;
  bool tc;  // bf16 model: contractions on the tensor cores
  std::vector<void*> allocs;
  cudaError_t err = cudaSuccess;
  // bf16 weight copies (plain [M][K] and transposed [K][M]) by (address, pitch, rows, cols); a copy is
  // remade at its first use in each pass (begin_pass), since the weights may change between passes
  using WKey = std::tuple<const float*, int64_t, int, int>;
  struct WCopy {
    bf16* p;
    bool fresh;
  };
  std::map<WKey, WCopy> w_plain, w_trans;
  // per-contraction operand scratch and the split-K exchange area, grown on demand
  bf16* sa = nullptr; size_t sa_n = 0;
  bf16* sb = nullptr; size_t sb_n = 0;
  float* ws = nullptr; size_t ws_n = 0;
  // Operations issued so far, and which fp32 rows the bf16 activation copy
  // in `sb` holds (the operand of the contraction issued as operation `at`):
  // a contraction that directly follows one of the same rows reuses it.
  int64_t ops = 0;
  struct XCopy {
    const float* x;
    int64_t ld, rows;
    int cols;
    int64_t at;
  } xc{nullptr, 0, 0, 0, -2};
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
    ++ops;
    if (err == cudaSuccess && n) err = cudaMemsetAsync(p, 0, n * sizeof(T), st);
  }
  template <class T> void copy(T* dst, const T* src, size_t n) {
    ++ops;
    if (err == cudaSuccess && n) err = cudaMemcpyAsync(dst, src, n * sizeof(T), cudaMemcpyDeviceToDevice, st);
  }
  template <class T> void upload(T* dst, const T* src, size_t n) {
    ++ops;
    if (err == cudaSuccess && n) err = cudaMemcpyAsync(dst, src, n * sizeof(T), cudaMemcpyHostToDevice, st);
    if (err == cudaSuccess) err = cudaStreamSynchronize(st);  // the host source is the engine's own vector
  }
  template <class K> void launch(const K& k, int64_t n) {
    ++ops;
    launch_impl(k, n);
  }
  template <class K> void launch_impl(const K& k, int64_t n) {
    if (err != cudaSuccess || n <= 0) return;
    const int64_t blocks = (n + 255) / 256;
    err = launch_pdl(functor_kernel<K>, dim3((unsigned)blocks), dim3(256), 0, st, k, n);
  }
  int ok() const { return err == cudaSuccess ? 0 : -1; }
  void range_push(const char* name) { nvtxRangePushA(name); }
  void range_pop() { nvtxRangePop(); }

  // ---- row and attention functors, warp or block per unit
  template <class K> void launch_rows(void (*kern)(K, int64_t), const K& k, int64_t n) {
    ++ops;
    if (err != cudaSuccess || n <= 0) return;
    err = launch_pdl(kern, dim3((unsigned)((n + 7) / 8)), dim3(256), 0, st, k, n);
  }
  void launch(const Xent<float>& k, int64_t n) {
    ++ops;
    if (err != cudaSuccess || n <= 0) return;
    err = launch_pdl(xent_kernel, dim3((unsigned)n), dim3(kXentThreads), 0, st, k);
  }
  void launch(const RmsF<float>& k, int64_t n) { launch_rows(rmsf_kernel, k, n); }
  void launch(const RmsBX<float>& k, int64_t n) { launch_rows(rmsbx_kernel, k, n); }
  void launch(const AttnF<float>& k, int64_t n) { launch_rows(attnf_kernel, k, n); }
  void launch(const AttnBQ<float>& k, int64_t n) { launch_rows(attnbq_kernel, k, n); }
  void launch(const AttnBKV<float>& k, int64_t n) { launch_rows(attnbkv_kernel, k, n); }

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
    launch_impl(ToBf16{src, ld, dst, cols}, rows * cols);
  }
  void to_bf16_t(const float* src, int64_t ld, int R, int C, int Rp, bf16* dst) {
    if (err != cudaSuccess) return;
    err = launch_pdl(to_bf16_t_kernel, dim3((unsigned)((C + 31) / 32), (unsigned)(Rp / 32)), dim3(32, 8), 0, st, src,
                     ld, R, C, Rp, dst);
  }
  void begin_pass() {
    for (auto& e : w_plain) e.second.fresh = false;
    for (auto& e : w_trans) e.second.fresh = false;
  }
  // bf16 copy of the weight block W[M][K] (pitch ldw), plain or transposed, once per pass
  const bf16* weight(const float* W, int64_t ldw, int M, int K, bool transposed) {
    if (err != cudaSuccess) return nullptr;
    auto& cache = transposed ? w_trans : w_plain;
    const WKey key{W, ldw, M, K};
    auto it = cache.find(key);
    if (it != cache.end() && it->second.fresh) return it->second.p;
    bf16* b = nullptr;
    if (it != cache.end()) {
      b = it->second.p;
    } else {
      void* q = nullptr;
      err = cudaMalloc(&q, (size_t)M * K * sizeof(bf16));
      if (err != cudaSuccess) { cudaGetLastError(); return nullptr; }
      allocs.push_back(q);
      b = static_cast<bf16*>(q);
    }
    if (transposed) to_bf16_t(W, ldw, M, K, M, b);  // [K][M]; M % 64 == 0 where used
    else to_bf16(W, ldw, M, K, b);
    cache[key] = WCopy{b, true};
    return b;
  }
  // C[n][m] (+)= sum_k Bop[n][k] Aop[m][k] into fp32 rows `ldc` apart.  A
  // grid of output tiles that already fills the GPU runs unsplit; smaller
  // ones split K inside clusters (the decode plan).  The backward has no
  // batch-invariance constraint, so the choice may follow N.
  void gemm(const bf16* Aop, int M, const bf16* Bop, int N, int K, float* C, int64_t ldc, bool acc) {
    if (err != cudaSuccess) return;
    EpiParams ep{};
    ep.out = C;
    ep.out_map = plain_rows(ldc);
    ep.aux0_map = plain_rows(0);
    const int split = (int64_t)(M / 128) * ((N + 255) / 256) >= kSmCount ? 0 : 1;
    const size_t wsn = gemm_tc_workspace_floats(M, N, K, split);
    float* w = wsn ? workspace(wsn) : nullptr;
    if (err != cudaSuccess) return;
    err = gemm_tc(Aop, K, Bop, K, M, N, K, acc ? EPI_RESID : EPI_STORE, ep, split, w, wsn, st);
  }
  static int64_t round64(int64_t x) { return (x + 63) / 64 * 64; }

  // true when the rows [a, a + (ra-1)*lda + ca) and [b, b + (rb-1)*ldb + cb) share memory
  static bool spans_overlap(const float* a, int64_t lda, int64_t ra, int64_t ca, const float* b, int64_t ldb,
                            int64_t rb, int64_t cb) {
    const float* a1 = a + (ra - 1) * lda + ca;
    const float* b1 = b + (rb - 1) * ldb + cb;
    return a < b1 && b < a1;
  }
  // Y[r][m] (+)= sum_k X[r][k] W[m][k]
  void launch(const MmNT<float>& k, int64_t n) {
    const int64_t op = ++ops;
    const int64_t R = n / k.M;
    if (!tc || k.M % 128 || k.K % 64) return launch_impl<MmNT<float>>(k, n);
    const bf16* Wb = weight(k.Wm, k.ldw, k.M, k.K, false);
    bf16* Xb = grow(&sb, &sb_n, (size_t)R * k.K);
    if (!Wb || !Xb) return;
    // the operation just before was a contraction of the same rows, whose
    // bf16 copy is still in sb (the q/k/v and W1/W3 projections of one input)
    const bool reuse = xc.at == op - 1 && xc.x == k.X && xc.ld == k.ldx && xc.rows == R && xc.cols == k.K;
    if (!reuse) to_bf16(k.X, k.ldx, R, k.K, Xb);
    gemm(Wb, k.M, Xb, (int)R, k.K, k.Y, k.ldy, k.acc != 0);
    const bool wrote_source = spans_overlap(k.Y, k.ldy, R, k.M, k.X, k.ldx, R, k.K);
    xc = XCopy{k.X, k.ldx, R, k.K, wrote_source ? -2 : op};
  }
  // Y[r][c] (+)= sum_m D[r][m] W[m][c]   (c < K)
  void launch(const MmNN<float>& k, int64_t n) {
    ++ops;
    const int64_t R = n / k.K;
    if (!tc || k.K % 128 || k.M % 64) return launch_impl<MmNN<float>>(k, n);
    const bf16* Wt = weight(k.Wm, k.ldw, k.M, k.K, true);  // [K][M]
    bf16* Db = grow(&sb, &sb_n, (size_t)R * k.M);
    if (!Wt || !Db) return;
    to_bf16(k.Dm, k.ldd, R, k.M, Db);
    gemm(Wt, k.K, Db, (int)R, k.M, k.Y, k.ldy, k.acc != 0);
  }
  // G[m][c] += sum_r D[r][m] X[r][c]   (m < M = n / K, c < K), reduction padded to 64
  void launch(const MmTN<float>& k, int64_t n) {
    ++ops;
    const int64_t M = n / k.K;
    if (!tc || k.K % 128) return launch_impl<MmTN<float>>(k, n);
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

// ---------------------------------------------------------------- runner
namespace {
// Above this many kernels a pass runs its launches directly: a graph of that
// size costs more to instantiate and hold than its launches cost.
constexpr int64_t kMaxGraphKernels = 400000;

struct StreamSet {
  cudaStream_t s = nullptr;
  cudaEvent_t in = nullptr, out = nullptr;
  ~StreamSet() {
    if (in) cudaEventDestroy(in);
    if (out) cudaEventDestroy(out);
    if (s) cudaStreamDestroy(s);
  }
};
}  // namespace

struct Runner {
  Dims D;
  int seg;
  StreamSet ss;  // destroyed after the backend below, which drains the stream
  CudaBackend bk;
  Engine<CudaBackend, float> eng;
  int32_t* tok = nullptr;
  float* wts = nullptr;
  float* logp = nullptr;
  int passes = 0;
  bool graph_ok = true;
  cudaGraphExec_t exec = nullptr;
  int64_t kernels = 0;  // kernels of one pass
  Runner(const Dims& d, int sg, cudaStream_t s, bool tc, const float* const* W32, float* const* G32)
      : D(d), seg(sg), bk(s, tc), eng(bk, d, W32, G32) {}
  ~Runner() {
    if (exec) cudaGraphExecDestroy(exec);
  }
};

cudaError_t runner_create(const Dims& D, int seg, bool tensor_cores, const float* const* W32, float* const* G32,
                          Runner** out) {
  *out = nullptr;
  cudaStream_t s = nullptr;
  cudaError_t e = cudaStreamCreateWithFlags(&s, cudaStreamNonBlocking);
  if (e != cudaSuccess) return e;
  Runner* r = new Runner(D, seg, s, tensor_cores, W32, G32);
  r->ss.s = s;
  e = cudaEventCreateWithFlags(&r->ss.in, cudaEventDisableTiming);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&r->ss.out, cudaEventDisableTiming);
  if (e == cudaSuccess) {
    r->tok = r->bk.alloc<int32_t>((size_t)D.B * D.S);
    r->wts = r->bk.alloc<float>((size_t)D.B * (D.S - 1));
    r->logp = r->bk.alloc<float>((size_t)D.B * (D.S - 1));
    e = r->bk.err;
  }
  if (e != cudaSuccess) {
    delete r;
    return e;
  }
  *out = r;
  return cudaSuccess;
}

void runner_free(Runner* r) { delete r; }

cudaError_t runner_run(Runner* r, cudaError_t (*prologue)(void* ctx, cudaStream_t s), void* ctx, const int32_t* tok,
                       const float* wts, float* logp, cudaStream_t st) {
  const Dims& D = r->D;
  cudaStream_t gs = r->ss.s;
  cudaError_t e = cudaEventRecord(r->ss.in, st);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(gs, r->ss.in, 0);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(r->tok, tok, (size_t)D.B * D.S * 4, cudaMemcpyDeviceToDevice, gs);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(r->wts, wts, (size_t)D.B * (D.S - 1) * 4, cudaMemcpyDeviceToDevice, gs);
  if (e != cudaSuccess) return e;
  // the pass: widen the weights, then the engine (forward sweep, segments in reverse, encoder)
  auto pass = [&]() -> cudaError_t {
    cudaError_t pe = prologue(ctx, gs);
    if (pe != cudaSuccess) return pe;
    r->bk.begin_pass();
    const int rc = r->eng.run(r->tok, r->wts, r->seg, r->logp);
    if (r->bk.err != cudaSuccess) return r->bk.err;
    return rc == 0 ? cudaSuccess : cudaErrorInvalidValue;
  };
  if (r->exec) {
    for (int64_t i = 0; i < r->kernels; ++i) note_launch();
    e = cudaGraphLaunch(r->exec, gs);
  } else if (r->passes == 0 || !r->graph_ok || r->kernels > kMaxGraphKernels) {
    const int64_t n0 = launch_count();
    e = pass();
    if (r->passes == 0) r->kernels = launch_count() - n0;
  } else {
    // second pass: capture it (every buffer and bf16 weight copy exists by
    // now, so the pass allocates nothing), then launch the graph
    cudaGraph_t g = nullptr;
    bool ok = cudaStreamBeginCapture(gs, cudaStreamCaptureModeThreadLocal) == cudaSuccess;
    const int64_t n0 = launch_count();
    const cudaError_t pe = ok ? pass() : cudaSuccess;
    const int64_t n1 = launch_count();
    if (ok) ok = cudaStreamEndCapture(gs, &g) == cudaSuccess && pe == cudaSuccess;
    if (ok) ok = cudaGraphInstantiate(&r->exec, g, 0) == cudaSuccess;
    if (g) cudaGraphDestroy(g);
    if (ok) {
      r->kernels = n1 - n0;
      e = cudaGraphLaunch(r->exec, gs);
    } else {  // graphs off for this runner; this pass launches its kernels
      cudaGetLastError();
      r->exec = nullptr;
      r->graph_ok = false;
      r->bk.err = cudaSuccess;
      e = pass();
    }
  }
  if (e != cudaSuccess) return e;
  ++r->passes;
  if (logp) e = cudaMemcpyAsync(logp, r->logp, (size_t)D.B * (D.S - 1) * 4, cudaMemcpyDeviceToDevice, gs);
  if (e == cudaSuccess) e = cudaEventRecord(r->ss.out, gs);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st, r->ss.out, 0);
  return e;
}

}  // namespace bptt
}  // namespace rlt
