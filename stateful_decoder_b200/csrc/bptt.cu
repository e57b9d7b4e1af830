// bptt.cu -- CUDA backend of the full-BPTT engine (bptt_core.h): every
// functor of the engine runs as a kernel with one thread per output index.
// Also the widening of stored weights (fp32 or bf16, possibly pitched views)
// into the fp32 copies the engine differentiates.
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

// Device backend of Engine: plain stream-ordered launches (no dependent
// launch), buffers from cudaMalloc released after the stream drains.
struct CudaBackend {
  cudaStream_t st;
  std::vector<void*> allocs;
  cudaError_t err = cudaSuccess;
  explicit CudaBackend(cudaStream_t s) : st(s) {}
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
                                const float* wts, int seg, float* logp, cudaStream_t st) {
  cudaError_t e;
  {
    CudaBackend bk(st);
    Engine<CudaBackend, float> eng(bk, D, W32, G32);
    eng.run(tok, wts, seg, logp);
    e = bk.err;
  }  // the backend drains the stream and frees the engine's buffers here
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace bptt
}  // namespace rlt
