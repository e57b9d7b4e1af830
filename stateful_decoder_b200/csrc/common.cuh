// common.cuh -- shared device helpers of librlt (types, conversions, warp
// reductions, Philox4x32-10, bounded mbarrier waits, row addressing).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace rlt {

using bf16 = __nv_bfloat16;

// ---------------------------------------------------------------- errors
// Device word set by any bounded wait that ran out (never expected in a
// correct launch); the host reads and clears it with rlt_check_device().
extern __device__ int g_device_error;

// Bounded waits give up after this many nanoseconds of %globaltimer (far
// above any legitimate wait in these kernels) and raise g_device_error.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// ---------------------------------------------------------------- dependent launch
// Every kernel of the library is launched with programmatic stream
// serialisation, so it may start while the previous kernel of the stream is
// still running.  It must call griddep_wait() before it reads anything the
// previous kernels write or writes anything they read (weights and the rotary
// table are never written during a step and may be read before).  After the
// wait it lets its own dependents begin launching.
__device__ __forceinline__ void griddep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void griddep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void griddep_enter() {
  griddep_wait();
  griddep_launch_dependents();
}

// ---------------------------------------------------------------- types
template <typename T> struct TypeOf;
template <> struct TypeOf<float> { static constexpr int dtype = 0; };
template <> struct TypeOf<bf16> { static constexpr int dtype = 1; };

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(bf16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float x) { return __float2bfloat16_rn(x); }

// Load 8 consecutive elements (16 B for bf16: one vector; fp32: two) as floats.
__device__ __forceinline__ void load8(const bf16* p, float* f) {
  uint4 u = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void load8(const float* p, float* f) {
  float4 a = *reinterpret_cast<const float4*>(p);
  float4 b = *reinterpret_cast<const float4*>(p + 4);
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
// Read-only, streaming (evict-first) variants for KV streams read once.
__device__ __forceinline__ void load8_stream(const bf16* p, float* f) {
  uint4 u = __ldcs(reinterpret_cast<const uint4*>(p));
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void load8_stream(const float* p, float* f) {
  float4 a = __ldcs(reinterpret_cast<const float4*>(p));
  float4 b = __ldcs(reinterpret_cast<const float4*>(p + 4));
  f[0] = a.x; f[1] = a.y; f[2] = a.z; f[3] = a.w;
  f[4] = b.x; f[5] = b.y; f[6] = b.z; f[7] = b.w;
}
__device__ __forceinline__ void store8(bf16* p, const float* f) {
  uint32_t w[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    __nv_bfloat162 h = __floats2bfloat162_rn(f[2 * i], f[2 * i + 1]);
    w[i] = *reinterpret_cast<uint32_t*>(&h);
  }
  *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
}
__device__ __forceinline__ void store8(float* p, const float* f) {
  *reinterpret_cast<float4*>(p) = make_float4(f[0], f[1], f[2], f[3]);
  *reinterpret_cast<float4*>(p + 4) = make_float4(f[4], f[5], f[6], f[7]);
}

// ---------------------------------------------------------------- reductions
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
// Block-wide reductions for blockDim.x a multiple of 32 (<= 1024); `red`
// must hold 32 floats.  Every thread gets the result.
__device__ __forceinline__ float block_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_sum(v);
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  float r = lane < nw ? red[lane] : 0.f;
  r = warp_sum(r);
  return r;
}
__device__ __forceinline__ float block_max(float v, float* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  float r = lane < nw ? red[lane] : -INFINITY;
  r = warp_max(r);
  return r;
}

// ---------------------------------------------------------------- Philox
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, SC'11): ten rounds of the 4x32
// multiply-xor round with a Weyl-sequence key schedule.
__host__ __device__ __forceinline__ void philox4x32_10(uint32_t c[4], uint32_t k0, uint32_t k1) {
  const uint32_t mA = 0xD2511F53u, mB = 0xCD9E8D57u;
  for (int r = 0; r < 10; ++r) {
    if (r) { k0 += 0x9E3779B9u; k1 += 0xBB67AE85u; }
#ifdef __CUDA_ARCH__
    const uint32_t hA = __umulhi(mA, c[0]), lA = mA * c[0];
    const uint32_t hB = __umulhi(mB, c[2]), lB = mB * c[2];
#else
    const uint64_t pA = (uint64_t)mA * c[0], pB = (uint64_t)mB * c[2];
    const uint32_t hA = (uint32_t)(pA >> 32), lA = (uint32_t)pA;
    const uint32_t hB = (uint32_t)(pB >> 32), lB = (uint32_t)pB;
#endif
    const uint32_t n0 = hB ^ c[1] ^ k0, n2 = hA ^ c[3] ^ k1;
    c[0] = n0; c[1] = lB; c[2] = n2; c[3] = lA;
  }
}

// ---------------------------------------------------------------- rows
// Address of logical row r in a buffer whose rows come in groups:
// offset = (r / per_group) * group_stride + (r % per_group) * ld
// (per_group == 0: plain offset r * ld).  Used where token rows of several
// sequences live in a [B][max_len][d] store.
struct RowMap {
  int64_t ld;
  int32_t per_group;
  int64_t group_stride;
  __host__ __device__ __forceinline__ int64_t off(int64_t r) const {
    if (per_group <= 0) return r * ld;
    return (r / per_group) * group_stride + (r % per_group) * ld;
  }
};
__host__ __device__ inline RowMap plain_rows(int64_t ld) { return RowMap{ld, 0, 0}; }

// ---------------------------------------------------------------- positions
// Per-sequence positions of a state, as device arrays of B entries (report
// §4.1: every sequence of a batch has its own position).  `dec` counts the
// decoder transitions applied (n_dec), `enc` the tokens encoded (n_enc); the
// transition in flight for sequence b is at t_b = dec[b] + 1.  In a masked
// phase (catching up over appended spans of different lengths) `lim` is set
// and sequence b takes part in a transition only while dec[b] < lim[b]; an
// idle sequence reads only rows that exist and writes nothing.  All pointers
// null: the kernel takes the scalar position it is given instead.
struct SeqPos {
  const int32_t* dec;
  const int32_t* enc;
  const int32_t* lim;
  __host__ __device__ bool on() const { return dec != nullptr; }
  __device__ __forceinline__ bool active(int b) const { return lim == nullptr || dec[b] < lim[b]; }
  // keys an attention query of sequence b reads: 1..t_b when active, else
  // the rows an idle sequence already holds (at least one)
  __device__ __forceinline__ int n_keys(int b) const { return active(b) ? dec[b] + 1 : max(1, dec[b]); }
  // the transition's encoder step writes position t_b of sequence b
  __device__ __forceinline__ bool encodes(int b) const { return active(b) && enc[b] <= dec[b]; }
};
__host__ __device__ inline SeqPos no_pos() { return SeqPos{nullptr, nullptr, nullptr}; }

// ---------------------------------------------------------------- mbarrier / PTX
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// Bounded wait for the completion of the phase with the given parity.
// Returns false (and raises the device error word) when the limit runs out.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, uint64_t limit_ns = kWaitLimitNs) {
  uint64_t t0 = 0;
  for (uint32_t it = 0;; ++it) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    if (ok) return true;
    if (it == 0) t0 = globaltimer_ns();
    else if ((it & 255u) == 0 && globaltimer_ns() - t0 > limit_ns) break;
  }
  atomicExch(&g_device_error, 1);
  return false;
}

}  // namespace rlt
