// gemm_tc.cu -- bf16 GEMM on the sm_100a tensor cores (tcgen05.mma, fp32
// accumulators in tensor memory, operands staged by TMA).
//
// C[n][m] = sum_k X[n][k] * W[m][k]: the weight rows are the 128-row A operand
// (M = output features) and the activation rows are the N operand, so a
// decode step with a handful of sequences still fills the 128-lane MMA
// ("swap-AB"), and the same kernel serves the token-parallel encoder where N
// is the number of tokens.  Both operands are K-major bf16 in global memory,
// loaded by TMA with 128-byte swizzling into a multi-stage ring; one thread
// issues the TMA copies, one thread issues the MMAs, and all four warps drain
// the tensor-memory accumulator through the fused epilogue.  Work over K can
// be split across CTAs (the number of splits depends only on M and K, never on
// N, so a sequence's result does not depend on how many sequences share the
// step); partial sums then go to a workspace and a second kernel adds them in
// split order and applies the epilogue.
//
// No TMA multicast is used anywhere: every CTA loads its own tiles.
#include <cuda.h>

#include "common.cuh"
#include "epilogue.cuh"
#include "internal.h"

namespace rlt {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;

template <int BN>
struct TcCfg {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = BN >= 256 ? 4 : (BN >= 128 ? 6 : 8);
  static constexpr int SMEM = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;
  static constexpr int TMEM_COLS = BN;  // power of two >= 32
};

// UMMA shared-memory matrix descriptor for a K-major tile whose rows are 128
// bytes (64 bf16) with the 128-byte swizzle: 8-row core groups 1024 bytes
// apart (stride byte offset), descriptor version 1, layout SWIZZLE_128B.
__device__ __forceinline__ uint64_t sdesc_k128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)1 << 16;            // leading byte offset (unused for this layout)
  d |= (uint64_t)(1024 >> 4) << 32;  // stride byte offset
  d |= (uint64_t)1 << 46;            // descriptor version
  d |= (uint64_t)2 << 61;            // SWIZZLE_128B
  return d;
}

// Instruction descriptor: D fp32, A and B bf16, both K-major, shape 128 x BN.
template <int BN>
__device__ __forceinline__ constexpr uint32_t idesc_bf16() {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* tm, uint32_t bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

template <int BN, int EPI>
__global__ void __launch_bounds__(128, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int M, int N,
                   int K, int kb_per_split, EpiParams ep, float* partial) {
  using C = TcCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::STAGES;
  uint64_t* done = bars + 2 * C::STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * C::STAGES + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tile = blockIdx.x, n_tile = blockIdx.y, split = blockIdx.z;
  const int kb_total = K / BK;
  const int kb0 = split * kb_per_split;
  const int kb1 = min(kb_total, kb0 + kb_per_split);
  const int nkb = kb1 - kb0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(smem_u32(&full[s]), 1);
      mbar_init(smem_u32(&empty[s]), 1);
    }
    mbar_init(smem_u32(done), 1);
    *abort_flag = 0;
    fence_mbar_init();
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(C::TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // TMA producer
    int issued = 0;
    for (int i = 0; i < nkb && nkb > 0; ++i) {
      const int s = i % C::STAGES;
      const uint32_t ph = (uint32_t)(i / C::STAGES) & 1u;
      if (i >= C::STAGES) {
        if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1u)) { *abort_flag = 1; break; }
      }
      if (*abort_flag) break;
      const uint32_t a_s = smem_u32(smem + s * C::STAGE_BYTES);
      const uint32_t b_s = a_s + C::A_BYTES;
      mbar_arrive_expect_tx(smem_u32(&full[s]), C::STAGE_BYTES);
      tma_load_2d(a_s, &tmA, smem_u32(&full[s]), (kb0 + i) * BK, m_tile * BM);
      tma_load_2d(b_s, &tmB, smem_u32(&full[s]), (kb0 + i) * BK, n_tile * BN);
      ++issued;
    }
    if (*abort_flag) {
      // drain copies that may still be in flight before the CTA exits
      const int lo = issued > C::STAGES ? issued - C::STAGES : 0;
      for (int i = lo; i < issued; ++i)
        mbar_wait(smem_u32(&full[i % C::STAGES]), (uint32_t)(i / C::STAGES) & 1u);
    }
  } else if (warp == 1 && lane == 0) {
    // MMA issuer
    constexpr uint32_t idesc = idesc_bf16<BN>();
    for (int i = 0; i < nkb; ++i) {
      const int s = i % C::STAGES;
      const uint32_t ph = (uint32_t)(i / C::STAGES) & 1u;
      if (!mbar_wait(smem_u32(&full[s]), ph)) { *abort_flag = 1; break; }
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
      const uint32_t a_s = smem_u32(smem + s * C::STAGE_BYTES);
      const uint32_t b_s = a_s + C::A_BYTES;
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk) {
        umma_bf16(tmem_base, sdesc_k128(a_s + kk * 32), sdesc_k128(b_s + kk * 32), idesc,
                  (i > 0 || kk > 0) ? 1u : 0u);
      }
      umma_commit(smem_u32(&empty[s]));
    }
    umma_commit(smem_u32(done));
  }
  __syncwarp();

  // Epilogue: warp w owns accumulator lanes 32w..32w+31 (output features).
  const bool ok = mbar_wait(smem_u32(done), 0);
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  if (ok && !*abort_flag && nkb > 0) {
    const int m = m_tile * BM + warp * 32 + lane;
    const int64_t n_base = (int64_t)n_tile * BN;
#pragma unroll 1
    for (int c = 0; c < BN; c += 32) {
      if (n_base + c >= N) break;
      float v[32];
      tmem_ld32(tmem_base + ((uint32_t)(warp * 32) << 16) + (uint32_t)c, v);
      if (partial != nullptr) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int64_t n = n_base + c + j;
          if (n < N) partial[((int64_t)split * N + n) * M + m] = v[j];
        }
      } else if constexpr (EPI == EPI_SWIGLU) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const float other = __shfl_xor_sync(0xffffffffu, v[j], 1);
          const int64_t n = n_base + c + j;
          if (n < N && (lane & 1) == 0) epi_swiglu(ep, n, m >> 1, v[j], other);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int64_t n = n_base + c + j;
          if (n < N) epi_apply<EPI>(ep, n, m, v[j]);
        }
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(C::TMEM_COLS));
  }
}

// Sums split partials in split order and applies the epilogue; one thread
// per (n, pair of m).
template <int EPI>
__global__ void splitk_reduce_kernel(const float* __restrict__ partial, int splits, int M, int N, EpiParams ep) {
  const int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t pairs = (int64_t)N * (M / 2);
  if (idx >= pairs) return;
  const int64_t n = idx / (M / 2);
  const int m = (int)(idx % (M / 2)) * 2;
  float a = 0.f, b = 0.f;
  for (int s = 0; s < splits; ++s) {
    const float2 v = *reinterpret_cast<const float2*>(partial + ((int64_t)s * N + n) * M + m);
    a += v.x;
    b += v.y;
  }
  if constexpr (EPI == EPI_SWIGLU) {
    epi_swiglu(ep, n, m >> 1, a, b);
  } else {
    epi_apply<EPI>(ep, n, m, a);
    epi_apply<EPI>(ep, n, m + 1, b);
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D bf16 tensor map over a row-major [rows][cols] matrix with row pitch
// `ld` elements, box = 64 columns x box_rows rows, 128-byte swizzle.
bool make_tmap(CUtensorMap* tm, const void* base, int64_t rows, int64_t cols, int64_t ld, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int BN, int EPI>
cudaError_t launch_bn(const CUtensorMap& ta, const CUtensorMap& tb, int M, int N, int K, int splits,
                      int kb_per_split, const EpiParams& ep, float* partial, cudaStream_t st) {
  using C = TcCfg<BN>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc_kernel<BN, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  dim3 grid(M / BM, (N + BN - 1) / BN, splits);
  gemm_tc_kernel<BN, EPI><<<grid, 128, C::SMEM, st>>>(ta, tb, M, N, K, kb_per_split, ep, partial);
  note_launch();
  return cudaGetLastError();
}

template <int EPI>
cudaError_t launch_epi(const CUtensorMap& ta, const CUtensorMap& tb, int bn, int M, int N, int K, int splits,
                       int kb_per_split, const EpiParams& ep, float* partial, cudaStream_t st) {
  switch (bn) {
    case 32: return launch_bn<32, EPI>(ta, tb, M, N, K, splits, kb_per_split, ep, partial, st);
    case 64: return launch_bn<64, EPI>(ta, tb, M, N, K, splits, kb_per_split, ep, partial, st);
    case 128: return launch_bn<128, EPI>(ta, tb, M, N, K, splits, kb_per_split, ep, partial, st);
    default: return launch_bn<256, EPI>(ta, tb, M, N, K, splits, kb_per_split, ep, partial, st);
  }
}

template <int EPI>
cudaError_t launch_reduce(const float* partial, int splits, int M, int N, const EpiParams& ep, cudaStream_t st) {
  const int64_t pairs = (int64_t)N * (M / 2);
  const int threads = 256;
  splitk_reduce_kernel<EPI><<<(unsigned)((pairs + threads - 1) / threads), threads, 0, st>>>(partial, splits, M, N, ep);
  note_launch();
  return cudaGetLastError();
}

}  // namespace

int gemm_tc_splits(int M, int K, int N) {
  if (N > 256) return 1;
  const int tiles = M / BM;
  const int kb = K / BK;
  int s = (kSmCount + tiles / 2) / tiles;
  if (s < 1) s = 1;
  if (s > kb / 2) s = kb / 2 > 0 ? kb / 2 : 1;
  const int per = (kb + s - 1) / s;
  return (kb + per - 1) / per;
}

int gemm_tc_bn(int N) {
  if (N <= 32) return 32;
  if (N <= 64) return 64;
  if (N <= 128) return 128;
  return 256;
}

cudaError_t gemm_tc(const bf16* W, int64_t ldw, const bf16* X, int64_t ldx, int M, int N, int K, int epi,
                    const EpiParams& ep, float* workspace, size_t workspace_floats, cudaStream_t st) {
  if (M % BM || K % BK || N <= 0) return cudaErrorInvalidValue;
  const int bn = gemm_tc_bn(N);
  const int splits = gemm_tc_splits(M, K, N);
  const int kb = K / BK;
  const int per = (kb + splits - 1) / splits;
  CUtensorMap ta, tb;
  if (!make_tmap(&ta, W, M, K, ldw, BM)) return cudaErrorInvalidValue;
  if (!make_tmap(&tb, X, N, K, ldx, bn)) return cudaErrorInvalidValue;
  float* partial = nullptr;
  if (splits > 1) {
    if (!workspace || (size_t)splits * N * M > workspace_floats) return cudaErrorInvalidValue;
    partial = workspace;
  }
  cudaError_t e;
  switch (epi) {
    case EPI_STORE: e = launch_epi<EPI_STORE>(ta, tb, bn, M, N, K, splits, per, ep, partial, st); break;
    case EPI_RESID: e = launch_epi<EPI_RESID>(ta, tb, bn, M, N, K, splits, per, ep, partial, st); break;
    case EPI_SWIGLU: e = launch_epi<EPI_SWIGLU>(ta, tb, bn, M, N, K, splits, per, ep, partial, st); break;
    case EPI_GATE: e = launch_epi<EPI_GATE>(ta, tb, bn, M, N, K, splits, per, ep, partial, st); break;
    case EPI_MERGE: e = launch_epi<EPI_MERGE>(ta, tb, bn, M, N, K, splits, per, ep, partial, st); break;
    case EPI_CONVEX: e = launch_epi<EPI_CONVEX>(ta, tb, bn, M, N, K, splits, per, ep, partial, st); break;
    default: return cudaErrorInvalidValue;
  }
  if (e != cudaSuccess || splits == 1) return e;
  switch (epi) {
    case EPI_STORE: return launch_reduce<EPI_STORE>(partial, splits, M, N, ep, st);
    case EPI_RESID: return launch_reduce<EPI_RESID>(partial, splits, M, N, ep, st);
    case EPI_SWIGLU: return launch_reduce<EPI_SWIGLU>(partial, splits, M, N, ep, st);
    case EPI_GATE: return launch_reduce<EPI_GATE>(partial, splits, M, N, ep, st);
    case EPI_MERGE: return launch_reduce<EPI_MERGE>(partial, splits, M, N, ep, st);
    default: return launch_reduce<EPI_CONVEX>(partial, splits, M, N, ep, st);
  }
}

size_t gemm_tc_workspace_floats(int M, int K, int N) {
  const int s = gemm_tc_splits(M, K, N);
  return s > 1 ? (size_t)s * N * M : 0;
}

}  // namespace rlt
