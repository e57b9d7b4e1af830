// gemm_tc_kernel.cuh -- device code of the bf16 tensor-core GEMM (sm_100a:
// tcgen05.mma with fp32 accumulators in tensor memory, operands staged by TMA).
//
// C[n][m] = sum_k X[n][k] * W[m][k].  The weight rows are the 128-row A
// operand (M = output features); the activation rows are the N operand
// (N = sequences in a decode step, tokens in the encoder), so a decode step
// with few sequences still fills the 128-lane MMA.  Both operands are K-major
// bf16 in global memory, loaded by TMA with 128-byte swizzling into a
// multi-stage ring.  One thread issues the TMA copies, one thread issues the
// MMAs, and eight warps (two groups of four) drain the accumulator through
// the fused epilogue; the four warps without a main-loop role prepare the
// folded RMSNorm scales while the MMAs run.
//
// Split over K inside a thread-block cluster: the CS CTAs of one cluster own
// the same output tile and consecutive K ranges, so every weight byte is read
// from HBM once while all SMs stream.  CTA r finishes columns
// [r*BN/CS, (r+1)*BN/CS) of the tile: every CTA writes the other CTAs'
// shares of its fp32 partial to a global (L2-resident) exchange area, the
// cluster barrier publishes them, and each owner adds the CS partials of its
// columns in rank order 0..CS-1 (a fixed order, so results never depend on
// timing) before applying the epilogue.  Distributed shared memory was
// measured slower for this exchange than a round trip through L2.
//
// No TMA multicast is used anywhere: every CTA loads its own tiles.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "epilogue.cuh"
#include "internal.h"

namespace rlt {
namespace gemm_detail {

constexpr int BM = 128;
constexpr int BK = 64;

template <int BN>
struct TcCfg {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BN * BK * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = BN >= 256 ? 4 : (BN >= 128 ? 6 : 8);
  static constexpr int PIPE_BYTES = STAGES * STAGE_BYTES;
  static constexpr int EXTRA_OFF = PIPE_BYTES + 256;  // after the barriers
  static constexpr int SMEM = PIPE_BYTES + 1024 /*align*/ + 256 /*barriers*/ + 1024 /*1/rms per column*/ +
                              1024 /*per-warp column sums, two groups*/;
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

// Loads CNT (4, 8, 16 or 32) consecutive accumulator columns of this warp's 32
// lanes.
template <int CNT>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, float* v) {
  if constexpr (CNT == 32) {
    tmem_ld32(taddr, v);
  } else if constexpr (CNT == 16) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
  } else if constexpr (CNT == 4) {
    uint32_t r[4];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(r[i]);
  } else {
    static_assert(CNT == 8, "column count");
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < CNT; ++i) v[i] = __uint_as_float(r[i]);
  }
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}


// Barrier of one 128-thread epilogue group (named barrier 1 or 2; the block
// barrier 0 is __syncthreads).
__device__ __forceinline__ void group_sync(int g) {
  asm volatile("bar.sync %0, 128;" ::"r"(1 + g) : "memory");
}

// Butterfly transpose-reduction over the 32 lanes of a warp: on entry zv[j]
// is this lane's value for column j; on exit zv[0] of lane j is the sum over
// all lanes of column j (31 shuffles, fixed order).
__device__ __forceinline__ void warp_column_sums(float* zv, int lane) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < off; ++i) {
      const float send = upper ? zv[i] : zv[i + off];
      const float keep = upper ? zv[i + off] : zv[i];
      zv[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
  }
}

// Epilogue of CNT accumulator columns n0.. of this thread's row m: loads of
// each run of up to 16 outputs are issued before their stores.  `full` (all
// CNT columns exist) selects straight-line code; the ragged tail of N checks
// every column.  On return v[j] holds z^2 of producers (0 otherwise).
template <int EPI, int CNT, bool OBF, bool ZB>
__device__ __forceinline__ void epi_columns(const EpiParams& ep, const EpiRowConst& rc, int64_t n0, int64_t N,
                                            bool full, int m, int64_t my_o, int64_t my_a, float* v) {
  constexpr int RUN = CNT < 16 ? CNT : 16;
#pragma unroll
  for (int h = 0; h < CNT; h += RUN) {
    int64_t orow[RUN], arow[RUN];
    EpiPre pre[RUN];
#pragma unroll
    for (int j = 0; j < RUN; ++j) {
      orow[j] = __shfl_sync(0xffffffffu, my_o, h + j);
      arow[j] = epi_uses_aux0<EPI>() ? __shfl_sync(0xffffffffu, my_a, h + j) : 0;
    }
    if (full) {
#pragma unroll
      for (int j = 0; j < RUN; ++j) pre[j] = epi_load<EPI>(ep, n0 + h + j, orow[j], arow[j], m);
#pragma unroll
      for (int j = 0; j < RUN; ++j) {
        const float z = epi_store<EPI, OBF, ZB>(ep, rc, n0 + h + j, orow[j], m, v[h + j], pre[j]);
        v[h + j] = z * z;
      }
    } else {
#pragma unroll
      for (int j = 0; j < RUN; ++j)
        pre[j] = n0 + h + j < N ? epi_load<EPI>(ep, n0 + h + j, orow[j], arow[j], m) : EpiPre{0.f, 0.f};
#pragma unroll
      for (int j = 0; j < RUN; ++j) {
        const float z = n0 + h + j < N ? epi_store<EPI, OBF, ZB>(ep, rc, n0 + h + j, orow[j], m, v[h + j], pre[j]) : 0.f;
        v[h + j] = z * z;
      }
    }
  }
}

template <int CNT, bool OBF>
__device__ __forceinline__ void swiglu_columns(const EpiParams& ep, int64_t n0, int64_t N, bool full, int m,
                                               int lane, int64_t my_o, const float* v) {
  // Lanes 2k and 2k+1 hold the gate and up rows of hidden unit k.  For each
  // pair of columns (j, j+1) they swap one value, so that the even lane
  // finishes unit k of column j and the odd lane unit k of column j+1: every
  // lane evaluates one silu per column pair, with no branch, and stores one
  // output.
  static_assert(CNT % 2 == 0, "column pairs");
  const bool odd = (lane & 1) != 0;
  float hv[CNT / 2];
#pragma unroll
  for (int j = 0; j < CNT; j += 2) {
    const float send = odd ? v[j] : v[j + 1];  // up of column j / gate of column j+1
    const float recv = __shfl_xor_sync(0xffffffffu, send, 1);
    const float gate = odd ? recv : v[j];
    const float up = odd ? v[j + 1] : recv;
    hv[j / 2] = siluf_(gate) * up;
  }
#pragma unroll
  for (int j = 0; j < CNT; j += 2) {
    const int64_t orow_e = __shfl_sync(0xffffffffu, my_o, j);
    const int64_t orow_o = __shfl_sync(0xffffffffu, my_o, j + 1);
    const int jj = odd ? j + 1 : j;
    const int64_t orow = odd ? orow_o : orow_e;
    if (full || n0 + jj < N) {
      if constexpr (OBF) reinterpret_cast<bf16*>(ep.out)[orow + (m >> 1)] = __float2bfloat16_rn(hv[j / 2]);
      else reinterpret_cast<float*>(ep.out)[orow + (m >> 1)] = hv[j / 2];
    }
  }
}

// Finishes accumulator columns [n0, n0 + CNT) of this thread's row m (row
// `row` of weight tile m_tile): folded RMSNorm scale (consumers), the
// epilogue, and for producers the tile's per-column sums of z^2.  Called by
// the four warps of one epilogue group together (g: group, q: the warp's
// quarter of the 128 accumulator rows; it contains group barriers).  Row
// offsets, which may need a division for grouped rows, are computed once per
// column by lane j and broadcast.
template <int EPI, int CNT>
__device__ __forceinline__ void finish_chunk(const EpiParams& ep, const EpiRowConst& rc, int64_t n0, int64_t N, int m,
                                             int m_tile, int g, int q, int lane, float* v, const float* rinv,
                                             float* red) {
  if (ep.ss_in != nullptr) {
#pragma unroll
    for (int j = 0; j < CNT; ++j) v[j] *= rinv[j];
  }
  const int64_t my_n = n0 + lane;
  const bool my_ok = lane < CNT && my_n < N;
  const int64_t my_o = my_ok ? ep.out_map.off(my_n) : 0;
  const int64_t my_a = (epi_uses_aux0<EPI>() && my_ok) ? ep.aux0_map.off(my_n) : 0;
  const bool full = n0 + CNT <= N;
  if constexpr (EPI == EPI_SWIGLU) {
    if (ep.out_bf16) swiglu_columns<CNT, true>(ep, n0, N, full, m, lane, my_o, v);
    else swiglu_columns<CNT, false>(ep, n0, N, full, m, lane, my_o, v);
  } else if constexpr (EPI == EPI_STORE) {
    if (ep.out_bf16) epi_columns<EPI, CNT, true, false>(ep, rc, n0, N, full, m, my_o, my_a, v);
    else epi_columns<EPI, CNT, false, false>(ep, rc, n0, N, full, m, my_o, my_a, v);
  } else if constexpr (epi_produces_z<EPI>()) {
    if (ep.zb != nullptr) {
      epi_columns<EPI, CNT, false, true>(ep, rc, n0, N, full, m, my_o, my_a, v);
      if (ep.ss_out != nullptr) {
#pragma unroll
        for (int j = CNT; j < 32; ++j) v[j] = 0.f;
        warp_column_sums(v, lane);
        float* rg = red + g * 128;
        rg[q * 32 + lane] = v[0];
        group_sync(g);
        if (q == 0 && lane < CNT && n0 + lane < N)
          ep.ss_out[(int64_t)m_tile * ep.ss_ld + n0 + lane] = rg[lane] + rg[32 + lane] + rg[64 + lane] + rg[96 + lane];
        group_sync(g);
      }
    } else {
      epi_columns<EPI, CNT, false, false>(ep, rc, n0, N, full, m, my_o, my_a, v);
    }
  } else {
    epi_columns<EPI, CNT, false, false>(ep, rc, n0, N, full, m, my_o, my_a, v);
  }
}

template <int BN, int EPI, int CS>
__global__ void __launch_bounds__(256, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, int M, int N,
                   int K, int kb_per_split, float* split_ws, EpiParams ep) {
  using C = TcCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::PIPE_BYTES);
  uint64_t* full = bars;
  uint64_t* empty = bars + C::STAGES;
  uint64_t* done = bars + 2 * C::STAGES;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * C::STAGES + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tile = blockIdx.x, n_tile = blockIdx.y, split = blockIdx.z;  // cluster spans z: rank == split
  const int kb_total = K / BK;
  const int kb0 = split * kb_per_split;
  const int kb1 = min(kb_total, kb0 + kb_per_split);
  const int nkb = kb1 > kb0 ? kb1 - kb0 : 0;

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
    // TMA producer.  Weights do not depend on earlier kernels of the step, so
    // the first stages' weight tiles are requested before waiting for the
    // previous kernel (dependent launch); activation tiles follow the wait.
    const int pre = nkb < C::STAGES ? nkb : C::STAGES;
    for (int i = 0; i < pre; ++i) {
      const uint32_t a_s = smem_u32(smem + i * C::STAGE_BYTES);
      mbar_arrive_expect_tx(smem_u32(&full[i]), C::STAGE_BYTES);
      tma_load_2d(a_s, &tmA, smem_u32(&full[i]), (kb0 + i) * BK, m_tile * BM);
    }
    griddep_wait();
    for (int i = 0; i < pre; ++i) {
      const uint32_t b_s = smem_u32(smem + i * C::STAGE_BYTES) + C::A_BYTES;
      tma_load_2d(b_s, &tmB, smem_u32(&full[i]), (kb0 + i) * BK, n_tile * BN);
    }
    int issued = pre;
    for (int i = pre; i < nkb; ++i) {
      const int s = i % C::STAGES;
      const uint32_t ph = (uint32_t)(i / C::STAGES) & 1u;
      if (!mbar_wait(smem_u32(&empty[s]), ph ^ 1u)) { *abort_flag = 1; break; }
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

  // Epilogue: eight warps in two groups of four.  Warp w reads accumulator
  // lanes 32(w%4)..+31 (the tensor-memory quarter its SM sub-partition may
  // access) and its group g = w/4 takes every other column chunk, so two
  // warps per scheduler overlap their epilogue work.
  const int g = warp >> 2, q = warp & 3;
  const int row = q * 32 + lane;
  const int m = m_tile * BM + row;
  const EpiRowConst rc = epi_row_const<EPI>(ep, m);  // weights only: no wait needed
  const int64_t n_base = (int64_t)n_tile * BN;
  float* rinv = reinterpret_cast<float*>(smem + C::EXTRA_OFF);  // [BN] folded RMSNorm scale per column
  float* red = rinv + 256;                                        // [2][4][32] per-warp column sums
  if (warp >= 4) {
    // Warps 4..7 have no main-loop role: while the MMAs run they wait for
    // the previous kernel and turn its sums of squares into the per-column
    // 1/rms of the folded RMSNorm (8-load batches keep the summation order).
    griddep_wait();
    if (ep.ss_in != nullptr) {
      for (int i = threadIdx.x - 128; i < BN; i += 128) {
        const int64_t n = n_base + i;
        float ss = 0.f;
        if (n < N) {
          int mt = 0;
          for (; mt + 8 <= ep.n_ss; mt += 8) {
            float t8[8];
#pragma unroll
            for (int j = 0; j < 8; ++j) t8[j] = ep.ss_in[(int64_t)(mt + j) * ep.ss_ld + n];
#pragma unroll
            for (int j = 0; j < 8; ++j) ss += t8[j];
          }
          for (; mt < ep.n_ss; ++mt) ss += ep.ss_in[(int64_t)mt * ep.ss_ld + n];
        }
        rinv[i] = rsqrtf(ss * ep.norm_scale + ep.norm_eps);
      }
    }
  }
  const bool ok = mbar_wait(smem_u32(done), 0);
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  griddep_wait();  // epilogue reads/writes buffers of earlier kernels
  griddep_launch_dependents();
  const bool good = ok && !*abort_flag && nkb > 0;
  __syncthreads();
  if constexpr (CS == 1) {
#pragma unroll 1
    for (int c = 32 * g; c < BN; c += 64) {
      if (n_base + c >= N) break;
      float v[32];
      if (good) {
        tmem_ld32(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)c, v);
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) v[j] = 0.f;
      }
      finish_chunk<EPI, 32>(ep, rc, n_base + c, N, m, m_tile, g, q, lane, v, rinv + c, red);
    }
  } else {
    // Cluster split-K through L2: this CTA's exchange area holds CS slots of
    // COLS x 128 floats, slot o for owner o (its own slot stays unused).
    constexpr int COLS = BN / CS;
    // chunk width: two or more chunks per share where possible, so that both
    // epilogue groups have work
    constexpr int CNT = COLS >= 64 ? 32 : (COLS >= 8 ? COLS / 2 : COLS);
    constexpr int64_t SLICE = (int64_t)COLS * BM;  // floats of one share, column-major [COLS][128]
    const int rank = split;
    const int64_t col_cta = blockIdx.x + (int64_t)gridDim.x * blockIdx.y;  // same for every rank of the cluster
    const int64_t lin_stride = (int64_t)gridDim.x * gridDim.y;             // linear CTA id = col_cta + z * lin_stride
    float* mine = split_ws + (col_cta + rank * lin_stride) * CS * SLICE;
    int e = 0;  // chunk counter: group g takes the chunks with e % 2 == g
#pragma unroll 1
    for (int o = 0; o < CS; ++o) {
      if (o == rank) continue;
#pragma unroll 1
      for (int c = 0; c < COLS; c += CNT, ++e) {
        if ((e & 1) != g) continue;
        float v[32];
        if (good && n_base + o * COLS + c < N) {
          tmem_ld_cols<CNT>(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(o * COLS + c), v);
        } else {
#pragma unroll
          for (int j = 0; j < CNT; ++j) v[j] = 0.f;
        }
#pragma unroll
        for (int j = 0; j < CNT; ++j) __stcg(mine + o * SLICE + (int64_t)(c + j) * BM + row, v[j]);
      }
    }
    cluster_sync_all();  // release/acquire at cluster scope: the shares are visible to their owners
#pragma unroll 1
    for (int cc = CNT * g; cc < COLS; cc += 2 * CNT) {
      const int c0 = rank * COLS + cc;
      if (n_base + c0 >= N) break;
      float own[32], v[32];
      if (good) {
        tmem_ld_cols<CNT>(tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)c0, own);
      } else {
#pragma unroll
        for (int j = 0; j < CNT; ++j) own[j] = 0.f;
      }
#pragma unroll
      for (int j = 0; j < CNT; ++j) {
        float acc = 0.f;
#pragma unroll
        for (int p = 0; p < CS; ++p) {
          const float* src = split_ws + ((col_cta + p * lin_stride) * CS + rank) * SLICE + (int64_t)(cc + j) * BM + row;
          acc += p == rank ? own[j] : __ldcg(src);
        }
        v[j] = acc;
      }
#pragma unroll
      for (int j = CNT; j < 32; ++j) v[j] = 0.f;
      finish_chunk<EPI, CNT>(ep, rc, n_base + c0, N, m, m_tile, g, q, lane, v, rinv + c0, red);
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(C::TMEM_COLS));
  }
}

template <int BN, int EPI, int CS>
cudaError_t launch_gemm(const CUtensorMap& ta, const CUtensorMap& tb, int M, int N, int K, int kb_per_split, float* split_ws,
                        const EpiParams& ep, cudaStream_t st) {
  using C = TcCfg<BN>;
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e =
        cudaFuncSetAttribute(gemm_tc_kernel<BN, EPI, CS>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(M / BM, (N + BN - 1) / BN, CS);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = C::SMEM;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = CS;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, gemm_tc_kernel<BN, EPI, CS>, ta, tb, M, N, K, kb_per_split, split_ws, ep);
  note_launch();
  return e != cudaSuccess ? e : cudaGetLastError();
}

template <int EPI, int CS>
cudaError_t launch_gemm_bn(const CUtensorMap& ta, const CUtensorMap& tb, int bn, int M, int N, int K, int kb_per_split, float* split_ws,
                           const EpiParams& ep, cudaStream_t st) {
  switch (bn) {
    case 32: return launch_gemm<32, EPI, CS>(ta, tb, M, N, K, kb_per_split, split_ws, ep, st);
    case 64: return launch_gemm<64, EPI, CS>(ta, tb, M, N, K, kb_per_split, split_ws, ep, st);
    case 128: return launch_gemm<128, EPI, CS>(ta, tb, M, N, K, kb_per_split, split_ws, ep, st);
    default:
      return launch_gemm<256, EPI, CS>(ta, tb, M, N, K, kb_per_split, split_ws, ep, st);
  }
}

// All (BN, CS) variants of one epilogue; instantiated per epilogue in the
// gemm_tc_epi_*.cu files so the variants compile in parallel.
template <int EPI>
cudaError_t launch_gemm_epi(const CUtensorMap& ta, const CUtensorMap& tb, int bn, int cs, int M, int N, int K,
                            int kb_per_split, float* split_ws, const EpiParams& ep, cudaStream_t st) {
  switch (cs) {
    case 1: return launch_gemm_bn<EPI, 1>(ta, tb, bn, M, N, K, kb_per_split, split_ws, ep, st);
    case 2: return launch_gemm_bn<EPI, 2>(ta, tb, bn, M, N, K, kb_per_split, split_ws, ep, st);
    case 4: return launch_gemm_bn<EPI, 4>(ta, tb, bn, M, N, K, kb_per_split, split_ws, ep, st);
    case 8: return launch_gemm_bn<EPI, 8>(ta, tb, bn, M, N, K, kb_per_split, split_ws, ep, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace gemm_detail
}  // namespace rlt
