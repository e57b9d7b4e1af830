// attn_prefill_tc.cu -- token-parallel causal self-attention of the encoder
// ("Recurrent Looped Transformer" §2.2, eq. 2.1) on the sm_100a tensor cores.
//
// One CTA owns 128 queries of one (sequence, head).  Keys come in 128-row
// tiles up to the diagonal.  Two passes over the key tiles:
//   pass 1: S = Q K^T (tcgen05.mma, fp32 in tensor memory); every thread
//           reads its query row of S and keeps the running row maximum;
//   pass 2: S again; p = exp2(S*scale - max) is summed per row and written to
//           shared memory as the bf16 A operand of O += P V (tcgen05.mma, O in
//           tensor memory).
// With the final maximum known in pass 2, O is never rescaled, at the price
// of one more Q K^T (cheap: the tensor cores are far from busy here).
// Q, K (K-major) and V (read as an MN-major operand straight from its
// [key][hd] rows) are staged by TMA with 128-byte swizzling.  Four warps:
// thread 0 issues TMA and MMA, every thread owns one query row.
#include <cuda.h>

#include "common.cuh"
#include "internal.h"

namespace rlt {

namespace {

constexpr int FQ = 128;   // queries per CTA (MMA M)
constexpr int FKV = 128;  // keys per tile (MMA N of Q K^T, K of P V)

template <int HD>
struct FaCfg {
  static constexpr int SUB = HD / 64;                  // 64-wide swizzle sub-tiles along hd
  static constexpr int TILE_BYTES = 128 * HD * 2;      // a [128][HD] bf16 tile
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = TILE_BYTES;             // K tile, then reused for P ([128][128] bf16)
  static constexpr int V_OFF = K_OFF + (TILE_BYTES > 32768 ? TILE_BYTES : 32768);
  static constexpr int BAR_OFF = V_OFF + TILE_BYTES;
  static constexpr int SMEM = BAR_OFF + 64 + 1024;
  static constexpr int TMEM_COLS = 256;                // S in [0,128), O in [128,128+HD)
};

__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// kind::f16 instruction descriptor, fp32 accumulate, bf16 operands, M = 128;
// b_mn = 1 reads B as MN-major.
__device__ __forceinline__ constexpr uint32_t idesc_fa(int n, int b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)b_mn << 16) | ((uint32_t)(n >> 3) << 17) |
         ((uint32_t)(128 >> 4) << 24);
}

__device__ __forceinline__ void fa_tma(uint32_t dst, const CUtensorMap* tm, uint32_t bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(tm)), "r"(bar), "r"(x), "r"(y)
      : "memory");
}

__device__ __forceinline__ void fa_mma(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ void fa_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void fa_ld32(uint32_t taddr, float* v) {
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

// One full tile-sized transfer: TMA the [128][HD] tile at row `row0` of the
// 2-D [rows][HD] view into dst (HD/64 swizzled boxes, 16 KB apart).
template <int HD>
__device__ __forceinline__ void load_tile(uint32_t dst, const CUtensorMap* tm, uint32_t bar, int row0) {
#pragma unroll
  for (int s = 0; s < HD / 64; ++s) fa_tma(dst + s * 16384, tm, bar, s * 64, row0);
}

template <int HD>
__global__ void __launch_bounds__(128, 2)
    causal_attn_tc_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                          const __grid_constant__ CUtensorMap tmV, int64_t ld_tq, int64_t ld_tkv, int H, int T,
                          int q_off, bf16* out, int64_t ld_out, float scale_log2) {
  using C = FaCfg<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::BAR_OFF);
  const uint32_t bar_q = smem_u32(&bars[0]);   // Q landed
  const uint32_t bar_kv = smem_u32(&bars[1]);  // K (and V) landed
  const uint32_t bar_s = smem_u32(&bars[2]);   // S = Q K^T done
  const uint32_t bar_o = smem_u32(&bars[3]);   // O += P V done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(&bars[4]);
  const uint32_t sQ = smem_u32(smem + C::Q_OFF), sK = smem_u32(smem + C::K_OFF), sV = smem_u32(smem + C::V_OFF);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, row = threadIdx.x;
  const int q0 = blockIdx.x * FQ, h = blockIdx.y, b = blockIdx.z;
  const int qrow0 = (int)(((int64_t)b * H + h) * ld_tq + q0);
  const int krow0 = (int)(((int64_t)b * H + h) * ld_tkv);
  // queries: chunk rows q0 + row at positions q_off + q0 + row; keys 0..Tk-1
  const int Tk = q_off + T;
  const int n_tiles = (min(Tk, q_off + q0 + FQ) + FKV - 1) / FKV;
  const int qi = q0 + row;
  const int qpos = q_off + qi;

  griddep_enter();
  if (threadIdx.x == 0) {
    for (int i = 0; i < 4; ++i) mbar_init(smem_u32(&bars[i]), 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(C::TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  const uint32_t tmem = *tmem_slot;
  const uint32_t tS = tmem, tO = tmem + 128;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

  constexpr uint32_t ID_S = idesc_fa(FKV, 0);
  constexpr uint32_t ID_O = idesc_fa(HD, 1);
  bool ok = true;
  uint32_t ph_kv = 0, ph_s = 0, ph_o = 0;

  if (threadIdx.x == 0) {
    mbar_arrive_expect_tx(bar_q, C::TILE_BYTES);
    load_tile<HD>(sQ, &tmQ, bar_q, qrow0);
  }
  ok = mbar_wait(bar_q, 0) && ok;

  // S = Q K_j^T into tS (issued by thread 0)
  auto issue_s = [&](int j, bool with_v) {
    mbar_arrive_expect_tx(bar_kv, with_v ? 2 * C::TILE_BYTES : C::TILE_BYTES);
    load_tile<HD>(sK, &tmK, bar_kv, krow0 + j * FKV);
    if (with_v) load_tile<HD>(sV, &tmV, bar_kv, krow0 + j * FKV);
  };
  auto mma_s = [&]() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll
    for (int kk = 0; kk < HD / 16; ++kk) {
      const uint32_t off = (uint32_t)((kk / 4) * 16384 + (kk % 4) * 32);
      fa_mma(tS, desc_sw128(sQ + off, 16, 1024), desc_sw128(sK + off, 16, 1024), ID_S, kk > 0 ? 1u : 0u);
    }
    fa_commit(bar_s);
  };

  // ---------------- pass 1: row maxima
  float mrow = -INFINITY;
  for (int j = 0; j < n_tiles; ++j) {
    if (threadIdx.x == 0) {
      issue_s(j, false);
      ok = mbar_wait(bar_kv, ph_kv) && ok;
      mma_s();
    }
    ph_kv ^= 1u;
    ok = mbar_wait(bar_s, ph_s) && ok;
    ph_s ^= 1u;
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll 1
    for (int c = 0; c < FKV; c += 32) {
      float v[32];
      fa_ld32(tS + lane_off + (uint32_t)c, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int kj = j * FKV + c + i;
        if (kj <= qpos && kj < Tk) mrow = fmaxf(mrow, v[i] * scale_log2);
      }
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();  // S fully read and K buffer free before the next tile
  }

  // ---------------- pass 2: P = exp2(S*scale - m), O += P V
  float lrow = 0.f;
  for (int j = 0; j < n_tiles; ++j) {
    if (threadIdx.x == 0) {
      issue_s(j, true);
      ok = mbar_wait(bar_kv, ph_kv) && ok;
      mma_s();
    } else {
      ok = mbar_wait(bar_kv, ph_kv) && ok;  // V rows below are rewritten by this thread
    }
    ph_kv ^= 1u;
    // Value rows past the sequence end (rows of another head, or cache rows
    // never written) get probability 0, but 0 * NaN would still poison O:
    // zero them.
    if (j * FKV + row >= Tk) {
#pragma unroll
      for (int s = 0; s < HD / 64; ++s) {
        const uint32_t vrow = sV + (uint32_t)(s * 16384 + (row >> 3) * 1024 + (row & 7) * 128);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          asm volatile("st.shared.v4.b32 [%0], {%1, %1, %1, %1};" ::"r"(vrow + q * 16), "r"(0u) : "memory");
      }
    }
    ok = mbar_wait(bar_s, ph_s) && ok;
    ph_s ^= 1u;
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    // P row -> the K buffer (its MMA is complete) in the swizzled K-major
    // layout of a [128 rows][128 keys] bf16 A operand (two 64-key sub-tiles)
    const uint32_t prow = sK + (uint32_t)((row >> 3) * 1024 + (row & 7) * 128);
#pragma unroll 1
    for (int c = 0; c < FKV; c += 32) {
      float v[32];
      fa_ld32(tS + lane_off + (uint32_t)c, v);
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 32; i += 2) {
        const int kj = j * FKV + c + i;
        const float p0 = (kj <= qpos && kj < Tk) ? exp2f(v[i] * scale_log2 - mrow) : 0.f;
        const float p1 = (kj + 1 <= qpos && kj + 1 < Tk) ? exp2f(v[i + 1] * scale_log2 - mrow) : 0.f;
        lrow += p0 + p1;
        __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);
        pk[i / 2] = *reinterpret_cast<uint32_t*>(&h2);
      }
      const int sub = c / 64;
#pragma unroll
      for (int q = 0; q < 4; ++q) {  // four 16-byte chunks of 8 keys
        const int chunk = ((c % 64) / 8) + q;
        const uint32_t addr = prow + (uint32_t)(sub * 16384 + ((chunk ^ (row & 7)) * 16));
        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(pk[4 * q]), "r"(pk[4 * q + 1]),
                     "r"(pk[4 * q + 2]), "r"(pk[4 * q + 3])
                     : "memory");
      }
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (threadIdx.x == 0) {
      asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
#pragma unroll
      for (int kk = 0; kk < FKV / 16; ++kk) {
        const uint32_t aoff = (uint32_t)((kk / 4) * 16384 + (kk % 4) * 32);
        fa_mma(tO, desc_sw128(sK + aoff, 16, 1024), desc_sw128(sV + (uint32_t)(kk * 2048), 16384, 1024), ID_O,
               (j > 0 || kk > 0) ? 1u : 0u);
      }
      fa_commit(bar_o);
      ok = mbar_wait(bar_o, ph_o) && ok;  // P and V buffers are reused by the next tile
    }
    ph_o ^= 1u;
    __syncthreads();
  }

  // ---------------- epilogue: O / l
  if (n_tiles > 0) {
    ok = mbar_wait(bar_o, ph_o ^ 1u) && ok;
  }
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
  // every thread takes part in the (warp-collective) tensor-memory loads;
  // only rows inside the sequence are stored
  const bool store = ok && qi < T;
  const float inv = 1.0f / lrow;
  bf16* orow = out + ((int64_t)b * T + (qi < T ? qi : 0)) * ld_out + (int64_t)h * HD;
#pragma unroll 1
  for (int c = 0; c < HD; c += 32) {
    float v[32];
    fa_ld32(tO + lane_off + (uint32_t)c, v);
    if (store) {
#pragma unroll
      for (int i = 0; i < 32; i += 8) {
        float f[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) f[u] = v[i + u] * inv;
        store8(orow + c + i, f);
      }
    }
  }
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
  __syncthreads();
  if (warp == 0) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(C::TMEM_COLS));
  }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool fa_tmap(CUtensorMap* tm, const void* base, int64_t rows, int hd) {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return false;
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  cuuint64_t dims[2] = {(cuuint64_t)hd, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)hd * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  return fn(tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int HD>
cudaError_t launch_fa(const bf16* q, const bf16* k, const bf16* v, int64_t ld_tq, int64_t ld_tkv, int B, int H, int T,
                      int q_off, bf16* out, int64_t ld_out, cudaStream_t st) {
  using C = FaCfg<HD>;
  CUtensorMap tq, tk, tv;
  if (!fa_tmap(&tq, q, (int64_t)B * H * ld_tq, HD) || !fa_tmap(&tk, k, (int64_t)B * H * ld_tkv, HD) ||
      !fa_tmap(&tv, v, (int64_t)B * H * ld_tkv, HD))
    return cudaErrorInvalidValue;
  static bool attr = false;
  if (!attr) {
    const cudaError_t e =
        cudaFuncSetAttribute(causal_attn_tc_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr = true;
  }
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)HD);
  return launch_pdl(causal_attn_tc_kernel<HD>, dim3((T + FQ - 1) / FQ, H, B), dim3(128), (size_t)C::SMEM, st, tq, tk,
                    tv, ld_tq, ld_tkv, H, T, q_off, out, ld_out, scale_log2);
}

}  // namespace

cudaError_t causal_attn_tc(const bf16* q, const bf16* k, const bf16* v, int64_t ld_tq, int64_t ld_tkv, int B, int H,
                           int hd, int T, int q_off, bf16* out, int64_t ld_out, cudaStream_t st) {
  if (T <= 0 || B <= 0 || q_off < 0) return cudaErrorInvalidValue;
  if ((int64_t)B * H * (ld_tq > ld_tkv ? ld_tq : ld_tkv) >= ((int64_t)1 << 31)) return cudaErrorInvalidValue;
  switch (hd) {
    case 64: return launch_fa<64>(q, k, v, ld_tq, ld_tkv, B, H, T, q_off, out, ld_out, st);
    case 128: return launch_fa<128>(q, k, v, ld_tq, ld_tkv, B, H, T, q_off, out, ld_out, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace rlt
