// ops.cu -- elementwise and row kernels of the RLT step: weight generator,
// embedding gather, RMSNorm, merge operand, head scatter with rotary map,
// readout log-probabilities and the behaviour sampler.
#include <float.h>

#include <atomic>

#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace rlt {

__device__ int g_device_error = 0;
// Time the last bounded_wait_probe launch waited (ns), for the host to read.
__device__ unsigned long long g_probe_waited_ns = 0;

namespace {
std::atomic<int64_t> g_launches{0};
}
void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }
int64_t launch_count() { return g_launches.load(std::memory_order_relaxed); }

namespace {

// ------------------------------------------------------------------ init
// Element i of generator stream `sid`: init_std * (Irwin-Hall(12) - 6), the
// twelve uniforms being the words of three Philox4x32-10 blocks with counters
// (i_lo, i_hi, sid, j), key = seed.  Integer sum, exact double arithmetic,
// then fp32 and (bf16 storage) round-to-nearest-even.
template <typename WT>
__global__ void init_normal_kernel(WT* dst, int64_t rows, int64_t cols, int64_t pitch, uint32_t k0, uint32_t k1,
                                   uint32_t sid, float std) {
  griddep_enter();
  const int64_t n = rows * cols;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    uint64_t sum = 0;
#pragma unroll
    for (uint32_t j = 0; j < 3; ++j) {
      uint32_t c[4] = {(uint32_t)i, (uint32_t)((uint64_t)i >> 32), sid, j};
      philox4x32_10(c, k0, k1);
      sum += (uint64_t)c[0] + c[1] + c[2] + c[3];
    }
    const double z = (double)sum * (1.0 / 4294967296.0) - 6.0;
    const float f = __double2float_rn((double)std * z);
    dst[(i / cols) * pitch + (i % cols)] = from_f32<WT>(f);
  }
}

template <typename WT>
__global__ void init_const_kernel(WT* dst, int64_t rows, int64_t cols, int64_t pitch, float value) {
  griddep_enter();
  const int64_t n = rows * cols;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    dst[(i / cols) * pitch + (i % cols)] = from_f32<WT>(value);
}

// ------------------------------------------------------------------ embed
template <typename WT>
__global__ void embed_kernel(const int32_t* __restrict__ tok, int tok_per_seq, int64_t tok_seq_stride,
                             const WT* __restrict__ emb, int d, int vocab, float* out, RowMap out_map) {
  griddep_enter();
  const int64_t r = blockIdx.x;
  int32_t id = tok[(r / tok_per_seq) * tok_seq_stride + (r % tok_per_seq)];
  if (id < 0 || id >= vocab) {
    if (threadIdx.x == 0) atomicExch(&g_device_error, 2);
    id = 0;
  }
  float* o = out + out_map.off(r);
  const WT* e = emb + (int64_t)id * d;
  for (int i = threadIdx.x; i < d; i += blockDim.x) o[i] = to_f32(e[i]);
}

// ------------------------------------------------------------------ rmsnorm
template <typename WT, typename OT>
__global__ void rmsnorm_kernel(const float* __restrict__ x, RowMap x_map, const WT* __restrict__ gamma, int d,
                               float eps, OT* out, int64_t ld_out) {
  griddep_enter();
  __shared__ float red[32];
  const int64_t r = blockIdx.x;
  const float* xr = x + x_map.off(r);
  float ss = 0.f;
  for (int i = threadIdx.x; i < d; i += blockDim.x) ss = fmaf(xr[i], xr[i], ss);
  ss = block_sum(ss, red);
  const float inv = rsqrtf(ss / (float)d + eps);
  OT* o = out + r * ld_out;
  for (int i = threadIdx.x; i < d; i += blockDim.x) o[i] = from_f32<OT>(to_f32(gamma[i]) * xr[i] * inv);
}

// The same, one warp per row for d = 128 * NV: the row stays in registers
// (NV float4 per lane), the sum of squares is a warp butterfly, and the
// output is written with 16-byte stores.  Used for every row count at these
// widths (rows 16-byte aligned).
template <typename WT, typename OT, int NV>
__global__ void __launch_bounds__(256) rmsnorm_warp_kernel(const float* __restrict__ x, RowMap x_map, int64_t rows,
                                                           const WT* __restrict__ gamma, float eps, OT* out,
                                                           int64_t ld_out) {
  griddep_enter();
  constexpr int d = 128 * NV;
  const int lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (r >= rows) return;
  const float4* xr = reinterpret_cast<const float4*>(x + x_map.off(r));
  float4 v[NV];
  float ss = 0.f;
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    v[k] = xr[k * 32 + lane];
    ss = fmaf(v[k].x, v[k].x, ss);
    ss = fmaf(v[k].y, v[k].y, ss);
    ss = fmaf(v[k].z, v[k].z, ss);
    ss = fmaf(v[k].w, v[k].w, ss);
  }
  ss = warp_sum(ss);
  const float inv = rsqrtf(ss / (float)d + eps);
  OT* o = out + r * ld_out;
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int i = 4 * (k * 32 + lane);  // this lane's float4 of chunk k
    const float y0 = to_f32(gamma[i]) * v[k].x * inv, y1 = to_f32(gamma[i + 1]) * v[k].y * inv;
    const float y2 = to_f32(gamma[i + 2]) * v[k].z * inv, y3 = to_f32(gamma[i + 3]) * v[k].w * inv;
    if constexpr (std::is_same<OT, bf16>::value) {
      __nv_bfloat162 p0 = __floats2bfloat162_rn(y0, y1);
      __nv_bfloat162 p1 = __floats2bfloat162_rn(y2, y3);
      uint2 w;
      w.x = *reinterpret_cast<uint32_t*>(&p0);
      w.y = *reinterpret_cast<uint32_t*>(&p1);
      *reinterpret_cast<uint2*>(o + i) = w;
    } else {
      *reinterpret_cast<float4*>(o + i) = make_float4(y0, y1, y2, y3);
    }
  }
}

// Merge operand (eqs. 2.9-2.10): row b = [e_t ; RMSNorm_s(s_{t-1})] for the
// report's merge, [e_t ; s_{t-1}] for the convex gate.
template <typename WT, typename OT>
__global__ void merge_prep_kernel(const float* __restrict__ e, RowMap e_map, const float* __restrict__ s,
                                  const WT* __restrict__ gamma, int d, float eps, int kind, OT* out) {
  griddep_enter();
  __shared__ float red[32];
  const int b = blockIdx.x;
  const float* er = e + e_map.off(b);
  const float* sr = s + (int64_t)b * d;
  OT* o = out + (int64_t)b * 2 * d;
  float ss = 0.f;
  for (int i = threadIdx.x; i < d; i += blockDim.x) ss = fmaf(sr[i], sr[i], ss);
  ss = block_sum(ss, red);
  const float inv = rsqrtf(ss / (float)d + eps);
  for (int i = threadIdx.x; i < d; i += blockDim.x) {
    o[i] = from_f32<OT>(er[i]);
    o[d + i] = from_f32<OT>(kind == 0 ? to_f32(gamma[i]) * sr[i] * inv : sr[i]);
  }
}

// ------------------------------------------------------------------ scatter
// Row r of x (columns col0 + h*hd + i) goes to dst[b][h][dst_row0 + i_seq][i]
// with b = r / rows_per_seq, i_seq = r % rows_per_seq, rotating the pair
// (i, i+hd/2) by (pos0 + i_seq) * base^(-2i/hd) when rope != 0.  A thread
// moves eight consecutive pairs with 16-byte accesses (hd % 16 == 0).
template <typename XT, typename KT>
__global__ void head_scatter_kernel(const XT* __restrict__ x, int64_t ld_x, int64_t col0, int64_t rows,
                                    int rows_per_seq, int pos0, int dst_row0, int H, int hd, int rope,
                                    const float* __restrict__ rope_cs, KT* dst, int64_t ld_t) {
  griddep_enter();
  const int half = hd / 2, oct = half / 8;
  const int64_t n = rows * H * oct;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < n; idx += (int64_t)gridDim.x * blockDim.x) {
    const int i = (int)(idx % oct) * 8;
    const int h = (int)((idx / oct) % H);
    const int64_t r = idx / ((int64_t)oct * H);
    const int64_t b = r / rows_per_seq;
    const int i_seq = (int)(r % rows_per_seq);
    const int pos = pos0 + i_seq;
    const XT* xr = x + r * ld_x + col0 + (int64_t)h * hd;
    float a[8], c[8];
    load8(xr + i, a);
    load8(xr + i + half, c);
    if (rope) {
      const float4* cs = reinterpret_cast<const float4*>(rope_cs + ((int64_t)pos * half + i) * 2);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float4 t = cs[u];  // (cos, sin) of pairs i+2u and i+2u+1
        const float a0 = a[2 * u] * t.x - c[2 * u] * t.y, c0 = a[2 * u] * t.y + c[2 * u] * t.x;
        const float a1 = a[2 * u + 1] * t.z - c[2 * u + 1] * t.w, c1 = a[2 * u + 1] * t.w + c[2 * u + 1] * t.z;
        a[2 * u] = a0;
        c[2 * u] = c0;
        a[2 * u + 1] = a1;
        c[2 * u + 1] = c1;
      }
    }
    KT* o = dst + ((b * H + h) * ld_t + dst_row0 + i_seq) * hd;
    store8(o + i, a);
    store8(o + i + half, c);
  }
}

// One row per sequence (the encoder step's keys/values or memory row of the
// token at t_b), written to store row t_b - 1 and rotated at t_b - 1, for the
// sequences whose transition encodes its token; the same 16-byte moves as
// head_scatter_kernel.
template <typename XT, typename KT>
__global__ void head_insert_kernel(const XT* __restrict__ x, int64_t ld_x, int64_t col0, int B, SeqPos sp, int H,
                                   int hd, int rope, const float* __restrict__ rope_cs, KT* dst, int64_t ld_t) {
  griddep_enter();
  const int half = hd / 2, oct = half / 8;
  const int64_t n = (int64_t)B * H * oct;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < n; idx += (int64_t)gridDim.x * blockDim.x) {
    const int i = (int)(idx % oct) * 8;
    const int h = (int)((idx / oct) % H);
    const int b = (int)(idx / ((int64_t)oct * H));
    if (!sp.encodes(b)) continue;
    const int pos = sp.dec[b];  // t_b - 1
    const XT* xr = x + (int64_t)b * ld_x + col0 + (int64_t)h * hd;
    float a[8], c[8];
    load8(xr + i, a);
    load8(xr + i + half, c);
    if (rope) {
      const float4* cs = reinterpret_cast<const float4*>(rope_cs + ((int64_t)pos * half + i) * 2);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float4 t = cs[u];
        const float a0 = a[2 * u] * t.x - c[2 * u] * t.y, c0 = a[2 * u] * t.y + c[2 * u] * t.x;
        const float a1 = a[2 * u + 1] * t.z - c[2 * u + 1] * t.w, c1 = a[2 * u + 1] * t.w + c[2 * u + 1] * t.z;
        a[2 * u] = a0;
        c[2 * u] = c0;
        a[2 * u + 1] = a1;
        c[2 * u + 1] = c1;
      }
    }
    KT* o = dst + (((int64_t)b * H + h) * ld_t + pos) * hd;
    store8(o + i, a);
    store8(o + i + half, c);
  }
}

// ------------------------------------------------------------------ positions
// et[b] = e[b][row_b]: the encoder output the merge of sequence b's
// transition reads (row t_b - 1; an idle sequence copies a row it holds).
__global__ void erow_gather_kernel(const float* __restrict__ e, int max_len, int d, SeqPos sp, float* et) {
  griddep_enter();
  const int b = blockIdx.x;
  const int row = min(sp.dec[b], max_len - 1);
  const float4* src = reinterpret_cast<const float4*>(e + ((int64_t)b * max_len + row) * d);
  float4* dst = reinterpret_cast<float4*>(et + (int64_t)b * d);
  for (int i = threadIdx.x; i < d / 4; i += blockDim.x) dst[i] = src[i];
}

// e[b][t_b - 1] = et[b] for the sequences whose transition encoded their token.
__global__ void erow_scatter_kernel(const float* __restrict__ et, int max_len, int d, SeqPos sp, float* e) {
  griddep_enter();
  const int b = blockIdx.x;
  if (!sp.encodes(b)) return;
  const float4* src = reinterpret_cast<const float4*>(et + (int64_t)b * d);
  float4* dst = reinterpret_cast<float4*>(e + ((int64_t)b * max_len + sp.dec[b]) * d);
  for (int i = threadIdx.x; i < d / 4; i += blockDim.x) dst[i] = src[i];
}

__global__ void save_rows_kernel(const float* __restrict__ s, float* s_save, const bf16* __restrict__ zb,
                                 bf16* zb_save, const float* __restrict__ ss, float* ss_save, int B, int d, int n_ss) {
  griddep_enter();
  const int b = blockIdx.x;
  for (int i = threadIdx.x; i < d; i += blockDim.x) s_save[(int64_t)b * d + i] = s[(int64_t)b * d + i];
  if (zb)
    for (int i = threadIdx.x; i < d; i += blockDim.x) zb_save[(int64_t)b * d + i] = zb[(int64_t)b * d + i];
  if (ss)
    for (int i = threadIdx.x; i < n_ss; i += blockDim.x) ss_save[(int64_t)i * B + b] = ss[(int64_t)i * B + b];
}

// One block per sequence: the active ones advance (n_dec = t_b, n_enc at
// least t_b); in a masked phase the idle ones get their saved rows back.
__global__ void advance_kernel(int32_t* dec, int32_t* enc, const int32_t* __restrict__ lim, int B, int d, float* s,
                               const float* __restrict__ s_save, bf16* zb, const bf16* __restrict__ zb_save, float* ss,
                               const float* __restrict__ ss_save, int n_ss) {
  griddep_wait();
  const int b = blockIdx.x;
  const int db = dec[b];
  const bool act = lim == nullptr || db < lim[b];
  if (!act && s_save) {
    for (int i = threadIdx.x; i < d; i += blockDim.x) s[(int64_t)b * d + i] = s_save[(int64_t)b * d + i];
    if (zb)
      for (int i = threadIdx.x; i < d; i += blockDim.x) zb[(int64_t)b * d + i] = zb_save[(int64_t)b * d + i];
    if (ss)
      for (int i = threadIdx.x; i < n_ss; i += blockDim.x) ss[(int64_t)i * B + b] = ss_save[(int64_t)i * B + b];
  }
  __syncthreads();  // every thread has read dec[b] before it changes
  if (threadIdx.x == 0 && act) {
    dec[b] = db + 1;
    if (enc[b] < db + 1) enc[b] = db + 1;
  }
  griddep_launch_dependents();
}

__global__ void set_positions_kernel(int32_t* n, int b0, int b1, int32_t value) {
  griddep_enter();
  for (int b = b0 + (int)(blockIdx.x * blockDim.x + threadIdx.x); b < b1; b += (int)(gridDim.x * blockDim.x))
    n[b] = value;
}

// ------------------------------------------------------------------ readout
__global__ void logp_gather_kernel(const float* __restrict__ logits, int V, const int32_t* __restrict__ next,
                                   int64_t next_stride, float* logp, int64_t ld_logp, const int32_t* __restrict__ dec,
                                   const int32_t* __restrict__ lim) {
  griddep_enter();
  __shared__ float red[32];
  const int b = blockIdx.x;
  if (lim != nullptr && !(dec[b] < lim[b])) return;  // this sequence's phase has no next token here
  const float* l = logits + (int64_t)b * V;
  // 16-byte loads when every row starts 16-byte aligned (V % 4 == 0); the
  // second pass finds the row in L1/L2
  const bool vec = (V & 3) == 0;
  const float4* l4 = reinterpret_cast<const float4*>(l);
  float mx = -INFINITY;
  if (vec) {
    for (int i = threadIdx.x; i < V / 4; i += blockDim.x) {
      const float4 x = l4[i];
      mx = fmaxf(mx, fmaxf(fmaxf(x.x, x.y), fmaxf(x.z, x.w)));
    }
  } else {
    for (int i = threadIdx.x; i < V; i += blockDim.x) mx = fmaxf(mx, l[i]);
  }
  mx = block_max(mx, red);
  float s = 0.f;
  if (vec) {
    for (int i = threadIdx.x; i < V / 4; i += blockDim.x) {
      const float4 x = l4[i];
      s += __expf(x.x - mx) + __expf(x.y - mx) + __expf(x.z - mx) + __expf(x.w - mx);
    }
  } else {
    for (int i = threadIdx.x; i < V; i += blockDim.x) s += __expf(l[i] - mx);
  }
  s = block_sum(s, red);
  if (threadIdx.x == 0) {
    int32_t id = next[(int64_t)b * next_stride];
    if (id < 0 || id >= V) {
      atomicExch(&g_device_error, 2);
      id = 0;
    }
    logp[(int64_t)b * ld_logp] = l[id] - (mx + logf(s));
  }
}

// RL replay ratios (eq. 5.5): per token r = exp(log p - log mu) where the
// token is a sampled action, 1 (no action factor) elsewhere; per sequence
// the log of the product of the action ratios.  One block per sequence; the
// sum runs in double in a fixed order (thread-strided partials, then a fixed
// tree), so it does not depend on timing.
__global__ void replay_ratio_kernel(const float* __restrict__ logp, const float* __restrict__ logmu,
                                    const uint8_t* __restrict__ mask, int n, float* ratio, float* seq_logratio) {
  griddep_enter();
  __shared__ double part[256];
  const int b = blockIdx.x;
  const int64_t base = (int64_t)b * n;
  double acc = 0.0;
  for (int i = threadIdx.x; i < n; i += 256) {
    const bool act = mask[base + i] != 0;
    const float dl = logp[base + i] - logmu[base + i];
    if (ratio) ratio[base + i] = act ? expf(dl) : 1.0f;
    if (act) acc += (double)dl;
  }
  part[threadIdx.x] = acc;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0 && seq_logratio) seq_logratio[b] = (float)part[0];
}

// order-preserving key of a float (larger float -> larger key); -0 and +0
// share a key so equal values compare equal as floats do
__device__ __forceinline__ uint32_t fkey(float f) {
  if (f == 0.0f) f = 0.0f;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

constexpr int kSampleThreads = 1024;
constexpr int kMaxTopK = 256;

// One block per sequence.  (1) radix-select the key of the top_k-th largest
// logit; (2) gather every logit above it plus the lowest-id ones equal to it;
// (3) sort the candidates by (value desc, id asc); (4) thread 0 forms the
// tempered weights, their running sums in that order, draws the Philox
// uniform for counter (t, b, 0, 0) and picks the first candidate whose
// running sum exceeds u * total.
__global__ void __launch_bounds__(kSampleThreads)
    sample_kernel(const float* __restrict__ logits, int V, float temperature, int top_k, uint32_t k0, uint32_t k1,
                  uint32_t t, const int32_t* __restrict__ t_rows, int32_t* token, float* logp_tok, float* logmu) {
  griddep_enter();
  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_sel[2];
  __shared__ float red[32];
  __shared__ uint32_t cand_key[kMaxTopK];
  __shared__ int32_t cand_id[kMaxTopK];
  __shared__ uint32_t scan[kSampleThreads];
  __shared__ uint32_t n_gt;
  const int b = blockIdx.x, tid = threadIdx.x;
  const float* l = logits + (int64_t)b * V;
  const int k = top_k < V ? top_k : V;

  uint32_t prefix = 0, mask = 0, need = (uint32_t)k;
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < 256; i += kSampleThreads) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < V; i += kSampleThreads) {
      const uint32_t u = fkey(l[i]);
      if ((u & mask) == prefix) atomicAdd(&hist[(u >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid == 0) {
      uint32_t cum = 0, sel = 0;
      for (int dg = 255; dg >= 0; --dg) {
        if (cum + hist[dg] >= need) { sel = (uint32_t)dg; break; }
        cum += hist[dg];
      }
      s_sel[0] = sel;
      s_sel[1] = need - cum;
    }
    __syncthreads();
    prefix |= s_sel[0] << shift;
    mask |= 255u << shift;
    need = s_sel[1];
    __syncthreads();
  }
  const uint32_t thr = prefix;  // key of the k-th largest logit; `need` ties at it are taken

  // ordered pass over contiguous id ranges so ties are taken by ascending id
  const int per = (V + kSampleThreads - 1) / kSampleThreads;
  const int lo = tid * per, hi = min(V, lo + per);
  uint32_t my_eq = 0;
  for (int i = lo; i < hi; ++i) my_eq += fkey(l[i]) == thr;
  scan[tid] = my_eq;
  if (tid == 0) n_gt = 0;
  __syncthreads();
  for (int off = 1; off < kSampleThreads; off <<= 1) {  // inclusive scan
    const uint32_t v = tid >= off ? scan[tid - off] : 0u;
    __syncthreads();
    scan[tid] += v;
    __syncthreads();
  }
  uint32_t eq_rank = scan[tid] - my_eq;
  const uint32_t n_above = (uint32_t)k - need;
  for (int i = lo; i < hi; ++i) {
    const uint32_t u = fkey(l[i]);
    if (u > thr) {
      const uint32_t slot = atomicAdd(&n_gt, 1u);
      cand_key[slot] = u;
      cand_id[slot] = i;
    } else if (u == thr) {
      if (eq_rank < need) {
        cand_key[n_above + eq_rank] = u;
        cand_id[n_above + eq_rank] = i;
      }
      ++eq_rank;
    }
  }
  __syncthreads();
  // bitonic sort of kMaxTopK entries (padding sorts last)
  for (int i = tid; i < kMaxTopK; i += kSampleThreads)
    if (i >= k) { cand_key[i] = 0u; cand_id[i] = 0x7FFFFFFF; }
  __syncthreads();
  for (int size = 2; size <= kMaxTopK; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      if (tid < kMaxTopK) {
        const int j = tid ^ stride;
        if (j > tid) {
          // "a before b": larger key, or equal key and smaller id
          const bool asc = (tid & size) == 0;
          const uint32_t ka = cand_key[tid], kb = cand_key[j];
          const int32_t ia = cand_id[tid], ib = cand_id[j];
          const bool a_first = ka > kb || (ka == kb && ia < ib);
          if (asc ? !a_first : a_first) {
            cand_key[tid] = kb; cand_key[j] = ka;
            cand_id[tid] = ib; cand_id[j] = ia;
          }
        }
      }
      __syncthreads();
    }
  }
  // raw log-softmax normaliser over the whole vocabulary
  const float mx = l[cand_id[0]];
  float s = 0.f;
  for (int i = tid; i < V; i += kSampleThreads) s += __expf(l[i] - mx);
  s = block_sum(s, red);
  if (tid == 0) {
    const float z0 = l[cand_id[0]] / temperature;
    float w[kMaxTopK];
    float total = 0.f;
    for (int r = 0; r < k; ++r) {
      w[r] = expf(l[cand_id[r]] / temperature - z0);
      total += w[r];
    }
    uint32_t c[4] = {t_rows ? (uint32_t)t_rows[b] : t, (uint32_t)b, 0u, 0u};
    philox4x32_10(c, k0, k1);
    const float u = (float)(c[0] >> 8) * (1.0f / 16777216.0f);
    const float target = u * total;
    float run = 0.f;
    int pick = k - 1;
    for (int r = 0; r < k; ++r) {
      run += w[r];
      if (run > target) { pick = r; break; }
    }
    const int32_t id = cand_id[pick];
    if (token) token[b] = id;
    if (logmu) logmu[b] = (l[id] / temperature - z0) - logf(total);
    if (logp_tok) logp_tok[b] = l[id] - (mx + logf(s));
  }
}

template <typename WT>
__global__ void broadcast_kernel(const WT* __restrict__ src, int d, float* dst, int B) {
  griddep_enter();
  const int64_t n = (int64_t)B * d;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    dst[i] = to_f32(src[i % d]);
}

__global__ void copy_kernel(float* dst, const float* src, int64_t n) {
  griddep_enter();
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    dst[i] = src[i];
}

inline unsigned grid_for(int64_t n, int threads, int cap = 148 * 16) {
  int64_t g = (n + threads - 1) / threads;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return (unsigned)g;
}

}  // namespace

template <typename WT>
cudaError_t init_normal(WT* dst, int64_t rows, int64_t cols, int64_t pitch, uint64_t seed, uint32_t sid, float std,
                        cudaStream_t st) {
  const int64_t n = rows * cols;
  {
    const cudaError_t e_l = launch_pdl(init_normal_kernel<WT>, dim3(grid_for(n, 256, 148 * 64)), dim3(256), 0, st, dst, rows, cols, pitch, (uint32_t)seed,
                                                                     (uint32_t)(seed >> 32), sid, std);
    if (e_l != cudaSuccess) return e_l;
  }
  return cudaGetLastError();
}

template <typename WT>
cudaError_t init_const(WT* dst, int64_t rows, int64_t cols, int64_t pitch, float value, cudaStream_t st) {
  {
    const cudaError_t e_l = launch_pdl(init_const_kernel<WT>, dim3(grid_for(rows * cols, 256)), dim3(256), 0, st, dst, rows, cols, pitch, value);
    if (e_l != cudaSuccess) return e_l;
  }
  return cudaGetLastError();
}

template <typename WT>
cudaError_t embed(const int32_t* tok, int64_t n_rows, int tok_per_seq, int64_t tok_seq_stride, const WT* emb, int d,
                  int vocab, float* out, RowMap out_map, cudaStream_t st) {
  {
    const cudaError_t e_l = launch_pdl(embed_kernel<WT>, dim3((unsigned)n_rows), dim3(128), 0, st, tok, tok_per_seq, tok_seq_stride, emb, d, vocab, out, out_map);
    if (e_l != cudaSuccess) return e_l;
  }
  return cudaGetLastError();
}

// The kernel (and with it the order of the sum of squares) is chosen from the
// row width and layout alone, never from the number of rows, so a row's
// result does not depend on how many rows share the launch (the batch).
template <typename WT, typename OT>
cudaError_t rmsnorm(const float* x, RowMap x_map, const WT* gamma, int64_t rows, int d, float eps, OT* out,
                    int64_t ld_out, cudaStream_t st) {
  const bool rows16 = x_map.ld % 4 == 0 && (x_map.per_group <= 0 || x_map.group_stride % 4 == 0) && ld_out % 4 == 0;
  if (rows16 && (d == 256 || d == 512 || d == 1024 || d == 2048)) {
    const dim3 grid((unsigned)((rows + 7) / 8));
    cudaError_t e_l;
    switch (d) {
      case 256: e_l = launch_pdl(rmsnorm_warp_kernel<WT, OT, 2>, grid, dim3(256), 0, st, x, x_map, rows, gamma, eps, out, ld_out); break;
      case 512: e_l = launch_pdl(rmsnorm_warp_kernel<WT, OT, 4>, grid, dim3(256), 0, st, x, x_map, rows, gamma, eps, out, ld_out); break;
      case 1024: e_l = launch_pdl(rmsnorm_warp_kernel<WT, OT, 8>, grid, dim3(256), 0, st, x, x_map, rows, gamma, eps, out, ld_out); break;
      default: e_l = launch_pdl(rmsnorm_warp_kernel<WT, OT, 16>, grid, dim3(256), 0, st, x, x_map, rows, gamma, eps, out, ld_out); break;
    }
    return e_l != cudaSuccess ? e_l : cudaGetLastError();
  }
  const int threads = d >= 1024 ? 256 : 128;
  {
    const cudaError_t e_l = launch_pdl(rmsnorm_kernel<WT, OT>, dim3((unsigned)rows), dim3(threads), 0, st, x, x_map, gamma, d, eps, out, ld_out);
    if (e_l != cudaSuccess) return e_l;
  }
  return cudaGetLastError();
}

template <typename WT, typename OT>
cudaError_t merge_prep(const float* e, RowMap e_map, const float* s, const WT* gamma, int B, int d, float eps,
                       int kind, OT* out, cudaStream_t st) {
  {
    const cudaError_t e_l = launch_pdl(merge_prep_kernel<WT, OT>, dim3(B), dim3(d >= 1024 ? 256 : 128), 0, st, e, e_map, s, gamma, d, eps, kind, out);
    if (e_l != cudaSuccess) return e_l;
  }
  return cudaGetLastError();
}

template <typename XT, typename KT>
cudaError_t head_scatter(const XT* x, int64_t ld_x, int64_t col0, int64_t rows, int rows_per_seq, int pos0, int dst_row0, int H,
                         int hd, int rope, const float* rope_cs, KT* dst, int64_t ld_t, cudaStream_t st) {
  if (hd % 16) return cudaErrorInvalidValue;
  const int64_t n = rows * H * (hd / 16);
  {
    const cudaError_t e_l = launch_pdl(head_scatter_kernel<XT, KT>, dim3(grid_for(n, 256, 148 * 32)), dim3(256), 0, st, x, ld_x, col0, rows, rows_per_seq, pos0, dst_row0, H,
                                                                          hd, rope, rope_cs, dst, ld_t);
    if (e_l != cudaSuccess) return e_l;
  }
  return cudaGetLastError();
}

template <typename XT, typename KT>
cudaError_t head_insert(const XT* x, int64_t ld_x, int64_t col0, int B, const SeqPos& sp, int H, int hd, int rope,
                        const float* rope_cs, KT* dst, int64_t ld_t, cudaStream_t st) {
  if (hd % 16 || !sp.on()) return cudaErrorInvalidValue;
  const int64_t n = (int64_t)B * H * (hd / 16);
  const cudaError_t e_l = launch_pdl(head_insert_kernel<XT, KT>, dim3(grid_for(n, 256, 148 * 32)), dim3(256), 0, st, x,
                                     ld_x, col0, B, sp, H, hd, rope, rope_cs, dst, ld_t);
  return e_l != cudaSuccess ? e_l : cudaGetLastError();
}

cudaError_t erow_gather(const float* e, int max_len, int d, int B, const SeqPos& sp, float* et, cudaStream_t st) {
  if (d % 4 || !sp.on()) return cudaErrorInvalidValue;
  const cudaError_t e_l = launch_pdl(erow_gather_kernel, dim3(B), dim3(128), 0, st, e, max_len, d, sp, et);
  return e_l != cudaSuccess ? e_l : cudaGetLastError();
}

cudaError_t erow_scatter(const float* et, int max_len, int d, int B, const SeqPos& sp, float* e, cudaStream_t st) {
  if (d % 4 || !sp.on()) return cudaErrorInvalidValue;
  const cudaError_t e_l = launch_pdl(erow_scatter_kernel, dim3(B), dim3(128), 0, st, et, max_len, d, sp, e);
  return e_l != cudaSuccess ? e_l : cudaGetLastError();
}

cudaError_t advance_positions(int32_t* dec, int32_t* enc, const int32_t* lim, int B, int d, float* s,
                              const float* s_save, bf16* zb, const bf16* zb_save, float* ss, const float* ss_save,
                              int n_ss, cudaStream_t st) {
  const cudaError_t e_l = launch_pdl(advance_kernel, dim3(B), dim3(128), 0, st, dec, enc, lim, B, d, s, s_save, zb,
                                     zb_save, ss, ss_save, n_ss);
  return e_l != cudaSuccess ? e_l : cudaGetLastError();
}

cudaError_t save_rows(const float* s, float* s_save, const bf16* zb, bf16* zb_save, const float* ss, float* ss_save,
                      int B, int d, int n_ss, cudaStream_t st) {
  const cudaError_t e_l =
      launch_pdl(save_rows_kernel, dim3(B), dim3(128), 0, st, s, s_save, zb, zb_save, ss, ss_save, B, d, n_ss);
  return e_l != cudaSuccess ? e_l : cudaGetLastError();
}

cudaError_t set_positions(int32_t* n, int b0, int b1, int32_t value, cudaStream_t st) {
  if (b1 <= b0) return cudaSuccess;
  const cudaError_t e_l = launch_pdl(set_positions_kernel, dim3(grid_for(b1 - b0, 128)), dim3(128), 0, st, n, b0, b1,
                                     value);
  return e_l != cudaSuccess ? e_l : cudaGetLastError();
}

cudaError_t logp_gather(const float* logits, int B, int V, const int32_t* next, int64_t next_stride, float* logp,
                        int64_t ld_logp, const int32_t* dec, const int32_t* lim, cudaStream_t st) {
  {
    const cudaError_t e_l = launch_pdl(logp_gather_kernel, dim3(B), dim3(256), 0, st, logits, V, next, next_stride, logp, ld_logp,
                                       dec, lim);
    if (e_l != cudaSuccess) return e_l;
  }
  return cudaGetLastError();
}

cudaError_t replay_ratios(const float* logp, const float* logmu, const uint8_t* mask, int B, int n, float* ratio,
                          float* seq_logratio, cudaStream_t st) {
  {
    const cudaError_t e_l = launch_pdl(replay_ratio_kernel, dim3(B), dim3(256), 0, st, logp, logmu, mask, n, ratio,
                                       seq_logratio);
    if (e_l != cudaSuccess) return e_l;
  }
  return cudaGetLastError();
}

cudaError_t sample_topk(const float* logits, int B, int V, float temperature, int top_k, uint64_t seed, uint32_t t,
                        const int32_t* t_rows, int32_t* token, float* logp_tok, float* logmu, cudaStream_t st) {
  if (top_k < 1 || top_k > kMaxTopK || !(temperature > 0.f)) return cudaErrorInvalidValue;
  {
    const cudaError_t e_l = launch_pdl(sample_kernel, dim3(B), dim3(kSampleThreads), 0, st, logits, V, temperature, top_k, (uint32_t)seed, (uint32_t)(seed >> 32), t,
                                             t_rows, token, logp_tok, logmu);
    if (e_l != cudaSuccess) return e_l;
  }
  return cudaGetLastError();
}

template <typename WT>
cudaError_t broadcast_row(const WT* src, int d, float* dst, int B, cudaStream_t st) {
  {
    const cudaError_t e_l = launch_pdl(broadcast_kernel<WT>, dim3(grid_for((int64_t)B * d, 256)), dim3(256), 0, st, src, d, dst, B);
    if (e_l != cudaSuccess) return e_l;
  }
  return cudaGetLastError();
}

cudaError_t copy_f32(float* dst, const float* src, int64_t n, cudaStream_t st) {
  {
    const cudaError_t e_l = launch_pdl(copy_kernel, dim3(grid_for(n, 256)), dim3(256), 0, st, dst, src, n);
    if (e_l != cudaSuccess) return e_l;
  }
  return cudaGetLastError();
}

#define RLT_INST_W(WT)                                                                                              \
  template cudaError_t init_normal<WT>(WT*, int64_t, int64_t, int64_t, uint64_t, uint32_t, float, cudaStream_t);  \
  template cudaError_t init_const<WT>(WT*, int64_t, int64_t, int64_t, float, cudaStream_t);                      \
  template cudaError_t embed<WT>(const int32_t*, int64_t, int, int64_t, const WT*, int, int, float*, RowMap,     \
                                 cudaStream_t);                                                                   \
  template cudaError_t rmsnorm<WT, WT>(const float*, RowMap, const WT*, int64_t, int, float, WT*, int64_t,        \
                                       cudaStream_t);                                                             \
  template cudaError_t merge_prep<WT, WT>(const float*, RowMap, const float*, const WT*, int, int, float, int,    \
                                          WT*, cudaStream_t);                                                     \
  template cudaError_t head_scatter<float, WT>(const float*, int64_t, int64_t, int64_t, int, int, int, int, int, int,   \
                                               const float*, WT*, int64_t, cudaStream_t);                         \
  template cudaError_t head_insert<float, WT>(const float*, int64_t, int64_t, int, const SeqPos&, int, int, int,  \
                                              const float*, WT*, int64_t, cudaStream_t);                          \
  template cudaError_t broadcast_row<WT>(const WT*, int, float*, int, cudaStream_t);

RLT_INST_W(float)
RLT_INST_W(bf16)
template cudaError_t head_scatter<bf16, bf16>(const bf16*, int64_t, int64_t, int64_t, int, int, int, int, int, int,
                                              const float*, bf16*, int64_t, cudaStream_t);

// ------------------------------------------------------------------ failure-detection probe
namespace {
// One thread waits on an mbarrier that expects one arrival which no thread
// ever makes, so the bounded wait must run out after limit_ns: the same
// mbar_wait the tensor-core kernels use, which then raises the device error
// word and returns instead of spinning on.
__global__ void bounded_wait_probe_kernel(uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  fence_mbar_init();
  const uint64_t t0 = globaltimer_ns();
  const bool ok = mbar_wait(b, 0, limit_ns);
  g_probe_waited_ns = ok ? 0ull : (unsigned long long)(globaltimer_ns() - t0);
}
}  // namespace

cudaError_t bounded_wait_probe(uint64_t limit_ns, uint64_t* waited_ns, cudaStream_t st) {
  bounded_wait_probe_kernel<<<1, 32, 0, st>>>(limit_ns);
  note_launch();
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return e;
  unsigned long long v = 0;
  e = cudaMemcpyFromSymbol(&v, g_probe_waited_ns, sizeof(v));
  *waited_ns = v;
  return e;
}

}  // namespace rlt
