// gemm_tc.cu -- host side of the tensor-core GEMM (kernel in
// gemm_tc_kernel.cuh): TMA tensor maps, tile and cluster policy, dispatch.
#include <cuda.h>

#include <mutex>
#include <unordered_map>

#include "gemm_tc_kernel.cuh"

namespace rlt {

namespace gemm_detail {
template <int EPI>
cudaError_t launch_gemm_epi(const CUtensorMap& ta, const CUtensorMap& tb, int bn, int cs, int M, int N, int K,
                            int kb_per_split, float* split_ws, const EpiParams& ep, cudaStream_t st);
}

namespace {

// Shape-only stand-in used to ask the runtime how many clusters of a given
// size fit at once with a GEMM's shared-memory footprint.
__global__ void cluster_probe_kernel() {}

using gemm_detail::BK;
using gemm_detail::BM;

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
bool encode_tmap(CUtensorMap* tm, const void* base, int64_t rows, int64_t cols, int64_t ld, int box_rows) {
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

// Tensor maps depend only on (address, shape, pitch, box); weights and state
// buffers keep their addresses, so encoded maps are cached on the host.
struct TmapKey {
  const void* base;
  int64_t rows, cols, ld;
  int box_rows;
  bool operator==(const TmapKey& o) const {
    return base == o.base && rows == o.rows && cols == o.cols && ld == o.ld && box_rows == o.box_rows;
  }
};
struct TmapKeyHash {
  size_t operator()(const TmapKey& k) const {
    size_t h = std::hash<const void*>()(k.base);
    h ^= std::hash<int64_t>()(k.rows * 1000003 + k.cols * 7919 + k.ld * 31 + k.box_rows) + 0x9e3779b97f4a7c15ull +
         (h << 6) + (h >> 2);
    return h;
  }
};

bool make_tmap(CUtensorMap* tm, const void* base, int64_t rows, int64_t cols, int64_t ld, int box_rows) {
  static std::mutex mu;
  static std::unordered_map<TmapKey, CUtensorMap, TmapKeyHash> cache;
  const TmapKey key{base, rows, cols, ld, box_rows};
  {
    std::lock_guard<std::mutex> g(mu);
    auto it = cache.find(key);
    if (it != cache.end()) {
      *tm = it->second;
      return true;
    }
  }
  if (!encode_tmap(tm, base, rows, cols, ld, box_rows)) return false;
  std::lock_guard<std::mutex> g(mu);
  if (cache.size() > 65536) cache.clear();
  cache.emplace(key, *tm);
  return true;
}

}  // namespace

// How many clusters of `cs` CTAs, each holding the shared memory of a GEMM
// with 256-wide activation tiles, the device runs at once (queried once).
int max_active_clusters(int cs) {
  static int cache[9] = {0};
  if (cache[cs] == 0) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1, 1, cs);
    cfg.blockDim = dim3(256, 1, 1);
    cfg.dynamicSmemBytes = gemm_detail::TcCfg<256>::SMEM;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = cs;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    cudaFuncSetAttribute(cluster_probe_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         gemm_detail::TcCfg<256>::SMEM);
    if (cudaOccupancyMaxActiveClusters(&n, cluster_probe_kernel, &cfg) != cudaSuccess || n <= 0) {
      cudaGetLastError();
      n = kSmCount / cs;
    }
    cache[cs] = n;
  }
  return cache[cs];
}

// Decode-step plan (activation tile width and K-split cluster size) for an
// M x K weight, worked out once for the design batch of 256 rows: prefer an
// unsplit grid of 128- or 256-wide tiles that gives 80..148 CTAs (one wave,
// no reduction); otherwise the cluster split with the most CTAs that still
// fit in one wave (cluster occupancy included), wider tiles first.  The
// cluster size therefore depends on M and K only -- never on the actual
// batch -- so a sequence's result does not depend on the batch it shares a
// step with; only the tile width follows the batch (which does not change
// the accumulation order).
struct DecodePlan {
  int bn, cs;
};

DecodePlan decode_plan(int M, int K) {
  const int tiles = M / BM, kb = K / BK;
  for (int bn : {256, 128}) {
    const int ctas = tiles * (256 / bn);
    if (ctas >= 80 && ctas <= kSmCount) {
      // A long K split in two over 256-wide tiles keeps the same CTA count
      // with half the k-blocks each: the main loop (about 0.5 us per
      // 256-wide k-block against 0.35 us at 128) then ends sooner.
      if (bn == 128 && kb >= 32 && 2 * tiles <= kSmCount && tiles <= max_active_clusters(2))
        return {256, 2};
      return {bn, 1};
    }
  }
  if (tiles >= 80) return {256, 1};
  DecodePlan best{256, 1};
  int best_ctas = tiles;
  for (int cs = 2; cs <= 8; cs *= 2) {
    if (kb < 2 * cs) break;
    for (int bn : {256, 128}) {
      const int clusters = tiles * (256 / bn), ctas = clusters * cs;
      if (ctas > kSmCount || clusters > max_active_clusters(cs)) continue;
      if (ctas > best_ctas || (ctas == best_ctas && bn > best.bn)) {
        best = {bn, cs};
        best_ctas = ctas;
      }
    }
  }
  return best;
}

int gemm_tc_cluster(int M, int K, int split_mode) { return split_mode ? decode_plan(M, K).cs : 1; }

// Activation tile width: the smallest of 32/64/128/256 that covers N, except
// that decode steps with more than 128 rows use the planned width.
int gemm_tc_bn(int M, int N, int K, int split_mode) {
  if (split_mode && N > 128) return decode_plan(M, K).bn;
  return N <= 32 ? 32 : N <= 64 ? 64 : N <= 128 ? 128 : 256;
}

size_t gemm_tc_workspace_floats(int M, int N, int K, int split_mode) {
  if (M % BM || K % BK || N <= 0) return 0;
  const int cs = gemm_tc_cluster(M, K, split_mode);
  if (cs == 1) return 0;
  const int bn = gemm_tc_bn(M, N, K, split_mode);
  // every CTA of the grid owns cs slots of (bn / cs) x 128 floats
  return (size_t)(M / BM) * (size_t)((N + bn - 1) / bn) * cs * (size_t)bn * BM;
}

cudaError_t gemm_tc(const bf16* W, int64_t ldw, const bf16* X, int64_t ldx, int M, int N, int K, int epi,
                    const EpiParams& ep, int split_mode, float* ws, size_t ws_floats, cudaStream_t st) {
  if (M % BM || K % BK || N <= 0) return cudaErrorInvalidValue;
  const int bn = gemm_tc_bn(M, N, K, split_mode);
  const int cs = gemm_tc_cluster(M, K, split_mode);
  if (cs > 1 && (ws == nullptr || ws_floats < gemm_tc_workspace_floats(M, N, K, split_mode)))
    return cudaErrorInvalidValue;
  const int kb = K / BK;
  const int per = (kb + cs - 1) / cs;
  CUtensorMap ta, tb;
  if (!make_tmap(&ta, W, M, K, ldw, BM)) return cudaErrorInvalidValue;
  if (!make_tmap(&tb, X, N, K, ldx, bn)) return cudaErrorInvalidValue;
  using namespace gemm_detail;
  switch (epi) {
    case EPI_STORE: return launch_gemm_epi<EPI_STORE>(ta, tb, bn, cs, M, N, K, per, ws, ep, st);
    case EPI_RESID: return launch_gemm_epi<EPI_RESID>(ta, tb, bn, cs, M, N, K, per, ws, ep, st);
    case EPI_SWIGLU: return launch_gemm_epi<EPI_SWIGLU>(ta, tb, bn, cs, M, N, K, per, ws, ep, st);
    case EPI_GATE: return launch_gemm_epi<EPI_GATE>(ta, tb, bn, cs, M, N, K, per, ws, ep, st);
    case EPI_MERGE: return launch_gemm_epi<EPI_MERGE>(ta, tb, bn, cs, M, N, K, per, ws, ep, st);
    case EPI_CONVEX: return launch_gemm_epi<EPI_CONVEX>(ta, tb, bn, cs, M, N, K, per, ws, ep, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace rlt
