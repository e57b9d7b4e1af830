// gemm_tc_epi_b.cu -- instantiates the tensor-core GEMM for the EPI_SWIGLU and
// EPI_GATE epilogues (split from the other epilogues to compile in parallel).
#include "gemm_tc_kernel.cuh"

namespace rlt {
namespace gemm_detail {
template cudaError_t launch_gemm_epi<EPI_SWIGLU>(const CUtensorMap&, const CUtensorMap&, int, int, int, int, int, int, float*,
                                             const EpiParams&, cudaStream_t);
template cudaError_t launch_gemm_epi<EPI_GATE>(const CUtensorMap&, const CUtensorMap&, int, int, int, int, int, int, float*,
                                             const EpiParams&, cudaStream_t);
}  // namespace gemm_detail
}  // namespace rlt
