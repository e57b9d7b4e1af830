// gemm_tc_epi_a.cu -- instantiates the tensor-core GEMM for the EPI_STORE and
// EPI_RESID epilogues (split from the other epilogues to compile in parallel).
#include "gemm_tc_kernel.cuh"

namespace rlt {
namespace gemm_detail {
template cudaError_t launch_gemm_epi<EPI_STORE>(const CUtensorMap&, const CUtensorMap&, int, int, int, int, int, int, float*,
                                             const EpiParams&, cudaStream_t);
template cudaError_t launch_gemm_epi<EPI_RESID>(const CUtensorMap&, const CUtensorMap&, int, int, int, int, int, int, float*,
                                             const EpiParams&, cudaStream_t);
}  // namespace gemm_detail
}  // namespace rlt
