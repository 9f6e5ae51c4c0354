// gemm_tc.cu -- placeholder until the tcgen05 grouped GEMM lands.
#include "common.cuh"
#include "kernels.h"

namespace moe {
bool gemm_tc_supported(const GemmArgs&, bool, bool) { return false; }
cudaError_t launch_gemm_tc(const GemmArgs&, bool, bool, moe_diag*, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace moe
