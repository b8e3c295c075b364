// tcgen05 GEMM (placeholder until the tensor-core GEMM lands): reports no
// supported shapes, so the layer uses the CUDA-core GEMM.
#include "common.cuh"
#include "kernels.cuh"

namespace hstu {
bool tc_gemm_supported(const GemmParams&, int) { return false; }
cudaError_t launch_gemm_tc(const GemmParams&, cudaStream_t) { return cudaErrorNotSupported; }
}  // namespace hstu
