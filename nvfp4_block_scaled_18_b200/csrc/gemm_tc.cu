// tcgen05 block-scaled FP4 GEMM (large M).  Not built yet: the entry point
// reports "not supported" so nvfp4_gemm returns NVFP4_ERR_UNSUPPORTED.
#include "kernels.h"

namespace nvfp4 {

cudaError_t launch_gemm_tc(const GemmArgs&, int, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace nvfp4
