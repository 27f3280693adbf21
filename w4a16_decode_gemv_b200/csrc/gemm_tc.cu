// Tensor-core W4A16 skinny GEMM for M >= 16 (not yet built).
#include "internal.h"

namespace w4a16 {

cudaError_t launch_gemm_tc(const GemmProblem&, const Workspace&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace w4a16
