// attn_bwd.cu -- attention backward for one rank's head slice (placeholder
// until the tensor-core kernels land).
#include "ulysses_internal.cuh"

namespace uly {

cudaError_t launch_attn_bwd(const BwdLaunch &, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace uly
