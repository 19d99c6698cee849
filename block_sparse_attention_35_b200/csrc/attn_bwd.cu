// attn_bwd.cu - PBSA backward (placeholder until the kernel lands).
#include "pbsa_internal.cuh"

namespace pbsa {

cudaError_t launch_attn_bwd(const BwdArgs&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace pbsa
