// bf16 split attention (placeholder routing to the CUDA-core kernel until the tcgen05
// kernel lands).
#include "common.cuh"

namespace ispa {
cudaError_t launch_attn_bf16(const AttnArgs &a, cudaStream_t s) { return launch_attn_simt_bf16(a, s); }
}  // namespace ispa
