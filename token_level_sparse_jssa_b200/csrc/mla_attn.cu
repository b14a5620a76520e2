// MLA indexed attention (one latent row per token serves as key and value).
#include "common.cuh"
#include "launch.h"

namespace jssa {

cudaError_t launch_mla_attention(const AttnArgs&, cudaStream_t) { return cudaErrorNotSupported; }

}  // namespace jssa
