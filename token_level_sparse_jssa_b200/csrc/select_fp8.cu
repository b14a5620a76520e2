// Fused selection of the decode step over an FP8 E4M3 projected-key cache: the E4M3
// instantiations of the kernel in select_kernel.cuh ("Joint Subspace Sparse Attention for
// Efficient Long-Context Decoding", §A.3 and §E.2: the deployed scoring cache is FP8, which
// halves the bytes of the scan; the final attention stays on the bf16 K/V rows).
#include "select_kernel.cuh"

namespace jssa {

cudaError_t launch_select_fp8(const SelectArgs& a, int num_sms, cudaStream_t s) {
  switch (a.r) {  // rows of at least 16 bytes
    case 16: return launch_select_rd<16, true>(a, num_sms, s);
    case 32: return launch_select_rd<32, true>(a, num_sms, s);
    case 64: return launch_select_rd<64, true>(a, num_sms, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace jssa
