// Fused selection of the decode step: the bf16-Kp instantiations of the kernel in
// select_kernel.cuh and the dispatch over the Kp storage type; the E4M3-Kp
// instantiations are built in select_fp8.cu.
#include "select_kernel.cuh"

namespace jssa {

int64_t select_max_candidates() { return 8 * static_cast<int64_t>(kSelMaxSlice); }
int select_max_new_rows() { return kSelMaxNew; }

cudaError_t launch_select(const SelectArgs& a, int num_sms, cudaStream_t s) {
  if (a.T_cap > select_max_candidates() || a.n_new > kSelMaxNew || a.n_new < 0) return cudaErrorInvalidValue;
  if (a.d % 8 != 0 || a.d / 8 > 8 * (kSelMaxDn / 8)) return cudaErrorInvalidValue;
  if (a.kp_fp8) return launch_select_fp8(a, num_sms, s);
  switch (a.r) {
    case 8: return launch_select_rd<8, false>(a, num_sms, s);
    case 16: return launch_select_rd<16, false>(a, num_sms, s);
    case 32: return launch_select_rd<32, false>(a, num_sms, s);
    case 64: return launch_select_rd<64, false>(a, num_sms, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace jssa
