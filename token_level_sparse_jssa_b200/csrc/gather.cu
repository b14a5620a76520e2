// Gather-then-attend comparator: copy each (sequence, KV head) row's attended K/V rows (the
// selection, then the window) into a compact buffer, so that the dense flash-decode can run over
// it.  This is the gather-based baseline that "Joint Subspace Sparse Attention for Efficient
// Long-Context Decoding" compares its gather-free kernel against (§2.2, §3.3, §4.7): the copy
// costs about as much as the reduced attention itself.  It is not part of the method's path.
//
// Grid (position blocks of kGatherTile, rows); each CTA copies the K and V rows of its block of
// list positions with 16-byte loads and stores.  Invalid selected indices are flagged and their
// rows written as zeros.
#include "common.cuh"
#include "launch.h"

namespace jssa {
namespace {

constexpr int kGatherTile = 64;      // list positions per CTA
constexpr int kGatherThreads = 256;

__global__ void __launch_bounds__(kGatherThreads) gather_rows_kernel(GatherArgs a) {
  const int row = blockIdx.y;
  const int b = row / a.Hkv, h = row % a.Hkv;
  int64_t T = a.seq_lens[b];
  if (T < 0 || T > a.T_cap) {
    if (blockIdx.x == 0 && threadIdx.x == 0) flag_error(a.status, DEVFLAG_BAD_SEQ_LEN);
    T = T < 0 ? 0 : a.T_cap;
  }
  const int64_t Wc = min64(max64(a.window, 0), T);
  const int64_t win_start = T - Wc;
  int64_t nsel = a.n_sel[row];
  const int64_t nsel_max = min64(a.idx_ld, win_start);
  if (nsel < 0 || nsel > nsel_max) {
    if (blockIdx.x == 0 && threadIdx.x == 0) flag_error(a.status, DEVFLAG_BAD_NSEL);
    nsel = nsel < 0 ? 0 : nsel_max;
  }
  const int64_t list_len = nsel + Wc;
  if (blockIdx.x == 0 && threadIdx.x == 0) a.glen[row] = static_cast<int32_t>(list_len);
  const int64_t p0 = static_cast<int64_t>(blockIdx.x) * kGatherTile;
  if (p0 >= list_len) return;
  const int cpr = a.d / 8;  // 16-byte chunks per row
  const uint4* Kb = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.K) + b * a.ks[0] + h * a.ks[1]);
  const uint4* Vb = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.V) + b * a.vs[0] + h * a.vs[1]);
  uint4* Kg = reinterpret_cast<uint4*>(a.Kg) + static_cast<int64_t>(row) * a.Lmax * cpr;
  uint4* Vg = reinterpret_cast<uint4*>(a.Vg) + static_cast<int64_t>(row) * a.Lmax * cpr;
  const int64_t ks2 = a.ks[2] / 8, vs2 = a.vs[2] / 8;  // row strides in 16-byte chunks
  const int n_items = kGatherTile * cpr;
  for (int it = threadIdx.x; it < n_items; it += kGatherThreads) {
    const int jp = it / cpr, ch = it % cpr;
    const int64_t p = p0 + jp;
    if (p >= list_len) break;  // items are in position order
    int64_t t;
    if (p < nsel) {
      t = a.idx[static_cast<int64_t>(row) * a.idx_ld + p];
      if (t < 0 || t >= win_start) {
        if (ch == 0) flag_error(a.status, DEVFLAG_BAD_INDEX);
        t = -1;
      }
    } else {
      t = win_start + (p - nsel);
    }
    const uint4 z = make_uint4(0u, 0u, 0u, 0u);
    Kg[p * cpr + ch] = (t >= 0) ? __ldg(Kb + t * ks2 + ch) : z;
    Vg[p * cpr + ch] = (t >= 0) ? __ldg(Vb + t * vs2 + ch) : z;
  }
}

}  // namespace

cudaError_t launch_gather_rows(const GatherArgs& a, cudaStream_t s) {
  if (a.d % 8 != 0 || a.Lmax < 1) return cudaErrorInvalidValue;
  const dim3 grid(static_cast<unsigned>(ceil_div(a.Lmax, kGatherTile)), static_cast<unsigned>(a.B * a.Hkv));
  gather_rows_kernel<<<grid, kGatherThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace jssa
