// Per-(sequence, KV head) top-k selection over fp32 scores.
//
// "Joint Subspace Sparse Attention for Efficient Long-Context Decoding", Figure 1
// (top-B positions per KV head), §A.3 / §E.3 (independent selections per KV head
// and sequence), §E.1 (top-B selection dominates the step at small batch).
//
// Exact radix select on order-preserving 32-bit keys, one thread-block cluster per
// (sequence, KV head) row.  Each CTA of the cluster owns a contiguous slice of the
// row, staged once from L2 into shared memory.  Three histogram passes (12, 12 and
// 8 key bits) find the k-th largest key K*: each CTA histograms its slice, pushes
// the non-zero bins into rank 0's shared memory (distributed shared memory atomics),
// and rank 0 finds the digit and broadcasts it.  A last pass compacts, in index
// order, every key > K* plus the lowest-indexed keys == K* up to the quota, using
// warp ballots; per-CTA and per-warp counts give each output position, so the
// selection comes out sorted ascending.  Cluster barriers are hardware barriers
// over co-scheduled CTAs, so no wait here can hang.
#include <cooperative_groups.h>

#include "common.cuh"
#include "launch.h"

namespace cg = cooperative_groups;

namespace jssa {

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kBins = 4096;
constexpr int kMaxCluster = 8;

// Exclusive prefix sum over the block (every thread contributes v); returns the
// sum of the values of lower-numbered threads and writes the block total.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* warp_tmp, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, x, off);
    if (lane >= off) x += y;
  }
  if (lane == 31) warp_tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = (lane < kTopkWarps) ? warp_tmp[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, w, off);
      if (lane >= off) w += y;
    }
    if (lane < kTopkWarps) warp_tmp[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  const uint32_t warp_base = (warp > 0) ? warp_tmp[warp - 1] : 0;
  const uint32_t res = warp_base + x - v;
  if (total) *total = warp_tmp[kTopkWarps - 1];
  __syncthreads();
  return res;
}

template <bool STAGED>
__global__ void __launch_bounds__(kTopkThreads) topk_kernel(TopkArgs a, int per_cap) {
  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int crank = static_cast<int>(cluster.block_rank());
  extern __shared__ __align__(16) unsigned char smem_raw[];
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem_raw);  // [kBins] this CTA's histogram
  uint32_t* tot = hist + kBins;                             // [kBins] cluster total (rank 0)
  uint32_t* keys = tot + kBins;                             // [per_cap] staged keys
  __shared__ uint32_t bc_digit, bc_krem;                    // written by rank 0
  __shared__ uint32_t cta_gt[kMaxCluster], cta_eq[kMaxCluster];
  __shared__ uint32_t warp_gt[kTopkWarps], warp_eq[kTopkWarps];
  __shared__ uint32_t scan_tmp[32];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row = blockIdx.y;
  const int b = row / a.Hkv;
  int64_t T = a.seq_lens[b];
  if (T < 0 || T > a.T_cap) {
    if (crank == 0 && tid == 0) flag_error(a.status, DEVFLAG_BAD_SEQ_LEN);
    T = T < 0 ? 0 : a.T_cap;
  }
  const int64_t W = min64(max64(a.window, 0), T);
  const int64_t n = T - W;
  const int64_t k_eff = min64(a.k, n);
  int32_t* out = a.idx + static_cast<int64_t>(row) * a.k;
  if (crank == 0 && tid == 0) a.n_sel[row] = static_cast<int32_t>(k_eff);
  for (int64_t j = k_eff + crank * kTopkThreads + tid; j < a.k; j += static_cast<int64_t>(C) * kTopkThreads) out[j] = -1;
  if (k_eff == n) {  // everything is selected (includes n == 0)
    for (int64_t j = crank * kTopkThreads + tid; j < n; j += static_cast<int64_t>(C) * kTopkThreads)
      out[j] = static_cast<int32_t>(j);
    return;
  }

  // this CTA's slice [lo, lo + len)
  const int64_t per = ceil_div(n, C);
  const int64_t lo = crank * per;
  const int len = static_cast<int>(max64(0, min64(n, lo + per) - lo));
  const float* srow = a.scores + static_cast<int64_t>(row) * a.sc_ld + lo;
  if (STAGED) {
    for (int i = tid; i < len; i += kTopkThreads) keys[i] = float_to_ordered(__ldg(srow + i));
  }
  auto key_at = [&](int i) -> uint32_t { return STAGED ? keys[i] : float_to_ordered(__ldg(srow + i)); };

  uint32_t prefix = 0, mask = 0, krem = static_cast<uint32_t>(k_eff);
  for (int i = tid; i < kBins; i += kTopkThreads) tot[i] = 0;
  uint32_t* tot0 = cluster.map_shared_rank(tot, 0);
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = (pass == 0) ? 20 : (pass == 1) ? 8 : 0;
    const int nb = (pass == 2) ? 256 : kBins;
    for (int i = tid; i < nb; i += kTopkThreads) hist[i] = 0;
    if (pass == 0) cluster.sync();  // every CTA runs and rank 0's totals are zero
    else __syncthreads();
    for (int i = tid; i < len; i += kTopkThreads) {
      const uint32_t key = key_at(i);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & (nb - 1)], 1u);
    }
    __syncthreads();
    for (int i = tid; i < nb; i += kTopkThreads) {
      const uint32_t v = hist[i];
      if (v) atomicAdd(&tot0[i], v);
    }
    cluster.sync();
    if (crank == 0) {
      // digit D: the largest bin whose suffix count (bins >= D) reaches krem
      const int per_t = (nb + kTopkThreads - 1) / kTopkThreads;
      const int b0 = tid * per_t, b1 = min(nb, b0 + per_t);
      uint32_t s = 0;
      for (int i = b0; i < b1; ++i) s += tot[i];
      // count in the bins above this thread's range: total - inclusive prefix
      uint32_t total;
      const uint32_t below = block_exclusive_scan(s, scan_tmp, &total);
      const uint32_t above = total - below - s;
      if (b0 < b1 && above < krem && above + s >= krem) {
        uint32_t acc = above;
        for (int i = b1 - 1; i >= b0; --i) {
          if (acc + tot[i] >= krem) {
            for (int c = 0; c < C; ++c) {
              *cluster.map_shared_rank(&bc_digit, c) = static_cast<uint32_t>(i);
              *cluster.map_shared_rank(&bc_krem, c) = krem - acc;
            }
            break;
          }
          acc += tot[i];
        }
      }
      __syncthreads();
      for (int i = tid; i < nb; i += kTopkThreads) tot[i] = 0;
    }
    cluster.sync();
    prefix |= bc_digit << shift;
    mask |= static_cast<uint32_t>(nb - 1) << shift;
    krem = bc_krem;
  }
  const uint32_t kstar = prefix;  // the k-th largest key
  const uint32_t need = krem;     // keys equal to kstar to take, lowest index first

  // ---- ordered compaction: warp w owns [w*wc, min(len, (w+1)*wc))
  const int wc = static_cast<int>(ceil_div(ceil_div(len, kTopkWarps), 32) * 32);
  const int w_lo = warp * wc, w_hi = min(len, w_lo + wc);
  uint32_t ngt = 0, neq = 0;
  for (int base = w_lo; base < w_hi; base += 32) {
    const int i = base + lane;
    const uint32_t key = (i < w_hi) ? key_at(i) : 0u;
    ngt += __popc(__ballot_sync(0xFFFFFFFFu, i < w_hi && key > kstar));
    neq += __popc(__ballot_sync(0xFFFFFFFFu, i < w_hi && key == kstar));
  }
  if (lane == 0) { warp_gt[warp] = ngt; warp_eq[warp] = neq; }
  __syncthreads();
  if (tid < C) {
    uint32_t g = 0, e = 0;
    for (int w = 0; w < kTopkWarps; ++w) { g += warp_gt[w]; e += warp_eq[w]; }
    *cluster.map_shared_rank(&cta_gt[crank], tid) = g;
    *cluster.map_shared_rank(&cta_eq[crank], tid) = e;
  }
  cluster.sync();  // last access to another CTA's shared memory
  // output base of this CTA and its quota of equal keys
  uint32_t base_out = 0, eq_before = 0;
  for (int c = 0; c < crank; ++c) {
    const uint32_t q = (need > eq_before) ? min(cta_eq[c], need - eq_before) : 0u;
    base_out += cta_gt[c] + q;
    eq_before += cta_eq[c];
  }
  const uint32_t quota = (need > eq_before) ? min(cta_eq[crank], need - eq_before) : 0u;
  // this warp's base and its first equal-key rank inside the CTA
  uint32_t pos = base_out, eq_rank = 0;
  for (int w = 0; w < warp; ++w) {
    const uint32_t q = (quota > eq_rank) ? min(warp_eq[w], quota - eq_rank) : 0u;
    pos += warp_gt[w] + q;
    eq_rank += warp_eq[w];
  }
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int base = w_lo; base < w_hi; base += 32) {
    const int i = base + lane;
    const uint32_t key = (i < w_hi) ? key_at(i) : 0u;
    const bool gt = i < w_hi && key > kstar;
    const bool eq = i < w_hi && key == kstar;
    const uint32_t eq_m = __ballot_sync(0xFFFFFFFFu, eq);
    const bool sel = gt || (eq && (eq_rank + __popc(eq_m & lt_mask)) < quota);
    const uint32_t sel_m = __ballot_sync(0xFFFFFFFFu, sel);
    if (sel) {
      const uint32_t p = pos + __popc(sel_m & lt_mask);
      if (p < static_cast<uint32_t>(k_eff)) out[p] = static_cast<int32_t>(lo + i);
      else flag_error(a.status, DEVFLAG_BAD_INDEX);  // unreachable when the counts are consistent
    }
    pos += __popc(sel_m);
    eq_rank += __popc(eq_m);
  }
}

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t s) {
  const int64_t n_max = a.T_cap;
  int C = 1;
  while (C < kMaxCluster && ceil_div(n_max, C) > 16384) C *= 2;
  const int64_t per = ceil_div(n_max, C);
  const bool staged = per <= 40960;
  const int per_cap = staged ? static_cast<int>(per) : 0;
  const size_t smem = 2 * kBins * sizeof(uint32_t) + static_cast<size_t>(per_cap) * sizeof(uint32_t);
  void (*kern)(TopkArgs, int) = staged ? topk_kernel<true> : topk_kernel<false>;
  static int done_staged[64] = {0}, done_plain[64] = {0};
  cudaError_t e = set_smem_limit_once(kern, smem, staged ? done_staged : done_plain);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C, a.B * a.Hkv, 1);
  cfg.blockDim = dim3(kTopkThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, a, per_cap);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace jssa
