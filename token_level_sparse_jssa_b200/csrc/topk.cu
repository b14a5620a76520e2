// Per-(sequence, KV head) top-k selection over fp32 scores.
//
// "Joint Subspace Sparse Attention for Efficient Long-Context Decoding", Figure 1
// (top-B positions per KV head), §A.3 / §E.3 (independent selections per KV head
// and sequence), §E.1 (top-B selection dominates the step at small batch).
//
// Exact radix select on order-preserving 32-bit keys (larger score -> larger key,
// -0 == +0), one thread-block cluster per (sequence, KV head) row; ties go to the
// lower token index and the selection is written in ascending index order.
//
//   digit 1 (key bits 31..20): from the row's histogram, which the score scan builds
//           as it streams the projected cache (or topk_hist_kernel for standalone
//           calls); each CTA stages it with its slice and finds the digit itself.
//   scan 1 (the only pass over the whole slice): each warp lists, in index order, its
//           keys above bin D1 ("definites", all selected) and inside bin D1
//           ("candidates", about 1 % of the keys for the workloads here).
//   digits 2 and 3 (bits 19..10, 9..0): the candidate keys of the whole row are
//           gathered into rank 0's shared memory (distributed shared memory stores);
//           after one cluster barrier every CTA copies them and finds both digits
//           locally.  If the candidates do not fit, the cluster instead resolves each
//           digit with a histogram summed in rank 0 (atomics) and read back by all.
//   output: every key > K* plus, in index order, the first `need` keys == K*.  Per-warp
//           and per-CTA counts exchanged across the cluster give each warp its output
//           position; a warp marks its selected offsets in a bitmap and emits them in
//           order (or, with overflowing lists, rescans its range with ballots).
//
// Each CTA's slice of scores is staged once into shared memory with one bulk copy
// (TMA engine).  Three cluster barriers (five when the gather overflows); cluster barriers are hardware
// barriers over co-scheduled CTAs, so no wait here can hang; the bulk-copy wait is
// bounded in time.
#include <cooperative_groups.h>

#include <mutex>

#include "common.cuh"
#include "launch.h"

namespace cg = cooperative_groups;

namespace jssa {

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kBins1 = 4096;   // digit 1: key bits [31:20]
constexpr int kBins2 = 1024;   // digits 2 and 3: bits [19:10] and [9:0]
constexpr int kMaxCluster = 8;
constexpr int kSliceTarget = 16384;   // keys per CTA the cluster size aims for
constexpr int kMaxStaged = 32768;     // keys per CTA that still fit in shared memory
constexpr int kCapW = 64;             // per-warp capacity of the definite and candidate lists
constexpr int kMaskWords = 64;        // per-warp output bitmap: ranges of up to 2048 keys
constexpr uint32_t kGather = 3072;    // candidate keys of a row gathered into rank 0

// Exclusive prefix sum over the block; returns the sum over lower-numbered threads and
// writes the block total.
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
  *total = warp_tmp[kTopkWarps - 1];
  __syncthreads();
  return warp_base + x - v;
}

// Given a histogram (any address space, generic pointer) and the number of keys still
// to select, find the digit D whose suffix count (bins >= D) first reaches krem.  Writes
// D and the count still to take inside bin D to *digit / *krem_out (shared memory).
template <int NB>
__device__ __forceinline__ void find_digit(const uint32_t* hist, uint32_t krem, uint32_t* scan_tmp,
                                           uint32_t* digit, uint32_t* krem_out) {
  constexpr int PER = (NB + kTopkThreads - 1) / kTopkThreads;
  const int b0 = threadIdx.x * PER;
  uint32_t c[PER];
  uint32_t s = 0;
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    c[q] = (b0 + q < NB) ? hist[b0 + q] : 0u;
    s += c[q];
  }
  uint32_t total;
  const uint32_t below = block_exclusive_scan(s, scan_tmp, &total);
  const uint32_t above = total - below - s;  // keys in the bins above this thread's group
  if (b0 < NB && above < krem && above + s >= krem) {
    uint32_t acc = above;
#pragma unroll
    for (int q = PER - 1; q >= 0; --q) {
      if (acc + c[q] >= krem) {
        *digit = static_cast<uint32_t>(b0 + q);
        *krem_out = krem - acc;
        break;
      }
      acc += c[q];
    }
  }
  __syncthreads();
}

template <bool STAGED>
__global__ void __launch_bounds__(kTopkThreads) topk_kernel(TopkArgs a, int per_cap) {
  cg::cluster_group cluster = cg::this_cluster();
  const int C = static_cast<int>(cluster.num_blocks());
  const int crank = static_cast<int>(cluster.block_rank());
  extern __shared__ __align__(128) unsigned char smem_raw[];
  float* fs = reinterpret_cast<float*>(smem_raw);                      // [per_cap] staged scores
  uint32_t* h1s = reinterpret_cast<uint32_t*>(fs + per_cap);           // [kBins1] the row's digit-1 histogram
  uint32_t* gbuf = h1s + kBins1;                                        // [kGather] candidate keys of the row
  uint32_t* hloc = gbuf + kGather;                                      // [kBins2] local histogram / bitmaps
  uint32_t* defs = hloc + kBins2;                                       // [warps][kCapW] keys above bin D1
  uint32_t* cands = defs + kTopkWarps * kCapW;                          // [warps][kCapW] keys inside bin D1
  uint32_t* totA = gbuf;                                                // fallback totals (rank 0) alias gbuf
  uint32_t* totB = gbuf + kBins2;
  uint32_t* masks = hloc;                                               // output bitmaps alias hloc
  __shared__ uint64_t bar;
  __shared__ uint32_t dig, krem_s, gcnt, gbase;
  __shared__ uint32_t cta_gt[kMaxCluster], cta_eq[kMaxCluster], cta_ab[kMaxCluster];
  __shared__ uint32_t warp_gt[kTopkWarps], warp_eq[kTopkWarps], warp_nc[kTopkWarps];
  __shared__ uint32_t scan_tmp[32];

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row = blockIdx.y;
  const int b = row / a.Hkv;
  const WaitTest wt = wait_test_read(a.status, row == 0 && crank == 0);
  if (tid == 0) {
    gcnt = 0;
    mbar_init(&bar, 1);
    fence_mbarrier_init();
  }
  int64_t T = a.seq_lens[b];
  if (T < 0 || T > a.T_cap) {
    if (crank == 0 && tid == 0) flag_error(a.status, DEVFLAG_BAD_SEQ_LEN);
    T = T < 0 ? 0 : a.T_cap;
  }
  const int64_t W = min64(max64(a.window, 0), T);
  const int n = static_cast<int>(T - W);
  const int k_eff = static_cast<int>(min64(a.k, n));
  int32_t* out = a.idx + static_cast<int64_t>(row) * a.k;
  if (crank == 0 && tid == 0) a.n_sel[row] = k_eff;
  for (int j = k_eff + crank * kTopkThreads + tid; j < a.k; j += C * kTopkThreads) out[j] = -1;
  uint32_t* hrow_w = a.hist + static_cast<int64_t>(row) * kBins1;
  if (k_eff == n) {  // everything is selected (includes n == 0)
    for (int j = crank * kTopkThreads + tid; j < n; j += C * kTopkThreads) out[j] = j;
    if (crank == 0)  // leave the row's histogram zeroed for the next scan
      for (int i = tid; i < kBins1; i += kTopkThreads) hrow_w[i] = 0u;
    return;
  }

  // this CTA's slice [lo, lo + len); warp w owns slice offsets [w * wc, min(len, (w + 1) * wc))
  const int per = (((n + C - 1) / C) + 3) & ~3;
  const int lo = crank * per;
  const int len = max(0, min(n, lo + per) - lo);
  const int wc = ((len + kTopkWarps - 1) / kTopkWarps + 31) & ~31;
  const float* srow = a.scores + static_cast<int64_t>(row) * a.sc_ld + lo;
  const uint32_t* hrow = a.hist + static_cast<int64_t>(row) * kBins1;
  __syncthreads();
  const bool bulk = STAGED && (reinterpret_cast<uintptr_t>(srow) & 15u) == 0;
  const int nbulk = bulk ? (len & ~3) : 0;
  if (wt.withhold && tid == 0) wait_test_disarm(a.status);  // every thread has read it
  if (tid == 0 && !wt.withhold) {  // the slice (when staged) and the row's digit-1 histogram, in one transaction
    const uint64_t pol = l2_policy_evict_first();
    mbar_arrive_expect_tx(&bar, static_cast<uint32_t>(nbulk) * 4u + kBins1 * 4u);
    if (nbulk > 0) bulk_g2s(fs, srow, static_cast<uint32_t>(nbulk) * 4u, &bar, pol);
    bulk_g2s(h1s, hrow, kBins1 * 4u, &bar, pol);
  }
  if (STAGED)
    for (int i = nbulk + tid; i < len; i += kTopkThreads) fs[i] = __ldg(srow + i);
  auto key_at = [&](int i) -> uint32_t { return float_to_ordered(STAGED ? fs[i] : __ldg(srow + i)); };
  cluster.sync();  // S0: every CTA runs and rank 0's gather count is zero (overlaps the copies)
  const bool staged_ok = mbar_wait_bounded(&bar, 0, a.status, wt.limit_ns);
  const bool aborted = __syncthreads_or(!staged_ok);

  // digit 1 from the row's histogram (every CTA computes the same digit)
  find_digit<kBins1>(h1s, static_cast<uint32_t>(k_eff), scan_tmp, &dig, &krem_s);
  const uint32_t d1 = dig;
  const uint32_t k1 = krem_s;

  // scan 1, the only pass over the whole slice: each warp lists, in index order, its
  // keys above bin d1 ("definites", all selected) and inside bin d1 ("candidates")
  const int w_lo = warp * wc, w_hi = aborted ? w_lo : min(len, w_lo + wc);
  const uint32_t lt_mask = (1u << lane) - 1u;
  uint32_t* my_defs = defs + warp * kCapW;
  uint32_t* my_cands = cands + warp * kCapW;
  uint32_t nd = 0, nca = 0;
  constexpr int U = 4;  // 32-key groups per step: independent loads and ballots, in index order
  for (int base = w_lo; base < w_hi; base += 32 * U) {
    uint32_t dk[U], mdef[U], mcan[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int i = base + u * 32 + lane;
      dk[u] = (i < w_hi) ? (key_at(i) >> 20) : 0u;
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const bool valid = base + u * 32 + lane < w_hi;
      mdef[u] = __ballot_sync(0xFFFFFFFFu, valid && dk[u] > d1);
      mcan[u] = __ballot_sync(0xFFFFFFFFu, valid && dk[u] == d1);
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const uint32_t i = static_cast<uint32_t>(base + u * 32 + lane);
      if ((mdef[u] >> lane) & 1u) {
        const uint32_t p = nd + __popc(mdef[u] & lt_mask);
        if (p < kCapW) my_defs[p] = i;
      }
      if ((mcan[u] >> lane) & 1u) {
        const uint32_t p = nca + __popc(mcan[u] & lt_mask);
        if (p < kCapW) my_cands[p] = i;
      }
      nd += __popc(mdef[u]);
      nca += __popc(mcan[u]);
    }
  }
  const bool cand_list = nca <= kCapW;   // warp-uniform: else this warp rescans its range
  if (lane == 0) warp_nc[warp] = cand_list ? nca : (kGather + 1u);
  __syncthreads();

  // gather the keys of bin d1 from the whole row into rank 0 (distributed shared memory)
  uint32_t* gcnt0 = cluster.map_shared_rank(&gcnt, 0);
  uint32_t* gbuf0 = cluster.map_shared_rank(gbuf, 0);
  if (tid == 0) {
    uint32_t tot = 0;
    for (int w = 0; w < kTopkWarps; ++w) tot += warp_nc[w];
    tot = min(tot, kGather + 1u);
    gbase = (tot > 0) ? atomicAdd(gcnt0, tot) : 0u;
  }
  __syncthreads();
  {
    uint32_t off = gbase;
    for (int w = 0; w < warp; ++w) off += warp_nc[w];
    if (cand_list && off + nca <= kGather)
      for (int j = lane; j < static_cast<int>(nca); j += 32) gbuf0[off + j] = key_at(static_cast<int>(my_cands[j]));
  }
  cluster.sync();  // S1: the row's candidate keys (or an overflowed count) are in rank 0
  const uint32_t gtotal = *gcnt0;
  if (crank == 0)  // every CTA has staged the row's histogram: leave it zeroed for the next scan
    for (int i = tid; i < kBins1; i += kTopkThreads) hrow_w[i] = 0u;
  uint32_t prefix = d1 << 20, mask = 0xFFF00000u, krem = k1;
  if (gtotal <= kGather) {
    // exact selection among the gathered keys, locally in every CTA: digits 2 and 3
    if (crank != 0)
      for (int j = tid; j < static_cast<int>(gtotal); j += kTopkThreads) gbuf[j] = gbuf0[j];
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
      const int shift = (pass == 0) ? 10 : 0;
      for (int i = tid; i < kBins2; i += kTopkThreads) hloc[i] = 0;
      __syncthreads();
      for (int j = tid; j < static_cast<int>(gtotal); j += kTopkThreads) {
        const uint32_t key = gbuf[j];
        if ((key & mask) == prefix) atomicAdd(&hloc[(key >> shift) & (kBins2 - 1)], 1u);
      }
      __syncthreads();
      find_digit<kBins2>(hloc, krem, scan_tmp, &dig, &krem_s);
      prefix |= dig << shift;
      mask |= static_cast<uint32_t>(kBins2 - 1) << shift;
      krem = krem_s;
    }
  } else {
    // too many candidates for the gather buffer: resolve digits 2 and 3 with cluster-wide
    // histograms in rank 0 (every CTA takes this branch: gtotal is the same everywhere)
    uint32_t* totA0 = cluster.map_shared_rank(totA, 0);
    uint32_t* totB0 = cluster.map_shared_rank(totB, 0);
    if (crank == 0)
      for (int i = tid; i < kBins2; i += kTopkThreads) { totA[i] = 0; totB[i] = 0; }
    cluster.sync();
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
      const int shift = (pass == 0) ? 10 : 0;
      uint32_t* tot0 = (pass == 0) ? totA0 : totB0;
      for (int i = tid; i < kBins2; i += kTopkThreads) hloc[i] = 0;
      __syncthreads();
      if (cand_list) {
        for (int j = lane; j < static_cast<int>(nca); j += 32) {
          const uint32_t key = key_at(static_cast<int>(my_cands[j]));
          if ((key & mask) == prefix) atomicAdd(&hloc[(key >> shift) & (kBins2 - 1)], 1u);
        }
      } else {
        for (int i = w_lo + lane; i < w_hi; i += 32) {
          const uint32_t key = key_at(i);
          if ((key & mask) == prefix) atomicAdd(&hloc[(key >> shift) & (kBins2 - 1)], 1u);
        }
      }
      __syncthreads();
      for (int i = tid; i < kBins2; i += kTopkThreads) {
        const uint32_t v = hloc[i];
        if (v) atomicAdd(&tot0[i], v);
      }
      cluster.sync();
      find_digit<kBins2>(tot0, krem, scan_tmp, &dig, &krem_s);
      prefix |= dig << shift;
      mask |= static_cast<uint32_t>(kBins2 - 1) << shift;
      krem = krem_s;
    }
  }
  const uint32_t kstar = prefix;  // the k-th largest key
  const uint32_t need = krem;     // keys equal to kstar to take, lowest index first

  // per-warp counts of keys > kstar (all definites + candidates above) and == kstar
  {
    uint32_t ngt = nd, neq = 0;
    if (cand_list) {
      for (int j0 = 0; j0 < static_cast<int>(nca); j0 += 32) {
        const int j = j0 + lane;
        const uint32_t key = (j < static_cast<int>(nca)) ? key_at(static_cast<int>(my_cands[j])) : 0u;
        ngt += __popc(__ballot_sync(0xFFFFFFFFu, j < static_cast<int>(nca) && key > kstar));
        neq += __popc(__ballot_sync(0xFFFFFFFFu, j < static_cast<int>(nca) && key == kstar));
      }
    } else {
      for (int base = w_lo; base < w_hi; base += 32) {
        const int i = base + lane;
        const uint32_t key = (i < w_hi) ? key_at(i) : 0u;
        ngt += __popc(__ballot_sync(0xFFFFFFFFu, i < w_hi && key > kstar && (key >> 20) == d1));
        neq += __popc(__ballot_sync(0xFFFFFFFFu, i < w_hi && key == kstar));
      }
    }
    if (lane == 0) { warp_gt[warp] = ngt; warp_eq[warp] = neq; }
  }
  __syncthreads();
  if (tid < C) {
    uint32_t g = 0, e = 0;
    for (int w = 0; w < kTopkWarps; ++w) { g += warp_gt[w]; e += warp_eq[w]; }
    *cluster.map_shared_rank(&cta_gt[crank], tid) = g;
    *cluster.map_shared_rank(&cta_eq[crank], tid) = e;
    *cluster.map_shared_rank(&cta_ab[crank], tid) = aborted ? 1u : 0u;
  }
  cluster.sync();  // S2: last access to another CTA's shared memory
  bool any_aborted = false;
  for (int c = 0; c < C; ++c) any_aborted |= (cta_ab[c] != 0u);
  if (any_aborted) {  // a staging copy of the row never completed (flagged): the selection is empty
    for (int j = crank * kTopkThreads + tid; j < k_eff; j += C * kTopkThreads) out[j] = -1;
    if (crank == 0 && tid == 0) a.n_sel[row] = 0;
    if (aborted && tid == 0) mbar_wait_bounded(&bar, 0, nullptr, wt.limit_ns);  // a late copy lands before exit
    return;
  }
  // output base and quota of keys == kstar: of this CTA, then of this warp
  uint32_t base_out = 0, eq_before = 0;
  for (int c = 0; c < crank; ++c) {
    const uint32_t q = (need > eq_before) ? min(cta_eq[c], need - eq_before) : 0u;
    base_out += cta_gt[c] + q;
    eq_before += cta_eq[c];
  }
  const uint32_t quota = (need > eq_before) ? min(cta_eq[crank], need - eq_before) : 0u;
  uint32_t pos = base_out, eq_rank = 0;
  for (int w = 0; w < warp; ++w) {
    const uint32_t q = (quota > eq_rank) ? min(warp_eq[w], quota - eq_rank) : 0u;
    pos += warp_gt[w] + q;
    eq_rank += warp_eq[w];
  }
  const uint32_t wquota = (quota > eq_rank) ? min(warp_eq[warp], quota - eq_rank) : 0u;
  const int words = wc / 32;
  if (cand_list && nd <= kCapW && words <= kMaskWords) {
    // mark the selected offsets of this warp's range in a bitmap, then emit them in order
    uint32_t* m = masks + warp * kMaskWords;
    for (int j = lane; j < words; j += 32) m[j] = 0u;
    __syncwarp();
    for (int j = lane; j < static_cast<int>(nd); j += 32) {
      const uint32_t o = my_defs[j] - static_cast<uint32_t>(w_lo);
      atomicOr(&m[o >> 5], 1u << (o & 31));
    }
    uint32_t eq_run = 0;
    for (int j0 = 0; j0 < static_cast<int>(nca); j0 += 32) {
      const int j = j0 + lane;
      const uint32_t i = (j < static_cast<int>(nca)) ? my_cands[j] : 0u;
      const uint32_t key = (j < static_cast<int>(nca)) ? key_at(static_cast<int>(i)) : 0u;
      const bool gt = j < static_cast<int>(nca) && key > kstar;
      const bool eq = j < static_cast<int>(nca) && key == kstar;
      const uint32_t eq_m = __ballot_sync(0xFFFFFFFFu, eq);
      if (gt || (eq && (eq_run + __popc(eq_m & lt_mask)) < wquota)) {
        const uint32_t o = i - static_cast<uint32_t>(w_lo);
        atomicOr(&m[o >> 5], 1u << (o & 31));
      }
      eq_run += __popc(eq_m);
    }
    __syncwarp();
    const uint32_t w0 = (lane < words) ? m[lane] : 0u;
    const uint32_t w1 = (lane + 32 < words) ? m[lane + 32] : 0u;
    const uint32_t c0 = __popc(w0), c1 = __popc(w1);
    uint32_t x0 = c0, x1 = c1;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t y0 = __shfl_up_sync(0xFFFFFFFFu, x0, off);
      const uint32_t y1 = __shfl_up_sync(0xFFFFFFFFu, x1, off);
      if (lane >= off) { x0 += y0; x1 += y1; }
    }
    const uint32_t tot0 = __shfl_sync(0xFFFFFFFFu, x0, 31);
    uint32_t p0 = pos + x0 - c0, p1 = pos + tot0 + x1 - c1;
    const int gb = lo + w_lo;
    for (uint32_t v = w0; v; v &= v - 1) {
      if (p0 < static_cast<uint32_t>(k_eff)) out[p0] = gb + lane * 32 + (__ffs(v) - 1);
      else flag_error(a.status, DEVFLAG_BAD_INDEX);  // unreachable when the counts are consistent
      ++p0;
    }
    for (uint32_t v = w1; v; v &= v - 1) {
      if (p1 < static_cast<uint32_t>(k_eff)) out[p1] = gb + (lane + 32) * 32 + (__ffs(v) - 1);
      else flag_error(a.status, DEVFLAG_BAD_INDEX);
      ++p1;
    }
  } else {
    // long lists: rescan this warp's range and compact with ballots
    uint32_t eq_run = 0;
    for (int base = w_lo; base < w_hi; base += 32) {
      const int i = base + lane;
      const uint32_t key = (i < w_hi) ? key_at(i) : 0u;
      const bool gt = i < w_hi && key > kstar;
      const bool eq = i < w_hi && key == kstar;
      const uint32_t eq_m = __ballot_sync(0xFFFFFFFFu, eq);
      const bool sel = gt || (eq && (eq_run + __popc(eq_m & lt_mask)) < wquota);
      const uint32_t sel_m = __ballot_sync(0xFFFFFFFFu, sel);
      if (sel) {
        const uint32_t p = pos + __popc(sel_m & lt_mask);
        if (p < static_cast<uint32_t>(k_eff)) out[p] = lo + i;
        else flag_error(a.status, DEVFLAG_BAD_INDEX);
      }
      pos += __popc(sel_m);
      eq_run += __popc(eq_m);
    }
  }
}

// Standalone path: histogram of key bits [31:20] per row, 8192 scores per CTA.
constexpr int kHistChunk = 8192;
__global__ void __launch_bounds__(256) topk_hist_kernel(TopkArgs a) {
  __shared__ uint32_t h[kBins1];
  const int row = blockIdx.y;
  const int b = row / a.Hkv;
  int64_t T = a.seq_lens[b];
  T = T < 0 ? 0 : (T > a.T_cap ? a.T_cap : T);
  const int64_t n = T - min64(max64(a.window, 0), T);
  const int64_t lo = static_cast<int64_t>(blockIdx.x) * kHistChunk;
  if (lo >= n) return;
  const int64_t hi = min64(n, lo + kHistChunk);
  for (int i = threadIdx.x; i < kBins1; i += blockDim.x) h[i] = 0;
  __syncthreads();
  const float* srow = a.scores + static_cast<int64_t>(row) * a.sc_ld;
  for (int64_t t = lo + threadIdx.x; t < hi; t += blockDim.x)
    atomicAdd(&h[float_to_ordered(__ldg(srow + t)) >> 20], 1u);
  __syncthreads();
  uint32_t* g = a.hist + static_cast<int64_t>(row) * kBins1;
  for (int i = threadIdx.x; i < kBins1; i += blockDim.x)
    if (h[i]) atomicAdd(g + i, h[i]);
}

// ------------------------------------------------------------------ allocation-free variant
// Scratch of jssa_topk_noalloc: the first-digit histograms (4096 counters, 16 KB) of up to
// kNoAllocMaxRows (sequence, KV head) rows, in a file-scope device array: 4 MB that every
// GPU which loads the library keeps until the process exits.  All calls share it.
constexpr int kNoAllocMaxRows = 256;
static __device__ __align__(256) uint32_t g_noalloc_hist[kNoAllocMaxRows * kBins1];

int topk_noalloc_max_rows() { return kNoAllocMaxRows; }

// Device address of g_noalloc_hist on the current device.  Host code cannot use the
// array's name as a pointer (it denotes a host-side stand-in), so the address is looked
// up with cudaGetSymbolAddress once per device, with that device current, and cached.
cudaError_t topk_noalloc_scratch(uint32_t** out) {
  static std::mutex mu;
  static uint32_t* ptrs[64] = {nullptr};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (ptrs[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_hist);
    if (e != cudaSuccess) return e;
    ptrs[dev] = static_cast<uint32_t*>(p);
  }
  *out = ptrs[dev];
  return cudaSuccess;
}

cudaError_t launch_topk_histogram(const TopkArgs& a, int, cudaStream_t s) {
  dim3 grid(static_cast<unsigned>(ceil_div(a.T_cap, kHistChunk)), a.B * a.Hkv);
  topk_hist_kernel<<<grid, 256, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_topk(const TopkArgs& a, cudaStream_t s) {
  const int64_t n_max = a.T_cap;
  int C = 1;
  while (C < kMaxCluster && ceil_div(n_max, C) > kSliceTarget) C *= 2;
  const int64_t per = ceil_div(ceil_div(n_max, C), 4) * 4;
  const bool staged = per <= kMaxStaged;
  void (*kern)(TopkArgs, int) = staged ? topk_kernel<true> : topk_kernel<false>;
  const int per_cap = staged ? static_cast<int>(per) : 0;
  static_assert(kTopkWarps * kMaskWords <= kBins2 && 2 * kBins2 <= kGather, "aliased shared-memory regions");
  const size_t smem = static_cast<size_t>(per_cap) * sizeof(float) +
                      (kBins1 + kGather + kBins2 + 2 * kTopkWarps * kCapW) * sizeof(uint32_t);
  static int done_staged[64] = {0}, done_plain[64] = {0};
  cudaError_t e = set_smem_limit_once(kern, smem, staged ? done_staged : done_plain);
  if (e != cudaSuccess) return e;
  return launch_ex(kern, dim3(C, a.B * a.Hkv, 1), dim3(kTopkThreads), smem, s, C, a, per_cap);
}

}  // namespace jssa
