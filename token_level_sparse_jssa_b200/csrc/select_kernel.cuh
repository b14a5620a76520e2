// The fused selection kernel of the decode step (template over the projected rank, the
// attention head dimension, the query-head tiles and the Kp storage type) and its launcher.
// Included by select.cu (bf16 Kp) and select_fp8.cu (E4M3 Kp), one instantiation set each.
//
// Fused selection of the decode step: query projection, projection of the newest keys,
// score scan and top-k, in one kernel with one thread-block cluster per (sequence, KV head).
//
// "Joint Subspace Sparse Attention for Efficient Long-Context Decoding", Figure 1 and
// §3.1-§3.2: the group query is projected with the head's orthonormal basis (qs = sum_g
// P^T q_g), every candidate position of the projected-key cache is scored (fp32 dot
// product with qs) and the top-k positions are selected per (sequence, KV head), ties to
// the lower index, output ascending; §3.2 (keys projected on write): the newest key rows
// are projected into the scoring cache inside the same step.
//
// The cluster's C CTAs (2 to 16, chosen at launch) split the row's candidates into
// contiguous slices of at most `per` tokens.  Each CTA streams its slice of Kp through a
// ring of 16 KB stages (one producer warp, 1-D bulk copies, full/empty mbarriers; eight
// consumer warps), keeps the order-preserving score keys of its slice in shared memory and
// counts the top 12 key bits in a packed 16-bit histogram.  The row's histogram is then
// assembled in distributed shared memory (each CTA owns an even-sized share of the 4096
// bins); each CTA finds the first radix digit, lists its keys above and inside that bin,
// gathers the row's in-bin keys into rank 0, resolves digits 2 and 3 locally and writes its
// selected positions in order.  Neither the scores nor the histogram leave the chip.
#pragma once

#include <cooperative_groups.h>

#include <map>
#include <mutex>
#include <tuple>

#include "attn_core.cuh"
#include "common.cuh"
#include "launch.h"

namespace jssa {
namespace {

constexpr int kSelConsumers = 256;                 // 8 consumer warps
constexpr int kSelThreads = kSelConsumers + 32;    // + 1 producer warp
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kSelStage = 16384;                   // bytes per ring stage
constexpr int kSelMaxCluster = 16;                 // up to 8 (portable) or 16 CTAs per row
constexpr int kSelMinCluster = 2;                  // fewer than 8 only to keep every row in one wave
constexpr int kSelMinSlice = 512;                  // or when slices would be shorter than this (latency-bound rows)
constexpr int kSelBins1 = 4096;                    // digit 1: key bits [31:20]
constexpr int kSelBins2 = 1024;                    // digits 2 and 3: bits [19:10] and [9:0]
constexpr int kSelCapW = 64;                       // per-warp capacity of the definite / candidate lists
constexpr int kSelMaskWords = 64;                  // per-warp bitmaps: ranges of up to 2048 keys
static_assert(((16384 + 8) / 9 + 31) / 32 <= 64, "a slice's warp ranges fit the bitmaps");
constexpr uint32_t kSelGather = 2048;              // in-bin keys of a row gathered into rank 0
constexpr int kSelMaxNew = 16;                     // newest rows projected inside the kernel
constexpr int kSelMaxR = 64;
constexpr int kSelKeysMin = 16384;                 // the keys area also holds the projection scratch
constexpr int kSelMaxDn = 72;                      // dims per CTA of the split projections (576 / 8)

// Words of the owned-bins area: the CTA's share of the row's first-digit histogram (an even
// number of bins), later its share of the attended token list; at least 512 words, so that
// clusters of 8 or more CTAs share one layout.
__host__ __device__ constexpr int sel_own_bins(int C) { return (((kSelBins1 + C - 1) / C) + 1) & ~1; }
__host__ __device__ constexpr int sel_own_words(int C) {
  return sel_own_bins(C) > kSelBins1 / 8 ? sel_own_bins(C) : kSelBins1 / 8;
}

__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kSelConsumers) : "memory"); }

__device__ __forceinline__ void mbar_arrive_one(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }

// Exclusive prefix sum over the block; returns the sum over lower-numbered threads and
// writes the block total.
__device__ __forceinline__ uint32_t sel_block_scan(uint32_t v, uint32_t* warp_tmp, uint32_t* total) {
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
    uint32_t w = (lane < kSelWarps) ? warp_tmp[lane] : 0;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, w, off);
      if (lane >= off) w += y;
    }
    if (lane < kSelWarps) warp_tmp[lane] = w;  // inclusive over warps
  }
  __syncthreads();
  const uint32_t warp_base = (warp > 0) ? warp_tmp[warp - 1] : 0;
  *total = warp_tmp[kSelWarps - 1];
  __syncthreads();
  return warp_base + x - v;
}

// The digit D whose suffix count (bins >= D) first reaches krem, and the count still to
// take inside bin D, written to *digit / *krem_out (shared memory).
template <int NB>
__device__ __forceinline__ void sel_find_digit(const uint32_t* hist, uint32_t krem, uint32_t* scan_tmp,
                                               uint32_t* digit, uint32_t* krem_out) {
  constexpr int PER = (NB + kSelThreads - 1) / kSelThreads;
  const int b0 = threadIdx.x * PER;
  uint32_t c[PER];
  uint32_t s = 0;
#pragma unroll
  for (int q = 0; q < PER; ++q) {
    c[q] = (b0 + q < NB) ? hist[b0 + q] : 0u;
    s += c[q];
  }
  uint32_t total;
  const uint32_t below = sel_block_scan(s, scan_tmp, &total);
  const uint32_t above = total - below - s;
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

template <int R, int D, int NTILE, bool F8>
__global__ void __launch_bounds__(kSelThreads, 2) select_kernel(SelectArgs a) {
  constexpr int EB = F8 ? 1 : 2;                   // bytes per Kp element (E4M3 or bf16)
  constexpr int EPV = 16 / EB;                     // Kp elements per 16-byte vector
  constexpr int CH = kSelStage / (R * EB);         // tokens per stage
  constexpr int V = R * EB / 16;                   // 16-byte vectors per token
  constexpr int TPT = (R >= 64) ? 2 : 1;           // consumer threads per token
  constexpr int VPT = V / TPT;
  static_assert(V >= 1 && V % TPT == 0, "Kp rows of at least 16 bytes");
  constexpr int TOK_PER_PASS = kSelConsumers / TPT;
  constexpr int PASSES = CH / TOK_PER_PASS;
  static_assert(PASSES >= 1 && CH % TOK_PER_PASS == 0, "stage / thread mapping");

  cg::cluster_group cluster = cg::this_cluster();
  const int crank = static_cast<int>(cluster.block_rank());
  const int C = static_cast<int>(cluster.num_blocks());  // 8 or 16
  const int own_bins = sel_own_bins(C);  // even: a packed bin pair has one owner
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const int S = a.stages;
  const int keys_words = a.keys_words;
  unsigned char* ring = smem_raw;                                                        // [S][16 KB]
  uint32_t* keys = reinterpret_cast<uint32_t*>(ring + S * kSelStage);                   // [keys_words]
  uint32_t* histp = keys + keys_words;                                                   // [2048] packed 16-bit bins
  uint32_t* own = histp + kSelBins1 / 2;                                                 // [4096 / C] owned row bins
  float* qpart = reinterpret_cast<float*>(own + sel_own_words(C));                     // [R] this CTA's share of qs
  double* npart = reinterpret_cast<double*>(qpart + kSelMaxR);                          // [n_new][R] newest-row shares
  unsigned char* kpn = reinterpret_cast<unsigned char*>(npart + a.n_new * R);           // [n_new][R] newest Kp rows
  // after the scan the ring holds the row histogram copy and the selection scratch
  uint32_t* ghist = reinterpret_cast<uint32_t*>(ring);                                   // [4096]
  uint32_t* hloc = ghist + kSelBins1;                                                    // [1024]
  uint32_t* masks = hloc + kSelBins2;                                                    // [warps][kSelMaskWords]
  uint32_t* cands = masks + kSelWarps * kSelMaskWords;                                   // [warps][kSelCapW]
  uint32_t* cmasks = cands + kSelWarps * kSelCapW;                                       // [warps][kSelMaskWords]
  // after the row histogram is assembled the packed histogram holds the gathered keys
  uint32_t* gbuf = histp;                                                                // [kSelGather]
  uint32_t* totA = histp;                                                                // fallback totals
  uint32_t* totB = histp + kSelBins2;
  // before the scan the keys area holds the projection scratch
  double* red = reinterpret_cast<double*>(keys);                                         // [256]
  float* qsum = reinterpret_cast<float*>(red + kSelConsumers);                          // [d / 8 chunks * 8]
  float* qgrp = qsum + kSelMaxDn;                                                        // [head groups][dn]

  __shared__ __align__(8) uint64_t full[8], empty[8];
  __shared__ float qs[kSelMaxR];
  __shared__ uint32_t dig, krem_s, gcnt, gbase;
  __shared__ uint32_t cta_gt[kSelMaxCluster], cta_eq[kSelMaxCluster], cta_ab[kSelMaxCluster];
  __shared__ uint32_t warp_gt[kSelWarps], warp_eq[kSelWarps], warp_nc[kSelWarps];
  __shared__ uint32_t scan_tmp[32];
  __shared__ int aborted_s;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row = blockIdx.y;
  const int b = row / a.Hkv, h = row % a.Hkv;
  const int G = a.Hq / a.Hkv;
  const int d = a.d;

  int64_t T = a.seq_lens[b];
  if (T < 0 || T > a.T_cap) {
    if (crank == 0 && tid == 0) flag_error(a.status, DEVFLAG_BAD_SEQ_LEN);
    T = T < 0 ? 0 : a.T_cap;
  }
  const int64_t Wc = min64(max64(a.window, 0), T);
  const int n = static_cast<int>(T - Wc);
  const int k_eff = static_cast<int>(min64(a.k, n));
  const int per = min(a.per, ((((n + C - 1) / C) + 31) & ~31));
  const int lo = crank * per;
  const int len = max(0, min(n, lo + per) - lo);
  const int n_new = static_cast<int>(min64(max64(a.n_new, 0), T));
  const int64_t t_new0 = T - n_new;  // newest rows [t_new0, T) are projected here
  int32_t* out = a.idx + static_cast<int64_t>(row) * a.k;
  const WaitTest wt = wait_test_read(a.status, row == 0 && crank == 0);

  if (tid == 0) {
    gcnt = 0;
    aborted_s = 0;
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kSelConsumers / 32);
    }
    fence_mbarrier_init();
  }
  for (int i = tid; i < own_bins; i += kSelThreads) own[i] = 0u;
  for (int i = tid; i < kSelBins1 / 2; i += kSelThreads) histp[i] = 0u;
  if (crank == 0 && tid == 0) {
    a.n_sel[row] = k_eff;
    if (a.counters) a.counters[row] = 0;
  }
  for (int j = k_eff + crank * kSelThreads + tid; j < a.k; j += C * kSelThreads) out[j] = -1;
  __syncthreads();
  if (wt.withhold && tid == 0) wait_test_disarm(a.status);  // every thread has read it

  // ---- the producer warp streams the slice's Kp rows.  The consumers form this CTA's share
  // of the projections (dims [dlo, dlo + dn): the d / 8 chunks of 8 dims split over the
  // cluster), exchange the shares through one cluster barrier and add them in rank order.
  const int nch = (len + CH - 1) / CH;
  const bool select_all = (k_eff == n);  // includes n == 0: no scan needed
  const unsigned char* Kprow = static_cast<const unsigned char*>(a.Kp) + (b * a.ps[0] + h * a.ps[1]) * EB;
  if (warp == kSelWarps - 1) {
    cluster_arrive_release();  // own[] and gcnt are zero (the producer has no share to publish)
    if (lane == 0 && !select_all) {
      const uint64_t policy = l2_policy_evict_first();
      for (int c = 0; c < nch; ++c) {
        const int s = c % S;
        if (c >= S && !mbar_wait_bounded(&empty[s], static_cast<uint32_t>((c / S - 1) & 1), a.status)) {
          atomicExch(&aborted_s, 1);
          break;
        }
        if (wt.withhold && c == 0) continue;  // the armed test: this stage's copy never comes
        const int t0 = lo + c * CH;
        const uint32_t cnt = static_cast<uint32_t>(min(CH, lo + len - t0));
        mbar_arrive_expect_tx(&full[s], cnt * R * EB);
        bulk_g2s(ring + s * kSelStage, Kprow + static_cast<int64_t>(t0) * a.ps[2] * EB, cnt * R * EB, &full[s], policy);
      }
    }
    __syncwarp();
    cluster_wait_acquire();
  } else {
    const int chunks = d / 8;
    const int c_lo = chunks * crank / C, c_hi = chunks * (crank + 1) / C;
    const int dlo = c_lo * 8, dn = (c_hi - c_lo) * 8;
    const int parts = kSelConsumers / R, j = tid % R, part = tid / R;
    const float* Ph = a.P + static_cast<int64_t>(h) * d * R;
    const __nv_bfloat16* Kb = static_cast<const __nv_bfloat16*>(a.K) + b * a.ks[0] + h * a.ks[1];
    if (!select_all) {
      // group sum of this CTA's dims: thread = (16-byte chunk, head group); fixed-order adds
      const int nc = dn / 8;
      const int ng = nc > 0 ? min(G, kSelConsumers / nc) : 0;
      const __nv_bfloat16* Qg = static_cast<const __nv_bfloat16*>(a.Q) + (static_cast<int64_t>(b) * a.Hq + h * G) * d;
      if (nc > 0 && tid < nc * ng) {
        const int c = tid % nc, hg = tid / nc;
        float s8[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int g = hg; g < G; g += ng) {
          const uint4 v = __ldg(reinterpret_cast<const uint4*>(Qg + static_cast<int64_t>(g) * d + dlo + c * 8));
          s8[0] += __uint_as_float(v.x << 16); s8[1] += __uint_as_float(v.x & 0xFFFF0000u);
          s8[2] += __uint_as_float(v.y << 16); s8[3] += __uint_as_float(v.y & 0xFFFF0000u);
          s8[4] += __uint_as_float(v.z << 16); s8[5] += __uint_as_float(v.z & 0xFFFF0000u);
          s8[6] += __uint_as_float(v.w << 16); s8[7] += __uint_as_float(v.w & 0xFFFF0000u);
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) qgrp[hg * dn + c * 8 + e] = s8[e];
      }
      consumers_sync();
      for (int i = tid; i < dn; i += kSelConsumers) {
        float s1 = 0.f;
        for (int hg = 0; hg < ng; ++hg) s1 += qgrp[hg * dn + i];
        qsum[i] = s1;
      }
      consumers_sync();
      // this CTA's share of qs = P_h^T (sum_g q_g) over its dims
      float acc = 0.f;
      for (int i = part; i < dn; i += parts) acc = fmaf(__ldg(Ph + (dlo + i) * R + j), qsum[i], acc);
      red[part * R + j] = acc;
      consumers_sync();
      if (tid < R) {
        float t2 = 0.f;
        for (int p = 0; p < parts; ++p) t2 += static_cast<float>(red[p * R + tid]);
        qpart[tid] = t2;
      }
      consumers_sync();
    }
    // this CTA's share of the projection of each newest row (fp64)
    for (int q = 0; q < n_new; ++q) {
      const __nv_bfloat16* krow = Kb + (t_new0 + q) * a.ks[2];
      double acc = 0.0;
      for (int i = part; i < dn; i += parts)
        acc = fma(static_cast<double>(__bfloat162float(krow[dlo + i])), static_cast<double>(__ldg(Ph + (dlo + i) * R + j)),
                  acc);
      red[part * R + j] = acc;
      consumers_sync();
      if (tid < R) {
        double t2 = 0.0;
        for (int p = 0; p < parts; ++p) t2 += red[p * R + tid];
        npart[q * R + tid] = t2;
      }
      consumers_sync();
    }
    cluster_arrive_release();  // shares published; own[] and gcnt are zero
    cluster_wait_acquire();
    // add the shares in rank order: qs, and the newest rows this CTA owns (rows inside
    // its slice, or rank C-1 for rows in the window), stored to Kp and kept for the scan
    if (tid < R) {
      if (!select_all) {
        float t2 = 0.f;
        for (int c = 0; c < C; ++c) t2 += *(cluster.map_shared_rank(qpart, c) + tid);
        qs[tid] = t2;
      }
      for (int q = 0; q < n_new; ++q) {
        const int64_t t = t_new0 + q;
        const bool mine = (t < n) ? (t >= lo && t < lo + len) : (crank == C - 1);
        if (!mine) continue;
        double t2 = 0.0;
        for (int c = 0; c < C; ++c) t2 += *(cluster.map_shared_rank(npart, c) + q * R + tid);
        const int64_t off = b * a.ps[0] + h * a.ps[1] + t * a.ps[2] + tid;
        if constexpr (F8) {
          const uint8_t v = f64_to_e4m3_rne_sat(t2);
          kpn[q * R + tid] = v;
          static_cast<uint8_t*>(a.Kp)[off] = v;
        } else {
          const uint16_t v = f64_to_bf16_rne(t2);
          reinterpret_cast<uint16_t*>(kpn)[q * R + tid] = v;
          static_cast<uint16_t*>(a.Kp)[off] = v;
        }
      }
    }
    consumers_sync();
    if (!select_all) {
      // ---- score scan of the slice
      const int sub = (TPT == 2) ? (tid & 1) : 0;
      const int tok_in_pass = tid / TPT;
      const int rot = kp_vector_rotation<VPT>(tid);
      float q[VPT][EPV];
#pragma unroll
      for (int jj = 0; jj < VPT; ++jj)
#pragma unroll
        for (int e = 0; e < EPV; ++e) q[jj][e] = qs[(sub * VPT + (jj + rot) % VPT) * EPV + e];
      bool dead = false;
      for (int c = 0; c < nch; ++c) {
        const int s = c % S;
        if (!dead && !mbar_wait_bounded(&full[s], static_cast<uint32_t>((c / S) & 1), a.status, wt.limit_ns)) {
          dead = true;
          atomicExch(&aborted_s, 1);
        }
        const int t0 = lo + c * CH;
        const int cnt = min(CH, lo + len - t0);
        const unsigned char* buf = ring + s * kSelStage;
        if (!dead) {
#pragma unroll
          for (int p = 0; p < PASSES; ++p) {
            const int tok = p * TOK_PER_PASS + tok_in_pass;
            const int64_t tg = t0 + tok;
            const unsigned char* trow = (tg >= t_new0 && tok < cnt) ? kpn + (tg - t_new0) * (R * EB)
                                                                    : buf + tok * (R * EB);
            float accv[VPT];
#pragma unroll
            for (int jj = 0; jj < VPT; ++jj) {
              const uint4 raw = *reinterpret_cast<const uint4*>(trow + (sub * VPT + (jj + rot) % VPT) * 16);
              accv[jj] = kp_vector_dot<F8>(q[jj], raw);
            }
            float sc = kp_rotated_sum<VPT>(accv);
            if (TPT == 2) sc += __shfl_xor_sync(0xFFFFFFFFu, sc, 1);
            if (sub == 0 && tok < cnt) {
              const uint32_t key = float_to_ordered(sc);
              keys[c * CH + tok] = key;
              atomicAdd(&histp[key >> 21], 1u << (((key >> 20) & 1u) * 16u));
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive_one(&empty[s]);
      }
    }
  }
  __syncthreads();

  // the attended list of the row (selection, then the window) and this CTA's share of it
  // when the attention runs here: positions [crank * L, crank * L + L) of the list
  const int list_len = k_eff + static_cast<int>(Wc);
  const int L = (list_len + C - 1) / C;
  int32_t* tok_list = reinterpret_cast<int32_t*>(own);  // own[] is free once the selection is known
  if (select_all) {  // every candidate is selected (also n == 0)
    for (int j = crank * kSelThreads + tid; j < n; j += C * kSelThreads) out[j] = j;
    cluster.sync();  // no CTA exits while another may still read its shares
    if constexpr (D == 0) return;
  } else {
    const bool aborted = aborted_s != 0;
    if (aborted && tid == kSelConsumers) {  // let every copy still in flight land before the CTA moves on
      for (int s = 0; s < S; ++s)
        for (int par = 0; par < 2; ++par)
          mbar_wait_bounded(&full[s], par, nullptr, wt.limit_ns < 50000000ull ? wt.limit_ns : 50000000ull);
    }
    __syncthreads();

    // ---- the row's first-digit histogram, assembled in the owners' shared memory
    for (int i = tid; i < kSelBins1 / 2; i += kSelThreads) {
      const uint32_t v = histp[i];
      if (v == 0u) continue;
      const int bin0 = 2 * i;
      uint32_t* dst = cluster.map_shared_rank(own, bin0 / own_bins) + (bin0 % own_bins);
      if (v & 0xFFFFu) atomicAdd(dst, v & 0xFFFFu);
      if (v >> 16) atomicAdd(dst + 1, v >> 16);
    }
    cluster.sync();  // the row histogram is complete
    {
      constexpr int kPerT = (kSelBins1 + kSelThreads - 1) / kSelThreads;
      uint32_t v[kPerT];
#pragma unroll
      for (int u = 0; u < kPerT; ++u) {  // all remote loads in flight before the first store
        const int i = tid + u * kSelThreads;
        v[u] = (i < kSelBins1) ? *(cluster.map_shared_rank(own, i / own_bins) + i % own_bins) : 0u;
      }
#pragma unroll
      for (int u = 0; u < kPerT; ++u) {
        const int i = tid + u * kSelThreads;
        if (i < kSelBins1) ghist[i] = v[u];
      }
    }
    __syncthreads();
    sel_find_digit<kSelBins1>(ghist, static_cast<uint32_t>(k_eff), scan_tmp, &dig, &krem_s);
    const uint32_t d1 = dig;
    const uint32_t k1 = krem_s;

    // ---- one pass over the slice: each warp marks its keys above bin d1 ("definites", all
    // selected) in a bitmap of its range and lists its keys inside bin d1 ("candidates", in
    // any order: ties are later ranked by position).
    const int wc = ((len + kSelWarps - 1) / kSelWarps + 31) & ~31;
    const int w_lo = warp * wc, w_hi = min(len, w_lo + wc);
    const uint32_t lt_mask = (1u << lane) - 1u;
    uint32_t* my_mask = masks + warp * kSelMaskWords;
    uint32_t* my_cands = cands + warp * kSelCapW;
    uint32_t nd = 0, nca = 0;
    const bool use_mask = wc <= 32 * kSelMaskWords;  // block-uniform
    {
      uint32_t* my_cmask = cmasks + warp * kSelMaskWords;
      for (int base = w_lo; base < w_hi; base += 128) {
        // lane L reads keys base + 32 e + L: the ballots of key-slot e are bitmap words
        // (base - w_lo) / 32 + e of the definites and of the candidates, in index order
        uint32_t kk[4], mdef[4], mcan[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) kk[e] = keys[min(base + 32 * e + lane, w_hi - 1)];  // all loads first
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const bool ok = base + 32 * e + lane < w_hi;
          mdef[e] = __ballot_sync(0xFFFFFFFFu, ok && (kk[e] >> 20) > d1);
          mcan[e] = __ballot_sync(0xFFFFFFFFu, ok && (kk[e] >> 20) == d1);
        }
        nd += __popc(mdef[0]) + __popc(mdef[1]) + __popc(mdef[2]) + __popc(mdef[3]);
        // one lane stores the step's four words of each bitmap (16-byte aligned: 4 words a step)
        const int wb = (base - w_lo) / 32;
        if (use_mask && lane == 0 && wb < kSelMaskWords) {
          *reinterpret_cast<uint4*>(my_mask + wb) = make_uint4(mdef[0], mdef[1], mdef[2], mdef[3]);
          *reinterpret_cast<uint4*>(my_cmask + wb) = make_uint4(mcan[0], mcan[1], mcan[2], mcan[3]);
        }
      }
      __syncwarp();
      // the candidates' positions from their bitmap (lane L: words L and L + 32)
      const int nwords = (w_hi > w_lo) ? (w_hi - w_lo + 31) / 32 : 0;
      const uint32_t cw0 = (use_mask && lane < nwords) ? my_cmask[lane] : 0u;
      const uint32_t cw1 = (use_mask && lane + 32 < nwords) ? my_cmask[lane + 32] : 0u;
      const uint32_t cnt = __popc(cw0) + __popc(cw1);
      uint32_t incl = cnt;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const uint32_t y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
        if (lane >= off) incl += y;
      }
      nca = use_mask ? __shfl_sync(0xFFFFFFFFu, incl, 31) : kSelCapW + 1u;  // no bitmap: rescan later
      uint32_t p = incl - cnt;
      for (uint32_t v = cw0; v; v &= v - 1, ++p)
        if (p < kSelCapW) my_cands[p] = static_cast<uint32_t>(w_lo + lane * 32 + (__ffs(v) - 1));
      for (uint32_t v = cw1; v; v &= v - 1, ++p)
        if (p < kSelCapW) my_cands[p] = static_cast<uint32_t>(w_lo + (lane + 32) * 32 + (__ffs(v) - 1));
      __syncwarp();
    }
    const bool cand_list = nca <= kSelCapW;  // warp-uniform: else this warp rescans its range
    if (lane == 0) warp_nc[warp] = cand_list ? nca : (kSelGather + 1u);
    __syncthreads();

    // ---- gather the row's in-bin keys into rank 0 (its packed histogram is no longer read)
    uint32_t* gcnt0 = cluster.map_shared_rank(&gcnt, 0);
    uint32_t* gbuf0 = cluster.map_shared_rank(gbuf, 0);
    if (tid == 0) {
      uint32_t tot = 0;
      for (int w = 0; w < kSelWarps; ++w) tot += warp_nc[w];
      tot = min(tot, kSelGather + 1u);
      gbase = (tot > 0) ? atomicAdd(gcnt0, tot) : 0u;
    }
    __syncthreads();
    {
      uint32_t off = gbase;
      for (int w = 0; w < warp; ++w) off += warp_nc[w];
      if (cand_list && off + nca <= kSelGather)
        for (int j = lane; j < static_cast<int>(nca); j += 32) gbuf0[off + j] = keys[my_cands[j]];
    }
    cluster.sync();  // the row's in-bin keys (or an overflowed count) are in rank 0
    const uint32_t gtotal = *gcnt0;
    uint32_t prefix = d1 << 20, mask = 0xFFF00000u, krem = k1;
    if (gtotal <= kSelGather) {
      // exact selection among the gathered keys, locally in every CTA: digits 2 and 3
      if (crank != 0) {  // copy the gathered keys: all remote loads in flight before the stores
        constexpr int kCopy = (kSelGather + kSelThreads - 1) / kSelThreads;
        uint32_t v[kCopy];
#pragma unroll
        for (int u = 0; u < kCopy; ++u) {
          const int j = tid + u * kSelThreads;
          v[u] = (j < static_cast<int>(gtotal)) ? gbuf0[j] : 0u;
        }
#pragma unroll
        for (int u = 0; u < kCopy; ++u) {
          const int j = tid + u * kSelThreads;
          if (j < static_cast<int>(gtotal)) gbuf[j] = v[u];
        }
      }
#pragma unroll 1
      for (int pass = 0; pass < 2; ++pass) {
        const int shift = (pass == 0) ? 10 : 0;
        for (int i = tid; i < kSelBins2; i += kSelThreads) hloc[i] = 0;
        __syncthreads();
        for (int j = tid; j < static_cast<int>(gtotal); j += kSelThreads) {
          const uint32_t key = gbuf[j];
          if ((key & mask) == prefix) atomicAdd(&hloc[(key >> shift) & (kSelBins2 - 1)], 1u);
        }
        __syncthreads();
        sel_find_digit<kSelBins2>(hloc, krem, scan_tmp, &dig, &krem_s);
        prefix |= dig << shift;
        mask |= static_cast<uint32_t>(kSelBins2 - 1) << shift;
        krem = krem_s;
      }
    } else {
      // too many in-bin keys for the gather buffer: digits 2 and 3 from cluster-wide
      // histograms in rank 0 (every CTA takes this branch: gtotal is the same everywhere)
      uint32_t* totA0 = cluster.map_shared_rank(totA, 0);
      uint32_t* totB0 = cluster.map_shared_rank(totB, 0);
      if (crank == 0)
        for (int i = tid; i < kSelBins2; i += kSelThreads) { totA[i] = 0; totB[i] = 0; }
      cluster.sync();
#pragma unroll 1
      for (int pass = 0; pass < 2; ++pass) {
        const int shift = (pass == 0) ? 10 : 0;
        uint32_t* tot0 = (pass == 0) ? totA0 : totB0;
        for (int i = tid; i < kSelBins2; i += kSelThreads) hloc[i] = 0;
        __syncthreads();
        if (cand_list) {
          for (int j = lane; j < static_cast<int>(nca); j += 32) {
            const uint32_t key = keys[my_cands[j]];
            if ((key & mask) == prefix) atomicAdd(&hloc[(key >> shift) & (kSelBins2 - 1)], 1u);
          }
        } else {
          for (int i = w_lo + lane; i < w_hi; i += 32) {
            const uint32_t key = keys[i];
            if ((key & mask) == prefix) atomicAdd(&hloc[(key >> shift) & (kSelBins2 - 1)], 1u);
          }
        }
        __syncthreads();
        for (int i = tid; i < kSelBins2; i += kSelThreads) {
          const uint32_t v = hloc[i];
          if (v) atomicAdd(&tot0[i], v);
        }
        cluster.sync();
        sel_find_digit<kSelBins2>(tot0, krem, scan_tmp, &dig, &krem_s);
        prefix |= dig << shift;
        mask |= static_cast<uint32_t>(kSelBins2 - 1) << shift;
        krem = krem_s;
      }
    }
    const uint32_t kstar = prefix;  // the k-th largest key
    const uint32_t need = krem;     // keys equal to kstar to take, lowest index first

    // ---- per-warp counts of keys > kstar and == kstar, published to every CTA
    {
      uint32_t ngt = nd, neq = 0;
      if (cand_list) {
        for (int j0 = 0; j0 < static_cast<int>(nca); j0 += 32) {
          const int j = j0 + lane;
          const uint32_t key = (j < static_cast<int>(nca)) ? keys[my_cands[j]] : 0u;
          ngt += __popc(__ballot_sync(0xFFFFFFFFu, j < static_cast<int>(nca) && key > kstar));
          neq += __popc(__ballot_sync(0xFFFFFFFFu, j < static_cast<int>(nca) && key == kstar));
        }
      } else {
        for (int base = w_lo; base < w_hi; base += 32) {
          const int i = base + lane;
          const uint32_t key = (i < w_hi) ? keys[i] : 0u;
          ngt += __popc(__ballot_sync(0xFFFFFFFFu, i < w_hi && key > kstar && (key >> 20) == d1));
          neq += __popc(__ballot_sync(0xFFFFFFFFu, i < w_hi && key == kstar));
        }
      }
      if (lane == 0) { warp_gt[warp] = ngt; warp_eq[warp] = neq; }
    }
    __syncthreads();
    if (tid < C) {
      uint32_t g = 0, e = 0;
      for (int w = 0; w < kSelWarps; ++w) { g += warp_gt[w]; e += warp_eq[w]; }
      *cluster.map_shared_rank(&cta_gt[crank], tid) = g;
      *cluster.map_shared_rank(&cta_eq[crank], tid) = e;
      *cluster.map_shared_rank(&cta_ab[crank], tid) = aborted ? 1u : 0u;
    }
    cluster.sync();  // the counts are everywhere; other CTAs' memory is no longer read
    bool any_aborted = false;
    for (int c = 0; c < C; ++c) any_aborted |= (cta_ab[c] != 0u);
    if (any_aborted) {  // a wait gave up in some CTA of the row (flagged): the row's selection is empty
      for (int j = crank * kSelThreads + tid; j < k_eff; j += C * kSelThreads) out[j] = -1;
      if (crank == 0 && tid == 0) a.n_sel[row] = 0;
      if constexpr (D > 0) for (int j = tid; j < L; j += kSelThreads) tok_list[j] = -1;
    } else {

      // ---- output positions: CTAs in rank order, warps in index order
      uint32_t base_out = 0, eq_before = 0;
      for (int c = 0; c < crank; ++c) {
        const uint32_t qv = (need > eq_before) ? min(cta_eq[c], need - eq_before) : 0u;
        base_out += cta_gt[c] + qv;
        eq_before += cta_eq[c];
      }
      const uint32_t quota = (need > eq_before) ? min(cta_eq[crank], need - eq_before) : 0u;
      uint32_t pos = base_out, eq_rank = 0;
      for (int w = 0; w < warp; ++w) {
        const uint32_t qv = (quota > eq_rank) ? min(warp_eq[w], quota - eq_rank) : 0u;
        pos += warp_gt[w] + qv;
        eq_rank += warp_eq[w];
      }
      const uint32_t wquota = (quota > eq_rank) ? min(warp_eq[warp], quota - eq_rank) : 0u;
      const int words = (w_hi > w_lo) ? (w_hi - w_lo + 31) / 32 : 0;  // bitmap words written by the scan
      if (cand_list && use_mask) {
        // add the selected candidates to the bitmap of definites, then emit the range in order
        uint32_t* m = my_mask;
        for (int j0 = 0; j0 < static_cast<int>(nca); j0 += 32) {
          const int j = j0 + lane;
          const uint32_t i = (j < static_cast<int>(nca)) ? my_cands[j] : 0u;
          const uint32_t key = (j < static_cast<int>(nca)) ? keys[i] : 0u;
          const bool gt = j < static_cast<int>(nca) && key > kstar;
          bool take = gt;
          if (j < static_cast<int>(nca) && key == kstar) {
            // rank among this warp's keys equal to kstar by position (the list may be unordered)
            uint32_t rank = 0;
            for (int jj = 0; jj < static_cast<int>(nca); ++jj) {
              const uint32_t o2 = my_cands[jj];
              rank += (o2 < i && keys[o2] == kstar) ? 1u : 0u;
            }
            take = rank < wquota;
          }
          if (take) {
            const uint32_t o = i - static_cast<uint32_t>(w_lo);
            atomicOr(&m[o >> 5], 1u << (o & 31));
          }
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
          if (p0 < static_cast<uint32_t>(k_eff)) {
            const int t = gb + lane * 32 + (__ffs(v) - 1);
            out[p0] = t;
            if constexpr (D > 0) *(cluster.map_shared_rank(tok_list, p0 / L) + p0 % L) = t;
          } else {
            flag_error(a.status, DEVFLAG_BAD_INDEX);  // unreachable when the counts are consistent
          }
          ++p0;
        }
        for (uint32_t v = w1; v; v &= v - 1) {
          if (p1 < static_cast<uint32_t>(k_eff)) {
            const int t = gb + (lane + 32) * 32 + (__ffs(v) - 1);
            out[p1] = t;
            if constexpr (D > 0) *(cluster.map_shared_rank(tok_list, p1 / L) + p1 % L) = t;
          } else {
            flag_error(a.status, DEVFLAG_BAD_INDEX);
          }
          ++p1;
        }
      } else {
        // long lists: rescan this warp's range and compact with ballots
        uint32_t eq_run = 0;
        for (int base = w_lo; base < w_hi; base += 32) {
          const int i = base + lane;
          const uint32_t key = (i < w_hi) ? keys[i] : 0u;
          const bool gt = i < w_hi && key > kstar;
          const bool eq = i < w_hi && key == kstar;
          const uint32_t eq_m = __ballot_sync(0xFFFFFFFFu, eq);
          const bool sel = gt || (eq && (eq_run + __popc(eq_m & lt_mask)) < wquota);
          const uint32_t sel_m = __ballot_sync(0xFFFFFFFFu, sel);
          if (sel) {
            const uint32_t p = pos + __popc(sel_m & lt_mask);
            if (p < static_cast<uint32_t>(k_eff)) {
              out[p] = lo + i;
              if constexpr (D > 0) *(cluster.map_shared_rank(tok_list, p / L) + p % L) = lo + i;
            } else {
              flag_error(a.status, DEVFLAG_BAD_INDEX);
            }
          }
          pos += __popc(sel_m);
          eq_run += __popc(eq_m);
        }
      }
    }  // selection written
  }  // not every candidate selected

  if constexpr (D > 0) {
    // ---- attention of the row's list: this CTA takes positions [my_lo, my_lo + my_len); the
    // selected ones were scattered into tok_list above, the window ones are filled here
    const int my_lo = crank * L;
    const int my_len = max(0, min(list_len, my_lo + L) - my_lo);
    const int64_t win_start = T - Wc;
    for (int j = tid; j < my_len; j += kSelThreads) {
      const int p = my_lo + j;
      if (select_all) tok_list[j] = p;  // selection [0, n) then window [n, T): token p
      else if (p >= k_eff) tok_list[j] = static_cast<int32_t>(win_start + (p - k_eff));
    }
    const int64_t hq0 = static_cast<int64_t>(b) * a.Hq + static_cast<int64_t>(h) * G;
    uint32_t qf[NTILE][D / 16][2];
    load_q_frags<D, NTILE>(a.Q, hq0, G, qf);
    cluster_arrive_release();  // the scattered positions are in place
    cluster_wait_acquire();
    AttnArgs at{};
    at.K = a.K;
    at.V = a.V;
    for (int i = 0; i < 3; ++i) { at.ks[i] = a.ks[i]; at.vs[i] = a.vs[i]; }
    at.B = a.B;
    at.Hq = a.Hq;
    at.Hkv = a.Hkv;
    at.dk = D;
    at.dv = D;
    at.T_cap = a.T_cap;
    at.window = a.window;
    at.sm_scale = a.sm_scale;
    at.S = C;
    at.split_len = L;
    at.O = a.O;
    at.lse = a.lse;
    at.out_bf16 = a.out_bf16;
    at.status = a.status;
    attn_core<D, NTILE, false>(at, row, crank, b, h, G, hq0, qf, tok_list, win_start, my_lo, my_len, smem_raw);
  }
}

constexpr int kSelMaxSlice = 16384;    // keys per CTA kept in shared memory
constexpr int kSelStaticBytes = 3072;  // static shared memory of the kernel, rounded up

// Number of clusters of this shape that can be resident at once (cached per device).
template <typename Kernel>
int active_clusters(Kernel kernel, int C, size_t smem, int rows) {
  static std::mutex mu;
  static std::map<std::tuple<int, int, size_t, const void*>, int> cache;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  const auto key = std::make_tuple(dev, C, smem, reinterpret_cast<const void*>(kernel));
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C, rows > 0 ? rows : 1);
  cfg.blockDim = dim3(kSelThreads);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kernel, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    n = 0;
  }
  cache[key] = n;
  return n;
}

template <int R, int D, int NTILE, bool F8>
cudaError_t launch_select_r(SelectArgs a, int num_sms, cudaStream_t s) {
  auto kernel = select_kernel<R, D, NTILE, F8>;
  static int done[64] = {0};
  cudaError_t e = set_smem_limit_once(kernel, 227u * 1024u - kSelStaticBytes, done);
  if (e != cudaSuccess) return e;
  static int np_done[64] = {0};
  int dev = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  if (!np_done[dev]) {  // clusters above 8 CTAs are non-portable sizes
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess)
      np_done[dev] = 1;
    else
      np_done[dev] = -1, (void)cudaGetLastError();
  }
  const int rows = a.B * a.Hkv;
  // Cluster size and ring depth.  Sizes are tried from the largest down: 9..16 CTAs per row
  // only when 8 per row would leave SMs idle, fewer than 8 (down to 2) only when 8 per row
  // cannot all be resident at once, and no size whose slices would be shorter than
  // kSelMinSlice tokens (on short rows the fixed cost of a larger cluster dominates).  The first size whose clusters are all resident wins, with
  // the deepest ring that keeps them so: a second wave of clusters would pay the scan and the
  // selection's serial tail twice.  If no size fits in one wave, 8 CTAs per row run in two.
  // With the attention inside, the ring and keys areas also hold the attention's buffers, and
  // each CTA's share of the attended list must fit its token list.
  int C = 0, stages = 2, per_c = 0, kw_c = 0;
  size_t fixed = 0;
  int fb_per = 0, fb_kw = 0;  // the two-wave fallback at 8 CTAs per row
  size_t fb_fixed = 0;
  const int64_t list_max = a.k + min64(max64(a.window, 0), a.T_cap);
  const int c_max = (np_done[dev] > 0 && static_cast<int64_t>(rows) * 8 < num_sms) ? kSelMaxCluster : 8;
  for (int c_try = c_max; c_try >= kSelMinCluster; --c_try) {
    const int per = static_cast<int>(ceil_div(ceil_div(a.T_cap, c_try), 32) * 32);
    if (per > kSelMaxSlice) continue;
    if (c_try > kSelMinCluster && per < kSelMinSlice) continue;               // short rows: fewer, fuller CTAs
    if (ceil_div(a.d / 8, c_try) * 8 > kSelMaxDn) continue;                    // share of the projections
    const int own_words = sel_own_words(c_try);
    if (D > 0 && ceil_div(list_max, c_try) > own_words) continue;             // token list lives in own[]
    const size_t tail = (kSelBins1 / 2) * 4 + static_cast<size_t>(own_words) * 4 + kSelMaxR * 4 +
                        static_cast<size_t>(a.n_new) * R * 8 + static_cast<size_t>((a.n_new * R + 7) & ~7) * 2;
    int st_ok = 0, kw_ok = 0;
    for (int st = 8; st >= 2; --st) {
      int kw = max(per, kSelKeysMin / 4);
      if (D > 0) {
        const int need = attn_main_bytes<D>() - st * kSelStage;
        if (need > kw * 4) kw = (need + 3) / 4;
      }
      const size_t smem = static_cast<size_t>(st) * kSelStage + static_cast<size_t>(kw) * 4 + tail;
      if (smem + kSelStaticBytes > 227u * 1024u) continue;
      if (active_clusters(kernel, c_try, smem, rows) >= rows) { st_ok = st; kw_ok = kw; break; }
    }
    if (st_ok == 0) {  // these clusters would need a second wave
      if (c_try == 8) {
        fb_kw = max(per, kSelKeysMin / 4);
        if (D > 0) fb_kw = max(fb_kw, (attn_main_bytes<D>() - 2 * kSelStage + 3) / 4);
        fb_per = per;
        fb_fixed = static_cast<size_t>(fb_kw) * 4 + tail;
      }
      continue;
    }
    C = c_try;
    stages = st_ok;
    fixed = static_cast<size_t>(kw_ok) * 4 + tail;
    per_c = per;
    kw_c = kw_ok;
    break;
  }
  if (C == 0 && fb_fixed > 0) {
    C = 8;
    stages = 2;
    fixed = fb_fixed;
    per_c = fb_per;
    kw_c = fb_kw;
  }
  if (fixed == 0) return D > 0 ? cudaErrorNotSupported : cudaErrorInvalidValue;
  a.per = per_c;
  a.keys_words = kw_c;
  a.stages = stages;
  const size_t smem = static_cast<size_t>(stages) * kSelStage + fixed;
  if (smem + kSelStaticBytes > 227u * 1024u) return D > 0 ? cudaErrorNotSupported : cudaErrorInvalidValue;
  return launch_ex(kernel, dim3(C, rows), dim3(kSelThreads), smem, s, C, a);
}

template <int R, bool F8>
cudaError_t launch_select_rd(const SelectArgs& a, int num_sms, cudaStream_t s) {
  if (a.V == nullptr) return launch_select_r<R, 0, 1, F8>(a, num_sms, s);
  const int G = a.Hq / a.Hkv;
  if (G > 16) return cudaErrorNotSupported;
  switch (a.d) {
    case 64:
      return G <= 8 ? launch_select_r<R, 64, 1, F8>(a, num_sms, s) : launch_select_r<R, 64, 2, F8>(a, num_sms, s);
    case 128:
      return G <= 8 ? launch_select_r<R, 128, 1, F8>(a, num_sms, s) : launch_select_r<R, 128, 2, F8>(a, num_sms, s);
    default: return cudaErrorNotSupported;
  }
}

}  // namespace
}  // namespace jssa
