// Shared pieces of the GQA attention kernels: the per-split flash-decode core (main loop,
// combine of the warps' states and the split's output path) and the two ways splits are
// merged.  Used by the standalone attention kernel (attn.cu) and by the selection kernel when
// it runs the attention of its row itself (select.cu).
//
// "Joint Subspace Sparse Attention for Efficient Long-Context Decoding", §3.3: the selected
// K/V rows are read in place from the standard GQA cache; split-T partials are combined by
// log-sum-exp.  The design of the core is described at the top of attn.cu.
#pragma once

#include <cooperative_groups.h>

#include <cmath>

#include "common.cuh"
#include "launch.h"

namespace cg = cooperative_groups;

namespace jssa {

constexpr int kAttnWarps = 4;
constexpr int kSub = 16;                 // tokens per warp subtile
constexpr int kMaxTokList = 4096;        // indexed mode: split length bound (token list in smem)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// Per head dimension D: kAttnWarps warp groups stream the subtiles; a group is one warp, or,
// for D = 256, a pair of warps that each take half of the head dims (the score partials of
// the two halves are added through shared memory, then both warps run the same softmax and
// each accumulates its half of the output), which halves the dependency chain of a warp and
// doubles the warps that hide each other's latency.
template <int D>
struct AttnCfg {
  static constexpr int HALVES = (D >= 256) ? 2 : 1;    // warps per group
  static constexpr int DW = D / HALVES;                // head dims per warp
  static constexpr int WARPS = kAttnWarps * HALVES;
  static constexpr int THREADS = WARPS * 32;
  static constexpr int STAGES = (DW <= 64) ? 4 : 3;
  static constexpr int CPR = DW / 8;                   // 16-byte chunks per row and warp
  static constexpr int SUB_BYTES = kSub * DW * 2;      // one K or V subtile (this warp's dims)
  static constexpr int STAGE_BYTES = 2 * SUB_BYTES;
  static constexpr int RING_BYTES = WARPS * STAGES * STAGE_BYTES;
  static constexpr int XCH_BYTES = (HALVES > 1) ? WARPS * 2 * 32 * 8 * 4 : 0;  // [warp][parity][lane][<= 8]
  static constexpr int COMBINE_BYTES = kAttnWarps * 16 * D * 4 + 2 * kAttnWarps * 16 * 4;
  static constexpr int PART_BYTES = 16 * D * 4 + 16 * 4;   // this CTA's partial (o, lse) for the cluster merge
  static constexpr int MAIN_BYTES = RING_BYTES + XCH_BYTES > COMBINE_BYTES + PART_BYTES ? RING_BYTES + XCH_BYTES
                                                                                        : COMBINE_BYTES + PART_BYTES;
};

template <int D>
constexpr int attn_main_bytes() { return AttnCfg<D>::MAIN_BYTES; }


// Combine the S split partials of query heads [hq0, hq0 + G) into O (and lse):
// O = sum_s w_s o_s with w_s = exp(lse_s - M) / sum_s' exp(lse_s' - M), M = max lse;
// lse = M + log(sum exp(lse_s - M)).  Run by the last CTA of a row to finish, on
// partials every CTA made visible with a device-scope fence before counting itself
// in.  The split weights go through shared memory (wsm: G * S floats); every thread
// then issues all the loads of two outputs (up to 16 splits each) before using them,
// so the merge costs about one memory round trip per two outputs.
constexpr int kMergeUnroll = 16;
template <int D>
__device__ __forceinline__ void merge_row(const AttnArgs& a, int64_t hq0, int G, float* wsm) {
  const int S = a.S;
  for (int i = threadIdx.x; i < G * S; i += blockDim.x) wsm[i] = __ldcg(a.part_lse + (hq0 + i / S) * S + i % S);
  __syncthreads();
  if (threadIdx.x < G) {
    float* w = wsm + threadIdx.x * S;
    float M = -INFINITY;
    for (int s = 0; s < S; ++s) M = fmaxf(M, w[s]);
    float L = 0.f;
    if (M != -INFINITY)
      for (int s = 0; s < S; ++s) { w[s] = expf(w[s] - M); L += w[s]; }
    const float inv = (M != -INFINITY) ? 1.f / L : 0.f;
    for (int s = 0; s < S; ++s) w[s] = (M != -INFINITY) ? w[s] * inv : 0.f;
    if (a.lse) a.lse[hq0 + threadIdx.x] = (M == -INFINITY) ? -INFINITY : M + logf(L);
  }
  __syncthreads();
  for (int i0 = threadIdx.x; i0 < G * D; i0 += 2 * blockDim.x) {
    const int i1 = i0 + blockDim.x;
    const bool has1 = i1 < G * D;
    const int h0 = i0 / D, d0 = i0 % D, h1 = has1 ? i1 / D : h0, d1 = has1 ? i1 % D : d0;
    const float* o0 = a.part_o + (hq0 + h0) * S * D + d0;
    const float* o1 = a.part_o + (hq0 + h1) * S * D + d1;
    float acc0 = 0.f, acc1 = 0.f;
    for (int s0 = 0; s0 < S; s0 += kMergeUnroll) {
      float v0[kMergeUnroll], v1[kMergeUnroll];
#pragma unroll
      for (int u = 0; u < kMergeUnroll; ++u) {
        const bool ok = s0 + u < S;
        v0[u] = ok ? __ldcg(o0 + static_cast<int64_t>(s0 + u) * D) : 0.f;
        v1[u] = (ok && has1) ? __ldcg(o1 + static_cast<int64_t>(s0 + u) * D) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kMergeUnroll; ++u) {
        if (s0 + u < S) {
          acc0 = fmaf(wsm[h0 * S + s0 + u], v0[u], acc0);
          acc1 = fmaf(wsm[h1 * S + s0 + u], v1[u], acc1);
        }
      }
    }
    const int64_t q0 = hq0 + h0, q1 = hq0 + h1;
    if (a.out_bf16) {
      static_cast<__nv_bfloat16*>(a.O)[q0 * D + d0] = __float2bfloat16_rn(acc0);
      if (has1) static_cast<__nv_bfloat16*>(a.O)[q1 * D + d1] = __float2bfloat16_rn(acc1);
    } else {
      static_cast<float*>(a.O)[q0 * D + d0] = acc0;
      if (has1) static_cast<float*>(a.O)[q1 * D + d1] = acc1;
    }
  }
}

// Count this CTA's finished partial in; the CTA that completes the row merges it and
// re-arms the counter for the next call.
template <int D>
__device__ __forceinline__ void finish_split(const AttnArgs& a, int row, int64_t hq0, int G, float* wsm) {
  __shared__ int is_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const int prev = atomicAdd(a.counters + row, 1);
    is_last = (prev == a.S - 1);
  }
  __syncthreads();
  if (!is_last) return;
  __threadfence();
  merge_row<D>(a, hq0, G, wsm);
  if (threadIdx.x == 0) a.counters[row] = 0;
}

// Split merge inside a thread-block cluster (one CTA per split of the row, S <= 16):
// every CTA keeps its normalised partial (o, lse) in its own shared memory; after a
// cluster barrier CTA c combines output slice c of the row.  Each thread reads, in one
// round of distributed-shared-memory loads, the S partials of its element and the S
// log-sum-exps of its head, forms the weights itself and writes the element (and the
// head's lse, from the thread of the head's first element).  A second barrier keeps the
// partials alive until every CTA has read them.
template <int D>
__device__ __forceinline__ void cluster_merge(const AttnArgs& a, int64_t hq0, int G, const float* pbuf,
                                              const float* plse) {
  cg::cluster_group cl = cg::this_cluster();
  const int S = static_cast<int>(cl.num_blocks());
  const int c = static_cast<int>(cl.block_rank());
  cl.sync();
  const int per = (G * D + S - 1) / S;
  const int lo = c * per, hi = min(G * D, lo + per);
  for (int i = lo + threadIdx.x; i < hi; i += blockDim.x) {
    const int head = i / D;
    float v[16], l[16];
#pragma unroll
    for (int q = 0; q < 16; ++q) {  // all remote loads in flight before the first use
      v[q] = (q < S) ? cl.map_shared_rank(pbuf, q)[i] : 0.f;
      l[q] = (q < S) ? cl.map_shared_rank(plse, q)[head] : -INFINITY;
    }
    float M = -INFINITY;
#pragma unroll
    for (int q = 0; q < 16; ++q) M = fmaxf(M, l[q]);
    float L = 0.f, o = 0.f;
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const float w = (M == -INFINITY || q >= S) ? 0.f : expf(l[q] - M);
      L += w;
      o = fmaf(w, v[q], o);
    }
    o = (L > 0.f) ? o / L : 0.f;
    const int64_t qi = hq0 + head;
    if (a.lse && i % D == 0) a.lse[qi] = (M == -INFINITY) ? -INFINITY : M + logf(L);
    if (a.out_bf16) static_cast<__nv_bfloat16*>(a.O)[qi * D + (i % D)] = __float2bfloat16_rn(o);
    else static_cast<float*>(a.O)[qi * D + (i % D)] = o;
  }
  cl.sync();
}

// Q^T as MMA B fragments: head nt*8 + g, dims dim0 + kk*16 + 2c (+8) (g = lane / 4, c = lane % 4),
// for the KS K-steps of 16 dims from dim0.
template <int D, int NTILE, int KS = D / 16>
__device__ __forceinline__ void load_q_frags(const void* Q, int64_t hq0, int G, uint32_t (&qf)[NTILE][KS][2],
                                             int dim0 = 0) {
  const int lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const __nv_bfloat16* Qg = static_cast<const __nv_bfloat16*>(Q) + hq0 * D;
#pragma unroll
  for (int nt = 0; nt < NTILE; ++nt) {
    const int head = nt * 8 + g;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      if (head < G) {
        const uint32_t* qp =
            reinterpret_cast<const uint32_t*>(Qg + static_cast<int64_t>(head) * D + dim0 + kk * 16 + 2 * c);
        qf[nt][kk][0] = __ldg(qp);
        qf[nt][kk][1] = __ldg(qp + 4);
      } else {
        qf[nt][kk][0] = 0u;
        qf[nt][kk][1] = 0u;
      }
    }
  }
}

// One split of a row: the attended tokens are tok_s[0, my_len) (indexed) or the contiguous
// range win_start + my_lo + [0, my_len) (dense).  The first AttnCfg<D>::WARPS warps stream and
// multiply (qf holds the Q fragments of the warp's dims); every thread of the block must call
// this (it holds block and cluster barriers).
// Writes the split's partial through the cluster merge (indexed, and dense launches of at
// most 8 splits) or the workspace and the row's last CTA (dense with more splits).
// smem_raw: AttnCfg<D>::MAIN_BYTES of shared memory.
template <int D, int NTILE, bool DENSE>
__device__ __forceinline__ void attn_core(const AttnArgs& a, int row, int split, int b, int h, int G, int64_t hq0,
                                          const uint32_t (&qf)[NTILE][AttnCfg<D>::DW / 16][2], const int32_t* tok_s,
                                          int64_t win_start, int64_t my_lo, int my_len, unsigned char* smem_raw) {
  using Cfg = AttnCfg<D>;
  constexpr int STAGES = Cfg::STAGES, CPR = Cfg::CPR, HALVES = Cfg::HALVES, DW = Cfg::DW;
  constexpr int KSTEPS = DW / 16;  // K-steps of the score MMA and M-tiles of the output, this warp's dims
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  const bool streams = warp < Cfg::WARPS;
  const int grp = warp % kAttnWarps, hf = (warp / kAttnWarps) % HALVES;  // warp group, half of the dims
  unsigned char* ring = smem_raw + (streams ? warp : 0) * STAGES * Cfg::STAGE_BYTES;
  float* pbuf = reinterpret_cast<float*>(smem_raw + Cfg::COMBINE_BYTES);   // [16][D] (cluster merge)
  float* plse = pbuf + 16 * D;                                              // [16]
  const bool in_cluster = !DENSE || a.cluster_merge != 0;  // the row's splits merge over DSMEM
  const float scale_log2 = a.sm_scale * kLog2e;
  const bool pack = NTILE == 1 && G <= 4;  // hi and lo parts of P in one value MMA
  float m_run[NTILE][2], l_run[NTILE][2];
  float acc[KSTEPS][NTILE][4];
#pragma unroll
  for (int nt = 0; nt < NTILE; ++nt) {
    m_run[nt][0] = m_run[nt][1] = -INFINITY;
    l_run[nt][0] = l_run[nt][1] = 0.f;
#pragma unroll
    for (int mt = 0; mt < KSTEPS; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
  }

  const __nv_bfloat16* Kb = static_cast<const __nv_bfloat16*>(a.K) + b * a.ks[0] + h * a.ks[1] + hf * DW;
  const __nv_bfloat16* Vb = static_cast<const __nv_bfloat16*>(a.V) + b * a.vs[0] + h * a.vs[1] + hf * DW;
  const int nsub = (my_len + kSub - 1) / kSub;
  // warps beyond the streaming ones (a larger block) only join the barriers
  const int my_count = (streams && nsub > grp) ? (nsub - grp + kAttnWarps - 1) / kAttnWarps : 0;

  auto token_at = [&](int j) -> int64_t {
    if (j >= my_len) return -1;
    return DENSE ? (win_start + my_lo + j) : static_cast<int64_t>(tok_s[j]);
  };
  auto issue = [&](int i) {  // i-th subtile of this warp's group into stage i % STAGES
    const int sub = grp + i * kAttnWarps;
    unsigned char* kbuf = ring + (i % STAGES) * Cfg::STAGE_BYTES;
    unsigned char* vbuf = kbuf + Cfg::SUB_BYTES;
#pragma unroll
    for (int q = 0; q < (kSub * CPR) / 32; ++q) {
      const int cid = lane + q * 32;
      const int tin = cid / CPR, ch = cid % CPR;
      const int64_t t = token_at(sub * kSub + tin);
      const uint32_t nbytes = (t >= 0) ? 16u : 0u;
      const int64_t tt = (t >= 0) ? t : 0;
      const int soff = (tin * CPR + (ch ^ (tin & 7))) * 16;
      cp_async16(kbuf + soff, Kb + tt * a.ks[2] + ch * 8, nbytes);
      cp_async16(vbuf + soff, Vb + tt * a.vs[2] + ch * 8, nbytes);
    }
  };

#pragma unroll
  for (int s = 0; s < STAGES - 1; ++s) {
    if (s < my_count) issue(s);
    cp_async_commit();
  }
  for (int i = 0; i < my_count; ++i) {
    if (i + STAGES - 1 < my_count) issue(i + STAGES - 1);
    cp_async_commit();
    cp_async_wait<STAGES - 1>();
    __syncwarp();
    const int sub = grp + i * kAttnWarps;
    const unsigned char* kbuf = ring + (i % STAGES) * Cfg::STAGE_BYTES;
    const unsigned char* vbuf = kbuf + Cfg::SUB_BYTES;

    // ---- S^T = K_sub . Q^T
    // (even and odd K-steps accumulate separately: two dependency chains of D/32 MMAs)
    float sacc[NTILE][4], sacc_odd[NTILE][4];
#pragma unroll
    for (int nt = 0; nt < NTILE; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[nt][e] = sacc_odd[nt][e] = 0.f;
    {
      const int tin = (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
      for (int kk = 0; kk < KSTEPS; ++kk) {
        const int ch = 2 * kk + (lane >> 4);
        uint32_t af[4];
        ldmatrix_x4(af, kbuf + (tin * CPR + (ch ^ (tin & 7))) * 16);
#pragma unroll
        for (int nt = 0; nt < NTILE; ++nt)
          mma_bf16_16816((kk & 1) ? sacc_odd[nt] : sacc[nt], af, qf[nt][kk][0], qf[nt][kk][1]);
      }
    }
#pragma unroll
    for (int nt = 0; nt < NTILE; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[nt][e] += sacc_odd[nt][e];
    if constexpr (HALVES > 1) {
      // add the other half's score partial (double-buffered by subtile parity; the pair's
      // barrier orders every write before the partner's read, and a buffer is written again
      // only after the partner has passed the next barrier, i.e. finished reading it)
      static_assert(NTILE * 4 <= 8, "exchange slot of 8 floats per lane");
      float* xch = reinterpret_cast<float*>(smem_raw + Cfg::RING_BYTES);
      const int partner = grp + (1 - hf) * kAttnWarps;
      float* mine = xch + ((warp * 2 + (i & 1)) * 32 + lane) * 8;
      const float* theirs = xch + ((partner * 2 + (i & 1)) * 32 + lane) * 8;
#pragma unroll
      for (int nt = 0; nt < NTILE; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) mine[nt * 4 + e] = sacc[nt][e];
      asm volatile("bar.sync %0, 64;" ::"r"(8 + grp) : "memory");
#pragma unroll
      for (int nt = 0; nt < NTILE; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) sacc[nt][e] += theirs[nt * 4 + e];
    }
    // ---- online softmax over the 16 tokens of this subtile
    // (with at most 4 heads, the hi and lo parts of P share one MMA: B columns 0-3 carry the
    // hi parts of heads 0-3 and columns 4-7 the lo parts, which the lanes holding columns 4-7
    // take from the lanes two to their left; those lanes' accumulators then follow the
    // rescaling of the head whose lo part they hold)
    const bool v0 = token_at(sub * kSub + g) >= 0;
    const bool v1 = token_at(sub * kSub + g + 8) >= 0;
    uint32_t bhi[NTILE][2], blo[NTILE][2];
#pragma unroll
    for (int nt = 0; nt < NTILE; ++nt) {
      float x[4];
      x[0] = v0 ? sacc[nt][0] * scale_log2 : -INFINITY;
      x[1] = v0 ? sacc[nt][1] * scale_log2 : -INFINITY;
      x[2] = v1 ? sacc[nt][2] * scale_log2 : -INFINITY;
      x[3] = v1 ? sacc[nt][3] * scale_log2 : -INFINITY;
      float p[4];
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float mx = fmaxf(x[e], x[2 + e]);
        mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 4));
        mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 8));
        mx = fmaxf(mx, __shfl_xor_sync(0xFFFFFFFFu, mx, 16));
        const float m_new = fmaxf(m_run[nt][e], mx);
        const float m_use = (m_new == -INFINITY) ? 0.f : m_new;
        const float alpha = exp2f(m_run[nt][e] - m_use);
        p[e] = exp2f(x[e] - m_use);
        p[2 + e] = exp2f(x[2 + e] - m_use);
        l_run[nt][e] = l_run[nt][e] * alpha + p[e] + p[2 + e];
        m_run[nt][e] = m_new;
        const float alpha_lo = __shfl_xor_sync(0xFFFFFFFFu, alpha, 2);
        const float alpha_acc = (pack && c >= 2) ? alpha_lo : alpha;
#pragma unroll
        for (int mt = 0; mt < KSTEPS; ++mt) {
          acc[mt][nt][e] *= alpha_acc;
          acc[mt][nt][2 + e] *= alpha_acc;
        }
      }
      // P^T as B fragments (tokens x heads) via an in-register 8x8 transpose
      const uint32_t h0 = pack_bf16x2(p[0], p[1]);
      const uint32_t h1 = pack_bf16x2(p[2], p[3]);
      const uint32_t l0 = pack_bf16x2(p[0] - bf16_bits_to_float(h0 & 0xFFFFu), p[1] - bf16_bits_to_float(h0 >> 16));
      const uint32_t l1 = pack_bf16x2(p[2] - bf16_bits_to_float(h1 & 0xFFFFu), p[3] - bf16_bits_to_float(h1 >> 16));
      if (pack) {
        const uint32_t x0 = __shfl_xor_sync(0xFFFFFFFFu, l0, 2), x1 = __shfl_xor_sync(0xFFFFFFFFu, l1, 2);
        bhi[nt][0] = movmatrix_trans(c < 2 ? h0 : x0);
        bhi[nt][1] = movmatrix_trans(c < 2 ? h1 : x1);
      } else {
        bhi[nt][0] = movmatrix_trans(h0);
        bhi[nt][1] = movmatrix_trans(h1);
        blo[nt][0] = movmatrix_trans(l0);
        blo[nt][1] = movmatrix_trans(l1);
      }
    }
    // ---- O^T += V_sub^T . P^T
    {
      const int tin = (lane & 7) + (lane >> 4) * 8;
#pragma unroll
      for (int mt = 0; mt < KSTEPS; ++mt) {
        const int ch = 2 * mt + ((lane >> 3) & 1);
        uint32_t vf[4];
        ldmatrix_x4_trans(vf, vbuf + (tin * CPR + (ch ^ (tin & 7))) * 16);
#pragma unroll
        for (int nt = 0; nt < NTILE; ++nt) {
          mma_bf16_16816(acc[mt][nt], vf, bhi[nt][0], bhi[nt][1]);
          if (!pack) mma_bf16_16816(acc[mt][nt], vf, blo[nt][0], blo[nt][1]);
        }
      }
    }
    __syncwarp();
  }
  cp_async_wait<0>();
  if (pack) {  // the lo parts' accumulators (columns 4-7) onto the hi parts' (columns 0-3)
#pragma unroll
    for (int mt = 0; mt < KSTEPS; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][0][e] += __shfl_xor_sync(0xFFFFFFFFu, acc[mt][0][e], 2);
  }

  // ---- merge the 4 warps' states in shared memory
#pragma unroll
  for (int nt = 0; nt < NTILE; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      float l = l_run[nt][e];
      l += __shfl_xor_sync(0xFFFFFFFFu, l, 4);
      l += __shfl_xor_sync(0xFFFFFFFFu, l, 8);
      l += __shfl_xor_sync(0xFFFFFFFFu, l, 16);
      l_run[nt][e] = l;
    }
  __syncthreads();  // ring no longer needed
  float* o_w = reinterpret_cast<float*>(smem_raw);           // [warps][16 heads][D]
  float* m_w = o_w + kAttnWarps * 16 * D;                     // [groups][16]
  float* l_w = m_w + kAttnWarps * 16;                         // [groups][16]
#pragma unroll
  for (int nt = 0; nt < NTILE && streams; ++nt) {
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int head = nt * 8 + 2 * c + e;
      if (g == 0 && hf == 0) {  // both halves hold the same softmax state
        m_w[grp * 16 + head] = m_run[nt][e];
        l_w[grp * 16 + head] = l_run[nt][e];
      }
#pragma unroll
      for (int mt = 0; mt < KSTEPS; ++mt) {
        o_w[(grp * 16 + head) * D + hf * DW + mt * 16 + g] = acc[mt][nt][e];
        o_w[(grp * 16 + head) * D + hf * DW + mt * 16 + g + 8] = acc[mt][nt][2 + e];
      }
    }
  }
  __syncthreads();
  for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
    const int head = i / D, dim = i % D;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kAttnWarps; ++w) M = fmaxf(M, m_w[w * 16 + head]);
    float o = 0.f, lse = -INFINITY;
    if (M != -INFINITY) {
      float L = 0.f;
#pragma unroll
      for (int w = 0; w < kAttnWarps; ++w) {
        const float sc = exp2f(m_w[w * 16 + head] - M);
        L += l_w[w * 16 + head] * sc;
        o += o_w[(w * 16 + head) * D + dim] * sc;
      }
      o /= L;
      lse = (M + log2f(L)) * kLn2;
    }
    if (in_cluster) {
      pbuf[i] = o;
      if (dim == 0) plse[head] = lse;
    } else {
      a.part_o[((hq0 + head) * a.S + split) * D + dim] = o;
      if (dim == 0) a.part_lse[(hq0 + head) * a.S + split] = lse;
    }
  }
  if (in_cluster) {
    __syncthreads();
    cluster_merge<D>(a, hq0, G, pbuf, plse);
    return;
  }
  finish_split<D>(a, row, hq0, G, reinterpret_cast<float*>(smem_raw));
}

}  // namespace jssa
