// MLA attention over many 128-token tiles per CTA on the fifth-generation tensor cores, with
// the split merge inside a thread-block cluster: one kernel for the indexed form (the selected
// tokens plus the sliding window) and for the dense form (the full-cache comparator).
//
// Joint Subspace Sparse Attention, §3.3 and §A.3 (MLA / latent caches: one 576-dim latent row
// per token, 512 latent dims followed by 64 RoPE dims; the 128 absorbed query heads form one
// group, the logit of head h for token t is sm_scale * q_h . C_t over all 576 dims and the
// value is C_t[:512]); §4.5 (the full-KV decode the method is compared against).
//
// Work split: grid (G, 2, B).  CTA (g, hh, b) takes token group g of the attended list of
// sequence b (contiguous positions of the list) for query heads [64 hh, 64 hh + 64); the G
// groups of one (b, hh) form a cluster.  Per tile of 128 attended tokens, in the transposed
// orientation so that both MMAs have M = 128:
//   S^T  = C_tile . Q_hh^T    M = 128 tokens, N = 64 heads, K = 576 (9 K-blocks of 64 dims)
//   O^T += V_tile^T . P^T     M = 128 dims (4 blocks cover 512), N = 64 heads, K = 128 tokens
// TMEM (512 columns): S^T in [0, 64), O^T in [256, 512) (dims block j at 256 + 64 j); O^T stays
// resident over the CTA's tiles.  The latent tile (128-byte swizzled, 147 KB) is the K-major A
// operand of the score MMA and the MN-major A operand of the value MMA; the query streams
// through a four-stage ring; P^T (bf16 hi + lo parts, rows = tokens) is the MN-major B
// operand of the value MMA, whose MMAs take the four dims blocks' accumulators in turn.  The
// next tile's cache rows are resolved, and prefetched into L2 line by line, while a tile runs.
// Softmax over S^T: one thread per (token, 32 heads); the running maximum of a head moves only
// when a tile brings a logit more than 2^8 above it (then the resident O^T columns and the
// sums are rescaled), so most tiles need no reduction across threads.
// After the last tile each CTA pushes its lse of every head to all CTAs of the cluster, writes
// its normalised partial o into shared memory, and the cluster merges the G partials of every
// output element over distributed shared memory with per-head weights formed once.
// Every wait is bounded; on a timeout the kernel raises DEVFLAG_TIMEOUT, stops issuing, writes
// an empty partial, drains its copies and MMAs, and frees its tensor memory.
#include <cooperative_groups.h>

#include "common.cuh"
#include "launch.h"
#include "tcgen05.cuh"

namespace cg = cooperative_groups;

namespace jssa {
namespace {

constexpr int kSpHeads = 64;                 // query heads per CTA
constexpr int kSpTile = 128;                 // tokens per tile
constexpr int kSpDk = 576, kSpDv = 512;
constexpr int kSpKB = kSpDk / 64;            // K-blocks of the score MMA
constexpr int kSpThreads = 256;
constexpr int kSpBlkC = 128 * 128;           // latent block: 128 tokens x 64 dims (16 KB)
constexpr int kSpBlkQ = kSpHeads * 128;      // query block: 64 heads x 64 dims (8 KB)
constexpr int kSpQStages = 4;
constexpr int kSpBlkP = kSpTile * 128;       // P^T: 128 tokens x 64 heads (16 KB), hi then lo
constexpr int kSpCBytes = kSpKB * kSpBlkC;
constexpr int kSpSmem = kSpCBytes + kSpQStages * kSpBlkQ + 2 * kSpBlkP + 1024;
constexpr int kSpMaxCluster = 8;
constexpr uint32_t kSpTmemCols = 512;
constexpr uint32_t kSpOCol = 256;            // first TMEM column of O^T
constexpr float kSpRescale = 8.f;            // log2 margin before the running maximum moves

static_assert(kSpHeads * kSpDv * 4 <= kSpCBytes, "the normalised partial reuses the latent tile");

// cp.async groups that may still be pending when the score MMA of K-block kb is issued: one
// group per latent block (query blocks 0-2 ride in the first three) and, while kb < 6, one for
// query block kb + 3.
__device__ __forceinline__ void sp_wait_groups(int kb) {
  switch (kb) {
    case 0: case 1: case 2: cp_async_wait<8>(); break;
    case 3: case 4: case 5: case 6: cp_async_wait<2>(); break;
    case 7: cp_async_wait<1>(); break;
    default: cp_async_wait<0>(); break;
  }
}

__device__ __forceinline__ void cluster_arrive_relaxed() { asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }

// Bring the 128-byte line at `p` into L2.
__device__ __forceinline__ void prefetch_l2_line(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

template <bool DENSE>
__global__ void __launch_bounds__(kSpThreads, 1) mla_split_kernel(AttnArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ int32_t tok_s[2][kSpTile];               // cache rows of this tile and the next
  __shared__ __align__(8) uint64_t bars[kSpKB + 1];  // [kb]: score MMAs through block kb; [9]: value MMAs
  __shared__ uint32_t tmem_base_s;
  __shared__ float m_s[kSpHeads];                     // running maximum per head (log2 units)
  __shared__ float alpha_s[kSpHeads];
  __shared__ float red_s[4][kSpHeads];                // per TMEM lane quadrant: tile maxima, then sums
  __shared__ __align__(16) float invl_s[kSpHeads];
  __shared__ float lse_all[kSpMaxCluster][kSpHeads];  // every CTA's lse, pushed before the merge
  __shared__ float w_s[kSpMaxCluster][kSpHeads];      // merge weight of each partial per head

  cg::cluster_group cluster = cg::this_cluster();
  const int G = static_cast<int>(cluster.num_blocks());
  const int g = static_cast<int>(cluster.block_rank());
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int quad = warp & 3, hw = warp >> 2;  // TMEM lane quadrant; which 32 of the 64 heads
  const int hh = blockIdx.y, b = blockIdx.z;
  const int64_t qrow0 = static_cast<int64_t>(b) * a.Hq + kSpHeads * hh;  // first (b, head) row of Q and O

  // ---- this CTA's range of the attended list
  int64_t T = a.seq_lens[b];
  if (T < 0 || T > a.T_cap) {
    if (g == 0 && hh == 0 && tid == 0) flag_error(a.status, DEVFLAG_BAD_SEQ_LEN);
    T = T < 0 ? 0 : a.T_cap;
  }
  int64_t win_start, nsel = 0, list_len;
  if (DENSE) {
    win_start = (a.window > 0) ? max64(0, T - a.window) : 0;
    list_len = T - win_start;
  } else {
    const int64_t Wc = min64(max64(a.window, 0), T);
    win_start = T - Wc;
    nsel = a.n_sel[b];
    const int64_t nsel_max = min64(a.idx_ld, win_start);
    if (nsel < 0 || nsel > nsel_max) {
      if (g == 0 && hh == 0 && tid == 0) flag_error(a.status, DEVFLAG_BAD_NSEL);
      nsel = nsel < 0 ? 0 : nsel_max;
    }
    list_len = nsel + Wc;
  }
  const int64_t my_lo = static_cast<int64_t>(g) * a.split_len;
  const int64_t my_len = max64(0, min64(list_len, my_lo + a.split_len) - my_lo);
  const int ntiles = static_cast<int>(ceil_div(my_len, kSpTile));
  auto token_at = [&](int64_t pos) -> int64_t {  // list position -> cache row (or -1)
    if (pos < 0 || pos >= list_len) return -1;
    if (DENSE || pos >= nsel) return win_start + (DENSE ? pos : pos - nsel);
    const int64_t t = a.idx[static_cast<int64_t>(b) * a.idx_ld + pos];
    if (t < 0 || t >= win_start) {
      flag_error(a.status, DEVFLAG_BAD_INDEX);
      return -1;
    }
    return t;
  };

  if (tid == 0) {
    for (int i = 0; i <= kSpKB; ++i) mbar_init(&bars[i], 1);
    fence_mbarrier_init();
  }
  if (tid < kSpHeads) m_s[tid] = -INFINITY;
  if (warp == 0) tmem_alloc(&tmem_base_s, kSpTmemCols);
  cluster_arrive_relaxed();  // matched by the wait before the first access to a peer's shared memory
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;

  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t c_s = base;                              // latent tile: 9 blocks [128 tokens][64 dims]
  const uint32_t q_s = base + kSpCBytes;                  // query ring: 4 blocks [64 heads][64 dims]
  const uint32_t p_s = q_s + kSpQStages * kSpBlkQ;        // P^T hi, lo: [128 tokens][64 heads] each
  float* ob = reinterpret_cast<float*>(smem_raw + (base - raw));   // after the last tile: [64 heads][512]
  const __nv_bfloat16* Cb = static_cast<const __nv_bfloat16*>(a.K) + static_cast<int64_t>(b) * a.ks[0];
  const __nv_bfloat16* Qb = static_cast<const __nv_bfloat16*>(a.Q) + qrow0 * kSpDk;
  const uint64_t pol_c = l2_policy_evict_first(), pol_q = l2_policy_evict_last();
  const int ch = tid & 7, r0 = tid >> 3;
  const int t_lane = quad * 32 + lane;                    // this thread's token row of S^T
  const uint32_t trow = tmem + (static_cast<uint32_t>(quad * 32) << 16);
  const uint32_t idesc_s = instr_desc(128, kSpHeads, false, false);
  const uint32_t idesc_v = instr_desc(128, kSpHeads, true, true);
  const float scale = a.sm_scale * 1.4426950408889634f;   // logits in log2 units

  float l_part[32];  // this thread's share of the softmax sums of its 32 heads
#pragma unroll
  for (int i = 0; i < 32; ++i) l_part[i] = 0.f;
  bool dead = false;
  int last_commit = -1;
  uint32_t par = 0;  // phase parity of the per-tile barriers

  // cache row of list position pos of this CTA's range (-1 past it)
  auto row_at = [&](int64_t pos) -> int32_t {
    return (pos < my_lo + my_len) ? static_cast<int32_t>(token_at(pos)) : -1;
  };
  if (ntiles > 0 && tid < kSpTile) tok_s[0][tid] = row_at(my_lo + tid);

  for (int tile = 0; tile < ntiles && !dead; ++tile, par ^= 1u) {
    const int64_t pos0 = my_lo + static_cast<int64_t>(tile) * kSpTile;
    const int tlen = static_cast<int>(min64(kSpTile, my_lo + my_len - pos0));
    const int32_t* tok = tok_s[tile & 1];
    // this thread's row of the next tile: loaded now, stored once this tile's copies are issued
    const int32_t next_row = (tid < kSpTile && tile + 1 < ntiles) ? row_at(pos0 + kSpTile + tid) : -1;
    __syncthreads();
    const int N = (tlen + 15) & ~15;  // K extent of the value MMA

    // ---- every latent load of the tile and the first three query blocks
    const __nv_bfloat16* src_c[4];
    uint32_t bytes_c[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int32_t t = tok[r0 + 32 * u];
      src_c[u] = (t >= 0) ? Cb + static_cast<int64_t>(t) * a.ks[2] + ch * 8 : Cb;
      bytes_c[u] = (t >= 0) ? 16u : 0u;  // masked rows are zero-filled
    }
#pragma unroll
    for (int kb = 0; kb < kSpKB; ++kb) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int j = r0 + 32 * u;
        cp_async16_hint(c_s + kb * kSpBlkC + sw128(j, ch), src_c[u] + (bytes_c[u] ? kb * 64 : 0), bytes_c[u], pol_c);
      }
      if (kb < kSpQStages - 1) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int hr = r0 + 32 * u;
          cp_async16_hint(q_s + kb * kSpBlkQ + sw128(hr, ch), Qb + hr * kSpDk + kb * 64 + ch * 8, 16u, pol_q);
        }
      }
      cp_async_commit();
    }
    // the next tile's rows: into tok_s (the other buffer, free since the previous tile) and L2
    if (tid < kSpTile && tile + 1 < ntiles) {
      tok_s[(tile + 1) & 1][tid] = next_row;
      // one head half prefetches each row, a line at a time (the plain prefetch is issued by the
      // load unit; bulk prefetches of whole rows queue on the copy engine behind one another)
      if (next_row >= 0 && (tid >> 6) == hh) {
        const char* rp = reinterpret_cast<const char*>(Cb + static_cast<int64_t>(next_row) * a.ks[2]);
#pragma unroll
        for (int l = 0; l < kSpDk * 2 / 128; ++l) prefetch_l2_line(rp + l * 128);
      }
    }

    // ---- S^T over the 9 K-blocks, the query ring refilled behind it
#pragma unroll
    for (int kb = 0; kb < kSpKB; ++kb) {
      sp_wait_groups(kb);
      fence_async_smem();
      dead = __syncthreads_or(dead) != 0;
      if (tid == 0 && !dead) {
        tc_fence_after();
        const uint32_t qa = q_s + (kb % kSpQStages) * kSpBlkQ, ca = c_s + kb * kSpBlkC;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16(tmem, smem_desc(ca + kk * 32, 16, 1024), smem_desc(qa + kk * 32, 16, 1024), idesc_s,
                    (kb | kk) != 0 ? 1u : 0u);
        umma_commit(&bars[kb]);
        last_commit = kb;
      }
      if (kb + kSpQStages - 1 < kSpKB) {
        // query block kb+3 goes to the stage of block kb-1: wait for that block's MMAs
        if (kb >= 1 && !dead && !mbar_wait_bounded(&bars[kb - 1], par, a.status)) dead = true;
        if (!dead) {
          const int nb = kb + kSpQStages - 1;
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int hr = r0 + 32 * u;
            cp_async16_hint(q_s + (nb % kSpQStages) * kSpBlkQ + sw128(hr, ch), Qb + hr * kSpDk + nb * 64 + ch * 8,
                            16u, pol_q);
          }
        }
        cp_async_commit();  // also when dead: keeps the group count of every thread in step
      }
    }
    if (!dead && !mbar_wait_bounded(&bars[kSpKB - 1], par, a.status)) dead = true;
    tc_fence_after();
    dead = __syncthreads_or(dead) != 0;
    if (dead) break;

    // ---- softmax of this thread's token over its 32 heads
    float x[32];
    tmem_ld32(trow + hw * 32, x);
    const bool valid = t_lane < tlen && tok[t_lane] >= 0;
    bool big = false;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      x[i] = valid ? x[i] * scale : -INFINITY;
      big |= x[i] > m_s[hw * 32 + i] + kSpRescale;
    }
    if (__syncthreads_or(big)) {
      // the running maxima move: this tile's maximum of every head, then the rescale
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        float v = x[i];
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, off));
        if (lane == 0) red_s[quad][hw * 32 + i] = v;
      }
      __syncthreads();
      if (tid < kSpHeads) {
        const float mt = fmaxf(fmaxf(red_s[0][tid], red_s[1][tid]), fmaxf(red_s[2][tid], red_s[3][tid]));
        const float mo = m_s[tid];
        const float mn = fmaxf(mo, mt);
        alpha_s[tid] = (mo == -INFINITY) ? 0.f : exp2f(mo - mn);
        m_s[tid] = mn;
      }
      __syncthreads();
#pragma unroll
      for (int i = 0; i < 32; ++i) l_part[i] *= alpha_s[hw * 32 + i];
      if (tile > 0) {  // the resident O^T columns of this thread's heads (the value MMAs are done)
        tc_fence_after();
#pragma unroll 1
        for (int j = 0; j < 4; ++j) {
          float v[32];
          const uint32_t ta = trow + kSpOCol + 64 * j + hw * 32;
          tmem_ld32(ta, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] *= alpha_s[hw * 32 + i];
          tmem_st32(ta, v);
        }
      }
    }
    // P^T row of this token (bf16 hi in the first block, lo in the second)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i0 = c * 8 + 2 * e;
        const float m0 = m_s[hw * 32 + i0], m1 = m_s[hw * 32 + i0 + 1];
        const float p0 = (x[i0] == -INFINITY || m0 == -INFINITY) ? 0.f : exp2f(x[i0] - m0);
        const float p1 = (x[i0 + 1] == -INFINITY || m1 == -INFINITY) ? 0.f : exp2f(x[i0 + 1] - m1);
        l_part[i0] += p0;
        l_part[i0 + 1] += p1;
        const __nv_bfloat16 h0 = __float2bfloat16_rn(p0), h1 = __float2bfloat16_rn(p1);
        hi[e] = static_cast<uint32_t>(__bfloat16_as_ushort(h0)) | (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
        lo[e] = pack_bf16x2(p0 - __bfloat162float(h0), p1 - __bfloat162float(h1));
      }
      const uint32_t off = sw128(t_lane, hw * 4 + c);
      st_shared_v4(p_s + off, hi[0], hi[1], hi[2], hi[3]);
      st_shared_v4(p_s + kSpBlkP + off, lo[0], lo[1], lo[2], lo[3]);
    }
    fence_async_smem();
    tc_fence_before();
    __syncthreads();

    // ---- O^T += V^T . P^T (hi and lo parts), accumulated over the CTA's tiles
    if (tid == 0) {
      tc_fence_after();
      // the four dims blocks' accumulators take turns, so consecutive MMAs are independent
      for (int kt = 0; kt < N / 16; ++kt) {
#pragma unroll
        for (int pl = 0; pl < 2; ++pl) {
          const uint64_t bdesc = smem_desc(p_s + pl * kSpBlkP + kt * 2048, kSpBlkP, 1024);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint64_t adesc = smem_desc(c_s + (2 * j) * kSpBlkC + kt * 2048, kSpBlkC, 1024);
            umma_bf16(tmem + kSpOCol + 64 * j, adesc, bdesc, idesc_v, (tile > 0 || kt > 0 || pl > 0) ? 1u : 0u);
          }
        }
      }
      umma_commit(&bars[kSpKB]);
      last_commit = kSpKB;
    }
    if (!mbar_wait_bounded(&bars[kSpKB], par, a.status)) dead = true;
    tc_fence_after();
    dead = __syncthreads_or(dead) != 0;
  }

  // ---- this CTA's softmax sums per head (over its 128 token lanes), lse and 1 / sum
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    float v = l_part[i];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
    if (lane == 0) red_s[quad][hw * 32 + i] = v;
  }
  cp_async_wait<0>();
  if (tid == 0 && dead && last_commit >= 0) mbar_wait_bounded(&bars[last_commit], par, a.status);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  cluster_wait();  // every CTA of the cluster has started
  if (tid < kSpHeads) {
    const float L = red_s[0][tid] + red_s[1][tid] + red_s[2][tid] + red_s[3][tid];
    const float m = m_s[tid];
    const bool ok = !dead && ntiles > 0 && L > 0.f && m != -INFINITY;
    const float lse = ok ? (m + log2f(L)) * 0.6931471805599453f : -INFINITY;
    invl_s[tid] = ok ? 1.f / L : 0.f;
    for (int q = 0; q < G; ++q) cluster.map_shared_rank(&lse_all[0][0], q)[g * kSpHeads + tid] = lse;
  }
  __syncthreads();
  // normalised partial o[head][dim] into shared memory (the latent tile is free)
  if (!dead && ntiles > 0) {
    float il[32];
#pragma unroll
    for (int i = 0; i < 32; i += 4) {
      const float4 v4 = *reinterpret_cast<const float4*>(&invl_s[hw * 32 + i]);
      il[i] = v4.x, il[i + 1] = v4.y, il[i + 2] = v4.z, il[i + 3] = v4.w;
    }
#pragma unroll 1
    for (int j = 0; j < 4; ++j) {
      float v[32];
      tmem_ld32(trow + kSpOCol + 64 * j + hw * 32, v);
      const int d = 128 * j + quad * 32 + lane;
#pragma unroll
      for (int i = 0; i < 32; ++i) ob[(hw * 32 + i) * kSpDv + d] = v[i] * il[i];
    }
  } else {
    for (int i = tid; i < kSpHeads * kSpDv; i += kSpThreads) ob[i] = 0.f;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kSpTmemCols);
  }

  // ---- merge the G partials of the cluster: CTA g writes its share of the 64 x 512 outputs.
  // The weight of partial q for head h is exp(lse_q - M) / sum_q' exp(lse_q' - M), computed
  // once per head from the lse values every CTA pushed; the partial rows are then read over
  // distributed shared memory 16 bytes at a time, a batch of loads in flight before the first
  // is used.
  cluster.sync();
  if (tid < kSpHeads) {
    float l[kSpMaxCluster];
#pragma unroll
    for (int q = 0; q < kSpMaxCluster; ++q) l[q] = (q < G) ? lse_all[q][tid] : -INFINITY;
    float M = -INFINITY;
#pragma unroll
    for (int q = 0; q < kSpMaxCluster; ++q) M = fmaxf(M, l[q]);
    float L = 0.f;
#pragma unroll
    for (int q = 0; q < kSpMaxCluster; ++q) {
      l[q] = (M == -INFINITY) ? 0.f : expf(l[q] - M);
      L += l[q];
    }
#pragma unroll
    for (int q = 0; q < kSpMaxCluster; ++q) w_s[q][tid] = (L > 0.f) ? l[q] / L : 0.f;
    if (a.lse && g == 0) a.lse[qrow0 + tid] = (M == -INFINITY) ? -INFINITY : M + logf(L);
  }
  __syncthreads();
  constexpr int kVec = kSpHeads * kSpDv / 4;  // float4 elements of the output block
  const int per4 = (kVec + G - 1) / G;
  const int v_lo = g * per4, v_hi = min(kVec, v_lo + per4);
  const float4* obq[kSpMaxCluster];
#pragma unroll
  for (int q = 0; q < kSpMaxCluster; ++q)
    obq[q] = reinterpret_cast<const float4*>(cluster.map_shared_rank(ob, q < G ? q : 0));
  constexpr int kBatch = 2;
  const bool o_vec = (reinterpret_cast<uintptr_t>(a.O) & 15u) == 0;  // 16-byte stores (8 for bf16)
  for (int v0 = v_lo + tid; v0 < v_hi; v0 += kBatch * kSpThreads) {
    float4 x[kBatch][kSpMaxCluster];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int v = v0 + u * kSpThreads;
#pragma unroll
      for (int q = 0; q < kSpMaxCluster; ++q)
        x[u][q] = (q < G && v < v_hi) ? obq[q][v] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int v = v0 + u * kSpThreads;
      if (v >= v_hi) break;
      const int h = (v * 4) / kSpDv, d = (v * 4) % kSpDv;
      float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int q = 0; q < kSpMaxCluster; ++q) {
        const float wq = (q < G) ? w_s[q][h] : 0.f;
        o.x = fmaf(wq, x[u][q].x, o.x);
        o.y = fmaf(wq, x[u][q].y, o.y);
        o.z = fmaf(wq, x[u][q].z, o.z);
        o.w = fmaf(wq, x[u][q].w, o.w);
      }
      const int64_t off = (qrow0 + h) * kSpDv + d;
      if (a.out_bf16) {
        __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(a.O) + off;
        if (o_vec) {
          uint2 pk;
          pk.x = pack_bf16x2(o.x, o.y);
          pk.y = pack_bf16x2(o.z, o.w);
          *reinterpret_cast<uint2*>(dst) = pk;
        } else {
          dst[0] = __float2bfloat16_rn(o.x), dst[1] = __float2bfloat16_rn(o.y);
          dst[2] = __float2bfloat16_rn(o.z), dst[3] = __float2bfloat16_rn(o.w);
        }
      } else {
        float* dst = static_cast<float*>(a.O) + off;
        if (o_vec) *reinterpret_cast<float4*>(dst) = o;
        else dst[0] = o.x, dst[1] = o.y, dst[2] = o.z, dst[3] = o.w;
      }
    }
  }
  cluster.sync();  // the partials stay until every CTA has read them
}

}  // namespace

int mla_split_groups(int B, int num_sms) {
  // token groups per (sequence, head half): the largest cluster (up to 8) that keeps every
  // CTA resident at one per SM
  int G = num_sms / (2 * (B > 0 ? B : 1));
  return G < 1 ? 1 : (G > kSpMaxCluster ? kSpMaxCluster : G);
}

cudaError_t launch_mla_split(const AttnArgs& a, bool dense, cudaStream_t s) {
  if (a.Hkv != 1 || a.Hq != 2 * kSpHeads || a.dk != kSpDk || a.dv != kSpDv) return cudaErrorNotSupported;
  if (!dense && (a.idx == nullptr || a.n_sel == nullptr)) return cudaErrorInvalidValue;
  if (a.S < 1 || a.S > kSpMaxCluster || a.split_len < 1) return cudaErrorInvalidValue;
  auto kernel = dense ? mla_split_kernel<true> : mla_split_kernel<false>;
  static int done[2][64] = {{0}};
  cudaError_t e = set_smem_limit_once(kernel, kSpSmem, done[dense ? 1 : 0]);
  if (e != cudaSuccess) return e;
  return launch_ex(kernel, dim3(a.S, 2, a.B), dim3(kSpThreads), kSpSmem, s, a.S, a);
}

}  // namespace jssa
