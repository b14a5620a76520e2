// Gather-free indexed flash-decode (GQA) with split-T partials, and their LSE merge.
//
// "Joint Subspace Sparse Attention for Efficient Long-Context Decoding", §3.3: one
// launch per layer handles distinct per-KV-head index sets and reads the selected
// K/V entries in place from the standard GQA cache layout, with no gather buffer and
// no per-head launches; §2.2 / §4.7: gathering first would cost about as much as the
// reduced attention itself.  The same kernel with a contiguous range instead of an
// index list is the dense full-KV decode used as the baseline (§4.5).
//
// Grid: (split, sequence * KV head).  Each CTA owns one contiguous slice of the
// attended list (selected positions followed by the sliding window).  Its 4 warp groups
// take 16-token subtiles in turn (a group is one warp, or for d = 256 a pair of warps
// that each take half of the head dims and add their score partials through shared
// memory); each warp streams its part of the subtile's K and V rows with 16-byte cp.async
// copies (XOR-swizzled in shared memory) through a private multi-stage ring, so no block
// barrier sits in the main loop.  All G query heads of the group stay in registers as MMA
// operands:
//   S^T[16 tok x 8 heads] = K_sub[16 x d] . Q^T         (mma.sync m16n8k16, bf16 -> fp32,
//                                                        even and odd K-steps in two chains)
//   online softmax per head in fp32 (exp2 domain)
//   O^T[d x 8 heads]     += V_sub^T . P^T               (P split into bf16 hi + lo parts,
//                                                        so the weights keep ~16 bits; with at
//                                                        most 4 heads both parts share one MMA,
//                                                        the lo parts in columns 4-7)
// The 4 groups' states are merged in shared memory into one normalised partial (o, lse)
// per query head.  Indexed attention, and the dense decode when it uses at most 8 splits (a
// short window), runs the splits of a row as one thread-block cluster and combines the
// partials by log-sum-exp through distributed shared memory; the dense decode with more
// splits writes partials to the workspace and the last CTA of each row to finish (a per-row
// arrival counter) combines them.
#include "attn_core.cuh"

namespace jssa {

template <int D, bool DENSE>
static size_t attn_smem_bytes() {
  return AttnCfg<D>::MAIN_BYTES + (DENSE ? 0 : kMaxTokList * sizeof(int32_t));
}

template <int D, int NTILE, bool DENSE>
__global__ void __launch_bounds__(AttnCfg<D>::THREADS) attn_kernel(AttnArgs a) {
  using Cfg = AttnCfg<D>;
  constexpr int KSTEPS = Cfg::DW / 16;  // Q fragments of this warp's head dims
  constexpr int NT = Cfg::THREADS;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  int32_t* tok_s = reinterpret_cast<int32_t*>(smem_raw + Cfg::MAIN_BYTES);

  const int split = blockIdx.x, row = blockIdx.y;
  const int b = row / a.Hkv, h = row % a.Hkv;
  const int G = a.Hq / a.Hkv;
  const int64_t hq0 = static_cast<int64_t>(b) * a.Hq + static_cast<int64_t>(h) * G;
  const int64_t my_lo = static_cast<int64_t>(split) * a.split_len;
  // Issue every independent load of the prologue before using any of them: the sequence
  // length, the selection count, this split's index entries (speculatively, validated
  // below) and the query fragments.
  int64_t T = a.seq_lens[b];
  int64_t nsel = DENSE ? 0 : a.n_sel[row];
  constexpr int kPre = 4;  // index entries per thread loaded up front (4 x block size tokens)
  int32_t pre[kPre];
  if (!DENSE) {
    const int32_t* irow = a.idx + static_cast<int64_t>(row) * a.idx_ld;
#pragma unroll
    for (int u = 0; u < kPre; ++u) {
      const int64_t pos = my_lo + threadIdx.x + u * NT;
      pre[u] = (threadIdx.x + u * NT < a.split_len && pos < a.idx_ld) ? __ldg(irow + pos) : -1;
    }
  }
  uint32_t qf[NTILE][KSTEPS][2];
  load_q_frags<D, NTILE, KSTEPS>(a.Q, hq0, G, qf, ((threadIdx.x >> 5) / kAttnWarps % Cfg::HALVES) * Cfg::DW);
  if (T < 0 || T > a.T_cap) {
    if (split == 0 && threadIdx.x == 0) flag_error(a.status, DEVFLAG_BAD_SEQ_LEN);
    T = T < 0 ? 0 : a.T_cap;
  }
  int64_t list_len, win_start;
  if (DENSE) {
    win_start = (a.window > 0) ? max64(0, T - a.window) : 0;
    list_len = T - win_start;
  } else {
    const int64_t Wc = min64(max64(a.window, 0), T);
    win_start = T - Wc;
    const int64_t nsel_max = min64(a.idx_ld, win_start);
    if (nsel < 0 || nsel > nsel_max) {
      if (split == 0 && threadIdx.x == 0) flag_error(a.status, DEVFLAG_BAD_NSEL);
      nsel = nsel < 0 ? 0 : nsel_max;
    }
    list_len = nsel + Wc;
  }
  const int my_len = static_cast<int>(max64(0, min64(list_len, my_lo + a.split_len) - my_lo));

  float* pbuf = reinterpret_cast<float*>(smem_raw + Cfg::COMBINE_BYTES);   // [16][D] (cluster merge)
  float* plse = pbuf + 16 * D;                                              // [16]
  if (my_len == 0) {  // empty split: weight zero in the merge
    if (!DENSE || a.cluster_merge) {
      for (int i = threadIdx.x; i < G * D; i += NT) pbuf[i] = 0.f;
      if (threadIdx.x < G) plse[threadIdx.x] = -INFINITY;
      cluster_merge<D>(a, hq0, G, pbuf, plse);
    } else {
      for (int i = threadIdx.x; i < G * D; i += NT) {
        const int head = i / D, dim = i % D;
        a.part_o[((hq0 + head) * a.S + split) * D + dim] = 0.f;
        if (dim == 0) a.part_lse[(hq0 + head) * a.S + split] = -INFINITY;
      }
      finish_split<D>(a, row, hq0, G, reinterpret_cast<float*>(smem_raw));
    }
    return;
  }
  if (!DENSE) {
    const int32_t* irow = a.idx + static_cast<int64_t>(row) * a.idx_ld;
    auto resolve = [&](int j, int64_t t) {  // selected entry (validated) or window position
      const int64_t pos = my_lo + j;
      if (pos < nsel) {
        if (t < 0 || t >= win_start) {
          flag_error(a.status, DEVFLAG_BAD_INDEX);
          t = -1;
        }
      } else {
        t = win_start + (pos - nsel);
      }
      tok_s[j] = static_cast<int32_t>(t);
    };
#pragma unroll
    for (int u = 0; u < kPre; ++u) {
      const int j = threadIdx.x + u * NT;
      if (j < my_len) resolve(j, pre[u]);
    }
    for (int j = threadIdx.x + kPre * NT; j < my_len; j += NT)
      resolve(j, (my_lo + j < nsel) ? irow[my_lo + j] : 0);
    __syncthreads();
  }

  attn_core<D, NTILE, DENSE>(a, row, split, b, h, G, hq0, qf, DENSE ? nullptr : tok_s, win_start, my_lo, my_len,
                             smem_raw);
}

// ------------------------------------------------------------------ host side
void attn_split_policy(bool indexed, int rows, int64_t list_max, int num_sms, int d, int* S_out,
                       int* split_out) {
  // Choose the split length (a multiple of the 16-token subtile, at least 64 tokens) that
  // keeps the last wave of CTAs fullest; fewer splits win ties.
  const int min_split = 64;
  if (list_max <= 0) { *S_out = 1; *split_out = min_split; return; }
  if (d >= 256) {
    // One resident CTA per SM (the eight-warp ring takes 208 KB), and a fixed cost per CTA
    // (prologue, ring fill, merge) worth about 256 tokens of streaming: minimise
    // waves x (1 + len / 256), fewer splits on ties.
    const int cap = indexed ? 8 : 256;
    int best_S = 1;
    int64_t best_len = ceil_div(list_max, 16) * 16;
    double best_cost = 1e300;
    for (int S = 1; S <= cap; ++S) {
      int64_t len = ceil_div(ceil_div(list_max, S), 16) * 16;
      if (len < min_split) len = min_split;
      if (ceil_div(list_max, len) != S) continue;
      if (indexed && len > kMaxTokList) continue;  // the token list lives in shared memory
      const int64_t waves = ceil_div(static_cast<int64_t>(rows) * S, num_sms);
      const double cost = static_cast<double>(waves) * (1.0 + static_cast<double>(len) / 256.0);
      if (cost < best_cost - 1e-9) { best_cost = cost; best_S = S; best_len = len; }
    }
    *S_out = best_S;
    *split_out = static_cast<int>(best_len);
    return;
  }
  const int slots = num_sms * 2;  // two resident CTAs per SM (at most 112 KB of shared memory each)
  int best_S = 0;
  int64_t best_len = 0;
  double best_eff = -1.0;
  for (int S = 1; S <= 256; ++S) {
    int64_t len = ceil_div(ceil_div(list_max, S), 16) * 16;
    if (len < min_split) len = min_split;
    const int64_t Sr = ceil_div(list_max, len);
    if (Sr != S) continue;
    if (indexed && len > kMaxTokList) continue;  // the token list lives in shared memory
    if (indexed && S > 8) break;                 // one cluster per row
    const int64_t ctas = static_cast<int64_t>(rows) * Sr;
    const int64_t waves = ceil_div(ctas, slots);
    const double eff = static_cast<double>(ctas) / static_cast<double>(waves * slots);
    if (eff > best_eff + 0.02) { best_eff = eff; best_S = S; best_len = len; }
  }
  if (best_S == 0) {  // only reachable for very long lists
    const int cap = indexed ? 8 : 256;
    best_len = ceil_div(ceil_div(list_max, cap), 16) * 16;
    best_S = static_cast<int>(ceil_div(list_max, best_len));
  }
  *S_out = best_S;
  *split_out = static_cast<int>(best_len);
}

template <int D, int NTILE, bool DENSE>
static cudaError_t launch_attn_t(const AttnArgs& a, cudaStream_t s) {
  const size_t smem = attn_smem_bytes<D, DENSE>();
  static int done[64] = {0};
  cudaError_t e = set_smem_limit_once(attn_kernel<D, NTILE, DENSE>, smem, done);
  if (e != cudaSuccess) return e;
  // indexed, and dense with at most 8 splits: the S splits of a row form one cluster and
  // merge through distributed shared memory; dense with more splits merges through the
  // workspace (the row's last CTA to finish)
  AttnArgs c = a;
  c.cluster_merge = (!DENSE || a.S <= 8) ? 1 : 0;
  return launch_ex(attn_kernel<D, NTILE, DENSE>, dim3(a.S, a.B * a.Hkv), dim3(AttnCfg<D>::THREADS), smem, s,
                   c.cluster_merge ? a.S : 0, c);
}

template <int D, bool DENSE>
static cudaError_t launch_attn_d(const AttnArgs& a, cudaStream_t s) {
  const int G = a.Hq / a.Hkv;
  return (G <= 8) ? launch_attn_t<D, 1, DENSE>(a, s) : launch_attn_t<D, 2, DENSE>(a, s);
}

cudaError_t launch_attention(const AttnArgs& a, cudaStream_t s) {
  const bool dense = (a.idx == nullptr);
  if (!dense && (a.split_len > kMaxTokList || a.S > 8)) return cudaErrorNotSupported;
  switch (a.dk) {
    case 64: return dense ? launch_attn_d<64, true>(a, s) : launch_attn_d<64, false>(a, s);
    case 128: return dense ? launch_attn_d<128, true>(a, s) : launch_attn_d<128, false>(a, s);
    case 256: return dense ? launch_attn_d<256, true>(a, s) : launch_attn_d<256, false>(a, s);
    default: return cudaErrorInvalidValue;
  }
}


}  // namespace jssa
