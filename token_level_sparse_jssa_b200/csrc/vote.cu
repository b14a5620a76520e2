// Head-shared soft voting: one index set for all KV heads of a sequence.
//
// "Joint Subspace Sparse Attention for Efficient Long-Context Decoding", §1 and §E.3 /
// Table 15: the variant that the per-KV-head selection is compared against.  The pages
// do not define the vote; the reading implemented: every KV head h turns its subspace
// scores over the candidates [0, T_b - W) into a distribution
//   p_h(t) = exp(c s_h(t) - m_h) / Z_h,   c = sm_scale / G,
// m_h = max_t c s_h(t), Z_h = sum_t exp(c s_h(t) - m_h), the distributions are summed over
// the KV heads, v(t) = sum_h p_h(t), and the top-k of v (ties to the lower index, output
// ascending) is copied to every KV head's row of the index list.
//
// Kernels (after the score scan has written the fp32 scores of every (b, h) row):
//   vote_stats_kernel   — grid (8 slices, b * Hkv + h): the slice's max logit and fp64 sum
//                         of the fp32 exponentials relative to it;
//   vote_combine_kernel — grid (token blocks, b): merges the slices into m_h and Z_h, then
//                         v(t) for every candidate, written over the score row of KV head 0
//                         (the thread that reads s_0(t) writes v(t));
//   then the standalone top-k over the B vote rows, and
//   vote_broadcast_kernel — the B index sets copied to all B * Hkv rows.
#include <cfloat>

#include "common.cuh"
#include "launch.h"

namespace jssa {
namespace {

constexpr int kVoteThreads = 256;
constexpr int kVoteSlices = 8;   // CTAs per (b, h) row of the statistics
constexpr int kVoteMaxHkv = 64;  // KV heads merged in shared memory by the combine kernel
constexpr int kCombineThreads = 256;
constexpr int kCombineTok = 4;  // tokens per thread

__device__ __forceinline__ int64_t vote_candidates(const VoteArgs& a, int b, bool flag) {
  int64_t T = a.seq_lens[b];
  if (T < 0 || T > a.T_cap) {
    if (flag) flag_error(a.status, DEVFLAG_BAD_SEQ_LEN);
    T = T < 0 ? 0 : a.T_cap;
  }
  return T - min64(max64(a.window, 0), T);
}

__global__ void __launch_bounds__(kVoteThreads) vote_stats_kernel(VoteArgs a) {
  __shared__ float smax[kVoteThreads / 32];
  __shared__ double ssum[kVoteThreads / 32];
  const int row = blockIdx.y, b = row / a.Hkv;
  const int64_t n_all = vote_candidates(a, b, threadIdx.x == 0 && blockIdx.x == 0 && row % a.Hkv == 0);
  const int64_t lo = n_all * blockIdx.x / kVoteSlices, n = n_all * (blockIdx.x + 1) / kVoteSlices - lo;
  const float* s = a.scores + static_cast<int64_t>(row) * a.sc_ld + lo;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  float m = -FLT_MAX;
  for (int64_t t = threadIdx.x; t < n; t += kVoteThreads) m = fmaxf(m, a.c * s[t]);
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
  if (lane == 0) smax[warp] = m;
  __syncthreads();
  m = smax[0];
  for (int w = 1; w < kVoteThreads / 32; ++w) m = fmaxf(m, smax[w]);
  double z = 0.0;
  for (int64_t t = threadIdx.x; t < n; t += kVoteThreads) z += static_cast<double>(expf(a.c * s[t] - m));
  for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xFFFFFFFFu, z, off);
  if (lane == 0) ssum[warp] = z;
  __syncthreads();
  if (threadIdx.x == 0) {
    double t = 0.0;
    for (int w = 0; w < kVoteThreads / 32; ++w) t += ssum[w];
    a.stats[2 * (row * kVoteSlices + blockIdx.x)] = static_cast<double>(m);
    a.stats[2 * (row * kVoteSlices + blockIdx.x) + 1] = t;
  }
}

__global__ void __launch_bounds__(kCombineThreads) vote_combine_kernel(VoteArgs a) {
  __shared__ float mh[kVoteMaxHkv], invz[kVoteMaxHkv];
  const int b = blockIdx.y;
  const int64_t n = vote_candidates(a, b, false);
  // merge the slices of each head: m = max m_i, Z = sum_i Z_i exp(m_i - m) (slices in order)
  for (int h = threadIdx.x; h < a.Hkv; h += blockDim.x) {
    const double* st = a.stats + 2 * static_cast<int64_t>(b * a.Hkv + h) * kVoteSlices;
    float m = -FLT_MAX;
    for (int i = 0; i < kVoteSlices; ++i) m = fmaxf(m, static_cast<float>(st[2 * i]));
    double Z = 0.0;
    for (int i = 0; i < kVoteSlices; ++i)
      if (st[2 * i + 1] > 0.0) Z += st[2 * i + 1] * static_cast<double>(expf(static_cast<float>(st[2 * i]) - m));
    mh[h] = m;
    invz[h] = Z > 0.0 ? static_cast<float>(1.0 / Z) : 0.f;
  }
  __syncthreads();
  const int64_t t0 = (static_cast<int64_t>(blockIdx.x) * kCombineThreads + threadIdx.x) * kCombineTok;
  if (t0 >= n) return;
  float v[kCombineTok] = {0.f, 0.f, 0.f, 0.f};
  float* s0 = a.scores + static_cast<int64_t>(b) * a.Hkv * a.sc_ld;
  for (int h = 0; h < a.Hkv; ++h) {
    const float m = mh[h], inv = invz[h];
    const float* s = s0 + static_cast<int64_t>(h) * a.sc_ld;
#pragma unroll
    for (int j = 0; j < kCombineTok; ++j)
      if (t0 + j < n) v[j] += expf(a.c * s[t0 + j] - m) * inv;
  }
#pragma unroll
  for (int j = 0; j < kCombineTok; ++j)
    if (t0 + j < n) s0[t0 + j] = v[j];
}

__global__ void vote_broadcast_kernel(VoteArgs a) {
  const int b = blockIdx.x;
  const int32_t* src = a.idx_shared + static_cast<int64_t>(b) * a.k;
  for (int h = 0; h < a.Hkv; ++h) {
    int32_t* dst = a.idx + (static_cast<int64_t>(b) * a.Hkv + h) * a.k;
    for (int j = threadIdx.x; j < a.k; j += blockDim.x) dst[j] = src[j];
    if (threadIdx.x == 0) a.n_sel[b * a.Hkv + h] = a.nsel_shared[b];
  }
}

}  // namespace

cudaError_t launch_vote_stats(const VoteArgs& a, cudaStream_t s) {
  if (a.Hkv > kVoteMaxHkv) return cudaErrorInvalidValue;
  vote_stats_kernel<<<dim3(kVoteSlices, a.B * a.Hkv), kVoteThreads, 0, s>>>(a);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t per_cta = static_cast<int64_t>(kCombineThreads) * kCombineTok;
  const dim3 grid(static_cast<unsigned>(ceil_div(a.T_cap, per_cta)), static_cast<unsigned>(a.B));
  vote_combine_kernel<<<grid, kCombineThreads, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_vote_broadcast(const VoteArgs& a, cudaStream_t s) {
  vote_broadcast_kernel<<<a.B, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace jssa
