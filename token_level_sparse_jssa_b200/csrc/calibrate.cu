// Spectral calibration of the scoring basis P, one basis per KV head.
//
// "Joint Subspace Sparse Attention for Efficient Long-Context Decoding", §3.2 (one
// orthonormal basis for queries and keys minimising the expected bilinear score error;
// a marginal upper bound with a closed-form spectral solution; the group-mean query; the
// query and key second moments each normalised to unit trace), §A.4 (a basis per layer
// and KV head from packed calibration sequences), §B.1-§B.3.  The closed form is not
// printed; the reading implemented here: P = the top-r eigenvectors of
//   M = S_q / tr S_q + S_k / tr S_k,
// S_q and S_k the uncentred second moments of the group-mean query and of the key over
// the calibration tokens (the 1/N factors cancel in the normalisation; a moment with zero
// trace contributes nothing).  Columns in descending eigenvalue order; each column's sign
// makes its largest-magnitude entry positive (the lowest index among equal magnitudes).
// A run that has not converged after the bounded number of sweeps raises the timeout bit
// of the status word.
//
// Two kernels:
//   moments_kernel — the two Gram matrices, fp64 throughout (bf16 inputs are exact in
//                    fp64 and so is the group mean for G <= 16): grid (upper-triangle 64x64
//                    tile pairs, token chunks, KV head x {query, key}); each CTA stages 32
//                    tokens at a time in shared memory, every thread accumulates a 4x4
//                    block, and the chunk's tile is added to the result with fp64 atomics.
//   jacobi_kernel  — one 8-CTA cluster per KV head diagonalises M by cyclic Jacobi in the
//                    round-robin parallel order: every round rotates d/2 disjoint index
//                    pairs at once.  The CTA owning a pair computes the new rows of that
//                    pair directly (each 2x2 block of the new matrix is R_ab^T B R_ef, so
//                    rows a and b of the old matrix and all the round's angles suffice),
//                    into the other buffer of a double-buffered matrix, and rotates the
//                    same two rows of the transposed eigenvector matrix in place.  One
//                    cluster barrier per round; the loop stops when the off-diagonal mass
//                    falls below 1e-12 of the (rotation-invariant) Frobenius norm, or
//                    after a bounded number of sweeps.
#include <cooperative_groups.h>

#include "common.cuh"
#include "launch.h"

namespace jssa {
namespace {

namespace cg = cooperative_groups;

constexpr int kMomTile = 64;      // tile edge of the d x d moments
constexpr int kMomThreads = 256;  // 16 x 16 threads, 4 x 4 entries each
constexpr int kMomSub = 32;       // tokens staged per step
constexpr int kMomChunk = 8192;   // tokens per CTA
constexpr int kJacCluster = 8;
constexpr int kJacThreads = 256;
constexpr int kJacMaxSweeps = 40;

__device__ __forceinline__ double bf16_bits_to_f64(uint32_t u16) {
  return static_cast<double>(__uint_as_float(u16 << 16));
}

// acc [Hkv][2][d][d]: sums over tokens of qbar qbar^T (slot 0) and k k^T (slot 1); only
// tiles (ti <= tj) are written.
__global__ void __launch_bounds__(kMomThreads) moments_kernel(CalibArgs a) {
  __shared__ double xi[kMomSub][kMomTile];
  __shared__ double xj[kMomSub][kMomTile];
  const int d = a.d, nt = d / kMomTile;
  // tile pair (ti <= tj) from the linear index
  int pid = blockIdx.x, ti = 0;
  while (pid >= nt - ti) { pid -= nt - ti; ++ti; }
  const int tj = ti + pid;
  const int which = blockIdx.z & 1, h = blockIdx.z >> 1;
  const int G = a.Hq / a.Hkv;
  const int64_t N = static_cast<int64_t>(a.B) * a.n_tokens;
  const int64_t u0 = static_cast<int64_t>(blockIdx.y) * kMomChunk;
  const int64_t u1 = min64(N, u0 + kMomChunk);
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  double acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
  const double inv_g = 1.0 / G;
  for (int64_t s0 = u0; s0 < u1; s0 += kMomSub) {
    // stage tokens [s0, s0 + 32): 32 tokens x 64 dims per tile = 256 chunks of 8 dims, one
    // per thread and tile; rows past the chunk end are zeros
    {
      const int tok = threadIdx.x / 8, ch = threadIdx.x % 8;
      const int64_t u = s0 + tok;
      double vi[8], vj[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) { vi[e] = 0.0; vj[e] = 0.0; }
      if (u < u1) {
        const int64_t b = u / a.n_tokens, t = u % a.n_tokens;
        const int ci = ti * kMomTile + ch * 8, cj = tj * kMomTile + ch * 8;
        if (which == 1) {
          const __nv_bfloat16* row = static_cast<const __nv_bfloat16*>(a.K) + b * a.ks[0] + h * a.ks[1] + t * a.ks[2];
          const uint4 ri = __ldg(reinterpret_cast<const uint4*>(row + ci));
          const uint4 rj = __ldg(reinterpret_cast<const uint4*>(row + cj));
          const uint32_t wi[4] = {ri.x, ri.y, ri.z, ri.w}, wj[4] = {rj.x, rj.y, rj.z, rj.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            vi[2 * e] = bf16_bits_to_f64(wi[e] & 0xFFFFu); vi[2 * e + 1] = bf16_bits_to_f64(wi[e] >> 16);
            vj[2 * e] = bf16_bits_to_f64(wj[e] & 0xFFFFu); vj[2 * e + 1] = bf16_bits_to_f64(wj[e] >> 16);
          }
        } else {  // group mean of the KV head's G query heads (exact in fp64)
          const __nv_bfloat16* q0 = static_cast<const __nv_bfloat16*>(a.Qc) +
                                    ((b * a.Hq + static_cast<int64_t>(h) * G) * a.n_tokens + t) * d;
          const int64_t hstride = a.n_tokens * d;
          for (int g = 0; g < G; ++g) {
            const uint4 ri = __ldg(reinterpret_cast<const uint4*>(q0 + g * hstride + ci));
            const uint4 rj = __ldg(reinterpret_cast<const uint4*>(q0 + g * hstride + cj));
            const uint32_t wi[4] = {ri.x, ri.y, ri.z, ri.w}, wj[4] = {rj.x, rj.y, rj.z, rj.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              vi[2 * e] += bf16_bits_to_f64(wi[e] & 0xFFFFu); vi[2 * e + 1] += bf16_bits_to_f64(wi[e] >> 16);
              vj[2 * e] += bf16_bits_to_f64(wj[e] & 0xFFFFu); vj[2 * e + 1] += bf16_bits_to_f64(wj[e] >> 16);
            }
          }
#pragma unroll
          for (int e = 0; e < 8; ++e) { vi[e] *= inv_g; vj[e] *= inv_g; }
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        xi[tok][ch * 8 + e] = vi[e];
        xj[tok][ch * 8 + e] = vj[e];
      }
    }
    __syncthreads();
#pragma unroll 4
    for (int t = 0; t < kMomSub; ++t) {
      double p[4], q[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { p[i] = xi[t][ty * 4 + i]; q[i] = xj[t][tx * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fma(p[i], q[j], acc[i][j]);
    }
    __syncthreads();
  }
  double* out = a.acc + (static_cast<int64_t>(h) * 2 + which) * d * d;
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
      atomicAdd(out + static_cast<int64_t>(ti * kMomTile + ty * 4 + i) * d + tj * kMomTile + tx * 4 + j, acc[i][j]);
}

// Round-robin pairing of d indices (d even) in round m of a sweep (d - 1 rounds): pair 0
// is (d - 1, m); pair k > 0 is ((m + k) mod (d - 1), (m - k) mod (d - 1)).  Returned with
// the smaller index first.
__device__ __forceinline__ void rr_pair(int d, int m, int k, int* lo, int* hi) {
  int x, y;
  if (k == 0) {
    x = d - 1;
    y = m;
  } else {
    x = (m + k) % (d - 1);
    y = (m - k + (d - 1)) % (d - 1);
  }
  *lo = min(x, y);
  *hi = max(x, y);
}

__global__ void __launch_bounds__(kJacThreads) jacobi_kernel(CalibArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  cg::cluster_group cl = cg::this_cluster();
  const int C = static_cast<int>(cl.num_blocks()), crank = static_cast<int>(cl.block_rank());
  const int h = blockIdx.x / C;
  const int d = a.d, np = d / 2, tid = threadIdx.x;
  double* cs_c = reinterpret_cast<double*>(smem_raw);  // [np] cosines of the round
  double* cs_s = cs_c + np;                            // [np] sines
  int* plo = reinterpret_cast<int*>(cs_s + np);        // [np] smaller index of each pair
  int* phi = plo + np;                                 // [np] larger index
  __shared__ double red[kJacThreads / 32];
  __shared__ double fro2_s;
  __shared__ int stop_s;
  double* A0 = a.jac + static_cast<int64_t>(h) * 3 * d * d;  // two matrix buffers, then W = V^T
  double* A1 = A0 + static_cast<int64_t>(d) * d;
  double* W = A1 + static_cast<int64_t>(d) * d;
  double* offp = a.jac_off + static_cast<int64_t>(h) * 2 * kJacCluster;  // [2 parities][C] partial off-norms
  const double* Sq = a.acc + static_cast<int64_t>(h) * 2 * d * d;
  const double* Sk = Sq + static_cast<int64_t>(d) * d;

  // M = S_q / tr S_q + S_k / tr S_k (the accumulated sums hold the upper tile triangle)
  double trq = 0.0, trk = 0.0;
  for (int i = 0; i < d; ++i) { trq += Sq[static_cast<int64_t>(i) * d + i]; trk += Sk[static_cast<int64_t>(i) * d + i]; }
  const double wq = trq > 0.0 ? 1.0 / trq : 0.0, wk = trk > 0.0 ? 1.0 / trk : 0.0;
  double fro_part = 0.0;
  for (int64_t e = static_cast<int64_t>(crank) * kJacThreads + tid; e < static_cast<int64_t>(d) * d;
       e += static_cast<int64_t>(C) * kJacThreads) {
    const int x = static_cast<int>(e / d), y = static_cast<int>(e % d);
    const int64_t src = (x / kMomTile <= y / kMomTile) ? e : static_cast<int64_t>(y) * d + x;
    const double m = Sq[src] * wq + Sk[src] * wk;
    A0[e] = m;
    W[e] = (x == y) ? 1.0 : 0.0;
    fro_part += m * m;
  }
  // the Frobenius norm (invariant under the rotations) from the partials, in rank order
  for (int off = 16; off > 0; off >>= 1) fro_part += __shfl_down_sync(0xFFFFFFFFu, fro_part, off);
  if ((tid & 31) == 0) red[tid >> 5] = fro_part;
  __syncthreads();
  if (tid == 0) {
    double s = 0.0;
    for (int w = 0; w < kJacThreads / 32; ++w) s += red[w];
    offp[crank] = s;  // parity slot 0 doubles as the norm exchange before the first round
  }
  cl.sync();
  if (tid == 0) {
    double s = 0.0;
    for (int c = 0; c < C; ++c) s += offp[c];
    fro2_s = s;
    stop_s = 0;
  }
  cl.sync();  // everyone has read the norm partials before they are reused
  const double thresh = fro2_s * 1e-24;  // off-diagonal mass below 1e-12 of the norm
  const int k_lo = np * crank / C, k_hi = np * (crank + 1) / C;  // this CTA's pairs

  const int rounds_max = kJacMaxSweeps * (d - 1);
  double* Acur = A0;
  double* Anext = A1;
  int round = 0;
  for (; round < rounds_max; ++round) {
    const int m = round % (d - 1);
    // the round's pairs and angles (every CTA computes all of them from the current matrix)
    for (int k = tid; k < np; k += kJacThreads) {
      int p, q;
      rr_pair(d, m, k, &p, &q);
      plo[k] = p;
      phi[k] = q;
      const double app = Acur[static_cast<int64_t>(p) * d + p], aqq = Acur[static_cast<int64_t>(q) * d + q];
      const double apq = Acur[static_cast<int64_t>(p) * d + q];
      double c = 1.0, s = 0.0;
      if (apq != 0.0) {
        // zero the (p, q) entry: with t = tan(theta), t^2 + 2 tau t - 1 = 0, smaller root
        const double tau = (aqq - app) / (2.0 * apq);
        const double t = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(1.0 + tau * tau));
        c = 1.0 / sqrt(1.0 + t * t);
        s = t * c;
      }
      cs_c[k] = c;
      cs_s[k] = s;
    }
    __syncthreads();
    // new rows of this CTA's pairs: block (pair k rows) x (pair l columns) = R_k^T B R_l,
    // R = [[c, s], [-s, c]]; the transposed eigenvector rows rotate with R_k^T
    double off_part = 0.0;
    const int items = (k_hi - k_lo) * np;
    for (int it = tid; it < items; it += kJacThreads) {
      const int k = k_lo + it / np, l = it % np;
      const int a0 = plo[k], a1 = phi[k], e0 = plo[l], e1 = phi[l];
      const double ck = cs_c[k], sk = cs_s[k], cl2 = cs_c[l], sl = cs_s[l];
      const double b00 = Acur[static_cast<int64_t>(a0) * d + e0], b01 = Acur[static_cast<int64_t>(a0) * d + e1];
      const double b10 = Acur[static_cast<int64_t>(a1) * d + e0], b11 = Acur[static_cast<int64_t>(a1) * d + e1];
      // left: rows (a0, a1) <- (c b0 - s b1, s b0 + c b1)
      const double t00 = ck * b00 - sk * b10, t01 = ck * b01 - sk * b11;
      const double t10 = sk * b00 + ck * b10, t11 = sk * b01 + ck * b11;
      // right: columns (e0, e1) <- (c t0 - s t1, s t0 + c t1)
      const double n00 = cl2 * t00 - sl * t01, n01 = sl * t00 + cl2 * t01;
      const double n10 = cl2 * t10 - sl * t11, n11 = sl * t10 + cl2 * t11;
      Anext[static_cast<int64_t>(a0) * d + e0] = n00;
      Anext[static_cast<int64_t>(a0) * d + e1] = n01;
      Anext[static_cast<int64_t>(a1) * d + e0] = n10;
      Anext[static_cast<int64_t>(a1) * d + e1] = n11;
      off_part += (a0 != e0 ? n00 * n00 : 0.0) + (a0 != e1 ? n01 * n01 : 0.0) + (a1 != e0 ? n10 * n10 : 0.0) +
                  (a1 != e1 ? n11 * n11 : 0.0);
    }
    for (int it = tid; it < (k_hi - k_lo) * d; it += kJacThreads) {
      const int k = k_lo + it / d, col = it % d;
      const int a0 = plo[k], a1 = phi[k];
      const double ck = cs_c[k], sk = cs_s[k];
      const double w0 = W[static_cast<int64_t>(a0) * d + col], w1 = W[static_cast<int64_t>(a1) * d + col];
      W[static_cast<int64_t>(a0) * d + col] = ck * w0 - sk * w1;
      W[static_cast<int64_t>(a1) * d + col] = sk * w0 + ck * w1;
    }
    for (int off = 16; off > 0; off >>= 1) off_part += __shfl_down_sync(0xFFFFFFFFu, off_part, off);
    if ((tid & 31) == 0) red[tid >> 5] = off_part;
    __syncthreads();
    if (tid == 0) {
      double s = 0.0;
      for (int w = 0; w < kJacThreads / 32; ++w) s += red[w];
      offp[(round & 1) * kJacCluster + crank] = s;
    }
    cl.sync();  // the new matrix and the round's off-diagonal partials are complete
    if (tid == 0) {
      double s = 0.0;
      for (int c = 0; c < C; ++c) s += offp[(round & 1) * kJacCluster + c];
      stop_s = (s <= thresh) ? 1 : 0;
    }
    __syncthreads();
    double* tmp = Acur;
    Acur = Anext;
    Anext = tmp;
    if (stop_s) break;
  }
  if (crank == 0 && tid == 0 && round >= rounds_max) flag_error(a.status, DEVFLAG_TIMEOUT);  // did not converge

  // eigenvalues = diag(Acur); rank by value (descending, lower index first on ties)
  if (crank != 0) return;
  int* rank_of = plo;  // reuse of the pair ends: [d]
  for (int i = tid; i < d; i += kJacThreads) {
    const double li = Acur[static_cast<int64_t>(i) * d + i];
    int rk = 0;
    for (int j = 0; j < d; ++j) {
      const double lj = Acur[static_cast<int64_t>(j) * d + j];
      rk += (lj > li || (lj == li && j < i)) ? 1 : 0;
    }
    rank_of[i] = rk;
    if (a.eigvals) a.eigvals[static_cast<int64_t>(h) * d + rk] = li;
  }
  __syncthreads();
  // the top r eigenvectors (rows of W), sign-fixed, as the columns of P_h (fp32)
  const int warp = tid >> 5, lane = tid & 31;
  for (int i = warp; i < d; i += kJacThreads / 32) {
    const int col = rank_of[i];
    if (col >= a.r) continue;
    const double* v = W + static_cast<int64_t>(i) * d;
    double best = -1.0;
    int bi = d;
    for (int x = lane; x < d; x += 32) {
      const double m = fabs(v[x]);
      if (m > best || (m == best && x < bi)) { best = m; bi = x; }
    }
    for (int off = 16; off > 0; off >>= 1) {
      const double ob = __shfl_down_sync(0xFFFFFFFFu, best, off);
      const int oi = __shfl_down_sync(0xFFFFFFFFu, bi, off);
      if (ob > best || (ob == best && oi < bi)) { best = ob; bi = oi; }
    }
    bi = __shfl_sync(0xFFFFFFFFu, bi, 0);
    const double sign = (v[bi] < 0.0) ? -1.0 : 1.0;
    float* Ph = a.P + static_cast<int64_t>(h) * d * a.r;
    for (int x = lane; x < d; x += 32) Ph[static_cast<int64_t>(x) * a.r + col] = static_cast<float>(sign * v[x]);
  }
}

}  // namespace

size_t calib_workspace_doubles(int Hkv, int d) {
  return static_cast<size_t>(Hkv) * (2 + 3) * d * d + static_cast<size_t>(Hkv) * 2 * kJacCluster;
}

cudaError_t launch_calibrate(const CalibArgs& in, cudaStream_t s) {
  CalibArgs a = in;
  if (a.d % kMomTile != 0 || a.d < kMomTile || a.r < 1 || a.r > a.d || a.n_tokens < 1) return cudaErrorInvalidValue;
  const int nt = a.d / kMomTile;
  const int64_t N = static_cast<int64_t>(a.B) * a.n_tokens;
  cudaError_t e = cudaMemsetAsync(a.acc, 0, sizeof(double) * static_cast<size_t>(a.Hkv) * 2 * a.d * a.d, s);
  if (e != cudaSuccess) return e;
  const dim3 g1(static_cast<unsigned>(nt * (nt + 1) / 2), static_cast<unsigned>(ceil_div(N, kMomChunk)),
                static_cast<unsigned>(a.Hkv * 2));
  if (g1.y > 65535u) return cudaErrorInvalidValue;
  moments_kernel<<<g1, kMomThreads, 0, s>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // cosines and sines (d / 2 each), pair ends (d / 2 each, later the d eigenvalue ranks)
  const size_t smem = static_cast<size_t>(a.d) * sizeof(double) + static_cast<size_t>(a.d) * sizeof(int);
  static int done[64] = {0};
  if ((e = set_smem_limit_once(jacobi_kernel, smem, done)) != cudaSuccess) return e;
  return launch_ex(jacobi_kernel, dim3(a.Hkv * kJacCluster), dim3(kJacThreads), smem, s, kJacCluster, a);
}

}  // namespace jssa
