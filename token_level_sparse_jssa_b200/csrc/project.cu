// Projected scoring cache on write, and the step prologue.
//
// "Joint Subspace Sparse Attention for Efficient Long-Context Decoding", §3.1 and
// §3.4 (a projected-key cache per layer and KV head, used for scoring only), §3.2
// (one basis for queries and keys) and §E.1 (the newly generated key is projected on
// write; at most 3.2 % of the step).
//
// Kp[t] = rnd(K[t] . P_h): the products K[t,i] * P[i,j] (bf16 x fp32) are exact in fp64
// and are accumulated in fp64, then rounded once to the cache's type (bf16, or FP8 E4M3
// saturated to +-448 as in the paper's deployed scoring cache, §A.3 and §E.2; nearest,
// ties to even), so the stored cache equals the rounding of the exact product except when
// that product lies within about 1e-16 relative of a rounding midpoint.
//
// Two kernels:
//   project_keys_kernel  — many rows (the prefill fill of the cache): 32 rows per CTA,
//                          P_h and the rows staged in shared memory.
//   step_prologue_kernel — one CTA per (sequence, KV head) per decode step: stages
//                          P_h once, forms the projected group query
//                          qs = sum_g P_h^T q_g (fp32; the group sum first) and
//                          projects the newest row(s) into Kp; every output column is
//                          split over 256/r threads whose partial sums are added in a
//                          fixed order.  It also re-arms the attention's split counters.
#include "common.cuh"
#include "launch.h"

namespace jssa {

// Stage P_h [d][r] (fp32) into shared memory with 16-byte loads.
__device__ __forceinline__ void stage_basis(float* Psm, const float* Ph, int n) {
  const float4* src = reinterpret_cast<const float4*>(Ph);
  float4* dst = reinterpret_cast<float4*>(Psm);
  for (int i = threadIdx.x; i < n / 4; i += blockDim.x) dst[i] = __ldg(src + i);
}

// Store one projected value, rounded to the cache's element type, at element offset `off`.
__device__ __forceinline__ void store_kp(void* Kp, int fp8, int64_t off, double v) {
  if (fp8) static_cast<uint8_t*>(Kp)[off] = f64_to_e4m3_rne_sat(v);
  else static_cast<uint16_t*>(Kp)[off] = f64_to_bf16_rne(v);
}

constexpr int kProjRows = 32;     // rows of K per CTA
constexpr int kProjThreads = 256;

__global__ void __launch_bounds__(kProjThreads) project_keys_kernel(ProjectArgs a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const int d = a.d, r = a.r;
  float* Psm = reinterpret_cast<float*>(smem_raw);                                 // [d][r]
  __nv_bfloat16* krows = reinterpret_cast<__nv_bfloat16*>(Psm + d * r);          // [kProjRows][d]
  const int b = blockIdx.z, h = blockIdx.y;
  int64_t tb;
  if (a.t_begin) {
    tb = a.t_begin[b];
  } else {
    int64_t T = a.seq_lens[b];
    if (T < 0 || T > a.T_cap) {
      if (threadIdx.x == 0) flag_error(a.status, DEVFLAG_BAD_SEQ_LEN);
      T = T < 0 ? 0 : a.T_cap;
    }
    tb = T - a.n_tokens;
  }
  stage_basis(Psm, a.P + static_cast<int64_t>(h) * d * r, d * r);
  const int64_t row0 = static_cast<int64_t>(blockIdx.x) * kProjRows;  // offset within [0, n_tokens)
  const int nrows = static_cast<int>(min64(kProjRows, a.n_tokens - row0));
  const __nv_bfloat16* Kb = static_cast<const __nv_bfloat16*>(a.K) + b * a.ks[0] + h * a.ks[1];
  // stage the rows (16-byte chunks); rows outside [0, T_cap) become zeros and are not stored
  const int cpr = d / 8;
  for (int c = threadIdx.x; c < nrows * cpr; c += blockDim.x) {
    const int rr = c / cpr, ch = c % cpr;
    const int64_t t = tb + row0 + rr;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (t >= 0 && t < a.T_cap) v = *reinterpret_cast<const uint4*>(Kb + t * a.ks[2] + ch * 8);
    *reinterpret_cast<uint4*>(krows + rr * d + ch * 8) = v;
  }
  __syncthreads();
  const int groups = kProjThreads / r;   // row groups
  const int j = threadIdx.x % r, g = threadIdx.x / r;
  constexpr int kMaxRowsPerThread = kProjRows / 4;   // r <= 64 -> at least 4 groups
  double acc[kMaxRowsPerThread];
#pragma unroll
  for (int q = 0; q < kMaxRowsPerThread; ++q) acc[q] = 0.0;
  const int my_rows = (nrows - g + groups - 1) / groups;  // rows g, g+groups, ...
#pragma unroll 4
  for (int i = 0; i < d; ++i) {
    const double p = static_cast<double>(Psm[i * r + j]);
#pragma unroll
    for (int q = 0; q < kMaxRowsPerThread; ++q)
      if (q < my_rows) acc[q] = fma(static_cast<double>(__bfloat162float(krows[(g + q * groups) * d + i])), p, acc[q]);
  }
  const int64_t kp0 = b * a.ps[0] + h * a.ps[1];
#pragma unroll
  for (int q = 0; q < kMaxRowsPerThread; ++q) {
    if (q < my_rows) {
      const int64_t t = tb + row0 + g + q * groups;
      if (t >= 0 && t < a.T_cap) store_kp(a.Kp, a.kp_fp8, kp0 + t * a.ps[2] + j, acc[q]);
    }
  }
}

cudaError_t launch_project_keys(const ProjectArgs& a, cudaStream_t s) {
  if (a.n_tokens <= 0) return cudaSuccess;
  dim3 grid(static_cast<unsigned>(ceil_div(a.n_tokens, kProjRows)), a.Hkv, a.B);
  const size_t smem = static_cast<size_t>(a.d) * a.r * sizeof(float) +
                      static_cast<size_t>(kProjRows) * a.d * sizeof(__nv_bfloat16);
  static int done[64] = {0};
  cudaError_t e = set_smem_limit_once(project_keys_kernel, smem, done);
  if (e != cudaSuccess) return e;
  project_keys_kernel<<<grid, kProjThreads, smem, s>>>(a);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ append on write
// One CTA per (sequence, KV head): the newest key (and value) row, 16 bytes per thread,
// from the contiguous [B, Hkv, d] input into row t_pos[b] of the strided caches.
constexpr int kAppendThreads = 64;

__global__ void __launch_bounds__(kAppendThreads) append_rows_kernel(AppendArgs a) {
  const int row = blockIdx.x;
  const int b = row / a.Hkv, h = row % a.Hkv;
  const int64_t t = a.t_pos[b];
  if (t < 0 || t >= a.T_cap) return;
  const uint4* ks = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.K_new) +
                                                   static_cast<int64_t>(row) * a.dk);
  uint4* kd = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.K) + b * a.ks[0] + h * a.ks[1] + t * a.ks[2]);
  for (int i = threadIdx.x; i < a.dk / 8; i += kAppendThreads) kd[i] = __ldg(ks + i);
  if (a.V_new) {
    const uint4* vs = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(a.V_new) +
                                                     static_cast<int64_t>(row) * a.dv);
    uint4* vd = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(a.V) + b * a.vs[0] + h * a.vs[1] + t * a.vs[2]);
    for (int i = threadIdx.x; i < a.dv / 8; i += kAppendThreads) vd[i] = __ldg(vs + i);
  }
}

cudaError_t launch_append_rows(const AppendArgs& a, cudaStream_t s) {
  append_rows_kernel<<<a.B * a.Hkv, kAppendThreads, 0, s>>>(a);
  return cudaGetLastError();
}

// Staging copy of n16 16-byte words (device or device-addressable pinned host memory on
// either side): grid-stride, all of a thread's loads issued before its stores.
__global__ void __launch_bounds__(256) copy16_kernel(uint4* __restrict__ dst, const uint4* __restrict__ src,
                                                     size_t n16) {
  const size_t stride = static_cast<size_t>(gridDim.x) * blockDim.x;
  size_t i = static_cast<size_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (; i + 3 * stride < n16; i += 4 * stride) {
    const uint4 v0 = src[i], v1 = src[i + stride], v2 = src[i + 2 * stride], v3 = src[i + 3 * stride];
    dst[i] = v0;
    dst[i + stride] = v1;
    dst[i + 2 * stride] = v2;
    dst[i + 3 * stride] = v3;
  }
  for (; i < n16; i += stride) dst[i] = src[i];
}

cudaError_t launch_copy16(void* dst, const void* src, size_t n16, int num_sms, cudaStream_t s) {
  if (n16 == 0) return cudaSuccess;
  // one 256-thread block per 4 KB, at most 2 per SM: enough 16-byte requests in flight to
  // cover the host link's latency for the few tens of KB a decode step moves
  const size_t want = (n16 + 255) / 256;
  const size_t cap = static_cast<size_t>(num_sms > 0 ? 2 * num_sms : 256);
  const unsigned blocks = static_cast<unsigned>(want < cap ? want : cap);
  copy16_kernel<<<blocks, 256, 0, s>>>(static_cast<uint4*>(dst), static_cast<const uint4*>(src), n16);
  return cudaGetLastError();
}

// ------------------------------------------------------------------ step prologue
constexpr int kPrologueThreads = 256;
constexpr int kMaxNewRowsInPrologue = 16;
constexpr int kQStageBytes = 16384;  // query groups up to this size are staged with one bulk copy

// One CTA per (sequence, KV head).  P_h, the group's queries and the newest key rows
// arrive through bulk copies (TMA engine) issued together, so the whole prologue costs
// about two memory round trips: one for P_h / Q (and the sequence length), one for
// the key rows, whose position depends on the sequence length.
__global__ void __launch_bounds__(kPrologueThreads) step_prologue_kernel(PrologueArgs a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const int d = a.d, r = a.r;
  const int row = blockIdx.x;
  const int b = row / a.Hkv, h = row % a.Hkv;
  const int G = a.Hq / a.Hkv;
  const int tid = threadIdx.x;
  const bool q_bulk = G * d * 2 <= kQStageBytes;
  const int n_new = a.n_new > 0 ? a.n_new : 0;
  float* Psm = reinterpret_cast<float*>(smem_raw);                                  // [d][r]
  __nv_bfloat16* Qsm = reinterpret_cast<__nv_bfloat16*>(Psm + d * r);              // [G][d] (q_bulk)
  __nv_bfloat16* Ksm = Qsm + (q_bulk ? G * d : 0);                                  // [n_new][d]
  float* vec = reinterpret_cast<float*>(Ksm + ((n_new * d + 7) & ~7));              // [d]
  double* red = reinterpret_cast<double*>(vec + ((d + 1) & ~1));                    // [256]
  __shared__ uint64_t bars[2];
  __shared__ int64_t tb_s;
  if (tid == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  const __nv_bfloat16* Q = static_cast<const __nv_bfloat16*>(a.Q) + (static_cast<int64_t>(b) * a.Hq + h * G) * d;
  const __nv_bfloat16* Kb = static_cast<const __nv_bfloat16*>(a.K) + b * a.ks[0] + h * a.ks[1];
  if (tid == 0) {
    const uint32_t pbytes = static_cast<uint32_t>(d) * r * 4, qbytes = q_bulk ? static_cast<uint32_t>(G) * d * 2 : 0u;
    mbar_arrive_expect_tx(&bars[0], pbytes + qbytes);
    bulk_g2s(Psm, a.P + static_cast<int64_t>(h) * d * r, pbytes, &bars[0], l2_policy_evict_last());
    if (q_bulk) bulk_g2s(Qsm, Q, qbytes, &bars[0], l2_policy_evict_first());
    if (n_new > 0) {
      int64_t T = a.seq_lens[b];
      if (T < 0 || T > a.T_cap) {
        flag_error(a.status, DEVFLAG_BAD_SEQ_LEN);
        T = T < 0 ? 0 : a.T_cap;
      }
      const int64_t t0 = max64(0, T - n_new);
      tb_s = t0;
      const int rows = static_cast<int>(T - t0);
      mbar_arrive_expect_tx(&bars[1], static_cast<uint32_t>(rows) * d * 2);
      for (int q = 0; q < rows; ++q)  // one copy per row: rows may be strided
        bulk_g2s(Ksm + q * d, Kb + (t0 + q) * a.ks[2], static_cast<uint32_t>(d) * 2, &bars[1], l2_policy_evict_first());
    }
  }
  if (a.counters && tid == 0) a.counters[row] = 0;
  // group-summed query (fp32, heads in ascending order)
  bool ok = mbar_wait_bounded(&bars[0], 0, a.status);
  for (int i = tid; i < d; i += blockDim.x) {
    float sacc = 0.f;
    if (q_bulk) {
      for (int g = 0; g < G; ++g) sacc += __bfloat162float(Qsm[g * d + i]);
    } else {
#pragma unroll 8
      for (int g = 0; g < G; ++g) sacc += __bfloat162float(Q[static_cast<int64_t>(g) * d + i]);
    }
    vec[i] = sacc;
  }
  __syncthreads();
  // output column j = tid % r; this thread sums i = part, part + parts, ...; the partial
  // sums are then added in a fixed order (a warp reads consecutive columns of P: no conflicts)
  const int parts = kPrologueThreads / r, j = tid % r, part = tid / r;
  {
    float acc = 0.f;
    for (int i = part; i < d; i += parts) acc = fmaf(Psm[i * r + j], vec[i], acc);
    red[part * r + j] = acc;
    __syncthreads();
    if (tid < r) {
      float t = 0.f;
      for (int q = 0; q < parts; ++q) t += static_cast<float>(red[q * r + tid]);
      a.qs[static_cast<int64_t>(row) * r + tid] = t;
    }
  }
  if (n_new == 0) return;
  // project the newest rows [T_b - n_new, T_b) into Kp (fp64 accumulation, one rounding)
  __syncthreads();
  ok = mbar_wait_bounded(&bars[1], 0, a.status) && ok;
  const int64_t t0 = tb_s;
  const int64_t kp0 = b * a.ps[0] + h * a.ps[1];
  for (int64_t t = t0; t < t0 + n_new; ++t) {
    int64_t T = a.seq_lens[b];
    T = T < 0 ? 0 : (T > a.T_cap ? a.T_cap : T);
    if (t >= T) break;
    const __nv_bfloat16* krow = Ksm + (t - t0) * d;
    double acc = 0.0;
    for (int i = part; i < d; i += parts)
      acc = fma(static_cast<double>(__bfloat162float(krow[i])), static_cast<double>(Psm[i * r + j]), acc);
    red[part * r + j] = acc;
    __syncthreads();
    if (tid < r && ok) {
      double t2 = 0.0;
      for (int q = 0; q < parts; ++q) t2 += red[q * r + tid];
      store_kp(a.Kp, a.kp_fp8, kp0 + t * a.ps[2] + tid, t2);
    }
    __syncthreads();
  }
}

cudaError_t launch_step_prologue(const PrologueArgs& a, cudaStream_t s) {
  if (a.n_new > kMaxNewRowsInPrologue) return cudaErrorInvalidValue;
  const int G = a.Hq / a.Hkv;
  const bool q_bulk = G * a.d * 2 <= kQStageBytes;
  const int n_new = a.n_new > 0 ? a.n_new : 0;
  const size_t smem = static_cast<size_t>(a.d) * a.r * 4 + (q_bulk ? static_cast<size_t>(G) * a.d * 2 : 0) +
                      static_cast<size_t>((n_new * a.d + 7) & ~7) * 2 + static_cast<size_t>((a.d + 1) & ~1) * 4 +
                      kPrologueThreads * sizeof(double);
  static int done[64] = {0};
  cudaError_t e = set_smem_limit_once(step_prologue_kernel, smem, done);
  if (e != cudaSuccess) return e;
  return launch_ex(step_prologue_kernel, dim3(a.B * a.Hkv), dim3(kPrologueThreads), smem, s, 0, a);
}

}  // namespace jssa
