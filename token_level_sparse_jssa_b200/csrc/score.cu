// Subspace scoring: the full-context score scan.
//
// "Joint Subspace Sparse Attention for Efficient Long-Context Decoding", Figure 1
// and §3.1-§3.2: the group's query heads are projected with the same orthonormal
// basis as the keys and score every cached position of the projected-key cache;
// §E.1: this scan grows with batch size and dominates at large batch.
//
// score:  s[b,h,t] = qs[b,h,:] . Kp[b,h,t,:] (fp32) for t in [0, T_b - W), with the
//         projected group query qs formed by the step prologue (project.cu).
// The scan also builds, per (sequence, KV head) row, the histogram of the top 12 bits
// of the order-preserving score keys (the first radix digit of the top-k selection):
// a shared-memory histogram per CTA, flushed to the row's global histogram with one
// atomic add per non-zero bin whenever the CTA moves to another row.  The ALU work is
// hidden under the memory stream.
//
// The scan is HBM-bound (about r*2 bytes read and 4 bytes written per token).  A
// persistent grid walks the flattened (row, token) space in 16 KB chunks; one
// thread per CTA streams chunks into a 4-stage shared-memory ring with 1-D bulk
// copies (TMA engine, L2 evict-first), completion tracked by mbarriers.  Each chunk
// is consumed with 16-byte shared loads: r/8 consecutive threads share a token,
// each holding a fixed 8-wide slice of qs in registers, and reduce by shuffles.
#include "common.cuh"
#include "launch.h"

namespace jssa {

// ---------------------------------------------------------------- score scan
constexpr int kScoreThreads = 256;
constexpr int kScoreStages = 4;
constexpr int kChunkBytes = 16384;
constexpr int kMaxBatch = 1024;
constexpr int kHistBins = 4096;  // first radix digit of the selection: key bits [31:20]

struct ChunkLoc {
  int row;
  int64_t t0;
  int cnt;
};

template <int R>
__device__ __forceinline__ ChunkLoc locate_chunk(int64_t c, const int64_t* cum, const int64_t* nb, int B, int Hkv) {
  constexpr int CH = kChunkBytes / (R * 2);
  int lo = 0, hi = B - 1;  // last b with cum[b] <= c
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (cum[mid] <= c) lo = mid; else hi = mid - 1;
  }
  const int b = lo;
  const int64_t per_head = ceil_div(nb[b], CH);
  const int64_t local = c - cum[b];
  const int h = static_cast<int>(local / per_head);
  const int64_t ci = local % per_head;
  ChunkLoc L;
  L.row = b * Hkv + h;
  L.t0 = ci * CH;
  L.cnt = static_cast<int>(min64(CH, nb[b] - L.t0));
  return L;
}

template <int R>
__global__ void __launch_bounds__(kScoreThreads) score_kernel(ScoreArgs a) {
  constexpr int CH = kChunkBytes / (R * 2);  // tokens per chunk
  constexpr int V = R / 8;                    // 16-byte vectors per token = threads per token
  extern __shared__ __align__(128) unsigned char smem_raw[];
  unsigned char* ring = smem_raw;                                           // [stages][16 KB]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem_raw + kScoreStages * kChunkBytes);
  uint32_t* hist = reinterpret_cast<uint32_t*>(bars + kScoreStages);        // [kHistBins]
  int64_t* cum = reinterpret_cast<int64_t*>(hist + kHistBins);              // [B + 1]
  int64_t* nb = cum + (a.B + 1);                                            // [B]

  const int tid = threadIdx.x;
  for (int i = tid; i < kHistBins; i += blockDim.x) hist[i] = 0;
  // candidate counts and chunk prefix per batch entry
  for (int b = tid; b < a.B; b += blockDim.x) {
    int64_t T = a.seq_lens[b];
    if (T < 0 || T > a.T_cap) {
      if (blockIdx.x == 0) flag_error(a.status, DEVFLAG_BAD_SEQ_LEN);
      T = T < 0 ? 0 : a.T_cap;
    }
    const int64_t W = min64(max(a.window, 0), T);
    nb[b] = T - W;
  }
  __syncthreads();
  if (tid == 0) {
    int64_t c = 0;
    for (int b = 0; b < a.B; ++b) {
      cum[b] = c;
      c += static_cast<int64_t>(a.Hkv) * ceil_div(nb[b], CH);
    }
    cum[a.B] = c;
    for (int s = 0; s < kScoreStages; ++s) mbar_init(&bars[s], 1);
    fence_mbarrier_init();
  }
  __syncthreads();
  const int64_t total = cum[a.B];
  const int64_t c_begin = total * blockIdx.x / gridDim.x;
  const int64_t c_end = total * (blockIdx.x + 1) / gridDim.x;
  const int64_t n_mine = c_end - c_begin;
  if (n_mine <= 0) return;

  const __nv_bfloat16* Kp = static_cast<const __nv_bfloat16*>(a.Kp);
  uint64_t policy = 0;
  auto issue = [&](int64_t it) {
    const ChunkLoc L = locate_chunk<R>(c_begin + it, cum, nb, a.B, a.Hkv);
    const int b = L.row / a.Hkv, h = L.row % a.Hkv;
    const __nv_bfloat16* src = Kp + b * a.ps[0] + h * a.ps[1] + L.t0 * a.ps[2];
    const uint32_t bytes = static_cast<uint32_t>(L.cnt) * R * 2;
    const int s = static_cast<int>(it % kScoreStages);
    mbar_arrive_expect_tx(&bars[s], bytes);
    bulk_g2s(ring + s * kChunkBytes, src, bytes, &bars[s], policy);
  };
  if (tid == 0) {
    policy = l2_policy_evict_first();
    for (int64_t it = 0; it < min64(kScoreStages, n_mine); ++it) issue(it);
  }

  const int vec = tid % V;            // this thread's 8-wide slice of the token
  float q[8];
  int cur_row = -1;
  // add this CTA's histogram of row `row` into the global one and clear it (block-uniform)
  auto flush = [&](int row) {
    if (a.hist) {
      uint32_t* g = a.hist + static_cast<int64_t>(row) * kHistBins;
      for (int i = tid; i < kHistBins; i += blockDim.x) {
        const uint32_t v = hist[i];
        if (v) { atomicAdd(g + i, v); hist[i] = 0; }
      }
    }
    __syncthreads();
  };
  int64_t it = 0;
  bool aborted = false;
  for (; it < n_mine; ++it) {
    const int s = static_cast<int>(it % kScoreStages);
    const uint32_t parity = static_cast<uint32_t>((it / kScoreStages) & 1);
    const ChunkLoc L = locate_chunk<R>(c_begin + it, cum, nb, a.B, a.Hkv);
    if (L.row != cur_row) {
      if (cur_row >= 0) flush(cur_row);
      cur_row = L.row;
      const float4* qp = reinterpret_cast<const float4*>(a.qs + static_cast<int64_t>(cur_row) * R + vec * 8);
      const float4 q0 = qp[0], q1 = qp[1];
      q[0] = q0.x; q[1] = q0.y; q[2] = q0.z; q[3] = q0.w;
      q[4] = q1.x; q[5] = q1.y; q[6] = q1.z; q[7] = q1.w;
    }
    const bool ok = mbar_wait_bounded(&bars[s], parity, a.status);
    if (ok) {
      const unsigned char* buf = ring + s * kChunkBytes;
      float* out = a.scores + static_cast<int64_t>(L.row) * a.sc_ld + L.t0;
#pragma unroll
      for (int m = 0; m < (CH * V) / kScoreThreads; ++m) {
        const int slot = tid + m * kScoreThreads;
        const int tok = slot / V;
        const uint4 raw = *reinterpret_cast<const uint4*>(buf + static_cast<size_t>(slot) * 16);
        float acc = 0.f;
        acc = fmaf(q[0], __uint_as_float(raw.x << 16), acc);
        acc = fmaf(q[1], __uint_as_float(raw.x & 0xFFFF0000u), acc);
        acc = fmaf(q[2], __uint_as_float(raw.y << 16), acc);
        acc = fmaf(q[3], __uint_as_float(raw.y & 0xFFFF0000u), acc);
        acc = fmaf(q[4], __uint_as_float(raw.z << 16), acc);
        acc = fmaf(q[5], __uint_as_float(raw.z & 0xFFFF0000u), acc);
        acc = fmaf(q[6], __uint_as_float(raw.w << 16), acc);
        acc = fmaf(q[7], __uint_as_float(raw.w & 0xFFFF0000u), acc);
#pragma unroll
        for (int off = V / 2; off >= 1; off >>= 1) acc += __shfl_xor_sync(0xFFFFFFFFu, acc, off);
        if (vec == 0 && tok < L.cnt) {
          out[tok] = acc;
          atomicAdd(&hist[float_to_ordered(acc) >> 20], 1u);
        }
      }
    }
    // one barrier per chunk: everyone is done with stage s, and all agree on a timeout
    if (__syncthreads_or(!ok)) { aborted = true; break; }
    if (tid == 0 && it + kScoreStages < n_mine) issue(it + kScoreStages);
  }
  if (aborted) {
    if (tid == 0) {
      // give every copy still in flight a bounded chance to land before the CTA exits
      for (int64_t j = it; j < min64(it + kScoreStages, n_mine); ++j) {
        const int s = static_cast<int>(j % kScoreStages);
        mbar_wait_bounded(&bars[s], static_cast<uint32_t>((j / kScoreStages) & 1), a.status, 100000000ull);
      }
    }
    return;
  }
  if (cur_row >= 0) flush(cur_row);
}

template <int R>
static cudaError_t launch_score_r(const ScoreArgs& a, int num_sms, cudaStream_t s) {
  const size_t smem = kScoreStages * kChunkBytes + kScoreStages * sizeof(uint64_t) + kHistBins * sizeof(uint32_t) +
                      (2 * a.B + 1) * sizeof(int64_t);
  static int done[64] = {0};
  cudaError_t e = set_smem_limit_once(score_kernel<R>, smem, done);
  if (e != cudaSuccess) return e;
  const int grid = num_sms * 2;
  score_kernel<R><<<grid, kScoreThreads, smem, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_score(const ScoreArgs& a, int num_sms, cudaStream_t s) {
  if (a.B > kMaxBatch) return cudaErrorInvalidValue;
  switch (a.r) {
    case 8: return launch_score_r<8>(a, num_sms, s);
    case 16: return launch_score_r<16>(a, num_sms, s);
    case 32: return launch_score_r<32>(a, num_sms, s);
    case 64: return launch_score_r<64>(a, num_sms, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace jssa
