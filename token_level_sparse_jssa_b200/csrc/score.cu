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
// atomic add per non-zero bin whenever the CTA moves to another row.
//
// The scan is HBM-bound (r*2 bytes of bf16 Kp, or r of E4M3, read and 4 bytes written per token).  A persistent
// grid walks the flattened (row, token) space in 16 KB chunks, each CTA a contiguous
// range of chunks.  One producer warp streams chunks into a shared-memory ring with
// 1-D bulk copies (TMA engine, L2 evict-first) and full/empty mbarrier pairs; eight
// consumer warps score them without any block-wide barrier.  A consumer thread owns
// whole tokens (two threads per token for r = 64): it reads a token's 16-byte
// vectors in a per-thread rotated order, so that every 8-thread phase of a 16-byte
// shared load touches 8 different bank groups, and holds the matching rotated slice
// of qs in registers.  Chunk bookkeeping advances incrementally (no divisions).
// The projected group queries of the rows a CTA covers (formed by the step prologue)
// are loaded into shared memory in one batch at start, while the first chunks stream in.
#include "common.cuh"
#include "launch.h"

namespace jssa {

constexpr int kScoreConsumers = 256;                 // 8 consumer warps
constexpr int kScoreThreads = kScoreConsumers + 32;  // + 1 producer warp
constexpr int kScoreStages = 3;
constexpr int kChunkBytes = 16384;
constexpr int kMaxBatch = 1024;
constexpr int kHistBins = 4096;  // first radix digit of the selection: key bits [31:20]
constexpr int kQRows = 8;        // projected queries preloaded per CTA

// Position in the flattened chunk space: sequence b, KV head h, chunk ci of the row.
struct ChunkIter {
  int b, h;
  int64_t ci;
};

__device__ __forceinline__ void chunk_advance(ChunkIter& c, const int64_t* per_head, int B, int Hkv) {
  if (++c.ci < per_head[c.b]) return;
  c.ci = 0;
  if (++c.h < Hkv) return;
  c.h = 0;
  do { ++c.b; } while (c.b < B && per_head[c.b] == 0);
}

__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kScoreConsumers) : "memory"); }

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

template <int R, bool F8>
__global__ void __launch_bounds__(kScoreThreads, 3) score_kernel(ScoreArgs a) {
  constexpr int EB = F8 ? 1 : 2;                      // bytes per Kp element (E4M3 or bf16)
  constexpr int EPV = 16 / EB;                        // Kp elements per 16-byte vector
  constexpr int CH = kChunkBytes / (R * EB);          // tokens per chunk
  constexpr int V = R * EB / 16;                      // 16-byte vectors per token
  constexpr int TPT = (R >= 64) ? 2 : 1;              // threads per token
  constexpr int VPT = V / TPT;                        // vectors per thread (<= 4)
  static_assert(V >= 1 && V % TPT == 0, "Kp rows of at least 16 bytes");
  constexpr int TOK_PER_PASS = kScoreConsumers / TPT;
  constexpr int PASSES = CH / TOK_PER_PASS;
  static_assert(PASSES >= 1 && CH % TOK_PER_PASS == 0, "chunk / thread mapping");
  extern __shared__ __align__(128) unsigned char smem_raw[];
  unsigned char* ring = smem_raw;                                                   // [stages][16 KB]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem_raw + kScoreStages * kChunkBytes);
  uint64_t* empty = full + kScoreStages;
  uint32_t* hist = reinterpret_cast<uint32_t*>(empty + kScoreStages);               // [kHistBins]
  float* qtab = reinterpret_cast<float*>(hist + kHistBins);                         // [kQRows][R] projected queries
  int64_t* cum = reinterpret_cast<int64_t*>(qtab + kQRows * R);                     // [B + 1] chunk prefix
  int64_t* per_head = cum + (a.B + 1);                                              // [B] chunks per row
  int64_t* nb = per_head + a.B;                                                     // [B] candidates
  __shared__ int aborted;

  const int tid = threadIdx.x;
  const bool producer = tid >= kScoreConsumers;
  for (int i = tid; i < kHistBins; i += blockDim.x) hist[i] = 0;
  for (int b = tid; b < a.B; b += blockDim.x) {
    int64_t T = a.seq_lens[b];
    if (T < 0 || T > a.T_cap) {
      if (blockIdx.x == 0) flag_error(a.status, DEVFLAG_BAD_SEQ_LEN);
      T = T < 0 ? 0 : a.T_cap;
    }
    nb[b] = T - min64(max64(a.window, 0), T);
    per_head[b] = ceil_div(nb[b], CH);
  }
  __syncthreads();
  if (tid == 0) {
    aborted = 0;
    int64_t c = 0;
    for (int b = 0; b < a.B; ++b) {
      cum[b] = c;
      c += static_cast<int64_t>(a.Hkv) * per_head[b];
    }
    cum[a.B] = c;
    for (int s = 0; s < kScoreStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kScoreConsumers / 32);
    }
    fence_mbarrier_init();
  }
  __syncthreads();
  const int64_t total = cum[a.B];
  const int64_t c_begin = total * blockIdx.x / gridDim.x;
  const int64_t c_end = total * (blockIdx.x + 1) / gridDim.x;
  const int64_t n_mine = c_end - c_begin;
  if (n_mine <= 0) return;

  // iterator at c_begin (the only divisions of the kernel)
  ChunkIter it0;
  {
    int b = 0;
    while (b + 1 < a.B && cum[b + 1] <= c_begin) ++b;
    const int64_t local = c_begin - cum[b];
    it0.b = b;
    it0.h = static_cast<int>(local / per_head[b]);
    it0.ci = local % per_head[b];
  }

  if (producer) {
    if ((tid & 31) == 0) {
      const uint64_t policy = l2_policy_evict_first();
      const unsigned char* Kp = static_cast<const unsigned char*>(a.Kp);
      ChunkIter c = it0;
      for (int64_t it = 0; it < n_mine; ++it) {
        const int s = static_cast<int>(it % kScoreStages);
        if (it >= kScoreStages &&
            !mbar_wait_bounded(&empty[s], static_cast<uint32_t>((it / kScoreStages - 1) & 1), a.status)) {
          atomicExch(&aborted, 1);
          break;
        }
        const int64_t t0 = c.ci * CH;
        const uint32_t cnt = static_cast<uint32_t>(min64(CH, nb[c.b] - t0));
        const unsigned char* src = Kp + (c.b * a.ps[0] + c.h * a.ps[1] + t0 * a.ps[2]) * EB;
        mbar_arrive_expect_tx(&full[s], cnt * R * EB);
        bulk_g2s(ring + s * kChunkBytes, src, cnt * R * EB, &full[s], policy);
        chunk_advance(c, per_head, a.B, a.Hkv);
      }
    }
  } else {
    // projected queries of the first kQRows rows this CTA covers, in one batch
    const int row0 = it0.b * a.Hkv + it0.h;
    for (int i = tid; i < kQRows * R; i += kScoreConsumers) {
      const int64_t rr = row0 + i / R;
      if (rr < static_cast<int64_t>(a.B) * a.Hkv) qtab[i] = __ldg(a.qs + rr * R + i % R);
    }
    consumers_sync();
    // this thread's token within a pass, its slice of the token and its rotation
    const int sub = (TPT == 2) ? (tid & 1) : 0;
    const int tok_in_pass = tid / TPT;
    const int rot = kp_vector_rotation<VPT>(tid);
    float q[VPT][EPV];
    ChunkIter c = it0;
    int cur_row = -1;
    bool dead = false;  // a wait gave up: keep the loop's barrier structure, skip the work
    for (int64_t it = 0; it < n_mine; ++it) {
      const int s = static_cast<int>(it % kScoreStages);
      const int row = c.b * a.Hkv + c.h;
      if (row != cur_row) {
        if (cur_row >= 0) {  // flush the finished row's histogram (all consumers)
          consumers_sync();
          if (a.hist) {
            uint32_t* g = a.hist + static_cast<int64_t>(cur_row) * kHistBins;
            for (int i = tid; i < kHistBins; i += kScoreConsumers) {
              const uint32_t v = hist[i];
              if (v) { atomicAdd(g + i, v); hist[i] = 0; }
            }
          }
          consumers_sync();
        }
        cur_row = row;
        const float* qsrc = (row - row0 < kQRows) ? qtab + (row - row0) * R : a.qs + static_cast<int64_t>(row) * R;
#pragma unroll
        for (int j = 0; j < VPT; ++j) {
          const float4* qp = reinterpret_cast<const float4*>(qsrc + (sub * VPT + (j + rot) % VPT) * EPV);
#pragma unroll
          for (int u = 0; u < EPV / 4; ++u) {
            const float4 q4 = qp[u];
            q[j][4 * u] = q4.x; q[j][4 * u + 1] = q4.y; q[j][4 * u + 2] = q4.z; q[j][4 * u + 3] = q4.w;
          }
        }
      }
      if (!dead && !mbar_wait_bounded(&full[s], static_cast<uint32_t>((it / kScoreStages) & 1), a.status)) {
        dead = true;
        atomicExch(&aborted, 1);
      }
      const int64_t t0 = c.ci * CH;
      const int cnt = static_cast<int>(min64(CH, nb[c.b] - t0));
      const unsigned char* buf = ring + s * kChunkBytes;
      if (!dead) {
        float* out = a.scores + static_cast<int64_t>(row) * a.sc_ld + t0;
#pragma unroll
        for (int p = 0; p < PASSES; ++p) {
          const int tok = p * TOK_PER_PASS + tok_in_pass;
          const unsigned char* trow = buf + tok * (R * EB);
          float acc[VPT];
#pragma unroll
          for (int j = 0; j < VPT; ++j) {
            const uint4 raw = *reinterpret_cast<const uint4*>(trow + (sub * VPT + (j + rot) % VPT) * 16);
            acc[j] = kp_vector_dot<F8>(q[j], raw);
          }
          float sc = kp_rotated_sum<VPT>(acc);
          if (TPT == 2) sc += __shfl_xor_sync(0xFFFFFFFFu, sc, 1);
          if (sub == 0 && tok < cnt) {
            out[tok] = sc;
            atomicAdd(&hist[float_to_ordered(sc) >> 20], 1u);
          }
        }
      }
      __syncwarp();
      if ((tid & 31) == 0) mbar_arrive(&empty[s]);
      chunk_advance(c, per_head, a.B, a.Hkv);
    }
    consumers_sync();
    if (a.hist && cur_row >= 0) {
      uint32_t* g = a.hist + static_cast<int64_t>(cur_row) * kHistBins;
      for (int i = tid; i < kHistBins; i += kScoreConsumers) {
        const uint32_t v = hist[i];
        if (v) atomicAdd(g + i, v);
      }
    }
  }
  __syncthreads();
  if (aborted && tid == kScoreConsumers) {
    // give every copy still in flight a bounded chance to land before the CTA exits
    for (int s = 0; s < kScoreStages; ++s) {
      for (int par = 0; par < 2; ++par) mbar_wait_bounded(&full[s], par, nullptr, 50000000ull);
    }
  }
}

template <int R, bool F8>
static cudaError_t launch_score_r(const ScoreArgs& a, int num_sms, cudaStream_t s) {
  const size_t smem = kScoreStages * kChunkBytes + 2 * kScoreStages * sizeof(uint64_t) +
                      kHistBins * sizeof(uint32_t) + kQRows * R * sizeof(float) + (3 * a.B + 1) * sizeof(int64_t);
  static int done[64] = {0};
  cudaError_t e = set_smem_limit_once(score_kernel<R, F8>, smem, done);
  if (e != cudaSuccess) return e;
  const int grid = num_sms * 3;
  return launch_ex(score_kernel<R, F8>, dim3(grid), dim3(kScoreThreads), smem, s, 0, a);
}

cudaError_t launch_score(const ScoreArgs& a, int num_sms, cudaStream_t s) {
  if (a.B > kMaxBatch) return cudaErrorInvalidValue;
  if (a.kp_fp8) {
    switch (a.r) {  // E4M3 rows of at least 16 bytes
      case 16: return launch_score_r<16, true>(a, num_sms, s);
      case 32: return launch_score_r<32, true>(a, num_sms, s);
      case 64: return launch_score_r<64, true>(a, num_sms, s);
      default: return cudaErrorInvalidValue;
    }
  }
  switch (a.r) {
    case 8: return launch_score_r<8, false>(a, num_sms, s);
    case 16: return launch_score_r<16, false>(a, num_sms, s);
    case 32: return launch_score_r<32, false>(a, num_sms, s);
    case 64: return launch_score_r<64, false>(a, num_sms, s);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace jssa
