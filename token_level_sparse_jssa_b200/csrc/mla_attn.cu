// MLA indexed attention on the fifth-generation tensor cores (tcgen05, accumulators in TMEM).
//
// Joint Subspace Sparse Attention, §3.3 (MLA / latent caches) and §A.3: every token keeps one
// latent row of 576 bf16 values (512 latent dims followed by 64 RoPE dims).  The 128 absorbed
// query heads of a sequence form a single group: the logit of head h for token t is
// sm_scale * q_h . C_t over all 576 dims, and the value is C_t[:512].  Attention runs over the
// selected tokens of the sequence plus its sliding window, split into tiles of at most 128 tokens;
// each split's partial (o normalised by its own softmax sum, lse) goes to the workspace and the
// log-sum-exp merge kernel combines the splits.
//
// One CTA handles one (sequence, split) and 128 heads x up to 128 tokens:
//   S = Q . C_tile^T   M = 128 heads, N = tokens, K = 576   (9 K-blocks of 64 dims)
//   P = softmax rows of S (fp32 in registers), stored as bf16 hi + lo parts
//   O = P_hi . V + P_lo . V   M = 128 heads, N = 512 dims (two N = 256 MMAs), K = tokens
// The latent tile is staged once in shared memory (128-byte swizzled rows) and serves both
// MMAs: K-major B operand of the score MMA, MN-major B operand of the value MMA.  The query
// streams through a four-stage ring, which then holds P.  TMEM: S in columns [0, 128), then O
// in all 512 columns (S has been read out by then).  Every wait is bounded; on a timeout the
// kernel raises DEVFLAG_TIMEOUT, stops issuing, drains its copies and MMAs and frees TMEM.
#include "common.cuh"
#include "launch.h"
#include "tcgen05.cuh"

namespace jssa {
namespace {

constexpr int kMlaHeads = 128;
constexpr int kMlaDk = 576;
constexpr int kMlaDv = 512;
constexpr int kMlaKB = kMlaDk / 64;     // 9 K-blocks of the score MMA
constexpr int kMlaTile = 128;           // tokens per CTA at most
constexpr int kMlaThreads = 256;
constexpr int kBlk = 128 * 128;         // one 128-row x 128-byte block (16 KB)
constexpr int kQStages = 4;
constexpr int kCBytes = kMlaKB * kBlk;  // latent tile, 147,456 B
constexpr int kQBytes = kQStages * kBlk;
constexpr int kMlaSmem = kCBytes + kQBytes + 1024;  // + slack to align the tile to 1024 B
constexpr int kStgLd = 36;              // epilogue staging row stride (floats)
constexpr uint32_t kTmemCols = 512;

static_assert(kQBytes >= 4 * kBlk, "the query ring holds P hi and lo (two 64-token blocks each)");
static_assert(8 * 32 * kStgLd * 4 <= kCBytes, "epilogue staging reuses the latent tile");

// cp.async groups still allowed in flight when the score MMA of K-block kb is issued: the
// prologue commits one group per latent block (query blocks 0-2 ride in the first three) and
// iteration kb < 6 commits query block kb + 3.
__device__ __forceinline__ void wait_groups_for_block(int kb) {
  switch (kb) {
    case 0: case 1: case 2: cp_async_wait<8>(); break;
    case 3: case 4: case 5: case 6: cp_async_wait<2>(); break;
    case 7: cp_async_wait<1>(); break;
    default: cp_async_wait<0>(); break;
  }
}

__global__ void __launch_bounds__(kMlaThreads, 1) mla_attn_kernel(AttnArgs a) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  __shared__ int32_t tok_s[kMlaTile];
  __shared__ __align__(8) uint64_t bars[kMlaKB + 1];  // [kb]: score MMAs through block kb; [9]: value MMAs
  __shared__ uint32_t tmem_base_s;
  __shared__ float red_m[2][kMlaHeads], red_l[2][kMlaHeads];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int split = blockIdx.x, b = blockIdx.y;
  const int64_t qrow0 = static_cast<int64_t>(b) * kMlaHeads;  // first (b, head) row of Q, O, partials

  // ---- token list of this split (same rules as the GQA kernels)
  int64_t T = a.seq_lens[b];
  if (T < 0 || T > a.T_cap) {
    if (split == 0 && tid == 0) flag_error(a.status, DEVFLAG_BAD_SEQ_LEN);
    T = T < 0 ? 0 : a.T_cap;
  }
  const int64_t Wc = min64(max64(a.window, 0), T);
  const int64_t win_start = T - Wc;
  int64_t nsel = a.n_sel[b];
  const int64_t nsel_max = min64(a.idx_ld, win_start);
  if (nsel < 0 || nsel > nsel_max) {
    if (split == 0 && tid == 0) flag_error(a.status, DEVFLAG_BAD_NSEL);
    nsel = nsel < 0 ? 0 : nsel_max;
  }
  const int64_t list_len = nsel + Wc;
  const int64_t my_lo = static_cast<int64_t>(split) * a.split_len;
  const int my_len = static_cast<int>(max64(0, min64(list_len, my_lo + a.split_len) - my_lo));

  if (my_len == 0) {  // empty split: weight zero in the merge
    for (int i = tid; i < kMlaHeads * kMlaDv; i += kMlaThreads) {
      const int head = i / kMlaDv, dim = i % kMlaDv;
      a.part_o[((qrow0 + head) * a.S + split) * kMlaDv + dim] = 0.f;
      if (dim == 0) a.part_lse[(qrow0 + head) * a.S + split] = -INFINITY;
    }
    return;
  }

  if (tid < kMlaTile) {
    int32_t t = -1;
    if (tid < my_len) {
      const int64_t pos = my_lo + tid;
      if (pos < nsel) {
        t = a.idx[static_cast<int64_t>(b) * a.idx_ld + pos];
        if (t < 0 || t >= win_start) {
          flag_error(a.status, DEVFLAG_BAD_INDEX);
          t = -1;
        }
      } else {
        t = static_cast<int32_t>(win_start + (pos - nsel));
      }
    }
    tok_s[tid] = t;
  }
  if (tid == 0) {
    for (int i = 0; i <= kMlaKB; ++i) mbar_init(&bars[i], 1);
    fence_mbarrier_init();
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(&tmem_base_s)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_s;

  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t c_s = base;            // latent tile: 9 blocks [128 tokens][64 dims]
  const uint32_t q_s = base + kCBytes;  // query ring: 4 blocks [128 heads][64 dims]; then P hi | P lo
  float* stg_base = reinterpret_cast<float*>(smem_raw + (base - raw));

  // ---- issue every latent load and the first three query blocks
  const int N = (my_len + 15) & ~15;  // MMA N of the score MMA and K extent of the value MMA
  const int ch = tid & 7, r0 = tid >> 3;
  const __nv_bfloat16* Cb = static_cast<const __nv_bfloat16*>(a.K) + static_cast<int64_t>(b) * a.ks[0];
  const __nv_bfloat16* Qb = static_cast<const __nv_bfloat16*>(a.Q) + qrow0 * kMlaDk;
  const uint64_t pol_c = l2_policy_evict_first(), pol_q = l2_policy_evict_last();
  const __nv_bfloat16* src_c[4];
  uint32_t bytes_c[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int j = r0 + 32 * u;
    const int32_t t = tok_s[j];
    src_c[u] = (t >= 0) ? Cb + static_cast<int64_t>(t) * a.ks[2] + ch * 8 : Cb;
    bytes_c[u] = (t >= 0) ? 16u : 0u;  // masked slots are zero-filled
  }
#pragma unroll
  for (int kb = 0; kb < kMlaKB; ++kb) {
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = r0 + 32 * u;
      if (j < N) cp_async16_hint(c_s + kb * kBlk + sw128(j, ch), src_c[u] + (bytes_c[u] ? kb * 64 : 0), bytes_c[u], pol_c);
    }
    if (kb < kQStages - 1) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int h = r0 + 32 * u;
        cp_async16_hint(q_s + kb * kBlk + sw128(h, ch), Qb + h * kMlaDk + kb * 64 + ch * 8, 16u, pol_q);
      }
    }
    cp_async_commit();
  }

  // ---- score MMA over the 9 K-blocks, query ring refilled behind it
  bool dead = false;
  int last_commit = -1;
  const uint32_t idesc_s = instr_desc(128, N, false);
#pragma unroll
  for (int kb = 0; kb < kMlaKB; ++kb) {
    wait_groups_for_block(kb);
    fence_async_smem();  // this thread's cp.async data -> visible to the tensor core's async proxy
    dead = __syncthreads_or(dead) != 0;
    if (tid == 0 && !dead) {
      tc_fence_after();
      const uint32_t qa = q_s + (kb % kQStages) * kBlk, ca = c_s + kb * kBlk;
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        umma_bf16(tmem, smem_desc(qa + kk * 32, 16, 1024), smem_desc(ca + kk * 32, 16, 1024), idesc_s,
                  (kb | kk) != 0 ? 1u : 0u);
      umma_commit(&bars[kb]);
      last_commit = kb;
    }
    if (kb + kQStages - 1 < kMlaKB) {
      // query block kb+3 goes to the stage of block kb-1: wait for that block's MMAs
      if (kb >= 1 && !dead && !mbar_wait_bounded(&bars[kb - 1], 0, a.status)) dead = true;
      if (!dead) {
        const int nb = kb + kQStages - 1;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int h = r0 + 32 * u;
          cp_async16_hint(q_s + (nb % kQStages) * kBlk + sw128(h, ch), Qb + h * kMlaDk + nb * 64 + ch * 8, 16u,
                          pol_q);
        }
      }
      cp_async_commit();  // also when dead: keeps the group count of every thread in step
    }
  }
  if (!dead && !mbar_wait_bounded(&bars[kMlaKB - 1], 0, a.status)) dead = true;
  tc_fence_after();

  // ---- softmax: warp w reads TMEM lanes 32*(w%4).. (one head per thread), token half w/4
  const int quad = warp & 3, half = warp >> 2;
  const int head = quad * 32 + lane;
  const uint32_t trow = tmem + (static_cast<uint32_t>(quad * 32) << 16);
  float m = -INFINITY, l = 0.f;
  dead = __syncthreads_or(dead) != 0;
  if (!dead) {
    float s[2][32];
    tmem_ld32(trow + half * 64, s[0]);
    tmem_ld32(trow + half * 64 + 32, s[1]);
    const float scale = a.sm_scale * 1.4426950408889634f;  // logits in log2 units
    float mx = -INFINITY;
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      const int j = half * 64 + i;
      const bool valid = (j < my_len) && (tok_s[j] >= 0);
      s[i >> 5][i & 31] = valid ? s[i >> 5][i & 31] * scale : -INFINITY;
      mx = fmaxf(mx, s[i >> 5][i & 31]);
    }
    red_m[half][head] = mx;
    __syncthreads();
    m = fmaxf(red_m[0][head], red_m[1][head]);
    float ls = 0.f;
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      const float p = (m == -INFINITY) ? 0.f : exp2f(s[i >> 5][i & 31] - m);
      s[i >> 5][i & 31] = p;
      ls += p;
    }
    red_l[half][head] = ls;
    // P rows (heads) x 64 tokens of this half, bf16 hi in the first two ring stages, lo in the last two
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      uint32_t hi[4], lo[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int i0 = c * 8 + 2 * e;
        const float p0 = s[i0 >> 5][i0 & 31], p1 = s[(i0 + 1) >> 5][(i0 + 1) & 31];
        const __nv_bfloat16 h0 = __float2bfloat16_rn(p0), h1 = __float2bfloat16_rn(p1);
        hi[e] = static_cast<uint32_t>(__bfloat16_as_ushort(h0)) | (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
        lo[e] = pack_bf16x2(p0 - __bfloat162float(h0), p1 - __bfloat162float(h1));
      }
      const uint32_t off = half * kBlk + sw128(head, c);
      st_shared_v4(q_s + off, hi[0], hi[1], hi[2], hi[3]);
      st_shared_v4(q_s + 2 * kBlk + off, lo[0], lo[1], lo[2], lo[3]);
    }
    fence_async_smem();
  } else {
    __syncthreads();  // matches the exchange barrier above
  }
  tc_fence_before();
  dead = __syncthreads_or(dead) != 0;
  l = red_l[0][head] + red_l[1][head];

  // ---- value MMA: O[128 x 512] = P_hi V + P_lo V over N tokens
  if (tid == 0 && !dead) {
    tc_fence_after();
    const uint32_t idesc_o = instr_desc(128, 256, true);
    for (int kt = 0; kt < N / 16; ++kt) {
#pragma unroll
      for (int nh = 0; nh < 2; ++nh) {
        // V = latent dims [256 nh, 256 nh + 256): MN-major, 64-dim blocks 16 KB apart, 8-token groups 1 KB apart
        const uint64_t bdesc = smem_desc(c_s + nh * 4 * kBlk + kt * 2048, kBlk, 1024);
#pragma unroll
        for (int pl = 0; pl < 2; ++pl) {
          const uint64_t adesc = smem_desc(q_s + pl * 2 * kBlk + (kt >> 2) * kBlk + (kt & 3) * 32, 16, 1024);
          umma_bf16(tmem + nh * 256, adesc, bdesc, idesc_o, (kt > 0 || pl > 0) ? 1u : 0u);
        }
      }
    }
    umma_commit(&bars[kMlaKB]);
    last_commit = kMlaKB;
  }
  if (!dead && !mbar_wait_bounded(&bars[kMlaKB], 0, a.status)) dead = true;
  tc_fence_after();
  dead = __syncthreads_or(dead) != 0;

  // ---- epilogue: normalised partial o (coalesced through a per-warp staging tile) and lse
  if (!dead) {
    const float inv_l = (l > 0.f) ? 1.f / l : 0.f;
    float* stg = stg_base + warp * 32 * kStgLd;
    for (int cj = 0; cj < 8; ++cj) {
      const int col0 = half * 256 + cj * 32;
      float v[32];
      tmem_ld32(trow + col0, v);
#pragma unroll
      for (int u = 0; u < 8; ++u)
        *reinterpret_cast<float4*>(stg + lane * kStgLd + 4 * u) =
            make_float4(v[4 * u] * inv_l, v[4 * u + 1] * inv_l, v[4 * u + 2] * inv_l, v[4 * u + 3] * inv_l);
      __syncwarp();
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const int rr = i * 4 + (lane >> 3), c4 = (lane & 7) * 4;
        const float4 x = *reinterpret_cast<const float4*>(stg + rr * kStgLd + c4);
        float* dst = a.part_o + ((qrow0 + quad * 32 + rr) * a.S + split) * kMlaDv + col0 + c4;
        *reinterpret_cast<float4*>(dst) = x;
      }
      __syncwarp();
    }
    if (half == 0)
      a.part_lse[(qrow0 + head) * a.S + split] = (m == -INFINITY) ? -INFINITY : (m + log2f(l)) * 0.6931471805599453f;
  }

  // ---- drain and free TMEM
  cp_async_wait<0>();
  if (tid == 0 && dead && last_commit >= 0) mbar_wait_bounded(&bars[last_commit], 0, a.status);
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

}  // namespace

int mla_max_split() { return kMlaTile; }

cudaError_t launch_mla_attention(const AttnArgs& a, cudaStream_t s) {
  // The tensor-core kernel covers indexed attention (selection plus window) only; a dense
  // pass over the whole latent cache would need per-tile partials of 256 KB each.
  if (a.idx == nullptr || a.n_sel == nullptr) return cudaErrorNotSupported;
  if (a.Hkv != 1 || a.Hq != kMlaHeads || a.dk != kMlaDk || a.dv != kMlaDv) return cudaErrorNotSupported;
  if (a.split_len < 1 || a.split_len > kMlaTile || a.S < 1) return cudaErrorInvalidValue;
  static int done[64] = {0};
  cudaError_t e = set_smem_limit_once(mla_attn_kernel, kMlaSmem, done);
  if (e != cudaSuccess) return e;
  mla_attn_kernel<<<dim3(a.S, a.B), kMlaThreads, kMlaSmem, s>>>(a);
  return cudaGetLastError();
}

}  // namespace jssa
