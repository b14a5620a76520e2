/*
 * jssa.h — C ABI of libjssa.so: the decode-step hot path of Joint Subspace Sparse
 * Attention on NVIDIA B200 (sm_100a).
 *
 * Method: "Joint Subspace Sparse Attention for Efficient Long-Context Decoding"
 * (Song, Kim, Kim; arXiv 2610.19026v1, paperlayer.ai summary).  At each decoding
 * step, per KV head, the projected group query scores a projected-key cache
 * Kp = K P, the top-B positions are selected per sequence and KV head, and the
 * group's query heads attend over the original full-dimensional K/V rows at those
 * positions, read in place (Figure 1; §3.1 Overview; §3.3 Gather-free indexed
 * attention; §3.4 Projected scoring cache; §E.1 the new key is projected on write).
 * "B" (the token budget) is called k here.
 *
 * Conventions fixed by this library (the summary leaves them open):
 *   - group query = SUM of the G query heads of a KV head (the page's "mean" times
 *     G; the ranking is identical);
 *   - score of token t for KV head h = fp32 dot product of (sum_g P_h^T q_g) with
 *     Kp[t] — the projected query is formed in fp32 from bf16 Q and fp32 P;
 *   - ties in the top-k break toward the lower token index; selected indices are
 *     written in ascending order; unused slots are -1;
 *   - Kp is stored in bf16 or, with kp_dtype = JSSA_KP_FP8_E4M3, in FP8 E4M3 (the
 *     paper's deployed scoring cache, §A.3, §E.2), rounded to nearest-even once
 *     from an fp64 accumulation of K P (bit-identical to rounding the exact product,
 *     except in cases where the exact value lies within ~1e-16 relative of a
 *     rounding midpoint).  E4M3 is the OCP format (bias 7, subnormals, max 448)
 *     with a unit scale and saturation to +-448; a per-head scale s_h is expressed
 *     by passing P_h / s_h, which scales every score of the (sequence, head) row by
 *     the same positive factor and leaves the selection unchanged;
 *   - attention uses an explicit softmax scale sm_scale (logit = sm_scale * q . k);
 *     split partials are combined by a log-sum-exp merge;
 *   - with a sliding window W > 0 (hybrid local/global models, §A.1/§A.3), the
 *     candidates are [0, T - W) and the attended set is the selection plus the
 *     window [T - W, T);
 *   - MLA (§3.3, §A.3): one latent row per token per layer (Hkv = 1) serves as the
 *     key (d_k dims) and, on its first d_v dims, as the value; all query heads
 *     share one index set.
 *
 * Memory model.  Every pointer argument named "device" points to GPU memory owned
 * by the caller; the library never allocates, frees or synchronises on the compute
 * calls.  All compute calls are asynchronous on `stream` (a cudaStream_t passed as
 * void*; NULL = the legacy default stream) and contain no host synchronisation, so
 * they can be captured into a CUDA graph.  Scratch memory is a caller-provided
 * workspace of at least jssa_workspace_size() bytes, 256-byte aligned, zeroed once
 * with jssa_workspace_init() before its first use; every call leaves it ready for the
 * next (some scratch, such as the selection histograms and the split counters, must
 * be zero on entry and is cleared by the kernel that consumes it).  After a call
 * that returned an error, initialise the workspace again.
 *
 * Errors.  Arguments are validated on the host before any launch; an invalid call
 * returns an error status and launches nothing.  A launch failure returns
 * JSSA_ERR_CUDA.  Values only visible on the device (seq_lens, n_sel, indices) are
 * clamped or skipped by the kernels, which record what they saw in a status word
 * inside the workspace; jssa_read_device_status() returns and clears it.
 * No C++ exception crosses this interface.
 */
#ifndef JSSA_H_
#define JSSA_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define JSSA_API __attribute__((visibility("default")))
#else
#define JSSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  JSSA_OK = 0,
  JSSA_ERR_INVALID_ARG = 1,  /* null pointer, bad size, stride or alignment      */
  JSSA_ERR_UNSUPPORTED = 2,  /* a valid but unimplemented shape (d, r, G, mode)  */
  JSSA_ERR_WORKSPACE = 3,    /* workspace missing, misaligned or too small       */
  JSSA_ERR_CUDA = 4,         /* a CUDA runtime call or launch failed             */
  JSSA_ERR_DEVICE_CHECK = 5, /* the kernels flagged out-of-range device data     */
  JSSA_ERR_TIMEOUT = 6,      /* a bounded wait inside a kernel gave up           */
  JSSA_ERR_SCRATCH_LIMIT = 7 /* beyond the built-in scratch of jssa_topk_noalloc */
} jssa_status;

enum { JSSA_MODE_GQA = 0, JSSA_MODE_MLA = 1 };
enum { JSSA_OUT_F32 = 0, JSSA_OUT_BF16 = 1 };
enum { JSSA_KP_BF16 = 0, JSSA_KP_FP8_E4M3 = 1 };

/* Device status bits reported by jssa_read_device_status(). */
enum {
  JSSA_DEV_BAD_SEQ_LEN = 1, /* a seq_lens[b] outside [0, T_cap] (clamped)        */
  JSSA_DEV_BAD_INDEX = 2,   /* an index outside its candidate range (skipped)    */
  JSSA_DEV_BAD_NSEL = 4,    /* an n_sel outside [0, k] (clamped)                 */
  JSSA_DEV_TIMEOUT = 8      /* a bounded wait gave up                            */
};

/*
 * Shapes and cache layout.  Element strides, last dimension contiguous.
 *   Q    [B, Hq, d_k]      bf16, contiguous
 *   K    element (b, h, t, i) at K[b*k_stride[0] + h*k_stride[1] + t*k_stride[2] + i], i < d_k
 *   V    element (b, h, t, i) at V[b*v_stride[0] + h*v_stride[1] + t*v_stride[2] + i], i < d_v
 *   Kp   element (b, h, t, j) at Kp[b*kp_stride[0] + h*kp_stride[1] + t*kp_stride[2] + j], j < r,
 *        bf16 or E4M3 bytes (kp_dtype); kp_stride[2] = r (rows contiguous)
 *   P    [Hkv, d_k, r]     fp32, contiguous (column j of P_h is the j-th basis vector)
 *   O    [B, Hq, d_v]      fp32 or bf16 (out_dtype), contiguous
 *   lse  [B, Hq]           fp32 natural-log log-sum-exp of the scaled logits (optional)
 * GQA: Hq = G * Hkv; query head hq belongs to KV head hq / G.  Supported: d_k = d_v in
 * {64, 128, 256}, G in {1, 2, 4, 8, 16}, r in {8, 16, 32, 64} (r <= d_k).
 * MLA: Hkv = 1, d_k = 576, d_v = 512, Hq = 128, r in {16, 32, 64}; V may alias K.
 * An E4M3 Kp needs r >= 16 (rows of at least 16 bytes).
 * Q, P, K, V and Kp base pointers and the K/V/Kp strides (except the unit inner
 * stride) must be multiples of 16 bytes.  A zero-initialised kp_dtype means bf16.
 */
typedef struct {
  int32_t mode;      /* JSSA_MODE_GQA or JSSA_MODE_MLA                    */
  int32_t B, Hq, Hkv;
  int32_t d_k, d_v, r;
  int32_t out_dtype; /* JSSA_OUT_F32 or JSSA_OUT_BF16                      */
  int64_t T_cap;     /* rows allocated per (b, h) in K, V and Kp            */
  int64_t k_stride[3];
  int64_t v_stride[3];
  int64_t kp_stride[3];
  int32_t kp_dtype;  /* JSSA_KP_BF16 or JSSA_KP_FP8_E4M3                   */
} jssa_layout;

/* Human-readable name of a status code (static string). */
JSSA_API const char* jssa_status_string(jssa_status s);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
JSSA_API int32_t jssa_version(void);

/*
 * Bytes of workspace needed by every compute call below for this layout, a budget
 * of at most k tokens and a window of at most `window` tokens, on the current
 * device.  Host-only.
 */
JSSA_API jssa_status jssa_workspace_size(const jssa_layout* L, int32_t k, int32_t window, size_t* bytes);

/*
 * Append on write (§3.1, §E.1: a generated key enters the cache, and is projected, when it
 * is written): copies the newest key and value rows of every (sequence, KV head) into
 * row t_pos[b] of the caches; jssa_decode_step with n_new = 1 then projects that row.
 *   K_new  device bf16 [B, Hkv, d_k], contiguous, 16-byte aligned;
 *   V_new  device bf16 [B, Hkv, d_v], contiguous, 16-byte aligned (GQA); NULL in MLA mode,
 *          where V is the leading d_v dims of the latent row K (V is then ignored);
 *   K, V   the layout's caches;
 *   t_pos  device int32 [B]; sequences whose t_pos lies outside [0, T_cap) are not written.
 * Asynchronous on `stream`; allocates nothing.
 */
JSSA_API jssa_status jssa_append_kv(const jssa_layout* L, const void* K_new, const void* V_new, void* K, void* V,
                                    const int32_t* t_pos, void* stream);

/*
 * Staging copy by a kernel instead of a copy engine, for the small per-step transfers of a
 * decode loop (the query and the newest K/V rows in, the attention output out): copies
 * `bytes` from src to dst, where each of dst and src is device memory or page-locked host
 * memory that the device can address (cudaHostAlloc / pinned tensors under unified
 * addressing).  Both pointers 16-byte aligned, bytes a multiple of 16; pageable host memory,
 * misalignment or a null pointer return JSSA_ERR_INVALID_ARG without launching anything.
 * Asynchronous on `stream` and ordered with the calls around it like any kernel; allocates
 * nothing.  The kernel reads or writes host memory over the host link, 16 bytes per thread.
 */
JSSA_API jssa_status jssa_copy_mapped(void* dst, const void* src, size_t bytes, void* stream);

/*
 * Projected scoring cache on write (§3.1, §3.4, §E.1):
 *   Kp[b, h, t, :] = rnd(K[b, h, t, :] . P_h)   for t in [t_begin[b], t_begin[b] + n_tokens)
 * with rnd = bf16 or E4M3 (saturating) rounding to nearest even, by kp_dtype.
 * t_begin: device int32 [B] (rows past T_cap are skipped), or NULL to mean
 * t_begin[b] = seq_lens[b] - n_tokens (the last n_tokens rows; then seq_lens is
 * required).  n_tokens = 0 is a no-op.
 */
JSSA_API jssa_status jssa_project_keys(const jssa_layout* L, const void* K, const float* P, void* Kp,
                              const int32_t* t_begin, const int32_t* seq_lens, int64_t n_tokens,
                              void* stream);

/*
 * Subspace score scan (Figure 1; §2 "score every candidate position"):
 *   scores[b, h, t] = fp32( (sum_g P_h^T q_{hG+g}) . Kp[b, h, t] )   for t in [0, T_b - W)
 * with T_b = seq_lens[b] (device int32 [B]) and W = window clamped to [0, T_b].
 * scores: device fp32 [B, Hkv, T_cap]; entries at t >= T_b - W are not written.
 */
JSSA_API jssa_status jssa_score(const jssa_layout* L, const void* Q, const float* P, const void* Kp,
                       const int32_t* seq_lens, int32_t window, float* scores,
                       void* workspace, size_t ws_bytes, void* stream);

/*
 * Per-(sequence, KV head) top-k (Figure 1 "top-B positions"; §E.3 per-KV-head
 * selection) over scores[b, h, 0 : T_b - W):
 *   idx[b, h, :]  the k_eff = min(k, T_b - W) positions of largest score, ties to the
 *                 lower index, ascending; slots >= k_eff are -1      (device int32 [B, Hkv, k])
 *   n_sel[b, h]   k_eff                                               (device int32 [B, Hkv])
 * scores: device fp32 [B, Hkv, T_cap]; must be finite.  The workspace (required) holds
 * the per-row first-digit histogram this call builds before selecting.
 */
JSSA_API jssa_status jssa_topk(const jssa_layout* L, const float* scores, const int32_t* seq_lens,
                      int32_t k, int32_t window, int32_t* idx, int32_t* n_sel,
                      void* workspace, size_t ws_bytes, void* stream);

/*
 * Allocation-free top-k: the same selection as jssa_topk, with no workspace argument.
 * The paper has no counterpart to this entry point; it exists for callers that cannot
 * allocate device memory for a workspace: code running inside a host framework that owns
 * all device memory and hands plug-ins no allocator, or code that must not allocate
 * while a stream is being captured.  Its scratch (the per-row first-digit histograms) is
 * a 4 MB array inside the library, present on every GPU that loads the library until the
 * process exits; it holds at most 256 (sequence, KV head) rows: larger batches return
 * JSSA_ERR_SCRATCH_LIMIT and launch nothing.  The call allocates nothing: it clears the
 * part of the scratch it uses (the previous call's contents remain otherwise) and runs
 * the selection kernels.  The first call on a device looks up the scratch's device
 * address (once per device); make that first call before any stream capture.  All
 * calls share one scratch, so calls that may overlap on the GPU (other streams, other
 * host threads) race and must be serialised by the caller.  No device status word is
 * kept: a row whose bounded wait gave up returns an empty selection (n_sel = 0, idx all
 * -1), which is how a caller of this entry point detects it.
 */
JSSA_API jssa_status jssa_topk_noalloc(const jssa_layout* L, const float* scores, const int32_t* seq_lens,
                                       int32_t k, int32_t window, int32_t* idx, int32_t* n_sel, void* stream);

/*
 * Gather-free indexed attention (§3.3) with split-T partials and a log-sum-exp merge.
 * For query head hq of KV head h: attended set = {idx[b, h, j] : j < n_sel[b, h]} plus
 * the window [T_b - W, T_b); logits = sm_scale * q . K_t; O = softmax . V.  K/V rows
 * are read in place.  idx entries must be distinct and in [0, T_b - W); out-of-range
 * entries are skipped and flagged.  lse may be NULL.
 */
JSSA_API jssa_status jssa_indexed_attn(const jssa_layout* L, const void* Q, const void* K, const void* V,
                              const int32_t* idx, int32_t k, const int32_t* n_sel,
                              const int32_t* seq_lens, int32_t window, float sm_scale,
                              void* O, float* lse, void* workspace, size_t ws_bytes, void* stream);

/*
 * The selection half of a decode step (Figure 1 up to the "top-B positions"; §3.2 keys
 * projected on write): project the last n_new rows of each sequence into Kp, form the
 * projected group query, score every candidate [0, T_b - W) and select the top-k per
 * (sequence, KV head), with the ties, ordering and padding rules of jssa_topk.
 *   idx    device int32 [B, Hkv, k]      n_sel  device int32 [B, Hkv]
 * When T_cap <= 131072 all of this runs in one kernel with one thread-block cluster per
 * (sequence, KV head) of 2 to 16 CTAs (the largest size that keeps every row's cluster
 * resident at once), the scores never leaving shared memory; longer caches take the
 * jssa_score + jssa_topk kernels.  Up to 16 appended rows are projected inside the
 * selection; more are projected by the bulk projection kernel first.
 */
JSSA_API jssa_status jssa_select(const jssa_layout* L, const void* Q, const void* K, void* Kp, const float* P,
                                 const int32_t* seq_lens, int32_t n_new, int32_t k, int32_t window, int32_t* idx,
                                 int32_t* n_sel, void* workspace, size_t ws_bytes, void* stream);

/*
 * Head-shared soft voting (§1, §E.3 / Table 15: the variant that per-KV-head selection is
 * compared with; the vote is not defined on the pages, this is the library's reading):
 * the same projections and score scan as jssa_select, then per (sequence, KV head) the
 * distribution p_h(t) = softmax_t(c * s_h(t)) over the candidates [0, T_b - W) with
 * c = sm_scale / G (the logit of the group-mean query), the vote v(t) = sum_h p_h(t), and
 * the top-k of v (ties to the lower index, ascending, -1 padded) written to EVERY KV head's
 * row of idx.  Runs the unfused kernels (score scan, vote statistics and combination,
 * top-k, broadcast) for any T_cap.  Arguments as jssa_select, plus sm_scale > 0.
 */
JSSA_API jssa_status jssa_vote_select(const jssa_layout* L, const void* Q, const void* K, void* Kp, const float* P,
                                      const int32_t* seq_lens, int32_t n_new, int32_t k, int32_t window,
                                      float sm_scale, int32_t* idx, int32_t* n_sel, void* workspace, size_t ws_bytes,
                                      void* stream);

/*
 * One fused decode step (Figure 1): project the last n_new rows of each sequence
 * into Kp (n_new may be 0 when Kp is already current), score, select the top-k per
 * (sequence, KV head), attend over the selection (plus the window) and merge.
 * idx_out / n_sel_out (nullable) receive the selection; otherwise it stays in the
 * workspace.  lse may be NULL.
 */
JSSA_API jssa_status jssa_decode_step(const jssa_layout* L, const void* Q, const void* K, const void* V,
                             void* Kp, const float* P, const int32_t* seq_lens, int32_t n_new,
                             int32_t k, int32_t window, float sm_scale, void* O, float* lse,
                             int32_t* idx_out, int32_t* n_sel_out, void* workspace,
                             size_t ws_bytes, void* stream);

/*
 * Gather-then-attend comparator (§2.2, §3.3, §4.7): not the method's path, but the
 * gather-based baseline its gather-free kernel is measured against.  The attended rows of every
 * (sequence, KV head), exactly as jssa_indexed_attn defines them, are first copied into a compact
 * buffer; then the dense flash-decode runs over that buffer.  GQA only.
 * jssa_gather_size gives the bytes of the caller-owned gather buffer (16-byte aligned):
 * gathered K and V [B*Hkv, Lmax, d] bf16 with Lmax = k + min(window, T_cap), plus the row
 * lengths.  The workspace is the one jssa_workspace_size(L, k, window) sizes.
 */
JSSA_API jssa_status jssa_gather_size(const jssa_layout* L, int32_t k, int32_t window, size_t* bytes);
JSSA_API jssa_status jssa_gather_decode(const jssa_layout* L, const void* Q, const void* K, const void* V,
                                        const int32_t* idx, int32_t k, const int32_t* n_sel,
                                        const int32_t* seq_lens, int32_t window, float sm_scale, void* O,
                                        float* lse, void* gather_buf, size_t gather_bytes, void* workspace,
                                        size_t ws_bytes, void* stream);

/*
 * Dense full-KV flash-decode (the full-KV baseline of §4.5), same kernel family as
 * jssa_indexed_attn with the index list replaced by the contiguous range
 * [T_b - W, T_b) (W = window clamped to T_b; window = 0 means all of [0, T_b)).
 */
JSSA_API jssa_status jssa_dense_decode(const jssa_layout* L, const void* Q, const void* K, const void* V,
                              const int32_t* seq_lens, int32_t window, float sm_scale, void* O,
                              float* lse, void* workspace, size_t ws_bytes, void* stream);

/*
 * Spectral calibration of the basis (§3.2, §A.4, §B.1-§B.3; offline, once per layer):
 *   P_h = the top-r eigenvectors of M_h = S_q / tr S_q + S_k / tr S_k, where
 *   S_q = sum_t qbar_t qbar_t^T over the calibration tokens, qbar_t the mean of KV head h's
 *   G query heads at token t, and S_k = sum_t k_t k_t^T (a moment with zero trace
 *   contributes nothing).  This is the library's reading of the marginal bound's closed
 *   form, which the summary does not print: Cauchy-Schwarz on the product of marginals
 *   and the arithmetic-geometric mean of the two unit-trace residuals give the surrogate
 *   2 - tr(P^T M P), minimised by those eigenvectors.
 *   Qc  device bf16 [B, Hq, n_tokens, d_k], contiguous: the calibration queries;
 *   K   the layout's key cache; rows [0, n_tokens) of every sequence (n_tokens <= T_cap);
 *   P   device fp32 [Hkv, d_k, r] out: columns in descending eigenvalue order, each
 *       column's largest-magnitude entry positive (lowest index on ties);
 *   eigvals  device fp64 [Hkv, d_k] out (nullable): the eigenvalues of M_h, descending.
 * Moments in fp64 (exact products of bf16), eigenvectors by cyclic Jacobi in fp64 (one
 * 8-CTA cluster per KV head).  d_k must be a multiple of 64.  The workspace holds the
 * status word: a diagonalisation that did not converge raises JSSA_DEV_TIMEOUT there.
 */
JSSA_API jssa_status jssa_calibrate_workspace_size(const jssa_layout* L, size_t* bytes);
JSSA_API jssa_status jssa_calibrate(const jssa_layout* L, const void* Qc, const void* K, int64_t n_tokens,
                                    float* P, double* eigvals, void* workspace, size_t ws_bytes, void* stream);

/*
 * Zero a freshly allocated workspace (asynchronously on `stream`): required once before
 * its first use by any compute call, and again after a call that returned an error.
 */
JSSA_API jssa_status jssa_workspace_init(void* workspace, size_t ws_bytes, void* stream);

/*
 * Test of the bounded waits (the paper has no counterpart; this is for checking the
 * library's failure path on a working GPU, without faulting it).  Arms a one-shot request
 * in the workspace, asynchronously on `stream`: the next selection launch that scans with
 * this workspace (jssa_select, jssa_decode_step, jssa_topk; rows of at least k + 1
 * candidates) withholds one bulk copy in the first CTA of row (0, 0), whose wait on it
 * then gives up after wait_limit_us microseconds (1 .. 1,000,000).  The launch returns
 * normally: its device status has JSSA_DEV_TIMEOUT (jssa_read_device_status returns
 * JSSA_ERR_TIMEOUT), row (0, 0) has an empty selection (n_sel = 0, idx all -1; with the
 * attention inside the step, its output is the attention over the window alone, zero
 * without one) and the other rows are unaffected.  The launch disarms the request.
 */
JSSA_API jssa_status jssa_test_withhold_copy(void* workspace, size_t ws_bytes, int32_t wait_limit_us, void* stream);

/*
 * Read and clear the device status word kept in the workspace (JSSA_DEV_* bits).
 * Synchronises `stream`.  Returns JSSA_ERR_DEVICE_CHECK if any bit other than
 * JSSA_DEV_TIMEOUT was set, JSSA_ERR_TIMEOUT if that bit was set, else JSSA_OK.
 */
JSSA_API jssa_status jssa_read_device_status(void* workspace, size_t ws_bytes, int32_t* flags, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* JSSA_H_ */
