// C ABI of libjssa.so (declared in include/jssa.h): host-side validation, workspace
// carving, split policy and the launch sequence of each entry point.  No entry point
// allocates, frees or synchronises, except jssa_read_device_status.
#include <cstdio>
#include <cstring>

#include "jssa.h"
#include "common.cuh"
#include "launch.h"

namespace jssa {
namespace {

constexpr size_t kAlign = 256;
constexpr int kMaxDevices = 64;
constexpr int64_t kMaxK = 1 << 24;
constexpr int kMaxPrologueRows = 16;  // appended rows projected inside the step prologue

size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

int num_sms_current() {
  static int cache[kMaxDevices] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return -1;
    cache[dev] = n;
  }
  return cache[dev];
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool is_pow2_in(int x, int lo, int hi) { return x >= lo && x <= hi && (x & (x - 1)) == 0; }

jssa_status check_layout(const jssa_layout* L) {
  if (!L) return JSSA_ERR_INVALID_ARG;
  if (L->mode != JSSA_MODE_GQA && L->mode != JSSA_MODE_MLA) return JSSA_ERR_INVALID_ARG;
  if (L->B < 1 || L->Hq < 1 || L->Hkv < 1 || L->d_k < 1 || L->d_v < 1 || L->r < 1 || L->T_cap < 1)
    return JSSA_ERR_INVALID_ARG;
  if (L->T_cap > (int64_t(1) << 31) - 1) return JSSA_ERR_INVALID_ARG;
  if (L->Hq % L->Hkv != 0) return JSSA_ERR_INVALID_ARG;
  if (L->r > L->d_k || L->d_v > L->d_k) return JSSA_ERR_INVALID_ARG;
  if (L->out_dtype != JSSA_OUT_F32 && L->out_dtype != JSSA_OUT_BF16) return JSSA_ERR_INVALID_ARG;
  if (L->kp_dtype != JSSA_KP_BF16 && L->kp_dtype != JSSA_KP_FP8_E4M3) return JSSA_ERR_INVALID_ARG;
  if (L->kp_dtype == JSSA_KP_FP8_E4M3 && L->r < 16) return JSSA_ERR_UNSUPPORTED;  // rows under 16 bytes
  const int64_t kp_align = (L->kp_dtype == JSSA_KP_FP8_E4M3) ? 16 : 8;  // elements per 16 bytes
  if (L->B > 1024) return JSSA_ERR_UNSUPPORTED;
  for (int i = 0; i < 3; ++i) {
    if (L->k_stride[i] < 0 || L->v_stride[i] < 0 || L->kp_stride[i] < 0) return JSSA_ERR_INVALID_ARG;
    if (L->k_stride[i] % 8 || L->v_stride[i] % 8) return JSSA_ERR_INVALID_ARG;
    if (L->kp_stride[i] % kp_align) return JSSA_ERR_INVALID_ARG;
  }
  if (L->k_stride[2] < L->d_k || L->v_stride[2] < L->d_v) return JSSA_ERR_INVALID_ARG;
  if (L->kp_stride[2] != L->r) return JSSA_ERR_UNSUPPORTED;  // Kp rows are streamed as one block
  if (!is_pow2_in(L->r, 8, 64)) return JSSA_ERR_UNSUPPORTED;
  const int G = L->Hq / L->Hkv;
  if (L->mode == JSSA_MODE_GQA) {
    if (L->d_k != L->d_v) return JSSA_ERR_UNSUPPORTED;
    if (L->d_k != 64 && L->d_k != 128 && L->d_k != 256) return JSSA_ERR_UNSUPPORTED;
    if (!is_pow2_in(G, 1, 16)) return JSSA_ERR_UNSUPPORTED;
  } else {
    if (L->Hkv != 1 || L->d_k != 576 || L->d_v != 512 || L->Hq != 128) return JSSA_ERR_UNSUPPORTED;
  }
  return JSSA_OK;
}

struct Workspace {
  int* status;
  float* qs;
  uint32_t* hist;   // [rows, 4096] first radix digit of the selection
  float* scores;    // [rows, sc_ld]
  int64_t sc_ld;
  int32_t* idx;
  int32_t* n_sel;
  int* counters;    // [rows] split arrival counters of the attention
  float* part_lse;
  float* part_o;
  int S_cap;
  size_t bytes;
};

// Carve the workspace for (layout, k, window).  With base == nullptr only sizes.
jssa_status carve(const jssa_layout* L, int64_t k, int64_t window, void* base, Workspace* w) {
  const int num_sms = num_sms_current();
  if (num_sms <= 0) return JSSA_ERR_CUDA;
  const int rows = L->B * L->Hkv;
  // partials for every split count a call with this (k, window) can use
  int S_cap = 1, S = 1, len = 0;
  if (L->mode != JSSA_MODE_MLA) {  // (the MLA kernel merges its splits inside a cluster: no partials)
    attn_split_policy(true, rows, min64(k + window, L->T_cap), num_sms, L->d_k, &S, &len);
    S_cap = S > S_cap ? S : S_cap;
    attn_split_policy(false, rows, L->T_cap, num_sms, L->d_k, &S, &len);
    S_cap = S > S_cap ? S : S_cap;
  }
  if (window > 0 && L->mode != JSSA_MODE_MLA) {
    attn_split_policy(false, rows, min64(window, L->T_cap), num_sms, L->d_k, &S, &len);
    S_cap = S > S_cap ? S : S_cap;
  }
  size_t off = 0;
  auto take = [&](size_t n) {
    const size_t o = off;
    off += align_up(n);
    return o;
  };
  const size_t o_status = take(sizeof(int));
  const size_t o_qs = take(sizeof(float) * rows * L->r);
  const size_t o_hist = take(sizeof(uint32_t) * static_cast<size_t>(rows) * 4096);
  const int64_t sc_ld = ceil_div(L->T_cap, 32) * 32;  // 128-byte aligned rows for bulk staging
  const size_t o_scores = take(sizeof(float) * static_cast<size_t>(rows) * sc_ld);
  const size_t o_idx = take(sizeof(int32_t) * static_cast<size_t>(rows) * k);
  const size_t o_nsel = take(sizeof(int32_t) * rows);
  const size_t o_cnt = take(sizeof(int) * rows);
  const size_t o_lse = take(sizeof(float) * static_cast<size_t>(L->B) * L->Hq * S_cap);
  const size_t o_po = take(sizeof(float) * static_cast<size_t>(L->B) * L->Hq * S_cap * L->d_v);
  w->bytes = off;
  w->S_cap = S_cap;
  char* p = static_cast<char*>(base);
  w->status = p ? reinterpret_cast<int*>(p + o_status) : nullptr;
  w->qs = p ? reinterpret_cast<float*>(p + o_qs) : nullptr;
  w->hist = p ? reinterpret_cast<uint32_t*>(p + o_hist) : nullptr;
  w->scores = p ? reinterpret_cast<float*>(p + o_scores) : nullptr;
  w->sc_ld = sc_ld;
  w->idx = p ? reinterpret_cast<int32_t*>(p + o_idx) : nullptr;
  w->n_sel = p ? reinterpret_cast<int32_t*>(p + o_nsel) : nullptr;
  w->counters = p ? reinterpret_cast<int*>(p + o_cnt) : nullptr;
  w->part_lse = p ? reinterpret_cast<float*>(p + o_lse) : nullptr;
  w->part_o = p ? reinterpret_cast<float*>(p + o_po) : nullptr;
  return JSSA_OK;
}

jssa_status get_ws(const jssa_layout* L, int64_t k, int64_t window, void* ws, size_t ws_bytes, Workspace* w) {
  if (!ws || !aligned(ws, kAlign)) return JSSA_ERR_WORKSPACE;
  jssa_status st = carve(L, k, window, ws, w);
  if (st != JSSA_OK) return st;
  if (ws_bytes < w->bytes) return JSSA_ERR_WORKSPACE;
  return JSSA_OK;
}

// Arms the one-shot test of the bounded waits (words 1 and 2 after the status word).
__global__ void arm_wait_test_kernel(int* status, int limit_us) {
  status[2] = limit_us;
  status[1] = 1;
}

jssa_status cu(cudaError_t e) {
  if (e == cudaSuccess) return JSSA_OK;
  if (e == cudaErrorNotSupported) return JSSA_ERR_UNSUPPORTED;
  return JSSA_ERR_CUDA;
}

ProjectArgs project_args(const jssa_layout* L, const void* K, const float* P, void* Kp, const int32_t* t_begin,
                         const int32_t* seq_lens, int64_t n, int* status) {
  ProjectArgs a{};
  a.K = K;
  memcpy(a.ks, L->k_stride, sizeof a.ks);
  a.P = P;
  a.Kp = Kp;
  memcpy(a.ps, L->kp_stride, sizeof a.ps);
  a.kp_fp8 = (L->kp_dtype == JSSA_KP_FP8_E4M3);
  a.t_begin = t_begin;
  a.seq_lens = seq_lens;
  a.n_tokens = n;
  a.B = L->B;
  a.Hkv = L->Hkv;
  a.d = L->d_k;
  a.r = L->r;
  a.T_cap = L->T_cap;
  a.status = status;
  return a;
}

jssa_status run_prologue(const jssa_layout* L, const void* Q, const float* P, const void* K, void* Kp,
                         const int32_t* seq_lens, int n_new, const Workspace& w, cudaStream_t s) {
  PrologueArgs q{};
  q.Q = Q;
  q.P = P;
  q.qs = w.qs;
  q.K = K;
  memcpy(q.ks, L->k_stride, sizeof q.ks);
  q.Kp = Kp;
  memcpy(q.ps, L->kp_stride, sizeof q.ps);
  q.kp_fp8 = (L->kp_dtype == JSSA_KP_FP8_E4M3);
  q.seq_lens = seq_lens;
  q.counters = w.counters;
  q.n_new = n_new;
  q.B = L->B;
  q.Hq = L->Hq;
  q.Hkv = L->Hkv;
  q.d = L->d_k;
  q.r = L->r;
  q.T_cap = L->T_cap;
  q.status = w.status;
  return cu(launch_step_prologue(q, s));
}

jssa_status run_score(const jssa_layout* L, const void* Kp, const int32_t* seq_lens, int window, float* scores,
                      int64_t sc_ld, const Workspace& w, cudaStream_t s, bool with_hist = true) {
  ScoreArgs a{};
  a.Kp = Kp;
  memcpy(a.ps, L->kp_stride, sizeof a.ps);
  a.kp_fp8 = (L->kp_dtype == JSSA_KP_FP8_E4M3);
  a.qs = w.qs;
  a.scores = scores;
  a.sc_ld = sc_ld;
  a.hist = with_hist ? w.hist : nullptr;
  a.seq_lens = seq_lens;
  a.B = L->B;
  a.Hkv = L->Hkv;
  a.r = L->r;
  a.T_cap = L->T_cap;
  a.window = window;
  a.status = w.status;
  return cu(launch_score(a, num_sms_current(), s));
}

jssa_status run_topk(const jssa_layout* L, const float* scores, int64_t sc_ld, const int32_t* seq_lens, int k,
                     int window, int32_t* idx, int32_t* n_sel, const Workspace& w, bool build_hist, cudaStream_t s) {
  TopkArgs a{};
  a.scores = scores;
  a.sc_ld = sc_ld;
  a.hist = w.hist;
  a.seq_lens = seq_lens;
  a.B = L->B;
  a.Hkv = L->Hkv;
  a.T_cap = L->T_cap;
  a.k = k;
  a.window = window;
  a.idx = idx;
  a.n_sel = n_sel;
  a.status = w.status;
  if (build_hist) {  // standalone selection: the first-digit histogram is not there yet
    jssa_status st = cu(cudaMemsetAsync(w.hist, 0, sizeof(uint32_t) * 4096 * L->B * L->Hkv, s));
    if (st != JSSA_OK) return st;
    st = cu(launch_topk_histogram(a, num_sms_current(), s));
    if (st != JSSA_OK) return st;
  }
  return cu(launch_topk(a, s));
}

jssa_status run_attention(const jssa_layout* L, const void* Q, const void* K, const void* V, const int32_t* idx,
                          int idx_ld, const int32_t* n_sel, const int32_t* seq_lens, int window, float sm_scale,
                          void* O, float* lse, const Workspace& w, bool counters_zeroed, cudaStream_t s) {
  if (!counters_zeroed && L->mode != JSSA_MODE_MLA) {  // (the MLA kernel keeps no arrival counters)
    jssa_status st = cu(cudaMemsetAsync(w.counters, 0, sizeof(int) * L->B * L->Hkv, s));
    if (st != JSSA_OK) return st;
  }
  AttnArgs a{};
  a.Q = Q;
  a.K = K;
  memcpy(a.ks, L->k_stride, sizeof a.ks);
  a.V = V;
  memcpy(a.vs, L->v_stride, sizeof a.vs);
  a.idx = idx;
  a.idx_ld = idx_ld;
  a.n_sel = n_sel;
  a.seq_lens = seq_lens;
  a.B = L->B;
  a.Hq = L->Hq;
  a.Hkv = L->Hkv;
  a.dk = L->d_k;
  a.dv = L->d_v;
  a.T_cap = L->T_cap;
  a.window = window;
  a.sm_scale = sm_scale;
  const bool indexed = idx != nullptr;
  a.list_max = indexed ? static_cast<int64_t>(idx_ld) + window : (window > 0 ? window : L->T_cap);
  if (a.list_max > L->T_cap) a.list_max = L->T_cap;
  if (L->mode == JSSA_MODE_MLA) {  // token groups merged inside a cluster per (sequence, head half)
    a.S = mla_split_groups(L->B, num_sms_current());
    a.split_len = static_cast<int>(ceil_div(a.list_max > 0 ? a.list_max : 1, a.S));
    a.O = O;
    a.lse = lse;
    a.out_bf16 = (L->out_dtype == JSSA_OUT_BF16);
    a.status = w.status;
    return cu(launch_mla_split(a, !indexed, s));
  }
  attn_split_policy(indexed, L->B * L->Hkv, a.list_max, num_sms_current(), L->d_k, &a.S, &a.split_len);
  if (a.S > w.S_cap) return JSSA_ERR_WORKSPACE;
  a.part_o = w.part_o;
  a.part_lse = w.part_lse;
  a.counters = w.counters;
  a.O = O;
  a.lse = lse;
  a.out_bf16 = (L->out_dtype == JSSA_OUT_BF16);
  a.status = w.status;
  return cu(launch_attention(a, s));  // merges in its last CTA per row
}

// Attention to run inside the selection kernel (nullptr: none).
struct FusedAttn {
  const void* V;
  float sm_scale;
  void* O;
  float* lse;
};

// The selection half of the step: newest-key projection, query projection, scan, top-k;
// with `fa`, also the attention of the selected rows when the selection kernel can run it
// (*fused is then set).
jssa_status run_select(const jssa_layout* L, const void* Q, const void* K, void* Kp, const float* P,
                       const int32_t* seq_lens, int n_new, int k, int window, int32_t* idx, int32_t* nsel,
                       const Workspace& w, cudaStream_t s, const FusedAttn* fa = nullptr, bool* fused = nullptr) {
  if (fused) *fused = false;
  jssa_status st = JSSA_OK;
  if (n_new > kMaxPrologueRows) {  // long appends go through the bulk projection kernel
    ProjectArgs pa = project_args(L, K, P, Kp, nullptr, seq_lens, n_new, w.status);
    st = cu(launch_project_keys(pa, s));
    if (st != JSSA_OK) return st;
  }
  const int n_in = n_new > kMaxPrologueRows ? 0 : n_new;
  if (L->T_cap <= select_max_candidates()) {
    // rows that fit a cluster's shared memory: projections, scan and top-k in one kernel
    SelectArgs sa{};
    sa.Q = Q;
    sa.P = P;
    sa.K = K;
    memcpy(sa.ks, L->k_stride, sizeof sa.ks);
    sa.Kp = Kp;
    memcpy(sa.ps, L->kp_stride, sizeof sa.ps);
    sa.kp_fp8 = (L->kp_dtype == JSSA_KP_FP8_E4M3);
    sa.seq_lens = seq_lens;
    sa.n_new = n_in;
    sa.B = L->B;
    sa.Hq = L->Hq;
    sa.Hkv = L->Hkv;
    sa.d = L->d_k;
    sa.r = L->r;
    sa.T_cap = L->T_cap;
    sa.window = window;
    sa.k = k;
    sa.idx = idx;
    sa.n_sel = nsel;
    sa.counters = w.counters;
    sa.status = w.status;
    if (fa && L->mode == JSSA_MODE_GQA) {
      sa.V = fa->V;
      memcpy(sa.vs, L->v_stride, sizeof sa.vs);
      sa.sm_scale = fa->sm_scale;
      sa.O = fa->O;
      sa.lse = fa->lse;
      sa.out_bf16 = (L->out_dtype == JSSA_OUT_BF16);
      const cudaError_t e = launch_select(sa, num_sms_current(), s);
      if (e == cudaSuccess) {
        if (fused) *fused = true;
        return JSSA_OK;
      }
      if (e != cudaErrorNotSupported) return cu(e);
      (void)cudaGetLastError();
      sa.V = nullptr;  // this shape keeps the attention in its own kernel
    }
    return cu(launch_select(sa, num_sms_current(), s));
  }
  st = run_prologue(L, Q, P, K, Kp, seq_lens, n_in, w, s);
  if (st != JSSA_OK) return st;
  st = run_score(L, Kp, seq_lens, window, w.scores, w.sc_ld, w, s);
  if (st != JSSA_OK) return st;
  return run_topk(L, w.scores, w.sc_ld, seq_lens, k, window, idx, nsel, w, false, s);
}

}  // namespace
}  // namespace jssa

using namespace jssa;

extern "C" {

const char* jssa_status_string(jssa_status s) {
  switch (s) {
    case JSSA_OK: return "ok";
    case JSSA_ERR_INVALID_ARG: return "invalid argument";
    case JSSA_ERR_UNSUPPORTED: return "unsupported shape or mode";
    case JSSA_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case JSSA_ERR_CUDA: return "CUDA error";
    case JSSA_ERR_DEVICE_CHECK: return "device-side check failed";
    case JSSA_ERR_TIMEOUT: return "bounded wait timed out";
    case JSSA_ERR_SCRATCH_LIMIT: return "request exceeds the built-in scratch of the allocation-free entry point";
  }
  return "unknown status";
}

int32_t jssa_version(void) { return 10200; }

jssa_status jssa_workspace_size(const jssa_layout* L, int32_t k, int32_t window, size_t* bytes) {
  jssa_status st = check_layout(L);
  if (st != JSSA_OK) return st;
  if (!bytes || k < 1 || k > kMaxK || window < 0) return JSSA_ERR_INVALID_ARG;
  Workspace w{};
  st = carve(L, k, window, nullptr, &w);
  if (st != JSSA_OK) return st;
  *bytes = w.bytes;
  return JSSA_OK;
}

jssa_status jssa_project_keys(const jssa_layout* L, const void* K, const float* P, void* Kp, const int32_t* t_begin,
                              const int32_t* seq_lens, int64_t n_tokens, void* stream) {
  jssa_status st = check_layout(L);
  if (st != JSSA_OK) return st;
  if (n_tokens < 0 || n_tokens > L->T_cap) return JSSA_ERR_INVALID_ARG;
  if (n_tokens == 0) return JSSA_OK;
  if (!K || !P || !Kp || (!t_begin && !seq_lens)) return JSSA_ERR_INVALID_ARG;
  if (!aligned(K, 16) || !aligned(Kp, 16) || !aligned(P, 16)) return JSSA_ERR_INVALID_ARG;
  ProjectArgs a = project_args(L, K, P, Kp, t_begin, seq_lens, n_tokens, nullptr);
  return cu(launch_project_keys(a, static_cast<cudaStream_t>(stream)));
}

jssa_status jssa_append_kv(const jssa_layout* L, const void* K_new, const void* V_new, void* K, void* V,
                           const int32_t* t_pos, void* stream) {
  jssa_status st = check_layout(L);
  if (st != JSSA_OK) return st;
  const bool mla = L->mode == JSSA_MODE_MLA;
  if (!K_new || !K || !t_pos || (!mla && (!V_new || !V)) || (mla && V_new)) return JSSA_ERR_INVALID_ARG;
  if (!aligned(K_new, 16) || !aligned(K, 16) || (V_new && (!aligned(V_new, 16) || !aligned(V, 16))) ||
      !aligned(t_pos, 4))
    return JSSA_ERR_INVALID_ARG;
  AppendArgs a{};
  a.K_new = K_new;
  a.V_new = mla ? nullptr : V_new;
  a.K = K;
  memcpy(a.ks, L->k_stride, sizeof a.ks);
  a.V = V;
  memcpy(a.vs, L->v_stride, sizeof a.vs);
  a.t_pos = t_pos;
  a.B = L->B;
  a.Hkv = L->Hkv;
  a.dk = L->d_k;
  a.dv = L->d_v;
  a.T_cap = L->T_cap;
  return cu(launch_append_rows(a, static_cast<cudaStream_t>(stream)));
}

// Address the current device dereferences for p: device (or managed) memory as is, page-locked
// host memory through its mapping; nullptr for pageable host memory or an unknown pointer.
static const void* device_view(const void* p) {
  cudaPointerAttributes at{};
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  switch (at.type) {
    case cudaMemoryTypeDevice:
    case cudaMemoryTypeManaged:
    case cudaMemoryTypeHost: return at.devicePointer;
    default: return nullptr;
  }
}

jssa_status jssa_copy_mapped(void* dst, const void* src, size_t bytes, void* stream) {
  if (bytes == 0) return JSSA_OK;
  if (!dst || !src || bytes % 16 != 0 || !aligned(dst, 16) || !aligned(src, 16)) return JSSA_ERR_INVALID_ARG;
  void* d = const_cast<void*>(device_view(dst));
  const void* sv = device_view(src);
  if (!d || !sv || !aligned(d, 16) || !aligned(sv, 16)) return JSSA_ERR_INVALID_ARG;
  return cu(launch_copy16(d, sv, bytes / 16, num_sms_current(), static_cast<cudaStream_t>(stream)));
}

jssa_status jssa_score(const jssa_layout* L, const void* Q, const float* P, const void* Kp, const int32_t* seq_lens,
                       int32_t window, float* scores, void* workspace, size_t ws_bytes, void* stream) {
  jssa_status st = check_layout(L);
  if (st != JSSA_OK) return st;
  if (!Q || !P || !Kp || !seq_lens || !scores || window < 0) return JSSA_ERR_INVALID_ARG;
  if (!aligned(Q, 16) || !aligned(P, 16) || !aligned(Kp, 16) || !aligned(scores, 4)) return JSSA_ERR_INVALID_ARG;
  Workspace w{};
  st = get_ws(L, 1, window, workspace, ws_bytes, &w);
  if (st != JSSA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = cu(cudaMemsetAsync(w.hist, 0, sizeof(uint32_t) * 4096 * L->B * L->Hkv, s));
  if (st != JSSA_OK) return st;
  st = run_prologue(L, Q, P, nullptr, nullptr, seq_lens, 0, w, s);
  if (st != JSSA_OK) return st;
  return run_score(L, Kp, seq_lens, window, scores, L->T_cap, w, s);
}

jssa_status jssa_topk(const jssa_layout* L, const float* scores, const int32_t* seq_lens, int32_t k, int32_t window,
                      int32_t* idx, int32_t* n_sel, void* workspace, size_t ws_bytes, void* stream) {
  jssa_status st = check_layout(L);
  if (st != JSSA_OK) return st;
  if (!scores || !seq_lens || !idx || !n_sel || k < 1 || k > kMaxK || window < 0) return JSSA_ERR_INVALID_ARG;
  if (!aligned(scores, 4) || !aligned(idx, 4) || !aligned(n_sel, 4)) return JSSA_ERR_INVALID_ARG;
  Workspace w{};
  st = get_ws(L, k, window, workspace, ws_bytes, &w);
  if (st != JSSA_OK) return st;
  return run_topk(L, scores, L->T_cap, seq_lens, k, window, idx, n_sel, w, true, static_cast<cudaStream_t>(stream));
}

jssa_status jssa_topk_noalloc(const jssa_layout* L, const float* scores, const int32_t* seq_lens, int32_t k,
                              int32_t window, int32_t* idx, int32_t* n_sel, void* stream) {
  jssa_status st = check_layout(L);
  if (st != JSSA_OK) return st;
  if (!scores || !seq_lens || !idx || !n_sel || k < 1 || k > kMaxK || window < 0) return JSSA_ERR_INVALID_ARG;
  if (!aligned(scores, 4) || !aligned(idx, 4) || !aligned(n_sel, 4)) return JSSA_ERR_INVALID_ARG;
  const int rows = L->B * L->Hkv;
  if (rows > topk_noalloc_max_rows()) return JSSA_ERR_SCRATCH_LIMIT;
  uint32_t* hist = nullptr;
  st = cu(topk_noalloc_scratch(&hist));
  if (st != JSSA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the shared scratch keeps the previous call's contents: clear the histograms first
  st = cu(cudaMemsetAsync(hist, 0, sizeof(uint32_t) * 4096 * rows, s));
  if (st != JSSA_OK) return st;
  TopkArgs a{};
  a.scores = scores;
  a.sc_ld = L->T_cap;
  a.hist = hist;
  a.seq_lens = seq_lens;
  a.B = L->B;
  a.Hkv = L->Hkv;
  a.T_cap = L->T_cap;
  a.k = k;
  a.window = window;
  a.idx = idx;
  a.n_sel = n_sel;
  a.status = nullptr;
  st = cu(launch_topk_histogram(a, num_sms_current(), s));
  if (st != JSSA_OK) return st;
  return cu(launch_topk(a, s));
}

jssa_status jssa_indexed_attn(const jssa_layout* L, const void* Q, const void* K, const void* V, const int32_t* idx,
                              int32_t k, const int32_t* n_sel, const int32_t* seq_lens, int32_t window, float sm_scale,
                              void* O, float* lse, void* workspace, size_t ws_bytes, void* stream) {
  jssa_status st = check_layout(L);
  if (st != JSSA_OK) return st;
  if (!Q || !K || !V || !idx || !n_sel || !seq_lens || !O || k < 1 || k > kMaxK || window < 0)
    return JSSA_ERR_INVALID_ARG;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(idx, 4) || !aligned(O, 4))
    return JSSA_ERR_INVALID_ARG;
  Workspace w{};
  st = get_ws(L, k, window, workspace, ws_bytes, &w);
  if (st != JSSA_OK) return st;
  return run_attention(L, Q, K, V, idx, k, n_sel, seq_lens, window, sm_scale, O, lse, w, false,
                       static_cast<cudaStream_t>(stream));
}

jssa_status jssa_select(const jssa_layout* L, const void* Q, const void* K, void* Kp, const float* P,
                        const int32_t* seq_lens, int32_t n_new, int32_t k, int32_t window, int32_t* idx,
                        int32_t* n_sel, void* workspace, size_t ws_bytes, void* stream) {
  jssa_status st = check_layout(L);
  if (st != JSSA_OK) return st;
  if (!Q || !K || !Kp || !P || !seq_lens || !idx || !n_sel || k < 1 || k > kMaxK || window < 0 || n_new < 0 ||
      n_new > L->T_cap)
    return JSSA_ERR_INVALID_ARG;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(Kp, 16) || !aligned(P, 16) || !aligned(idx, 4) ||
      !aligned(n_sel, 4))
    return JSSA_ERR_INVALID_ARG;
  Workspace w{};
  st = get_ws(L, k, window, workspace, ws_bytes, &w);
  if (st != JSSA_OK) return st;
  return run_select(L, Q, K, Kp, P, seq_lens, n_new, k, window, idx, n_sel, w, static_cast<cudaStream_t>(stream));
}

jssa_status jssa_vote_select(const jssa_layout* L, const void* Q, const void* K, void* Kp, const float* P,
                             const int32_t* seq_lens, int32_t n_new, int32_t k, int32_t window, float sm_scale,
                             int32_t* idx, int32_t* n_sel, void* workspace, size_t ws_bytes, void* stream) {
  jssa_status st = check_layout(L);
  if (st != JSSA_OK) return st;
  if (!Q || !K || !Kp || !P || !seq_lens || !idx || !n_sel || k < 1 || k > kMaxK || window < 0 || n_new < 0 ||
      !(sm_scale > 0.f))
    return JSSA_ERR_INVALID_ARG;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(Kp, 16) || !aligned(P, 16) || !aligned(idx, 4) ||
      !aligned(n_sel, 4))
    return JSSA_ERR_INVALID_ARG;
  Workspace w{};
  st = get_ws(L, k, window, workspace, ws_bytes, &w);
  if (st != JSSA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (n_new > kMaxPrologueRows) {
    ProjectArgs pa = project_args(L, K, P, Kp, nullptr, seq_lens, n_new, w.status);
    st = cu(launch_project_keys(pa, s));
    if (st != JSSA_OK) return st;
  }
  st = run_prologue(L, Q, P, K, Kp, seq_lens, n_new > kMaxPrologueRows ? 0 : n_new, w, s);
  if (st != JSSA_OK) return st;
  st = run_score(L, Kp, seq_lens, window, w.scores, w.sc_ld, w, s, false);
  if (st != JSSA_OK) return st;
  VoteArgs v{};
  v.scores = w.scores;
  v.sc_ld = w.sc_ld;
  v.stats = reinterpret_cast<double*>(w.hist);  // free until the vote rows' histograms are built
  v.seq_lens = seq_lens;
  v.B = L->B;
  v.Hkv = L->Hkv;
  v.T_cap = L->T_cap;
  v.window = window;
  v.k = k;
  v.c = sm_scale / static_cast<float>(L->Hq / L->Hkv);
  v.idx_shared = w.idx;
  v.nsel_shared = w.n_sel;
  v.idx = idx;
  v.n_sel = n_sel;
  v.status = w.status;
  st = cu(launch_vote_stats(v, s));
  if (st != JSSA_OK) return st;
  // top-k over the B vote rows (row b of the vote layout is score row b * Hkv)
  jssa_layout Lv = *L;
  Lv.Hkv = 1;
  Lv.Hq = L->Hq / L->Hkv;
  st = run_topk(&Lv, w.scores, w.sc_ld * L->Hkv, seq_lens, k, window, w.idx, w.n_sel, w, true, s);
  if (st != JSSA_OK) return st;
  return cu(launch_vote_broadcast(v, s));
}

jssa_status jssa_decode_step(const jssa_layout* L, const void* Q, const void* K, const void* V, void* Kp,
                             const float* P, const int32_t* seq_lens, int32_t n_new, int32_t k, int32_t window,
                             float sm_scale, void* O, float* lse, int32_t* idx_out, int32_t* n_sel_out, void* workspace,
                             size_t ws_bytes, void* stream) {
  jssa_status st = check_layout(L);
  if (st != JSSA_OK) return st;
  if (!Q || !K || !V || !Kp || !P || !seq_lens || !O || k < 1 || k > kMaxK || window < 0 || n_new < 0 ||
      n_new > L->T_cap)
    return JSSA_ERR_INVALID_ARG;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(Kp, 16) || !aligned(P, 16) || !aligned(O, 4))
    return JSSA_ERR_INVALID_ARG;
  if ((idx_out && !aligned(idx_out, 4)) || (n_sel_out && !aligned(n_sel_out, 4))) return JSSA_ERR_INVALID_ARG;
  Workspace w{};
  st = get_ws(L, k, window, workspace, ws_bytes, &w);
  if (st != JSSA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t* idx = idx_out ? idx_out : w.idx;
  int32_t* nsel = n_sel_out ? n_sel_out : w.n_sel;
  const FusedAttn fa{V, sm_scale, O, lse};
  bool fused = false;
  st = run_select(L, Q, K, Kp, P, seq_lens, n_new, k, window, idx, nsel, w, s, &fa, &fused);
  if (st != JSSA_OK || fused) return st;
  return run_attention(L, Q, K, V, idx, k, nsel, seq_lens, window, sm_scale, O, lse, w, true, s);
}

namespace {
// Bytes of the gather buffer and its pieces: K and V [rows, Lmax, d] bf16, then the row lengths.
size_t gather_layout(const jssa_layout* L, int64_t k, int64_t window, int64_t* Lmax, size_t* off_v,
                     size_t* off_len) {
  *Lmax = k + min64(window, L->T_cap);
  const size_t rows = static_cast<size_t>(L->B) * L->Hkv;
  const size_t kv = align_up(rows * static_cast<size_t>(*Lmax) * L->d_k * 2);
  *off_v = kv;
  *off_len = 2 * kv;
  return 2 * kv + align_up(rows * sizeof(int32_t));
}
}  // namespace

jssa_status jssa_gather_size(const jssa_layout* L, int32_t k, int32_t window, size_t* bytes) {
  jssa_status st = check_layout(L);
  if (st != JSSA_OK) return st;
  if (L->mode == JSSA_MODE_MLA) return JSSA_ERR_UNSUPPORTED;
  if (!bytes || k < 1 || k > kMaxK || window < 0) return JSSA_ERR_INVALID_ARG;
  int64_t Lmax;
  size_t ov, ol;
  *bytes = gather_layout(L, k, window, &Lmax, &ov, &ol);
  return JSSA_OK;
}

jssa_status jssa_gather_decode(const jssa_layout* L, const void* Q, const void* K, const void* V, const int32_t* idx,
                               int32_t k, const int32_t* n_sel, const int32_t* seq_lens, int32_t window,
                               float sm_scale, void* O, float* lse, void* gather_buf, size_t gather_bytes,
                               void* workspace, size_t ws_bytes, void* stream) {
  jssa_status st = check_layout(L);
  if (st != JSSA_OK) return st;
  if (L->mode == JSSA_MODE_MLA) return JSSA_ERR_UNSUPPORTED;
  if (!Q || !K || !V || !idx || !n_sel || !seq_lens || !O || !gather_buf || k < 1 || k > kMaxK || window < 0)
    return JSSA_ERR_INVALID_ARG;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 4) || !aligned(gather_buf, 16))
    return JSSA_ERR_INVALID_ARG;
  int64_t Lmax;
  size_t off_v, off_len;
  const size_t need = gather_layout(L, k, window, &Lmax, &off_v, &off_len);
  if (gather_bytes < need) return JSSA_ERR_WORKSPACE;
  Workspace w{};
  st = get_ws(L, k, window, workspace, ws_bytes, &w);
  if (st != JSSA_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* gb = static_cast<char*>(gather_buf);
  GatherArgs g{};
  g.K = K;
  memcpy(g.ks, L->k_stride, sizeof g.ks);
  g.V = V;
  memcpy(g.vs, L->v_stride, sizeof g.vs);
  g.idx = idx;
  g.idx_ld = k;
  g.n_sel = n_sel;
  g.seq_lens = seq_lens;
  g.B = L->B;
  g.Hkv = L->Hkv;
  g.d = L->d_k;
  g.window = window;
  g.T_cap = L->T_cap;
  g.Lmax = Lmax;
  g.Kg = gb;
  g.Vg = gb + off_v;
  g.glen = reinterpret_cast<int32_t*>(gb + off_len);
  g.status = w.status;
  st = cu(launch_gather_rows(g, s));
  if (st != JSSA_OK) return st;
  // the buffer as a cache of B*Hkv sequences with one KV head and G query heads each
  jssa_layout Lg = *L;
  Lg.B = L->B * L->Hkv;
  Lg.Hkv = 1;
  Lg.Hq = L->Hq / L->Hkv;
  Lg.T_cap = Lmax;
  const int64_t kst[3] = {Lmax * L->d_k, Lmax * L->d_k, L->d_k};
  memcpy(Lg.k_stride, kst, sizeof kst);
  memcpy(Lg.v_stride, kst, sizeof kst);
  const int64_t pst[3] = {Lmax * L->r, Lmax * L->r, L->r};
  memcpy(Lg.kp_stride, pst, sizeof pst);
  int S = 0, len = 0;
  attn_split_policy(false, Lg.B * Lg.Hkv, Lmax, num_sms_current(), Lg.d_k, &S, &len);
  if (S > w.S_cap) return JSSA_ERR_WORKSPACE;
  return run_attention(&Lg, Q, gb, gb + off_v, nullptr, 0, nullptr, g.glen, 0, sm_scale, O, lse, w, false, s);
}

jssa_status jssa_dense_decode(const jssa_layout* L, const void* Q, const void* K, const void* V,
                              const int32_t* seq_lens, int32_t window, float sm_scale, void* O, float* lse,
                              void* workspace, size_t ws_bytes, void* stream) {
  jssa_status st = check_layout(L);
  if (st != JSSA_OK) return st;
  if (!Q || !K || !V || !seq_lens || !O || window < 0) return JSSA_ERR_INVALID_ARG;
  if (!aligned(Q, 16) || !aligned(K, 16) || !aligned(V, 16) || !aligned(O, 4)) return JSSA_ERR_INVALID_ARG;
  Workspace w{};
  st = get_ws(L, 1, window, workspace, ws_bytes, &w);
  if (st != JSSA_OK) return st;
  return run_attention(L, Q, K, V, nullptr, 0, nullptr, seq_lens, window, sm_scale, O, lse, w, false,
                       static_cast<cudaStream_t>(stream));
}

namespace {
size_t calib_bytes(const jssa_layout* L) {
  return align_up(sizeof(int)) + align_up(calib_workspace_doubles(L->Hkv, L->d_k) * sizeof(double));
}
}  // namespace

jssa_status jssa_calibrate_workspace_size(const jssa_layout* L, size_t* bytes) {
  jssa_status st = check_layout(L);
  if (st != JSSA_OK) return st;
  if (!bytes) return JSSA_ERR_INVALID_ARG;
  if (L->d_k % 64 != 0) return JSSA_ERR_UNSUPPORTED;
  *bytes = calib_bytes(L);
  return JSSA_OK;
}

jssa_status jssa_calibrate(const jssa_layout* L, const void* Qc, const void* K, int64_t n_tokens, float* P,
                           double* eigvals, void* workspace, size_t ws_bytes, void* stream) {
  jssa_status st = check_layout(L);
  if (st != JSSA_OK) return st;
  if (L->d_k % 64 != 0) return JSSA_ERR_UNSUPPORTED;
  if (!Qc || !K || !P || n_tokens < 1 || n_tokens > L->T_cap) return JSSA_ERR_INVALID_ARG;
  if (!aligned(Qc, 16) || !aligned(K, 16) || !aligned(P, 4) || (eigvals && !aligned(eigvals, 8)))
    return JSSA_ERR_INVALID_ARG;
  if (!workspace || !aligned(workspace, kAlign) || ws_bytes < calib_bytes(L)) return JSSA_ERR_WORKSPACE;
  unsigned char* base = static_cast<unsigned char*>(workspace);
  double* scratch = reinterpret_cast<double*>(base + align_up(sizeof(int)));
  CalibArgs a{};
  a.Qc = Qc;
  a.K = K;
  memcpy(a.ks, L->k_stride, sizeof a.ks);
  a.n_tokens = n_tokens;
  a.B = L->B;
  a.Hq = L->Hq;
  a.Hkv = L->Hkv;
  a.d = L->d_k;
  a.r = L->r;
  a.P = P;
  a.eigvals = eigvals;
  a.acc = scratch;
  a.jac = scratch + static_cast<size_t>(L->Hkv) * 2 * L->d_k * L->d_k;
  a.jac_off = a.jac + static_cast<size_t>(L->Hkv) * 3 * L->d_k * L->d_k;
  a.status = reinterpret_cast<int*>(base);
  return cu(launch_calibrate(a, static_cast<cudaStream_t>(stream)));
}

jssa_status jssa_workspace_init(void* workspace, size_t ws_bytes, void* stream) {
  if (!workspace || !aligned(workspace, kAlign) || ws_bytes < sizeof(int)) return JSSA_ERR_WORKSPACE;
  return cu(cudaMemsetAsync(workspace, 0, ws_bytes, static_cast<cudaStream_t>(stream)));
}

jssa_status jssa_test_withhold_copy(void* workspace, size_t ws_bytes, int32_t wait_limit_us, void* stream) {
  if (!workspace || !aligned(workspace, kAlign) || ws_bytes < 3 * sizeof(int)) return JSSA_ERR_WORKSPACE;
  if (wait_limit_us < 1 || wait_limit_us > 1000000) return JSSA_ERR_INVALID_ARG;
  arm_wait_test_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<int*>(workspace), wait_limit_us);
  return cu(cudaGetLastError());
}

jssa_status jssa_read_device_status(void* workspace, size_t ws_bytes, int32_t* flags, void* stream) {
  if (!workspace || !aligned(workspace, kAlign) || ws_bytes < sizeof(int)) return JSSA_ERR_WORKSPACE;
  if (!flags) return JSSA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int32_t v = 0;
  if (cudaMemcpyAsync(&v, workspace, sizeof v, cudaMemcpyDeviceToHost, s) != cudaSuccess) return JSSA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return JSSA_ERR_CUDA;
  if (cudaMemsetAsync(workspace, 0, sizeof v, s) != cudaSuccess) return JSSA_ERR_CUDA;
  *flags = v;
  if (v & ~DEVFLAG_TIMEOUT) return JSSA_ERR_DEVICE_CHECK;
  if (v & DEVFLAG_TIMEOUT) return JSSA_ERR_TIMEOUT;
  return JSSA_OK;
}

}  // extern "C"
