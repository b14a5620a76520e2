// Internal launch interface between the C ABI layer (api.cu) and the kernel files.
// Host-side only; every launcher enqueues on `stream` and returns the launch error.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace jssa {

struct ProjectArgs {
  const void* K;
  int64_t ks[3];
  const float* P;
  void* Kp;
  int64_t ps[3];
  int kp_fp8;               // Kp elements are E4M3 bytes (else bf16)
  const int32_t* t_begin;   // nullable: then seq_lens[b] - n_tokens
  const int32_t* seq_lens;
  int64_t n_tokens;
  int B, Hkv, d, r;
  int64_t T_cap;
  int* status;
};
cudaError_t launch_project_keys(const ProjectArgs& a, cudaStream_t s);

// Append on write: the newest K (and V) row of every (sequence, KV head) into row t_pos[b].
struct AppendArgs {
  const void* K_new;   // [B, Hkv, dk] contiguous
  const void* V_new;   // [B, Hkv, dv] contiguous, nullable
  void* K;
  int64_t ks[3];
  void* V;
  int64_t vs[3];
  const int32_t* t_pos;
  int B, Hkv, dk, dv;
  int64_t T_cap;
};
cudaError_t launch_append_rows(const AppendArgs& a, cudaStream_t s);
// Copy of n16 16-byte words between device-addressable buffers (device or mapped pinned host).
cudaError_t launch_copy16(void* dst, const void* src, size_t n16, int num_sms, cudaStream_t s);

// Per-step prologue: projected group queries qs, plus the projection of the newest
// n_new (<= 16) rows of each sequence into Kp.
struct PrologueArgs {
  const void* Q;  // [B, Hq, d]
  const float* P; // [Hkv, d, r]
  float* qs;      // [B*Hkv, r]
  const void* K;
  int64_t ks[3];
  void* Kp;
  int64_t ps[3];
  int kp_fp8;       // Kp elements are E4M3 bytes (else bf16)
  const int32_t* seq_lens;
  int* counters;    // nullable: [B*Hkv] attention arrival counters zeroed here
  int n_new;
  int B, Hq, Hkv, d, r;
  int64_t T_cap;
  int* status;
};
cudaError_t launch_step_prologue(const PrologueArgs& a, cudaStream_t s);

struct ScoreArgs {
  const void* Kp;
  int64_t ps[3];
  int kp_fp8;        // Kp elements are E4M3 bytes (else bf16)
  const float* qs;   // [B*Hkv, r] projected group queries (from the step prologue)
  float* scores;     // [B*Hkv, sc_ld]
  int64_t sc_ld;
  uint32_t* hist;    // nullable: [B*Hkv, 4096] histogram of key bits [31:20], zero on entry
  const int32_t* seq_lens;
  int B, Hkv, r;
  int64_t T_cap;
  int window;
  int* status;
};
cudaError_t launch_score(const ScoreArgs& a, int num_sms, cudaStream_t s);

struct TopkArgs {
  const float* scores;
  int64_t sc_ld;
  uint32_t* hist;   // [B*Hkv, 4096] per-row histogram of key bits [31:20] (from the score scan)
  const int32_t* seq_lens;
  int B, Hkv;
  int64_t T_cap;
  int k, window;
  int32_t* idx;     // [B*Hkv, k]
  int32_t* n_sel;   // [B*Hkv]
  int* status;
};
cudaError_t launch_topk(const TopkArgs& a, cudaStream_t s);
// Standalone path: build the per-row first-digit histogram (hist must be zeroed).
cudaError_t launch_topk_histogram(const TopkArgs& a, int num_sms, cudaStream_t s);
// Allocation-free selection: device address of the built-in histogram scratch on the
// current device (looked up once per device), and the number of rows it holds.
cudaError_t topk_noalloc_scratch(uint32_t** hist);
int topk_noalloc_max_rows();

struct AttnArgs {
  const void* Q;    // [B, Hq, dk]
  const void* K;
  int64_t ks[3];
  const void* V;
  int64_t vs[3];
  const int32_t* idx;    // nullable => dense range
  int idx_ld;
  const int32_t* n_sel;
  const int32_t* seq_lens;
  int B, Hq, Hkv, dk, dv;
  int64_t T_cap;
  int window;
  float sm_scale;
  int64_t list_max;  // host upper bound on the attended list length
  float* part_o;     // [B, Hq, S, dv]
  float* part_lse;   // [B, Hq, S]
  int* counters;     // [B*Hkv] per-row arrival counters, zero on entry, re-armed on exit
  int S, split_len;
  void* O;           // [B, Hq, dv]
  float* lse;        // nullable
  int out_bf16;
  int* status;
  int cluster_merge;  // set by the launcher: the splits of a row form a cluster and merge over DSMEM
};
// Fused selection (query projection, newest-key projection, score scan, top-k) with one
// 2-16 CTA cluster per (sequence, KV head); rows of up to select_max_candidates() tokens.
struct SelectArgs {
  const void* Q;     // [B, Hq, d]
  const float* P;    // [Hkv, d, r]
  const void* K;     // newest rows projected from here
  int64_t ks[3];
  void* Kp;
  int64_t ps[3];
  int kp_fp8;        // Kp elements are E4M3 bytes (else bf16)
  const int32_t* seq_lens;
  int n_new;         // <= select_max_new_rows()
  int B, Hq, Hkv, d, r;
  int64_t T_cap;
  int window, k;
  int per, stages;   // set by the launcher
  int32_t* idx;      // [B*Hkv, k]
  int32_t* n_sel;    // [B*Hkv]
  int* counters;     // nullable: attention arrival counters zeroed here
  int* status;
  int keys_words;    // set by the launcher
  // attention of the selected rows inside the same kernel (GQA, d <= 128): V == nullptr skips it
  const void* V;
  int64_t vs[3];
  float sm_scale;
  void* O;           // [B, Hq, d]
  float* lse;        // nullable
  int out_bf16;
};
cudaError_t launch_select(const SelectArgs& a, int num_sms, cudaStream_t s);
cudaError_t launch_select_fp8(const SelectArgs& a, int num_sms, cudaStream_t s);  // E4M3 Kp, r >= 16
int64_t select_max_candidates();
int select_max_new_rows();

// Gather-then-attend comparator: copy each row's attended K/V rows into [B*Hkv, Lmax, d] buffers.
struct GatherArgs {
  const void* K;
  int64_t ks[3];
  const void* V;
  int64_t vs[3];
  const int32_t* idx;
  int idx_ld;
  const int32_t* n_sel;
  const int32_t* seq_lens;
  int B, Hkv, d, window;
  int64_t T_cap, Lmax;
  void* Kg;
  void* Vg;
  int32_t* glen;   // [B*Hkv] attended positions per row
  int* status;
};
cudaError_t launch_gather_rows(const GatherArgs& a, cudaStream_t s);

// Spectral calibration of the basis: second moments of the group-mean query and of the key
// over calibration tokens, then the top-r eigenvectors of their unit-trace sum.
struct CalibArgs {
  const void* Qc;     // [B, Hq, n_tokens, d] bf16, contiguous
  const void* K;      // cache rows [0, n_tokens) of every sequence
  int64_t ks[3];
  int64_t n_tokens;
  int B, Hq, Hkv, d, r;
  float* P;           // [Hkv, d, r] out
  double* eigvals;    // nullable: [Hkv, d] out, descending
  double* acc;        // [Hkv, 2, d, d] scratch
  double* jac;        // [Hkv, 3, d, d] scratch
  double* jac_off;    // [Hkv, 2, 8] scratch
  int* status;
};
size_t calib_workspace_doubles(int Hkv, int d);
cudaError_t launch_calibrate(const CalibArgs& a, cudaStream_t s);

// Head-shared soft voting over the fp32 score rows of the unfused scan.
struct VoteArgs {
  float* scores;          // [B*Hkv, sc_ld]; row b*Hkv receives the votes of sequence b
  int64_t sc_ld;
  double* stats;          // [B*Hkv, 8 slices, 2] (max logit, sum of exponentials)
  const int32_t* seq_lens;
  int B, Hkv;
  int64_t T_cap;
  int window, k;
  float c;                // logit scale: sm_scale / G
  const int32_t* idx_shared;    // [B, k] the selection over the vote rows
  const int32_t* nsel_shared;   // [B]
  int32_t* idx;           // [B*Hkv, k] out
  int32_t* n_sel;         // [B*Hkv] out
  int* status;
};
cudaError_t launch_vote_stats(const VoteArgs& a, cudaStream_t s);      // stats, then the votes
cudaError_t launch_vote_broadcast(const VoteArgs& a, cudaStream_t s);

// Split policy of the GQA attention, shared by the workspace sizing and the launch.
void attn_split_policy(bool indexed, int rows, int64_t list_max, int num_sms, int d, int* S, int* split_len);
cudaError_t launch_attention(const AttnArgs& a, cudaStream_t s);   // GQA path
// MLA attention, indexed or dense, many tiles per CTA with the split merge in a cluster of S
// CTAs per (sequence, head half); S from mla_split_groups, split_len = tokens per CTA.
int mla_split_groups(int B, int num_sms);
cudaError_t launch_mla_split(const AttnArgs& a, bool dense, cudaStream_t s);

}  // namespace jssa
