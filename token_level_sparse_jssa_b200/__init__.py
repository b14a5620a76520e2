"""JSSA decode step on B200 (sm_100a): C-ABI CUDA library (libjssa.so) and its binding.

The decode step of Joint Subspace Sparse Attention (arXiv 2610.19026v1): score a
projected-key cache with the projected group query, select the top-k tokens per
(sequence, KV head), and run gather-free indexed flash-decode over the selected rows
of the standard [B, Hkv, T, d] bf16 cache, merging split partials by log-sum-exp.

Importing this package does not load the CUDA library; the first call does, and
fails loudly if it has not been built.
"""
from ._binding import (  # noqa: F401
    EXPORTS, KP_BF16, KP_FP8_E4M3, LIB_PATH, MODE_GQA, MODE_MLA, OUT_BF16, OUT_F32, JssaError, Layout,
    alloc_calibration_workspace, alloc_gather_buffer, alloc_workspace, append_kv, arm_withheld_copy, calibrate,
    copy_mapped,
    decode_step, gather_decode,
    dense_decode, indexed_attn, load, make_layout, project_keys, read_device_status, score, select, status_string, topk,
    topk_noalloc, version, vote_select, workspace_init, workspace_size)
