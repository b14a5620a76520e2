"""The allocation-free top-k entry point (jssa_topk_noalloc) against jssa_topk.

jssa_topk_noalloc serves callers that cannot allocate device memory for a workspace
(for example code inside a host framework that owns all device memory, or code that
must not allocate while a stream is captured): its scratch is a fixed array inside the
library.  This file is collected last on purpose, so that a run stopping at the first
failure has already run every other test.
"""
import numpy as np
import pytest
import torch

import token_level_sparse_jssa_b200 as jssa
from token_level_sparse_jssa_b200 import synth

pytestmark = pytest.mark.gpu


def _layout(B, T):
    L = jssa.Layout()
    L.mode, L.B, L.Hq, L.Hkv, L.d_k, L.d_v, L.r, L.out_dtype, L.T_cap = 0, B, 4, 1, 128, 128, 16, 0, T
    for i, v in enumerate((T * 128, T * 128, 128)):
        L.k_stride[i] = v
        L.v_stride[i] = v
    for i, v in enumerate((T * 16, T * 16, 16)):
        L.kp_stride[i] = v
    return L


def _select(fn, L, scores, sl, k, window, B):
    idx = torch.full((B, 1, k), -7, dtype=torch.int32, device="cuda")
    nsel = torch.full((B, 1), -7, dtype=torch.int32, device="cuda")
    fn(idx, nsel)
    torch.cuda.synchronize()
    return idx, nsel


def test_noalloc_topk_matches_the_workspace_entry_point_on_two_calls_in_a_row():
    B, T, k, window = 5, 70000, 1500, 300
    L = _layout(B, T)
    sl = torch.tensor([70000, 69999, 1200, 50000, 1], dtype=torch.int32, device="cuda")
    ws = jssa.alloc_workspace(L, k, window)
    for call, seed in enumerate((11, 12)):  # the second call finds the first call's scratch contents
        scores = synth.random_scores(B, T, seed=seed, ties=40, zeros=8).cuda()
        ref_idx, ref_nsel = _select(lambda i, n: jssa.topk(L, scores, sl, k, window, i, n, ws), L, scores, sl, k,
                                    window, B)
        got_idx, got_nsel = _select(lambda i, n: jssa.topk_noalloc(L, scores, sl, k, window, i, n), L, scores, sl,
                                    k, window, B)
        # index work: bit-exact
        assert torch.equal(got_nsel, ref_nsel), call
        assert torch.equal(got_idx, ref_idx), call


def test_noalloc_topk_rejects_batches_beyond_its_scratch():
    B, T, k = 257, 64, 8   # 257 (sequence, KV head) rows > the 256-row scratch
    L = _layout(B, T)
    scores = torch.zeros(B, T, device="cuda")
    sl = torch.full((B,), T, dtype=torch.int32, device="cuda")
    idx = torch.full((B, 1, k), -7, dtype=torch.int32, device="cuda")
    nsel = torch.full((B, 1), -7, dtype=torch.int32, device="cuda")
    with pytest.raises(jssa.JssaError) as e:
        jssa.topk_noalloc(L, scores, sl, k, 0, idx, nsel)
    assert e.value.code == 7
    torch.cuda.synchronize()
    assert torch.all(idx == -7)
