"""Parity at the workloads' full sizes, in the launch configuration the benchmark times
(same shapes, k, window and split policy; fp32 output so that the attention tolerance
applies), on sampled (sequence, KV head) rows that the oracle recomputes one by one."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from tests._problem import Problem, assert_status_clean, check_attention, check_step_rows
from tests._util import u16, f32
import token_level_sparse_jssa_b200 as jssa
from token_level_sparse_jssa_b200 import synth

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS


def _sample_rows(w):
    rows = [(0, 0), (w.B - 1, w.Hkv - 1)]
    if w.B > 2:
        rows.append((w.B // 2, w.Hkv // 2))
    return rows


def _run_step(p, k, window, n_new=1):
    w = p.w
    ws = p.workspace(k, window)
    O = torch.full((w.B, w.Hq, w.dv), float("nan"), device="cuda")
    idx = torch.empty((w.B, w.Hkv, k), dtype=torch.int32, device="cuda")
    nsel = torch.empty((w.B, w.Hkv), dtype=torch.int32, device="cuda")
    jssa.decode_step(p.L, p.Q, p.K, p.V, p.Kp, p.P, p.seq_lens, n_new, k, window, w.sm_scale, O, None, idx, nsel,
                     ws)
    torch.cuda.synchronize()
    return O, idx, nsel, ws


@pytest.mark.parametrize("name", ["tiny", "h128k", "mla"])
def test_full_size_single_step(name):
    w = W[name]
    p = Problem(w)
    p.fill_kp()
    p.Kp[torch.arange(w.B), :, p.seq_lens.long() - 1] = 0  # the step projects the newest key itself
    O, idx, nsel, ws = _run_step(p, w.k, w.window)
    assert int(nsel.min()) == int(nsel.max()) == min(w.k, w.T - w.window)
    check_step_rows(p, w.k, w.window, O, idx, nsel, _sample_rows(w), f"{name} full size", kp_checked=True)
    assert_status_clean(ws)
    del p
    torch.cuda.empty_cache()


def test_full_size_llama8b_appending_loop():
    # the Llama-3.1-8B-shaped layer as its workload runs it: 1000 decode steps, each appending
    # one token (jssa_append_kv writes its K/V row into the cache) that the step projects into
    # the scoring cache on write, with a fresh query batch every step; the selection and the
    # output are checked against the oracle after the first, a middle and the last step
    w = W["llama8b"]
    steps = w.steps
    t0 = w.T - steps
    p = Problem(w, seq_lens=[t0] * w.B)
    new_k = p.K[:, :, t0:w.T].permute(2, 0, 1, 3).contiguous()   # the generated rows, step by step
    new_v = p.V[:, :, t0:w.T].permute(2, 0, 1, 3).contiguous()
    p.K[:, :, t0:].zero_()
    p.V[:, :, t0:].zero_()
    tb = torch.zeros(w.B, dtype=torch.int32, device="cuda")
    jssa.project_keys(p.L, p.K, p.P, p.Kp, t0, t_begin=tb)
    Qs = synth.fresh_queries(w, steps, p.A, device="cuda", seed=11)
    ws = p.workspace(w.k)
    O = torch.empty((w.B, w.Hq, w.dv), device="cuda")
    idx = torch.empty((w.B, w.Hkv, w.k), dtype=torch.int32, device="cuda")
    nsel = torch.empty((w.B, w.Hkv), dtype=torch.int32, device="cuda")
    checked = 0
    for i in range(steps):
        jssa.append_kv(p.L, new_k[i], new_v[i], p.K, p.V, p.seq_lens)   # row seq_len: the new token
        p.seq_lens += 1
        jssa.decode_step(p.L, Qs[i], p.K, p.V, p.Kp, p.P, p.seq_lens, 1, w.k, 0, w.sm_scale, O, None, idx, nsel,
                         ws)
        if i in (0, steps // 2, steps - 1):
            torch.cuda.synchronize()
            assert int(p.seq_lens.min()) == int(p.seq_lens.max()) == t0 + i + 1
            p.Q = Qs[i].contiguous()
            check_step_rows(p, w.k, 0, O, idx, nsel, _sample_rows(w), f"llama8b step {i}", kp_checked=True)
            assert_status_clean(ws)
            checked += 1
    assert checked == 3 and int(p.seq_lens.min()) == w.T
    del p
    torch.cuda.empty_cache()


def test_full_size_hybrid_global_and_local_layers():
    # the hybrid model's global layer (selection over [0, T - W) plus the window) and one of
    # its local layers (dense over the last W tokens)
    w = W["hybrid"]
    p = Problem(w)
    p.fill_kp()
    O, idx, nsel, ws = _run_step(p, w.k, w.window, n_new=0)
    check_step_rows(p, w.k, w.window, O, idx, nsel, _sample_rows(w), "hybrid global", kp_checked=True)
    assert_status_clean(ws)
    O_loc = torch.full((w.B, w.Hq, w.dv), float("nan"), device="cuda")
    jssa.dense_decode(p.L, p.Q, p.K, p.V, p.seq_lens, w.window, w.sm_scale, O_loc, ws=ws)
    torch.cuda.synchronize()
    G = w.G
    for (b, h) in _sample_rows(w):
        hst = p.host(b, h)
        T = int(p.seq_lens[b])
        O_ref, _ = oracle.attention(hst["Q"], hst["K"], hst["V"], np.arange(T - w.window, T), w.sm_scale)
        check_attention(O_loc[b, h * G:(h + 1) * G].cpu().numpy().astype(np.float64), O_ref,
                        f"hybrid local b={b} h={h}")
    assert_status_clean(ws)
    del p
    torch.cuda.empty_cache()


@pytest.mark.parametrize("k", [512, 4096])
def test_full_size_h128k_budget_sweep(k):
    # the 128K workload at the other budgets of its sweep (k = 4096 fills each CTA's token list)
    w = W["h128k"].with_(k=k)
    p = Problem(w)
    p.fill_kp()
    O, idx, nsel, ws = _run_step(p, k, 0, n_new=0)
    assert int(nsel.min()) == int(nsel.max()) == k
    check_step_rows(p, k, 0, O, idx, nsel, _sample_rows(w), f"h128k k={k}")
    assert_status_clean(ws)
    del p
    torch.cuda.empty_cache()
