"""The bounded waits give up, report and return: the failure path on a working GPU.

Every wait of the selection kernels on an mbarrier is bounded in time.  These tests arm
the library's one-shot test request (jssa_test_withhold_copy): the next selection launch
withholds one bulk copy in the first CTA of row (0, 0), so that CTA's wait on it can
never complete and gives up after a short limit.  Nothing faults and nothing hangs: the
call returns, the device status reports the timeout, row (0, 0) comes back as an empty
selection (n_sel = 0, idx all -1; inside the step, attention over the window alone), the
other rows are exactly those of a clean run, and the next call on the same workspace is
clean again.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import token_level_sparse_jssa_b200 as jssa
from token_level_sparse_jssa_b200 import synth
from tests._problem import Problem, check_attention
from tests._util import u16

pytestmark = pytest.mark.gpu

LIMIT_US = 2000
TIMEOUT = 6          # JSSA_ERR_TIMEOUT
DEV_TIMEOUT = 8      # JSSA_DEV_TIMEOUT


def _problem(kp_fp8: bool, T=16384):
    w = synth.WORKLOADS["h128k"].with_(B=2, Hq=8, Hkv=2, T=T, k=256)
    p = Problem(w, kp_fp8=kp_fp8)
    p.fill_kp()
    return p


def _outputs(p, window):
    w = p.w
    idx = torch.full((w.B, w.Hkv, w.k), -7, dtype=torch.int32, device="cuda")
    nsel = torch.full((w.B, w.Hkv), -7, dtype=torch.int32, device="cuda")
    O = torch.full((w.B, w.Hq, w.dv), float("nan"), device="cuda")
    return idx, nsel, O


def _expect_row00_empty_rest_clean(idx, nsel, ref_idx, ref_nsel):
    assert int(nsel[0, 0]) == 0
    assert torch.all(idx[0, 0] == -1)
    rest = torch.ones_like(nsel, dtype=torch.bool)
    rest[0, 0] = False
    assert torch.equal(nsel[rest], ref_nsel[rest])
    assert torch.equal(idx[rest], ref_idx[rest])


@pytest.mark.parametrize("kp_fp8", [False, True], ids=["bf16", "e4m3"])
def test_select_wait_gives_up_and_the_row_is_empty(kp_fp8):
    p = _problem(kp_fp8)
    w = p.w
    ws = p.workspace(w.k)
    ref_idx, ref_nsel, _ = _outputs(p, 0)
    jssa.select(p.L, p.Q, p.K, p.Kp, p.P, p.seq_lens, 0, w.k, 0, ref_idx, ref_nsel, ws)
    assert jssa.read_device_status(ws) == (0, 0)

    idx, nsel, _ = _outputs(p, 0)
    jssa.arm_withheld_copy(ws, LIMIT_US)
    jssa.select(p.L, p.Q, p.K, p.Kp, p.P, p.seq_lens, 0, w.k, 0, idx, nsel, ws)   # returns
    code, flags = jssa.read_device_status(ws)                                       # synchronises
    assert code == TIMEOUT and flags & DEV_TIMEOUT, (code, flags)
    _expect_row00_empty_rest_clean(idx, nsel, ref_idx, ref_nsel)

    # the request was one-shot and the context is usable: the next call is clean again
    idx2, nsel2, _ = _outputs(p, 0)
    jssa.select(p.L, p.Q, p.K, p.Kp, p.P, p.seq_lens, 0, w.k, 0, idx2, nsel2, ws)
    assert jssa.read_device_status(ws) == (0, 0)
    assert torch.equal(idx2, ref_idx) and torch.equal(nsel2, ref_nsel)


@pytest.mark.parametrize("window", [0, 300])
def test_step_wait_gives_up_and_attends_the_window_alone(window):
    p = _problem(False)
    w = p.w
    ws = p.workspace(w.k, window)
    ref_idx, ref_nsel, ref_O = _outputs(p, window)
    jssa.decode_step(p.L, p.Q, p.K, p.V, p.Kp, p.P, p.seq_lens, 0, w.k, window, w.sm_scale, ref_O, None,
                     ref_idx, ref_nsel, ws)
    assert jssa.read_device_status(ws) == (0, 0)

    idx, nsel, O = _outputs(p, window)
    jssa.arm_withheld_copy(ws, LIMIT_US)
    jssa.decode_step(p.L, p.Q, p.K, p.V, p.Kp, p.P, p.seq_lens, 0, w.k, window, w.sm_scale, O, None, idx, nsel, ws)
    code, flags = jssa.read_device_status(ws)
    assert code == TIMEOUT and flags & DEV_TIMEOUT, (code, flags)
    _expect_row00_empty_rest_clean(idx, nsel, ref_idx, ref_nsel)
    G = w.G
    # the other rows' outputs are those of the clean run, bit for bit
    assert torch.equal(O[0, G:], ref_O[0, G:]) and torch.equal(O[1:], ref_O[1:])
    # row (0, 0): attention over the window alone (no selected token), zero without a window
    O00 = O[0, :G].double().cpu().numpy()
    if window == 0:
        assert np.all(O00 == 0.0)
    else:
        T = int(p.seq_lens[0])
        toks = np.arange(T - window, T)
        O_ref, _ = oracle.attention(u16(p.Q[0, :G]), u16(p.K[0, 0, :T]), u16(p.V[0, 0, :T]), toks, w.sm_scale)
        check_attention(O00, O_ref, "window-only row")

    idx2, nsel2, O2 = _outputs(p, window)
    jssa.decode_step(p.L, p.Q, p.K, p.V, p.Kp, p.P, p.seq_lens, 0, w.k, window, w.sm_scale, O2, None, idx2, nsel2,
                     ws)
    assert jssa.read_device_status(ws) == (0, 0)
    assert torch.equal(idx2, ref_idx) and torch.equal(O2, ref_O)


def test_topk_wait_gives_up_and_the_row_is_empty():
    p = _problem(False)
    w = p.w
    ws = p.workspace(w.k)
    scores = synth.random_scores(w.B * w.Hkv, p.T_cap, seed=5, ties=20).cuda().view(w.B, w.Hkv, p.T_cap)
    ref_idx, ref_nsel, _ = _outputs(p, 0)
    jssa.topk(p.L, scores, p.seq_lens, w.k, 0, ref_idx, ref_nsel, ws)
    assert jssa.read_device_status(ws) == (0, 0)

    idx, nsel, _ = _outputs(p, 0)
    jssa.arm_withheld_copy(ws, LIMIT_US)
    jssa.topk(p.L, scores, p.seq_lens, w.k, 0, idx, nsel, ws)
    code, flags = jssa.read_device_status(ws)
    assert code == TIMEOUT and flags & DEV_TIMEOUT, (code, flags)
    _expect_row00_empty_rest_clean(idx, nsel, ref_idx, ref_nsel)

    idx2, nsel2, _ = _outputs(p, 0)
    jssa.topk(p.L, scores, p.seq_lens, w.k, 0, idx2, nsel2, ws)
    assert jssa.read_device_status(ws) == (0, 0)
    assert torch.equal(idx2, ref_idx) and torch.equal(nsel2, ref_nsel)


def test_arming_is_validated_on_the_host():
    p = _problem(False, T=2048)
    ws = p.workspace(p.w.k)
    for bad in (0, -5, 1000001):
        with pytest.raises(jssa.JssaError) as e:
            jssa.arm_withheld_copy(ws, bad)
        assert e.value.code == 1
    with pytest.raises(jssa.JssaError) as e:
        jssa.arm_withheld_copy(ws[:8], LIMIT_US)
    assert e.value.code == 3
