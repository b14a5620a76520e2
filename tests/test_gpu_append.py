"""Append on write: jssa_append_kv writes the newest key/value rows into the caches, and
the decode step then projects the appended key into the scoring cache (§3.1, §E.1).
Byte work, compared bit for bit."""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import token_level_sparse_jssa_b200 as jssa
from token_level_sparse_jssa_b200 import synth
from tests._problem import Problem, assert_status_clean
from tests._util import u16, f32

pytestmark = pytest.mark.gpu


def test_append_writes_the_rows_and_the_step_projects_them():
    w = synth.WORKLOADS["h128k"].with_(B=3, Hq=8, Hkv=2, T=4096, k=128)
    p = Problem(w, T_cap=4200, seq_lens=[4096, 4000, 17])
    p.fill_kp()
    g = torch.Generator(device="cuda")
    g.manual_seed(3)
    K_new = torch.randn(w.B, w.Hkv, w.dk, generator=g, device="cuda").to(torch.bfloat16)
    V_new = torch.randn(w.B, w.Hkv, w.dv, generator=g, device="cuda").to(torch.bfloat16)
    K0, V0 = p.K.clone(), p.V.clone()
    pos = torch.tensor([4096, 5000, 17], dtype=torch.int32, device="cuda")   # 5000 >= T_cap: not written
    jssa.append_kv(p.L, K_new, V_new, p.K, p.V, pos)
    torch.cuda.synchronize()
    expK, expV = K0.clone(), V0.clone()
    for b in (0, 2):
        expK[b, :, int(pos[b])] = K_new[b]
        expV[b, :, int(pos[b])] = V_new[b]
    assert torch.equal(p.K.view(torch.int16), expK.view(torch.int16))
    assert torch.equal(p.V.view(torch.int16), expV.view(torch.int16))

    # the step over the lengthened sequences projects the appended row (n_new = 1)
    sl = torch.tensor([4097, 4000, 18], dtype=torch.int32, device="cuda")
    ws = p.workspace(w.k)
    O = torch.empty(w.B, w.Hq, w.dv, device="cuda")
    idx = torch.empty(w.B, w.Hkv, w.k, dtype=torch.int32, device="cuda")
    nsel = torch.empty(w.B, w.Hkv, dtype=torch.int32, device="cuda")
    jssa.decode_step(p.L, p.Q, p.K, p.V, p.Kp, p.P, sl, 1, w.k, 0, w.sm_scale, O, None, idx, nsel, ws)
    torch.cuda.synchronize()
    assert_status_clean(ws)
    for b in range(w.B):
        t = int(sl[b]) - 1
        for h in range(w.Hkv):
            want, _ = oracle.project_rows(u16(p.K[b, h, t:t + 1]), f32(p.P[h]))
            np.testing.assert_array_equal(u16(p.Kp[b, h, t:t + 1]), want)


def test_append_in_latent_mode_writes_the_latent_row_only():
    w = synth.WORKLOADS["mla"].with_(B=2, T=512, k=64)
    p = Problem(w)
    K_new = torch.randn(w.B, 1, w.dk, device="cuda").to(torch.bfloat16)
    K0 = p.K.clone()
    pos = torch.tensor([7, 511], dtype=torch.int32, device="cuda")
    jssa.append_kv(p.L, K_new, None, p.K, p.V, pos)
    torch.cuda.synchronize()
    exp = K0.clone()
    exp[0, 0, 7] = K_new[0, 0]
    exp[1, 0, 511] = K_new[1, 0]
    assert torch.equal(p.K.view(torch.int16), exp.view(torch.int16))
    with pytest.raises(jssa.JssaError):   # a value row has no place in latent mode
        jssa.append_kv(p.L, K_new, K_new[..., :w.dv].contiguous(), p.K, p.V, pos)
