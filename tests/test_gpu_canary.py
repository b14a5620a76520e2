"""Canary-guarded outputs: every output of the step is a view into a larger buffer whose margins
hold sentinels; the calls must write the outputs in full and nothing outside them (fused step,
unfused long-cache step, head-shared voting)."""
import pytest
import torch

from tests._problem import Problem
import token_level_sparse_jssa_b200 as jssa
from token_level_sparse_jssa_b200 import synth

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS
PAD = 4096  # sentinel elements on each side


def _guarded(shape, dtype, fill):
    n = 1
    for s in shape:
        n *= s
    buf = torch.full((n + 2 * PAD,), fill, dtype=dtype, device="cuda")
    return buf, buf[PAD:PAD + n].view(*shape)


def _margins_intact(buf, fill):
    return bool(torch.all(buf[:PAD] == fill)) and bool(torch.all(buf[-PAD:] == fill))


@pytest.mark.parametrize("name,kw,voting", [
    ("h128k", dict(B=2, T=9000, k=512), False),                   # fused step
    ("h128k", dict(B=1, Hq=8, Hkv=2, T=140000, k=700), False),    # unfused path (beyond one cluster)
    ("tiny", dict(B=2, T=3000, k=200), True),                     # head-shared voting
])
def test_outputs_stay_inside_their_buffers(name, kw, voting):
    w = W[name].with_(**kw)
    p = Problem(w)
    p.fill_kp()
    ws = p.workspace(w.k)
    ob, O = _guarded((w.B, w.Hq, w.dv), torch.float32, -777.0)
    ib, idx = _guarded((w.B, w.Hkv, w.k), torch.int32, -555)
    nb, nsel = _guarded((w.B, w.Hkv), torch.int32, -333)
    lb, lse = _guarded((w.B, w.Hq), torch.float32, -999.0)
    if voting:
        jssa.vote_select(p.L, p.Q, p.K, p.Kp, p.P, p.seq_lens, 1, w.k, 0, w.sm_scale, idx, nsel, ws)
        jssa.indexed_attn(p.L, p.Q, p.K, p.V, idx, w.k, nsel, p.seq_lens, 0, w.sm_scale, O, lse, ws)
    else:
        jssa.decode_step(p.L, p.Q, p.K, p.V, p.Kp, p.P, p.seq_lens, 1, w.k, 0, w.sm_scale, O, lse, idx, nsel, ws)
    torch.cuda.synchronize()
    code, flags = jssa.read_device_status(ws)
    assert code == 0 and flags == 0
    for buf, fill in ((ob, -777.0), (ib, -555), (nb, -333), (lb, -999.0)):
        assert _margins_intact(buf, fill)
    assert torch.isfinite(O).all() and not (O == -777.0).any()
    assert torch.isfinite(lse).all() and not (lse == -999.0).any()
    assert bool(torch.all(nsel == min(w.k, w.T)))
    assert not (idx == -555).any()
