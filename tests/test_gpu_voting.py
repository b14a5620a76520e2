"""Head-shared soft voting (jssa_vote_select) and cross-layer index reuse against the oracle
("Joint Subspace Sparse Attention for Efficient Long-Context Decoding", §1, §E.3 / Table 15;
App. C: selection at indexer layers, indices reused by the adjacent layers).

The vote's error band is derived from the rigorous fp32 score bound: a score error e shifts a
head's logit by c*e, which moves p_h(t) by at most a factor exp(+-(c e(t) + max_u c e(u)));
the fp32 subtraction, the exponentials (also those that merge the statistics' slices), the
reciprocal and the product add at most ten units in the last place, and the fp32 sum over the
KV heads one more per head.  Selections may differ only by swaps
among tokens whose oracle vote lies within that band of the k-th vote.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import voting
from tests._problem import Problem, check_attention, score_error_bound
from tests._util import u16, f32
import token_level_sparse_jssa_b200 as jssa
from token_level_sparse_jssa_b200 import synth

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS
U = 2.0 ** -24


@pytest.fixture(scope="module", autouse=True)
def _lib():
    jssa.load()
    yield
    torch.cuda.synchronize()


def _vote_band(p, b, n):
    """Oracle votes of sequence b and their per-token error band."""
    w = p.w
    Hkv, G = w.Hkv, w.G
    c = w.sm_scale / G
    s, bands = [], []
    for h in range(Hkv):
        hst = p.host(b, h)
        Kp_or = p.project(hst["K"][:n], hst["P"])
        np.testing.assert_array_equal(hst["Kp"][:n], Kp_or)       # the GPU cache is the oracle's
        qs = oracle.query_proj(hst["Q"], hst["P"])
        if p.kp_fp8:
            vals = np.vectorize(oracle.e4m3_to_double, otypes=[np.float64])(Kp_or)
            s.append(oracle.scores_e4m3(qs, Kp_or))
            bands.append(score_error_bound(hst["Q"], hst["P"], vals))
        else:
            s.append(oracle.scores(qs, Kp_or))
            bands.append(score_error_bound(hst["Q"], hst["P"], Kp_or))
    s = np.stack(s)
    ph = voting.head_distributions(s, c)
    v = ph.sum(axis=0)
    x = c * s
    eps = c * np.stack(bands) + np.abs(x) * U
    rel = np.exp(eps + eps.max(axis=1, keepdims=True) + np.abs(x - x.max(axis=1, keepdims=True)) * U + 10 * U) - 1
    band = (ph * rel).sum(axis=0) + Hkv * U * v
    return v, band


def _check_vote_selection(g_idx, g_n, v, band, k):
    or_idx, k_eff = oracle.topk(v, k)
    assert g_n == k_eff
    sel = g_idx[:k_eff]
    assert np.all(g_idx[k_eff:] == -1) and np.all(np.diff(sel) > 0)
    A, B = set(sel.tolist()), set(or_idx[:k_eff].tolist())
    if A == B:
        return True
    kth_t = int(np.argsort(-v, kind="stable")[k_eff - 1])
    for t in A ^ B:
        assert abs(v[t] - v[kth_t]) <= band[t] + band[kth_t], (t, v[t], v[kth_t], band[t], band[kth_t])
    return False


@pytest.mark.parametrize("name,kw,seq,window,fp8", [
    ("tiny", {}, None, 0, False),
    ("h128k", dict(B=2, T=5000, k=256), [5000, 3001], 0, False),
    ("hybrid", dict(B=2, T=4000, k=300), [4000, 1200], 1024, False),
    ("h128k", dict(B=1, Hq=32, Hkv=2, T=3000, k=100), [3000], 0, False),     # G = 16
    ("h128k", dict(B=2, T=600, k=1024), [600, 2000], 0, False),             # k above the candidates in one row
    ("mla", dict(B=2, T=3000, k=300), [3000, 2222], 0, False),              # one latent head: the score ranking
    ("h128k", dict(B=2, T=5000, k=256), [5000, 4000], 0, True),             # E4M3 scoring cache
    ("h128k", dict(B=1, Hq=8, Hkv=2, T=140000, k=1024), [140000], 0, False),  # longer than one cluster's slices
])
def test_vote_select_matches_the_oracle(name, kw, seq, window, fp8):
    w = W[name].with_(**kw)
    p = Problem(w, T_cap=max(seq) if seq else None, seq_lens=seq, kp_fp8=fp8)
    p.fill_kp()
    ws = p.workspace(w.k, window)
    idx = torch.full((w.B, w.Hkv, w.k), -7, dtype=torch.int32, device="cuda")
    nsel = torch.full((w.B, w.Hkv), -7, dtype=torch.int32, device="cuda")
    jssa.vote_select(p.L, p.Q, p.K, p.Kp, p.P, p.seq_lens, 0, w.k, window, w.sm_scale, idx, nsel, ws)
    torch.cuda.synchronize()
    code, flags = jssa.read_device_status(ws)
    assert code == 0 and flags == 0
    for b in range(w.B):
        for h in range(1, w.Hkv):                                   # one set for every KV head
            assert torch.equal(idx[b, h], idx[b, 0]) and int(nsel[b, h]) == int(nsel[b, 0])
        T = int(p.seq_lens[b])
        n = T - min(window, T)
        v, band = _vote_band(p, b, n)
        _check_vote_selection(idx[b, 0].cpu().numpy(), int(nsel[b, 0]), v, band, w.k)


def test_vote_select_projects_the_newest_rows_and_feeds_the_attention():
    w = W["h128k"].with_(B=2, T=4000, k=300)
    p = Problem(w, seq_lens=[4000, 2500])
    p.fill_kp()
    for b, T in enumerate([4000, 2500]):
        p.Kp[b, :, T - 3:T] = 0
    ws = p.workspace(w.k)
    idx = torch.empty((w.B, w.Hkv, w.k), dtype=torch.int32, device="cuda")
    nsel = torch.empty((w.B, w.Hkv), dtype=torch.int32, device="cuda")
    jssa.vote_select(p.L, p.Q, p.K, p.Kp, p.P, p.seq_lens, 3, w.k, 0, w.sm_scale, idx, nsel, ws)
    O = torch.full((w.B, w.Hq, w.dv), float("nan"), device="cuda")
    jssa.indexed_attn(p.L, p.Q, p.K, p.V, idx, w.k, nsel, p.seq_lens, 0, w.sm_scale, O, None, ws)
    torch.cuda.synchronize()
    for b, T in enumerate([4000, 2500]):
        v, band = _vote_band(p, b, T)                                 # also checks the projected rows
        _check_vote_selection(idx[b, 0].cpu().numpy(), int(nsel[b, 0]), v, band, w.k)
        for h in range(w.Hkv):
            hst = p.host(b, h)
            toks = idx[b, h, :int(nsel[b, h])].cpu().numpy()
            O_ref, _ = oracle.attention(hst["Q"], hst["K"], hst["V"], toks, w.sm_scale)
            check_attention(O[b, h * w.G:(h + 1) * w.G].cpu().numpy().astype(np.float64), O_ref, f"b={b} h={h}")


def test_indices_selected_at_one_layer_serve_the_next_layer():
    # an indexer layer selects; the adjacent layer attends over its own K/V at those positions
    w = W["h128k"].with_(B=2, T=6000, k=512)
    pa = Problem(w, seq_lens=[6000, 4100], seed=21)
    pb = Problem(w, seq_lens=[6000, 4100], seed=22)
    pa.fill_kp()
    ws = pa.workspace(w.k)
    idx = torch.empty((w.B, w.Hkv, w.k), dtype=torch.int32, device="cuda")
    nsel = torch.empty((w.B, w.Hkv), dtype=torch.int32, device="cuda")
    jssa.select(pa.L, pa.Q, pa.K, pa.Kp, pa.P, pa.seq_lens, 0, w.k, 0, idx, nsel, ws)
    O = torch.full((w.B, w.Hq, w.dv), float("nan"), device="cuda")
    jssa.indexed_attn(pb.L, pb.Q, pb.K, pb.V, idx, w.k, nsel, pb.seq_lens, 0, w.sm_scale, O, None, ws)
    torch.cuda.synchronize()
    code, flags = jssa.read_device_status(ws)
    assert code == 0 and flags == 0
    for b in range(w.B):
        for h in range(w.Hkv):
            hb = pb.host(b, h)
            toks = idx[b, h, :int(nsel[b, h])].cpu().numpy()
            assert len(toks) == w.k and np.all(np.diff(toks) > 0)
            O_ref, _ = oracle.attention(hb["Q"], hb["K"], hb["V"], toks, w.sm_scale)
            check_attention(O[b, h * w.G:(h + 1) * w.G].cpu().numpy().astype(np.float64), O_ref, f"b={b} h={h}")
