"""Parity of the CUDA path (through the C ABI) with the CPU oracle, stage by stage and
end to end, on seeded synthetic inputs shaped like the pages' workloads.

Stages get independent inputs from the generator (the oracle never consumes an
output of the CUDA path): projection from K and P; scoring from Q, P and the
projected cache; top-k from generated score rows; attention from generated index
sets.  The fused step is compared on its selection (bit-exact up to swaps inside the
tie window) and on its output (fp64 oracle on the same index set).
"""
import math

import numpy as np
import pytest
import torch

import oracle
from tests._problem import Problem, check_attention, check_selection, check_step_rows, score_error_bound
from tests._util import u16, f32, rel_l2
import token_level_sparse_jssa_b200 as jssa
from token_level_sparse_jssa_b200 import synth

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS


@pytest.fixture(scope="module", autouse=True)
def _lib():
    jssa.load()
    yield
    torch.cuda.synchronize()


def _assert_status_clean(ws):
    code, flags = jssa.read_device_status(ws)
    assert code == 0 and flags == 0, (code, flags)


# ----------------------------------------------------------------------------- a1 projection
@pytest.mark.parametrize("name,kw", [
    ("tiny", dict(T=700)),
    ("tiny", dict(T=300, r=8, dk=64, dv=64)),
    ("h128k", dict(B=2, T=1100)),
    ("hybrid", dict(B=1, T=515)),
    ("mla", dict(B=2, T=333)),
])
def test_project_keys_is_bit_exact(name, kw):
    w = W[name].with_(**kw)
    p = Problem(w)
    p.fill_kp()
    torch.cuda.synchronize()
    for b in range(w.B):
        for h in range(w.Hkv):
            ref, _ = oracle.project_rows(u16(p.K[b, h]), f32(p.P[h]))
            np.testing.assert_array_equal(u16(p.Kp[b, h]), ref)


def test_project_keys_last_rows_only():
    w = W["tiny"].with_(B=3, T=500)
    p = Problem(w, T_cap=512, seq_lens=[500, 37, 512])
    jssa.project_keys(p.L, p.K, p.P, p.Kp, 3, seq_lens=p.seq_lens)   # rows [T_b-3, T_b)
    torch.cuda.synchronize()
    kp = u16(p.Kp)
    for b, T in enumerate([500, 37, 512]):
        for h in range(w.Hkv):
            ref, _ = oracle.project_rows(u16(p.K[b, h, T - 3:T]), f32(p.P[h]))
            np.testing.assert_array_equal(kp[b, h, T - 3:T], ref)
            assert np.all(kp[b, h, :T - 3] == 0) and np.all(kp[b, h, T:] == 0)


# ----------------------------------------------------------------------------- a2-a3 scoring
@pytest.mark.parametrize("name,kw,seq,window", [
    ("tiny", {}, None, 0),
    ("h128k", dict(B=3, T=5000), [5000, 17, 4097], 0),
    ("hybrid", dict(B=2, T=3000), [3000, 2100], 1024),
    ("tiny", dict(T=900, r=8, dk=64, dv=64, Hq=16, Hkv=1), None, 5),
    ("mla", dict(B=2, T=1200), [1200, 999], 0),
])
def test_score_within_fp32_error_bound(name, kw, seq, window):
    w = W[name].with_(**kw)
    p = Problem(w, seq_lens=seq)
    p.fill_kp()
    ws = p.workspace(1, window)
    scores = torch.full((w.B, w.Hkv, p.T_cap), float("nan"), device="cuda")
    jssa.score(p.L, p.Q, p.P, p.Kp, p.seq_lens, window, scores, ws)
    torch.cuda.synchronize()
    sc = scores.cpu().numpy().astype(np.float64)
    for b in range(w.B):
        T = int(p.seq_lens[b])
        n = T - min(window, T)
        for h in range(w.Hkv):
            hst = p.host(b, h)
            Kp_or, _ = oracle.project_rows(hst["K"][:n], hst["P"])
            np.testing.assert_array_equal(hst["Kp"][:n], Kp_or)
            s_or = oracle.scores(oracle.query_proj(hst["Q"], hst["P"]), Kp_or)
            bound = score_error_bound(hst["Q"], hst["P"], Kp_or)
            err = np.abs(sc[b, h, :n] - s_or)
            assert np.all(err <= bound * 1.0001 + 1e-30), float(np.max(err / np.maximum(bound, 1e-30)))
            assert np.all(np.isnan(sc[b, h, n:])), "entries past the candidates must not be written"
    _assert_status_clean(ws)


# ----------------------------------------------------------------------------- a4 top-k
@pytest.mark.parametrize("rows_T,k,seq,window,ties", [
    ((1, 64), 5, [64], 0, 3),
    ((1, 2048), 128, [2048], 0, 20),
    ((3, 20000), 2048, [20000, 1999, 15001], 0, 50),     # ragged, one row below k
    ((4, 131072), 2048, None, 0, 200),                    # 8-CTA clusters
    ((2, 65536), 1024, [65536, 40000], 1024, 100),        # window shrinks the candidates
    ((2, 4096), 4096, [4096, 100], 0, 10),                # k >= n: select everything
    ((1, 400000), 777, [400000], 0, 100),                 # 16-CTA cluster, large staged slices
    ((1, 600000), 3000, [599999], 0, 100),                # slice larger than shared memory
    ((2, 50000), 1000, [50000, 49000], 0, 30000),         # many exact ties
    ((2, 5000), 1, [5000, 1], 0, 2),
])
def test_topk_is_bit_exact(rows_T, k, seq, window, ties):
    B, T = rows_T
    Hkv = 1
    scores = synth.random_scores(B * Hkv, T, seed=T + k, ties=ties, zeros=8).cuda()
    seq = seq or [T] * B
    L = jssa.Layout()
    L.mode, L.B, L.Hq, L.Hkv, L.d_k, L.d_v, L.r, L.out_dtype, L.T_cap = 0, B, 4, Hkv, 128, 128, 16, 0, T
    for i, v in enumerate((Hkv * T * 128, T * 128, 128)):
        L.k_stride[i] = v
        L.v_stride[i] = v
    for i, v in enumerate((Hkv * T * 16, T * 16, 16)):
        L.kp_stride[i] = v
    sl = torch.tensor(seq, dtype=torch.int32, device="cuda")
    idx = torch.full((B, Hkv, k), -7, dtype=torch.int32, device="cuda")
    nsel = torch.full((B, Hkv), -7, dtype=torch.int32, device="cuda")
    ws = jssa.alloc_workspace(L, k, window)
    jssa.topk(L, scores, sl, k, window, idx, nsel, ws)
    torch.cuda.synchronize()
    _assert_status_clean(ws)
    s_host = scores.cpu().numpy().astype(np.float64)
    for b in range(B):
        n = seq[b] - min(window, seq[b])
        ref, k_eff = oracle.topk(s_host[b, :n], k)
        assert int(nsel[b, 0]) == k_eff
        np.testing.assert_array_equal(idx[b, 0].cpu().numpy(), ref)


def _topk_layout(B, T):
    L = jssa.Layout()
    L.mode, L.B, L.Hq, L.Hkv, L.d_k, L.d_v, L.r, L.out_dtype, L.T_cap = 0, B, 4, 1, 128, 128, 16, 0, T
    for i, v in enumerate((T * 128, T * 128, 128)):
        L.k_stride[i] = v
        L.v_stride[i] = v
    for i, v in enumerate((T * 16, T * 16, 16)):
        L.kp_stride[i] = v
    return L


def test_topk_with_the_winners_bunched_together():
    # increasing scores: all winners sit in the last warps' ranges (their lists overflow)
    B, T, k = 2, 131072, 3000
    scores = torch.arange(B * T, dtype=torch.float32).view(B, T).cuda() / 7.0
    scores[1] = scores[1].flip(0)
    L = _topk_layout(B, T)
    sl = torch.tensor([T, T - 5], dtype=torch.int32, device="cuda")
    idx = torch.empty((B, 1, k), dtype=torch.int32, device="cuda")
    nsel = torch.empty((B, 1), dtype=torch.int32, device="cuda")
    ws = jssa.alloc_workspace(L, k, 0)
    jssa.topk(L, scores, sl, k, 0, idx, nsel, ws)
    torch.cuda.synchronize()
    _assert_status_clean(ws)
    np.testing.assert_array_equal(idx[0, 0].cpu().numpy(), np.arange(T - k, T))
    np.testing.assert_array_equal(idx[1, 0].cpu().numpy(), np.arange(k))


@pytest.mark.parametrize("T,k,levels", [(131072, 2048, 1), (131072, 5000, 3), (70000, 300, 2)])
def test_topk_with_few_distinct_values(T, k, levels):
    # every key of a slice falls in one digit-1 bin: the candidate list overflows and the
    # CTAs scan their whole slices instead; ties resolve to the lowest indices
    B = 2
    g = torch.Generator().manual_seed(T + k)
    vals = torch.tensor([1.5, -0.25, 7.0][:levels])
    scores = vals[torch.randint(0, levels, (B, T), generator=g)].float().cuda()
    L = _topk_layout(B, T)
    sl = torch.tensor([T, T - 17], dtype=torch.int32, device="cuda")
    idx = torch.empty((B, 1, k), dtype=torch.int32, device="cuda")
    nsel = torch.empty((B, 1), dtype=torch.int32, device="cuda")
    ws = jssa.alloc_workspace(L, k, 0)
    jssa.topk(L, scores, sl, k, 0, idx, nsel, ws)
    torch.cuda.synchronize()
    _assert_status_clean(ws)
    s_host = scores.cpu().numpy().astype(np.float64)
    for b in range(B):
        ref, k_eff = oracle.topk(s_host[b, :int(sl[b])], k)
        assert int(nsel[b, 0]) == k_eff
        np.testing.assert_array_equal(idx[b, 0].cpu().numpy(), ref)


# ----------------------------------------------------------------------------- a5-a6 attention
@pytest.mark.parametrize("name,kw,seq,k,window,out", [
    ("tiny", {}, None, 128, 0, 0),
    ("tiny", dict(T=1000, dk=64, dv=64, r=8), None, 100, 0, 0),
    ("h128k", dict(B=2, T=9000), [9000, 4000], 2048, 0, 0),
    ("h128k", dict(B=2, T=3000, Hq=16, Hkv=16), [3000, 2500], 300, 0, 0),     # G = 1
    ("h128k", dict(B=2, T=3000, Hq=16, Hkv=8), [3000, 1700], 400, 0, 0),      # G = 2 (hi/lo parts in one MMA)
    ("h128k", dict(B=1, T=3000, Hq=32, Hkv=4), [3000], 500, 0, 0),           # G = 8
    ("h128k", dict(B=1, T=3000, Hq=32, Hkv=2), [3000], 257, 0, 0),           # G = 16
    ("hybrid", dict(B=2, T=6000), [6000, 1500], 1024, 1024, 0),              # d = 256 + window
    ("hybrid", dict(B=1, T=2000), [2000], 7, 3, 1),                          # bf16 output
    ("mla", dict(B=2, T=3000), [3000, 1234], 700, 0, 0),                     # tensor-core MLA kernel
    ("mla", dict(B=1, T=4100), [4100], 2048, 0, 0),                          # 16 full 128-token tiles
    ("mla", dict(B=3, T=2000), [2000, 333, 1999], 150, 64, 0),               # ragged tiles + window
    ("mla", dict(B=1, T=1000), [1000], 37, 5, 1),                            # bf16 output
    ("mla", dict(B=1, T=20000), [20000], 4096, 0, 0),                        # four tiles per CTA
    ("mla", dict(B=16, T=3000), None, 2048, 0, 0),                           # the workload's 16 sequences
])
def test_indexed_attention_matches_oracle(name, kw, seq, k, window, out):
    w = W[name].with_(**kw)
    p = Problem(w, seq_lens=seq, out_dtype=out)
    seq = seq or [w.T] * w.B
    ncand = [T - min(window, T) for T in seq]
    idx = synth.random_index_sets(w.B * w.Hkv, [n for n in ncand for _ in range(w.Hkv)], k, seed=k)
    nsel = (idx >= 0).sum(-1).to(torch.int32)
    idx = idx.view(w.B, w.Hkv, k).cuda()
    nsel = nsel.view(w.B, w.Hkv).cuda()
    ws = p.workspace(k, window)
    O = torch.full((w.B, w.Hq, w.dv), float("nan"), device="cuda",
                   dtype=torch.bfloat16 if out else torch.float32)
    lse = torch.full((w.B, w.Hq), float("nan"), device="cuda")
    jssa.indexed_attn(p.L, p.Q, p.K, p.V, idx, k, nsel, p.seq_lens, window, w.sm_scale, O, lse, ws)
    torch.cuda.synchronize()
    G = w.G
    for b in range(w.B):
        T = seq[b]
        for h in range(w.Hkv):
            hst = p.host(b, h)
            n = int(nsel[b, h])
            toks = np.concatenate([idx[b, h, :n].cpu().numpy(), np.arange(T - min(window, T), T)])
            O_ref, lse_ref = oracle.attention(hst["Q"], hst["K"], hst["V"], toks, w.sm_scale)
            O_gpu = O[b, h * G:(h + 1) * G].float().cpu().numpy().astype(np.float64)
            if out:
                # bf16 output: the fp32 result rounded once
                np.testing.assert_allclose(O_gpu, O_ref, atol=8e-3, rtol=8e-3)
            else:
                check_attention(O_gpu, O_ref, f"b={b} h={h}")
            np.testing.assert_allclose(lse[b, h * G:(h + 1) * G].cpu().numpy(), lse_ref, atol=1e-4, rtol=1e-5)
    _assert_status_clean(ws)


@pytest.mark.parametrize("name,kw,seq,k,window", [
    ("tiny", {}, None, 128, 0),
    ("h128k", dict(B=2, T=9000), [9000, 4000], 2048, 0),
    ("hybrid", dict(B=2, T=6000), [6000, 1500], 1024, 1024),    # d = 256 + window
    ("h128k", dict(B=1, T=3000, Hq=32, Hkv=2), [3000], 257, 0),  # G = 16
])
def test_gather_then_attend_comparator_matches_oracle(name, kw, seq, k, window):
    w = W[name].with_(**kw)
    p = Problem(w, seq_lens=seq)
    seq = seq or [w.T] * w.B
    ncand = [T - min(window, T) for T in seq]
    idx = synth.random_index_sets(w.B * w.Hkv, [n for n in ncand for _ in range(w.Hkv)], k, seed=k + 1)
    nsel = (idx >= 0).sum(-1).to(torch.int32).view(w.B, w.Hkv).cuda()
    idx = idx.view(w.B, w.Hkv, k).cuda()
    ws = p.workspace(k, window)
    gbuf = jssa.alloc_gather_buffer(p.L, k, window)
    O = torch.full((w.B, w.Hq, w.dv), float("nan"), device="cuda")
    lse = torch.full((w.B, w.Hq), float("nan"), device="cuda")
    jssa.gather_decode(p.L, p.Q, p.K, p.V, idx, k, nsel, p.seq_lens, window, w.sm_scale, O, lse, gbuf, ws)
    torch.cuda.synchronize()
    G = w.G
    for b in range(w.B):
        T = seq[b]
        for h in range(w.Hkv):
            hst = p.host(b, h)
            n = int(nsel[b, h])
            toks = np.concatenate([idx[b, h, :n].cpu().numpy(), np.arange(T - min(window, T), T)])
            O_ref, lse_ref = oracle.attention(hst["Q"], hst["K"], hst["V"], toks, w.sm_scale)
            check_attention(O[b, h * G:(h + 1) * G].cpu().numpy().astype(np.float64), O_ref, f"gather b={b} h={h}")
            np.testing.assert_allclose(lse[b, h * G:(h + 1) * G].cpu().numpy(), lse_ref, atol=1e-4, rtol=1e-5)
    _assert_status_clean(ws)


@pytest.mark.parametrize("name,kw,seq,window", [
    ("tiny", {}, None, 0),
    ("h128k", dict(B=2, T=7000), [7000, 333], 0),
    ("hybrid", dict(B=2, T=5000), [5000, 800], 1024),    # local layer: dense over the window
    ("h128k", dict(B=2, T=7000), [7000, 5000], 300),     # few splits per row: merged in a cluster
])
def test_dense_decode_matches_oracle(name, kw, seq, window):
    w = W[name].with_(**kw)
    p = Problem(w, seq_lens=seq)
    seq = seq or [w.T] * w.B
    ws = p.workspace(1, window)
    O = torch.full((w.B, w.Hq, w.dv), float("nan"), device="cuda")
    lse = torch.empty((w.B, w.Hq), device="cuda")
    jssa.dense_decode(p.L, p.Q, p.K, p.V, p.seq_lens, window, w.sm_scale, O, lse, ws)
    torch.cuda.synchronize()
    G = w.G
    for b in range(w.B):
        T = seq[b]
        lo = max(0, T - window) if window > 0 else 0
        for h in range(w.Hkv):
            hst = p.host(b, h)
            O_ref, lse_ref = oracle.attention(hst["Q"], hst["K"], hst["V"], np.arange(lo, T), w.sm_scale)
            check_attention(O[b, h * G:(h + 1) * G].cpu().numpy().astype(np.float64), O_ref, f"dense b={b} h={h}")
            np.testing.assert_allclose(lse[b, h * G:(h + 1) * G].cpu().numpy(), lse_ref, atol=1e-4, rtol=1e-5)


def test_sparse_with_k_equal_T_equals_dense():
    w = W["tiny"].with_(T=1500, k=1500)
    p = Problem(w)
    p.fill_kp()
    ws = p.workspace(w.k)
    O_s = torch.empty((w.B, w.Hq, w.dv), device="cuda")
    O_d = torch.empty_like(O_s)
    jssa.decode_step(p.L, p.Q, p.K, p.V, p.Kp, p.P, p.seq_lens, 0, w.k, 0, w.sm_scale, O_s, ws=ws)
    jssa.dense_decode(p.L, p.Q, p.K, p.V, p.seq_lens, 0, w.sm_scale, O_d, ws=ws)
    torch.cuda.synchronize()
    assert float((O_s - O_d).abs().max()) < 1e-5


def test_mla_single_token_returns_the_latent_value_row():
    # one selected token: P = 1 exactly, so O is the first 512 latent dims of that row, and
    # lse is the scaled logit q_h . C_t over all 576 dims
    w = W["mla"].with_(B=2, T=700)
    p = Problem(w)
    picks = [5, 699]
    idx = torch.full((w.B, 1, 4), -1, dtype=torch.int32, device="cuda")
    for b, t in enumerate(picks):
        idx[b, 0, 0] = t
    nsel = torch.ones((w.B, 1), dtype=torch.int32, device="cuda")
    ws = p.workspace(4)
    O = torch.empty((w.B, w.Hq, w.dv), device="cuda")
    lse = torch.empty((w.B, w.Hq), device="cuda")
    jssa.indexed_attn(p.L, p.Q, p.K, p.V, idx, 4, nsel, p.seq_lens, 0, w.sm_scale, O, lse, ws)
    torch.cuda.synchronize()
    for b, t in enumerate(picks):
        row = p.K[b, 0, t].double().cpu()
        assert torch.equal(O[b], p.K[b, 0, t, :w.dv].float().expand(w.Hq, -1))
        ref = (p.Q[b].double().cpu() @ row) * w.sm_scale
        np.testing.assert_allclose(lse[b].double().cpu().numpy(), ref.numpy(), atol=1e-4, rtol=1e-5)
    _assert_status_clean(ws)


@pytest.mark.parametrize("B,T,window,growth,qscale", [
    (1, 300, 0, 0.0, 1.0),        # one tile per CTA (eight CTAs, ragged)
    (2, 2500, 0, 0.0, 1.0),       # several tiles per CTA
    (3, 1800, 700, 0.0, 1.0),     # the window form (local layer of a latent model)
    (1, 4000, 0, 6.0, 24.0),      # logits growing along the cache: the running maxima move and the
                                  # resident output is rescaled on later tiles
])
def test_mla_dense_decode_matches_oracle(B, T, window, growth, qscale):
    # the full-cache comparator of the latent model (§4.5 full-KV baseline) on the tensor cores
    w = W["mla"].with_(B=B, T=T)
    p = Problem(w)
    if growth:
        ramp = 1.0 + growth * torch.arange(T, device="cuda", dtype=torch.float32) / T
        p.K.copy_((p.K.float() * ramp.view(1, 1, T, 1)).to(torch.bfloat16))
        p.Q.copy_((p.Q.float() * qscale).to(torch.bfloat16))
    ws = p.workspace(4, window)
    O = torch.full((w.B, w.Hq, w.dv), float("nan"), device="cuda")
    lse = torch.full((w.B, w.Hq), float("nan"), device="cuda")
    jssa.dense_decode(p.L, p.Q, p.K, p.V, p.seq_lens, window, w.sm_scale, O, lse, ws=ws)
    torch.cuda.synchronize()
    for b in range(w.B):
        hst = p.host(b, 0)
        toks = np.arange(T - window, T) if window else np.arange(T)
        O_ref, lse_ref = oracle.attention(hst["Q"], hst["K"], hst["V"], toks, w.sm_scale)
        check_attention(O[b].cpu().numpy().astype(np.float64), O_ref, f"b={b}")
        np.testing.assert_allclose(lse[b].cpu().numpy(), lse_ref, atol=1e-4, rtol=1e-5)
    _assert_status_clean(ws)


def test_single_token_selection_returns_the_value_row():
    w = W["tiny"].with_(T=600)
    p = Problem(w)
    idx = torch.full((1, w.Hkv, 4), -1, dtype=torch.int32, device="cuda")
    idx[0, :, 0] = torch.tensor([17, 599], dtype=torch.int32)
    nsel = torch.ones((1, w.Hkv), dtype=torch.int32, device="cuda")
    ws = p.workspace(4)
    O = torch.empty((1, w.Hq, w.dv), device="cuda")
    jssa.indexed_attn(p.L, p.Q, p.K, p.V, idx, 4, nsel, p.seq_lens, 0, w.sm_scale, O, None, ws)
    torch.cuda.synchronize()
    for h, t in enumerate([17, 599]):
        ref = p.V[0, h, t].float().expand(w.G, -1)
        assert torch.equal(O[0, h * w.G:(h + 1) * w.G], ref)


# ----------------------------------------------------------------------------- fused step
@pytest.mark.parametrize("name,kw,seq,window", [
    ("tiny", {}, None, 0),
    ("llama8b", dict(B=2, T=6000, k=512), [6000, 4321], 0),
    ("h128k", dict(B=2, T=20000, k=1024), [20000, 11111], 0),
    ("hybrid", dict(B=2, T=9000, k=512), [9000, 3000], 1024),
    ("mla", dict(B=2, T=5000, k=512), [5000, 3210], 0),
    ("h128k", dict(B=1, Hq=8, Hkv=2, T=140000, k=1024), [140000], 0),   # rows beyond one cluster: unfused path
    ("h128k", dict(B=2, T=3000, Hq=16, Hkv=16, k=300), [3000, 2500], 0),   # G = 1
    ("h128k", dict(B=2, T=3000, Hq=16, Hkv=8, k=400), [3000, 1700], 0),     # G = 2
    ("h128k", dict(B=1, T=3000, Hq=32, Hkv=2, k=257), [3000], 0),           # G = 16
    ("tiny", dict(T=1000, dk=64, dv=64, r=8, k=100), None, 0),               # d = 64
    ("h128k", dict(B=2, T=5000, k=512), [5000, 300], 700),                   # window; a row below k
    ("h128k", dict(B=8, T=6000, k=512), [6000, 5000, 4097, 6000, 3000, 2000, 6000, 5999], 0),  # 64 rows: 4-CTA clusters
    ("h128k", dict(B=16, T=3000, k=256), None, 0),                            # 128 rows: 2-CTA clusters
    ("hybrid", dict(B=8, T=5000, k=300), None, 1024),                         # 64 rows, d = 256, window
    ("h128k", dict(B=1, Hq=8, Hkv=2, T=131072, k=4096), None, 0),           # k = 4096 inside the fused kernel
])
def test_decode_step_end_to_end(name, kw, seq, window):
    w = W[name].with_(**kw)
    p = Problem(w, seq_lens=seq)
    p.fill_kp()
    ws = p.workspace(w.k, window)
    O = torch.full((w.B, w.Hq, w.dv), float("nan"), device="cuda")
    idx = torch.empty((w.B, w.Hkv, w.k), dtype=torch.int32, device="cuda")
    nsel = torch.empty((w.B, w.Hkv), dtype=torch.int32, device="cuda")
    p.Kp[torch.arange(w.B), :, p.seq_lens.long() - 1] = 0   # the step must project the newest key itself
    jssa.decode_step(p.L, p.Q, p.K, p.V, p.Kp, p.P, p.seq_lens, 1, w.k, window, w.sm_scale, O, None, idx, nsel, ws)
    torch.cuda.synchronize()
    for b in range(w.B):
        T = int(p.seq_lens[b])
        for h in range(w.Hkv):
            ref, _ = oracle.project_rows(u16(p.K[b, h, T - 1:T]), f32(p.P[h]))
            np.testing.assert_array_equal(u16(p.Kp[b, h, T - 1:T]), ref)
    rows = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    check_step_rows(p, w.k, window, O, idx, nsel, rows, name)
    _assert_status_clean(ws)


@pytest.mark.parametrize("name,kw,seq,window", [
    ("tiny", {}, None, 0),
    ("h128k", dict(B=3, T=20000, k=2048), [20000, 1500, 19999], 0),     # one row below k: select all
    ("hybrid", dict(B=2, T=9000, k=512), [9000, 1800], 1024),
    ("mla", dict(B=2, T=7000, k=700), [7000, 6001], 0),
    ("h128k", dict(B=1, Hq=8, Hkv=2, T=131073, k=512), [131073], 0),   # one token beyond the fused kernel
    ("llama8b", dict(B=8, T=9000, k=600), None, 0),                      # 64 rows: 4-CTA clusters
    ("h128k", dict(B=1, Hq=8, Hkv=2, T=131072, k=4096), None, 0),        # the largest budget of the k sweep
])
def test_select_matches_the_oracle_selection(name, kw, seq, window):
    w = W[name].with_(**kw)
    p = Problem(w, seq_lens=seq)
    p.fill_kp()
    ws = p.workspace(w.k, window)
    idx = torch.full((w.B, w.Hkv, w.k), -7, dtype=torch.int32, device="cuda")
    nsel = torch.full((w.B, w.Hkv), -7, dtype=torch.int32, device="cuda")
    jssa.select(p.L, p.Q, p.K, p.Kp, p.P, p.seq_lens, 0, w.k, window, idx, nsel, ws)
    torch.cuda.synchronize()
    for b in range(w.B):
        T = int(p.seq_lens[b])
        for h in range(w.Hkv):
            hst = p.host(b, h)
            Kp_or = p.project(hst["K"][:T], hst["P"])   # the oracle's own cache; the GPU's must equal it
            np.testing.assert_array_equal(hst["Kp"][:T], Kp_or)
            res = oracle.decode_head(hst["Q"], hst["K"][:T], hst["V"][:T], Kp_or, hst["P"], T, w.k, window,
                                     w.sm_scale)
            check_selection(idx[b, h].cpu().numpy(), int(nsel[b, h]), res["scores"], w.k)
    _assert_status_clean(ws)


@pytest.mark.parametrize("n_new", [3, 16, 40])
def test_decode_step_projects_many_appended_rows(n_new):
    # up to 16 appended rows are projected inside the selection kernel, more by the bulk kernel first
    w = W["tiny"].with_(B=2, T=3000, k=200)
    p = Problem(w, seq_lens=[3000, 2000])
    p.fill_kp()
    for b, T in enumerate([3000, 2000]):
        p.Kp[b, :, T - n_new:T] = 0
    ws = p.workspace(w.k)
    O = torch.full((w.B, w.Hq, w.dv), float("nan"), device="cuda")
    idx = torch.empty((w.B, w.Hkv, w.k), dtype=torch.int32, device="cuda")
    nsel = torch.empty((w.B, w.Hkv), dtype=torch.int32, device="cuda")
    jssa.decode_step(p.L, p.Q, p.K, p.V, p.Kp, p.P, p.seq_lens, n_new, w.k, 0, w.sm_scale, O, None, idx, nsel, ws)
    torch.cuda.synchronize()
    rows = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    check_step_rows(p, w.k, 0, O, idx, nsel, rows, f"n_new={n_new}", kp_checked=True)
    _assert_status_clean(ws)


def test_decode_step_bf16_output_is_the_rounded_fp32_result():
    w = W["h128k"].with_(B=2, T=6000, k=700)
    p32 = Problem(w, seq_lens=[6000, 4444])
    p16 = Problem(w, seq_lens=[6000, 4444], out_dtype=jssa.OUT_BF16)
    for p in (p32, p16):
        p.fill_kp()
    O32 = torch.empty((w.B, w.Hq, w.dv), device="cuda")
    O16 = torch.empty((w.B, w.Hq, w.dv), device="cuda", dtype=torch.bfloat16)
    jssa.decode_step(p32.L, p32.Q, p32.K, p32.V, p32.Kp, p32.P, p32.seq_lens, 0, w.k, 0, w.sm_scale, O32,
                     ws=p32.workspace(w.k))
    jssa.decode_step(p16.L, p16.Q, p16.K, p16.V, p16.Kp, p16.P, p16.seq_lens, 0, w.k, 0, w.sm_scale, O16,
                     ws=p16.workspace(w.k))
    torch.cuda.synchronize()
    assert torch.equal(O16, O32.to(torch.bfloat16))


def test_decode_step_append_loop_updates_the_scoring_cache():
    # workload 2 in miniature: each step appends one token (its K/V row is already in the
    # cache at position T_b) and projects it on write before scoring.
    w = W["llama8b"].with_(B=2, T=3000, k=256)
    p = Problem(w, T_cap=3010, seq_lens=[3000, 2500])
    tb = torch.zeros(w.B, dtype=torch.int32, device="cuda")
    jssa.project_keys(p.L, p.K, p.P, p.Kp, 3000, t_begin=tb)   # prefill rows [0, 3000)
    torch.cuda.synchronize()
    p.Kp[1, :, 2500:] = 0                                        # sequence 1 is shorter
    ws = p.workspace(w.k)
    O = torch.empty((w.B, w.Hq, w.dv), device="cuda")
    idx = torch.empty((w.B, w.Hkv, w.k), dtype=torch.int32, device="cuda")
    nsel = torch.empty((w.B, w.Hkv), dtype=torch.int32, device="cuda")
    for step in range(3):
        p.seq_lens += 1
        jssa.decode_step(p.L, p.Q, p.K, p.V, p.Kp, p.P, p.seq_lens, 1, w.k, 0, w.sm_scale, O, None, idx, nsel, ws)
        torch.cuda.synchronize()
        for b in range(w.B):
            T = int(p.seq_lens[b])
            for h in range(w.Hkv):
                ref, _ = oracle.project_rows(u16(p.K[b, h, T - 1:T]), f32(p.P[h]))
                np.testing.assert_array_equal(u16(p.Kp[b, h, T - 1:T]), ref)
        check_step_rows(p, w.k, 0, O, idx, nsel, [(0, 0), (1, 7), (1, 3)], f"append step {step}")


def test_decode_step_in_a_cuda_graph_matches_eager():
    w = W["h128k"].with_(B=2, T=8192, k=512)
    p = Problem(w)
    p.fill_kp()
    ws = p.workspace(w.k)
    O1 = torch.empty((w.B, w.Hq, w.dv), device="cuda")
    O2 = torch.empty_like(O1)
    jssa.decode_step(p.L, p.Q, p.K, p.V, p.Kp, p.P, p.seq_lens, 0, w.k, 0, w.sm_scale, O1, ws=ws)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            jssa.decode_step(p.L, p.Q, p.K, p.V, p.Kp, p.P, p.seq_lens, 0, w.k, 0, w.sm_scale, O2, ws=ws)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(O1, O2)


# ----------------------------------------------------------------------------- guards
def test_device_checks_flag_bad_indices_and_seq_lens():
    w = W["tiny"].with_(T=400)
    p = Problem(w, T_cap=400)
    ws = p.workspace(8)
    idx = torch.tensor([[[3, 5, 9999, -4, 7, -1, -1, -1], [1, 2, 3, 4, 5, 6, 7, 8]]], dtype=torch.int32,
                       device="cuda")
    nsel = torch.tensor([[5, 8]], dtype=torch.int32, device="cuda")
    O = torch.empty((1, w.Hq, w.dv), device="cuda")
    jssa.indexed_attn(p.L, p.Q, p.K, p.V, idx, 8, nsel, p.seq_lens, 0, w.sm_scale, O, None, ws)
    code, flags = jssa.read_device_status(ws)
    assert code == 5 and flags & jssa._binding.DEV_BAD_INDEX
    assert torch.isfinite(O).all()
    # the out-of-range entries were skipped: same as attending to {3, 5, 7}
    hst = p.host(0, 0)
    O_ref, _ = oracle.attention(hst["Q"], hst["K"], hst["V"], [3, 5, 7], w.sm_scale)
    check_attention(O[0, :w.G].cpu().numpy().astype(np.float64), O_ref, "skip")
    bad = torch.tensor([401], dtype=torch.int32, device="cuda")
    jssa.dense_decode(p.L, p.Q, p.K, p.V, bad, 0, w.sm_scale, O, None, ws)
    code, flags = jssa.read_device_status(ws)
    assert code == 5 and flags & jssa._binding.DEV_BAD_SEQ_LEN
    code, flags = jssa.read_device_status(ws)
    assert code == 0 and flags == 0


def test_invalid_calls_launch_nothing():
    w = W["tiny"].with_(T=256)
    p = Problem(w)
    ws = p.workspace(16)
    O = torch.full((w.B, w.Hq, w.dv), float("nan"), device="cuda")
    with pytest.raises(jssa.JssaError):
        jssa.decode_step(p.L, p.Q, p.K, p.V, p.Kp, p.P, p.seq_lens, 0, 0, 0, w.sm_scale, O, ws=ws)   # k = 0
    with pytest.raises(jssa.JssaError):
        jssa.decode_step(p.L, p.Q, p.K, p.V, p.Kp, p.P, p.seq_lens, 0, 16, 0, w.sm_scale, O,
                         ws=ws[:1024])                                                                 # too small
    with pytest.raises(jssa.JssaError):
        jssa.decode_step(p.L, p.Q, p.K, p.V, p.Kp, p.P, p.seq_lens, 0, 16, 0, w.sm_scale, O,
                         ws=ws[8:])                                                                    # misaligned
    torch.cuda.synchronize()
    assert torch.isnan(O).all()


def test_empty_sequences_and_short_rows():
    w = W["tiny"].with_(B=3, T=64, k=32)
    p = Problem(w, T_cap=64, seq_lens=[0, 5, 64])
    p.fill_kp()
    ws = p.workspace(w.k)
    O = torch.full((w.B, w.Hq, w.dv), float("nan"), device="cuda")
    idx = torch.empty((w.B, w.Hkv, w.k), dtype=torch.int32, device="cuda")
    nsel = torch.empty((w.B, w.Hkv), dtype=torch.int32, device="cuda")
    lse = torch.empty((w.B, w.Hq), device="cuda")
    jssa.decode_step(p.L, p.Q, p.K, p.V, p.Kp, p.P, p.seq_lens, 0, w.k, 0, w.sm_scale, O, lse, idx, nsel, ws)
    torch.cuda.synchronize()
    assert torch.all(O[0] == 0) and torch.all(torch.isneginf(lse[0]))
    assert torch.all(nsel[0] == 0) and torch.all(idx[0] == -1)
    assert torch.all(nsel[1] == 5) and torch.equal(idx[1, :, :5].cpu(), torch.arange(5).expand(w.Hkv, 5).int())
    check_step_rows(p, w.k, 0, O, idx, nsel, [(1, 0), (1, 1), (2, 0), (2, 1)], "short")
