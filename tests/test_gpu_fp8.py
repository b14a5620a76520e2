"""Parity of the FP8 E4M3 projected-key cache (the paper's deployed scoring cache, §A.3 and
§E.2 of "Joint Subspace Sparse Attention for Efficient Long-Context Decoding") with the
oracle: the GPU's E4M3 projection is the oracle's rounding of the exact product, bit for
bit (saturation and subnormals included); scores over the same codes stay within the fp32
error bound; the fused and unfused selections equal the oracle's up to swaps inside the tie
window, and the step's output matches the oracle's on the same index set.
"""
import numpy as np
import pytest
import torch

import oracle
from tests._problem import Problem, check_selection, check_step_rows, score_error_bound
from tests._util import u16, u8, f32
import token_level_sparse_jssa_b200 as jssa
from token_level_sparse_jssa_b200 import synth

pytestmark = pytest.mark.gpu
W = synth.WORKLOADS


@pytest.fixture(scope="module", autouse=True)
def _lib():
    jssa.load()
    yield
    torch.cuda.synchronize()


def _clean(ws):
    code, flags = jssa.read_device_status(ws)
    assert code == 0 and flags == 0, (code, flags)


def _upload_oracle_cache(p, window=0):
    """Fill Kp with the oracle's E4M3 projection of every cached row (inputs stay the oracle's)."""
    for b in range(p.w.B):
        for h in range(p.w.Hkv):
            hst = p.host(b, h)
            codes = p.project(hst["K"], hst["P"])
            p.Kp[b, h] = torch.from_numpy(codes).to(p.Kp.device)


@pytest.mark.parametrize("name,kw,pscale", [
    ("tiny", dict(T=700), 1.0),
    ("h128k", dict(B=2, T=1100), 1.0),
    ("h128k", dict(B=1, T=600, r=16), 1.0),
    ("tiny", dict(T=500, r=64), 1.0),
    ("mla", dict(B=1, T=333), 1.0),
    ("tiny", dict(T=400), 400.0),     # most products beyond 448: saturation
    ("tiny", dict(T=400), 2e-3),      # most products below 2^-6: subnormal codes and zeros
])
def test_project_keys_e4m3_is_bit_exact(name, kw, pscale):
    w = W[name].with_(**kw)
    p = Problem(w, kp_fp8=True)
    p.P.mul_(pscale)
    p.fill_kp()
    torch.cuda.synchronize()
    n_sat = n_sub = 0
    for b in range(w.B):
        for h in range(w.Hkv):
            ref, _ = oracle.project_rows_e4m3(u16(p.K[b, h]), f32(p.P[h]))
            got = u8(p.Kp[b, h])
            np.testing.assert_array_equal(got, ref)
            n_sat += int(np.sum((ref & 0x7F) == 0x7E))
            n_sub += int(np.sum((ref & 0x78) == 0))
    if pscale > 100:
        assert n_sat > 0
    if pscale < 1e-2:
        assert n_sub > 0


@pytest.mark.parametrize("name,kw,seq,window", [
    ("tiny", {}, None, 0),
    ("h128k", dict(B=2, T=5000), [5000, 4097], 0),
    ("hybrid", dict(B=2, T=3000), [3000, 2100], 1024),
    ("tiny", dict(T=900, r=64), None, 5),
    ("mla", dict(B=1, T=1200), [1200], 0),
])
def test_score_e4m3_within_fp32_error_bound(name, kw, seq, window):
    w = W[name].with_(**kw)
    p = Problem(w, seq_lens=seq, kp_fp8=True)
    _upload_oracle_cache(p)
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
            codes = hst["Kp"][:n]
            s_or = oracle.scores_e4m3(oracle.query_proj(hst["Q"], hst["P"]), codes)
            vals = np.vectorize(oracle.e4m3_to_double, otypes=[np.float64])(codes) if n else np.zeros((0, w.r))
            bound = score_error_bound(hst["Q"], hst["P"], vals)
            err = np.abs(sc[b, h, :n] - s_or)
            assert np.all(err <= bound * 1.0001 + 1e-30), float(np.max(err / np.maximum(bound, 1e-30)))
            assert np.all(np.isnan(sc[b, h, n:]))
    _clean(ws)


@pytest.mark.parametrize("name,kw,seq,window", [
    ("tiny", {}, None, 0),
    ("h128k", dict(B=3, T=20000, k=2048), [20000, 1500, 19999], 0),
    ("hybrid", dict(B=2, T=9000, k=512), [9000, 1800], 1024),
    ("mla", dict(B=2, T=7000, k=700), [7000, 6001], 0),
    ("h128k", dict(B=1, Hq=8, Hkv=2, T=131073, k=512), [131073], 0),   # beyond the fused kernel: unfused path
    ("tiny", dict(T=3000, r=16, k=200), None, 0),
    ("tiny", dict(T=3000, r=64, k=200), None, 0),
])
def test_select_e4m3_matches_the_oracle_selection(name, kw, seq, window):
    w = W[name].with_(**kw)
    p = Problem(w, seq_lens=seq, kp_fp8=True)
    _upload_oracle_cache(p)
    ws = p.workspace(w.k, window)
    idx = torch.full((w.B, w.Hkv, w.k), -7, dtype=torch.int32, device="cuda")
    nsel = torch.full((w.B, w.Hkv), -7, dtype=torch.int32, device="cuda")
    jssa.select(p.L, p.Q, p.K, p.Kp, p.P, p.seq_lens, 0, w.k, window, idx, nsel, ws)
    torch.cuda.synchronize()
    for b in range(w.B):
        T = int(p.seq_lens[b])
        for h in range(w.Hkv):
            hst = p.host(b, h)
            n = T - min(window, T)
            s = oracle.scores_e4m3(oracle.query_proj(hst["Q"], hst["P"]), hst["Kp"][:n])
            check_selection(idx[b, h].cpu().numpy(), int(nsel[b, h]), s, w.k)
    _clean(ws)


@pytest.mark.parametrize("name,kw,seq,window,n_new", [
    ("tiny", {}, None, 0, 1),
    ("h128k", dict(B=2, T=20000, k=1024), [20000, 11111], 0, 1),
    ("hybrid", dict(B=2, T=9000, k=512), [9000, 3000], 1024, 1),
    ("mla", dict(B=2, T=5000, k=512), [5000, 3210], 0, 1),
    ("h128k", dict(B=1, Hq=8, Hkv=2, T=140000, k=1024), [140000], 0, 1),   # unfused path
    ("tiny", dict(B=2, T=3000, k=200), [3000, 2000], 0, 16),              # newest rows inside the kernel
    ("tiny", dict(B=2, T=3000, k=200), [3000, 2000], 0, 40),              # bulk projection first
    ("h128k", dict(B=2, T=3000, Hq=32, Hkv=2, k=257), [3000, 2999], 0, 1),  # G = 16
])
def test_decode_step_e4m3_end_to_end(name, kw, seq, window, n_new):
    w = W[name].with_(**kw)
    p = Problem(w, seq_lens=seq, kp_fp8=True)
    _upload_oracle_cache(p)
    for b in range(w.B):   # the step must project its newest rows itself
        T = int(p.seq_lens[b])
        p.Kp[b, :, max(0, T - n_new):T] = 0
    ws = p.workspace(w.k, window)
    O = torch.full((w.B, w.Hq, w.dv), float("nan"), device="cuda")
    idx = torch.empty((w.B, w.Hkv, w.k), dtype=torch.int32, device="cuda")
    nsel = torch.empty((w.B, w.Hkv), dtype=torch.int32, device="cuda")
    jssa.decode_step(p.L, p.Q, p.K, p.V, p.Kp, p.P, p.seq_lens, n_new, w.k, window, w.sm_scale, O, None, idx, nsel,
                     ws)
    torch.cuda.synchronize()
    rows = [(b, h) for b in range(w.B) for h in range(w.Hkv)]
    check_step_rows(p, w.k, window, O, idx, nsel, rows, f"{name} e4m3", kp_checked=True)
    _clean(ws)


def test_e4m3_step_reads_half_the_scoring_bytes_of_bf16():
    # same inputs, both caches: the E4M3 cache holds the codes of the same exact products
    w = W["h128k"].with_(B=1, T=4096, k=256)
    p8 = Problem(w, kp_fp8=True, seed=5)
    p16 = Problem(w, seed=5)
    p8.fill_kp()
    p16.fill_kp()
    torch.cuda.synchronize()
    assert p8.Kp.element_size() * 2 == p16.Kp.element_size()
    ex = oracle.project_rows(u16(p16.K[0, 3, :64]), f32(p16.P[3]))[1]
    want = np.array([[oracle.double_to_e4m3(v) for v in row] for row in ex], np.uint8)
    np.testing.assert_array_equal(u8(p8.Kp[0, 3, :64]), want)
