"""Parity of the GPU basis calibration (jssa_calibrate) with the calibration oracle, and the
selection quality it buys on planted low-rank data ("Joint Subspace Sparse Attention for
Efficient Long-Context Decoding", §3.2, §A.4, §B.1-§B.3).

The eigenvectors are compared column by column (the sign convention makes them unique
when the eigenvalues are distinct, which the anisotropic test data guarantees), the
eigenvalues to fp64 accuracy.  The recall test measures, on the synthetic workload's
recipe, how often the decode step's selection contains the exact full-dimensional top-k.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import calibration as cal
from tests._util import u16
import token_level_sparse_jssa_b200 as jssa
from token_level_sparse_jssa_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    jssa.load()
    yield
    torch.cuda.synchronize()


def _layout(B, Hq, Hkv, d, r, T, mode=jssa.MODE_GQA, dv=None):
    K = torch.empty(B, Hkv, T, d, dtype=torch.bfloat16, device="cuda")
    V = K[..., : dv] if dv else K
    Kp = torch.empty(B, Hkv, T, r, dtype=torch.bfloat16, device="cuda")
    return jssa.make_layout(K, V, Kp, Hq, r, mode), K


def _anisotropic(shape, d, seed, spread=30.0):
    """bf16 rows with a spread of per-direction scales (distinct eigenvalues)."""
    g = torch.Generator().manual_seed(seed)
    rot = torch.linalg.qr(torch.randn(d, d, generator=g, dtype=torch.float64))[0]
    scales = torch.logspace(0, -np.log10(spread), d, dtype=torch.float64)
    x = torch.randn(*shape, d, generator=g, dtype=torch.float64) * scales
    return (x @ rot.T).to(torch.bfloat16)


@pytest.mark.parametrize("B,Hq,Hkv,d,r,n", [
    (2, 8, 2, 64, 16, 3000),
    (1, 16, 2, 128, 32, 5000),
    (2, 4, 4, 128, 64, 2100),       # G = 1
    (1, 16, 1, 256, 32, 1500),
])
def test_calibration_matches_the_oracle(B, Hq, Hkv, d, r, n):
    L, K = _layout(B, Hq, Hkv, d, r, n + 7)
    K.copy_(_anisotropic((B, Hkv, n + 7), d, seed=d + r))
    Qc = _anisotropic((B, Hq, n), d, seed=d * r + 1, spread=10.0).cuda().contiguous()
    P = torch.full((Hkv, d, r), float("nan"), device="cuda")
    ev = torch.full((Hkv, d), float("nan"), device="cuda", dtype=torch.float64)
    ws = jssa.alloc_calibration_workspace(L)
    jssa.calibrate(L, Qc, K, n, P, ws, ev)
    torch.cuda.synchronize()
    code, flags = jssa.read_device_status(ws)
    assert code == 0 and flags == 0, (code, flags)
    G = Hq // Hkv
    for h in range(Hkv):
        Qh = np.concatenate([u16(Qc[b, h * G:(h + 1) * G]) for b in range(B)], axis=1)   # [G, B*n, d]
        Kh = np.concatenate([u16(K[b, h, :n]) for b in range(B)], axis=0)
        P_or, w_or = cal.calibrate(Qh, Kh, r)
        np.testing.assert_allclose(ev[h].cpu().numpy(), w_or, rtol=1e-10, atol=1e-14)
        np.testing.assert_allclose(P[h].cpu().numpy(), P_or, atol=2e-6)


def test_calibration_of_the_mla_latent():
    # one latent head, 128 query heads, d = 576, r = 64 (a reduced token count)
    B, Hq, d, r, n = 1, 128, 576, 64, 400
    L, K = _layout(B, Hq, 1, d, r, n, mode=jssa.MODE_MLA, dv=512)
    K.copy_(_anisotropic((B, 1, n), d, seed=7))
    Qc = _anisotropic((B, Hq, n), d, seed=8, spread=10.0).cuda().contiguous()
    P = torch.empty((1, d, r), device="cuda")
    ev = torch.empty((1, d), device="cuda", dtype=torch.float64)
    ws = jssa.alloc_calibration_workspace(L)
    jssa.calibrate(L, Qc, K, n, P, ws, ev)
    torch.cuda.synchronize()
    code, flags = jssa.read_device_status(ws)
    assert code == 0 and flags == 0
    P_or, w_or = cal.calibrate(u16(Qc[0]), u16(K[0, 0]), r)
    np.testing.assert_allclose(ev[0].cpu().numpy(), w_or, rtol=1e-9, atol=1e-14)
    np.testing.assert_allclose(P[0].cpu().numpy(), P_or, atol=5e-6)


def test_calibrated_basis_is_orthonormal_and_scale_free():
    B, Hq, Hkv, d, r, n = 1, 8, 2, 128, 32, 2000
    L, K = _layout(B, Hq, Hkv, d, r, n)
    K.copy_(_anisotropic((B, Hkv, n), d, seed=3))
    Qc = _anisotropic((B, Hq, n), d, seed=4).cuda().contiguous()
    ws = jssa.alloc_calibration_workspace(L)
    P1 = torch.empty((Hkv, d, r), device="cuda")
    P2 = torch.empty_like(P1)
    jssa.calibrate(L, Qc, K, n, P1, ws)
    K.mul_(8.0)                                     # exact in bf16: trace normalisation removes it
    jssa.calibrate(L, Qc, K, n, P2, ws)
    torch.cuda.synchronize()
    assert torch.equal(P1, P2)
    for h in range(Hkv):
        G = P1[h].double().T @ P1[h].double()
        assert torch.allclose(G, torch.eye(r, dtype=torch.float64, device="cuda"), atol=1e-6)


def _recall(w, x, P, Qs, k):
    """Mean fraction of the exact full-dimensional top-k (group-mean query . key) that the
    decode step selects with basis P, over the query batches Qs."""
    Kp = torch.zeros(w.B, w.Hkv, w.T, w.r, dtype=torch.bfloat16, device="cuda")
    L = jssa.make_layout(x["K"], x["V"], Kp, w.Hq, w.r)
    tb = torch.zeros(w.B, dtype=torch.int32, device="cuda")
    jssa.project_keys(L, x["K"], P, Kp, w.T, t_begin=tb)
    ws = jssa.alloc_workspace(L, k)
    O = torch.empty(w.B, w.Hq, w.dv, device="cuda")
    idx = torch.empty(w.B, w.Hkv, k, dtype=torch.int32, device="cuda")
    nsel = torch.empty(w.B, w.Hkv, dtype=torch.int32, device="cuda")
    Kf = x["K"].double()
    rec = []
    for Q in Qs:
        jssa.decode_step(L, Q, x["K"], x["V"], Kp, P, x["seq_lens"], 0, k, 0, w.sm_scale, O, None, idx, nsel, ws)
        qbar = Q.double().view(w.B, w.Hkv, w.G, w.dk).mean(2)                       # [B, Hkv, d]
        s = torch.einsum("bhd,bhtd->bht", qbar, Kf)
        truth = torch.topk(s, k, dim=2).indices
        for b in range(w.B):
            for h in range(w.Hkv):
                a = set(truth[b, h].tolist())
                rec.append(len(a & set(idx[b, h].tolist())) / k)
    return float(np.mean(rec))


def test_calibrated_basis_selects_the_true_top_k_better_than_a_random_one():
    # the synthetic recipe plants a rank-16 query-key structure per KV head; calibrated on
    # other positions of the same sequences, the basis recovers it
    w = synth.WORKLOADS["h128k"].with_(B=2, Hq=8, Hkv=2, T=8192, k=256, heavy=0)
    x = synth.make_inputs(w, device="cuda")
    n = 4096
    Qc = synth.fresh_queries(w, n, x["A"], device="cuda", seed=11).permute(1, 2, 0, 3).contiguous()
    L, _ = _layout(w.B, w.Hq, w.Hkv, w.dk, w.r, w.T)
    P_cal = torch.empty_like(x["P"])
    ws = jssa.alloc_calibration_workspace(L)
    jssa.calibrate(L, Qc, x["K"], n, P_cal, ws)
    Qs = synth.fresh_queries(w, 4, x["A"], device="cuda", seed=12)
    r_cal = _recall(w, x, P_cal, Qs, w.k)
    r_rand = _recall(w, x, x["P"], Qs, w.k)
    assert r_cal > 0.8 and r_cal > r_rand + 0.2, (r_cal, r_rand)
