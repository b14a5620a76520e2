"""Test-side plumbing: build device caches from the seeded generator and compare the
CUDA path with the oracle.  Conversions and bookkeeping only."""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from tests._util import u16, u8, f32, rel_l2
import token_level_sparse_jssa_b200 as jssa
from token_level_sparse_jssa_b200 import synth

# Tolerances fixed by the method's parity target: selected index sets may differ only by
# swaps among tokens whose oracle score lies within 1e-5 relative of the k-th score;
# fp32 attention outputs within max-abs 2e-3 and rel-L2 1e-3 of the fp64 oracle.
TIE_REL = 1e-5
ATOL = 2e-3
RTOL_L2 = 1e-3


class Problem:
    """Device caches (K, V, Kp, Q, P, seq_lens) of one workload plus its layout."""

    def __init__(self, w: synth.Workload, T_cap=None, seq_lens=None, out_dtype=jssa.OUT_F32, device="cuda",
                 gen_device="cuda", seed=None, kp_fp8=False):
        self.w = w
        x = synth.make_inputs(w, device=gen_device, T_cap=T_cap, seq_lens=seq_lens, seed=seed)
        self.T_cap = x["T_cap"]
        self.A = x["A"]
        self.Q = x["Q"].to(device)
        self.K = x["K"].to(device)
        if w.mode == "mla":
            self.V = self.K[..., : w.dv]
        else:
            self.V = x["V"].to(device)
        self.P = x["P"].to(device).contiguous()
        self.seq_lens = x["seq_lens"].to(device)
        self.kp_fp8 = kp_fp8
        self.Kp = torch.zeros(w.B, w.Hkv, self.T_cap, w.r, dtype=torch.uint8 if kp_fp8 else torch.bfloat16,
                              device=device)
        self.L = jssa.make_layout(self.K, self.V, self.Kp, w.Hq, w.r,
                                  jssa.MODE_MLA if w.mode == "mla" else jssa.MODE_GQA, out_dtype)

    def fill_kp(self):
        """Project every row of the cache (the prefill-time fill of the scoring cache)."""
        tb = torch.zeros(self.w.B, dtype=torch.int32, device=self.K.device)
        jssa.project_keys(self.L, self.K, self.P, self.Kp, self.T_cap, t_begin=tb)

    def workspace(self, k, window=0):
        return jssa.alloc_workspace(self.L, k, window)

    # host copies for the oracle
    def host(self, b, h):
        G = self.w.G
        return dict(Q=u16(self.Q[b, h * G:(h + 1) * G]), K=u16(self.K[b, h]), V=u16(self.V[b, h]),
                    Kp=u8(self.Kp[b, h]) if self.kp_fp8 else u16(self.Kp[b, h]), P=f32(self.P[h]))

    def project(self, K_rows, P):
        """The oracle's scoring-cache rows for these key rows, in this problem's Kp type."""
        return (oracle.project_rows_e4m3 if self.kp_fp8 else oracle.project_rows)(K_rows, P)[0]


def check_selection(gpu_idx: np.ndarray, gpu_nsel: int, s: np.ndarray, k: int):
    """GPU selection vs the oracle's exact top-k of fp64 scores ``s``, allowing swaps within
    the tie window.  Returns (oracle_idx, identical?)."""
    or_idx, k_eff = oracle.topk(s, k)
    assert gpu_nsel == k_eff, (gpu_nsel, k_eff)
    sel = gpu_idx[:k_eff]
    assert np.all(gpu_idx[k_eff:] == -1)
    assert np.all(np.diff(sel) > 0), "selection must be strictly ascending"
    A, B = set(sel.tolist()), set(or_idx[:k_eff].tolist())
    if A == B:
        return or_idx, True
    kth = np.sort(s)[::-1][k_eff - 1]
    assert abs(kth) > 1e-3 * np.max(np.abs(s)), "k-th score too close to 0 for a relative tie window"
    for t in A ^ B:
        assert abs(s[t] - kth) <= TIE_REL * abs(kth), (t, s[t], kth)
    assert len(A) == len(B) == k_eff
    return or_idx, False


def check_attention(O_gpu: np.ndarray, O_ref: np.ndarray, what=""):
    err = float(np.max(np.abs(O_gpu - O_ref))) if O_ref.size else 0.0
    rl2 = rel_l2(O_gpu, O_ref)
    assert err <= ATOL and rl2 <= RTOL_L2, f"{what}: max-abs {err:.3e}, rel-L2 {rl2:.3e}"
    return err, rl2


def score_error_bound(Qg: np.ndarray, P: np.ndarray, Kp: np.ndarray) -> np.ndarray:
    """Rigorous bound on |fp32 score - exact score| for the GPU's evaluation order family:
    the group sum (G terms), the d-term projection and the r-term dot product, each in
    fp32 with any summation order (gamma_n = n u / (1 - n u), u = 2^-24).  Kp: bf16 codes
    (uint16) or the decoded values (float64)."""
    u = 2.0 ** -24
    gam = lambda n: n * u / (1 - n * u)
    q = oracle.bf16_to_f64(Qg)                 # [G, d]
    G, d = q.shape
    absP = np.abs(P.astype(np.float64))        # [d, r]
    qsum_abs = np.abs(q).sum(0)                # bound on |sum_g q| and on its rounding base
    qs_exact = P.astype(np.float64).T @ q.sum(0)
    err_qs = (gam(d) + gam(G) * (1 + gam(d))) * (absP.T @ qsum_abs)   # [r]
    kp = oracle.bf16_to_f64(Kp) if Kp.dtype == np.uint16 else np.asarray(Kp, np.float64)   # [n, r]
    r = kp.shape[1]
    qs_abs = np.abs(qs_exact) + err_qs
    return gam(r) * (np.abs(kp) @ qs_abs) + np.abs(kp) @ err_qs


def check_step_rows(p: Problem, k: int, window: int, O, idx, nsel, rows, what="", kp_checked=False):
    """Check sampled (b, h) rows of a decode step against the oracle run on the same inputs:
    the selection within the tie window, and the attention output against the oracle's
    (on the GPU's own index set when an allowed swap occurred).  Returns the number of rows
    whose selection was identical."""
    w = p.w
    G = w.G
    n_same = 0
    for (b, h) in rows:
        T = int(p.seq_lens[b])
        hst = p.host(b, h)
        Kp_or = p.project(hst["K"][:T], hst["P"])
        if kp_checked:  # the scoring cache the step read is the oracle's projection, bit for bit
            np.testing.assert_array_equal(hst["Kp"][:T], Kp_or)
        head = oracle.decode_head_e4m3 if p.kp_fp8 else oracle.decode_head
        res = head(hst["Q"], hst["K"][:T], hst["V"][:T], Kp_or, hst["P"], T, k, window, w.sm_scale)
        g_idx = idx[b, h].cpu().numpy()
        _, same = check_selection(g_idx, int(nsel[b, h]), res["scores"], k)
        O_gpu = O[b, h * G:(h + 1) * G].float().cpu().numpy().astype(np.float64)
        if same:
            O_ref = res["O"]
            n_same += 1
        else:  # an allowed swap inside the tie window: the oracle runs on the GPU's own set
            n = int(nsel[b, h])
            toks = np.concatenate([g_idx[:n], np.arange(T - min(window, T), T)])
            O_ref, _ = oracle.attention(hst["Q"], hst["K"], hst["V"], toks, w.sm_scale)
        check_attention(O_gpu, O_ref, f"{what} b={b} h={h}")
    return n_same


def assert_status_clean(ws):
    code, flags = jssa.read_device_status(ws)
    assert code == 0 and flags == 0, (code, flags)
