"""Exact ties and the overflow branches of the fused selection, compared bit for bit.

The fused kernel runs the whole selection of a (sequence, KV head) row inside one
thread-block cluster on caches of up to 131072 tokens, with its own radix select.  The
method selects the top-k positions per KV head (Figure 1, §E.3), and this build fixes
the order among equal scores: the lower token index wins.  These cases make that rule
and the kernel's rarely taken branches decide the result, and compare the selected sets
with the oracle's exact full sort without any tie-window allowance:

  * straddle      the k-th score is shared by a group of exactly equal scores, so only
                  part of the group is taken (gather path: the row's in-bin keys fit
                  the gather buffer, every warp lists its candidates);
  * warp overflow more than 64 keys of the k-th key's first-digit bin in one warp's
                  range: that warp rescans its range, and the row takes the cluster
                  histogram path for the later digits;
  * row overflow  more than 2048 in-bin keys in the row, no warp above 64: the cluster
                  histogram path with every warp's candidate list;
  * all equal     one score everywhere: the k lowest positions.

Scores are made exact in every precision: the basis is a coordinate selector and the
group query is the first unit vector, so a token's score is the first element of its
projected row, written directly into the cache (bf16 or E4M3 codes).  A second family
keeps the seeded generator, the real projection (newest row projected inside the step)
and a random orthonormal basis, and duplicates a key row near the boundary into 50
other positions, so that 51 identical projected rows straddle the k-th score.

Shapes: the 128K workload (B=4, Hkv=8: clusters of 8 CTAs) and one sequence of it
(B=1: clusters of 16 CTAs).
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
import token_level_sparse_jssa_b200 as jssa
from token_level_sparse_jssa_b200 import synth
from tests._problem import check_attention, score_error_bound, assert_status_clean
from tests._util import u16, u8, f32

pytestmark = pytest.mark.gpu

T = 131072
K_SEL = 2048
D = 128
R = 32
G = 4
GATHER = 2048      # in-bin keys of a row the kernel gathers into one CTA
WARP_CAP = 64      # per-warp capacity of the kernel's candidate lists
WARPS = 9          # warps of a selection CTA that list candidates


# --------------------------------------------------------------------------- branch bookkeeping
def _ordered(s32: np.ndarray) -> np.ndarray:
    """Order-preserving uint32 keys of fp32 scores (-0 and +0 equal)."""
    s32 = np.where(s32 == 0, np.float32(0), s32).astype(np.float32)
    u = s32.view(np.uint32)
    return np.where(u & 0x80000000, ~u, u | 0x80000000).astype(np.uint32)


def _branch_stats(s32: np.ndarray, k: int, C: int, T_cap: int):
    """How the kernel's selection meets this row: the in-bin keys of the k-th key's
    first-digit bin in the row, the most of them in one warp's range (the kernel's slice
    and warp partition), and the size of the exact-tie group at the k-th score together
    with how many of it are taken."""
    n = s32.size
    keys = _ordered(s32)
    bins = keys >> 20
    hist = np.bincount(bins, minlength=4096)
    suffix = np.cumsum(hist[::-1])[::-1]
    d1 = int(np.nonzero(suffix >= k)[0].max())
    inbin = bins == d1
    per0 = -(-(-(-T_cap // C)) // 32) * 32
    per = min(per0, ((-(-n // C)) + 31) & ~31)
    worst = 0
    for c in range(C):
        lo = c * per
        ln = max(0, min(n, lo + per) - lo)
        wc = ((ln + WARPS - 1) // WARPS + 31) & ~31
        for w in range(WARPS):
            a, b = lo + w * wc, lo + min(ln, w * wc + wc)
            if b > a:
                worst = max(worst, int(inbin[a:b].sum()))
    kth = np.sort(keys)[::-1][k - 1]
    group = int((keys == kth).sum())
    taken = k - int((keys > kth).sum())
    return dict(inbin=int(inbin.sum()), warp_max=worst, group=group, taken=taken)


# --------------------------------------------------------------------------- designed caches
def _designed(B: int, score_rows: torch.Tensor, kp_fp8: bool, seed: int):
    """Caches whose token scores are exactly score_rows [B, 8, T] (rounded once to the Kp
    type): selector basis, first unit vector as the group query, random K/V rows."""
    Hkv = 8
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    K = torch.randn(B, Hkv, T, D, generator=g, device="cuda").to(torch.bfloat16)
    V = torch.randn(B, Hkv, T, D, generator=g, device="cuda").to(torch.bfloat16)
    Q = torch.zeros(B, Hkv * G, D, dtype=torch.bfloat16, device="cuda")
    Q[:, ::G, 0] = 1.0                                  # head 0 of every group: e_0; the rest: 0
    P = torch.zeros(Hkv, D, R, device="cuda")
    P[:, torch.arange(R), torch.arange(R)] = 1.0        # coordinate selector (orthonormal)
    rest = torch.randn(B, Hkv, T, R, generator=g, device="cuda")
    rest[..., 0] = score_rows.to("cuda")
    if kp_fp8:
        Kp = rest.clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8)
    else:
        Kp = rest.to(torch.bfloat16)
    return Q, K, V, Kp.contiguous(), P


def _exact_scores(Kp_row: torch.Tensor, kp_fp8: bool) -> np.ndarray:
    """fp32 scores the designed caches give (the first element of each projected row)."""
    col = Kp_row[:, 0]
    if kp_fp8:
        return col.view(torch.float8_e4m3fn).float().cpu().numpy()
    return col.float().cpu().numpy()


def _plant(s: np.ndarray, value: float, positions: np.ndarray) -> np.ndarray:
    s = s.copy()
    s[positions] = value
    return s


def _kth_value(s: np.ndarray, k: int) -> float:
    return float(np.sort(s)[::-1][k - 1])


def _score_rows(B: int, case: str, kp_fp8: bool, C: int, seed: int) -> torch.Tensor:
    """Designed score rows [B, 8, T] for one case (values already on the Kp type's grid)."""
    gen = np.random.default_rng(seed)
    rows = np.empty((B, 8, T), np.float32)
    for b in range(B):
        for h in range(8):
            s = gen.standard_normal(T).astype(np.float32)
            s = _round_kp(s, kp_fp8)
            if case == "all_equal":
                s[:] = 1.0
            elif case == "straddle":
                # 20 more copies of the k-th value below it: the group then always extends
                # past the budget (only part of it is taken)
                v = _kth_value(s, K_SEL)
                cand = np.nonzero(s < v - 0.5)[0]
                s = _plant(s, v, cand[np.linspace(0, cand.size - 1, 20).astype(np.int64)])
            elif case == "warp_overflow":
                v = _kth_value(s, K_SEL)
                per = T // C
                wc = ((per + WARPS - 1) // WARPS + 31) & ~31
                c, w = (b * 8 + h) % C, (b + h) % WARPS      # one warp's range per row
                lo = c * per + w * wc
                cand = np.arange(lo, min(lo + wc, T))
                cand = cand[s[cand] < v][:100]
                s = _plant(s, v, cand)
            elif case == "row_overflow":
                v = _kth_value(s, K_SEL)
                m = 1300 if kp_fp8 else 1000
                cand = np.nonzero(s < v - 0.5)[0]
                pos = cand[np.linspace(0, cand.size - 1, m).astype(np.int64)]   # spread evenly
                s = _plant(s, v, pos)
            rows[b, h] = s
    return torch.from_numpy(rows)


def _round_kp(s: np.ndarray, kp_fp8: bool) -> np.ndarray:
    t = torch.from_numpy(s)
    if kp_fp8:
        return t.clamp(-448, 448).to(torch.float8_e4m3fn).float().numpy()
    return t.to(torch.bfloat16).float().numpy()


# --------------------------------------------------------------------------- oracle side
def _oracle_selection(Qg16, Kp_host, P32, n, k, kp_fp8):
    """The oracle's steps of Figure 1 on these inputs: projected group query, scores of
    the candidates [0, n) in fp64, exact top-k by a full sort (score desc, index asc)."""
    qs = oracle.query_proj(Qg16, P32)
    s = oracle.scores_e4m3(qs, Kp_host[:n]) if kp_fp8 else oracle.scores(qs, Kp_host[:n])
    idx, k_eff = oracle.topk(s, k)
    return idx, k_eff, s


def _check_exact(Q, K, V, Kp, P, seq_lens, k, window, idx, nsel, O=None, kp_fp8=False, sm_scale=None,
                 rows=None):
    """Every checked row: the selected set bit for bit against the oracle, n_sel, and (with O)
    the attention output against the oracle's fp64 attention over that set plus the window."""
    B, Hkv = idx.shape[0], idx.shape[1]
    rows = rows if rows is not None else [(b, h) for b in range(B) for h in range(Hkv)]
    idx_h, nsel_h = idx.cpu().numpy(), nsel.cpu().numpy()
    for (b, h) in rows:
        Tb = int(seq_lens[b])
        n = Tb - min(window, Tb)
        Qg = u16(Q[b, h * G:(h + 1) * G])
        Kp_host = u8(Kp[b, h]) if kp_fp8 else u16(Kp[b, h])
        or_idx, k_eff, _ = _oracle_selection(Qg, Kp_host, f32(P[h]), n, k, kp_fp8)
        assert int(nsel_h[b, h]) == k_eff, (b, h, nsel_h[b, h], k_eff)
        np.testing.assert_array_equal(idx_h[b, h], or_idx, err_msg=f"row b={b} h={h}")
        if O is not None:
            toks = np.concatenate([or_idx[:k_eff].astype(np.int64), np.arange(n, Tb, dtype=np.int64)])
            tt = torch.from_numpy(toks).to(K.device)
            Ks, Vs = u16(K[b, h].index_select(0, tt)), u16(V[b, h].index_select(0, tt))
            O_ref, _ = oracle.attention(Qg, Ks, Vs, np.arange(toks.size), sm_scale)
            O_gpu = O[b, h * G:(h + 1) * G].float().cpu().numpy().astype(np.float64)
            check_attention(O_gpu, O_ref, f"b={b} h={h}")


def _run_both(Q, K, V, Kp, P, seq_lens, k, window, n_new, kp_fp8, sm_scale, check_rows=None):
    """jssa_select and jssa_decode_step on the same inputs, both checked bit for bit."""
    B, Hkv = K.shape[0], K.shape[1]
    L = jssa.make_layout(K, V, Kp, Hkv * G, R, jssa.MODE_GQA, jssa.OUT_F32)
    ws = jssa.alloc_workspace(L, k, window)
    Kp0 = Kp.clone()
    for entry in ("select", "decode_step"):
        Kp.copy_(Kp0)
        idx = torch.full((B, Hkv, k), -7, dtype=torch.int32, device="cuda")
        nsel = torch.full((B, Hkv), -7, dtype=torch.int32, device="cuda")
        O = None
        if entry == "select":
            jssa.select(L, Q, K, Kp, P, seq_lens, n_new, k, window, idx, nsel, ws)
        else:
            O = torch.full((B, Hkv * G, D), float("nan"), device="cuda")
            jssa.decode_step(L, Q, K, V, Kp, P, seq_lens, n_new, k, window, sm_scale, O, None, idx, nsel, ws)
        torch.cuda.synchronize()
        assert_status_clean(ws)
        _check_exact(Q, K, V, Kp, P, seq_lens, k, window, idx, nsel, O, kp_fp8, sm_scale, check_rows)


# --------------------------------------------------------------------------- the designed cases
SHAPES = [(4, 8), (1, 16)]   # (sequences, CTAs per cluster the launch picks at T = 131072)
CASES = ["straddle", "warp_overflow", "row_overflow", "all_equal"]


@pytest.mark.parametrize("kp_fp8", [False, True], ids=["bf16", "e4m3"])
@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("B,C", SHAPES, ids=["8cta", "16cta"])
def test_fused_selection_is_exact_on_designed_ties(B, C, case, kp_fp8):
    seed = 4000 + 10 * CASES.index(case) + (1 if kp_fp8 else 0) + 100 * C
    srows = _score_rows(B, case, kp_fp8, C, seed)
    Q, K, V, Kp, P = _designed(B, srows, kp_fp8, seed)
    # the case reaches the branch it is named for, in every row
    for b in range(B):
        for h in range(8):
            st = _branch_stats(_exact_scores(Kp[b, h], kp_fp8), K_SEL, C, T)
            assert st["group"] > 1 and 0 < st["taken"] <= st["group"], st
            if case == "straddle":
                assert st["taken"] < st["group"] and st["inbin"] <= GATHER and st["warp_max"] <= WARP_CAP, st
            elif case == "warp_overflow":
                assert st["warp_max"] > WARP_CAP, st
            elif case == "row_overflow":
                assert st["inbin"] > GATHER and st["warp_max"] <= WARP_CAP, st
            else:
                assert st["group"] == T and st["taken"] == K_SEL, st
    seq_lens = torch.full((B,), T, dtype=torch.int32, device="cuda")
    _run_both(Q, K, V, Kp, P, seq_lens, K_SEL, 0, 0, kp_fp8, 1.0 / D ** 0.5)


@pytest.mark.parametrize("kp_fp8", [False, True], ids=["bf16", "e4m3"])
def test_fused_selection_is_exact_on_ties_with_a_window_and_ragged_rows(kp_fp8):
    """Exact ties with a sliding window (candidates [0, T - W)) and sequences of different
    lengths, 8-CTA clusters."""
    B = 4
    seed = 4500 + (1 if kp_fp8 else 0)
    srows = _score_rows(B, "straddle", kp_fp8, 8, seed)
    Q, K, V, Kp, P = _designed(B, srows, kp_fp8, seed)
    seq_lens = torch.tensor([T, T - 1, T - 4093, 70001], dtype=torch.int32, device="cuda")
    _run_both(Q, K, V, Kp, P, seq_lens, K_SEL, 1000, 0, kp_fp8, 1.0 / D ** 0.5)


# --------------------------------------------------------------------------- duplicated key rows
@pytest.mark.parametrize("kp_fp8", [False, True], ids=["bf16", "e4m3"])
def test_fused_selection_is_exact_on_duplicated_key_rows(kp_fp8):
    """The 128K workload's generator, the real projection and a random orthonormal basis;
    in every row a key ranked just inside the budget is copied to 50 positions ranked far
    below it, so that 51 identical projected rows straddle the k-th score (26 taken, the
    lowest positions).  The step projects the newest row itself (n_new = 1)."""
    w = synth.WORKLOADS["h128k"]
    x = synth.make_inputs(w, device="cuda")
    K, V, Q, P, sl = x["K"], x["V"], x["Q"], x["P"].contiguous(), x["seq_lens"]
    Kp = torch.zeros(w.B, w.Hkv, T, w.r, dtype=torch.uint8 if kp_fp8 else torch.bfloat16, device="cuda")
    L = jssa.make_layout(K, V, Kp, w.Hq, w.r)
    tb = torch.zeros(w.B, dtype=torch.int32, device="cuda")
    proj = oracle.project_rows_e4m3 if kp_fp8 else oracle.project_rows
    gen = np.random.default_rng(77 + kp_fp8)
    checked = []
    for b in range(w.B):
        for h in range(w.Hkv):
            Kh = u16(K[b, h])
            Kp_or, _ = proj(Kh, f32(P[h]))
            _, _, s = _oracle_selection(u16(Q[b, h * G:(h + 1) * G]), Kp_or, f32(P[h]), T, K_SEL, kp_fp8)
            order = np.lexsort((np.arange(T), -s))
            src = int(order[K_SEL - 26])
            low = order[K_SEL + 4096:]
            low = low[low < T - 1]                     # keep the newest row as it is
            dst = np.sort(gen.choice(low, 50, replace=False))
            K[b, h, torch.from_numpy(dst).cuda()] = K[b, h, src].clone()
            checked.append((b, h, src))
    jssa.project_keys(L, K, P, Kp, T, t_begin=tb)
    torch.cuda.synchronize()
    ws = jssa.alloc_workspace(L, K_SEL, 0)
    identical = 0
    for entry in ("select", "decode_step"):
        idx = torch.full((w.B, w.Hkv, K_SEL), -7, dtype=torch.int32, device="cuda")
        nsel = torch.full((w.B, w.Hkv), -7, dtype=torch.int32, device="cuda")
        O = None
        if entry == "select":
            jssa.select(L, Q, K, Kp, P, sl, 1, K_SEL, 0, idx, nsel, ws)
        else:
            O = torch.full((w.B, w.Hq, w.dv), float("nan"), device="cuda")
            jssa.decode_step(L, Q, K, V, Kp, P, sl, 1, K_SEL, 0, w.sm_scale, O, None, idx, nsel, ws)
        torch.cuda.synchronize()
        assert_status_clean(ws)
        for (b, h, src) in checked:
            Qg, Kp_host = u16(Q[b, h * G:(h + 1) * G]), (u8(Kp[b, h]) if kp_fp8 else u16(Kp[b, h]))
            or_idx, k_eff, s = _oracle_selection(Qg, Kp_host, f32(P[h]), T, K_SEL, kp_fp8)
            g_idx = idx[b, h].cpu().numpy()
            assert int(nsel[b, h]) == k_eff == K_SEL
            sel = g_idx[:k_eff]
            assert np.all(np.diff(sel) > 0) and np.all(g_idx[k_eff:] == -1)
            group = np.nonzero(s == s[src])[0]
            assert group.size >= 51
            # the tie rule on the path that ships: the selected members of the group of identical
            # projected rows are its lowest positions
            taken = np.intersect1d(sel, group)
            np.testing.assert_array_equal(taken, group[:taken.size], err_msg=f"b={b} h={h}")
            A, B = set(sel.tolist()), set(or_idx[:k_eff].tolist())
            if A == B:
                identical += 1
            else:  # only tokens whose fp32 score may round to either side of the group's score
                if kp_fp8:
                    kpv = np.array([oracle.e4m3_to_double(int(c)) for c in range(256)])[Kp_host[:T]]
                    bound = score_error_bound(Qg, f32(P[h]), kpv)
                else:
                    bound = score_error_bound(Qg, f32(P[h]), Kp_host[:T])
                for t in A ^ B:
                    assert t in set(group.tolist()) or abs(s[t] - s[src]) <= bound[t] + bound[src], (b, h, t)
            if O is not None:
                O_ref, _ = oracle.attention(Qg, u16(K[b, h]), u16(V[b, h]), sel, w.sm_scale)
                O_gpu = O[b, h * G:(h + 1) * G].float().cpu().numpy().astype(np.float64)
                check_attention(O_gpu, O_ref, f"b={b} h={h}")
    # rounding reorders a neighbour of the group only rarely: most rows match the oracle exactly
    assert identical >= 2 * len(checked) * 3 // 4, identical
