"""Pins for the CPU oracle (no GPU): the oracle is checked against closed forms,
special cases that reduce to independent library routines, brute force on tiny
inputs, invariants of the method and hand-derived worked examples, so that a
dropped term, a wrong sign or index or a transposed operand fails a test.

Method source: "Joint Subspace Sparse Attention for Efficient Long-Context
Decoding" (arXiv 2610.19026v1) — Figure 1, §2.1 (FASA = restricted orthonormal
projection), §3.1-§3.4, §4.5 (full-KV baseline), §A.3, §E.3.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from tests._util import u16, f32
from token_level_sparse_jssa_b200 import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _bf16_bits_of(x: np.ndarray) -> np.ndarray:
    return u16(torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16))


def _rand_bf16(shape, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return u16((torch.randn(*shape, generator=g) * scale).to(torch.bfloat16))


# ----------------------------------------------------------------------------- bf16
def test_bf16_round_matches_torch_cast_on_fp32_values():
    g = torch.Generator().manual_seed(1)
    x = torch.randn(200000, generator=g) * torch.exp2(torch.randint(-140, 120, (200000,), generator=g).float())
    x = x.to(torch.float32)
    ours = oracle.bf16_round(x.double().numpy())
    ref = u16(x.to(torch.bfloat16))
    np.testing.assert_array_equal(ours, ref)


def test_bf16_round_hand_cases():
    d = json.load(open(os.path.join(GOLD, "projection_small.json")))["rounding_cases"]
    got = [oracle.bf16_round_scalar(x) for x in d["x"]]
    assert got == d["bits"]


def test_bf16_decode_is_exact_inverse():
    bits = np.arange(0, 65536, dtype=np.uint32).astype(np.uint16)
    vals = oracle.bf16_to_f64(bits)
    finite = np.isfinite(vals)
    back = oracle.bf16_round(vals[finite])
    # every finite pattern round-trips, except that -0 keeps its sign bit
    np.testing.assert_array_equal(back, bits[finite])


# ----------------------------------------------------------------------------- projection
def test_projection_identity_basis_is_exact():
    K = _rand_bf16((300, 64), 2, scale=3.0)
    P = np.eye(64, dtype=np.float32)
    Kp, ex = oracle.project_rows(K, P)
    np.testing.assert_array_equal(Kp, K)


def test_projection_column_selector_is_channel_subset():
    # §2.1: keeping r original channels is a restricted orthonormal projection (FASA).
    K = _rand_bf16((257, 128), 3)
    cols = [5, 0, 77, 127, 64, 33, 2, 100]
    P = np.zeros((128, len(cols)), np.float32)
    for j, c in enumerate(cols):
        P[c, j] = 1.0
    Kp, _ = oracle.project_rows(K, P)
    np.testing.assert_array_equal(Kp, K[:, cols])


def test_projection_matches_numpy_matmul_and_rounds_once():
    K = _rand_bf16((500, 128), 4)
    P = synth.orthonormal_basis(128, 32, seed=9).numpy()
    Kp, ex = oracle.project_rows(K, P)
    ref = oracle.bf16_to_f64(K) @ P.astype(np.float64)
    np.testing.assert_allclose(ex, ref, rtol=0, atol=1e-12)
    # rounding the exact product once gives the stored cache
    np.testing.assert_array_equal(Kp, oracle.bf16_round(ref))


def test_projection_golden():
    d = json.load(open(os.path.join(GOLD, "projection_small.json")))
    K = _bf16_bits_of(np.array(d["K"]))
    P = np.array(d["P"], np.float32)
    Kp, ex = oracle.project_rows(K, P)
    np.testing.assert_array_equal(ex, np.array(d["Kp_exact"]))
    np.testing.assert_array_equal(Kp, np.array(d["Kp_bf16_bits"], np.uint16).reshape(Kp.shape))
    Q = _bf16_bits_of(np.array(d["Q"]))
    qs = oracle.query_proj(Q, P)
    np.testing.assert_array_equal(qs, np.array(d["qs"]))
    np.testing.assert_array_equal(oracle.scores(qs, Kp), np.array(d["scores"]))


# ----------------------------------------------------------------------------- query projection / scores
def test_query_projection_is_a_sum_over_the_group():
    # G copies of one head give G times the single-head projection (sum, not mean).
    q = _rand_bf16((1, 128), 5)
    P = synth.orthonormal_basis(128, 16, seed=3).numpy()
    one = oracle.query_proj(q, P)
    four = oracle.query_proj(np.repeat(q, 4, axis=0), P)
    np.testing.assert_allclose(four, 4 * one, rtol=1e-15, atol=0)
    ref = P.astype(np.float64).T @ oracle.bf16_to_f64(q[0])
    np.testing.assert_allclose(one, ref, rtol=0, atol=1e-14)


def test_query_projection_transposition_is_pinned():
    # A non-square, non-symmetric P: using P instead of P^T would not even type-check,
    # and swapping the roles of rows/columns changes every value.
    q = _rand_bf16((3, 6), 6)
    P = np.arange(12, dtype=np.float32).reshape(6, 2) / 7.0
    qs = oracle.query_proj(q, P)
    ref = (oracle.bf16_to_f64(q).sum(0)) @ P.astype(np.float64)
    np.testing.assert_allclose(qs, ref, rtol=1e-14)


def test_scores_identity_basis_equal_full_dot_products():
    G, d, T = 4, 64, 200
    Q = _rand_bf16((G, d), 7)
    K = _rand_bf16((T, d), 8)
    P = np.eye(d, dtype=np.float32)
    Kp, _ = oracle.project_rows(K, P)
    s = oracle.scores(oracle.query_proj(Q, P), Kp)
    ref = oracle.bf16_to_f64(K) @ oracle.bf16_to_f64(Q).sum(0)
    np.testing.assert_allclose(s, ref, rtol=1e-13, atol=1e-13)


# ----------------------------------------------------------------------------- top-k
def test_topk_golden_cases():
    d = json.load(open(os.path.join(GOLD, "topk_ties.json")))
    for c in d["cases"]:
        idx, k_eff = oracle.topk(np.array(c["scores"], np.float64), c["k"])
        assert k_eff == c["k_eff"], c
        assert idx.tolist() == c["idx"], c


def _pairwise_valid(s, sel_set):
    # every selected token beats every unselected one: larger score, or equal score and lower index
    for i in sel_set:
        for j in range(len(s)):
            if j in sel_set:
                continue
            if not (s[i] > s[j] or (s[i] == s[j] and i < j)):
                return False
    return True


@pytest.mark.parametrize("seed", range(25))
def test_topk_pairwise_brute_force(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 65))
    k = int(rng.integers(1, n + 3))
    # few distinct values to force many ties
    s = rng.integers(-4, 5, size=n).astype(np.float64) * 0.5
    idx, k_eff = oracle.topk(s, k)
    assert k_eff == min(k, n)
    sel = [int(i) for i in idx[:k_eff]]
    assert sel == sorted(sel) and len(set(sel)) == k_eff
    assert all(i == -1 for i in idx[k_eff:])
    assert _pairwise_valid(s, set(sel))


@pytest.mark.parametrize("seed", range(10))
def test_topk_exhaustive_subset_maximisation(seed):
    rng = np.random.default_rng(100 + seed)
    n = int(rng.integers(2, 13))
    k = int(rng.integers(1, n + 1))
    s = rng.integers(-3, 4, size=n).astype(np.float64)
    best = None
    for comb in itertools.combinations(range(n), k):
        key = (sum(s[list(comb)]), tuple(-c for c in comb))  # max sum, then lexicographically lowest
        if best is None or key > best[0]:
            best = (key, comb)
    idx, _ = oracle.topk(s, k)
    assert tuple(idx.tolist()) == best[1]


def test_topk_matches_numpy_lexsort():
    rng = np.random.default_rng(7)
    s = np.round(rng.standard_normal(5000), 2)    # many exact ties
    order = np.lexsort((np.arange(s.size), -s))   # primary: score desc, secondary: index asc
    idx, _ = oracle.topk(s, 300)
    np.testing.assert_array_equal(idx, np.sort(order[:300]))


def test_topk_permutation_invariance():
    rng = np.random.default_rng(3)
    s = rng.standard_normal(1000)                  # distinct values
    perm = rng.permutation(1000)
    idx, _ = oracle.topk(s, 50)
    idx_p, _ = oracle.topk(s[perm], 50)
    assert set(perm[idx_p].tolist()) == set(idx.tolist())


# ----------------------------------------------------------------------------- attention
def _torch_attention(Q, K, V, tokens, scale):
    q = torch.from_numpy(oracle.bf16_to_f64(Q))
    k = torch.from_numpy(oracle.bf16_to_f64(K))[tokens]
    v = torch.from_numpy(oracle.bf16_to_f64(V))[tokens]
    logits = scale * q @ k.T
    return (torch.softmax(logits, dim=-1) @ v).numpy(), torch.logsumexp(logits, dim=-1).numpy()


def test_attention_golden_two_tokens():
    d = json.load(open(os.path.join(GOLD, "attention_two_tokens.json")))
    Q, K, V = (_bf16_bits_of(np.array(d[x])) for x in ("Q", "K", "V"))
    O, lse = oracle.attention(Q, K, V, d["tokens"], d["scale"])
    np.testing.assert_allclose(O, np.array(d["O"]), rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, np.array(d["lse"]), rtol=0, atol=1e-15)


def test_attention_matches_torch_softmax_on_all_tokens():
    G, dk, dv, T = 4, 128, 96, 300
    Q, K, V = _rand_bf16((G, dk), 11, 0.2), _rand_bf16((T, dk), 12), _rand_bf16((T, dv), 13)
    tokens = np.arange(T)
    O, lse = oracle.attention(Q, K, V, tokens, 1 / math.sqrt(dk))
    Or, lr = _torch_attention(Q, K, V, tokens, 1 / math.sqrt(dk))
    np.testing.assert_allclose(O, Or, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse, lr, rtol=0, atol=1e-12)


def test_attention_single_token_returns_its_value_row():
    Q, K, V = _rand_bf16((3, 64), 14), _rand_bf16((50, 64), 15), _rand_bf16((50, 64), 16)
    O, _ = oracle.attention(Q, K, V, [37], 0.125)
    np.testing.assert_array_equal(O, np.repeat(oracle.bf16_to_f64(V[37:38]), 3, axis=0))


def test_attention_zero_query_is_value_mean():
    K, V = _rand_bf16((40, 32), 17), _rand_bf16((40, 32), 18)
    Q = np.zeros((2, 32), np.uint16)
    tokens = [1, 5, 9, 30]
    O, lse = oracle.attention(Q, K, V, tokens, 1.0)
    np.testing.assert_allclose(O[0], oracle.bf16_to_f64(V[tokens]).mean(0), rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, math.log(4.0), atol=1e-15)


def test_attention_is_order_free_and_empty_is_zero():
    Q, K, V = _rand_bf16((2, 32), 19), _rand_bf16((60, 32), 20), _rand_bf16((60, 16), 21)
    a, la = oracle.attention(Q, K, V, [3, 50, 7, 22], 0.3)
    b, lb = oracle.attention(Q, K, V, [22, 3, 7, 50], 0.3)
    np.testing.assert_allclose(a, b, atol=1e-15)
    np.testing.assert_allclose(la, lb, atol=1e-15)
    O, lse = oracle.attention(Q, K, V, [], 0.3)
    assert np.all(O == 0) and np.all(np.isneginf(lse))


# ----------------------------------------------------------------------------- whole step
def _small_problem(seed, G=4, d=64, r=16, T=400):
    Q = _rand_bf16((G, d), seed, 0.3)
    K = _rand_bf16((T, d), seed + 1)
    V = _rand_bf16((T, d), seed + 2)
    P = synth.orthonormal_basis(d, r, seed=seed + 3).numpy()
    Kp, _ = oracle.project_rows(K, P)
    return Q, K, V, P, Kp


def test_step_identity_basis_selects_full_score_topk():
    # r = d and P = I: the selection is the exact top-k of the full group scores.
    G, d, T, k = 4, 64, 500, 40
    Q, K, V, _, _ = _small_problem(30, G, d, d, T)
    P = np.eye(d, dtype=np.float32)
    Kp, _ = oracle.project_rows(K, P)
    res = oracle.decode_head(Q, K, V, Kp, P, T, k, 0, 0.125)
    full = oracle.bf16_to_f64(K) @ oracle.bf16_to_f64(Q).sum(0)
    order = np.lexsort((np.arange(T), -full))
    np.testing.assert_array_equal(res["idx"], np.sort(order[:k]))


def test_step_with_k_equal_T_is_dense_attention():
    # §4.5's full-KV baseline: with k = T the sparse step attends to every token.
    Q, K, V, P, Kp = _small_problem(40)
    T = K.shape[0]
    res = oracle.decode_head(Q, K, V, Kp, P, T, T, 0, 0.125)
    O, lse = _torch_attention(Q, K, V, np.arange(T), 0.125)
    np.testing.assert_allclose(res["O"], O, atol=1e-13)
    np.testing.assert_allclose(res["lse"], lse, atol=1e-12)
    assert res["k_eff"] == T


def test_step_window_covering_everything_is_dense():
    Q, K, V, P, Kp = _small_problem(50)
    T = K.shape[0]
    res = oracle.decode_head(Q, K, V, Kp, P, T, 16, T + 5, 0.125)
    O, _ = _torch_attention(Q, K, V, np.arange(T), 0.125)
    np.testing.assert_allclose(res["O"], O, atol=1e-13)
    assert res["k_eff"] == 0 and np.all(res["idx"] == -1)


def test_step_window_attends_selection_plus_recent_tokens():
    Q, K, V, P, Kp = _small_problem(60)
    T, k, W = K.shape[0], 20, 50
    res = oracle.decode_head(Q, K, V, Kp, P, T, k, W, 0.125)
    s = oracle.scores(oracle.query_proj(Q, P), Kp[: T - W])
    idx, _ = oracle.topk(s, k)
    assert np.all(idx < T - W)
    np.testing.assert_array_equal(res["idx"], idx)
    toks = np.concatenate([idx, np.arange(T - W, T)])
    O, _ = _torch_attention(Q, K, V, toks, 0.125)
    np.testing.assert_allclose(res["O"], O, atol=1e-13)


def test_step_permuting_cache_rows_keeps_selected_rows_and_output():
    Q, K, V, P, Kp = _small_problem(70, T=300)
    T, k = 300, 25
    res = oracle.decode_head(Q, K, V, Kp, P, T, k, 0, 0.125)
    s = res["scores"]
    kth = np.sort(s)[::-1][k - 1]
    assert np.sum(s == kth) == 1                  # no tie at the boundary for this seed
    perm = np.random.default_rng(1).permutation(T)
    res_p = oracle.decode_head(Q, K[perm], V[perm], Kp[perm], P, T, k, 0, 0.125)
    assert set(perm[res_p["idx"]].tolist()) == set(res["idx"].tolist())
    np.testing.assert_allclose(res_p["O"], res["O"], atol=1e-13)


def test_step_mla_shape_reduces_to_gqa_formula():
    # MLA (§3.3, §A.3): one latent row per token serves as the key (576 dims) and, on its
    # first 512 dims, as the value; all 128 query heads share one index set.
    G, dk, dv, r, T, k = 128, 576, 512, 64, 160, 12
    Q = _rand_bf16((G, dk), 80, 0.05)
    L = _rand_bf16((T, dk), 81)
    P = synth.orthonormal_basis(dk, r, seed=82).numpy()
    Kp, _ = oracle.project_rows(L, P)
    res = oracle.decode_head(Q, L, L[:, :dv], Kp, P, T, k, 0, 1 / math.sqrt(dk))
    full_q = P.astype(np.float64).T @ oracle.bf16_to_f64(Q).sum(0)
    s = oracle.bf16_to_f64(Kp) @ full_q
    order = np.lexsort((np.arange(T), -s))
    np.testing.assert_array_equal(res["idx"], np.sort(order[:k]))
    O, _ = _torch_attention(Q, L, np.ascontiguousarray(L[:, :dv]), res["idx"], 1 / math.sqrt(dk))
    np.testing.assert_allclose(res["O"], O, atol=1e-13)


# ----------------------------------------------------------------------------- FP8 E4M3 projected cache
def test_e4m3_decodes_the_format_constants():
    # OCP E4M3: bias 7, 3 mantissa bits, subnormals m * 2^-9, S.1111.111 is NaN, max 448
    assert oracle.e4m3_to_double(0x7E) == 448.0
    assert oracle.e4m3_to_double(0x08) == 2.0 ** -6      # smallest normal
    assert oracle.e4m3_to_double(0x07) == 7 * 2.0 ** -9  # largest subnormal
    assert oracle.e4m3_to_double(0x01) == 2.0 ** -9      # smallest subnormal
    assert oracle.e4m3_to_double(0x38) == 1.0
    assert oracle.e4m3_to_double(0x40) == 2.0
    assert oracle.e4m3_to_double(0x3C) == 1.5
    assert oracle.e4m3_to_double(0xB8) == -1.0
    assert oracle.e4m3_to_double(0x00) == 0.0 and math.copysign(1.0, oracle.e4m3_to_double(0x80)) == -1.0
    assert math.isnan(oracle.e4m3_to_double(0x7F)) and math.isnan(oracle.e4m3_to_double(0xFF))


def test_e4m3_agrees_with_torch_float8_on_every_code_and_on_in_range_rounding():
    codes = torch.arange(256, dtype=torch.uint8)
    tvals = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        v = oracle.e4m3_to_double(c)
        if math.isnan(v):
            assert math.isnan(tvals[c])
        else:
            assert v == tvals[c], (c, v, tvals[c])
    g = torch.Generator().manual_seed(7)
    x = torch.cat([torch.randn(4000, generator=g, dtype=torch.float64) * s for s in (1e-3, 0.05, 1.0, 30.0)])
    x = x[x.abs() < 440]
    mids = torch.tensor([1 + 1 / 16, 1 + 3 / 16, 2 ** -9 * 0.5, 2 ** -9 * 1.5, 2 ** -9 * 2.5, 240 + 8], dtype=torch.float64)
    x = torch.cat([x, mids, -mids])
    ref = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.double_to_e4m3(float(v)) for v in x.numpy()], np.uint8)
    np.testing.assert_array_equal(got, ref)


def test_e4m3_encoding_ties_to_even_and_saturates():
    assert oracle.double_to_e4m3(1 + 1 / 16) == 0x38           # midway 1.0 / 1.125 -> even mantissa
    assert oracle.double_to_e4m3(1 + 3 / 16) == 0x3A           # midway 1.125 / 1.25 -> even
    assert oracle.double_to_e4m3(0.5 * 2.0 ** -9) == 0x00      # midway 0 / 2^-9 -> 0
    assert oracle.double_to_e4m3(1.5 * 2.0 ** -9) == 0x02      # midway 1 / 2 subnormal steps -> 2
    assert oracle.double_to_e4m3(460.0) == 0x7E and oracle.double_to_e4m3(1e9) == 0x7E
    assert oracle.double_to_e4m3(-1e9) == 0xFE
    for c in list(range(0, 0x7F)) + list(range(0x80, 0xFF)):   # every finite code round-trips
        assert oracle.double_to_e4m3(oracle.e4m3_to_double(c)) == c


def test_e4m3_projection_is_the_rounded_exact_product():
    rng = np.random.default_rng(3)
    d, r, n = 64, 16, 50
    K = rng.standard_normal((n, d)).astype(np.float32)
    Kb = (K.view(np.uint32) >> 16).astype(np.uint16)        # bf16 truncation of the inputs
    P = np.linalg.qr(rng.standard_normal((d, r)))[0].astype(np.float32)
    Kp8, ex = oracle.project_rows_e4m3(Kb, P)
    Kd = oracle.bf16_to_f64(Kb)
    exact = Kd @ P.astype(np.float64)
    np.testing.assert_allclose(ex, exact, rtol=1e-12, atol=1e-12)
    want = np.array([[oracle.double_to_e4m3(v) for v in row] for row in exact], np.uint8)
    np.testing.assert_array_equal(Kp8, want)
    qs = rng.standard_normal(r)
    vals = np.vectorize(oracle.e4m3_to_double)(Kp8)
    np.testing.assert_allclose(oracle.scores_e4m3(qs, Kp8), vals @ qs, rtol=1e-13)


def test_e4m3_decode_head_equals_the_bf16_step_on_the_same_values():
    # every finite E4M3 value is exactly a bf16 value, so the FP8 step on codes c must equal the
    # bf16 step (the C decode_head) on bf16(value(c)): same scores, selection and output
    rng = np.random.default_rng(11)
    G, d, r, T, k, W = 4, 32, 16, 300, 20, 16
    bf = lambda a: oracle.bf16_round(np.asarray(a, np.float64))
    Qg, K, V = bf(rng.standard_normal((G, d))), bf(rng.standard_normal((T, d))), bf(rng.standard_normal((T, d)))
    P = np.linalg.qr(rng.standard_normal((d, r)))[0].astype(np.float32)
    codes = rng.integers(0, 256, (T, r)).astype(np.uint8)
    codes[(codes & 0x7F) == 0x7F] = 0x38                    # no NaN codes
    vals = np.vectorize(oracle.e4m3_to_double)(codes)
    a = oracle.decode_head_e4m3(Qg, K, V, codes, P, T, k, W, 0.125)
    b = oracle.decode_head(Qg, K, V, bf(vals), P, T, k, W, 0.125)
    np.testing.assert_array_equal(a["scores"], b["scores"])
    assert a["k_eff"] == b["k_eff"] == k
    np.testing.assert_array_equal(a["idx"], b["idx"])
    np.testing.assert_allclose(a["O"], b["O"], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(a["lse"], b["lse"], rtol=1e-13)
