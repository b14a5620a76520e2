"""Pins of the calibration oracle (oracle/calibration.py) against mathematics fixed
independently of its code: hand-derived moments, the product-of-marginals identity checked
by brute force over query-key pairs, the two bounds of the surrogate, optimality of the
spectral basis against random bases, the diagonal (channel-selection) special case, the
invariances that trace normalisation implies, and recall on planted low-rank data.
("Joint Subspace Sparse Attention for Efficient Long-Context Decoding", §3.2, §B.1-§B.3.)
"""
import numpy as np
import pytest

import oracle
from oracle import calibration as cal


def bf(a):
    return oracle.bf16_round(np.asarray(a, np.float64))


def orthonormal(rng, d, r):
    return np.linalg.qr(rng.standard_normal((d, r)))[0]


def test_moments_of_a_hand_example():
    # G = 2 heads, N = 2 tokens, d = 3.  Token 0: q = (2, 0, 0) and (0, 0, 4) -> mean (1, 0, 2);
    # token 1: q = (0, 2, 0) and (0, 2, 0) -> mean (0, 2, 0).  Keys (1, 0, 0) and (0, 0, -2).
    Qc = bf([[[2, 0, 0], [0, 2, 0]], [[0, 0, 4], [0, 2, 0]]])
    Kc = bf([[1, 0, 0], [0, 0, -2]])
    S_q, S_k = cal.moments(Qc, Kc)
    np.testing.assert_array_equal(S_q, np.array([[1, 0, 2], [0, 4, 0], [2, 0, 4]]) / 2.0)
    np.testing.assert_array_equal(S_k, np.diag([1.0, 0.0, 4.0]) / 2.0)


def test_product_of_marginals_identity_by_brute_force():
    # the mean over every (query, key) pair of the squared score error equals the trace form
    rng = np.random.default_rng(1)
    G, N, d, r = 2, 7, 6, 2
    Qc, Kc = bf(rng.standard_normal((G, N, d))), bf(rng.standard_normal((N, d)))
    S_q, S_k = cal.moments(Qc, Kc)
    P = orthonormal(rng, d, r)
    qbar = oracle.bf16_to_f64(Qc).mean(axis=0)
    k = oracle.bf16_to_f64(Kc)
    errs = [(qbar[s] @ k[t] - (P.T @ qbar[s]) @ (P.T @ k[t])) ** 2 for s in range(N) for t in range(N)]
    assert cal.marginal_objective(S_q, S_k, P) == pytest.approx(np.mean(errs), rel=1e-12)


@pytest.mark.parametrize("seed", range(5))
def test_the_surrogate_bounds_the_marginal_objective(seed):
    rng = np.random.default_rng(10 + seed)
    G, N, d, r = 4, 200, 16, 4
    A = rng.standard_normal((d, d)) * np.geomspace(3, 0.1, d)        # anisotropic, non-commuting
    Qc = bf(rng.standard_normal((G, N, d)) @ A)
    Kc = bf(rng.standard_normal((N, d)) @ rng.standard_normal((d, d)) * 5)
    S_q, S_k = cal.moments(Qc, Kc)
    assert np.linalg.norm(S_q @ S_k - S_k @ S_q) > 1e-3 * np.linalg.norm(S_q) * np.linalg.norm(S_k)
    for P in [orthonormal(rng, d, r) for _ in range(20)] + [cal.spectral_basis(S_q, S_k, r)[0]]:
        R = np.eye(d) - P @ P.T
        exact = cal.marginal_objective(S_q, S_k, P)
        cs = np.trace(R @ S_q) * np.trace(R @ S_k)                                   # Cauchy-Schwarz
        a, b = np.trace(R @ S_q) / np.trace(S_q), np.trace(R @ S_k) / np.trace(S_k)
        assert exact <= cs * (1 + 1e-12)
        assert cs <= np.trace(S_q) * np.trace(S_k) * ((a + b) / 2) ** 2 * (1 + 1e-12)
        assert cal.surrogate(S_q, S_k, P) == pytest.approx(a + b, rel=1e-12)


def test_the_spectral_basis_minimises_the_surrogate():
    rng = np.random.default_rng(3)
    d, r = 24, 5
    S_q = np.cov(rng.standard_normal((d, 300)) * np.linspace(4, 0.2, d)[:, None])
    S_k = np.cov(rng.standard_normal((d, 300)) * np.linspace(0.3, 6, d)[:, None])
    P, w = cal.spectral_basis(S_q, S_k, r)
    np.testing.assert_allclose(P.T @ P, np.eye(r), atol=1e-12)
    best = cal.surrogate(S_q, S_k, P)
    assert best == pytest.approx(2.0 - w[:r].sum(), rel=1e-12)
    assert np.all(np.diff(w) <= 0)
    for _ in range(300):
        assert cal.surrogate(S_q, S_k, orthonormal(rng, d, r)) >= best - 1e-12


def test_diagonal_moments_select_channels():
    # diagonal moments: the basis is the r coordinate axes with the largest normalised mass
    # (a channel selector, the FASA-style special case of §2.1)
    sq = np.array([5.0, 1.0, 0.5, 3.0, 0.1, 0.4])
    sk = np.array([0.2, 4.0, 0.3, 0.2, 0.1, 0.2])
    P, _ = cal.spectral_basis(np.diag(sq), np.diag(sk), 3)
    m = sq / sq.sum() + sk / sk.sum()
    want = np.argsort(-m)[:3]
    np.testing.assert_array_equal(np.argmax(np.abs(P), axis=0), want)
    np.testing.assert_allclose(np.abs(P).max(axis=0), 1.0)
    assert np.all(P.max(axis=0) == 1.0)      # sign convention: the largest entry is positive


def test_trace_normalisation_makes_the_basis_scale_free():
    rng = np.random.default_rng(4)
    G, N, d, r = 2, 300, 12, 3
    Qc = bf(rng.standard_normal((G, N, d)) * np.linspace(2, 0.5, d))
    Kc = bf(rng.standard_normal((N, d)) @ rng.standard_normal((d, d)))
    P1, _ = cal.calibrate(Qc, Kc, r)
    P2, _ = cal.calibrate(Qc, bf(oracle.bf16_to_f64(Kc) * 16.0), r)     # exact power-of-two rescale
    P3, _ = cal.calibrate(bf(oracle.bf16_to_f64(Qc) / 8.0), Kc, r)
    np.testing.assert_allclose(P2, P1, atol=1e-10)
    np.testing.assert_allclose(P3, P1, atol=1e-10)
    perm = rng.permutation(N)                                             # token order is irrelevant
    P4, _ = cal.calibrate(Qc[:, perm], Kc[perm], r)
    np.testing.assert_allclose(P4, P1, atol=1e-10)


def test_without_normalisation_the_larger_moment_would_dominate():
    # the reading's normalisation matters: unnormalised, a key moment 100x larger swamps the
    # query directions; normalised, both contribute (§B.2)
    d = 4
    S_q = np.diag([1.0, 0.0, 0.0, 0.0])
    S_k = np.diag([0.0, 100.0, 99.0, 0.0])
    P, _ = cal.spectral_basis(S_q, S_k, 2)
    assert set(np.argmax(np.abs(P), axis=0).tolist()) == {0, 1}
    w, V = np.linalg.eigh(S_q + S_k)
    assert set(np.argmax(np.abs(V[:, np.argsort(-w)[:2]]), axis=0).tolist()) == {1, 2}


def test_spectral_basis_recovers_the_planted_subspace_better_than_a_random_one():
    # keys and queries share a rank-8 structure plus noise (the synthetic recipe's form): the
    # calibrated r = 8 basis finds the true top-k of full-dimensional scores far more often
    rng = np.random.default_rng(5)
    G, N, d, r, R, k = 4, 4000, 64, 8, 8, 64
    A = rng.standard_normal((R, d)) / np.sqrt(R)
    Kc = bf(rng.standard_normal((N, R)) @ A + 0.3 * rng.standard_normal((N, d)))
    Qc = bf((rng.standard_normal((G, N, R)) @ A + 0.3 * rng.standard_normal((G, N, d))) / np.sqrt(d))
    P, _ = cal.calibrate(Qc, Kc, r)
    Prand = orthonormal(rng, d, r)
    keys = oracle.bf16_to_f64(Kc)
    rec = {"spectral": [], "random": []}
    for t in range(20):
        q = oracle.bf16_to_f64(Qc)[:, t].mean(axis=0)
        truth = set(np.argsort(-(keys @ q), kind="stable")[:k].tolist())
        for name, B in (("spectral", P), ("random", Prand)):
            s = (keys @ B) @ (B.T @ q)
            rec[name].append(len(truth & set(np.argsort(-s, kind="stable")[:k].tolist())) / k)
    assert np.mean(rec["spectral"]) > 0.8
    assert np.mean(rec["spectral"]) > np.mean(rec["random"]) + 0.3
