"""Pins of the head-shared soft-voting oracle (oracle/voting.py) against facts fixed
independently of its code: a hand example, the one-head reduction to the score ranking,
softmax shift invariance per head, a head with flat scores casting uniform votes, and a
brute-force restatement over tiny inputs ("Joint Subspace Sparse Attention for Efficient
Long-Context Decoding", §1, §E.3)."""
import math

import numpy as np

import oracle
from oracle import voting


def test_hand_example():
    # two heads, three tokens, c = 1: head 0 scores (0, ln 2, 0), head 1 (ln 3, 0, 0)
    s = np.array([[0.0, math.log(2.0), 0.0], [math.log(3.0), 0.0, 0.0]])
    v = voting.votes(s, 1.0)
    np.testing.assert_allclose(v, [1 / 4 + 3 / 5, 2 / 4 + 1 / 5, 1 / 4 + 1 / 5], rtol=1e-15)
    idx, k_eff = oracle.topk(v, 2)
    assert k_eff == 2 and idx.tolist() == [0, 1]


def test_one_head_votes_rank_like_the_scores():
    rng = np.random.default_rng(0)
    s = rng.standard_normal((1, 500)) * 3
    s[0, 17] = s[0, 40]                               # an exact tie keeps the lower index
    for c in (0.05, 1.0, 7.0):
        np.testing.assert_array_equal(oracle.topk(voting.votes(s, c), 60)[0], oracle.topk(s[0], 60)[0])


def test_each_head_is_shift_invariant_and_sums_to_one():
    rng = np.random.default_rng(1)
    s = rng.standard_normal((4, 300))
    p = voting.head_distributions(s, 0.7)
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=1e-14)
    shifted = s + np.array([[5.0], [-3.0], [0.0], [1e3]])
    np.testing.assert_allclose(voting.votes(shifted, 0.7), voting.votes(s, 0.7), rtol=1e-12)


def test_a_flat_head_casts_uniform_votes():
    rng = np.random.default_rng(2)
    s = np.vstack([rng.standard_normal(200), np.full(200, 3.25)])
    v = voting.votes(s, 1.3)
    np.testing.assert_allclose(v - 1.0 / 200, voting.head_distributions(s[:1], 1.3)[0], atol=1e-15)


def test_brute_force_restatement():
    rng = np.random.default_rng(3)
    for _ in range(20):
        H, n, c = rng.integers(1, 5), rng.integers(1, 9), float(rng.uniform(0.1, 3))
        s = rng.standard_normal((H, n))
        want = [sum(math.exp(c * s[h, t]) / sum(math.exp(c * s[h, u]) for u in range(n)) for h in range(H))
                for t in range(n)]
        np.testing.assert_allclose(voting.votes(s, c), want, rtol=1e-12)


def test_vote_select_composes_the_steps():
    rng = np.random.default_rng(4)
    Hkv, G, d, r, T, k, W = 2, 4, 32, 16, 90, 10, 5
    bf = lambda a: oracle.bf16_round(np.asarray(a, np.float64))
    Q = bf(rng.standard_normal((Hkv * G, d)))
    P = np.stack([np.linalg.qr(rng.standard_normal((d, r)))[0] for _ in range(Hkv)]).astype(np.float32)
    K = bf(rng.standard_normal((Hkv, T, d)))
    Kp = np.stack([oracle.project_rows(K[h], P[h])[0] for h in range(Hkv)])
    idx, k_eff, v, s = voting.vote_select(Q, P, Kp, T, k, W, 0.25)
    for h in range(Hkv):
        np.testing.assert_array_equal(s[h], oracle.scores(oracle.query_proj(Q[h * G:(h + 1) * G], P[h]), Kp[h][:T - W]))
    np.testing.assert_allclose(v, voting.votes(s, 0.25 / G), rtol=0)
    assert k_eff == k and np.all(np.diff(idx) > 0)
    assert set(idx.tolist()) == set(np.argsort(-v, kind="stable")[:k].tolist())
