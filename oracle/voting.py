"""CPU oracle of head-shared soft voting.  TEST INFRASTRUCTURE ONLY (like the rest of
``oracle``).

"Joint Subspace Sparse Attention for Efficient Long-Context Decoding", §1 (forcing the KV
heads to share one selected set can degrade accuracy) and §E.3 / Table 15 (per-KV-head
selection against head-shared soft voting).  The pages name the variant but do not define
the vote.  The reading used here: every KV head h of a sequence turns its subspace scores
over the candidates into a distribution,

  p_h(t) = softmax_t( c * s_h(t) ),   c = sm_scale / G,

(s_h is the score of the summed group query, so c * s_h is the softmax logit of the
group-mean query), the distributions are added, v(t) = sum_h p_h(t), and the top-k of v
(ties to the lower index, output ascending) is the one index set every KV head attends
over.  With one KV head the vote ranks exactly as the scores do.
"""
from __future__ import annotations

import numpy as np

from . import query_proj, scores as _scores, topk as _topk


def head_distributions(s: np.ndarray, c: float) -> np.ndarray:
    """p[h, t] = exp(c s[h, t] - max_t c s[h, t]) / sum_t exp(...) in fp64; s [Hkv, n]."""
    x = c * np.asarray(s, np.float64)
    if x.shape[1] == 0:
        return x.copy()
    e = np.exp(x - x.max(axis=1, keepdims=True))
    return e / e.sum(axis=1, keepdims=True)


def votes(s: np.ndarray, c: float) -> np.ndarray:
    """v[t] = sum_h p_h(t)."""
    return head_distributions(s, c).sum(axis=0)


def vote_select(Q_b, P, Kp_b, T: int, k: int, W: int, sm_scale: float):
    """Shared selection of one sequence.

    Q_b bf16 codes [Hq, d]; P float32 [Hkv, d, r]; Kp_b bf16 codes [Hkv, >= T, r].
    Returns (idx int32 [k] ascending, -1 padded; k_eff; v float64 [n]; s float64 [Hkv, n])."""
    Hkv = P.shape[0]
    G = Q_b.shape[0] // Hkv
    n = T - min(max(W, 0), T)
    s = np.stack([_scores(query_proj(Q_b[h * G:(h + 1) * G], P[h]), Kp_b[h][:n]) for h in range(Hkv)]) \
        if n > 0 else np.zeros((Hkv, 0))
    v = votes(s, sm_scale / G)
    idx, k_eff = _topk(v, k)
    return idx, k_eff, v, s
