"""CPU oracle of the JSSA basis calibration.  TEST INFRASTRUCTURE ONLY (like the rest of
``oracle``: only the tests, the smoke check and the benchmark's CPU legs may use it).

"Joint Subspace Sparse Attention for Efficient Long-Context Decoding", §3.2 (one
orthonormal basis for queries and keys, chosen to minimise the expected bilinear score
error; a marginal upper bound has a closed-form spectral solution; the group-mean query;
unit-trace normalisation of the query and key second moments), §A.4 (one basis per
layer and KV head from packed calibration sequences), §B.1 (query and key treated as
independent draws), §B.2 (trace normalisation), §B.3 (the bound needs no commuting
moments).  The pages do not print the closed form.  The reading used here:

  exact objective      E[(q^T k - (P^T q)^T (P^T k))^2] = E[(q^T (I - PP^T) k)^2]
  product of marginals = tr((I - PP^T) S_k (I - PP^T) S_q)          (q, k independent)
  Cauchy-Schwarz       <= tr((I - PP^T) S_q) * tr((I - PP^T) S_k)
  unit-trace moments   a = tr((I - PP^T) S_q / tr S_q), b = likewise for S_k, and
                       a * b <= ((a + b) / 2)^2 (arithmetic-geometric mean)
  surrogate            a + b = 2 - tr(P^T (S_q / tr S_q + S_k / tr S_k) P)

so the surrogate is minimised by the top-r eigenvectors of M = S_q / tr S_q + S_k / tr S_k
(Ky Fan), with S_q and S_k the uncentred second moments of the group-mean query and the
key over the calibration tokens.  Nothing in it needs S_q and S_k to commute.

Conventions (fixed here, shared with the GPU kernels only through this text): columns in
descending eigenvalue order; each column's sign makes its largest-magnitude entry
positive (the lowest index among equal magnitudes).  Numpy's symmetric eigensolver is
the library step.
"""
from __future__ import annotations

import numpy as np

from . import bf16_to_f64


def moments(Qc: np.ndarray, Kc: np.ndarray):
    """Second moments over N calibration tokens of one KV head.

    Qc: bf16 codes (uint16) [G, N, d], the KV head's G query heads; Kc: bf16 codes [N, d].
    Returns (S_q, S_k) float64 [d, d]: S_q = (1/N) sum_t qbar_t qbar_t^T with
    qbar_t = (1/G) sum_g q_{g,t} (the group-mean query, §3.2), S_k = (1/N) sum_t k_t k_t^T.
    """
    q = bf16_to_f64(np.asarray(Qc, np.uint16))
    k = bf16_to_f64(np.asarray(Kc, np.uint16))
    G, N, d = q.shape
    qbar = q.sum(axis=0) / G
    return qbar.T @ qbar / N, k.T @ k / N


def normalised_sum(S_q: np.ndarray, S_k: np.ndarray) -> np.ndarray:
    """M = S_q / tr S_q + S_k / tr S_k (§B.2: each moment scaled to unit trace)."""
    return S_q / np.trace(S_q) + S_k / np.trace(S_k)


def fix_signs(P: np.ndarray) -> np.ndarray:
    """Flip each column so that its largest-magnitude entry (lowest index on ties) is positive."""
    P = np.array(P, np.float64, copy=True)
    for j in range(P.shape[1]):
        i = int(np.argmax(np.abs(P[:, j])))
        if P[i, j] < 0:
            P[:, j] = -P[:, j]
    return P


def spectral_basis(S_q: np.ndarray, S_k: np.ndarray, r: int):
    """The rank-r basis minimising the surrogate: the top-r eigenvectors of M.

    Returns (P float64 [d, r], eigenvalues of M float64 [d], descending)."""
    M = normalised_sum(S_q, S_k)
    w, V = np.linalg.eigh(M)
    order = np.argsort(-w, kind="stable")
    return fix_signs(V[:, order[:r]]), w[order]


def surrogate(S_q: np.ndarray, S_k: np.ndarray, P: np.ndarray) -> float:
    """a + b of the module docstring for an orthonormal P [d, r]."""
    M = normalised_sum(S_q, S_k)
    return float(2.0 - np.trace(P.T @ M @ P))


def marginal_objective(S_q: np.ndarray, S_k: np.ndarray, P: np.ndarray) -> float:
    """tr((I - PP^T) S_k (I - PP^T) S_q): the product-of-marginals score error (§B.1)."""
    R = np.eye(P.shape[0]) - P @ P.T
    return float(np.trace(R @ S_k @ R @ S_q))


def calibrate(Qc: np.ndarray, Kc: np.ndarray, r: int):
    """Basis of one KV head from its calibration tokens: (P [d, r], eigenvalues)."""
    return spectral_basis(*moments(Qc, Kc), r)
