"""CPU oracle for the JSSA decode step.  TEST INFRASTRUCTURE ONLY.

A plain, slow, single-threaded fp64 restatement of what the decode step computes,
written from "Joint Subspace Sparse Attention for Efficient Long-Context Decoding"
(arXiv 2610.19026v1, paperlayer.ai summary: Figure 1, §3.1-§3.4, §A.3, §E.1, §E.3).
The arithmetic lives in ``oracle.c``; this module only marshals numpy arrays.

Only the tests, the smoke check and the CPU-baseline leg of the benchmark may use
it.  It imports nothing from the CUDA package and the CUDA package never imports it.

Array conventions: bf16 data is passed as ``numpy.uint16`` bit patterns, the basis P
as ``float32`` of shape [d, r] (one KV head) or [Hkv, d, r], scores as ``float64``.
The last dimension of every row array must be contiguous; rows may be strided.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = C.CDLL(_build.build())
        u16p, f32p, f64p = C.POINTER(C.c_uint16), C.POINTER(C.c_float), C.POINTER(C.c_double)
        i32p, i64p = C.POINTER(C.c_int32), C.POINTER(C.c_int64)
        lib.or_bf16_to_double.argtypes = [C.c_uint16]
        lib.or_bf16_to_double.restype = C.c_double
        lib.or_double_to_bf16.argtypes = [C.c_double]
        lib.or_double_to_bf16.restype = C.c_uint16
        lib.or_double_to_bf16_array.argtypes = [f64p, C.c_int64, u16p]
        lib.or_project_rows.argtypes = [u16p, C.c_int64, C.c_int, f32p, C.c_int, C.c_int64,
                                        u16p, C.c_int64, f64p]
        u8p = C.POINTER(C.c_uint8)
        lib.or_e4m3_to_double.argtypes = [C.c_uint8]
        lib.or_e4m3_to_double.restype = C.c_double
        lib.or_double_to_e4m3.argtypes = [C.c_double]
        lib.or_double_to_e4m3.restype = C.c_uint8
        lib.or_project_rows_e4m3.argtypes = [u16p, C.c_int64, C.c_int, f32p, C.c_int, C.c_int64, u8p, C.c_int64, f64p]
        lib.or_scores_e4m3.argtypes = [f64p, C.c_int, u8p, C.c_int64, C.c_int64, f64p]
        lib.or_query_proj.argtypes = [u16p, C.c_int, C.c_int, f32p, C.c_int, f64p]
        lib.or_scores.argtypes = [f64p, C.c_int, u16p, C.c_int64, C.c_int64, f64p]
        lib.or_topk.argtypes = [f64p, C.c_int64, C.c_int64, i32p]
        lib.or_topk.restype = C.c_int64
        lib.or_attention.argtypes = [u16p, C.c_int, C.c_int, u16p, C.c_int64, u16p, C.c_int64,
                                     C.c_int, i64p, C.c_int64, C.c_double, f64p, f64p]
        lib.or_decode_head.argtypes = [u16p, C.c_int, C.c_int, C.c_int, u16p, C.c_int64,
                                       u16p, C.c_int64, u16p, C.c_int64, f32p, C.c_int,
                                       C.c_int64, C.c_int64, C.c_int64, C.c_double,
                                       i32p, f64p, f64p, f64p]
        lib.or_decode_head.restype = C.c_int64
        _lib = lib
    return _lib


def _ptr(a: np.ndarray, ctype):
    return a.ctypes.data_as(C.POINTER(ctype))


def _rows(a: np.ndarray, dtype) -> tuple[np.ndarray, int]:
    """Return (array, row stride in elements) for a 2-D row array with a contiguous last dim."""
    assert a.dtype == dtype and a.ndim == 2, (a.dtype, a.shape)
    if a.shape[0] == 0:
        return np.zeros((1, max(a.shape[1], 1)), dtype), max(a.shape[1], 1)
    if a.strides[1] != a.itemsize:
        a = np.ascontiguousarray(a)
    return a, a.strides[0] // a.itemsize


# --------------------------------------------------------------------------- bf16
def bf16_to_f64(u: np.ndarray) -> np.ndarray:
    """Decode bf16 bit patterns (uint16) to float64 (exact)."""
    with np.errstate(invalid="ignore"):   # NaN patterns decode to NaN
        return (np.asarray(u, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """Round float64 values to bf16 (nearest, ties to even), returned as uint16 bit patterns."""
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty(x.shape, np.uint16)
    _load().or_double_to_bf16_array(_ptr(x, C.c_double), x.size, _ptr(out, C.c_uint16))
    return out


def bf16_round_scalar(x: float) -> int:
    return int(_load().or_double_to_bf16(float(x)))


# --------------------------------------------------------------------------- steps
def project_rows(K: np.ndarray, P: np.ndarray):
    """Projected scoring cache rows: Kp = bf16(K . P) from the exact product (§3.1, §3.4, §E.1).

    K: uint16 [n, d]; P: float32 [d, r].  Returns (Kp uint16 [n, r], exact float64 [n, r]).
    """
    K, k_ld = _rows(K, np.uint16)
    P = np.ascontiguousarray(P, np.float32)
    d, r = P.shape
    n = K.shape[0] if K.shape[1] == d else 0
    Kp = np.zeros((max(n, 1), r), np.uint16)
    ex = np.zeros((max(n, 1), r), np.float64)
    _load().or_project_rows(_ptr(K, C.c_uint16), k_ld, d, _ptr(P, C.c_float), r, n,
                            _ptr(Kp, C.c_uint16), r, _ptr(ex, C.c_double))
    return Kp[:n], ex[:n]


def e4m3_to_double(c: int) -> float:
    """Value of one FP8 E4M3 code."""
    return _load().or_e4m3_to_double(int(c))


def double_to_e4m3(x: float) -> int:
    """FP8 E4M3 code of x: round to nearest even, saturate to +-448."""
    return int(_load().or_double_to_e4m3(float(x)))


def project_rows_e4m3(K: np.ndarray, P: np.ndarray):
    """FP8 projected scoring cache rows: Kp8 = e4m3(K . P) from the exact product (the paper's
    deployed precision, §A.3 / §E.2).  Returns (Kp8 uint8 [n, r], exact float64 [n, r])."""
    K, k_ld = _rows(K, np.uint16)
    P = np.ascontiguousarray(P, np.float32)
    d, r = P.shape
    n = K.shape[0] if K.shape[1] == d else 0
    Kp = np.zeros((max(n, 1), r), np.uint8)
    ex = np.zeros((max(n, 1), r), np.float64)
    _load().or_project_rows_e4m3(_ptr(K, C.c_uint16), k_ld, d, _ptr(P, C.c_float), r, n,
                                 _ptr(Kp, C.c_uint8), r, _ptr(ex, C.c_double))
    return Kp[:n], ex[:n]


def scores_e4m3(qs: np.ndarray, Kp8: np.ndarray) -> np.ndarray:
    """fp64 scores against an FP8 projected cache: s_t = qs . value(Kp8_t)."""
    qs = np.ascontiguousarray(qs, np.float64)
    Kp8 = np.ascontiguousarray(Kp8, np.uint8)
    n, r = Kp8.shape
    s = np.zeros(max(n, 1), np.float64)
    _load().or_scores_e4m3(_ptr(qs, C.c_double), r, _ptr(Kp8, C.c_uint8), r, n, _ptr(s, C.c_double))
    return s[:n]


def query_proj(Qg: np.ndarray, P: np.ndarray) -> np.ndarray:
    """Projected group query qs = sum_g P^T q_g (Figure 1, §3.2).  Qg: uint16 [G, d]."""
    Qg = np.ascontiguousarray(Qg, np.uint16)
    P = np.ascontiguousarray(P, np.float32)
    G, d = Qg.shape
    r = P.shape[1]
    qs = np.zeros(r, np.float64)
    _load().or_query_proj(_ptr(Qg, C.c_uint16), G, d, _ptr(P, C.c_float), r, _ptr(qs, C.c_double))
    return qs


def scores(qs: np.ndarray, Kp: np.ndarray) -> np.ndarray:
    """Subspace scores s_t = qs . Kp_t for every row of Kp (uint16 [n, r])."""
    qs = np.ascontiguousarray(qs, np.float64)
    Kp, kp_ld = _rows(Kp, np.uint16)
    n = Kp.shape[0] if Kp.shape[1] == qs.shape[0] else 0
    s = np.zeros(max(n, 1), np.float64)
    _load().or_scores(_ptr(qs, C.c_double), qs.shape[0], _ptr(Kp, C.c_uint16), kp_ld, n,
                      _ptr(s, C.c_double))
    return s[:n]


def topk(s: np.ndarray, k: int):
    """Exact top-k by a full sort (score desc, index asc).  Returns (idx int32 [k], k_eff)."""
    s = np.ascontiguousarray(s, np.float64)
    idx = np.full(max(k, 1), -1, np.int32)
    k_eff = _load().or_topk(_ptr(s, C.c_double) if s.size else None, s.size, k, _ptr(idx, C.c_int32))
    return idx[:k], int(k_eff)


def attention(Qg: np.ndarray, K: np.ndarray, V: np.ndarray, tokens, scale: float):
    """Softmax attention of G heads over the listed tokens (§3.3).

    Qg uint16 [G, dk]; K uint16 [T, dk]; V uint16 [T, dv] (rows may be strided views).
    Returns (O float64 [G, dv], lse float64 [G]).
    """
    Qg = np.ascontiguousarray(Qg, np.uint16)
    K, k_ld = _rows(K, np.uint16)
    V, v_ld = _rows(V, np.uint16)
    tok = np.ascontiguousarray(np.asarray(tokens, np.int64).reshape(-1))
    G, dk = Qg.shape
    dv = V.shape[1]
    O = np.zeros((G, dv), np.float64)
    lse = np.zeros(G, np.float64)
    tp = _ptr(tok, C.c_int64) if tok.size else None
    _load().or_attention(_ptr(Qg, C.c_uint16), G, dk, _ptr(K, C.c_uint16), k_ld,
                         _ptr(V, C.c_uint16), v_ld, dv, tp, tok.size, float(scale),
                         _ptr(O, C.c_double), _ptr(lse, C.c_double))
    return O, lse


def decode_head(Qg, K, V, Kp, P, T: int, k: int, W: int, scale: float):
    """One decode step for one (sequence, KV head) problem (Figure 1).

    Candidates are [0, T-W); the attended list is the selection plus the window [T-W, T).
    Returns dict(idx int32 [k], k_eff, O [G, dv], lse [G], scores float64 [T-W]).
    """
    Qg = np.ascontiguousarray(Qg, np.uint16)
    K, k_ld = _rows(K, np.uint16)
    V, v_ld = _rows(V, np.uint16)
    Kp, kp_ld = _rows(Kp, np.uint16)
    P = np.ascontiguousarray(P, np.float32)
    G, dk = Qg.shape
    dv = V.shape[1]
    r = P.shape[1]
    Wc = min(max(W, 0), T)
    idx = np.full(max(k, 1), -1, np.int32)
    O = np.zeros((G, dv), np.float64)
    lse = np.zeros(G, np.float64)
    s = np.zeros(max(T - Wc, 1), np.float64)
    k_eff = _load().or_decode_head(_ptr(Qg, C.c_uint16), G, dk, dv, _ptr(K, C.c_uint16), k_ld,
                                   _ptr(V, C.c_uint16), v_ld, _ptr(Kp, C.c_uint16), kp_ld,
                                   _ptr(P, C.c_float), r, T, k, W, float(scale),
                                   _ptr(idx, C.c_int32), _ptr(O, C.c_double),
                                   _ptr(lse, C.c_double), _ptr(s, C.c_double))
    if k_eff < 0:
        raise ValueError("rank too large for the oracle")
    return dict(idx=idx[:k], k_eff=int(k_eff), O=O, lse=lse, scores=s[:T - Wc])


def decode_head_e4m3(Qg, K, V, Kp8, P, T: int, k: int, W: int, scale: float):
    """One decode step for one (sequence, KV head) problem over an FP8 E4M3 projected cache
    (§A.3, §E.2: only the scoring cache is FP8; attention reads the bf16 rows).  The steps of
    Figure 1 in order: projected group query, scores against the decoded codes, exact top-k,
    attention over the selection plus the window [T-W, T).  Same return as decode_head."""
    Wc = min(max(W, 0), T)
    n = T - Wc
    s = scores_e4m3(query_proj(Qg, P), np.asarray(Kp8, np.uint8)[:n])
    idx, k_eff = topk(s, k)
    toks = np.concatenate([idx[:k_eff].astype(np.int64), np.arange(n, T, dtype=np.int64)])
    O, lse = attention(Qg, K, V, toks, scale)
    return dict(idx=idx, k_eff=k_eff, O=O, lse=lse, scores=s)
