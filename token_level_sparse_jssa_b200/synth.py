"""Seeded synthetic inputs for the JSSA decode step.

This module only draws random tensors of the right shapes and statistics; it holds
none of the method's arithmetic (no projection, scoring, selection or attention).
The same tensors feed the CUDA path and, in the tests, the CPU oracle.

The workloads stand in for the models and datasets of "Joint Subspace Sparse
Attention for Efficient Long-Context Decoding" (arXiv 2610.19026v1): a GQA layer
shaped like LLaMA-3.1-8B (§4.5 throughput setting, 128K context, budget 2,048), a
hybrid sliding-window/global model (§A.1, §A.3) and an MLA latent cache (§3.3, §A.3).
No checkpoint or dataset is used.

Recipe (per KV head h, per sequence b):
  keys    K = Z . A_h + 0.3 * N(0, 1),   Z ~ N(0, 1) [T, R],  A_h ~ N(0, 1/R) [R, d]
          a set of "heavy" rows (16, or 1 % of T) at distinct uniform positions is scaled x4
  values  V ~ N(0, 1)
  queries q = (z . A_h + 0.3 * N(0, 1)) / sqrt(d) for each query head of the group
  basis   P_h = Q factor of QR(N(0, 1) [d, r]) with the signs fixed so that diag(R) > 0
  MLA     latent C[:, :512] = Z . A + 0.3 N (rank 32), C[:, 512:] ~ N(0, 1) (RoPE part);
          q_h = (z_h . A + 0.3 n) / sqrt(576) on the first 512 dims, N(0, 1) / sqrt(576) on the rest.
All bf16 tensors are drawn in fp32 and rounded by torch's own fp32 -> bf16 cast.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    mode: str            # "gqa" or "mla"
    B: int
    Hq: int
    Hkv: int
    dk: int
    dv: int
    r: int
    T: int
    k: int
    window: int = 0
    R: int = 16          # latent rank of the key generator
    heavy: float = 0.01  # heavy rows per (b, h): a count if >= 1, else a fraction of T
    seed: int = 1000
    layers: int = 1      # hybrid model: total layers (one global, the rest local)
    steps: int = 1       # decode steps in the workload (appending one token per step)
    extra: dict = field(default_factory=dict)

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def sm_scale(self) -> float:
        return 1.0 / math.sqrt(self.dk)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)


# The five workloads: shapes of the pages' settings (seed 1000 + i for workload i).
WORKLOADS = {
    "tiny": Workload("tiny", "gqa", B=1, Hq=8, Hkv=2, dk=128, dv=128, r=16, T=2048, k=128,
                     R=8, heavy=16, seed=1001),
    "llama8b": Workload("llama8b", "gqa", B=8, Hq=32, Hkv=8, dk=128, dv=128, r=32, T=32768,
                        k=2048, R=16, heavy=0.01, seed=1002, steps=1000),
    "h128k": Workload("h128k", "gqa", B=4, Hq=32, Hkv=8, dk=128, dv=128, r=32, T=131072,
                      k=2048, R=16, heavy=0.01, seed=1003),
    "hybrid": Workload("hybrid", "gqa", B=8, Hq=16, Hkv=8, dk=256, dv=256, r=32, T=65536,
                       k=1024, window=1024, R=16, heavy=0.01, seed=1004, layers=6),
    "mla": Workload("mla", "mla", B=16, Hq=128, Hkv=1, dk=576, dv=512, r=64, T=131072,
                    k=2048, R=32, heavy=0, seed=1005),
}


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def orthonormal_basis(d: int, r: int, seed: int) -> torch.Tensor:
    """P = Q of QR(N(0,1) [d, r]) with diag(R) > 0, as fp32 (drawn on the CPU)."""
    g = _gen("cpu", seed)
    X = torch.randn(d, r, generator=g, dtype=torch.float64)
    Qm, Rm = torch.linalg.qr(X)
    sgn = torch.sign(torch.diagonal(Rm))
    sgn[sgn == 0] = 1
    return (Qm * sgn).to(torch.float32)


def make_inputs(w: Workload, device="cpu", T_cap: int | None = None, seq_lens=None,
                seed: int | None = None) -> dict:
    """Draw Q, K, V, P and seq_lens for workload ``w``.

    GQA: K, V [B, Hkv, T_cap, d] bf16; MLA: one latent [B, 1, T_cap, 576] bf16 serving as K,
    with V its first 512 dims (a strided view).  Q [B, Hq, dk] bf16; P [Hkv, dk, r] fp32;
    seq_lens int32 [B] (default: all equal to w.T).  Rows >= seq_len are drawn too, so that
    appended tokens have data.
    """
    seed = w.seed if seed is None else seed
    T_cap = w.T if T_cap is None else T_cap
    g = _gen(device, seed)
    f32 = dict(device=device, dtype=torch.float32)
    B, Hkv, Hq, G = w.B, w.Hkv, w.Hq, w.G
    if w.mode == "mla":
        dl = w.dv                              # latent part (values)
        A = torch.randn(w.R, dl, generator=g, **f32) / math.sqrt(w.R)
        lat = torch.empty(B, 1, T_cap, w.dk, device=device, dtype=torch.bfloat16)
        for b in range(B):
            Z = torch.randn(T_cap, w.R, generator=g, **f32)
            part = Z @ A + 0.3 * torch.randn(T_cap, dl, generator=g, **f32)
            rope = torch.randn(T_cap, w.dk - dl, generator=g, **f32)
            lat[b, 0] = torch.cat([part, rope], dim=1).to(torch.bfloat16)
        zq = torch.randn(B, Hq, w.R, generator=g, **f32)
        qlat = zq @ A + 0.3 * torch.randn(B, Hq, dl, generator=g, **f32)
        qrope = torch.randn(B, Hq, w.dk - dl, generator=g, **f32)
        Q = (torch.cat([qlat, qrope], dim=2) / math.sqrt(w.dk)).to(torch.bfloat16)
        K = lat
        V = lat[..., :w.dv]
    else:
        d = w.dk
        A = torch.randn(Hkv, w.R, d, generator=g, **f32) / math.sqrt(w.R)
        K = torch.empty(B, Hkv, T_cap, d, device=device, dtype=torch.bfloat16)
        n_heavy = int(w.heavy) if w.heavy >= 1 else int(round(w.heavy * w.T))
        n_heavy = min(n_heavy, T_cap)
        for b in range(B):
            for h in range(Hkv):
                Z = torch.randn(T_cap, w.R, generator=g, **f32)
                kk = Z @ A[h] + 0.3 * torch.randn(T_cap, d, generator=g, **f32)
                if n_heavy > 0:
                    pos = torch.randperm(T_cap, generator=g, device=device)[:n_heavy]
                    kk[pos] *= 4.0
                K[b, h] = kk.to(torch.bfloat16)
        V = torch.randn(B, Hkv, T_cap, d, generator=g, **f32).to(torch.bfloat16)
        zq = torch.randn(B, Hq, w.R, generator=g, **f32)
        Ah = A.repeat_interleave(G, dim=0)                      # [Hq, R, d]
        q = torch.einsum("bhr,hrd->bhd", zq, Ah) + 0.3 * torch.randn(B, Hq, d, generator=g, **f32)
        Q = (q / math.sqrt(d)).to(torch.bfloat16)
    Q = Q.contiguous()
    P = torch.stack([orthonormal_basis(w.dk, w.r, seed * 1000 + h) for h in range(Hkv)]).to(device)
    if seq_lens is None:
        seq_lens = [min(w.T, T_cap)] * B
    sl = torch.as_tensor(seq_lens, dtype=torch.int32, device=device)
    return dict(Q=Q, K=K, V=V, P=P, seq_lens=sl, T_cap=T_cap, A=A)


def fresh_queries(w: Workload, n: int, A: torch.Tensor, device="cpu", seed: int = 0) -> torch.Tensor:
    """``n`` further query batches [n, B, Hq, dk] (bf16) drawn with the workload's query
    recipe and latent bases ``A`` (as returned by make_inputs); used to vary the query
    from step to step so that every timed step selects a different token set."""
    g = _gen(device, seed)
    f32 = dict(device=device, dtype=torch.float32)
    B, Hq = w.B, w.Hq
    A = A.to(device)
    if w.mode == "mla":
        dl = w.dv
        zq = torch.randn(n, B, Hq, w.R, generator=g, **f32)
        qlat = zq @ A + 0.3 * torch.randn(n, B, Hq, dl, generator=g, **f32)
        qrope = torch.randn(n, B, Hq, w.dk - dl, generator=g, **f32)
        q = torch.cat([qlat, qrope], dim=3)
    else:
        Ah = A.repeat_interleave(w.G, dim=0)                     # [Hq, R, d]
        zq = torch.randn(n, B, Hq, w.R, generator=g, **f32)
        q = torch.einsum("nbhr,hrd->nbhd", zq, Ah) + 0.3 * torch.randn(n, B, Hq, w.dk, generator=g, **f32)
    return (q / math.sqrt(w.dk)).to(torch.bfloat16).contiguous()


def random_scores(rows: int, n: int, device="cpu", seed: int = 0, ties: int = 0,
                  zeros: int = 0) -> torch.Tensor:
    """fp32 score rows [rows, n]: N(0,1) with a few large values, optional planted exact
    ties (groups of repeated values) and signed zeros."""
    g = _gen("cpu", seed)
    s = torch.randn(rows, n, generator=g, dtype=torch.float32)
    s += 3.0 * (torch.rand(rows, n, generator=g) < 0.02).float() * torch.rand(rows, n, generator=g)
    for i in range(rows):
        for _ in range(ties):
            m = int(torch.randint(2, 9, (1,), generator=g))
            pos = torch.randperm(n, generator=g)[:m]
            s[i, pos] = float(s[i, pos[0]])
        if zeros:
            pos = torch.randperm(n, generator=g)[:zeros]
            s[i, pos] = 0.0
            s[i, pos[: zeros // 2]] = -0.0
    return s.to(device)


def random_index_sets(rows: int, n_cand, k: int, seed: int = 0) -> torch.Tensor:
    """Sorted distinct token indices per row [rows, k] (int32, -1 padded when n_cand < k)."""
    g = _gen("cpu", seed)
    out = torch.full((rows, k), -1, dtype=torch.int32)
    for i in range(rows):
        n = int(n_cand[i]) if hasattr(n_cand, "__len__") else int(n_cand)
        m = min(k, n)
        if m > 0:
            sel = torch.randperm(n, generator=g)[:m].sort().values
            out[i, :m] = sel.to(torch.int32)
    return out
