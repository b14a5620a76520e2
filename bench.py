#!/usr/bin/env python
"""Benchmark of the JSSA decode step on B200 (one JSON line on rank 0).

Workload (default, ``--workload h128k``): the 128K headline GQA layer — B=4, Hq=32,
Hkv=8, d=128, r=32, T=131072 cached tokens, top-k budget k=2048, bf16 K/V/Q, synthetic
caches from the seeded generator (token_level_sparse_jssa_b200.synth).  One step =
project the newest key into the scoring cache, project the group queries, scan all
T projected keys, select the top-k per (sequence, KV head), attend over the selected
rows in place and merge the split partials.  Every timed step uses a fresh query
batch, so every step selects a different token set.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference] [--workload NAME] [--kp bf16|e4m3]

``--kp e4m3`` stores the projected scoring cache in FP8 E4M3 (the paper's deployed
configuration) instead of bf16; the default line also reports the step over an E4M3 cache
as a stage time.

N > 1 runs under torchrun: each rank owns an independent batch of sequences (weak
scaling, no collective on the data path); time is the max over ranks.
``--impl reference`` times the CPU oracle (fp64, single-threaded) on a bounded sample
of the same workload on this host instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode steps/s and µs/step at 128K (1×B200); % of HBM roofline; × vs own dense kernel"
UNIT = "steps/s"
# selection (query and newest-key projection, score scan, top-k) and attention (+ merge in the GQA
# kernel; the MLA path launches its merge separately)
FUSED_MAX_T = 131072  # caches up to this many tokens run projections, scan and top-k in one kernel


def step_kernels(w) -> tuple[int, bool]:
    """Kernels one decode step launches, and whether the attention runs inside the selection
    kernel (GQA with d <= 128 and G <= 16 on caches the selection kernel covers)."""
    if w.T > FUSED_MAX_T:
        return 4, False                                  # prologue, score, top-k, attention
    if w.mode == "mla":
        return 2, False                                  # selection, tensor-core attention (merge inside)
    fused = w.dk <= 128 and w.G <= 16
    return (1 if fused else 2) + (w.layers - 1), fused   # + one dense kernel per local layer


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="jssa", choices=["jssa", "reference"])
    ap.add_argument("--workload", default="h128k")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--kp", default="bf16", choices=["bf16", "e4m3"], help="projected scoring cache type")
    ap.add_argument("--k", type=int, default=0, help="token budget (default: the workload's)")
    ap.add_argument("--T", type=int, default=0,
                    help="cache length (default: the workload's); smaller caches are for profiler captures")
    return ap.parse_args()


# --------------------------------------------------------------------------- helpers
def byte_model(w, T, k, window, out_bytes=2, kp_bytes=2):
    """Algorithmic bytes of one step and of the dense step (HBM roofline numerator);
    kp_bytes = bytes per projected-cache element (2 bf16, 1 E4M3).  A hybrid model's step also
    runs w.layers - 1 local layers: dense attention over their window-sized caches."""
    n = T - min(window, T)
    keff = min(k, n)
    rows = w.B * w.Hkv
    kp = rows * n * w.r * kp_bytes
    kv_row = (w.dk if w.mode == "mla" else w.dk + w.dv) * 2
    sel = rows * (keff + min(window, T)) * kv_row
    qo = w.B * w.Hq * (w.dk * 2 + w.dv * out_bytes)
    dense = rows * T * kv_row + qo
    # the selection kernel: Kp scan, queries, bases, the newest key row in and its Kp row
    # out, indices and counts out (the scores and histograms stay on chip)
    select = (kp + w.B * w.Hq * w.dk * 2 + w.Hkv * w.dk * w.r * 4 + rows * (w.dk * 2 + w.r * kp_bytes)
              + rows * (k * 4 + 4))
    local = (w.layers - 1) * (rows * min(window, T) * kv_row + qo)
    return dict(kp=kp, selected=sel, qo=qo, step=kp + sel + qo + local, dense=dense + local, scores=rows * n * 4,
                select=select, local=local)


def tensor_peak():
    """Measured sustained dense bf16 tensor throughput (TFLOP/s), for kernels timed in long loops."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return d["bf16_tflops_sustained"], "measured"
    except Exception:
        return 1400.0, "fallback"


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return d["hbm_gbs"], "measured"
    except Exception:
        return 6650.0, "fallback"


def source_hash(*names):
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "token_level_sparse_jssa_b200", "csrc", n), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, workload: str, src_hash: str):
    """DRAM bytes per launch from a committed ncu summary, if taken on the current source."""
    p = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        d = json.load(open(p))
        e = d[kernel][workload]
        return e["bytes_per_launch"] if e.get("source_hash") == src_hash else None
    except Exception:
        return None


class ClockSampler:
    """Samples SM clock and throttle reasons with NVML while the timed region runs."""

    def __init__(self, dev_index: int, period=0.01):
        self.period, self.samples, self.reasons = period, [], set()
        self.max_mhz = None
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml as nv
            nv.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(dev_index).uuid)
            uuid = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
            self.h = nv.nvmlDeviceGetHandleByUUID(uuid.encode())
            self.nv = nv
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.h, nv.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover
            self.err = repr(e)

    def _run(self):
        nv = self.nv
        names = {
            "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4, "hw_slowdown": 0x8,
            "sync_boost": 0x10, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
            "hw_power_brake_slowdown": 0x80, "display_clock_setting": 0x100,
        }
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for k, bit in names.items():
                    if r & bit and k != "gpu_idle":
                        self.reasons.add(k)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# --------------------------------------------------------------------------- workload setup
class Setup:
    def __init__(self, w, device, seed_offset=0, kp="bf16"):
        import token_level_sparse_jssa_b200 as jssa
        from token_level_sparse_jssa_b200 import synth
        self.jssa, self.w = jssa, w
        x = synth.make_inputs(w, device=device, seed=w.seed + seed_offset)
        self.T_cap = x["T_cap"]
        self.K = x["K"]
        self.V = self.K[..., : w.dv] if w.mode == "mla" else x["V"]
        self.P = x["P"].contiguous()
        self.seq_lens = x["seq_lens"]
        self.A = x["A"]
        self.T_cap = x["T_cap"]
        # an appending workload (w.steps > 1 decode steps): the cache starts with T - steps
        # tokens; step i writes token T - steps + i (its K/V row, kept aside here as the stream
        # of generated rows) with jssa_append_kv, projects it on write (n_new = 1) and attends
        # over the lengthened sequence; the loop wraps after w.steps steps
        self.appending = w.steps > 1
        if self.appending:
            S, t0 = w.steps, w.T - w.steps
            self.Knew = self.K[:, :, t0:w.T].permute(2, 0, 1, 3).contiguous()
            self.Vnew = self.V[:, :, t0:w.T].permute(2, 0, 1, 3).contiguous() if w.mode != "mla" else None
            ar = torch.arange(S, device=device, dtype=torch.int32)
            self.SL = (t0 + 1 + ar).view(S, 1).repeat(1, w.B).contiguous()   # [S, B] lengths at step i
            self.POS = (self.SL - 1).contiguous()                              # [S, B] the row step i writes
        self.Kp, self.L = self.scoring_cache(kp)
        self.kp = kp
        self.ws = jssa.alloc_workspace(self.L, w.k, w.window)
        self.gbuf = jssa.alloc_gather_buffer(self.L, w.k, w.window) if w.mode != "mla" else None
        self.O = torch.empty(w.B, w.Hq, w.dv, dtype=torch.bfloat16, device=device)
        self.idx = torch.empty(w.B, w.Hkv, w.k, dtype=torch.int32, device=device)
        self.nsel = torch.empty(w.B, w.Hkv, dtype=torch.int32, device=device)
        # a hybrid model's local layers: each keeps a cache of its window of W tokens only
        self.local = []
        if w.layers > 1:
            g = torch.Generator(device=device)
            g.manual_seed(w.seed * 7 + seed_offset)
            W = w.window
            for _ in range(w.layers - 1):
                Kl = torch.randn(w.B, w.Hkv, W, w.dk, generator=g, device=device).to(torch.bfloat16)
                Vl = torch.randn(w.B, w.Hkv, W, w.dv, generator=g, device=device).to(torch.bfloat16)
                Kpl = torch.empty(w.B, w.Hkv, W, w.r, dtype=torch.bfloat16, device=device)   # unused by dense layers
                Ll = jssa.make_layout(Kl, Vl, Kpl, w.Hq, w.r, jssa.MODE_GQA, jssa.OUT_BF16)
                self.local.append((Kl, Vl, Ll))
            self.local_lens = torch.full((w.B,), W, dtype=torch.int32, device=device)
            self.local_ws = jssa.alloc_workspace(self.local[0][2], 1, 0)
        torch.cuda.synchronize()

    def local_layers(self, Q):
        for (Kl, Vl, Ll) in self.local:
            self.jssa.dense_decode(Ll, Q, Kl, Vl, self.local_lens, 0, self.w.sm_scale, self.O, None, self.local_ws)

    def scoring_cache(self, kp):
        """A projected scoring cache of this workload (bf16 or E4M3) filled from K, and its layout."""
        jssa, w = self.jssa, self.w
        Kp = torch.empty(w.B, w.Hkv, self.T_cap, w.r, dtype=torch.uint8 if kp == "e4m3" else torch.bfloat16,
                         device=self.K.device)
        L = jssa.make_layout(self.K, self.V, Kp, w.Hq, w.r, jssa.MODE_MLA if w.mode == "mla" else jssa.MODE_GQA,
                             jssa.OUT_BF16)
        tb = torch.zeros(w.B, dtype=torch.int32, device=self.K.device)
        filled = self.T_cap - (w.steps if self.appending else 0)
        jssa.project_keys(L, self.K, self.P, Kp, filled, t_begin=tb)   # prefill fill
        if filled < self.T_cap:
            Kp[:, :, filled:].zero_()   # rows the appending steps write
        return Kp, L

    def step(self, Q, i=0, Kp=None, L=None, kv_new=None):
        """Decode step i with query Q.  Appending workloads first write the step's token (from
        kv_new, else from the stream of generated rows) with jssa_append_kv; every step projects
        the newest key on write (n_new = 1)."""
        w = self.w
        L = self.L if L is None else L
        if self.appending:
            j = i % w.steps
            kn, vn = kv_new if kv_new is not None else (self.Knew[j], self.Vnew[j] if self.Vnew is not None else None)
            self.jssa.append_kv(L, kn, vn, self.K, self.V if vn is not None else None, self.POS[j])
            sl = self.SL[j]
        else:
            sl = self.seq_lens
        self.jssa.decode_step(L, Q, self.K, self.V, self.Kp if Kp is None else Kp, self.P,
                              sl, 1, w.k, w.window, w.sm_scale, self.O, None, self.idx, self.nsel, self.ws)
        self.local_layers(Q)

    def dense(self, Q):
        # an appending workload's comparator runs at the loop's mean length
        sl = self.SL[self.w.steps // 2] if self.appending else self.seq_lens
        self.jssa.dense_decode(self.L, Q, self.K, self.V, sl, 0, self.w.sm_scale, self.O, None, self.ws)
        self.local_layers(Q)


def graph_of(fn, qs):
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for q in qs:
                fn(q)
    torch.cuda.current_stream().wait_stream(s)
    return g


def timed_graph(g, barrier):
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    g.replay()
    e1.record()
    torch.cuda.synchronize()
    barrier()
    return e0.elapsed_time(e1)


def stage_times(st, Q, reps=50):
    """Device time of the public entry points that make up the step, each replayed from a
    CUDA graph of `reps` calls (CUDA events on the replay stream).  select = the selection
    half of the step (projections, score scan, top-k: one kernel when the cache fits a
    cluster); attention = indexed attention with its merge; dense = the full-KV comparator;
    gather_then_attend = the same attention done the gather-based way (copy, then dense);
    step_other_kp = the whole step over the other scoring-cache type (E4M3 when the run is bf16);
    vote_select = the head-shared soft-voting selection; local_layers = a hybrid model's local
    layers of one step."""
    jssa, w = st.jssa, st.w
    calls = {
        "select_us": lambda: jssa.select(st.L, Q, st.K, st.Kp, st.P, st.seq_lens, 1, w.k, w.window, st.idx,
                                         st.nsel, st.ws),
        "attention_us": lambda: jssa.indexed_attn(st.L, Q, st.K, st.V, st.idx, w.k, st.nsel, st.seq_lens,
                                                  w.window, w.sm_scale, st.O, None, st.ws),
        # the head-shared soft-voting variant of the selection (unfused kernels)
        "vote_select_us": lambda: jssa.vote_select(st.L, Q, st.K, st.Kp, st.P, st.seq_lens, 1, w.k, w.window,
                                                   w.sm_scale, st.idx, st.nsel, st.ws),
    }
    calls["dense_us"] = lambda: st.dense(Q)
    if st.local:  # a hybrid model's local layers (dense over their own window caches, together > L2)
        calls["local_layers_us"] = lambda: st.local_layers(Q)
    if st.w.mode != "mla":  # (the gather-based comparator is GQA only)
        # the gather-based baseline of the pages: copy the attended rows, then dense decode on them
        calls["gather_then_attend_us"] = lambda: jssa.gather_decode(st.L, Q, st.K, st.V, st.idx, w.k, st.nsel,
                                                                    st.seq_lens, w.window, w.sm_scale, st.O, None,
                                                                    st.gbuf, st.ws)
    other = "bf16" if st.kp == "e4m3" else "e4m3"
    Kp2, L2 = st.scoring_cache(other)
    calls[f"step_kp_{other}_us"] = lambda: st.step(Q, 0, Kp2, L2)
    out = {}
    for name, fn in calls.items():
        fn()
        torch.cuda.synchronize()
        g = graph_of(lambda _q: fn(), [None] * reps)
        g.replay()
        torch.cuda.synchronize()
        out[name] = timed_graph(g, lambda: None) * 1000.0 / reps
        del g
    del Kp2
    return out


# --------------------------------------------------------------------------- basis calibration
def calibration_leg(st, reps=3):
    """Offline calibration of the basis (jssa_calibrate) on calibration queries drawn with the
    workload's recipe at n positions of every sequence, timed with CUDA events (best of
    `reps`), and the selection quality it buys: the fraction of the exact full-dimensional
    top-k (group-mean query . key over all candidates) that the selection contains, with the
    calibrated basis and with the workload's random orthonormal basis, on two fresh queries."""
    from token_level_sparse_jssa_b200 import synth
    jssa, w = st.jssa, st.w
    n = min(w.T, 32768) if w.mode != "mla" else 1024
    Qc = synth.fresh_queries(w, n, st.A, device="cuda", seed=99).permute(1, 2, 0, 3).contiguous()
    P = torch.empty_like(st.P)
    ws = jssa.alloc_calibration_workspace(st.L)
    jssa.calibrate(st.L, Qc, st.K, n, P, ws)
    torch.cuda.synchronize()
    best = float("inf")
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        jssa.calibrate(st.L, Qc, st.K, n, P, ws)
        e1.record()
        torch.cuda.synchronize()
        best = min(best, e0.elapsed_time(e1))
    code, _ = jssa.read_device_status(ws)
    del Qc, ws
    Qs = synth.fresh_queries(w, 2, st.A, device="cuda", seed=98)
    rec = {}
    for name, basis in (("calibrated", P), ("random", st.P)):
        Kp = torch.empty(w.B, w.Hkv, st.T_cap, w.r, dtype=torch.bfloat16, device="cuda")
        L = jssa.make_layout(st.K, st.V, Kp, w.Hq, w.r, jssa.MODE_MLA if w.mode == "mla" else jssa.MODE_GQA,
                             jssa.OUT_BF16)
        jssa.project_keys(L, st.K, basis, Kp, st.T_cap, t_begin=torch.zeros(w.B, dtype=torch.int32, device="cuda"))
        got = []
        for Q in Qs:
            jssa.select(L, Q, st.K, Kp, basis, st.seq_lens, 0, w.k, w.window, st.idx, st.nsel, st.ws)
            n_cand = w.T - min(w.window, w.T)
            qbar = Q.float().view(w.B, w.Hkv, w.G, w.dk).mean(2)
            s = torch.einsum("bhd,bhtd->bht", qbar, st.K[:, :, :n_cand].float())
            truth = torch.topk(s, min(w.k, n_cand), dim=2).indices
            sel = torch.zeros_like(s, dtype=torch.bool).scatter_(2, st.idx.long().clamp(min=0), True)
            got.append(sel.gather(2, truth).float().mean().item())
            del s, sel
        rec[name] = sum(got) / len(got)
        del Kp
    return {"calibration_ms": best, "calibration_tokens_per_head": w.B * n, "status": code,
            "recall_at_k": rec}


# --------------------------------------------------------------------------- CPU oracle timing
def cpu_oracle_rate(w, seconds: float, data=None, kp="bf16"):
    """Time the fp64 oracle's decode step on sampled (sequence, KV head) rows of the workload
    on this host (single thread) for about ``seconds``; returns (steps/s, description)."""
    import numpy as np
    import oracle
    from token_level_sparse_jssa_b200 import synth
    from tests._util import u16, f32
    if data is None:
        # a bounded sample of the workload: sequence 0 only (its Hkv rows)
        x = synth.make_inputs(w.with_(B=1), device="cuda" if torch.cuda.is_available() else "cpu")
        K, V, Q, P = x["K"], (x["K"][..., : w.dv] if w.mode == "mla" else x["V"]), x["Q"], x["P"]
    else:
        K, V, Q, P = data
    rows = [(0, h) for h in range(min(2, w.Hkv))]
    proj = oracle.project_rows_e4m3 if kp == "e4m3" else oracle.project_rows
    head = oracle.decode_head_e4m3 if kp == "e4m3" else oracle.decode_head
    G, T = w.G, w.T
    host = []
    for (b, h) in rows:
        Kh, Vh = u16(K[b, h, :T]), u16(V[b, h, :T])
        Ph = f32(P[h])
        Kp, _ = proj(Kh, Ph)                      # cache state before the step (not timed)
        host.append((u16(Q[b, h * G:(h + 1) * G]), Kh, Vh, Kp, Ph))
    n, t0 = 0, time.perf_counter()
    while True:
        for (Qg, Kh, Vh, Kp, Ph) in host:
            proj(Kh[T - 1:T], Ph)                 # the newest key, projected on write
            head(Qg, Kh, Vh, Kp, Ph, T, w.k, w.window, w.sm_scale)
            for _ in range(w.layers - 1):         # local layers: dense over a window-sized cache
                oracle.attention(Qg, Kh[T - w.window:T], Vh[T - w.window:T], np.arange(w.window), w.sm_scale)
            n += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    per_row = el / n
    step_s = per_row * w.B * w.Hkv
    desc = (f"{n} (sequence, KV-head) problems of the {w.name} step ({len(rows)} distinct rows of sequence 0, "
            f"T={T}, k={w.k}) in {el:.1f} s on 1 thread; one step = {w.B * w.Hkv} such problems")
    return 1.0 / step_s, desc


def host_cpu() -> dict:
    """The host the CPU baseline runs on: its logical CPU count and model name."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"host_cpus": os.cpu_count(), "cpu_model": model}


# --------------------------------------------------------------------------- ranks
def rank_env():
    """(rank, world, local_rank) from the launcher's environment (1 process when absent)."""
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(x: float, dist=None, device="cuda") -> float:
    """The maximum of a per-rank scalar over all ranks (identity without a process group)."""
    if dist is None:
        return float(x)
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, steps: int, ms: float) -> float:
    """Steps per second of the whole job: every rank ran `steps` steps of its own batch and
    the slowest rank took `ms` milliseconds."""
    return world * steps / (ms / 1000.0)


# --------------------------------------------------------------------------- arms
def run_reference(args, w, cfg):
    rank, _, _ = rank_env()
    if rank != 0:
        return 0
    rate, desc = cpu_oracle_rate(w, max(0.2, args.cpu_seconds), kp=args.kp)
    line = {"impl": "reference", "metric": METRIC, "value": rate, "unit": UNIT, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 / rate, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
            "cpu_baseline": {"value": rate, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": desc,
                             **host_cpu()},
            "e2e": {"value": rate, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse()
    from token_level_sparse_jssa_b200 import synth
    w = synth.WORKLOADS[args.workload]
    if args.k > 0:
        w = w.with_(k=args.k)
    if args.T > 0:
        w = w.with_(T=args.T)
    rank, world, local = rank_env()
    # an appending workload's sequences grow from T - steps + 1 to T over its loop: bytes at the mean length
    T_bytes = w.T - w.steps // 2 if w.steps > 1 else w.T
    bm = byte_model(w, T_bytes, w.k, w.window, kp_bytes=1 if args.kp == "e4m3" else 2)
    cfg = {"workload": f"{w.name}: B={w.B} Hq={w.Hq} Hkv={w.Hkv} d_k={w.dk} d_v={w.dv} r={w.r} T={w.T} k={w.k}"
                       + (f" W={w.window}" if w.window else "") + f" ({w.mode.upper()})"
                       + (f"; {w.layers} layers: 1 global (sparse), {w.layers - 1} local (dense over the "
                          f"{w.window}-token window caches)" if w.layers > 1 else "")
                       + (f"; appending: each step writes one token (jssa_append_kv) and projects it on write, "
                          f"the sequences growing from T={w.T - w.steps + 1} to T={w.T} over a {w.steps}-step loop"
                          if w.steps > 1 else ""),
           "global_batch": w.B * max(world, args.gpus), "seq_len": w.T, "k": w.k, "r": w.r,
           "parallelism": f"dp{max(world, args.gpus)} (independent sequences per rank, no collective)",
           "kp": "FP8 E4M3 (unit scale)" if args.kp == "e4m3" else "bf16",
           "l2": "inputs larger than L2 (the projected cache alone is %.0f MB per step) and a fresh query every step"
                 % (bm["kp"] / 1e6)}
    if args.impl == "reference":
        return run_reference(args, w, cfg)

    if not torch.cuda.is_available():
        print(json.dumps({"error": "no CUDA device"}))
        return 1
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=torch.device("cuda", local))

    def barrier():
        if dist is not None:
            dist.barrier()

    st = Setup(w, "cuda", seed_offset=rank, kp=args.kp)
    nq = args.warmup + args.steps
    Qs = synth.fresh_queries(w, nq, st.A, device="cuda", seed=7 + rank)
    # warm-up (untimed), then exactly `steps` timed steps, each in one CUDA graph
    run = lambda it: st.step(it[1], it[0])   # (step index, query)
    g_warm = graph_of(run, [(i, Qs[i]) for i in range(args.warmup)])
    g_warm.replay()
    torch.cuda.synchronize()
    g_timed = graph_of(run, [(args.warmup + i, Qs[args.warmup + i]) for i in range(args.steps)])
    g_timed.replay()   # the graph's first launch uploads it to the device: keep that out of the timing
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        ms = timed_graph(g_timed, barrier)
    ms = max_over_ranks(ms, dist)
    ms_step = ms / args.steps
    value = whole_job_rate(world, args.steps, ms)
    del g_warm, g_timed

    # spread of the step time: 10 replays of a 50-step graph (fresh queries), per-replay means
    g_spread = graph_of(run, [(args.warmup + i, Qs[(args.warmup + i) % nq]) for i in range(50)])
    g_spread.replay()
    torch.cuda.synchronize()
    spread = sorted(max_over_ranks(timed_graph(g_spread, barrier), dist) * 1000.0 / 50 for _ in range(10))
    del g_spread

    # dense full-KV comparator at the same shape (the latent model's runs on the tensor cores)
    dense_ms = None
    if True:
        nd = max(5, min(200 if w.mode != "mla" else 20, args.steps // 10))
        g_dw = graph_of(st.dense, [Qs[i] for i in range(3)])
        g_dw.replay()
        g_d = graph_of(st.dense, [Qs[i % nq] for i in range(nd)])
        dense_ms = max_over_ranks(timed_graph(g_d, barrier) / nd, dist)
        del g_dw, g_d

    stages = stage_times(st, Qs[0])
    calib = calibration_leg(st)
    hbm, peak_kind = peaks()
    n_kernels, fused = step_kernels(w)
    sel_bytes = bm["step"] if fused else bm["select"]
    sel_s = stages["select_us"] * 1e-6
    shash = source_hash("select_kernel.cuh", "attn_core.cuh", "common.cuh")

    # end to end through the public API with host buffers.  Per step: ONE host-to-device copy
    # of a packed pinned buffer [query | newest K rows | newest V rows] into a device staging
    # buffer, the append-on-write call that writes the newest rows into every layer's cache
    # (jssa_append_kv), the decode step reading its query from the staging buffer, and ONE
    # device-to-host copy of the output.  Both copies are jssa_copy_mapped: a kernel that
    # reads (writes) the pinned host buffer over the host link, which for the few tens of KB
    # of a step avoids the copy engine's per-transfer latency.
    ne = max(10, min(500, args.steps // 4))
    jssa = st.jssa
    nq, nk = w.B * w.Hq * w.dk, w.B * w.Hkv * w.dk
    nv = w.B * w.Hkv * w.dv if w.mode != "mla" else 0
    stage_h = torch.empty(ne, nq + nk + nv, dtype=torch.bfloat16).pin_memory()
    stage_h[:, :nq] = Qs[:ne].reshape(ne, nq).cpu()
    stage_h[:, nq:nq + nk] = st.K[:, :, w.T - 1].reshape(1, nk).cpu()
    if nv:
        stage_h[:, nq + nk:] = st.V[:, :, w.T - 1].reshape(1, nv).cpu()
    stage_d = torch.empty(nq + nk + nv, dtype=torch.bfloat16, device="cuda")
    Qd = stage_d[:nq].view(w.B, w.Hq, w.dk)
    Kn = stage_d[nq:nq + nk].view(w.B, w.Hkv, w.dk)
    Vn = stage_d[nq + nk:].view(w.B, w.Hkv, w.dv) if nv else None
    pos = (st.seq_lens - 1).to(torch.int32)
    local_pos = torch.full((w.B,), w.window - 1, dtype=torch.int32, device="cuda") if st.local else None
    Oh_all = torch.empty((ne,) + tuple(st.O.shape), dtype=st.O.dtype).pin_memory()

    def e2e_step(i):
        jssa.copy_mapped(stage_d, stage_h[i])
        if not st.appending:   # (an appending workload's step appends from the staging buffer itself)
            jssa.append_kv(st.L, Kn, Vn, st.K, st.V if nv else None, pos)
        for (Kl, Vl, Ll) in st.local:   # the local layers' caches take the same newest rows
            jssa.append_kv(Ll, Kn, Vn, Kl, Vl, local_pos)
        st.step(Qd, i, kv_new=(Kn, Vn))
        jssa.copy_mapped(Oh_all[i], st.O)

    for i in range(3):
        e2e_step(i)
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(ne):
        e2e_step(i)
    e1.record()
    torch.cuda.synchronize()
    barrier()
    e2e_eager_ms = max_over_ranks(e0.elapsed_time(e1), dist)
    # the same loop as a decode server would run it: the ne steps' copies and calls captured in
    # one CUDA graph (the entry points are capturable), replayed once untimed, then timed
    g_e2e = graph_of(e2e_step, list(range(ne)))
    g_e2e.replay()
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(timed_graph(g_e2e, barrier), dist)
    del g_e2e
    h2d = (nq + nk + nv) * 2
    d2h = st.O.numel() * st.O.element_size()

    code, flags = st.jssa.read_device_status(st.ws)
    if rank == 0:
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            rate, desc = cpu_oracle_rate(w, args.cpu_seconds, data=(st.K, st.V, Qs[0], st.P), kp=args.kp)
            cpu = {"value": rate, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": desc, **host_cpu()}
        # the dominant kernel: with the attention inside, the step is that one kernel and its
        # launch time is the step time measured above; otherwise the selection kernel alone
        achieved = sel_bytes / (ms_step * 1e-3 if fused else sel_s) / 1e9
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg,
            "us_per_step": ms_step * 1000.0, "tokens_per_s": value * w.B,
            "us_per_step_spread": {"p10": spread[1], "p50": spread[5], "p90": spread[8],
                                   "of": "10 replays of a 50-step graph, mean step time of each"},
            "bytes_per_step": bm["step"], "effective_GBps": bm["step"] / (ms_step * 1e-3) / 1e9,
            "step_hbm_frac": bm["step"] / (ms_step * 1e-3) / 1e9 / hbm,
            "dense_us_per_step": dense_ms * 1000.0 if dense_ms else None,
            "speedup_vs_dense": dense_ms / ms_step if dense_ms else None,
            "byte_ratio": bm["dense"] / bm["step"],
            "dense_hbm_frac": bm["dense"] / (dense_ms * 1e-3) / 1e9 / hbm if dense_ms else None,
            # the latent model's dense step is a contraction (2 B Hq T (d_k + d_v) flops): its fraction
            # of the measured sustained bf16 tensor peak
            "dense_tensor_frac": (2.0 * w.B * w.Hq * w.T * (w.dk + w.dv) / (dense_ms * 1e-3) / 1e12 /
                                  tensor_peak()[0]) if (dense_ms and w.mode == "mla") else None,
            "stage_us": stages,
            "calibration": calib,
            "roofline": {"kernel": ("select_kernel (the whole step: query and newest-key projection, score scan, "
                                    "top-k, attention, merge)") if fused else
                                   "select_kernel (query and newest-key projection, score scan, top-k)",
                         "bound": "hbm", "achieved": achieved, "peak": hbm,
                         "unit": "GB/s", "frac": achieved / hbm, "peak_kind": peak_kind,
                         "frac_of_nominal_8000_GBps": achieved / 8000.0,
                         "traffic": traffic_for("select_kernel", w.name + ("-e4m3" if args.kp == "e4m3" else ""),
                                                shash),
                         "algorithmic_bytes_per_launch": sel_bytes},
            "cpu_baseline": cpu,
            "e2e": {"value": whole_job_rate(world, ne, e2e_ms), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": ne,
                    "mode": "per step: one H2D copy of a packed pinned buffer (query, newest K and V rows), "
                            "jssa_append_kv into every layer's cache, the decode_step call, one D2H copy of the "
                            "output; both copies by jssa_copy_mapped (a kernel reading / writing the pinned "
                            "host buffer); the steps captured in one CUDA graph"},
            "e2e_eager": {"value": whole_job_rate(world, ne, e2e_eager_ms), "unit": UNIT,
                          "mode": "the same loop issued call by call from Python"},
            "gpu_launches": n_kernels * args.steps,
            "clocks": clk.summary(),
            "device_status": flags,
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
