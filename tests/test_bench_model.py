"""The benchmark's algorithmic byte model (the roofline numerator) against byte counts worked
out by hand from the workloads' shapes: Kp rows read once, the attended K/V rows read once
(the latent row once for MLA), Q in and O out; the dense step reads every K/V row."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _model(name, **kw):
    import bench
    from token_level_sparse_jssa_b200 import synth
    w = synth.WORKLOADS[name].with_(**kw)
    return w, bench.byte_model(w, w.T, w.k, w.window)


def test_headline_step_bytes():
    w, bm = _model("h128k")
    kp = 4 * 8 * 131072 * 32 * 2                     # B Hkv T r, bf16
    kv = 4 * 8 * 2048 * (128 + 128) * 2              # selected K and V rows
    qo = 4 * 32 * (128 * 2 + 128 * 2)                # Q in, bf16 O out
    assert bm["step"] == kp + kv + qo == 302_055_424
    assert bm["dense"] == 4 * 8 * 131072 * 256 * 2 + qo == 2_147_549_184


@pytest.mark.parametrize("k,total", [(512, 276_889_600), (1024, 285_278_208), (4096, 335_609_856)])
def test_budget_sweep_bytes(k, total):
    _, bm = _model("h128k", k=k)
    assert bm["step"] == total


def test_e4m3_cache_halves_the_scoring_bytes():
    import bench
    from token_level_sparse_jssa_b200 import synth
    w = synth.WORKLOADS["h128k"]
    b16 = bench.byte_model(w, w.T, w.k, w.window, kp_bytes=2)
    b8 = bench.byte_model(w, w.T, w.k, w.window, kp_bytes=1)
    assert b16["kp"] == 2 * b8["kp"] and b16["step"] - b8["step"] == b8["kp"] == 134_217_728


def test_hybrid_model_step_has_one_global_and_five_local_layers():
    w, bm = _model("hybrid")
    rows, W, kv_row = 8 * 8, 1024, (256 + 256) * 2
    qo = 8 * 16 * (256 * 2 + 256 * 2)
    glob = rows * (65536 - W) * 32 * 2 + rows * (1024 + W) * kv_row + qo
    local = 5 * (rows * W * kv_row + qo)
    assert bm["step"] == glob + local == 734_789_632
    assert bm["dense"] == rows * 65536 * kv_row + qo + local


def test_mla_counts_the_latent_row_once():
    w, bm = _model("mla")
    kp = 16 * 131072 * 64 * 2
    lat = 16 * 2048 * 576 * 2                        # V is the first 512 dims of the same row
    qo = 16 * 128 * (576 * 2 + 512 * 2)
    assert bm["step"] == kp + lat + qo == 310_640_640
