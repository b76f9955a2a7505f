"""Host-side pieces of bench.py that the JSON line depends on, checked on the CPU: the whole-job
rate, the workload description, and the rule that reports the captured DRAM traffic only while
the GEMM sources still match the ones it was captured on."""
import hashlib
import json
import math
import os

import numpy as np

import pytest

import bench
import synth


def test_aggregate_rate_counts_every_rank():
    assert bench.aggregate_rate(1, 4096, 10, 20.0) == pytest.approx(4096 * 10 / 0.020)
    assert bench.aggregate_rate(8, 4096, 10, 20.0) == pytest.approx(8 * 4096 * 10 / 0.020)


def test_max_over_ranks_single_process():
    assert bench.max_over_ranks(3.5, 1) == 3.5


def test_workload_config_names_the_shape():
    w = bench.workload_config(synth.CONFIGS["mixtral"])
    for part in ("T=4096", "H=4096", "E=8", "k=2", "F=14336", "dropless", "GELU"):
        assert part in w
    assert "CF=1.25" in bench.workload_config(synth.CONFIGS["switch"])


def test_alg_flops_and_bytes_of_the_headline_workload():
    cfg = synth.CONFIGS["mixtral"]
    kept = cfg.T * cfg.k
    assert bench.alg_flops(cfg, kept) == pytest.approx(4.0 * cfg.H * cfg.F * kept + 2.0 * cfg.T * cfg.H * cfg.E)
    # every expert's W1 and W2 (bf16) dominate the algorithmic bytes
    assert bench.alg_bytes(cfg, cfg.E) > 2 * cfg.E * cfg.H * cfg.F * 2


def test_captured_traffic_follows_the_source_hashes(tmp_path, monkeypatch):
    src = tmp_path / "kernel.cu"
    src.write_text("// kernel v1\n")
    prof = tmp_path / "profiles"
    prof.mkdir()
    entry = {"grouped_gemm_bytes_per_launch": 123,
             "sources_sha256": {"kernel.cu": hashlib.sha256(b"// kernel v1\n").hexdigest()}}
    (prof / "traffic.json").write_text(json.dumps({"note": "test", "w": entry}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.captured_traffic("w") == 123
    assert bench.captured_traffic("other") is None
    src.write_text("// kernel v2\n")  # the kernel changed since the capture
    assert bench.captured_traffic("w") is None
    os.remove(src)
    assert bench.captured_traffic("w") is None


def test_committed_traffic_record_is_consistent():
    """The committed record names existing sources and a per-launch byte count near the
    algorithmic bytes of one moe_expert_ffn call (between 1x and 2x)."""
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "traffic.json")))["mixtral"]
    for rel in rec["sources_sha256"]:
        assert os.path.exists(os.path.join(bench.ROOT, rel)), rel
    cfg = synth.CONFIGS["mixtral"]
    rows = cfg.T * cfg.k
    alg = 2 * cfg.E * cfg.H * cfg.F * 2 + rows * cfg.H * 2 + 2 * rows * cfg.F * 2 + 2 * cfg.T * cfg.H * 4
    assert alg <= rec["grouped_gemm_bytes_per_launch"] <= 2 * alg
    assert math.isclose(sum(v["dram_read"] + v["dram_write"] for v in rec["per_kernel"].values()),
                        rec["grouped_gemm_bytes_per_launch"])


PEAKS = {"hbm_gbs": 6548.8, "bf16_tflops": 1661.1, "bf16_tflops_sustained": 1383.9, "source": "measured"}


def test_roofline_bound_follows_arithmetic_intensity():
    mix = synth.CONFIGS["mixtral"]
    r = bench.ffn_roofline(mix, mix.T * mix.k, mix.E, 1.75, PEAKS)
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(4.0 * mix.H * mix.F * mix.T * mix.k / 1.75e-3 / 1e12)
    # the call is timed alone: the burst peak is the denominator, the sustained fraction rides along
    assert r["frac"] == pytest.approx(r["achieved"] / PEAKS["bf16_tflops"])
    assert r["frac_of_sustained"] == pytest.approx(r["achieved"] / PEAKS["bf16_tflops_sustained"])
    assert "tensor_flop_per_sm_clk" not in r
    # a loop of 20 calls (35 ms) ends before the power cap's onset: burst peak; 500 calls (0.9 s): sustained
    short = bench.ffn_roofline(mix, mix.T * mix.k, mix.E, 1.75, PEAKS, None, 148, 20 * 1.75e-3)
    assert short["peak"] == PEAKS["bf16_tflops"] and short["frac"] == pytest.approx(r["frac"])
    long = bench.ffn_roofline(mix, mix.T * mix.k, mix.E, 1.75, PEAKS, None, 148, 500 * 1.75e-3)
    assert long["peak"] == PEAKS["bf16_tflops_sustained"] and "sustained" in long["peak_source"]
    assert long["frac"] == pytest.approx(r["frac_of_sustained"])
    assert long["frac_of_burst"] == pytest.approx(r["frac"])
    clk = bench.ffn_roofline(mix, mix.T * mix.k, mix.E, 1.75, PEAKS, {"sm_mhz": 1500.0}, 148)
    per_clk = 4.0 * mix.H * mix.F * mix.T * mix.k / (1.75e-3 * 1500e6 * 148)
    assert clk["tensor_flop_per_sm_clk"]["value"] == pytest.approx(per_clk)
    assert clk["tensor_flop_per_sm_clk"]["of_nominal"] == pytest.approx(per_clk / 8192)
    dec = synth.CONFIGS["decode"]
    r = bench.ffn_roofline(dec, dec.T * dec.k, dec.E, 0.35, PEAKS)
    assert r["bound"] == "hbm" and r["unit"] == "GB/s"
    weights = dec.E * (2 * dec.H * dec.F + dec.F + dec.H) * 2
    assert weights < r["algorithmic"]["bytes"] < 1.05 * weights  # weight streaming dominates
    assert r["frac"] == pytest.approx(r["algorithmic"]["bytes"] / 0.35e-3 / 1e9 / PEAKS["hbm_gbs"])
    sw = synth.CONFIGS["switch"]
    assert bench.ffn_roofline(sw, 8104, sw.E, 0.56, PEAKS)["bound"] == "hbm"


def test_stratified_rows_cover_every_tile():
    """The full-size parity rows: both ends of every segment, a row in every 128-row block of every
    segment, and every row of each segment's last block; empty segments contribute nothing."""
    from moe_testlib import stratified_columns, stratified_rows, stratified_tokens

    counts = np.array([1000, 0, 1, 128, 129, 256, 300, 0])
    offsets = np.concatenate([[0], np.cumsum(counts)])
    rows = stratified_rows(offsets, seed=3)
    for e, c in enumerate(counts):
        a, b = offsets[e], offsets[e + 1]
        mine = rows[(rows >= a) & (rows < b)]
        if c == 0:
            assert mine.size == 0
            continue
        assert a in mine and b - 1 in mine
        for m0 in range(a, b, 128):
            assert ((mine >= m0) & (mine < min(b, m0 + 128))).any()
        tail0 = a + ((c - 1) // 128) * 128
        assert set(range(tail0, b)) <= set(mine.tolist())
    row_token = np.arange(offsets[-1])[::-1] % 700
    toks = stratified_tokens(offsets, row_token, seed=3)
    assert set(toks.tolist()) == set(row_token[rows].tolist())
    cols = stratified_columns(14336, seed=1)
    assert len(cols) >= 56 and cols.max() == 14335
    for c0 in range(0, 14336, 256):
        assert ((cols >= c0) & (cols < c0 + 256)).any()
    assert ((cols >= 14080)).sum() >= 8
