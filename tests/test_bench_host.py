"""CPU checks of bench.py's host logic: the algorithmic byte and flop counts
the roofline divides by (against the figures derived by hand from the
workloads' shapes), the traffic record's source check, and the reference
arm's JSON line (the oracle on a bounded sample)."""
import io
import json
import os
import shutil
import contextlib
import types

import pytest

import bench
from weight_state_recurrence_b200 import inputs


def test_algorithmic_bytes_match_the_workloads():
    # causal_decay_d128: q, k, v read and y written once, 4 * 128 * 2 B per
    # head-token over 4 * 16 * 16384 head-tokens, plus S_final and z_final
    w = inputs.WORKLOADS["causal_decay_d128"]
    head_tokens = w.B * w.H * w.N
    assert bench.causal_bytes(w.B, w.H, w.N, w.d, w.d) == \
        head_tokens * 1024 + w.B * w.H * (128 * 128 + 128) * 4 == 1_077_968_896
    # decode_d128: per head-step S and z read and written (fp32), q, k, v read, y written
    wd = inputs.WORKLOADS["decode_d128"]
    assert bench.decode_bytes(wd.B, wd.H, 128, 128) == \
        wd.B * wd.H * (2 * 128 * 128 * 4 + 2 * 128 * 4 + 4 * 128 * 2) == 1_090_519_040
    # global_d64
    wg = inputs.WORKLOADS["global_d64"]
    assert bench.global_bytes(wg.B, wg.H, wg.N, 64, 64) == 404_250_624
    # Performer features: x read, 2m features written, omega once
    assert bench.features_bytes(1_048_576, 128, 64) == 1_048_576 * (128 + 128) * 2 + 64 * 128 * 2


def test_mma_flops_of_the_causal_kernel():
    # per 128-token chunk and head, the whole dv in one CTA: the score tile,
    # the carried term, the state update and the intra term, each 128 x 128
    # x 128 at d = 128, 2 flops per multiply-add
    per = 4 * 2 * 128 * 128 * 128
    assert bench.causal_mma_flops(4, 16, 16384, 128, 128) == 4 * 16 * 128 * per
    # 137.4 GFLOP for the headline workload (the count at C = 128)
    assert round(bench.causal_mma_flops(4, 16, 16384, 128, 128) / 1e9, 1) == 137.4
    # d = 64: the state update keeps its 128 rows of d_k (zero-padded)
    assert bench.causal_mma_flops(2, 8, 4096, 64, 64) == \
        16 * 32 * 2 * 128 * (128 * 64 + 64 * 64 + 64 * 128 + 64 * 128)


def test_backward_mma_count():
    g = 2 * 128 ** 3
    # one chunk: F has P, At V, W, B Kt; L has Ms; R has P^T, W^T, A^T w, B^T Q
    assert bench.bwd_mma_flops(1, 1, 128, 128) == 9 * g
    assert bench.bwd_mma_flops(1, 1, 100, 128, with_dlam=False) == 8 * g
    # two chunks: F 4n + 2(n-1) + (n-1) = 11, L n + 2(n-1) = 4, R 11
    assert bench.bwd_mma_flops(1, 1, 256, 128) == 26 * g
    # the headline workload: 2168 groups per head, 581.9 GFLOP
    assert bench.bwd_mma_flops(4, 16, 16384, 128) == 64 * 2168 * g
    assert bench.bwd_bytes(4, 16, 16384, 128) == 7 * 64 * 16384 * 128 * 2


def test_traffic_record_checks_its_sources(tmp_path, monkeypatch):
    src = tmp_path / "k.cuh"
    src.write_text("kernel v1\n")
    import hashlib
    sha = hashlib.sha256(b"kernel v1\n").hexdigest()
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.json").write_text(json.dumps(
        {"kern": {"bytes_per_launch": 123, "sources": ["k.cuh"], "sha256": sha}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_record("kern") == 123
    assert bench.traffic_record("other") is None
    src.write_text("kernel v2\n")          # the kernel changed since the capture
    assert bench.traffic_record("kern") is None


def test_committed_traffic_records_are_current():
    # the records in profiles/ are keyed to the sources they were taken on
    rec = json.load(open(os.path.join(bench.ROOT, "profiles", "traffic.json")))
    for name in rec:
        assert bench.traffic_record(name) == rec[name]["bytes_per_launch"], name


def test_reference_arm_prints_one_contract_line(monkeypatch):
    args = types.SimpleNamespace(gpus=1, steps=1, warmup=3)
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setattr(bench, "oracle_sample",
                        lambda target_s=12.0, heads=None: (1234.0, 2, "stub sample", 0.5))
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        assert bench.reference_arm(args) == 0
    line = json.loads(buf.getvalue().strip())
    assert line["impl"] == "reference" and line["value"] == 1234.0
    assert line["metric"] == bench.METRIC and line["unit"] == "tokens/s"
    assert line["higher_is_better"] is True and line["n_gpus"] == 1
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] == 2
    assert line["e2e"] == {"value": 1234.0, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_do_nothing(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        assert bench.reference_arm(types.SimpleNamespace(gpus=2, steps=1, warmup=3)) == 0
    assert buf.getvalue() == ""


def test_oracle_sample_is_bounded_and_consistent():
    tok_s, cores, desc, dt = bench.oracle_sample(target_s=0.5, heads=2)
    assert tok_s > 0 and cores >= 1 and dt > 0
    assert "causal_decay_d128" in desc
