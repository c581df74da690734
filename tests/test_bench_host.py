"""Host-side figures of bench.py (no GPU): the algorithmic work per launch that the roofline
divides by, and the source check that guards the DRAM traffic taken from a profile."""
import json
import os

import pytest

import bench
import inputs


def test_algorithmic_work_of_the_headline_field():
    w = inputs.WORKLOADS["field65k_bf16"]
    a = bench.algorithmic(dict(w))
    e = 2 * 8 * 65536 * 96 * 2  # bytes of one [B, H, N, d] bf16 tensor
    assert e == 201326592
    # summaries pass: k, v read, k_rot written, two summary tensors written, tables read
    assert a["summarize"]["bytes"] == 3 * e + 2 * 2 * 8 * 1024 * 96 * 2 + 65536 * 8
    assert a["summarize"]["bytes"] == 610795520
    # local branch: q, k_rot, v read, o_loc written, inverse map read
    assert a["local"]["bytes"] == 4 * e + 65536 * 4 == 805568512
    # global branch: QK and PV, 2 N M d flops each, per (batch, head)
    assert a["global"]["flops"] == pytest.approx(4.0 * 65536 * 1024 * 96 * 16)
    assert a["global"]["flops"] == pytest.approx(412316860416.0)


def test_traffic_is_reported_only_for_unchanged_sources(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("kernel v1\n")
    import hashlib
    entry = {"kernel": "k", "bytes_per_launch_full": 123.0, "sources": ["k.cu"],
             "sources_sha256": hashlib.sha256(b"kernel v1\n").hexdigest()}
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps({"x_w": entry}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.kernel_traffic("x_w") == 123.0
    assert bench.kernel_traffic("missing") is None
    src.write_text("kernel v2\n")  # the kernel changed since the counters were taken
    assert bench.kernel_traffic("x_w") is None


def test_committed_traffic_entries_name_existing_sources():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    t = json.load(open(os.path.join(root, "profiles", "traffic.json")))
    assert set(t) == {"summarize_field65k_bf16", "local_field65k_bf16", "global_field65k_bf16"}
    for e in t.values():
        for s in e["sources"]:
            assert os.path.exists(os.path.join(root, s)), s
        assert os.path.exists(os.path.join(root, e["capture"]))


def test_step_roofline_of_the_headline_field():
    w = inputs.WORKLOADS["field65k_bf16"]
    e = 201326592
    alg = bench.step_algorithmic(dict(w), index_bytes=8_000_000)
    # q, k, v read and o written, gate read, summaries written and read back, tables
    assert alg["bytes"] == 4 * e + 2 * 8 * 65536 * 2 + 4 * (2 * 8 * 1024 * 96 * 2) + 8_000_000
    assert alg["flops"] == pytest.approx(412316860416.0)
    peaks = dict(hbm=6508.8, bf16=1624.0, source="measured")
    r = bench.step_roofline(alg, 1.0, peaks)
    # tensor-bound: 412.3 GFLOP at 1,624 TFLOP/s is 0.2539 ms, more than 0.83 GB at 6.5 TB/s
    assert r["bound"] == "tensor"
    assert r["roofline_ms"] == pytest.approx(0.25389, rel=1e-4)
    assert r["frac"] == pytest.approx(0.25389, rel=1e-4)  # the step took 1 ms
    assert r["achieved"] == pytest.approx(412.3169, rel=1e-4)


def test_cores_used_is_cpu_time_over_wall_time():
    assert bench.cores_used(10.0, 10.2) == 1
    assert bench.cores_used(10.0, 38.0) == 4
    assert bench.cores_used(10.0, 0.1) == 1
