"""Host-side logic of bench.py that the JSON line depends on, checked without a GPU: the DRAM
traffic lookup is tied to the kernel sources it was captured on, the roofline denominators
come from the measured peaks (else the stated fallback), and the workload description both
arms print is the same dict."""
from __future__ import annotations

import hashlib
import json
import os

import bench
import synth


def _fake_root(tmp_path, src_text="kernel v1\n", value=12345):
    os.makedirs(tmp_path / "profiles")
    os.makedirs(tmp_path / "src")
    (tmp_path / "src" / "k.cuh").write_text(src_text)
    digest = hashlib.sha256(src_text.encode()).hexdigest()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"my_kernel": {"wl": {"dram_bytes_per_launch": value, "sources": {"src/k.cuh": digest}}}}))
    return tmp_path


def test_traffic_follows_the_recorded_sources(tmp_path, monkeypatch):
    root = _fake_root(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.kernel_traffic("my_kernel", "wl") == 12345
    assert bench.kernel_traffic("my_kernel", "other") is None
    assert bench.kernel_traffic("other_kernel", "wl") is None
    (root / "src" / "k.cuh").write_text("kernel v2\n")      # the kernel changed since the capture
    assert bench.kernel_traffic("my_kernel", "wl") is None
    os.remove(root / "src" / "k.cuh")
    assert bench.kernel_traffic("my_kernel", "wl") is None


def test_recorded_traffic_entries_name_their_sources_and_command():
    d = json.load(open(os.path.join(bench.ROOT, "profiles", "traffic.json")))
    for kernel, per_wl in d.items():
        if kernel.startswith("_"):
            continue
        for wl, e in per_wl.items():
            assert e["dram_bytes_per_launch"] > 0
            assert e["sources"] and all(os.path.exists(os.path.join(bench.ROOT, s)) for s in e["sources"])
            assert "--clock-control none" in e["command"]


def test_peaks_measured_else_fallback(tmp_path, monkeypatch):
    p = bench.load_peaks()
    if os.path.exists(os.path.join(bench.ROOT, "MEASURED_PEAKS.json")):
        m = json.load(open(os.path.join(bench.ROOT, "MEASURED_PEAKS.json")))
        assert p["source"] == "measured" and p["hbm"] == m["hbm_gbs"] and p["bf16"] == m["bf16_tflops"]
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    f = bench.load_peaks()
    assert f["source"] == "fallback" and f["hbm"] == 6650.0 and f["bf16"] == 1590.0


def test_workload_config_is_one_dict_for_both_arms():
    wl = synth.get_workload("prefill20m")
    a = bench.workload_config(wl, 1)
    b = bench.workload_config(wl, 1)
    assert a == b
    assert a["workload"] == "prefill20m" and a["B"] == 32 and a["T"] == 8192
    assert a["tokens_per_step_per_gpu"] == 32 * 8192 and a["table_rows"] == 9_999_991
    assert abs(a["table_GiB"] - 95.37) < 0.01
