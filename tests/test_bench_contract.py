"""Parts of the bench line that need no GPU.

- The DRAM traffic figure beside the roofline comes from the last ncu
  capture of the fused kernel (profiles/attn_tc_traffic.json). It stands
  only for the captured workload and only while the kernel's source is the
  captured one; otherwise the bench reports null.
- The reference arm (the oracle on the host cores) prints the GPU arm's
  metric, unit, direction and config; each of its steps is one whole frame
  and its ms_per_step is the measured time of one.
- The GPU arm's CPU baseline times whole frames the same way, so that the
  two timings of the oracle agree."""
import json
import os
import shutil
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _record():
    with open(os.path.join(ROOT, "profiles", "attn_tc_traffic.json")) as f:
        return json.load(f)


def test_traffic_for_the_captured_workload_and_source():
    d = _record()
    workload = d["workload"].split()[0]
    assert bench.measured_traffic(workload) == d["dram_bytes_per_launch"]
    assert d["dram_bytes_per_launch"] == d["dram_bytes_read"] + d["dram_bytes_write"]


@pytest.mark.parametrize("other", ["720p_bf16", "long_stream_bf16", "tiny_fp32"])
def test_no_traffic_for_another_workload(other):
    assert bench.measured_traffic(other) is None


def test_no_traffic_once_the_source_changes(tmp_path, monkeypatch):
    d = _record()
    workload = d["workload"].split()[0]
    os.makedirs(tmp_path / "profiles")
    shutil.copy(os.path.join(ROOT, "profiles", "attn_tc_traffic.json"), tmp_path / "profiles")
    for rel in d["source_files"]:
        dst = tmp_path / rel
        os.makedirs(dst.parent, exist_ok=True)
        shutil.copy(os.path.join(ROOT, rel), dst)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic(workload) == d["dram_bytes_per_launch"]
    with open(tmp_path / d["source_files"][0], "a") as f:
        f.write("\n// edited\n")
    assert bench.measured_traffic(workload) is None


def test_reference_arm_line_matches_the_gpu_arm(monkeypatch, capsys):
    # The reference arm (the oracle on the host) prints the same metric,
    # unit, direction and config as the GPU arm; the oracle's arithmetic is
    # stubbed out here, only the line is checked.
    import argparse

    import oracle
    import workloads

    monkeypatch.setattr(oracle, "build", lambda: None)
    monkeypatch.setattr(oracle, "frame_pass", lambda q, k, v, wq, wk, wv, a, b, S, clean: (None, S))
    monkeypatch.setattr(bench, "dist_env", lambda: (1, 0, 0))
    w = workloads.WORKLOADS["tiny_fp32"]
    args = argparse.Namespace(gpus=1, steps=1, warmup=0, gating="headwise", access="frame", gates="given")
    assert bench.run_reference(args, w) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["metric"] == bench.METRIC
    assert line["unit"] == "frames/s" and line["higher_is_better"] is True
    assert line["config"] == bench.arm_config(args, w, 1)
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]


def test_reference_arm_times_whole_frames(monkeypatch, capsys):
    # every pass of every step goes through the oracle's whole-pass call,
    # and ms_per_step is the measured time of one step
    import argparse
    import time

    import oracle
    import workloads

    calls = []

    def fake_pass(q, k, v, wq, wk, wv, a, b, S, clean):
        calls.append(clean)
        time.sleep(0.01)
        return None, S

    monkeypatch.setattr(oracle, "build", lambda: None)
    monkeypatch.setattr(oracle, "frame_pass", fake_pass)
    monkeypatch.setattr(bench, "dist_env", lambda: (1, 0, 0))
    w = workloads.WORKLOADS["480p_bf16"]
    args = argparse.Namespace(gpus=1, steps=2, warmup=1, gating="headwise", access="frame", gates="given")
    assert bench.run_reference(args, w) == 0
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    assert calls == [False, False, False, True] * 3  # (warm-up + steps) x passes, the last one clean
    assert 40.0 <= line["ms_per_step"] <= 400.0  # 4 passes x 10 ms each, measured
    assert abs(line["value"] - 1e3 / line["ms_per_step"]) < 1e-6 * line["value"]


def test_cpu_baseline_times_the_same_whole_frames(monkeypatch):
    import time

    import oracle
    import workloads

    calls = []

    def fake_pass(q, k, v, wq, wk, wv, a, b, S, clean):
        calls.append(clean)
        time.sleep(0.005)
        return None, S

    monkeypatch.setattr(oracle, "build", lambda: None)
    monkeypatch.setattr(oracle, "frame_pass", fake_pass)
    spf, threads, desc = bench.oracle_frame_seconds(workloads.WORKLOADS["480p_bf16"], budget_s=0.1)
    assert len(calls) % 4 == 0 and calls[:4] == [False, False, False, True]
    assert 0.02 <= spf <= 0.2 and threads >= 1 and "whole" in desc
