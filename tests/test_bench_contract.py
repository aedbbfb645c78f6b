"""bench.py's two arms report the same metric, unit and config.

The reference arm times the oracle on a bounded sample (for a batched
workload: one stream as old as the oldest of the batch), but its JSON line
must name the workload exactly as the GPU arm does. The oracle timing is
stubbed here, so this checks only the reporting, on the CPU.
"""
import json
import types

import pytest

import bench
import workload


@pytest.mark.parametrize("w", [1, 2, 3, 4, 5])
def test_reference_arm_reports_the_gpu_arms_metric_and_config(w, monkeypatch, capsys):
    monkeypatch.setattr(bench, "cpu_baseline", lambda *a, **k: {"value": 1.0, "sample": "stub"})
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setenv("RANK", "0")
    bench.run_reference(types.SimpleNamespace(workload=w, seed=1, steps=1, warmup=0, cpu_budget=20.0))
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    wl = workload.WORKLOADS[w]
    assert line["impl"] == "reference"
    assert line["metric"] == bench.metric_name(w, wl)     # what the GPU arm prints
    assert line["config"] == bench.arm_config(wl, 1, 1)
    assert line["unit"] == "frames/s" and line["higher_is_better"] is True
    assert line["e2e"] == {"value": 1.0, "unit": "frames/s", "h2d_bytes_per_step": 0,
                           "d2h_bytes_per_step": 0}
    if wl.streams > 1:
        assert len(line["config"]["stream_ages"]) == wl.streams


def test_reference_arm_prints_on_rank_0_only(monkeypatch, capsys):
    monkeypatch.setattr(bench, "cpu_baseline", lambda *a, **k: {"value": 1.0, "sample": "stub"})
    monkeypatch.setenv("WORLD_SIZE", "2")
    monkeypatch.setenv("RANK", "1")
    bench.run_reference(types.SimpleNamespace(workload=1, seed=1, steps=1, warmup=0, cpu_budget=20.0))
    assert capsys.readouterr().out == ""


@pytest.mark.parametrize("w", [1, 3, 4])
def test_both_arms_time_the_oracle_on_one_sample(w, monkeypatch, capsys):
    """The reference arm's steps and the GPU arm's cpu_baseline call the
    oracle on the same frames and rows, so their frames/s agree up to noise."""
    seen = []

    def stub(wl, seed, budget_s=20.0, frames_sample=None, rows=None):
        seen.append((wl.frames, tuple(frames_sample), rows))
        return {"value": 1.0, "sample": "stub"}

    monkeypatch.setattr(bench, "cpu_baseline", stub)
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setenv("RANK", "0")
    bench.run_reference(types.SimpleNamespace(workload=w, seed=1, steps=2, warmup=1, cpu_budget=20.0))
    wl = workload.WORKLOADS[w]
    timed = seen[1:]                       # after the warm-up call
    assert len(timed) == 2
    n = wl.frames if wl.streams == 1 else wl.age_hi
    want = tuple(sorted({min(wl.S + wl.W, n) - 1, n - 1}))
    assert all(t == (n, want, None) for t in timed)
    if wl.streams == 1:
        assert bench.oracle_sample_frames(wl) == want   # what run_gpu passes to cpu_baseline
