"""The benchmark's host-side contract without a GPU: the reference arm (the fp64 oracle, the
only reference this subject has) prints one JSON line with the required keys on a small
configuration, and the 50-step schedule rule it reports matches the planner's."""

import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
                          "--density", "0.25", "--steps", "1", "--warmup", "1"],
                         capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    for key in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "higher_is_better", "config",
                "cpu_baseline", "e2e"):
        assert key in rec, key
    assert rec["impl"] == "reference" and rec["value"] > 0 and rec["higher_is_better"] is False
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["cpu_baseline"]["cores"] >= 1
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["e2e"]["d2h_bytes_per_step"] == 0
    # ms_per_step is the measured time of one step (one head's reuse step); value scales it to
    # the layer's B*H = 2 heads
    assert abs(rec["value"] - 2 * rec["ms_per_step"]) < 1e-9 * rec["value"]


def test_reference_arm_other_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "tiny",
                          "--steps", "1", "--warmup", "0"], capture_output=True, text=True, timeout=300, cwd=ROOT,
                         env=env)
    assert out.returncode == 0 and not out.stdout.strip()


def test_clock_sampler_parses_samples(tmp_path, monkeypatch):
    # a fake nvidia-smi writes three samples (one idle); the sampler keeps the loaded ones for
    # the median and reports every active throttle reason
    import subprocess
    import sys as _sys
    _sys.path.insert(0, ROOT)
    import bench

    lines = ("0, 1965, 1965, 950.1, 0x4, Not Active, Not Active, Not Active, Active\n"
             "0, 1900, 1965, 990.0, 0x4, Not Active, Not Active, Not Active, Active\n"
             "0, 600, 1965, 120.0, 0x0, Not Active, Not Active, Not Active, Not Active\n")

    class FakeProc:
        def __init__(self, args, stdout=None, stderr=None):
            stdout.write(lines)
            stdout.flush()

        def poll(self):
            return None

        def terminate(self):
            pass

        def wait(self, timeout=None):
            return 0

    monkeypatch.setattr(subprocess, "Popen", FakeProc)
    s = bench.ClockSampler(0, str(tmp_path / "clocks.csv"))
    s.start()
    out = s.stop()
    assert out["sm_mhz"] == 1932.5 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"] and out["samples"] == 2
