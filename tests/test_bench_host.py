"""bench.py's CPU parts on the host.  The reference arm (the oracle timed on a bounded sample)
prints one JSON line with the contract's keys (the same metric, unit and direction as the GPU
arm, the oracle described as the CPU baseline, an end-to-end object without copies), and ranks
other than 0 print nothing and exit 0.  The GPU arm's cpu_baseline objects are built the same
way for every pass."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
KEYS = {"impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
        "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"}


def _bench(*args, env=None):
    e = dict(os.environ)
    e.update(env or {})
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", *args],
                       capture_output=True, text=True, timeout=600, cwd=ROOT, env=e)
    assert r.returncode == 0, r.stderr[-2000:]
    return r.stdout


@pytest.mark.parametrize("which,workload", [("forward", "vmamba_t_stage1"), ("backward", "tiny"),
                                            ("train", "tiny"), ("forward", "proj")])
def test_reference_arm_prints_one_contract_line(which, workload):
    out = _bench("--steps", "2", "--warmup", "1", "--pass", which, "--workload", workload)
    lines = [l for l in out.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert KEYS <= set(line)
    assert line["impl"] == "reference"
    assert line["unit"] == "Gelem/s" and line["higher_is_better"] is True and line["scaling"] == "weak"
    # the GPU arm's metric for the same pass
    assert line["metric"] == {"forward": "SS2D core Gelem/s (B*4*D*L)",
                              "backward": "SS2D core backward Gelem/s (B*4*D*L)",
                              "train": "SS2D core training step Gelem/s (B*4*D*L)"}[which]
    assert line["steps"] == 2 and line["warmup"] == 3  # fewer than 3 warm-up steps are raised to 3
    assert line["value"] > 0 and line["vs_baseline"] is None
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] == 1 and cb["value"] == line["value"] and cb["sample"]
    e2e = line["e2e"]
    assert e2e["value"] == line["value"] and e2e["unit"] == line["unit"]
    assert e2e["h2d_bytes_per_step"] == 0 and e2e["d2h_bytes_per_step"] == 0


def test_reference_arm_is_silent_on_other_ranks():
    assert _bench("--steps", "2", "--workload", "tiny", env={"RANK": "1", "WORLD_SIZE": "2"}).strip() == ""


@pytest.mark.parametrize("kind", ["forward", "backward", "train"])
def test_cpu_baseline_object(kind):
    """The cpu_baseline object the GPU arm adds to its line (the oracle on a bounded sample)."""
    sys.path.insert(0, ROOT)
    import bench
    from selective_scan_02_b200.inputs import WORKLOADS

    wl = WORKLOADS["tiny"]
    cb = bench.cpu_baseline(wl, 0.2) if kind == "forward" else \
        bench.cpu_baseline_backward(wl, 0.2, train=kind == "train")
    assert cb["unit"] == "Gelem/s" and cb["kind"] == "oracle" and cb["cores"] == 1
    assert cb["value"] > 0 and "scan elements" in cb["sample"]


def test_algorithmic_bytes_match_the_stated_figures():
    """The roofline numerators: the bytes each workload must move at least once."""
    sys.path.insert(0, ROOT)
    import bench
    from selective_scan_02_b200.inputs import WORKLOADS

    mb = lambda n: n / 1e6
    # stage 1 forward: x 38.5 (bf16) + dts 154.1 (bf16) + B, C 51.4 + y 77.1 MB
    assert abs(mb(bench.algorithmic_bytes(WORKLOADS["vmamba_t_stage1"])) - 321.1) < 0.5
    # projection form: x read twice 154.1 + x_dbl written and read 244.1 + y 154.1 MB
    assert abs(mb(bench.algorithmic_bytes(WORKLOADS["proj"])) - 552.4) < 0.5
    # stage 1 backward: x, dts, B, C, dy read; dx, ddts, dB, dC written
    assert abs(mb(bench.bwd_algorithmic_bytes(WORKLOADS["vmamba_t_stage1"])) - 758.0) < 1.0


def test_recorded_traffic_follows_the_kernel_sources():
    """The committed ncu traffic is reported only for its workload and only while the hashed
    kernel sources are the ones it was captured from."""
    sys.path.insert(0, ROOT)
    import bench
    from selective_scan_02_b200.inputs import WORKLOADS

    rec = json.load(open(bench.TRAFFIC_FILE))
    got = bench.recorded_traffic(WORKLOADS["vmamba_t_stage1"])
    if rec["kernel_hash"] == bench.kernel_source_hash():
        assert got == float(rec["bytes_per_launch_full_size"])
    else:
        assert got is None
    assert bench.recorded_traffic(WORKLOADS["tiny"]) is None
