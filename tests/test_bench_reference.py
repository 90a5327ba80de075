"""The reference arm of bench.py (the fp64 oracle on the host cores) prints
one well-formed contract line; it needs no GPU."""
import json
import os
import subprocess
import sys

ROOT = os.path.join(os.path.dirname(__file__), "..")


def test_reference_arm_prints_contract_line():
    out = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--config", "1", "--steps", "2",
                          "--warmup", "1"], cwd=ROOT, capture_output=True, text=True, timeout=300)
    assert out.returncode == 0, out.stderr[-2000:]
    line = json.loads(out.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in line, key
    assert line["value"] > 0 and line["steps"] == 2 and line["warmup"] == 1
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["d2h_bytes_per_step"] == 0
    assert line["config"]["workload"].startswith("tiny")


def test_schedule_inputs_drift_step_by_step_like_the_generator():
    """bench.py --schedule makes each step's inputs from the previous step's in
    worker processes; they must equal the generator's own step tensors."""
    sys.path.insert(0, ROOT)
    import numpy as np

    import bench
    import synth
    w = synth.workload(1).with_(steps=3)
    got = list(bench.schedule_inputs(w))
    assert [s for s, _ in got] == [1, 2, 3]
    for step, tensors in got:
        ref = synth.layer_tensors(w, step=step)
        for a, b in zip(tensors, ref):
            assert a.shape == b.shape and np.array_equal(a, b), step
