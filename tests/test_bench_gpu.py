"""bench.py on the GPU, on the small 1,024-token workload.

The end-to-end leg splits the heads into groups with pitched copies and
checks, bit for bit, that the host results of its last step equal the
device-timed step's; a run that exits 0 has passed that check.  The JSON line
must carry the contract's keys.
"""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("groups,path", [(1, "bf16"), (2, "bf16"), (2, "fp8")])
def test_bench_end_to_end_leg(cuda_device, groups, path):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--workload", "pr1_s1024", "--steps", "3",
                        "--warmup", "3", "--e2e-steps", "3", "--e2e-head-groups", str(groups), "--path", path,
                        "--no-cpu-baseline"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = json.loads(r.stdout.strip().splitlines()[-1])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better", "scaling",
                "dtype", "config", "roofline", "e2e", "clocks", "gpu_launches"):
        assert key in line, key
    e2e = line["e2e"]
    assert e2e["head_groups"] == groups
    assert e2e["h2d_bytes_per_step"] == 3 * 2 * 1024 * 2 * 128   # q, k, v: B=1, S=1024, H=2, D=128, bf16
    assert e2e["d2h_bytes_per_step"] == 1024 * 2 * 128 * 2 + 2 * 1024 * 4
    assert e2e["value"] > 0 and line["value"] > 0
