"""The bench runs its avq arm end to end on the GPU for workloads whose
shapes differ from the headline one: no child refinement (P = 0, an empty
selection output), the flat 192-codeword VQ, and a ragged token count, each
printing one JSON line with the contract's keys."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("config", ["sweep:0:4096", "flat192:4096", "vit28"])
def test_bench_line(config):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--config", config, "--steps", "2",
                        "--warmup", "3", "--no-cpu-baseline", "--profile"],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    line = [x for x in r.stdout.splitlines() if x.startswith("{")][-1]
    d = json.loads(line)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "config", "roofline",
                "gpu_launches", "clocks"):
        assert key in d, key
    assert d["value"] > 0 and d["steps"] == 2 and d["config"]["workload"] == config
