"""bench.py on one GPU prints one JSON line with every key of its report
(tiny workload, a few steps): metric, value, timing, roofline, CPU baseline,
end-to-end number, launch count and clock record; also in the head-sharded
mode."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*extra):
    p = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--config", "tiny", "--steps", "3",
                        "--warmup", "3", *extra], capture_output=True, text=True, timeout=600)
    assert p.returncode == 0, p.stderr[-2000:]
    lines = [ln for ln in p.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, lines
    return json.loads(lines[0])


@pytest.mark.parametrize("extra,scaling", [((), "weak"), (("--shard", "heads"), "strong")])
def test_bench_prints_the_whole_report(cuda_ok, extra, scaling):
    rec = run_bench(*extra)
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e",
                "gpu_launches", "clocks"):
        assert key in rec, key
    assert rec["n_gpus"] == 1 and rec["steps"] == 3 and rec["warmup"] == 3 and rec["scaling"] == scaling
    assert rec["value"] > 0 and rec["higher_is_better"] is False and rec["dtype"] == "bf16"
    assert rec["config"]["workload"].startswith("ISA fwd tiny")
    roof = rec["roofline"]
    for key in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert key in roof, key
    assert roof["bound"] == "tensor" and roof["peak"] > 0
    cpu = rec["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["cores"] >= 1 and cpu["value"] > 0
    e2e = rec["e2e"]
    assert e2e["value"] > 0 and e2e["h2d_bytes_per_step"] == 3 * 2 * 512 * 64 * 2
    assert e2e["d2h_bytes_per_step"] == 2 * 512 * 64 * 2
    assert rec["gpu_launches"] > 0
    assert {"sm_mhz", "sm_max_mhz", "reasons"} <= set(rec["clocks"])
