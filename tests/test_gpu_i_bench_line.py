"""GPU: one short run of bench.py prints one JSON line that carries every key
of its contract, with figures consistent with each other."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu


@pytest.mark.timeout(900)
def test_bench_line_contract():
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("WORLD_SIZE", "RANK", "LOCAL_RANK")}
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--steps", "2", "--warmup", "3",
                        "--no-configs", "--no-cpu-baseline"], capture_output=True, text=True, timeout=800,
                       env=env, cwd=root)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = lines[0]
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert key in d, key
    assert d["n_gpus"] == 1 and d["steps"] == 2 and d["warmup"] == 3
    assert d["unit"] == "TFLOP/s" and d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["dtype"] == "bf16" and d["data"] == "synthetic" and d["vs_baseline"] is None
    assert d["config"]["workload"].startswith("wan1.3b_6x")
    assert 0 < d["value"] < 2500 and d["ms_per_step"] > 0

    rf = d["roofline"]
    assert rf["bound"] == "tensor" and rf["unit"] == "TFLOP/s"
    assert abs(rf["frac"] - rf["achieved"] / rf["peak"]) < 1e-9
    assert 0.2 < rf["frac"] < 1.2                      # a little above 1.0 is possible, far above is not
    assert rf["traffic"] is None or rf["traffic"] > 0

    e2e = d["e2e"]
    assert e2e["unit"] == d["unit"] and e2e["value"] > 0
    assert e2e["h2d_bytes_per_step"] == 3 * 196560 * 12 * 128 * 2
    assert e2e["d2h_bytes_per_step"] == 196560 * 12 * 128 * 2 + 12 * 196560 * 4

    assert d["gpu_launches"] == 4 * d["steps"]
    ck = d["clocks"]
    assert ck["sm_mhz"] > 0 and ck["sm_max_mhz"] >= ck["sm_mhz"] and isinstance(ck["reasons"], list)
