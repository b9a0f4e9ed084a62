"""The JSON line of bench.py's reference (oracle) arm carries every key of the contract;
it runs on the host, so no GPU is needed."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.parametrize("workload,unit", [("ouro14_g16_32k", "tokens/s"), ("ouro26_prefill_32k", "vectors/s")])
def test_reference_arm_line_has_the_contract_keys(workload, unit):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "0", "--ref-sample", "1", "--oracle-procs", "2", "--workload", workload],
                       capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["config"]["workload"] == workload and d["unit"] == unit
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["cores"] == 2 and cb["value"] == d["value"] and cb["sample"]
    assert d["e2e"]["value"] == d["value"] and d["e2e"]["h2d_bytes_per_step"] == 0


def test_oracle_processes_default_to_the_usable_cores():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.oracle_procs(3) == 3
    n = bench.oracle_procs()
    assert 1 <= n <= bench.ORACLE_MAX_PROCS and n <= len(os.sched_getaffinity(0))
