"""The parts of the benchmark's contract that need no GPU: the reference arm's
JSON line, and the source hashes that tie recorded ncu traffic to the exact
kernels it was measured on."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def run_bench(*args, timeout=300):
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args],
                         capture_output=True, text=True, timeout=timeout, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    return out.stdout.strip().splitlines()


@pytest.mark.parametrize("workload", ["b4h16t4096", "kda_b4h16t4096"])
def test_reference_arm_prints_one_contract_line(workload):
    lines = run_bench("--impl", "reference", "--steps", "1", "--warmup", "0",
                      "--workload", workload)
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "Mtokens/s" and d["value"] > 0
    assert d["higher_is_better"] is True and d["steps"] == 1 and d["warmup"] == 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
    assert d["config"]["workload"] == workload
    assert ("channel-wise" in d["metric"]) == workload.startswith("kda")


def test_traffic_records_name_known_kernel_sets():
    hashes = json.loads(run_bench("--source-hashes")[0])
    assert set(hashes) == {"chunk_fwd_step", "kda_chunk_fwd_step", "decode", "bwd_step"}
    assert all(len(h) == 16 for h in hashes.values())
    records = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    for key, rec in records.items():
        kind, workload = key.split("/")
        assert kind in hashes, key
        assert rec["dram_bytes_per_launch"] > 0 and rec["note"]
        # every summary names the hash its counters were taken on
        assert len(rec["src_hash"]) == 16
