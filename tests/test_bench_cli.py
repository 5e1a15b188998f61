"""bench.py's host-side pieces on CPU: workload overrides, the traffic table
lookup, and the reference arm's JSON line."""
import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_with_overrides():
    out = subprocess.run(
        [sys.executable, os.path.join(ROOT, "bench.py"), "--config", "tiny", "--set", "causal=false",
         "--set", "S=64", "--impl", "reference", "--steps", "1", "--warmup", "3", "--ref-rows", "8"],
        capture_output=True, text=True, check=True, cwd=ROOT).stdout
    line = json.loads(out.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    assert line["config"]["causal"] is False and line["config"]["S"] == 64
    assert line["config"]["workload"] == "tiny[causal=false,S=64]"
    assert line["value"] > 0 and line["cpu_baseline"]["kind"] == "oracle"
    assert line["e2e"]["h2d_bytes_per_step"] == 0


def test_traffic_lookup_matches_sources():
    sha = bench.kernel_sources_sha()
    assert len(sha) == 16 and sha == bench.kernel_sources_sha()
    # a line for other sources never matches
    assert bench.measured_traffic("dsa_prefill", "0" * 16) is None
    assert bench.measured_traffic("no_such_workload", sha) is None
    # every recorded line parses to a positive byte count for its own sha
    with open(os.path.join(ROOT, "profiles", "traffic.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, _, line_sha, nbytes = line.split()[:4]
            assert int(nbytes) > 0
            if line_sha == sha:
                assert bench.measured_traffic(name, sha) == int(nbytes)
