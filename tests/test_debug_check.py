"""The debug build's index checks (-DCSA_DEBUG).

On the CPU: the function that records a failed check is run by a host
program (it is plain C++ there), which shows the device error word's layout
-- code, site, index, bound -- and that the first failure is the one kept; and
the whole library builds with the checks in and exports the same symbols.
On the GPU: the debug build gives the same results as the release build's
parity cases and reports no failed check.
"""
import os
import subprocess
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(ROOT, "lightning_indexer_top_02_b200", "csrc")


def test_failed_check_is_recorded(tmp_path):
    exe = str(tmp_path / "debug_check_host")
    subprocess.check_call(["g++", "-std=c++17", "-O1", "-I", CSRC, "-o", exe,
                           os.path.join(HERE, "debug_check_host.cpp")])
    out = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.splitlines()
    # kErrDebugCheck = 6, kChkListPos = 6, kChkTmemEpi = 4
    assert out[0] == "in_bounds 1 word 0 0 0 0"
    assert out[1] == "past_end 0 word 6 6 2560 2560"
    assert out[2] == "negative 0 word 6 6 2560 2560"   # the first failure is kept


@pytest.mark.slow
def test_debug_library_builds_and_exports_the_abi():
    sys.path.insert(0, ROOT)
    from lightning_indexer_top_02_b200 import EXPORTS
    from lightning_indexer_top_02_b200.build import build

    lib = build(debug=True)
    out = subprocess.run(["nm", "-D", "--defined-only", lib], capture_output=True, text=True,
                         check=True).stdout
    names = {line.split()[-1] for line in out.splitlines() if line.strip()}
    missing = [e for e in EXPORTS if e not in names]
    assert not missing, missing


_GPU_SCRIPT = r"""
import sys
sys.path.insert(0, {root!r}); sys.path.insert(0, {here!r})
import torch, lightning_indexer_top_02_b200 as L, workloads
from test_gpu_parity import run_gpu, run_oracle
from parity import check_exact
assert L.LIB_PATH.endswith("libcsa_indexer_debug.so"), L.LIB_PATH
L.load_library()
cases = [
    (workloads.CONFIGS["tiny"], 0, 0),
    (workloads.Workload("dbg1", B=2, S=300, T=1200, H=64, d=128, m=2, topk=300, values="integer", seed=41), 1, 0),
    (workloads.Workload("dbg2", B=3, S=3, T=9000, H=64, d=128, m=4, topk=512, values="integer", seed=42), 0, 0),
    (workloads.Workload("dbg3", B=1, S=200, T=700, H=16, d=64, m=1, topk=100, values="integer", seed=43, key_fp8=True), 0, 0),
]
for wl, mode, _ in cases:
    inp = workloads.make_inputs(wl)
    gi, gs = run_gpu(L, inp, wl, mode=mode)
    assert L.csa_last_device_error(None) == L.CSA_OK
    ri, rs, _, _ = run_oracle(inp, wl, mode=mode)
    check_exact(gi.reshape(-1, wl.topk), gs.reshape(-1, wl.topk), ri, rs, label=wl.name)
print("debug build ok")
"""


@pytest.mark.gpu
def test_debug_build_on_gpu():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    sys.path.insert(0, ROOT)
    from lightning_indexer_top_02_b200.build import build

    lib = build(debug=True)
    env = dict(os.environ, CSA_INDEXER_LIB=lib)
    r = subprocess.run([sys.executable, "-c", _GPU_SCRIPT.format(root=ROOT, here=HERE)],
                       capture_output=True, text=True, env=env, timeout=600)
    assert r.returncode == 0, r.stdout[-2000:] + r.stderr[-2000:]
    assert "debug build ok" in r.stdout
