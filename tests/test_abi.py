"""The C-ABI library loads without a GPU, exports every function the header
declares, and rejects bad arguments before touching a device."""
import ctypes
import os
import re
import subprocess

import pytest

import lightning_indexer_top_02_b200 as L
from lightning_indexer_top_02_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build()
    return L.load_library()


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(csa_[a-z0-9_]+)\s*\(", text))
    return names


def test_header_symbols_exported(lib):
    declared = declared_functions()
    assert declared, "no functions found in include/*.h"
    out = subprocess.run(["nm", "-D", "--defined-only", L.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    missing = declared - exported
    assert not missing, f"declared but not exported: {sorted(missing)}"
    assert set(L.EXPORTS) <= declared


def test_status_strings(lib):
    for st in range(6):
        assert L.csa_status_string(st)
    assert L.csa_status_string(5) == "device-side wait timed out"
    assert L.csa_version() >= 100


def test_invalid_arguments_without_gpu(lib):
    a = L.CsaArgs()
    a.B, a.S, a.T, a.H_I, a.d, a.m, a.topk = 1, 4, 8, 4, 32, 1, 2
    # null pointers
    assert L.csa_indexer_topk_ex(a, None, 0, None) == L.CSA_ERR_INVALID_ARG
    a.q = a.w = a.k = a.out_idx = a.out_score = 4096
    a.H_I = 3
    assert L.csa_indexer_topk_ex(a, None, 0, None) == L.CSA_ERR_UNSUPPORTED
    a.H_I = 4
    a.d = 48
    assert L.csa_indexer_topk_ex(a, None, 0, None) == L.CSA_ERR_UNSUPPORTED
    a.d = 32
    a.topk = 0
    assert L.csa_indexer_topk_ex(a, None, 0, None) == L.CSA_ERR_INVALID_ARG
    a.topk = 2
    a.q = 4100  # not 16-byte aligned
    assert L.csa_indexer_topk_ex(a, None, 0, None) == L.CSA_ERR_INVALID_ARG
    assert L.csa_indexer_workspace_size(a) == 0
    assert lib.csa_indexer_topk_ex(None, None, 0, None) == L.CSA_ERR_INVALID_ARG
    # B*S == 0 is a valid no-op
    a.q = 4096
    a.S = 0
    assert L.csa_indexer_topk_ex(a, None, 0, None) == L.CSA_OK
