"""The allocation-free entry point, csa_indexer_topk_noalloc.

It exists for callers that cannot allocate device memory while they run
(serving loops that must not risk cudaMalloc's device-wide synchronisation
mid-step, hosts with a fixed up-front memory budget).  It keeps its scratch
in one fixed array inside the library, so these tests check, through the C
ABI, that two calls in a row -- the second one reusing the array the first
one left behind -- give exactly what the allocating entry point gives, and
that a shape too large for the array is refused before any launch.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import lightning_indexer_top_02_b200 as L
    from lightning_indexer_top_02_b200.build import build

    build()
    L.load_library()
    return L


def _call_both(L, wl, mode=0):
    inp = workloads.make_inputs(wl, device="cuda")
    q, w, k, ks = inp["q"], inp["w"], inp["k"], inp["k_scale"]
    shape = (wl.B, wl.S, wl.topk)
    outs = []
    for entry in ("ex", "noalloc"):
        idx = torch.full(shape, -7, dtype=torch.int32, device="cuda")
        sc = torch.full(shape, 7.0, dtype=torch.float32, device="cuda")
        a = L.make_args(q, w, k, k_scale=ks, m=wl.m, topk=wl.topk, causal=wl.causal,
                        mode=mode, out_idx=idx, out_score=sc)
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        if entry == "ex":
            st = L.csa_indexer_topk_ex(a, None, 0, stream)
        else:
            st = L.csa_indexer_topk_noalloc(a, stream)
        assert st == L.CSA_OK, L.csa_status_string(st)
        torch.cuda.synchronize()
        assert L.csa_last_device_error(None) == L.CSA_OK
        outs.append((idx.cpu().numpy(), sc.cpu().numpy()))
    return outs


def _same(a, b):
    (ia, sa), (ib, sb) = a, b
    assert np.array_equal(ia, ib), "indices differ from the allocating entry point"
    assert np.array_equal(sa.view(np.uint32), sb.view(np.uint32)), "scores differ"


def test_two_calls_match_allocating_entry_point(lib):
    """Two calls in a row on different problems: the second reuses the scratch
    the first one wrote and must not be affected by it."""
    first = workloads.Workload("na1", B=2, S=700, T=1500, H=64, d=128, m=2, topk=300,
                               values="integer", seed=3001)
    second = workloads.Workload("na2", B=1, S=1100, T=900, H=16, d=64, m=1, topk=64,
                                seed=3002)
    for wl in (first, second):
        ex, na = _call_both(lib, wl)
        _same(ex, na)


def test_split_shape_and_gate(lib):
    """A few-query shape that splits key ranges (partials live in the scratch
    too) and the sigmoid-gated mode."""
    wl = workloads.Workload("na3", B=3, S=5, T=20000, H=64, d=128, m=4, topk=512,
                            values="integer", seed=3003)
    for mode in (0, 1):
        ex, na = _call_both(lib, wl, mode=mode)
        _same(ex, na)


def test_too_large_is_refused(lib):
    """1024 sequences with top-2048 need ~134 MB of candidate lists for just
    one block of queries per sequence: more than the fixed array holds even
    when run in chunks, so the call must refuse before launching anything."""
    a = lib.CsaArgs()
    a.B, a.S, a.T, a.H_I, a.d, a.m, a.topk = 1024, 4, 8192, 64, 128, 4, 2048
    a.causal, a.q_offset = 1, -1
    a.q = a.w = a.k = a.out_idx = a.out_score = 1 << 20  # never dereferenced
    st = lib.csa_indexer_topk_noalloc(a, None)
    assert st == lib.CSA_ERR_WORKSPACE
