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
    """1024 sequences with top-2048 need ~84 MB of candidate lists for just
    one block of queries per sequence (1024 sequences x 4 queries x 2560 keys
    x 8 bytes): more than the fixed array holds even when run in chunks, so
    the call must refuse before launching anything."""
    a = lib.CsaArgs()
    a.B, a.S, a.T, a.H_I, a.d, a.m, a.topk = 1024, 4, 8192, 64, 128, 4, 2048
    a.causal, a.q_offset = 1, lib.CSA_Q_OFFSET_DEFAULT
    a.q = a.w = a.k = a.out_idx = a.out_score = 1 << 20  # never dereferenced
    st = lib.csa_indexer_topk_noalloc(a, None)
    assert st == lib.CSA_ERR_WORKSPACE


def _launches_of(L, call):
    """Kernel launches one call makes, counted with the launch-event hook:
    events the call re-records land after a ~1 ms sleep on the stream, the
    rest keep their earlier timestamps."""
    n = 2049
    base = torch.cuda.Event(enable_timing=True)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    base.record()
    for e in ev:
        e.record()
    torch.cuda._sleep(2_000_000)
    L.csa_set_launch_events(ev)
    try:
        call()
    finally:
        L.csa_set_launch_events(None)
    torch.cuda.synchronize()
    late = [base.elapsed_time(e) > 0.3 for e in ev]
    return sum(late) - 1  # events[L] follows the last launch


def _noalloc_vs_oracle(L, wl, rows=None, min_launches=0):
    import oracle
    from parity import check_exact

    inp = workloads.make_inputs(wl, device="cuda")
    q, w, k, ks = inp["q"], inp["w"], inp["k"], inp["k_scale"]
    shape = (wl.B, wl.S, wl.topk)
    idx = torch.full(shape, -7, dtype=torch.int32, device="cuda")
    sc = torch.full(shape, 7.0, dtype=torch.float32, device="cuda")
    a = L.make_args(q, w, k, k_scale=ks, m=wl.m, topk=wl.topk, causal=wl.causal,
                    out_idx=idx, out_score=sc)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)

    def call():
        st = L.csa_indexer_topk_noalloc(a, stream)
        assert st == L.CSA_OK, L.csa_status_string(st)

    launches = _launches_of(L, call)
    assert launches >= min_launches, f"{launches} launches, expected >= {min_launches}"
    torch.cuda.synchronize()
    assert L.csa_last_device_error(None) == L.CSA_OK
    qb, wb, kb, kb_s = workloads.as_numpy_bits(inp)
    ri, rs, _, _ = oracle.topk(qb, wb, kb, kb_s, B=wl.B, S=wl.S, T=wl.T, H=wl.H, d=wl.d, m=wl.m,
                               topk=wl.topk, causal=wl.causal, rows=rows)
    gi = idx.cpu().numpy().reshape(-1, wl.topk)
    gs = sc.cpu().numpy().reshape(-1, wl.topk)
    if rows is not None:
        gi, gs = gi[rows], gs[rows]
    check_exact(gi, gs, ri, rs, label=wl.name)
    return launches


def test_many_launch_chunks_match_oracle(lib):
    """8192 queries at top-2048 need ~168 MB of candidate lists, so the fixed
    array runs the call as a dozen launch chunks of query blocks; chunks past
    the first start at a nonzero query block.  Every row must equal the
    oracle's bit for bit (integer-valued inputs)."""
    wl = workloads.Workload("na_chunks", B=1, S=8192, T=4096, H=16, d=64, m=1, topk=2048,
                            values="integer", seed=3004)
    _noalloc_vs_oracle(lib, wl, min_launches=2 * 3)


def test_reduced_grid_matches_oracle(lib):
    """Items of 16,384 keys make the per-CTA score buffers of a full grid
    larger than the fixed array, so the call runs fewer CTAs than SMs, and
    again in many launch chunks.  Sampled rows (every row of the first,
    second and last chunks' boundaries among them) must equal the oracle's
    bit for bit."""
    wl = workloads.Workload("na_grid", B=1, S=2400, T=16384, H=64, d=128, m=1, topk=2048,
                            values="integer", seed=3005)
    rng = np.random.default_rng(3006)
    rows = np.unique(np.concatenate([rng.integers(0, wl.S, 160), np.arange(0, 40),
                                     np.arange(wl.S - 40, wl.S)])).astype(np.int64)
    _noalloc_vs_oracle(lib, wl, rows=rows, min_launches=2 * 3)
