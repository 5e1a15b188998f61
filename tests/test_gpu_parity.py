"""CUDA path vs the CPU oracle, through the C ABI (needs a B200)."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import check_exact, check_random_row

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


def run_gpu(L, inp, wl, *, mode=0, q_offset=None, num_splits=0):
    q = inp["q"].cuda()
    w = inp["w"].cuda()
    k = inp["k"].cuda()
    ks = None if inp["k_scale"] is None else inp["k_scale"].cuda()
    idx, sc = L.indexer_topk(q, w, k, k_scale=ks, m=wl.m, topk=wl.topk, causal=wl.causal,
                             mode=mode, q_offset=q_offset, num_splits=num_splits)
    torch.cuda.synchronize()
    assert L.csa_last_device_error(None) == L.CSA_OK
    return idx.cpu().numpy(), sc.cpu().numpy()


def run_oracle(inp, wl, *, mode=0, q_offset=None, rows=None):
    q, w, k, ks = workloads.as_numpy_bits(inp)
    return oracle.topk(q, w, k, ks, B=wl.B, S=wl.S, T=wl.T, H=wl.H, d=wl.d, m=wl.m,
                       topk=wl.topk, causal=wl.causal, mode=mode, q_offset=q_offset, rows=rows)


def exact_case(L, wl, *, mode=0, q_offset=None, num_splits=0, seed=None):
    inp = workloads.make_inputs(wl.replace(values="integer"), seed=seed)
    gi, gs = run_gpu(L, inp, wl, mode=mode, q_offset=q_offset, num_splits=num_splits)
    ri, rs, _, _ = run_oracle(inp, wl, mode=mode, q_offset=q_offset)
    check_exact(gi.reshape(-1, wl.topk), gs.reshape(-1, wl.topk), ri, rs, label=str(wl))


# ---------------------------------------------------------------- bit-exact (integer inputs)

def test_tiny_config_bit_exact(lib):
    """The tiny causal indexer workload, bit for bit."""
    exact_case(lib, workloads.CONFIGS["tiny"])


@pytest.mark.parametrize("H", [1, 2, 4, 8, 16, 32, 64, 128, 256])
def test_heads_bit_exact(lib, H):
    wl = workloads.Workload("h", B=1, S=300, T=333, H=H, d=64, m=1, topk=24, values="integer", seed=200 + H)
    exact_case(lib, wl)


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("m", [1, 2, 4])
def test_dims_bit_exact(lib, d, m):
    wl = workloads.Workload("d", B=2, S=517, T=261, H=64, d=d, m=m, topk=40, values="integer", seed=300 + d + m)
    exact_case(lib, wl)


@pytest.mark.parametrize("topk", [1, 7, 128, 300, 2048])
def test_topk_sizes_bit_exact(lib, topk):
    wl = workloads.Workload("k", B=1, S=700, T=2900, H=16, d=32, m=4, topk=topk, values="integer", seed=400 + topk)
    exact_case(lib, wl)


@pytest.mark.parametrize("causal", [True, False])
@pytest.mark.parametrize("mode", [0, 1])
def test_causal_and_gate_bit_exact(lib, causal, mode):
    wl = workloads.Workload("c", B=3, S=190, T=700, H=64, d=128, m=2, topk=100, causal=causal,
                            values="integer", seed=500 + 2 * causal + mode)
    exact_case(lib, wl, mode=mode)


@pytest.mark.parametrize("num_splits", [2, 3, 4])
def test_splits_bit_exact(lib, num_splits):
    wl = workloads.Workload("s", B=2, S=64, T=3000, H=64, d=128, m=4, topk=256, values="integer", seed=600 + num_splits)
    exact_case(lib, wl, num_splits=num_splits)


@pytest.mark.parametrize("q_offset", [0, 37, 11000, -60])
def test_q_offset_bit_exact(lib, q_offset):
    wl = workloads.Workload("o", B=1, S=129, T=2800, H=32, d=64, m=4, topk=64, values="integer", seed=700)
    exact_case(lib, wl, q_offset=q_offset)


def test_decode_shape_bit_exact(lib):
    """Few queries per sequence against many keys: split path plus merge."""
    wl = workloads.Workload("dec", B=4, S=3, T=9000, H=64, d=128, m=4, topk=512, values="integer", seed=800)
    exact_case(lib, wl)


def test_all_scores_tied(lib):
    """Every score equal (w = 0): the answer is the lowest visible indices."""
    wl = workloads.Workload("tie", B=1, S=260, T=600, H=64, d=128, m=1, topk=50, values="integer", seed=801)
    inp = workloads.make_inputs(wl)
    inp["w"].zero_()
    gi, gs = run_gpu(lib, inp, wl)
    ri, rs, _, _ = run_oracle(inp, wl)
    check_exact(gi.reshape(-1, wl.topk), gs.reshape(-1, wl.topk), ri, rs, label="ties")


def test_plain_entry_point(lib):
    """csa_indexer_topk (bf16, ReLU top-k, default offset) through raw pointers."""
    wl = workloads.CONFIGS["tiny"]
    inp = workloads.make_inputs(wl)
    q, w, k = inp["q"].cuda(), inp["w"].cuda(), inp["k"].cuda()
    idx = torch.empty((wl.B, wl.S, wl.topk), dtype=torch.int32, device="cuda")
    sc = torch.empty((wl.B, wl.S, wl.topk), dtype=torch.float32, device="cuda")
    st = lib.csa_indexer_topk(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(w.data_ptr()),
                              ctypes.c_void_p(k.data_ptr()), wl.B, wl.S, wl.T, wl.H, wl.d, wl.m,
                              wl.topk, 1, ctypes.c_void_p(idx.data_ptr()),
                              ctypes.c_void_p(sc.data_ptr()),
                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == lib.CSA_OK
    torch.cuda.synchronize()
    ri, rs, _, _ = run_oracle(inp, wl)
    check_exact(idx.cpu().numpy().reshape(-1, wl.topk), sc.cpu().numpy().reshape(-1, wl.topk), ri, rs)


# ---------------------------------------------------------------- edge cases

def test_no_keys(lib):
    wl = workloads.Workload("t0", B=2, S=5, T=0, H=4, d=32, m=4, topk=3, values="integer", seed=1)
    inp = workloads.make_inputs(wl)
    gi, gs = run_gpu(lib, inp, wl)
    assert np.all(gi == -1) and np.all(np.isneginf(gs))


def test_no_queries(lib):
    wl = workloads.Workload("s0", B=1, S=0, T=64, H=4, d=32, m=4, topk=3, values="integer", seed=1)
    inp = workloads.make_inputs(wl)
    gi, gs = run_gpu(lib, inp, wl)
    assert gi.size == 0


def test_rejects_bad_arguments(lib):
    wl = workloads.CONFIGS["tiny"]
    inp = workloads.make_inputs(wl)
    q, w, k = inp["q"].cuda(), inp["w"].cuda(), inp["k"].cuda()
    idx = torch.full((1, wl.S, wl.topk), 7, dtype=torch.int32, device="cuda")
    sc = torch.zeros((1, wl.S, wl.topk), dtype=torch.float32, device="cuda")
    a = lib.make_args(q, w, k, m=wl.m, topk=wl.topk, out_idx=idx, out_score=sc)
    a.H_I = 3
    assert lib.csa_indexer_topk_ex(a, None, 0, None) == lib.CSA_ERR_UNSUPPORTED
    a.H_I = wl.H
    a.topk = 4096
    assert lib.csa_indexer_topk_ex(a, None, 0, None) == lib.CSA_ERR_UNSUPPORTED
    a.topk = wl.topk
    a.mode = 9
    assert lib.csa_indexer_topk_ex(a, None, 0, None) == lib.CSA_ERR_INVALID_ARG
    a.mode = 0
    ws_need = lib.csa_indexer_workspace_size(a)
    assert ws_need > 0
    ws = torch.empty(ws_need - 256, dtype=torch.uint8, device="cuda")
    assert lib.csa_indexer_topk_ex(a, ctypes.c_void_p(ws.data_ptr()), ws.numel(), None) == lib.CSA_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert torch.all(idx == 7), "a rejected call must not touch the outputs"


def test_caller_workspace(lib):
    wl = workloads.CONFIGS["tiny"]
    inp = workloads.make_inputs(wl)
    q, w, k = inp["q"].cuda(), inp["w"].cuda(), inp["k"].cuda()
    a = lib.make_args(q, w, k, m=wl.m, topk=wl.topk)
    ws = torch.empty(lib.csa_indexer_workspace_size(a), dtype=torch.uint8, device="cuda")
    for _ in range(2):
        gi, gs = lib.indexer_topk(q, w, k, m=wl.m, topk=wl.topk, workspace=ws)
    torch.cuda.synchronize()
    ri, rs, _, _ = run_oracle(inp, wl)
    check_exact(gi.cpu().numpy().reshape(-1, wl.topk), gs.cpu().numpy().reshape(-1, wl.topk), ri, rs)


def test_wait_timeout_is_reported(lib):
    """A wait budget of one cycle makes the pipeline's waits run out: the
    kernel must record a timeout and exit cleanly, and the next call with the
    default budget must be correct again."""
    wl = workloads.CONFIGS["tiny"]
    inp = workloads.make_inputs(wl)
    q, w, k = inp["q"].cuda(), inp["w"].cuda(), inp["k"].cuda()
    lib.csa_set_wait_limit(1)
    try:
        lib.indexer_topk(q, w, k, m=wl.m, topk=wl.topk)
        st = lib.csa_last_device_error(None)
    finally:
        lib.csa_set_wait_limit(0)
    assert st == lib.CSA_ERR_TIMEOUT
    assert lib.csa_last_device_error(None) == lib.CSA_OK  # cleared
    exact_case(lib, wl)


# ---------------------------------------------------------------- random-normal inputs

def oracle_rows(q, w, k, ks, wl, rows):
    """The oracle's fp64 scores and visibility of each sampled row, computed
    on all host threads (the oracle's calls release the interpreter lock)."""
    import concurrent.futures
    import os

    def one(row):
        b, i = divmod(int(row), wl.S)
        return oracle.score_row(q, w, k, ks, B=wl.B, S=wl.S, T=wl.T, H=wl.H, d=wl.d, m=wl.m,
                                b=b, i=i, causal=wl.causal)

    with concurrent.futures.ThreadPoolExecutor(max_workers=os.cpu_count() or 4) as ex:
        return list(ex.map(one, rows))


def random_case(L, wl, rows, *, mode=0, rtol=1e-2, inp=None):
    if inp is None:
        inp = workloads.make_inputs(wl, device="cuda")
    gi, gs = run_gpu(L, inp, wl, mode=mode)
    q, w, k, ks = workloads.as_numpy_bits(inp)
    ri, _, _, rc = oracle.topk(q, w, k, ks, B=wl.B, S=wl.S, T=wl.T, H=wl.H, d=wl.d, m=wl.m,
                               topk=wl.topk, causal=wl.causal, mode=mode, rows=rows)
    gi = gi.reshape(-1, wl.topk)
    gs = gs.reshape(-1, wl.topk)
    recalls = []
    for n, (row, (I, vis)) in enumerate(zip(rows, oracle_rows(q, w, k, ks, wl, rows))):
        recalls.append(check_random_row(gi[row], gs[row], ri[n], rc[n], I, vis, topk=wl.topk,
                                        gate=mode == 1, rtol=rtol, label=f"{wl.name} row {row}"))
    return recalls


def sample_rows(wl, n, seed=0, heavy=4):
    """n random query rows, plus the first and last rows of the first and
    last sequences and the last `heavy` rows of the last sequence (the
    heaviest query block: the most visible keys)."""
    rng = np.random.default_rng(seed)
    last = wl.B * wl.S
    rows = np.unique(np.concatenate([rng.integers(0, last, n),
                                     [0, last - 1, wl.S - 1],
                                     np.arange(max(0, last - heavy), last)]))
    return rows.astype(np.int64)


def exact_sampled_case(L, wl, rows, *, mode=0):
    """Integer-valued inputs at any size: the GPU's rows must equal the
    oracle's bit for bit on the sampled rows."""
    inp = workloads.make_inputs(wl.replace(values="integer"), device="cuda")
    gi, gs = run_gpu(L, inp, wl, mode=mode)
    ri, rs, _, _ = run_oracle(inp, wl, mode=mode, rows=rows)
    check_exact(gi.reshape(-1, wl.topk)[rows], gs.reshape(-1, wl.topk)[rows], ri, rs,
                label=f"{wl.name} (integer, {len(rows)} sampled rows)")


def test_random_small_recall(lib):
    wl = workloads.Workload("r", B=2, S=1000, T=1000, H=64, d=128, m=1, topk=256, seed=900)
    random_case(lib, wl, sample_rows(wl, 40))


def test_random_gate(lib):
    wl = workloads.Workload("g", B=1, S=777, T=2000, H=64, d=128, m=2, topk=300, seed=901)
    random_case(lib, wl, sample_rows(wl, 30), mode=1)


def test_random_long_ranges(lib):
    """Decode-sized batches over long key ranges (random normal): items of
    about 15,000 keys whose k-th score often shares its quarter-binade histogram
    bucket with more than the candidate list holds, so the selector refines
    that bucket by a second histogram level; the select kernel merges three
    lists per query through its (two-level) prefilter."""
    wl = workloads.Workload("rlong", B=4, S=600, T=45000, H=64, d=128, m=4, topk=2048, seed=1900)
    recalls = random_case(lib, wl, sample_rows(wl, 24, seed=19))
    assert min(recalls) >= 0.999


@pytest.mark.slow
def test_dsa_prefill_full_size(lib):
    """DSA-style uncompressed prefill at its full size, 256+ sampled queries."""
    wl = workloads.CONFIGS["dsa_prefill"]
    random_case(lib, wl, sample_rows(wl, 256, seed=1))


@pytest.mark.slow
def test_v4flash_prefill_full_size(lib):
    """V4-Flash-shaped prefill at its full size (S=65,536, T=16,384), 256+ sampled queries."""
    wl = workloads.CONFIGS["v4flash_prefill"]
    random_case(lib, wl, sample_rows(wl, 256, seed=2))


@pytest.mark.slow
def test_dsa_prefill_integer_full_size(lib):
    """Integer-valued inputs at the full DSA prefill size (S=T=8192, top-2048):
    every key of the 8192-key items goes through the selector's histogram
    levels and near-tie cut with dense exact ties, and the GPU must match the
    oracle bit for bit on 512+ sampled rows."""
    wl = workloads.CONFIGS["dsa_prefill"]
    exact_sampled_case(lib, wl, sample_rows(wl, 512, seed=11))


@pytest.mark.slow
def test_v4flash_prefill_integer_full_size(lib):
    """Integer-valued inputs at the full V4-Flash prefill size (items of up
    to 16,384 keys), bit for bit on 512+ sampled rows."""
    wl = workloads.CONFIGS["v4flash_prefill"]
    exact_sampled_case(lib, wl, sample_rows(wl, 512, seed=12))
