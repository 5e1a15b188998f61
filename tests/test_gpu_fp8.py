"""E4M3 keys with per-key fp32 scales: CUDA path vs the CPU oracle (needs a B200).

The oracle reads the exact dequantised keys (scale * E4M3 value).  Integer
inputs use power-of-two scales, so every product and sum is exact in fp32
and the GPU must match bit for bit; random-normal inputs are judged by recall
and a 3e-2 relative score tolerance.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import check_random_row
from test_gpu_parity import exact_case, lib, random_case, run_gpu, run_oracle, sample_rows  # noqa: F401

pytestmark = pytest.mark.gpu


def fp8(wl):
    return wl.replace(key_fp8=True)


@pytest.mark.parametrize("H", [1, 4, 16, 32, 64, 128, 256])
def test_fp8_heads_bit_exact(lib, H):
    wl = workloads.Workload("f8h", B=2, S=300, T=700, H=H, d=128, m=2, topk=100, seed=1200 + H)
    exact_case(lib, fp8(wl))


@pytest.mark.parametrize("d", [32, 64, 128])
@pytest.mark.parametrize("m", [1, 4])
def test_fp8_dims_bit_exact(lib, d, m):
    wl = workloads.Workload("f8d", B=1, S=520, T=900, H=64, d=d, m=m, topk=160, seed=1300 + d + m)
    exact_case(lib, fp8(wl))


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("causal", [True, False])
def test_fp8_gate_and_causal_bit_exact(lib, mode, causal):
    wl = workloads.Workload("f8g", B=1, S=400, T=1500, H=64, d=128, m=4, topk=200, causal=causal,
                            seed=1400 + mode + 2 * causal)
    exact_case(lib, fp8(wl), mode=mode)


def test_fp8_decode_splits_bit_exact(lib):
    """Few queries per sequence against many keys: key-range splits, then the
    select merges the splits' lists."""
    wl = workloads.Workload("f8s", B=3, S=2, T=20000, H=64, d=128, m=4, topk=512, seed=1500)
    exact_case(lib, fp8(wl))


def test_fp8_single_query_bit_exact(lib):
    """One query per sequence and 64 heads (N = 64): both epilogue warpgroups
    take alternate groups of key tiles that share an accumulator slot."""
    wl = workloads.Workload("f8one", B=5, S=1, T=3000, H=64, d=128, m=4, topk=300, seed=1550)
    exact_case(lib, fp8(wl))


def test_fp8_scales_and_subnormals(lib):
    """Keys drawn from every finite E4M3 code (subnormals, zeros of both signs,
    the largest value) with scales spanning many binades: the GPU must decode
    every code and apply every scale as the oracle does.  The sums need more
    than fp32's 24 bits here, so scores are held to 1e-5 relative."""
    wl = fp8(workloads.Workload("f8c", B=1, S=130, T=256, H=32, d=128, m=1, topk=64,
                                values="integer", seed=1600))
    inp = workloads.make_inputs(wl)
    codes = torch.arange(256, dtype=torch.int32)
    finite = codes[(codes & 0x7F) != 0x7F].to(torch.uint8)          # drop the NaN codes
    g = torch.Generator().manual_seed(1601)
    inp["k"] = finite[torch.randint(0, finite.numel(), (1, wl.T, wl.d), generator=g)].contiguous()
    inp["k_scale"] = torch.pow(2.0, torch.randint(-8, 6, (1, wl.T), generator=g).float())
    gi, gs = run_gpu(lib, inp, wl)
    rows = np.arange(wl.S, dtype=np.int64)
    check_rows(inp, wl, gi, gs, rows, rtol=1e-5)


def test_fp8_query_split_wide_range(lib):
    """The tensor core takes each bf16 query row as sigma * (hi8 + lo8), two
    E4M3 pieces.  Query elements spread over 18 binades put most of them on
    the second piece (and some below E4M3's grid): the scores must still match
    the exact fp64 scores to 2e-4 relative, which fails if lo8 were dropped or
    mis-scaled (errors of order 2^-5 of each element)."""
    wl = fp8(workloads.Workload("f8w", B=1, S=300, T=2500, H=64, d=128, m=1, topk=256, seed=1650))
    inp = workloads.make_inputs(wl)
    g = torch.Generator().manual_seed(1651)
    shape = inp["q"].shape
    mag = torch.pow(2.0, torch.empty(shape).uniform_(-14.0, 4.0, generator=g))
    sign = torch.where(torch.rand(shape, generator=g) < 0.5, -1.0, 1.0)
    inp["q"] = (sign * mag).to(torch.bfloat16)
    gi, gs = run_gpu(lib, inp, wl)
    rows = np.arange(0, wl.S, 7, dtype=np.int64)
    check_rows(inp, wl, gi, gs, rows, rtol=2e-4)


def check_rows(inp, wl, gi, gs, rows, *, mode=0, rtol):
    q, w, k, ks = workloads.as_numpy_bits(inp)
    ri, _, _, rc = oracle.topk(q, w, k, ks, B=wl.B, S=wl.S, T=wl.T, H=wl.H, d=wl.d, m=wl.m,
                               topk=wl.topk, causal=wl.causal, mode=mode, rows=rows)
    gi = gi.reshape(-1, wl.topk)
    gs = gs.reshape(-1, wl.topk)
    for n, row in enumerate(rows):
        b, i = divmod(int(row), wl.S)
        I, vis = oracle.score_row(q, w, k, ks, B=wl.B, S=wl.S, T=wl.T, H=wl.H, d=wl.d, m=wl.m,
                                  b=b, i=i, causal=wl.causal)
        check_random_row(gi[row], gs[row], ri[n], rc[n], I, vis, topk=wl.topk, gate=mode == 1,
                         rtol=rtol, label=f"{wl.name} row {row}")


def test_fp8_random_recall(lib):
    wl = workloads.Workload("f8r", B=2, S=900, T=1200, H=64, d=128, m=1, topk=256, seed=1700)
    random_case(lib, fp8(wl), sample_rows(wl, 40), rtol=3e-2)


def test_fp8_random_gate(lib):
    wl = workloads.Workload("f8q", B=1, S=700, T=2400, H=64, d=128, m=2, topk=300, seed=1701)
    random_case(lib, fp8(wl), sample_rows(wl, 30), mode=1, rtol=3e-2)


@pytest.mark.slow
def test_long_prefill_fp8_full_size(lib):
    """Long prefill (S=262,144, T=65,536, E4M3 keys) at full size, 256+ sampled queries."""
    wl = workloads.CONFIGS["long_prefill_fp8"]
    random_case(lib, wl, sample_rows(wl, 256, seed=3), rtol=3e-2)


@pytest.mark.slow
def test_long_prefill_fp8_gated_full_size(lib):
    wl = workloads.CONFIGS["long_prefill_fp8_gated"]
    random_case(lib, wl, sample_rows(wl, 256, seed=4), mode=1, rtol=3e-2)


@pytest.mark.slow
def test_decode_fp8_full_size(lib):
    """Batched decode (B=32 x 64 queries at T=131,072, E4M3 keys), 256+ sampled queries."""
    wl = workloads.CONFIGS["decode_fp8"]
    random_case(lib, wl, sample_rows(wl, 256, seed=5), rtol=3e-2)


@pytest.mark.slow
def test_decode1_fp8_full_size(lib):
    """One query per sequence (B=32, T=131,072, E4M3 keys), every query."""
    wl = workloads.CONFIGS["decode1_fp8"]
    random_case(lib, wl, np.arange(wl.B * wl.S, dtype=np.int64), rtol=3e-2)


# ---------------------------------------------------------------- one-piece E4M3 query
# With query_pieces = 1 each bf16 query row meets the E4M3 keys as one E4M3
# rounding sigma * hi8 (half the tensor work of the exact two-piece split).
# Integer-valued queries are exact in one piece, so those cases stay bit-exact;
# random-normal queries lose up to 2^-4 relative per element, which the
# accuracy bars of the two-piece path do not allow for: the random test
# measures and records recall and score error against the oracle's exact
# scores and holds them to the looser bar this mode documents.

def one_piece_case(L, wl, *, mode=0):
    inp = workloads.make_inputs(wl.replace(values="integer"))
    q = inp["q"].cuda()
    w = inp["w"].cuda()
    k = inp["k"].cuda()
    ks = inp["k_scale"].cuda()
    idx, sc = L.indexer_topk(q, w, k, k_scale=ks, m=wl.m, topk=wl.topk, causal=wl.causal,
                             mode=mode, query_pieces=1)
    torch.cuda.synchronize()
    assert L.csa_last_device_error(None) == L.CSA_OK
    from parity import check_exact

    ri, rs, _, _ = run_oracle(inp, wl, mode=mode)
    check_exact(idx.cpu().numpy().reshape(-1, wl.topk), sc.cpu().numpy().reshape(-1, wl.topk),
                ri, rs, label=f"{wl.name} one-piece")


@pytest.mark.parametrize("d", [32, 64, 128])
def test_one_piece_query_integer_bit_exact(lib, d):
    wl = workloads.Workload("f8p1", B=2, S=300, T=900, H=64, d=d, m=2, topk=120, seed=1800 + d,
                            key_fp8=True)
    one_piece_case(lib, wl)


def test_one_piece_query_gate_and_splits_bit_exact(lib):
    one_piece_case(lib, workloads.Workload("f8p1g", B=1, S=400, T=1500, H=64, d=128, m=4,
                                           topk=200, seed=1810, key_fp8=True), mode=1)
    one_piece_case(lib, workloads.Workload("f8p1s", B=3, S=2, T=20000, H=64, d=128, m=4,
                                           topk=512, seed=1811, key_fp8=True))


def one_piece_recall(L, wl, rows):
    """Recall and worst score error of the one-piece query on random inputs,
    per sampled row, against the oracle's exact fp64 scores."""
    from test_gpu_parity import oracle_rows

    inp = workloads.make_inputs(wl, device="cuda")
    idx, sc = L.indexer_topk(inp["q"], inp["w"], inp["k"], k_scale=inp["k_scale"], m=wl.m,
                             topk=wl.topk, causal=wl.causal, query_pieces=1)
    torch.cuda.synchronize()
    assert L.csa_last_device_error(None) == L.CSA_OK
    q, w, k, ks = workloads.as_numpy_bits(inp)
    ri, _, _, rc = oracle.topk(q, w, k, ks, B=wl.B, S=wl.S, T=wl.T, H=wl.H, d=wl.d, m=wl.m,
                               topk=wl.topk, causal=wl.causal, rows=rows)
    gi = idx.cpu().numpy().reshape(-1, wl.topk)
    gs = sc.cpu().numpy().reshape(-1, wl.topk)
    recalls, errs = [], []
    for n, (row, (I, vis)) in enumerate(zip(rows, oracle_rows(q, w, k, ks, wl, rows))):
        cnt = int(rc[n])
        sel = gi[row][gi[row] >= 0]
        assert len(sel) == cnt and len(np.unique(sel)) == cnt and np.all(vis[sel])
        top = abs(I[ri[n][0]]) if cnt else 1.0       # the row's largest exact score
        errs.append(float(np.max(np.abs(gs[row][:cnt] - I[sel]) / np.maximum(np.abs(I[sel]), top)))
                    if cnt else 0.0)
        recalls.append(len(np.intersect1d(sel, ri[n][:cnt])) / cnt if cnt else 1.0)
    return np.array(recalls), np.array(errs)


@pytest.mark.slow
def test_one_piece_query_recall_long_prefill(lib):
    """The one-piece query on the long-prefill shape, 256+ sampled rows: the
    bar of this mode is mean recall >= 0.95 and every returned score within
    0.3 of its exact value (relative to the larger of that value and the
    row's top score: the head sum cancels, so one E4M3 rounding of q moves a
    score by a sizeable fraction of it); the exact-split default is the mode
    that meets recall >= 0.999."""
    wl = workloads.CONFIGS["long_prefill_fp8"]
    rows = sample_rows(wl, 256, seed=21)
    rec, err = one_piece_recall(lib, wl, rows)
    print(f"one-piece query, long_prefill_fp8: recall mean {rec.mean():.4f} min {rec.min():.4f}, "
          f"score error max {err.max():.3g} over {len(rows)} rows")
    assert rec.mean() >= 0.95 and err.max() <= 0.3


@pytest.mark.slow
def test_one_piece_query_recall_decode(lib):
    wl = workloads.CONFIGS["decode_fp8"]
    rows = sample_rows(wl, 256, seed=22)
    rec, err = one_piece_recall(lib, wl, rows)
    print(f"one-piece query, decode_fp8: recall mean {rec.mean():.4f} min {rec.min():.4f}, "
          f"score error max {err.max():.3g} over {len(rows)} rows")
    assert rec.mean() >= 0.95 and err.max() <= 0.3
