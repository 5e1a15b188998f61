"""Comparison of the CUDA path's output with the CPU oracle (test helper).

Two bars, as the method's accuracy targets state them:

* exact -- integer-valued inputs make every product and partial sum exact in
  fp32, so indices and scores must equal the oracle's bit for bit;
* random -- per query, the selected set must overlap the oracle's with
  recall >= 0.999, every returned score must lie within ``rtol`` of the fp64
  score of the key it names (relative to max(|that score|, |oracle's k-th
  score|, 1e-6)), the returned list must be ordered (score descending, equal
  scores by ascending index), indices visible and unique, and the count equal
  to the oracle's (ReLU top-k) or within the keys whose fp64 score is within
  ``rtol`` of zero (sigmoid gate).
"""
from __future__ import annotations

import numpy as np


def check_exact(gpu_idx, gpu_sc, ref_idx, ref_sc, label=""):
    gi = np.asarray(gpu_idx).reshape(ref_idx.shape)
    gs = np.asarray(gpu_sc).reshape(ref_sc.shape)
    bad = np.nonzero(~np.all(gi == ref_idx, axis=1))[0]
    assert bad.size == 0, f"{label}: index mismatch in {bad.size} rows, first row {bad[0]}: gpu {gi[bad[0]][:8]} ref {ref_idx[bad[0]][:8]}"
    same = (gs == ref_sc) | (np.isneginf(gs) & np.isneginf(ref_sc))
    bad = np.nonzero(~np.all(same, axis=1))[0]
    assert bad.size == 0, f"{label}: score mismatch in {bad.size} rows, first row {bad[0]}: gpu {gs[bad[0]][:8]} ref {ref_sc[bad[0]][:8]}"
    # bitwise: +0.0 vs -0.0 must agree as well
    assert np.array_equal(gs.view(np.uint32), ref_sc.view(np.uint32)), f"{label}: score bits differ"


def check_random_row(gi, gs, ri, rcount, I_row, vis, *, topk, gate=False, rtol=1e-2,
                     min_recall=0.999, label=""):
    """One query row: gi/gs GPU idx/score [topk]; ri oracle idx [topk]; rcount
    oracle count; I_row fp64 scores of every key of the row; vis its mask."""
    n = int(np.sum(gi >= 0))
    assert np.all(gi[:n] >= 0) and np.all(gi[n:] == -1), f"{label}: padding not at the end"
    assert np.all(np.isneginf(gs[n:])), f"{label}: padding scores not -inf"
    sel = gi[:n]
    assert len(np.unique(sel)) == n, f"{label}: duplicate indices"
    assert np.all(sel < len(vis)) and np.all(vis[sel]), f"{label}: invisible key returned"
    s = gs[:n]
    ordered = (s[:-1] > s[1:]) | ((s[:-1] == s[1:]) & (sel[:-1] < sel[1:]))
    assert np.all(ordered), f"{label}: output not ordered"
    ref = ri[:rcount]
    kth = abs(I_row[ref[-1]]) if rcount else 0.0
    denom = np.maximum(np.maximum(np.abs(I_row[sel]), kth), 1e-6)
    err = np.abs(s.astype(np.float64) - I_row[sel]) / denom
    assert np.all(err <= rtol), f"{label}: score error {err.max():.3g} > {rtol}"
    if gate:
        assert np.all(I_row[sel] > -rtol * max(kth, 1e-6)), f"{label}: gate passed a negative score"
        # keys only one side kept must be within rounding of zero or of the cut
        diff = np.setxor1d(sel, ref)
        near = (np.abs(I_row[diff]) <= rtol * max(kth, 1e-6)) | (np.abs(I_row[diff] - (I_row[ref[-1]] if rcount else 0)) <= rtol * max(kth, 1e-6))
        assert np.all(near), f"{label}: gate set differs beyond rounding"
    else:
        assert n == rcount, f"{label}: count {n} != oracle {rcount}"
    if rcount == 0:
        return 1.0
    recall = len(np.intersect1d(sel, ref)) / rcount
    assert recall >= min_recall, f"{label}: recall {recall:.5f} < {min_recall}"
    return recall
