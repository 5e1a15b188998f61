"""Pins for the CPU oracle: checks against facts fixed outside the oracle.

Each ``pin_*`` takes an ``oracle.Oracle`` and raises AssertionError when the
oracle disagrees with a hand-worked example, a closed form, an exact integer
re-derivation, a library routine on a special case, or the brute-force
restatement in ``brute.py``.  ``test_oracle.py`` runs them against the real
oracle; ``test_oracle_mutants.py`` runs them against copies with planted
mistakes and requires every mistake to be caught.
"""
from __future__ import annotations

import json
import os

import numpy as np
import torch

from brute import brute_scores, brute_topk, decode_bf16, decode_e4m3

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


# ---------------------------------------------------------------------------
# small input builders (numpy; bf16 bit patterns via torch's RNE cast)

def bf16_bits(x) -> np.ndarray:
    t = torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def e4m3_bytes(x) -> np.ndarray:
    t = torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.float8_e4m3fn)
    return t.view(torch.uint8).numpy()


def rand_case(rng, B, S, T, H, d, *, values="normal", fp8=False):
    if values == "integer":
        q = rng.integers(-4, 5, (B, S, H, d)) / 4.0
        k = rng.integers(-4, 5, (B, T, d)) / 4.0
        w = rng.choice([-1, -0.5, -0.25, 0.25, 0.5, 1.0], (B, S, H))
    elif values == "nonneg":
        q = rng.integers(0, 5, (B, S, H, d)) / 4.0
        k = rng.integers(0, 5, (B, T, d)) / 4.0
        w = rng.choice([-1, -0.5, -0.25, 0.25, 0.5, 1.0], (B, S, H))
    else:
        q = rng.standard_normal((B, S, H, d))
        k = rng.standard_normal((B, T, d))
        w = rng.standard_normal((B, S, H)) / np.sqrt(H)
    qb = bf16_bits(q)
    w = w.astype(np.float32)
    if fp8:
        amax = np.abs(k).max(axis=-1)
        scale = np.where(amax > 0, amax / 448.0, 1.0).astype(np.float32)
        kb = e4m3_bytes(k / scale[..., None])
        return qb, w, kb, scale
    return qb, w, bf16_bits(k), None


def shape_kw(B, S, T, H, d, m, topk):
    return dict(B=B, S=S, T=T, H=H, d=d, m=m, topk=topk)


# ---------------------------------------------------------------------------
# pins

def pin_hand_worked(orc):
    g = json.load(open(os.path.join(GOLDEN, "hand_worked.json")))
    sh = g["shape"]
    q = bf16_bits(np.array(g["q"], np.float32)[None])
    k = bf16_bits(np.array(g["k"], np.float32)[None])
    w = np.array(g["w"], np.float32)[None]
    kw = dict(B=sh["B"], S=sh["S"], T=sh["T"], H=sh["H"], d=sh["d"], m=sh["m"],
              topk=sh["topk"], q_offset=sh["q_offset"])
    for mode, key in ((0, "expect_topk"), (1, "expect_gate")):
        idx, sc, _, cnt = orc.topk(q, w, k, None, mode=mode, **kw)
        exp_idx = np.array(g[key]["idx"])
        exp_sc = np.array([[-np.inf if v is None else v for v in row] for row in g[key]["score"]],
                          np.float32)
        assert np.array_equal(idx, exp_idx), (key, idx, exp_idx)
        assert np.array_equal(sc, exp_sc), (key, sc, exp_sc)
        assert np.array_equal(cnt, (exp_idx >= 0).sum(1)), (key, cnt)
    idx, sc, _, _ = orc.topk(q, w, k, None, causal=False, **kw)
    assert list(idx[0]) == g["expect_noncausal_row0"]["idx"], idx[0]
    assert list(sc[0]) == g["expect_noncausal_row0"]["score"], sc[0]


def pin_decoders(orc):
    # E4M3: every byte against torch's float8_e4m3fn conversion, plus values
    # fixed by the format definition.
    allb = np.arange(256, dtype=np.uint8)
    ref = decode_e4m3(allb)
    got = np.array([orc.e4m3_value(int(b)) for b in allb])
    both_nan = np.isnan(ref) & np.isnan(got)
    assert np.array_equal(ref[~both_nan], got[~both_nan]), "E4M3 decode differs from torch"
    assert both_nan.sum() == 2 and np.isnan(got).sum() == 2  # S.1111.111 only
    assert orc.e4m3_value(0x7E) == 448.0 and orc.e4m3_value(0x01) == 2.0 ** -9
    assert orc.e4m3_value(0x08) == 2.0 ** -6 and orc.e4m3_value(0x38) == 1.0
    assert orc.e4m3_value(0xB8) == -1.0 and orc.e4m3_value(0x07) == 7 * 2.0 ** -9
    # bf16: a sweep of bit patterns against torch
    bits = np.concatenate([np.arange(0, 65536, 97, dtype=np.uint32),
                           [0x0000, 0x8000, 0x3F80, 0xBF80, 0x0001, 0x7F7F]]).astype(np.uint16)
    ref = decode_bf16(bits)
    got = np.array([orc.bf16_value(int(b)) for b in bits])
    fin = np.isfinite(ref)
    assert np.array_equal(ref[fin], got[fin]), "bf16 decode differs from torch"


def pin_brute_small(orc):
    rng = np.random.default_rng(7)
    cases = []
    for m in (1, 2, 4):
        for H in (1, 2, 4):
            for topk in (1, 7, 40):
                for causal in (True, False):
                    cases.append((m, H, topk, causal))
    for n, (m, H, topk, causal) in enumerate(cases):
        B, S, T, d = 2, 9, 11, 8
        values = ("integer", "normal")[n % 2]
        fp8 = n % 3 == 0
        q, w, k, ks = rand_case(rng, B, S, T, H, d, values=values, fp8=fp8)
        q_off = (0, 5, max(0, T * m - S))[n % 3]
        for gate in (False, True):
            bi, bs, bc = brute_topk(q, w, k, ks, B=B, S=S, T=T, H=H, d=d, m=m, topk=topk,
                                    causal=causal, gate=gate, q_offset=q_off)
            oi, os_, _, oc = orc.topk(q, w, k, ks, B=B, S=S, T=T, H=H, d=d, m=m, topk=topk,
                                      causal=causal, mode=int(gate), q_offset=q_off)
            ctx = dict(m=m, H=H, topk=topk, causal=causal, gate=gate, values=values, fp8=fp8)
            assert np.array_equal(oc, bc), ("count", ctx)
            assert np.array_equal(oi, bi), ("idx", ctx)
            if values == "integer":
                assert np.array_equal(os_, bs), ("score", ctx)
            else:
                np.testing.assert_allclose(os_, bs, rtol=1e-6, atol=1e-9)


def pin_integer_exact(orc):
    """Integer inputs: 64*I equals an int64 re-derivation exactly."""
    rng = np.random.default_rng(11)
    B, S, T, H, d, m = 1, 40, 12, 4, 32, 4
    a = rng.integers(-4, 5, (B, S, H, d))
    c = rng.integers(-4, 5, (B, T, d))
    e = rng.choice([-4, -2, -1, 1, 2, 4], (B, S, H))  # 4*w
    q, k, w = bf16_bits(a / 4.0), bf16_bits(c / 4.0), (e / 4.0).astype(np.float32)
    for i in (3, 17, 39):
        I, vis = orc.score_row(q, w, k, None, B=B, S=S, T=T, H=H, d=d, m=m, b=0, i=i,
                               q_offset=0)
        dots = a[0, i] @ c[0].T                       # int64 [H, T]
        exact64 = (e[0, i][:, None] * np.maximum(dots, 0)).sum(axis=0)
        assert np.array_equal(I * 64.0, exact64.astype(np.float64)), i
        assert np.array_equal(vis, (np.arange(T) + 1) * m - 1 <= i), i


def pin_relu_inactive(orc):
    """q, k >= 0: every logit is >= 0 so I = k . (sum_h w_h q_h); compare with a
    library matmul and numpy's stable argsort (exact on these integer values)."""
    rng = np.random.default_rng(13)
    B, S, T, H, d, m, topk = 1, 16, 48, 4, 16, 1, 9
    q, w, k, _ = rand_case(rng, B, S, T, H, d, values="nonneg")
    qf, kf = decode_bf16(q), decode_bf16(k)
    oi, osc, _, _ = orc.topk(q, w, k, None, causal=False, q_offset=0,
                             **shape_kw(B, S, T, H, d, m, topk))
    for i in range(S):
        v = w[0, i].astype(np.float64) @ qf[0, i]     # [d]
        I = kf[0] @ v                                 # [T]
        order = np.argsort(-I, kind="stable")[:topk]
        assert np.array_equal(oi[i], order), i
        assert np.array_equal(osc[i], I[order].astype(np.float32)), i


def pin_closed_form(orc):
    """H=1, w=1, q=e_0, k[s,0] = (perm[s]+1)/64: I[t,s] = (perm[s]+1)/64, so the
    answer is the visible keys ordered by perm, largest first."""
    rng = np.random.default_rng(17)
    B, S, T, H, d, m, topk = 1, 50, 40, 1, 16, 2, 6
    perm = rng.permutation(T)
    q = np.zeros((B, S, H, d)); q[..., 0] = 1.0
    k = np.zeros((B, T, d)); k[0, :, 0] = (perm + 1) / 64.0; k[0, :, 1:] = 0.25 * rng.integers(-4, 5, (T, d - 1))
    w = np.ones((B, S, H), np.float32)
    for q_off in (0, 7):
        oi, osc, _, oc = orc.topk(bf16_bits(q), w, bf16_bits(k), None, q_offset=q_off,
                                  **shape_kw(B, S, T, H, d, m, topk))
        for i in range(S):
            nvis = min(T, (i + q_off + 1) // m)
            want = sorted(range(nvis), key=lambda s: -perm[s])[:topk]
            assert list(oi[i][: len(want)]) == want, (q_off, i)
            assert oc[i] == min(topk, nvis), (q_off, i)
            assert np.array_equal(osc[i][: len(want)], ((perm[want] + 1) / 64.0).astype(np.float32))


def pin_counts(orc):
    """m=1, causal, T=S: query t sees t+1 keys; with an offset the count is
    min(k, T, floor((t+1)/m))."""
    rng = np.random.default_rng(19)
    B, S, T, H, d, topk = 1, 30, 30, 2, 8, 12
    q, w, k, _ = rand_case(rng, B, S, T, H, d)
    _, _, _, cnt = orc.topk(q, w, k, None, q_offset=0, **shape_kw(B, S, T, H, d, 1, topk))
    assert np.array_equal(cnt, np.minimum(topk, np.arange(S) + 1))
    for m, q_off in ((4, 0), (4, 90), (3, 11)):
        _, _, _, cnt = orc.topk(q, w, k, None, q_offset=q_off, **shape_kw(B, S, T, H, d, m, topk))
        t = np.arange(S) + q_off
        assert np.array_equal(cnt, np.minimum(topk, np.minimum(T, (t + 1) // m))), (m, q_off)


def pin_gate(orc):
    rng = np.random.default_rng(23)
    B, S, T, H, d, m, topk = 1, 20, 24, 4, 16, 1, 10
    q, w, k, _ = rand_case(rng, B, S, T, H, d)
    kw = shape_kw(B, S, T, H, d, m, topk)
    # all weights negative: every I <= 0, nothing passes sigmoid(I) > 0.5
    _, _, _, cnt = orc.topk(q, -np.abs(w), k, None, mode=1, q_offset=0, **kw)
    assert cnt.sum() == 0
    # all of q, k, w positive: every visible I > 0, the gate equals plain top-k
    qp, kp, wp = bf16_bits(np.abs(decode_bf16(q)) + 0.125), bf16_bits(np.abs(decode_bf16(k)) + 0.125), np.abs(w) + 0.01
    a = orc.topk(qp, wp, kp, None, mode=1, q_offset=0, **kw)
    b = orc.topk(qp, wp, kp, None, mode=0, q_offset=0, **kw)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
    # the gate keeps exactly the positive-score visible keys (capped)
    for i in (0, 9, 19):
        I, vis = orc.score_row(q, w, k, None, b=0, i=i, q_offset=0,
                               **{x: kw[x] for x in ("B", "S", "T", "H", "d", "m")})
        n_pos = int(((I > 0) & vis).sum())
        g = orc.topk(q, w, k, None, mode=1, q_offset=0, rows=np.array([i]), **kw)
        assert g[3][0] == min(topk, n_pos), i


def check_invariants(orc, q, w, k, ks, kw, mode=0, q_offset=None, rows=None):
    """Invariants every correct result satisfies; returns nothing, asserts."""
    idx, sc, sc64, cnt = orc.topk(q, w, k, ks, mode=mode, q_offset=q_offset, rows=rows, **kw)
    B, S, T, m, topk = kw["B"], kw["S"], kw["T"], kw["m"], kw["topk"]
    rows = np.arange(B * S) if rows is None else rows
    for r, row in enumerate(rows):
        b, i = divmod(int(row), S)
        I, vis = orc.score_row(q, w, k, ks, b=b, i=i, q_offset=q_offset,
                               **{x: kw[x] for x in ("B", "S", "T", "H", "d", "m")})
        n = cnt[r]
        sel = idx[r, :n]
        assert np.all(idx[r, n:] == -1) and np.all(sc[r, n:] == -np.inf)
        assert len(set(sel.tolist())) == n and np.all(vis[sel])
        eligible = vis & (I > 0) if mode == 1 else vis
        assert n == min(topk, int(eligible.sum()))
        assert np.array_equal(sc64[r, :n], I[sel]) and np.array_equal(sc[r, :n], I[sel].astype(np.float32))
        s64 = sc64[r, :n]
        assert np.all((s64[:-1] > s64[1:]) | ((s64[:-1] == s64[1:]) & (sel[:-1] < sel[1:])))
        if n:
            last, last_i = s64[-1], sel[-1]
            rest = np.setdiff1d(np.nonzero(eligible)[0], sel)
            assert np.all((I[rest] < last) | ((I[rest] == last) & (rest > last_i)))


def pin_invariants(orc):
    rng = np.random.default_rng(29)
    B, S, T, H, d, m, topk = 2, 24, 20, 4, 16, 2, 8
    for fp8 in (False, True):
        for values in ("normal", "integer"):
            q, w, k, ks = rand_case(rng, B, S, T, H, d, values=values, fp8=fp8)
            kw = shape_kw(B, S, T, H, d, m, topk)
            for mode in (0, 1):
                check_invariants(orc, q, w, k, ks, kw, mode=mode, q_offset=3)


def pin_rows_subset(orc):
    """Computing a subset of rows gives the same rows as computing all of them."""
    rng = np.random.default_rng(31)
    B, S, T, H, d, m, topk = 3, 10, 12, 2, 8, 2, 5
    q, w, k, ks = rand_case(rng, B, S, T, H, d, fp8=True)
    kw = shape_kw(B, S, T, H, d, m, topk)
    full = orc.topk(q, w, k, ks, q_offset=1, **kw)
    rows = np.array([29, 0, 13, 13, 7])
    part = orc.topk(q, w, k, ks, q_offset=1, rows=rows, **kw)
    for a, b in zip(full, part):
        assert np.array_equal(a[rows], b, equal_nan=a.dtype.kind == "f")


ALL_PINS = [pin_hand_worked, pin_decoders, pin_brute_small, pin_integer_exact,
            pin_relu_inactive, pin_closed_form, pin_counts, pin_gate, pin_invariants,
            pin_rows_subset]
