"""Brute-force restatement of the indexer top-k for tiny shapes (test helper).

Independent of ``oracle/``: it decodes the input formats with torch's own
dtype conversions, materialises every score with numpy (fp64), derives
visibility from the token span a compressed key covers, applies the literal
sigmoid for the gate, and selects with Python's stable ``sorted``.
"""
from __future__ import annotations

import math

import numpy as np
import torch


def decode_bf16(bits: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.to(torch.float64).numpy()


def decode_e4m3(raw: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(raw).view(np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def key_tokens(s: int, m: int):
    """Tokens summarised by compressed key s."""
    return range(s * m, (s + 1) * m)


def brute_scores(q_bits, w, k, k_scale, b, i):
    """All I[t, s] of row (b, i) as float64, fully materialised."""
    q = decode_bf16(q_bits[b, i])                      # [H, d]
    if k_scale is None:
        kk = decode_bf16(k[b])                         # [T, d]
    else:
        kk = decode_e4m3(k[b]) * k_scale[b][:, None].astype(np.float64)
    logits = q @ kk.T                                  # [H, T]
    return (w[b, i].astype(np.float64)[:, None] * np.maximum(logits, 0.0)).sum(axis=0)


def brute_topk(q_bits, w, k, k_scale, *, B, S, T, H, d, m, topk, causal=True, gate=False,
               q_offset=0):
    idx = np.full((B * S, topk), -1, np.int32)
    sc = np.full((B * S, topk), -np.inf, np.float32)
    cnt = np.zeros((B * S,), np.int32)
    for b in range(B):
        for i in range(S):
            t = i + q_offset
            I = brute_scores(q_bits, w, k, k_scale, b, i)
            cand = [s for s in range(T) if not causal or max(key_tokens(s, m)) <= t]
            if gate:
                cand = [s for s in cand if 1.0 / (1.0 + math.exp(-I[s])) > 0.5]
            chosen = sorted(cand, key=lambda s: (-I[s], s))[:topk]
            r = b * S + i
            cnt[r] = len(chosen)
            for slot, s in enumerate(chosen):
                idx[r, slot] = s
                sc[r, slot] = np.float32(I[s])
    return idx, sc, cnt
