"""CPU oracle for the CSA lightning-indexer top-k step -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  The product path (``lightning_indexer_top_02_b200``)
never imports it and shares no code with it.

The arithmetic lives in ``csa_oracle.c`` (plain C, fp64 accumulation, OpenMP
over query rows); this module only compiles it with gcc and marshals numpy
arrays into it.  What it computes, with the passages it follows, is written
at the top of ``csa_oracle.c``:

* score ``I[t,s] = sum_h w[t,h] * ReLU(q[t,h,:] . k[s,:])`` -- "StreamIndex:
  Memory-Bounded Compressed Sparse Attention via Streaming Top-k", abstract
  (the lightning indexer scores compressed keys per query);
* causal visibility of compressed key ``s`` (tokens ``[s*m, (s+1)*m)``) for
  the query at absolute position ``t``: ``(s+1)*m - 1 <= t``;
* top-k by (score desc, index asc), or the sigmoid gate ``sigmoid(I) > 0.5``
  ("FlashMemory-DeepSeek-V4: Lightning Index Ultra-Long Context via Lookahead
  Sparse Attention", "What carries the argument") capped at k.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csa_oracle.c")
_LIB = os.path.join(_HERE, "libcsa_oracle.so")

KEY_BF16 = 0
KEY_E4M3 = 1
MODE_TOPK = 0
MODE_GATE = 1


def build(force: bool = False) -> str:
    """Compile ``csa_oracle.c`` into ``libcsa_oracle.so`` (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-fopenmp", "-std=c99", "-Wall", "-shared", "-fPIC",
             "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class Oracle:
    """ctypes view of one compiled oracle library (the default one, or a copy
    the tests compile with a planted mistake to check that the pins catch it)."""

    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        P = ctypes.c_void_p
        I = ctypes.c_int
        LL = ctypes.c_longlong
        lib.csa_oracle_topk.argtypes = [P, P, P, P, I, I, I, I, I, I, I, I, I, I, LL,
                                        P, LL, P, P, P, P]
        lib.csa_oracle_topk.restype = I
        lib.csa_oracle_score_row.argtypes = [P, P, P, P, I, I, I, I, I, I, I, I, LL,
                                             I, LL, P, P]
        lib.csa_oracle_score_row.restype = I
        lib.csa_oracle_bf16_value.argtypes = [ctypes.c_uint16]
        lib.csa_oracle_bf16_value.restype = ctypes.c_double
        lib.csa_oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        lib.csa_oracle_e4m3_value.restype = ctypes.c_double
        lib.csa_oracle_num_threads.argtypes = []
        lib.csa_oracle_num_threads.restype = I
        self.lib = lib

    def topk(self, q_bits, w, k, k_scale, *, B, S, T, H, d, m, topk, causal=True,
             mode=MODE_TOPK, q_offset=None, rows=None):
        """Run the oracle.

        q_bits: uint16 [B,S,H,d] (bfloat16 bits); w: float32 [B,S,H];
        k: uint16 [B,T,d] (bf16 bits) or uint8 [B,T,d] (E4M3 bytes, then
        k_scale float32 [B,T] is required); rows: optional int64 flat row ids
        b*S+i.  Returns (idx int32 [n,topk], score float32 [n,topk], score64
        float64 [n,topk], count int32 [n]).
        """
        key_fmt = KEY_E4M3 if k_scale is not None else KEY_BF16
        q_bits = _c(q_bits, np.uint16)
        w = _c(w, np.float32)
        k = _c(k, np.uint8 if key_fmt == KEY_E4M3 else np.uint16)
        k_scale = _c(k_scale, np.float32)
        if q_offset is None:
            q_offset = default_q_offset(S, T, m)
        if rows is not None:
            rows = _c(rows, np.int64)
            n = rows.shape[0]
        else:
            n = B * S
        idx = np.empty((n, topk), np.int32)
        sc = np.empty((n, topk), np.float32)
        sc64 = np.empty((n, topk), np.float64)
        cnt = np.empty((n,), np.int32)
        rc = self.lib.csa_oracle_topk(_ptr(q_bits), _ptr(w), _ptr(k), _ptr(k_scale), key_fmt,
                                      B, S, T, H, d, m, topk, int(bool(causal)), int(mode),
                                      int(q_offset), _ptr(rows), n, _ptr(idx), _ptr(sc),
                                      _ptr(sc64), _ptr(cnt))
        if rc != 0:
            raise ValueError(f"oracle rejected its arguments (code {rc})")
        return idx, sc, sc64, cnt

    def score_row(self, q_bits, w, k, k_scale, *, B, S, T, H, d, m, b, i, causal=True,
                  q_offset=None):
        """All fp64 scores I[t,s] of query row (b, i) and the visibility mask."""
        key_fmt = KEY_E4M3 if k_scale is not None else KEY_BF16
        q_bits = _c(q_bits, np.uint16)
        w = _c(w, np.float32)
        k = _c(k, np.uint8 if key_fmt == KEY_E4M3 else np.uint16)
        k_scale = _c(k_scale, np.float32)
        if q_offset is None:
            q_offset = default_q_offset(S, T, m)
        out = np.empty((T,), np.float64)
        vis = np.empty((T,), np.int32)
        rc = self.lib.csa_oracle_score_row(_ptr(q_bits), _ptr(w), _ptr(k), _ptr(k_scale),
                                           key_fmt, B, S, T, H, d, m, int(bool(causal)),
                                           int(q_offset), b, i, _ptr(out), _ptr(vis))
        if rc != 0:
            raise ValueError(f"oracle rejected its arguments (code {rc})")
        return out, vis.astype(bool)

    def bf16_value(self, bits: int) -> float:
        return self.lib.csa_oracle_bf16_value(bits)

    def e4m3_value(self, byte: int) -> float:
        return self.lib.csa_oracle_e4m3_value(byte)

    def num_threads(self) -> int:
        return self.lib.csa_oracle_num_threads()


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def default_q_offset(S: int, T: int, m: int) -> int:
    """Bottom-right alignment: the last query sits at the last token the keys cover."""
    return max(0, T * m - S)


_default = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def topk(*args, **kw):
    return default().topk(*args, **kw)


def score_row(*args, **kw):
    return default().score_row(*args, **kw)


def bf16_value(bits: int) -> float:
    return default().bf16_value(bits)


def e4m3_value(byte: int) -> float:
    return default().e4m3_value(byte)


def num_threads() -> int:
    return default().num_threads()
