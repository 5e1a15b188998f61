"""CPU oracle of the sparse-attention step that consumes the indexer's
selection -- TEST INFRASTRUCTURE.

Only ``tests/`` and ``bench.py``'s CPU-baseline leg may import this module;
the product path never does.  The arithmetic lives in ``csa_attn_oracle.c``
(plain C, fp64, OpenMP over query rows), whose header states what it computes
and which passage it follows; this module compiles it with gcc and marshals
numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "csa_attn_oracle.c")
_LIB = os.path.join(_HERE, "libcsa_attn_oracle.so")


def build(force: bool = False, src: str = _SRC, lib: str = _LIB) -> str:
    """Compile the attention oracle into a shared library (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(lib) or os.path.getmtime(lib) < os.path.getmtime(src):
        tmp = lib + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-std=c99", "-Wall", "-shared", "-fPIC",
                               "-o", tmp, src, "-lm"])
        os.replace(tmp, lib)
    return lib


class AttentionOracle:
    def __init__(self, lib_path: str):
        lib = ctypes.CDLL(lib_path)
        P, I, LL = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong
        lib.csa_oracle_sparse_attention.argtypes = [P, P, P, LL, P, I, I, I, I, I, I, I,
                                                    ctypes.c_double, P, LL, P]
        lib.csa_oracle_sparse_attention.restype = I
        self.lib = lib

    def sparse_attention(self, qa_bits, kc_bits, vc_bits, idx, *, B, S, T, HA, Dk, Dv, topk,
                         scale, ld_v=None, rows=None):
        """o [n_rows, HA, Dv] (fp64) of the given flat query rows (all when None).

        qa_bits: uint16 [B,S,HA,Dk] (bf16 bits); kc_bits: uint16 [B,T,Dk];
        vc_bits: uint16 array whose row s of batch b starts at (b*T + s)*ld_v
        (ld_v defaults to Dv; pass kc_bits itself with ld_v=Dk for values that
        are a prefix of each key row); idx: int32 [B,S,topk], -1 = padding.
        """
        qa = np.ascontiguousarray(qa_bits, dtype=np.uint16)
        kc = np.ascontiguousarray(kc_bits, dtype=np.uint16)
        vc = np.ascontiguousarray(vc_bits, dtype=np.uint16)
        ix = np.ascontiguousarray(idx, dtype=np.int32)
        ld_v = Dv if ld_v is None else int(ld_v)
        if rows is None:
            n = B * S
            rows_arr = None
        else:
            rows_arr = np.ascontiguousarray(rows, dtype=np.int64)
            n = len(rows_arr)
        out = np.empty((n, HA, Dv), np.float64)

        def ptr(a):
            return None if a is None else a.ctypes.data_as(ctypes.c_void_p)

        rc = self.lib.csa_oracle_sparse_attention(ptr(qa), ptr(kc), ptr(vc), ld_v, ptr(ix), B, S,
                                                  T, HA, Dk, Dv, topk, float(scale),
                                                  ptr(rows_arr), n, ptr(out))
        if rc != 0:
            raise ValueError(f"attention oracle rejected its arguments (code {rc})")
        return out


_default = None


def default() -> AttentionOracle:
    global _default
    if _default is None:
        _default = AttentionOracle(build())
    return _default


def sparse_attention(*args, **kw):
    return default().sparse_attention(*args, **kw)
