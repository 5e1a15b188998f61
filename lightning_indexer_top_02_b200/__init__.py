"""Python binding of the B200 CSA lightning-indexer top-k library.

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libcsa_indexer.so`` (see ``include/csa_indexer.h`` for the
operation, layouts and error behaviour).  PyTorch provides device memory and
streams.  There is no CPU fallback: if the library is missing, importing the
functions below raises.

C-ABI names are mirrored one to one (``csa_indexer_topk``,
``csa_indexer_topk_ex``, ``csa_indexer_workspace_size``, ``csa_status_string``,
``csa_last_device_error``, ``csa_set_wait_limit``, ``csa_set_launch_events``,
``csa_version``);
``indexer_topk`` is the same call on torch tensors.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

from .build import LIB as _BUILT_LIB

# The library this binding loads: the in-tree build, or another build of the
# same sources named by CSA_INDEXER_LIB (e.g. the -DCSA_DEBUG build).
LIB_PATH = os.environ.get("CSA_INDEXER_LIB") or _BUILT_LIB

CSA_OK = 0
CSA_ERR_INVALID_ARG = 1
CSA_ERR_UNSUPPORTED = 2
CSA_ERR_WORKSPACE = 3
CSA_ERR_CUDA = 4
CSA_ERR_TIMEOUT = 5
CSA_ERR_DEBUG_CHECK = 6
CSA_KEY_BF16 = 0
CSA_KEY_E4M3 = 1
CSA_MODE_TOPK = 0
CSA_MODE_GATE = 1
CSA_Q_OFFSET_DEFAULT = -(1 << 63)

EXPORTS = ("csa_indexer_topk", "csa_indexer_topk_ex", "csa_indexer_workspace_size",
           "csa_indexer_plan", "csa_indexer_topk_noalloc", "csa_sparse_attention",
           "csa_union_selections", "csa_merge_topk", "csa_merge_workspace_size",
           "csa_status_string", "csa_last_device_error", "csa_set_wait_limit",
           "csa_set_launch_events", "csa_version")


class CsaError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        super().__init__(f"{what}: {csa_status_string(status)} (status {status})")


class CsaArgs(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("w", ctypes.c_void_p), ("k", ctypes.c_void_p),
        ("k_scale", ctypes.c_void_p),
        ("B", ctypes.c_int), ("S", ctypes.c_int), ("T", ctypes.c_int), ("H_I", ctypes.c_int),
        ("d", ctypes.c_int), ("m", ctypes.c_int), ("topk", ctypes.c_int),
        ("causal", ctypes.c_int), ("key_dtype", ctypes.c_int), ("mode", ctypes.c_int),
        ("q_offset", ctypes.c_longlong), ("num_splits", ctypes.c_int),
        ("out_idx", ctypes.c_void_p), ("out_score", ctypes.c_void_p),
        ("query_pieces", ctypes.c_int),
    ]


class CsaAttnArgs(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("ld_v", ctypes.c_longlong), ("idx", ctypes.c_void_p),
        ("B", ctypes.c_int), ("S", ctypes.c_int), ("T", ctypes.c_int), ("HA", ctypes.c_int),
        ("Dk", ctypes.c_int), ("Dv", ctypes.c_int), ("topk", ctypes.c_int),
        ("scale", ctypes.c_float), ("out", ctypes.c_void_p),
    ]


class CsaPlan(ctypes.Structure):
    _fields_ = [("grid", ctypes.c_int), ("threads", ctypes.c_int), ("smem_bytes", ctypes.c_int),
                ("stages", ctypes.c_int), ("queries_per_block", ctypes.c_int),
                ("num_splits", ctypes.c_int), ("launches", ctypes.c_int),
                ("workspace_bytes", ctypes.c_size_t)]

    def as_dict(self):
        return {name: getattr(self, name) for name, _ in self._fields_}


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load ``libcsa_indexer.so`` (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"CUDA library {path} is missing; build it with "
                          "lightning_indexer_top_02_b200.build.build()")
    lib = ctypes.CDLL(path)
    P, I, LL = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong
    lib.csa_indexer_topk.argtypes = [P, P, P, I, I, I, I, I, I, I, I, P, P, P]
    lib.csa_indexer_topk.restype = I
    lib.csa_indexer_topk_ex.argtypes = [ctypes.POINTER(CsaArgs), P, ctypes.c_size_t, P]
    lib.csa_indexer_topk_ex.restype = I
    lib.csa_indexer_workspace_size.argtypes = [ctypes.POINTER(CsaArgs)]
    lib.csa_indexer_workspace_size.restype = ctypes.c_size_t
    lib.csa_indexer_topk_noalloc.argtypes = [ctypes.POINTER(CsaArgs), P]
    lib.csa_indexer_topk_noalloc.restype = I
    lib.csa_merge_topk.argtypes = [P, P, P, I, I, I, I, P, P, P, ctypes.c_size_t, P]
    lib.csa_merge_topk.restype = I
    lib.csa_merge_workspace_size.argtypes = [I, I, I]
    lib.csa_merge_workspace_size.restype = ctypes.c_size_t
    lib.csa_union_selections.argtypes = [P, I, I, I, I, I, P, P, P]
    lib.csa_union_selections.restype = I
    lib.csa_sparse_attention.argtypes = [ctypes.POINTER(CsaAttnArgs), P]
    lib.csa_sparse_attention.restype = I
    lib.csa_indexer_plan.argtypes = [ctypes.POINTER(CsaArgs), ctypes.POINTER(CsaPlan)]
    lib.csa_indexer_plan.restype = I
    lib.csa_status_string.argtypes = [I]
    lib.csa_status_string.restype = ctypes.c_char_p
    lib.csa_last_device_error.argtypes = [P]
    lib.csa_last_device_error.restype = I
    lib.csa_set_wait_limit.argtypes = [ctypes.c_ulonglong]
    lib.csa_set_wait_limit.restype = None
    lib.csa_set_launch_events.argtypes = [P, I]
    lib.csa_set_launch_events.restype = I
    lib.csa_version.argtypes = []
    lib.csa_version.restype = I
    _lib = lib
    return lib


# ----------------------------------------------------------------- raw C-ABI mirrors

def csa_indexer_topk(q_ptr, w_ptr, k_ptr, B, S, T, H_I, d, m, topk, causal, out_idx_ptr,
                     out_score_ptr, stream_ptr) -> int:
    return load_library().csa_indexer_topk(q_ptr, w_ptr, k_ptr, B, S, T, H_I, d, m, topk,
                                           causal, out_idx_ptr, out_score_ptr, stream_ptr)


def csa_indexer_topk_ex(args: CsaArgs, workspace_ptr, workspace_bytes: int, stream_ptr) -> int:
    return load_library().csa_indexer_topk_ex(ctypes.byref(args), workspace_ptr,
                                              workspace_bytes, stream_ptr)


def csa_indexer_workspace_size(args: CsaArgs) -> int:
    return load_library().csa_indexer_workspace_size(ctypes.byref(args))


def csa_indexer_topk_noalloc(args: CsaArgs, stream_ptr) -> int:
    """The allocation-free entry point (fixed in-library scratch; see the header)."""
    return load_library().csa_indexer_topk_noalloc(ctypes.byref(args), stream_ptr)


def csa_sparse_attention(args: CsaAttnArgs, stream_ptr) -> int:
    return load_library().csa_sparse_attention(ctypes.byref(args), stream_ptr)


def csa_indexer_plan(args: CsaArgs) -> CsaPlan:
    plan = CsaPlan()
    st = load_library().csa_indexer_plan(ctypes.byref(args), ctypes.byref(plan))
    if st != CSA_OK:
        raise CsaError(st, "csa_indexer_plan")
    return plan


def csa_status_string(status: int) -> str:
    return load_library().csa_status_string(status).decode()


def csa_last_device_error(stream_ptr=None) -> int:
    return load_library().csa_last_device_error(stream_ptr)


def csa_set_wait_limit(cycles: int) -> None:
    load_library().csa_set_wait_limit(cycles)


def csa_set_launch_events(events) -> int:
    """Record ``events`` (torch.cuda.Event with timing, or raw cudaEvent_t
    handles) around every kernel launch of later calls on this thread; pass
    None or [] to stop.  The list must stay alive while set."""
    global _event_array
    if not events:
        _event_array = None
        return load_library().csa_set_launch_events(None, 0)
    handles = [e.cuda_event if hasattr(e, "cuda_event") else int(e) for e in events]
    _event_array = (ctypes.c_void_p * len(handles))(*handles)
    return load_library().csa_set_launch_events(_event_array, len(handles))


_event_array = None


def csa_version() -> int:
    return load_library().csa_version()


# ----------------------------------------------------------------- torch convenience

def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def make_args(q, w, k, *, k_scale=None, m: int, topk: int, causal: bool = True,
              mode: int = CSA_MODE_TOPK, q_offset: Optional[int] = None, num_splits: int = 0,
              query_pieces: int = 0, out_idx=None, out_score=None) -> CsaArgs:
    """Pack torch tensors into the C argument struct (shapes read from q and k)."""
    import torch

    B, S, H, d = q.shape
    T = k.shape[1]
    fp8 = k.dtype in (torch.uint8, torch.float8_e4m3fn)
    a = CsaArgs()
    a.q, a.w, a.k = q.data_ptr(), w.data_ptr(), k.data_ptr()
    a.k_scale = k_scale.data_ptr() if k_scale is not None else None
    a.B, a.S, a.T, a.H_I, a.d, a.m, a.topk = B, S, T, H, d, m, topk
    a.causal = int(bool(causal))
    a.key_dtype = CSA_KEY_E4M3 if fp8 else CSA_KEY_BF16
    a.mode = int(mode)
    a.q_offset = CSA_Q_OFFSET_DEFAULT if q_offset is None else int(q_offset)
    a.num_splits = int(num_splits)
    a.query_pieces = int(query_pieces)
    a.out_idx = out_idx.data_ptr() if out_idx is not None else None
    a.out_score = out_score.data_ptr() if out_score is not None else None
    return a


def indexer_topk(q, w, k, *, k_scale=None, m: int, topk: int, causal: bool = True,
                 mode: int = CSA_MODE_TOPK, q_offset: Optional[int] = None,
                 num_splits: int = 0, query_pieces: int = 0, out_idx=None, out_score=None,
                 workspace=None,
                 stream=None):
    """Run the indexer top-k on CUDA tensors; returns (out_idx, out_score).

    q: bf16 [B,S,H_I,d]; w: fp32 [B,S,H_I]; k: bf16 [B,T,d] or E4M3 bytes
    (uint8 / float8_e4m3fn) [B,T,d] with k_scale fp32 [B,T].  Outputs are
    allocated if not given.  ``workspace`` (uint8 CUDA tensor) is optional.
    """
    import torch

    for name, t in (("q", q), ("w", w), ("k", k)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if q.dtype != torch.bfloat16 or w.dtype != torch.float32:
        raise TypeError("q must be bfloat16 and w float32")
    B, S, H, d = q.shape
    if out_idx is None:
        out_idx = torch.empty((B, S, topk), dtype=torch.int32, device=q.device)
    if out_score is None:
        out_score = torch.empty((B, S, topk), dtype=torch.float32, device=q.device)
    a = make_args(q, w, k, k_scale=k_scale, m=m, topk=topk, causal=causal, mode=mode,
                  q_offset=q_offset, num_splits=num_splits, query_pieces=query_pieces,
                  out_idx=out_idx, out_score=out_score)
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    st = csa_indexer_topk_ex(a, ws_ptr, ws_bytes, ctypes.c_void_p(stream.cuda_stream))
    if st != CSA_OK:
        raise CsaError(st, "csa_indexer_topk_ex")
    return out_idx, out_score


def sparse_attention(q, k, idx, *, scale: float, v=None, dv: Optional[int] = None, out=None,
                     stream=None):
    """Attention of every head over the keys ``idx`` selects, on CUDA tensors.

    q: bf16 [B,S,HA,Dk]; k: bf16 [B,T,Dk]; idx: int32 [B,S,topk] (the
    indexer's out_idx); v: bf16 [B,T,Dv], or None to read the values as the
    first ``dv`` elements of each key row (one latent cache).  Returns out
    fp32 [B,S,HA,Dv] (allocated if not given).
    """
    import torch

    B, S, HA, Dk = q.shape
    T = k.shape[1]
    if v is None:
        Dv = int(dv) if dv is not None else Dk
        vt, ld_v = k, Dk
    else:
        Dv = v.shape[-1]
        vt, ld_v = v, Dv
    for name, t in (("q", q), ("k", k), ("v", vt), ("idx", idx)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if out is None:
        out = torch.empty((B, S, HA, Dv), dtype=torch.float32, device=q.device)
    a = CsaAttnArgs()
    a.q, a.k, a.v, a.ld_v, a.idx = q.data_ptr(), k.data_ptr(), vt.data_ptr(), ld_v, idx.data_ptr()
    a.B, a.S, a.T, a.HA, a.Dk, a.Dv, a.topk = B, S, T, HA, Dk, Dv, idx.shape[-1]
    a.scale = float(scale)
    a.out = out.data_ptr()
    if stream is None:
        stream = torch.cuda.current_stream(q.device)
    st = csa_sparse_attention(a, ctypes.c_void_p(stream.cuda_stream))
    if st != CSA_OK:
        raise CsaError(st, "csa_sparse_attention")
    return out


def csa_union_selections(list_ptrs, rows: int, topk: int, T: int, cap: int, out_ptr, count_ptr,
                         stream_ptr) -> int:
    arr = (ctypes.c_void_p * len(list_ptrs))(*list_ptrs)
    return load_library().csa_union_selections(arr, len(list_ptrs), rows, topk, T, cap, out_ptr,
                                               count_ptr, stream_ptr)


def union_selections(idx_lists, T: int, cap: Optional[int] = None, stream=None):
    """OR-union per row of several [.., topk] int32 CUDA selections (same
    shape); returns (keys [rows, cap] ascending with -1 padding, count [rows])."""
    import torch

    first = idx_lists[0]
    topk = first.shape[-1]
    rows = first.numel() // topk
    for t in idx_lists:
        if not t.is_cuda or not t.is_contiguous() or t.dtype != torch.int32 or t.shape != first.shape:
            raise ValueError("selections must be contiguous int32 CUDA tensors of one shape")
    cap = len(idx_lists) * topk if cap is None else int(cap)
    out = torch.empty(first.shape[:-1] + (cap,), dtype=torch.int32, device=first.device)
    count = torch.empty(first.shape[:-1], dtype=torch.int32, device=first.device)
    if stream is None:
        stream = torch.cuda.current_stream(first.device)
    st = csa_union_selections([t.data_ptr() for t in idx_lists], rows, topk, T, cap,
                              ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(count.data_ptr()),
                              ctypes.c_void_p(stream.cuda_stream))
    if st != CSA_OK:
        raise CsaError(st, "csa_union_selections")
    return out, count
