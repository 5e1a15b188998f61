"""Key-sharded selection across GPUs.

"Million-Token Memory Without the Global Bottleneck" (first and second
paragraphs): with the keys split across GPUs, each GPU selects over its own
keys and the selections are combined so that they cover the global top.  Here
each rank holds one contiguous range of the compressed keys; it runs the
indexer over its range (``csa_indexer_topk_ex`` with the query positions
shifted by the range start, so the causal rule still sees absolute key
positions), all ranks exchange their lists with one all-gather, and every
rank merges them (``csa_merge_topk``):

* exact -- each rank keeps its range's top k (``k_local = topk``): the merge
  is then exactly the top k over all keys, ties to the lower index;
* relaxed -- each rank keeps fewer (``k_local < topk``): less to exchange and
  merge, at a cost in recall that ``tests/`` measures.

The exchange is the one collective step of the method (NCCL over NVLink;
``gloo`` in the CPU tests).  ``select_fn`` and ``merge_fn`` default to the
CUDA entry points; the CPU tests pass their own to exercise the plumbing.
"""
from __future__ import annotations

import ctypes
from typing import Callable, Optional, Tuple

import lightning_indexer_top_02_b200 as L


def shard_range(T: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous, balanced key range [start, end) of rank ``rank``."""
    if not (0 <= rank < world):
        raise ValueError("rank out of range")
    return T * rank // world, T * (rank + 1) // world


def local_q_offset(S: int, T_total: int, m: int, start: int, q_offset: Optional[int] = None) -> int:
    """Query offset that makes a key range starting at ``start`` see the
    causal rule of the full key set: key s of the range is key start + s, and
    (start + s + 1) m - 1 <= t  <=>  (s + 1) m - 1 <= t - start m."""
    q_abs = max(0, T_total * m - S) if q_offset is None else int(q_offset)
    return q_abs - start * m


def select_local(q, w, k_range, *, start: int, T_total: int, m: int, k_local: int,
                 k_scale=None, causal: bool = True, mode: int = L.CSA_MODE_TOPK,
                 q_offset: Optional[int] = None, stream=None):
    """The indexer over one key range; indices are range-local."""
    S = q.shape[1]
    return L.indexer_topk(q, w, k_range, k_scale=k_scale, m=m, topk=k_local, causal=causal,
                          mode=mode, q_offset=local_q_offset(S, T_total, m, start, q_offset),
                          stream=stream)


def merge_topk(idx_lists, score_lists, offsets, topk: int, stream=None):
    """Exact top-k of the union of range-local lists (``csa_merge_topk``)."""
    import torch

    first = idx_lists[0]
    k_in = first.shape[-1]
    rows = first.numel() // k_in
    out_idx = torch.empty(first.shape[:-1] + (topk,), dtype=torch.int32, device=first.device)
    out_sc = torch.empty(first.shape[:-1] + (topk,), dtype=torch.float32, device=first.device)
    n = len(idx_lists)
    ip = (ctypes.c_void_p * n)(*[t.data_ptr() for t in idx_lists])
    sp = (ctypes.c_void_p * n)(*[t.data_ptr() for t in score_lists])
    op = (ctypes.c_longlong * n)(*[int(o) for o in offsets])
    if stream is None:
        stream = torch.cuda.current_stream(first.device)
    st = L.load_library().csa_merge_topk(ip, sp, op, n, rows, k_in, topk,
                                         ctypes.c_void_p(out_idx.data_ptr()),
                                         ctypes.c_void_p(out_sc.data_ptr()), None, 0,
                                         ctypes.c_void_p(stream.cuda_stream))
    if st != L.CSA_OK:
        raise L.CsaError(st, "csa_merge_topk")
    return out_idx, out_sc


def sharded_indexer_topk(q, w, k_range, *, start: int, T_total: int, m: int, topk: int,
                         k_local: Optional[int] = None, k_scale=None, causal: bool = True,
                         mode: int = L.CSA_MODE_TOPK, q_offset: Optional[int] = None,
                         group=None, select_fn: Optional[Callable] = None,
                         merge_fn: Optional[Callable] = None):
    """Every rank: select over its key range [start, start + k_range.shape[1]),
    all-gather the lists, merge.  Returns (idx, score) [B, S, topk] with
    global key indices, the same on every rank."""
    import torch
    import torch.distributed as dist

    k_local = topk if k_local is None else int(k_local)
    select_fn = select_fn or select_local
    merge_fn = merge_fn or merge_topk
    idx, sc = select_fn(q, w, k_range, start=start, T_total=T_total, m=m, k_local=k_local,
                        k_scale=k_scale, causal=causal, mode=mode, q_offset=q_offset)
    world = dist.get_world_size(group)
    idx_all = [torch.empty_like(idx) for _ in range(world)]
    sc_all = [torch.empty_like(sc) for _ in range(world)]
    starts = torch.tensor([start], dtype=torch.int64, device=idx.device)
    starts_all = [torch.empty_like(starts) for _ in range(world)]
    dist.all_gather(idx_all, idx.contiguous(), group=group)
    dist.all_gather(sc_all, sc.contiguous(), group=group)
    dist.all_gather(starts_all, starts, group=group)
    offsets = [int(s.item()) for s in starts_all]
    return merge_fn(idx_all, sc_all, offsets, topk)
