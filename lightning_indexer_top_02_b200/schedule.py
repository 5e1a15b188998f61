"""Cross-layer scheduling of the indexer over the library's entry points.

Three ways to give each layer of a decode step its selection, all built from
the C-ABI calls (``csa_indexer_topk_ex``, ``csa_sparse_attention``,
``csa_union_selections``); this module only orders the launches on CUDA
streams:

* ``"own"`` -- every layer runs its own indexer, then its attention reads
  that selection (the plain DeepSeek Sparse Attention order);
* ``"mli"`` -- the Multi-layer Indexer blog post (third paragraph): a layer's
  attention reads the selection the previous layer's indexer made, and the
  layer's own indexer runs for the next layer on a second CUDA stream, so the
  indexer scan overlaps the attention instead of preceding it (layer 0 reads
  its own selection);
* ``"indexcache"`` -- the same post (fourth paragraph): the indexer runs only
  on every ``refresh``-th layer and the layers in between reuse the latest
  selection.

``union_of_layers`` is the lookahead page's OR-union of gated selections of a
few layers ("FlashMemory-DeepSeek-V4 ...", "What carries the argument").
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional

import lightning_indexer_top_02_b200 as L


@dataclass
class Layer:
    """One layer's decode-step inputs (CUDA tensors).

    Indexer: ``iq`` bf16 [B,S,H_I,d], ``iw`` fp32 [B,S,H_I], ``ik`` bf16 or
    E4M3 [B,T,d] (``ik_scale`` fp32 [B,T] with E4M3).  Attention: ``aq`` bf16
    [B,S,HA,Dk], ``kc`` bf16 [B,T,Dk], ``vc`` bf16 [B,T,Dv] or None (values =
    the first ``dv`` elements of each ``kc`` row), ``scale``.
    """
    iq: object
    iw: object
    ik: object
    aq: object
    kc: object
    scale: float
    ik_scale: object = None
    vc: object = None
    dv: Optional[int] = None


def _select(layer: Layer, m: int, topk: int, mode: int, stream):
    return L.indexer_topk(layer.iq, layer.iw, layer.ik, k_scale=layer.ik_scale, m=m, topk=topk,
                          mode=mode, stream=stream)[0]


def _attend(layer: Layer, idx, stream):
    return L.sparse_attention(layer.aq, layer.kc, idx, scale=layer.scale, v=layer.vc, dv=layer.dv,
                              stream=stream)


def decode_layers(layers: List[Layer], *, m: int, topk: int, schedule: str = "mli",
                  mode: int = L.CSA_MODE_TOPK, refresh: int = 2, main=None, side=None):
    """Runs the layers' selections and sparse attentions in the given
    schedule; returns (outputs, selections), one per layer, where
    selections[l] is the selection layer l's attention read.  Both streams
    are ordered after everything already queued on ``main``."""
    import torch

    dev = layers[0].aq.device
    main = main or torch.cuda.current_stream(dev)
    outs, used = [], []
    if schedule == "own":
        for layer in layers:
            idx = _select(layer, m, topk, mode, main)
            used.append(idx)
            outs.append(_attend(layer, idx, main))
        return outs, used
    if schedule == "indexcache":
        idx = None
        for l, layer in enumerate(layers):
            if idx is None or l % refresh == 0:
                idx = _select(layer, m, topk, mode, main)
            used.append(idx)
            outs.append(_attend(layer, idx, main))
        return outs, used
    if schedule != "mli":
        raise ValueError(f"unknown schedule {schedule!r}")
    side = side or torch.cuda.Stream(dev)
    start = torch.cuda.Event()
    start.record(main)
    side.wait_event(start)
    n = len(layers)
    idx = [None] * n
    ready = [None] * n
    idx[0] = _select(layers[0], m, topk, mode, main)   # layer 0 has no earlier indexer
    for l in range(n):
        feeds_next = 1 <= l < n - 1
        if feeds_next:
            # layer l's indexer works for layer l+1, beside layer l's attention
            with torch.cuda.stream(side):
                idx[l] = _select(layers[l], m, topk, mode, side)
                idx[l].record_stream(main)
                ready[l] = torch.cuda.Event()
                ready[l].record(side)
        sel = idx[0] if l == 0 else idx[l - 1]
        used.append(sel)
        outs.append(_attend(layers[l], sel, main))
        if feeds_next:
            main.wait_event(ready[l])
    side.wait_stream(main)
    return outs, used


def union_of_layers(selections, T: int, cap: Optional[int] = None, stream=None):
    """OR-union of gated selections of several layers (ascending keys, -1 padding)."""
    return L.union_selections(selections, T=T, cap=cap, stream=stream)
