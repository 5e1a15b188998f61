"""CPU oracle of the OR-union of several layers' selections -- TEST
INFRASTRUCTURE (only ``tests/`` may import it).

"FlashMemory-DeepSeek-V4: Lightning Index Ultra-Long Context via Lookahead
Sparse Attention", "What carries the argument": the gated decisions of a few
layers are combined by OR-union.  Per row: the set of keys in [0, T) that any
list holds, in ascending order, the first ``cap`` of them, padded with -1.
Plain Python sets, row by row.
"""
from __future__ import annotations

import numpy as np


def union_selections(lists, T: int, cap: int):
    """lists: int arrays of one shape [..., topk]; returns (out [..., cap], count [...])."""
    shape = np.asarray(lists[0]).shape
    flat = [np.asarray(x).reshape(-1, shape[-1]) for x in lists]
    rows = flat[0].shape[0]
    out = np.full((rows, cap), -1, np.int32)
    count = np.zeros((rows,), np.int32)
    for r in range(rows):
        keys = set()
        for x in flat:
            for v in x[r].tolist():
                if 0 <= v < T:
                    keys.add(v)
        ordered = sorted(keys)[:cap]
        out[r, :len(ordered)] = ordered
        count[r] = len(ordered)
    return out.reshape(shape[:-1] + (cap,)), count.reshape(shape[:-1])
