"""Pyramidal schedule integers (LLaTTE notes, appendix A.2 "Transformer Layers
and Pyramidal Schedule": the next layer operates on the last T_{l+1} rows of
this layer's output, T_{l+1} <= T_l; three modes full / pyramidal / cross).

Reading taken: keep_l counts HISTORY rows only; the n_q query tokens are always
kept. With the pages' own count (which includes the query tokens),
T_l(pages) = n_l + n_q, so keep_l = T_l(pages) - n_q; keep_l = 0 is the cross
mode (only query tokens remain). A user whose history is shorter than keep_l
keeps all of it.

Per user u and layer l (1-based in the pages, 0-based here):
  T_{0,u}  = input history length
  n_{l,u}  = min(T_{l,u}, keep_l)          history rows kept as queries
  q_{l,u}  = n_{l,u} + n_q                 query rows of layer l
  T_{l+1,u} = n_{l,u}
  hist_off_l  = exclusive prefix sum of T_{l,u}     (history/key rows)
  query_off_l = exclusive prefix sum of q_{l,u}     (query rows = next layer's rows)
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Sequence

import numpy as np


@dataclass
class LayerPlan:
    T: np.ndarray           # int64 [B] history (key) rows entering the layer
    n: np.ndarray           # int64 [B] kept history rows (queries)
    hist_off: np.ndarray    # int64 [B+1]
    query_off: np.ndarray   # int64 [B+1]


def _exscan(v: np.ndarray) -> np.ndarray:
    out = np.zeros(v.shape[0] + 1, dtype=np.int64)
    acc = 0
    for i, x in enumerate(v.tolist()):      # plain loop: the definition, no tricks
        out[i] = acc
        acc += int(x)
    out[-1] = acc
    return out


def plan_layers(lengths: Sequence[int], keep: Sequence[int], n_q: int) -> List[LayerPlan]:
    lengths = np.asarray(lengths, dtype=np.int64)
    if np.any(lengths < 0):
        raise ValueError("negative history length")
    for a, b in zip(keep, keep[1:]):
        if b > a:
            raise ValueError("keep schedule must be non-increasing (T_{l+1} <= T_l)")
    if any(k < 0 for k in keep):
        raise ValueError("negative keep count")
    plans = []
    T = lengths.copy()
    for k in keep:
        n = np.minimum(T, k)
        plans.append(LayerPlan(T=T.copy(), n=n.copy(), hist_off=_exscan(T),
                               query_off=_exscan(n + n_q)))
        T = n
    return plans
