"""Attention-probability statistics of the query tokens, fp64.

TEST INFRASTRUCTURE ONLY (see the package docstring).

Source: LLaTTE notes (huaxiaozhuan.com), appendix A.4 "Attention Weight
Distribution": the probabilities P = softmax(Q K^T / sqrt(d_k)) of every query
token over the user's sequence are aggregated over many requests into
  * the cumulative attention on the most recent k events (Figure 3),
  * the cumulative attention on the k events with the largest weights (the
    most any k events can hold), and
  * the attention by hours before the request (Figures 5 and 6: 24-hour
    peaks).

Readings (the pages show plots, not formulas): per (user, query token, head)
of one layer, for k = 1, 2, 4, ..., 2^(n_k - 1),
  recent[k] = sum of P over the k most recent keys of that layer (all keys when
              k >= T; zero when the user has no key),
  topk[k]   = sum of the k largest entries of P (likewise);
and, when every history event has an age in hours before the request,
  hours[b]  = sum of P over keys whose age a has floor(a) = b, the last bin
              b = n_hours - 1 also taking every older key.
The keys of layer l are the T_l most recent history events of the user (the
pyramid keeps the most recent rows), so key t of layer l is event
T_0 - T_l + t of the user's input.  Aggregation over users and query tokens is
left to the caller.
"""
from __future__ import annotations

from typing import Optional, Sequence

import numpy as np

from .model import forward


def row_stats(p: np.ndarray, n_k: int, ages: Optional[np.ndarray] = None, n_hours: int = 0):
    """Statistics of one probability row p [T] (keys earliest first)."""
    p = np.asarray(p, dtype=np.float64)
    T = p.shape[0]
    recent = np.zeros(n_k)
    topk = np.zeros(n_k)
    desc = np.sort(p)[::-1]
    for i in range(n_k):
        k = 1 << i
        recent[i] = p[max(0, T - k):].sum()
        topk[i] = desc[:k].sum()
    hours = None
    if ages is not None:
        hours = np.zeros(n_hours)
        b = np.minimum(np.floor(np.asarray(ages, dtype=np.float64)), n_hours - 1).astype(np.int64)
        np.add.at(hours, b, p)
    return recent, topk, hours


def attention_stats(inputs, layer: int, n_k: int, ages: Optional[np.ndarray] = None,
                    n_hours: int = 0, users: Optional[Sequence[int]] = None):
    """Per (user, query token, head) statistics of layer `layer`.

    ages: float [sum of history lengths], hours before the request of every
    input event (same jagged layout as inputs.values), or None.
    Returns (recent [U, n_q, h, n_k], topk [U, n_q, h, n_k],
    hours [U, n_q, h, n_hours] or None).
    """
    dims = inputs.dims
    users = list(range(inputs.batch)) if users is None else [int(u) for u in users]
    _, probs = forward(inputs, users=users, return_probs=True)
    h, nq = dims.heads, dims.n_q
    R = np.zeros((len(users), nq, h, n_k))
    K = np.zeros((len(users), nq, h, n_k))
    H = np.zeros((len(users), nq, h, n_hours)) if ages is not None else None
    for ui, u in enumerate(users):
        a0 = int(inputs.offsets[u])
        T0 = int(inputs.offsets[u + 1]) - a0
        for j in range(h):
            P = probs[ui][layer][j]                    # [n + n_q, T_l]
            T = P.shape[1]
            n = P.shape[0] - nq
            key_ages = None
            if ages is not None:
                key_ages = np.asarray(ages[a0 + T0 - T: a0 + T0], dtype=np.float64)
            for i in range(nq):
                rec, top, hrs = row_stats(P[n + i], n_k, key_ages, n_hours)
                R[ui, i, j], K[ui, i, j] = rec, top
                if H is not None:
                    H[ui, i, j] = hrs
    return R, K, H
