"""Action tokenizer MLP_act, fp64 (test infrastructure only).

Source: LLaTTE notes (huaxiaozhuan.com), appendix A.2 "Sequence Module",
item 1 "Action Embeddings": every action a_t = (tau_t, type_t, item_t,
surface_t, meta_t) of the time-ordered history is embedded field by field
(E_type, E_item, E_surface, E_time, E_meta) and the embeddings are projected
to one token x_t in R^d by MLP_act; the tokens, earliest first, form X_seq.

Readings (the pages name the parts and give no formula):
  * every field, the timestamp included, is an integer id into its own
    embedding table (the timestamp's id being its time bucket);
  * MLP_act takes the concatenation of the field embeddings in the order
    the pages list its arguments' tables (the order of `tables`), and is a
    two-layer MLP with SiLU between, without biases like every other
    projection on the pages: x_t = W_a2 SiLU(W_a1 [e_1 ; ... ; e_F]);
  * an id outside its table is an input error: the token is not defined.
"""
from __future__ import annotations

from typing import Sequence

import numpy as np


def _silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def embed(ids: np.ndarray, tables: Sequence[np.ndarray]) -> np.ndarray:
    """[n, D_in]: per event the field embeddings, concatenated in table order."""
    ids = np.asarray(ids)
    n = ids.shape[0]
    if ids.ndim != 2 or ids.shape[1] != len(tables):
        raise ValueError("ids must be [n_events, n_fields]")
    cols = []
    for f, tab in enumerate(tables):
        tab = np.asarray(tab, dtype=np.float64)
        col = ids[:, f].astype(np.int64)
        if n and (col.min() < 0 or col.max() >= tab.shape[0]):
            raise ValueError(f"field {f}: id outside its table")
        cols.append(tab[col])
    return np.concatenate(cols, axis=1) if cols else np.zeros((n, 0))


def action_tokens(ids: np.ndarray, tables: Sequence[np.ndarray], W_a1: np.ndarray,
                  W_a2: np.ndarray) -> np.ndarray:
    """x_t = W_a2 SiLU(W_a1 e_t) for every event t: [n, d] fp64."""
    e = embed(ids, tables)
    h = _silu(e @ np.asarray(W_a1, dtype=np.float64).T)
    return h @ np.asarray(W_a2, dtype=np.float64).T
