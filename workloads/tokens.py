"""Seeded synthetic action events for the action tokenizer (MLP_act).

Shapes and random numbers only: no arithmetic of the method lives here.

An action a_t = (tau_t, type_t, item_t, surface_t, meta_t) is given as one
integer id per field, each indexing that field's embedding table; the time
field's id is the index of the event's time bucket (how a timestamp is cut
into buckets is the caller's choice, so the generator draws bucket ids
directly, recent buckets more often).

Draw order for a seed (NumPy PCG64), fixed so every consumer sees the same
numbers: the embedding tables field by field (N(0, 1)), W_a1 [d_hid, D_in]
N(0, 1/D_in), W_a2 [d, d_hid] N(0, 1/d_hid), then the ids field by field:
  type     uniform over the table
  item     Zipf(1.2) popularity ranks folded into the table, then mapped
           through a fixed random permutation (popular items spread out)
  surface  uniform
  time     geometric(0.05) bucket index, clipped to the table
  meta     uniform
Values are rounded to the storage type (bf16 RNE) before anyone sees them.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import List, Tuple

import numpy as np

from .gen import round_to_bf16

FIELDS = ("type", "item", "surface", "time", "meta")


@dataclass(frozen=True)
class TokDims:
    """Tokenizer dimensions: per field the table rows and embedding width,
    the MLP hidden width and the token width d."""
    rows: Tuple[int, ...]
    width: Tuple[int, ...]
    d_hid: int
    d: int
    dtype: str = "bf16"

    @property
    def n_fields(self) -> int:
        return len(self.rows)

    @property
    def d_in(self) -> int:
        return int(sum(self.width))


TOKENIZERS = {
    # small fp32 case: the oracle finishes in milliseconds
    "tiny": TokDims(rows=(8, 1000, 4, 32, 64), width=(8, 16, 8, 8, 8), d_hid=64, d=64,
                    dtype="fp32"),
    # the online ranker's token width (d = 256): D_in = 256, hidden 256
    "online": TokDims(rows=(64, 262144, 32, 256, 4096), width=(32, 128, 32, 32, 32),
                      d_hid=256, d=256),
    # widths the tensor-core GEMMs do not take (D_in = 48): CUDA-core GEMMs in bf16
    "odd_bf16": TokDims(rows=(8, 500, 4, 16, 32), width=(8, 16, 8, 8, 8), d_hid=96, d=64),
}


@dataclass
class TokInputs:
    dims: TokDims
    tables: List[np.ndarray]   # float32 [rows_f, width_f], storage-rounded
    W_a1: np.ndarray           # float32 [d_hid, d_in]
    W_a2: np.ndarray           # float32 [d, d_hid]
    ids: np.ndarray            # int32 [n_events, n_fields]


def draw_ids(dims: TokDims, n: int, rng: np.random.Generator) -> np.ndarray:
    ids = np.empty((n, dims.n_fields), dtype=np.int32)
    for f, rows in enumerate(dims.rows):
        name = FIELDS[f] if f < len(FIELDS) else "meta"
        if name == "item":
            perm = rng.permutation(rows)
            ranks = rng.zipf(1.2, size=n) - 1
            ids[:, f] = perm[ranks % rows]
        elif name == "time":
            ids[:, f] = np.minimum(rng.geometric(0.05, size=n) - 1, rows - 1)
        else:
            ids[:, f] = rng.integers(0, rows, size=n)
    return ids


def make_token_inputs(dims: TokDims, n_events: int, seed: int) -> TokInputs:
    rng = np.random.Generator(np.random.PCG64(seed))
    tables = [rng.standard_normal(size=(r, w), dtype=np.float32)
              for r, w in zip(dims.rows, dims.width)]
    W_a1 = rng.standard_normal(size=(dims.d_hid, dims.d_in), dtype=np.float32)
    W_a1 *= np.float32(1.0 / np.sqrt(dims.d_in))
    W_a2 = rng.standard_normal(size=(dims.d, dims.d_hid), dtype=np.float32)
    W_a2 *= np.float32(1.0 / np.sqrt(dims.d_hid))
    ids = draw_ids(dims, int(n_events), rng)
    if dims.dtype == "bf16":
        tables = [round_to_bf16(t) for t in tables]
        W_a1, W_a2 = round_to_bf16(W_a1), round_to_bf16(W_a2)
    elif dims.dtype != "fp32":
        raise ValueError(f"unknown storage dtype {dims.dtype!r}")
    return TokInputs(dims=dims, tables=tables, W_a1=W_a1, W_a2=W_a2, ids=ids)
