"""Seeded input generator (NumPy PCG64).

Draw order, fixed so that every consumer sees the same numbers for a seed:
  1. per-user history lengths
  2. W_sem (only for workloads with a semantic-content term)
  3. history tokens x: ID part N(0,1), then semantic codes N(0,1) (if any)
  4. candidate tokens: ID part, then semantic codes (if any)
  5. context vectors c ~ N(0,1)
  6. weights, layer by layer, in the order
     W_dkv, g_kv, W_q, W_uk, W_uv, W_o, g1, W1, W2, g2
     (matrices N(0, 1/fan_in); gains are 1 unless random gains are asked for,
     then N(1, 0.1^2)); with a low-rank query, W_q is replaced by
     W_dq [q_rank, d + d_ctx], g_q [q_rank], W_uq [h*d_h, q_rank] drawn in
     that order at its place
  7. W_e (readout) when d_out > 0.
  Event ages (hours before the request, for the timestamp encoding when
  d_time > 0) come from a generator of their own: make_event_ages with seed
  + 7919.
  8. sequence-summary weights when n_sum > 0, summary by summary:
     W_down [sum_rank, n_q*d] N(0, 1/(n_q*d)), then W_up [d_seq, sum_rank]
     N(0, 1/sum_rank).

All arrays are returned as float32 already rounded to the storage type
(round-to-nearest-even to bfloat16 for "bf16" workloads), so that the oracle
(which upcasts them to fp64) and the device path read identical values.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Dict, List, Optional

import numpy as np

from .configs import Dims, Workload

LAYER_KEYS = ("W_dkv", "g_kv", "W_q", "W_uk", "W_uv", "W_o", "g1", "W1", "W2", "g2")


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bfloat16 (ties to even), kept as float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32)
    # finite inputs cannot overflow 32 bits here (largest finite pattern + 0x8000)
    u = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
    return u.view(np.float32).reshape(a.shape)


@dataclass
class Inputs:
    dims: Dims
    lengths: np.ndarray        # int64 [B]
    offsets: np.ndarray        # int64 [B+1], exclusive prefix sum of lengths
    values: np.ndarray         # float32 [sum T, d]   history tokens, earliest first
    cand: np.ndarray           # float32 [B, n_q, d]  query tokens
    ctx: np.ndarray            # float32 [B, d_ctx]   non-sequence context
    layers: List[Dict[str, np.ndarray]]
    W_e: Optional[np.ndarray]  # float32 [d_out, d] or None
    summaries: Optional[List[Dict[str, np.ndarray]]] = None  # per summary W_down, W_up
    event_age: Optional[np.ndarray] = None  # float32 [sum T] hours before the request

    @property
    def batch(self) -> int:
        return int(self.lengths.shape[0])


def draw_lengths(spec: tuple, batch: int, rng: np.random.Generator) -> np.ndarray:
    kind = spec[0]
    if kind == "uniform":
        lo, hi = spec[1], spec[2]
        return rng.integers(lo, hi + 1, size=batch).astype(np.int64)
    if kind == "fixed":
        return np.full(batch, spec[1], dtype=np.int64)
    if kind == "lognormal":
        mu, sigma, lo, hi = spec[1:5]
        raw = rng.lognormal(mean=mu, sigma=sigma, size=batch)
        return np.clip(np.rint(raw), lo, hi).astype(np.int64)
    raise ValueError(f"unknown length law {spec!r}")


def _normal(rng, shape, std=1.0):
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return x


def draw_weights(dims: Dims, rng: np.random.Generator, random_gains: bool = False):
    d, hd, r, dc, f = dims.d, dims.heads * dims.d_head, dims.rank, dims.d_ctx, dims.d_ffn

    def gain(n):
        if random_gains:
            return (1.0 + 0.1 * rng.standard_normal(size=n)).astype(np.float32)
        return np.ones(n, dtype=np.float32)

    layers = []
    for _ in range(dims.n_layers):
        w = {}
        w["W_dkv"] = _normal(rng, (r, d), 1.0 / np.sqrt(d))
        w["g_kv"] = gain(r)
        if dims.q_rank > 0:
            rq = dims.q_rank
            w["W_dq"] = _normal(rng, (rq, d + dc), 1.0 / np.sqrt(d + dc))
            w["g_q"] = gain(rq)
            w["W_uq"] = _normal(rng, (hd, rq), 1.0 / np.sqrt(rq))
        else:
            w["W_q"] = _normal(rng, (hd, d + dc), 1.0 / np.sqrt(d + dc))
        w["W_uk"] = _normal(rng, (hd, r), 1.0 / np.sqrt(r))
        w["W_uv"] = _normal(rng, (hd, r), 1.0 / np.sqrt(r))
        w["W_o"] = _normal(rng, (d, hd), 1.0 / np.sqrt(hd))
        w["g1"] = gain(d)
        w["W1"] = _normal(rng, (f, d), 1.0 / np.sqrt(d))
        w["W2"] = _normal(rng, (d, f), 1.0 / np.sqrt(f))
        w["g2"] = gain(d)
        layers.append(w)
    W_e = _normal(rng, (dims.d_out, d), 1.0 / np.sqrt(d)) if dims.d_out > 0 else None
    return layers, W_e


def draw_summaries(dims: Dims, rng: np.random.Generator):
    """Weights of the n_sum summary MLPs (None when there are none)."""
    if dims.n_sum <= 0:
        return None
    kin = dims.n_q * dims.d
    out = []
    for _ in range(dims.n_sum):
        out.append({"W_down": _normal(rng, (dims.sum_rank, kin), 1.0 / np.sqrt(kin)),
                    "W_up": _normal(rng, (dims.d_seq, dims.sum_rank), 1.0 / np.sqrt(dims.sum_rank))})
    return out


def make_event_ages(lengths, seed: int, mean_gap_hours: float = 0.5) -> np.ndarray:
    """Hours before the request of every history event (jagged like values):
    exponential gaps between consecutive events (and between the most recent
    event and the request), so ages fall from the earliest event to the most
    recent one.  Drawn from a generator of its own (seed), after nothing else."""
    rng = np.random.Generator(np.random.PCG64(seed))
    out = []
    for T in np.asarray(lengths, dtype=np.int64):
        gaps = rng.exponential(mean_gap_hours, size=int(T))
        out.append(np.cumsum(gaps[::-1])[::-1])          # age of event t = sum of gaps t..T-1
    return np.concatenate(out).astype(np.float32) if out else np.zeros(0, np.float32)


def make_inputs(wl: Workload, batch: Optional[int] = None,
                lengths: Optional[np.ndarray] = None, seed: Optional[int] = None,
                random_gains: bool = False, dims: Optional[Dims] = None) -> Inputs:
    """Draw one batch of `wl` (optionally overriding batch size, lengths, seed, dims)."""
    dims = dims or wl.dims
    B = wl.batch if batch is None else int(batch)
    rng = np.random.Generator(np.random.PCG64(wl.seed if seed is None else seed))
    lens = draw_lengths(wl.lengths, B, rng)
    if lengths is not None:
        lens = np.asarray(lengths, dtype=np.int64).reshape(-1)
        B = lens.shape[0]
    offsets = np.zeros(B + 1, dtype=np.int64)
    np.cumsum(lens, out=offsets[1:])
    total = int(offsets[-1])
    d = dims.d

    W_sem = _normal(rng, (wl.sem_dim, d), 1.0 / np.sqrt(wl.sem_dim)) if wl.semantic else None

    def tokens(n):
        x = _normal(rng, (n, d))
        if W_sem is not None:
            codes = _normal(rng, (n, wl.sem_dim))
            x += codes @ W_sem
        return x

    values = tokens(total)
    cand = tokens(B * dims.n_q).reshape(B, dims.n_q, d)
    ctx = _normal(rng, (B, dims.d_ctx))
    layers, W_e = draw_weights(dims, rng, random_gains=random_gains)
    sums = draw_summaries(dims, rng)

    ages = None
    if dims.d_time > 0:
        ages = make_event_ages(lens, seed=(wl.seed if seed is None else seed) + 7919)

    if dims.dtype == "bf16":
        values, cand, ctx = round_to_bf16(values), round_to_bf16(cand), round_to_bf16(ctx)
        layers = [{k: round_to_bf16(v) for k, v in w.items()} for w in layers]
        W_e = round_to_bf16(W_e) if W_e is not None else None
        if sums is not None:
            sums = [{k: round_to_bf16(v) for k, v in w.items()} for w in sums]
    elif dims.dtype != "fp32":
        raise ValueError(f"unknown storage dtype {dims.dtype!r}")
    return Inputs(dims=dims, lengths=lens, offsets=offsets, values=values, cand=cand,
                  ctx=ctx, layers=layers, W_e=W_e, summaries=sums, event_age=ages)
