"""Algorithmic work of one forward pass, counted from the jagged lengths.

The count follows the cost structure of the pyramidal schedule (LLaTTE notes,
huaxiaozhuan.com appendix A.2: attention O(T_{l+1} T_l d), FFN O(T_{l+1} d^2),
i.e. projections and FFN on the kept query rows only, attention over the
visible (query, key) pairs only) with the constants of the absorbed MLA form
(appendix A.3: per-head queries in the rank-r latent, one shared K=V latent).

Per user and layer, with T history rows in, n = min(T, keep) kept, q = n + n_q:
  kv      2 T d r
  q       2 q d h r + 2 d_ctx h r          (context term once per user)
          low-rank query (rank R_q): 2 q d R_q + 2 d_ctx R_q + 2 q R_q h r
  attn    4 h r P,  P = n_q T + n T - n (n - 1) / 2  visible pairs
  o       2 q h r d
  ffn1    2 q d (m d)      ffn2  2 q (m d) d        (m = FFN multiplier)
  readout 2 d d_out per user (final layer)
Layers that run MLA in its per-head form (K, V = split(c_kv W_up^KV), scores
over d_h; same function) count what that form computes instead:
  kv      2 T d r + 2 T r (2 h d_h)        (latent, then every head's K and V)
  q       2 q d h d_h + 2 d_ctx h d_h
  attn    4 h d_h P
  o       2 q h d_h d
  summary 2 k R (n_q d + d_seq) per user: k sequence summaries, each a
          bottleneck of width R over the flattened n_q x d final query rows
          then the projection to d_seq (appendix A.2 item 4)
Masked pairs and padding are not counted.
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, List, Sequence

import numpy as np


@dataclass
class LayerWork:
    T: np.ndarray
    n: np.ndarray
    q: np.ndarray
    pairs: np.ndarray
    flops: Dict[str, float] = field(default_factory=dict)


def visible_pairs(T: np.ndarray, n: np.ndarray, n_q: int) -> np.ndarray:
    T = np.asarray(T, dtype=np.int64)
    n = np.asarray(n, dtype=np.int64)
    return n_q * T + n * T - n * (n - 1) // 2


def layer_work(lengths: Sequence[int], dims, per_head_layers: int = 0) -> List[LayerWork]:
    T = np.asarray(lengths, dtype=np.int64)
    d, h, r, dc, m = dims.d, dims.heads, dims.rank, dims.d_ctx, dims.ffn_mult
    rq = getattr(dims, "q_rank", 0)
    hd = h * dims.d_head
    out = []
    for li, k in enumerate(dims.keep):
        n = np.minimum(T, k)
        q = n + dims.n_q
        P = visible_pairs(T, n, dims.n_q)
        B = T.shape[0]
        f = {
            "kv": 2.0 * T.sum() * d * r,
            "q": (2.0 * q.sum() * d * h * r + 2.0 * B * dc * h * r) if not rq else
                 (2.0 * q.sum() * d * rq + 2.0 * B * dc * rq + 2.0 * q.sum() * rq * h * r),
            "attn": 4.0 * h * r * P.sum(),
            "o": 2.0 * q.sum() * h * r * d,
            "ffn1": 2.0 * q.sum() * d * m * d,
            "ffn2": 2.0 * q.sum() * m * d * d,
        }
        if (per_head_layers >> li) & 1:
            f["kv"] = 2.0 * T.sum() * d * r + 2.0 * T.sum() * r * 2 * hd
            f["q"] = 2.0 * q.sum() * d * hd + 2.0 * B * dc * hd
            f["attn"] = 4.0 * hd * P.sum()
            f["o"] = 2.0 * q.sum() * hd * d
        out.append(LayerWork(T=T.copy(), n=n, q=q, pairs=P, flops=f))
        T = n
    return out


def total_flops(lengths: Sequence[int], dims, per_head_layers: int = 0) -> float:
    work = layer_work(lengths, dims, per_head_layers)
    tot = sum(sum(w.flops.values()) for w in work)
    if dims.d_out:
        tot += 2.0 * len(lengths) * dims.d * dims.d_out
    tot += summary_flops(len(lengths), dims)
    return float(tot)


def summary_flops(B: int, dims) -> float:
    k = getattr(dims, "n_sum", 0)
    if not k:
        return 0.0
    return 2.0 * B * k * dims.sum_rank * (dims.n_q * dims.d + dims.d_seq)


def summary_bytes(B: int, dims, elem: int = 2) -> float:
    """Bytes the summary step must move at least: the final query rows and
    both projections read once (storage type), the summaries written (fp32)."""
    k = getattr(dims, "n_sum", 0)
    if not k:
        return 0.0
    rows = B * dims.n_q * dims.d * elem
    w = k * dims.sum_rank * (dims.n_q * dims.d + dims.d_seq) * elem
    return float(rows + w + B * k * dims.d_seq * 4)


def flops_by_step(lengths: Sequence[int], dims, per_head_layers: int = 0) -> Dict[str, float]:
    acc: Dict[str, float] = {}
    for w in layer_work(lengths, dims, per_head_layers):
        for k, v in w.flops.items():
            acc[k] = acc.get(k, 0.0) + float(v)
    if dims.d_out:
        acc["readout"] = 2.0 * len(lengths) * dims.d * dims.d_out
    acc["ffn"] = acc["ffn1"] + acc["ffn2"]      # the FFN as one fused step
    if getattr(dims, "n_sum", 0):
        acc["summary"] = summary_flops(len(lengths), dims)
    return acc


def io_bytes(lengths: Sequence[int], dims, elem: int = 2) -> float:
    """Bytes a forward must move at least: the inputs read once, the
    weights read once, the outputs written once (fp32)."""
    lengths = np.asarray(lengths, dtype=np.int64)
    B = lengths.shape[0]
    d, hd, r, dc, f = dims.d, dims.heads * dims.d_head, dims.rank, dims.d_ctx, dims.d_ffn
    inp = (lengths.sum() + B * dims.n_q) * d * elem + B * dc * elem + (B + 1) * 8
    rq = getattr(dims, "q_rank", 0)
    qw = rq * (d + dc) + rq + hd * rq if rq else hd * (d + dc)
    per_layer_w = (r * d + r + qw + 2 * hd * r + d * hd + 2 * d + 2 * f * d) * elem
    w = dims.n_layers * per_layer_w + dims.d_out * d * elem
    k = getattr(dims, "n_sum", 0)
    if k:
        w += k * dims.sum_rank * (dims.n_q * d + dims.d_seq) * elem
        out = B * k * dims.d_seq * 4
    else:
        out = B * (dims.d_out if dims.d_out else dims.n_q * d) * 4
    return float(inp + w + out)


def tokenizer_flops(tdims) -> float:
    """Algorithmic FLOPs of the action tokenizer per event: the two MLP_act
    products, 2 D_in d_hid + 2 d_hid d."""
    return 2.0 * tdims.d_in * tdims.d_hid + 2.0 * tdims.d_hid * tdims.d


def tokenizer_bytes(tdims) -> float:
    """Algorithmic bytes of the action tokenizer per event: its ids read, its
    embedding rows read once, its token written once (storage type)."""
    e = 2 if tdims.dtype == "bf16" else 4
    return 4.0 * tdims.n_fields + e * tdims.d_in + e * tdims.d
