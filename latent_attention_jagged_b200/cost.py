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


def bytes_by_step(lengths: Sequence[int], dims, per_head_layers: int = 0,
                  tensor_cores: bool = True) -> Dict[str, float]:
    """HBM bytes each step must move at least in this library's data flow:
    the step's inputs read once, its weights read once, its outputs written
    once (the rows that pass between steps live in HBM by design).

    Per layer, with T history rows in, n kept, q = n + n_q query rows, storage
    element e (2 for bf16), and the fp16 residual copies of the bf16 path:
      gather   read  sum T d e + B n_q d e          (history events, query tokens)
               write sum T d e + sum q_0 d e        (key rows, query rows)
                     + 4 sum_l sum q_l              (row -> user maps)
      kv       read  sum T d e + r d e              write sum T r e
               per-head form: + read sum T r e + 2 h d_h r e, write sum T 2 h d_h e
      q        read  sum q d e + w_q e + 4 B w      write sum q w e   (w = h r, or h d_h)
      attn     read  sum q w e + sum T r e          write sum q w e   (latent keys once per user;
               per-head form: the K | V rows, sum T 2 h d_h e)
      o        read  sum q w e + sum q d 2 + d w e  write sum q d 2   (fp16 Z)
      ffn      read  sum q d 2 + 2 f d e            write the next layer's rows
               (sum n d e history + sum q' d 2 query rows), or the fp32 output
               rows of the last layer (sum n_q d 4, or sum q d 4 for the readout)
      ffn1     read  sum q d 2 + f d e              write sum q f e
      ffn2     read  sum q f e + sum q d 2 + f d e  write as ffn
      readout  read  sum q_L d 4 + d_out d e        write B d_out 4
    """
    T = np.asarray(lengths, dtype=np.int64)
    B = T.shape[0]
    e = 2 if dims.dtype == "bf16" else 4
    res = 2 if e == 2 else 4                     # residual-stream copies
    d, h, r, dh, nq = dims.d, dims.heads, dims.rank, dims.d_head, dims.n_q
    f = dims.ffn_mult * d
    acc: Dict[str, float] = {}

    def add(k, v):
        acc[k] = acc.get(k, 0.0) + float(v)

    L = dims.n_layers
    Ts, ns = [], []
    t = T.copy()
    for k in dims.keep:
        n = np.minimum(t, k)
        Ts.append(t)
        ns.append(n)
        t = n
    qs = [n + nq for n in ns]
    add("gather", T.sum() * d * e + B * nq * d * e + T.sum() * d * e + qs[0].sum() * d * e
        + 4 * sum(q.sum() for q in qs))
    for l in range(L):
        Tl, nl, ql = Ts[l].sum(), ns[l].sum(), qs[l].sum()
        ph = (per_head_layers >> l) & 1
        w = h * dh if ph else h * r
        add("kv", Tl * d * e + r * d * e + Tl * r * e)
        if ph:
            add("kv", Tl * r * e + 2 * h * dh * r * e + Tl * 2 * h * dh * e)
        add("q", ql * d * e + w * (d + dims.d_ctx) * e + 4 * B * w + ql * w * e)
        add("attn", ql * w * e + (Tl * 2 * h * dh * e if ph else Tl * r * e) + ql * w * e)
        add("o", ql * w * e + ql * d * res + d * w * e + ql * d * res)
        if l == L - 1:
            out = (ql * d * 4) if dims.d_out else (B * nq * d * 4)
        else:
            out = ns[l].sum() * d * e + qs[l + 1].sum() * d * res
        add("ffn", ql * d * res + 2 * f * d * e + out)
        add("ffn1", ql * d * res + f * d * e + ql * f * e)
        add("ffn2", ql * f * e + ql * d * res + f * d * e + out)
    if dims.d_out:
        add("readout", qs[-1].sum() * d * 4 + dims.d_out * d * e + B * dims.d_out * 4)
    return acc


def step_roofline(flops: float, nbytes: float, ms: float, peak_tflops: float,
                  peak_gbs: float) -> Dict[str, float]:
    """Roofline of one step: the slower of its FLOPs at the tensor peak and its
    bytes at the HBM bandwidth, against the measured time."""
    s = ms / 1e3
    t_f = flops / (peak_tflops * 1e12) if flops else 0.0
    t_b = nbytes / (peak_gbs * 1e9) if nbytes else 0.0
    return {"ms": ms, "flops": flops, "bytes": nbytes,
            "tflops": flops / s / 1e12 if s > 0 else 0.0,
            "gbs": nbytes / s / 1e9 if s > 0 else 0.0,
            "frac_tensor": t_f / s if s > 0 else 0.0,
            "frac_hbm": t_b / s if s > 0 else 0.0,
            "bound": "tensor" if t_f >= t_b else "hbm",
            "frac": max(t_f, t_b) / s if s > 0 else 0.0}
