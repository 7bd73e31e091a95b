"""Form B of the layer: MLA as multi-query attention in the latent space, fp64.

Sources:
  * LLaTTE notes (huaxiaozhuan.com), appendix A.3: the KV latent
    RMSNorm(X W_down^KV); W_up^Q and (W_up^KV)^T fuse into one matrix acting
    on the query; the V half of W_up^KV folds into W_out; the result is MQA
    over the shared latent.
  * appendix A.2 display: Z = RMSNorm(R + MLA(R)), X = RMSNorm(Z + FFN(Z)),
    and the pyramid slice of the last T_{l+1} rows.
  * daiwk.github.io notes, "core formula": target-aware query
    q_t = W_Q [x_t ; c], h_t = sum_i softmax_i(q_t.k_i / sqrt(d)) W_V x_i.
  * appendix A.3 first display, the low-rank query of the MLA
    parameterisation: Q = RMSNorm(X W_down^Q) W_up^Q (when q_rank > 0).

Readings: the softmax scale is 1/sqrt(d_h) in both forms (the absorbed
display's sqrt(d_c) is read as garbled: only the same scale keeps the two forms
equal); history query at position p sees keys t <= p; a candidate sees every
history key of the current layer and no query token; with no visible key the
attention output is zero; RMSNorm(v) = v / sqrt(mean(v^2) + eps) * g;
FFN(z) = W2 SiLU(W1 z), SiLU(x) = x / (1 + exp(-x)), no biases; a sequence
summary is W_up SiLU(W_down Flatten(Z_raw)) (see `summaries`).

Low-rank query reading: the down-projection acts on the target-aware input
[x ; c] (so the query stays target-aware), with its own RMSNorm gain g_q;
W_up^Q then absorbs into the key up-projection like W_Q does.

Absorbed matrices per head j (rows j*d_h:(j+1)*d_h of the per-head blocks):
  W_QK_j = W_uk_j^T W_q_j / sqrt(d_h)      (r x (d + d_ctx))
  W_QK_j = W_uk_j^T W_uq_j / sqrt(d_h)     (r x q_rank, low-rank query)
  W_OV_j = W_o[:, j-block] W_uv_j          (d x r)
"""
from __future__ import annotations

from typing import List, Optional, Sequence

import numpy as np

from .plan import plan_layers


def time_encoding(ages: np.ndarray, d_time: int) -> np.ndarray:
    """Additive timestamp encoding of history events (LLaTTE notes,
    huaxiaozhuan.com, appendix A.2 item 1: added on a subset of the hidden
    dims).  Reading (the pages give no formula): the sinusoidal code of the
    Transformer applied to the event's age a in hours before the request, on
    the first d_time dims: pair i = 0 .. d_time/2 - 1 holds
    (sin(a w_i), cos(a w_i)) with w_i = 10000^(-2i / d_time).  [T, d_time]."""
    a = np.asarray(ages, dtype=np.float64).reshape(-1, 1)
    w = 10000.0 ** (-2.0 * np.arange(d_time // 2) / d_time)
    te = np.empty((a.shape[0], d_time))
    te[:, 0::2] = np.sin(a * w)
    te[:, 1::2] = np.cos(a * w)
    return te


def history_tokens(inputs, u: int) -> np.ndarray:
    """User u's history tokens as the first layer sees them: the input rows,
    plus the timestamp encoding on the first d_time dims when d_time > 0."""
    a, b = int(inputs.offsets[u]), int(inputs.offsets[u + 1])
    H = _f64(inputs.values[a:b]).copy()
    dt = getattr(inputs.dims, "d_time", 0)
    if dt:
        H[:, :dt] += time_encoding(inputs.event_age[a:b], dt)
    return H


def rmsnorm(v: np.ndarray, g: np.ndarray, eps: float) -> np.ndarray:
    ms = np.mean(v * v, axis=-1, keepdims=True)
    return v / np.sqrt(ms + eps) * g


def silu(x: np.ndarray) -> np.ndarray:
    return x / (1.0 + np.exp(-x))


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def absorb(w: dict, dims) -> dict:
    """Per-head absorbed matrices in fp64 from the non-absorbed weights."""
    h, dh = dims.heads, dims.d_head
    W_q = _f64(w["W_uq"] if getattr(dims, "q_rank", 0) else w["W_q"])
    W_uk, W_uv, W_o = _f64(w["W_uk"]), _f64(w["W_uv"]), _f64(w["W_o"])
    scale = 1.0 / np.sqrt(dh)
    W_QK, W_OV = [], []
    for j in range(h):
        blk = slice(j * dh, (j + 1) * dh)
        W_QK.append(W_uk[blk].T @ W_q[blk] * scale)
        W_OV.append(W_o[:, blk] @ W_uv[blk])
    return {"W_QK": W_QK, "W_OV": W_OV}


def layer_forward(H: np.ndarray, Y: np.ndarray, c: np.ndarray, w: dict, ab: dict, dims,
                  keep: int, probs: Optional[list] = None):
    """One layer for one user. H: [T, d] history (earliest first), Y: [n_q, d]
    query tokens, c: [d_ctx] context. Returns (H', Y') with T' = min(T, keep)."""
    T = H.shape[0]
    n = min(T, keep)
    eps = dims.eps

    L = H @ _f64(w["W_dkv"]).T                                   # [T, r]
    C = rmsnorm(L, _f64(w["g_kv"]), eps) if dims.kv_norm else L

    R = np.concatenate([H[T - n:], Y], axis=0)                   # query rows [q, d]
    q = R.shape[0]
    RC = np.concatenate([R, np.broadcast_to(c, (q, c.shape[0]))], axis=1)

    visible = np.zeros((q, T), dtype=bool)
    for i in range(q):
        if i < n:
            visible[i, : T - n + i + 1] = True                   # causal: keys <= own position
        else:
            visible[i, :] = True                                 # candidate: all history keys

    if getattr(dims, "q_rank", 0):
        Qin = rmsnorm(RC @ _f64(w["W_dq"]).T, _f64(w["g_q"]), eps)   # [q, q_rank]
    else:
        Qin = RC
    A = np.zeros((q, dims.d))
    for j in range(dims.heads):
        Qt = Qin @ ab["W_QK"][j].T                               # [q, r] latent queries
        S = Qt @ C.T                                             # [q, T]
        S = np.where(visible, S, -np.inf)
        P = np.zeros_like(S)
        rows = visible.any(axis=1)
        if rows.any():
            Sr = S[rows]
            Pr = np.exp(Sr - Sr.max(axis=1, keepdims=True))
            P[rows] = Pr / Pr.sum(axis=1, keepdims=True)
        if probs is not None:
            probs.append(P)
        Ot = P @ C                                               # [q, r] latent outputs
        A += Ot @ ab["W_OV"][j].T

    Z = rmsnorm(R + A, _f64(w["g1"]), eps)
    F = silu(Z @ _f64(w["W1"]).T) @ _f64(w["W2"]).T
    X = rmsnorm(Z + F, _f64(w["g2"]), eps)
    return X[:n], X[n:]


def summaries(z_raw: np.ndarray, sum_w: Sequence[dict]) -> np.ndarray:
    """Sequence summaries of one user from the final query-token rows.

    LLaTTE notes (huaxiaozhuan.com), appendix A.2 item 4 "Sequence Summaries":
    the final layer's rows at the query-token positions, Z_raw [n_q, d], are
    flattened and each of k low-rank adapted MLPs maps the flat vector to a
    fixed-size summary Z_seq^(k) of width d_seq.

    Reading (the pages name the block but give no formula): Flatten is
    row-major, token 0's d values first; LoRAMLP_k(v) = W_up,k SiLU(W_down,k v)
    with W_down,k [sum_rank, n_q*d] the low-rank bottleneck and W_up,k
    [d_seq, sum_rank], no biases (the layers have none either), SiLU as in
    the FFN.  Returns [k, d_seq].
    """
    v = _f64(z_raw).reshape(-1)
    return np.stack([_f64(w["W_up"]) @ silu(_f64(w["W_down"]) @ v) for w in sum_w])


def forward(inputs, users: Optional[Sequence[int]] = None, return_probs: bool = False,
            return_layers: bool = False):
    """fp64 forward of the whole sequence module for the chosen users.

    Returns out: [U, n_q, d] (final query-token rows) when d_out == 0 and
    n_sum == 0; [U, d_out] = W_e @ mean of the final layer's rows (zero if
    there are none) when d_out > 0; [U, n_sum, d_seq] sequence summaries of the
    final query-token rows when n_sum > 0.
    With return_probs, also a list (per user) of lists (per layer) of per-head
    probability matrices. With return_layers, also per user the list of
    (H, Y) after every layer.
    """
    dims = inputs.dims
    B = inputs.batch
    users = list(range(B)) if users is None else [int(u) for u in users]
    abs_w = [absorb(w, dims) for w in inputs.layers]
    outs, all_probs, all_layers = [], [], []
    for u in users:
        H = history_tokens(inputs, u)
        Y = _f64(inputs.cand[u])
        c = _f64(inputs.ctx[u])
        probs_u, layers_u = [], []
        for l, w in enumerate(inputs.layers):
            pl = [] if return_probs else None
            H, Y = layer_forward(H, Y, c, w, abs_w[l], dims, dims.keep[l], probs=pl)
            probs_u.append(pl)
            layers_u.append((H.copy(), Y.copy()))
        if dims.d_out > 0:
            rows = np.concatenate([H, Y], axis=0)
            m = rows.mean(axis=0) if rows.shape[0] > 0 else np.zeros(dims.d)
            outs.append(_f64(inputs.W_e) @ m)
        elif getattr(dims, "n_sum", 0) > 0:
            outs.append(summaries(Y, inputs.summaries))
        else:
            outs.append(Y)
        all_probs.append(probs_u)
        all_layers.append(layers_u)
    out = np.stack(outs) if outs else np.zeros((0,))
    res = [out]
    if return_probs:
        res.append(all_probs)
    if return_layers:
        res.append(all_layers)
    return res[0] if len(res) == 1 else tuple(res)


def layer_counts(inputs) -> List:
    """Per-layer schedule integers for the whole batch (see plan.py)."""
    return plan_layers(inputs.lengths, inputs.dims.keep, inputs.dims.n_q)
