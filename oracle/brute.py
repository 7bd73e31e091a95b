"""Form A brute force: the non-absorbed MLA layer applied to the WHOLE fused
sequence, followed by the pages' slice X[:, -T_{l+1}:, :].

Sources (LLaTTE notes, huaxiaozhuan.com):
  * appendix A.2 step 2: X_input = Concat(X_seq, Q), history first, query
    tokens appended;
  * appendix A.2 step 3: Z = RMSNorm(R + MLA(R)), X = RMSNorm(Z + FFN(Z));
    R^(l+1) = X^(l)[:, -T_{l+1}:, :] with T_l counting the query tokens;
  * appendix A.3 first display (non-absorbed MLA):
    K, V = split(RMSNorm(X W_down^KV) W_up^KV),
    MLA(X) = softmax(Q K^T / sqrt(d_k)) V W_out;
  * daiwk.github.io notes, "core formula": q_t = W_Q [x_t ; c];
  * appendix A.3 first display, low-rank query (q_rank > 0):
    Q = RMSNorm([x ; c] W_down^Q) W_up^Q.

Every row of the fused sequence is computed (also the rows the slice then
drops), with an explicit boolean mask over (row, key): a history row at fused
position i sees history keys t <= i; a query-token row sees every history key;
query tokens are never keys. This is deliberately the slow, literal order of
operations: it is what Form B (model.py), which only computes the kept rows in
the latent space, is checked against.
"""
from __future__ import annotations

import numpy as np

from .model import history_tokens


def _rms(v, g, eps):
    out = np.empty_like(v)
    for i in range(v.shape[0]):
        row = v[i]
        out[i] = row / np.sqrt(np.sum(row * row) / row.shape[0] + eps) * g
    return out


def _softmax_masked(S, mask):
    P = np.zeros_like(S)
    for i in range(S.shape[0]):
        idx = np.nonzero(mask[i])[0]
        if idx.size == 0:
            continue                      # no visible key: the attention output is zero
        s = S[i, idx]
        e = np.exp(s - s.max())
        P[i, idx] = e / e.sum()
    return P


def layer_brute(Xf: np.ndarray, T: int, c: np.ndarray, w: dict, dims):
    """Xf: fused rows [T + n_q, d] (history first). Returns all output rows."""
    f = lambda k: np.asarray(w[k], dtype=np.float64)
    h, dh, eps = dims.heads, dims.d_head, dims.eps
    N = Xf.shape[0]

    lat = Xf[:T] @ f("W_dkv").T
    C = _rms(lat, f("g_kv"), eps) if dims.kv_norm else lat          # latent of history rows
    K = C @ f("W_uk").T                                             # [T, h*dh]
    V = C @ f("W_uv").T
    Xc = np.concatenate([Xf, np.tile(c, (N, 1))], axis=1)
    if getattr(dims, "q_rank", 0):
        Q = _rms(Xc @ f("W_dq").T, f("g_q"), eps) @ f("W_uq").T        # [N, h*dh]
    else:
        Q = Xc @ f("W_q").T                                         # [N, h*dh]

    mask = np.zeros((N, T), dtype=bool)
    for i in range(N):
        for t in range(T):
            mask[i, t] = (t <= i) if i < T else True

    O = np.zeros((N, h * dh))
    for j in range(h):
        blk = slice(j * dh, (j + 1) * dh)
        S = (Q[:, blk] @ K[:, blk].T) / np.sqrt(dh)
        P = _softmax_masked(S, mask)
        O[:, blk] = P @ V[:, blk]
    A = O @ f("W_o").T

    Z = _rms(Xf + A, f("g1"), eps)
    hid = Z @ f("W1").T
    hid = hid / (1.0 + np.exp(-hid))
    X = _rms(Z + hid @ f("W2").T, f("g2"), eps)
    return X


def forward_brute(inputs, users=None, return_counts: bool = False):
    """Form A forward for the chosen users. Same output convention as
    model.forward. With return_counts, also per user the list of per-layer
    (fused rows in, history rows in, fused rows kept) integers."""
    dims = inputs.dims
    users = range(inputs.batch) if users is None else users
    outs, counts = [], []
    for u in users:
        a, b = int(inputs.offsets[u]), int(inputs.offsets[u + 1])
        Xf = np.concatenate([history_tokens(inputs, u),
                             np.asarray(inputs.cand[u], np.float64)], axis=0)
        T = b - a
        c = np.asarray(inputs.ctx[u], np.float64)
        cu = []
        for l, w in enumerate(inputs.layers):
            X = layer_brute(Xf, T, c, w, dims)
            T_next = min(T, dims.keep[l])
            rows_next = T_next + dims.n_q          # the pages' T_{l+1}, query tokens included
            cu.append((Xf.shape[0], T, rows_next))
            Xf = X[X.shape[0] - rows_next:]
            T = T_next
        counts.append(cu)
        if dims.d_out > 0:
            m = Xf.mean(axis=0) if Xf.shape[0] > 0 else np.zeros(dims.d)
            outs.append(np.asarray(inputs.W_e, np.float64) @ m)
        else:
            outs.append(Xf[T:])
    out = np.stack(outs)
    return (out, counts) if return_counts else out
