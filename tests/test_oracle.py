"""Pins for the fp64 oracle: it is checked against things other than itself.

* Form A (non-absorbed MLA on the whole fused sequence + the pages' slice,
  LLaTTE notes appendix A.2/A.3) equals Form B (absorbed latent MQA on the
  kept rows only): the absorption identity of appendix A.3.
* Textbook reduction: with no KV norm, r = d, W_down^KV = I, the layer is
  standard causal multi-head attention + post-norm + SiLU FFN; compared with
  torch's scaled_dot_product_attention / rms_norm / silu / linear on float64.
* One key (T = 1): the attention output is the value of that key whatever the
  query (daiwk.github.io "core formula" with a single term in the sum).
* Identical keys: the probabilities are uniform over the visible keys.
* Probability rows sum to one and are zero exactly where the causal /
  candidate mask hides a key.
* Key-permutation invariance of candidate outputs in cross mode (no
  positional term anywhere in the layer).
* Post-norm: every output row has RMS 1 when the final gain is 1.
* Pyramid integers against the fused-sequence slice and against the pages'
  three modes (golden fixture).
* The FLOP counter's visible-pair count against the oracle's masks.
"""
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle.plan import plan_layers
from latent_attention_jagged_b200 import cost
from workloads import Dims, Workload, make_inputs, workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _wl(dims, lengths=("uniform", 1, 8), seed=7, batch=3):
    return Workload(name="t", dims=dims, batch=batch, lengths=lengths, seed=seed)


def small_dims(**kw):
    base = dict(d=16, heads=2, d_head=8, rank=12, d_ctx=5, n_q=3, keep=(9, 4), dtype="fp32")
    base.update(kw)
    return Dims(**base)


# ---------------------------------------------------------------- Form A == Form B

@pytest.mark.parametrize("lengths", [[0, 1, 2, 5, 9, 13], [1], [20, 3], [0, 0]])
@pytest.mark.parametrize("dkw", [
    dict(),
    dict(n_q=0, d_ctx=0),
    dict(keep=(6, 6, 0)),                 # full, pyramidal, cross (keep = 0)
    dict(keep=(0,)),
    dict(kv_norm=0),
    dict(d_out=7, keep=(10, 3)),
    dict(heads=3, d_head=4, rank=20),     # r > h*d_h
    dict(q_rank=5),                       # low-rank RMSNorm'd query
    dict(q_rank=21, d_ctx=0, keep=(6, 0)),
])
def test_absorbed_equals_non_absorbed(lengths, dkw):
    dims = small_dims(**dkw)
    inp = make_inputs(_wl(dims), lengths=lengths, random_gains=True)
    a = oracle.forward(inp)
    b = oracle.forward_brute(inp)
    assert a.shape == b.shape
    if a.size:
        scale = max(1.0, float(np.abs(b).max()))
        assert np.abs(a - b).max() <= 1e-11 * scale


@pytest.mark.parametrize("name", ["tiny", "tiny_lq"])
def test_absorbed_equals_non_absorbed_tiny_workload(name):
    inp = make_inputs(workload(name))
    a = oracle.forward(inp)
    b = oracle.forward_brute(inp)
    assert np.abs(a - b).max() < 1e-12


# ---------------------------------------------------------------- textbook MHA

def _textbook_layer(x, c, w, dims, causal_rows, cand):
    """Standard MHA + post-norm + SiLU FFN, written with torch library routines.
    x: history [T, d], cand: [n_q, d]. Returns outputs of history and cand rows."""
    t = lambda a: torch.as_tensor(np.asarray(a, dtype=np.float64))
    h, dh, d = dims.heads, dims.d_head, dims.d
    X, Y = t(x), t(cand)
    cc = t(c)

    def q_of(rows):
        xc = torch.cat([rows, cc.expand(rows.shape[0], -1)], 1)
        if dims.q_rank:                           # Q = RMSNorm([x; c] W_down^Q) W_up^Q
            lat = F.rms_norm(F.linear(xc, t(w["W_dq"])), (dims.q_rank,), weight=t(w["g_q"]),
                             eps=dims.eps)
            return F.linear(lat, t(w["W_uq"]))
        return F.linear(xc, t(w["W_q"]))

    k = F.linear(X, t(w["W_uk"]))                 # C = X because W_dkv = I, no norm
    v = F.linear(X, t(w["W_uv"]))
    split = lambda m: m.reshape(m.shape[0], h, dh).transpose(0, 1)
    outs = []
    if X.shape[0]:
        oh = F.scaled_dot_product_attention(split(q_of(X)), split(k), split(v), is_causal=True)
        outs.append((X, oh.transpose(0, 1).reshape(X.shape[0], h * dh)))
    if Y.shape[0]:
        if X.shape[0]:
            oc = F.scaled_dot_product_attention(split(q_of(Y)), split(k), split(v))
            oc = oc.transpose(0, 1).reshape(Y.shape[0], h * dh)
        else:
            oc = torch.zeros(Y.shape[0], h * dh, dtype=torch.float64)
        outs.append((Y, oc))
    res = []
    for R, o in outs:
        Z = F.rms_norm(R + F.linear(o, t(w["W_o"])), (d,), weight=t(w["g1"]), eps=dims.eps)
        Hd = F.silu(F.linear(Z, t(w["W1"])))
        res.append(F.rms_norm(Z + F.linear(Hd, t(w["W2"])), (d,), weight=t(w["g2"]),
                              eps=dims.eps).numpy())
    hist = res[0] if X.shape[0] else np.zeros((0, d))
    cnd = res[-1] if Y.shape[0] else np.zeros((0, d))
    return hist, cnd


@pytest.mark.parametrize("n_q,d_ctx,keep,q_rank", [
    (0, 0, (11, 6), 0), (3, 4, (11, 6), 0), (2, 0, (5, 0), 0), (4, 3, (0,), 0),
    (3, 4, (11, 6), 5), (2, 0, (7, 0), 9)])
def test_textbook_reduction(n_q, d_ctx, keep, q_rank):
    d = 12
    dims = Dims(d=d, heads=3, d_head=4, rank=d, d_ctx=d_ctx, n_q=n_q, keep=keep,
                kv_norm=0, dtype="fp32", q_rank=q_rank)
    inp = make_inputs(_wl(dims, batch=2), lengths=[11, 7], random_gains=True)
    for w in inp.layers:
        w["W_dkv"] = np.eye(d, dtype=np.float32)
    _, layers = oracle.forward(inp, return_layers=True)
    for u in range(2):
        a, b = inp.offsets[u], inp.offsets[u + 1]
        H, Y = inp.values[a:b].astype(np.float64), inp.cand[u].astype(np.float64)
        c = inp.ctx[u]
        for l, w in enumerate(inp.layers):
            hist, cnd = _textbook_layer(H, c, w, dims, True, Y)
            n = min(H.shape[0], keep[l])
            H, Y = hist[hist.shape[0] - n:], cnd      # pyramid: keep the last n rows
            Ho, Yo = layers[u][l]
            np.testing.assert_allclose(Ho, H, rtol=0, atol=1e-12)
            np.testing.assert_allclose(Yo, Y, rtol=0, atol=1e-12)


def test_low_rank_query_is_scale_invariant_in_its_down_projection():
    """RMSNorm on the query latent: scaling W_down^Q by any positive factor
    leaves the layer unchanged (with eps -> 0); a full-rank or un-normed query
    would change."""
    dims = small_dims(q_rank=6, eps=1e-30)
    inp = make_inputs(_wl(dims), lengths=[9, 4, 1], random_gains=True)
    a = oracle.forward(inp)
    for w in inp.layers:
        w["W_dq"] = w["W_dq"] * np.float32(8.0)
    b = oracle.forward(inp)
    np.testing.assert_allclose(a, b, rtol=0, atol=1e-12)
    for w in inp.layers:
        w["W_uq"] = w["W_uq"] * np.float32(2.0)        # the up-projection is not normed
    c = oracle.forward(inp)
    assert np.abs(c - a).max() > 1e-3


# ---------------------------------------------------------------- special cases

def _one_layer(dims, lengths, mutate=None, seed=3):
    inp = make_inputs(_wl(dims, seed=seed), lengths=lengths, random_gains=True)
    if mutate:
        mutate(inp)
    return inp


def test_one_key_output_independent_of_query():
    """T = 1: softmax over one key is 1, so W_q and W_uk cannot matter."""
    dims = small_dims(keep=(1,), n_q=4)
    base = _one_layer(dims, [1, 1, 1])
    out0, lay0 = oracle.forward(base, return_layers=True)
    rng = np.random.default_rng(11)

    def scramble(inp):
        for w in inp.layers:
            w["W_q"] = rng.standard_normal(w["W_q"].shape).astype(np.float32) * 3
            w["W_uk"] = rng.standard_normal(w["W_uk"].shape).astype(np.float32) * 3

    other = _one_layer(dims, [1, 1, 1], mutate=scramble)
    out1, lay1 = oracle.forward(other, return_layers=True)
    np.testing.assert_allclose(out0, out1, atol=1e-13)
    for u in range(3):
        np.testing.assert_allclose(lay0[u][0][0], lay1[u][0][0], atol=1e-13)


def test_identical_keys_uniform_probabilities_and_query_independent():
    dims = small_dims(keep=(6,), n_q=3)

    def same_rows(inp):
        for u in range(inp.batch):
            a, b = inp.offsets[u], inp.offsets[u + 1]
            inp.values[a:b] = inp.values[a]

    inp = _one_layer(dims, [6, 4], mutate=same_rows)
    out, probs = oracle.forward(inp, return_probs=True)
    for u, T in enumerate([6, 4]):
        n = min(T, 6)
        for P in probs[u][0]:
            for i in range(P.shape[0]):
                vis = (T - n + i + 1) if i < n else T
                np.testing.assert_allclose(P[i, :vis], 1.0 / vis, rtol=1e-14)
                assert np.all(P[i, vis:] == 0)

    def scramble(inp2):
        same_rows(inp2)
        r = np.random.default_rng(5)
        inp2.layers[0]["W_q"] = r.standard_normal(inp2.layers[0]["W_q"].shape).astype(np.float32)

    out2 = oracle.forward(_one_layer(dims, [6, 4], mutate=scramble))
    np.testing.assert_allclose(out, out2, atol=1e-13)


def test_probability_rows_sum_to_one_and_mask_pattern():
    dims = small_dims(keep=(7, 3), n_q=2)
    inp = make_inputs(_wl(dims), lengths=[0, 1, 9, 4], random_gains=True)
    _, probs = oracle.forward(inp, return_probs=True)
    plans = plan_layers(inp.lengths, dims.keep, dims.n_q)
    for u in range(4):
        for l in range(dims.n_layers):
            T, n = int(plans[l].T[u]), int(plans[l].n[u])
            for P in probs[u][l]:
                assert P.shape == (n + dims.n_q, T)
                for i in range(P.shape[0]):
                    vis = (T - n + i + 1) if i < n else T
                    if vis == 0:
                        assert np.all(P[i] == 0)
                        continue
                    assert abs(P[i].sum() - 1.0) < 1e-14
                    assert np.all(P[i, :vis] > 0) and np.all(P[i, vis:] == 0)


def test_cross_mode_key_permutation_invariance():
    dims = small_dims(keep=(0,), n_q=4)
    inp = make_inputs(_wl(dims), lengths=[9, 5], random_gains=True)
    out = oracle.forward(inp)
    perm = make_inputs(_wl(dims), lengths=[9, 5], random_gains=True)
    rng = np.random.default_rng(2)
    for u in range(2):
        a, b = perm.offsets[u], perm.offsets[u + 1]
        perm.values[a:b] = perm.values[a:b][rng.permutation(b - a)]
    np.testing.assert_allclose(oracle.forward(perm), out, atol=1e-13)


def test_causal_history_is_order_sensitive():
    """Control for the test above: history rows are causal, so order matters."""
    dims = small_dims(keep=(9,), n_q=0, d_ctx=0)
    inp = make_inputs(_wl(dims), lengths=[9], random_gains=True)
    _, lay = oracle.forward(inp, return_layers=True)
    perm = make_inputs(_wl(dims), lengths=[9], random_gains=True)
    perm.values[:] = perm.values[::-1]
    _, lay2 = oracle.forward(perm, return_layers=True)
    assert np.abs(lay[0][0][0][::-1] - lay2[0][0][0]).max() > 1e-3


def test_post_norm_rows_have_unit_rms():
    inp = make_inputs(workload("tiny"))
    out, lay = oracle.forward(inp, return_layers=True)
    rms = np.sqrt((out ** 2).mean(-1))
    assert np.abs(rms - 1).max() < 1e-5
    for u in range(inp.batch):
        for H, Y in lay[u]:
            if H.shape[0]:
                assert np.abs(np.sqrt((H ** 2).mean(-1)) - 1).max() < 1e-5


def test_readout_is_mean_then_linear():
    dims = small_dims(d_out=6, keep=(8, 2))
    inp = make_inputs(_wl(dims), lengths=[0, 3, 12], random_gains=True)
    out, lay = oracle.forward(inp, return_layers=True)
    for u in range(3):
        H, Y = lay[u][-1]
        rows = torch.as_tensor(np.concatenate([H, Y], 0))
        proj = F.linear(rows, torch.as_tensor(inp.W_e.astype(np.float64)))
        np.testing.assert_allclose(out[u], proj.mean(0).numpy(), atol=1e-13)


def test_empty_history_candidates_see_nothing():
    """T = 0: no visible key, the attention output is zero, so the layer is the
    post-norm FFN block applied to RMSNorm(query token)."""
    dims = small_dims(keep=(4,), n_q=3)
    inp = make_inputs(_wl(dims), lengths=[0], random_gains=True)
    out = oracle.forward(inp)
    w = inp.layers[0]
    t = lambda a: torch.as_tensor(np.asarray(a, dtype=np.float64))
    Z = F.rms_norm(t(inp.cand[0]), (dims.d,), weight=t(w["g1"]), eps=dims.eps)
    X = F.rms_norm(Z + F.linear(F.silu(F.linear(Z, t(w["W1"]))), t(w["W2"])), (dims.d,),
                   weight=t(w["g2"]), eps=dims.eps)
    np.testing.assert_allclose(out[0], X.numpy(), atol=1e-13)


# ---------------------------------------------------------------- integers

def test_plan_matches_fused_sequence_slices():
    dims = small_dims(keep=(10, 6, 6, 2, 0), n_q=3)
    lengths = [0, 1, 2, 6, 7, 15]
    inp = make_inputs(_wl(dims), lengths=lengths)
    _, counts = oracle.forward_brute(inp, return_counts=True)
    plans = plan_layers(lengths, dims.keep, dims.n_q)
    for u in range(len(lengths)):
        for l, (rows_in, T_in, rows_out) in enumerate(counts[u]):
            assert plans[l].T[u] == T_in
            assert rows_in == T_in + dims.n_q
            assert plans[l].n[u] + dims.n_q == rows_out
            q = plans[l].query_off
            assert q[u + 1] - q[u] == rows_out
            h = plans[l].hist_off
            assert h[u + 1] - h[u] == T_in
    assert plans[0].hist_off[-1] == sum(lengths)


def test_plan_rejects_increasing_schedule():
    with pytest.raises(ValueError):
        plan_layers([5], (2, 3), 0)


def _read_golden(name):
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            kv = dict(tok.split("=", 1) for tok in line.split())
            rows.append(kv)
    return rows


def test_pyramid_modes_golden():
    ints = lambda s: [int(v) for v in s.split(",")]
    for row in _read_golden("pyramid_modes.txt"):
        T, n_q, keep = int(row["T"]), int(row["n_q"]), ints(row["keep"])
        plans = plan_layers([T], keep, n_q)
        rows_in = [int(p.T[0]) + n_q for p in plans]
        rows_out = [int(p.n[0]) + n_q for p in plans]
        assert rows_in == ints(row["rows_in"])
        assert rows_out == ints(row["rows_out"])
        modes = []
        for p in plans:
            Tl = int(p.n[0]) + n_q           # the pages' T_{l+1}, query tokens included
            if Tl == int(p.T[0]) + n_q:
                modes.append("full")
            elif Tl == n_q:
                modes.append("cross")
            else:
                modes.append("pyramidal")
        assert modes == row["modes"].split(",")


def test_flop_counter_pairs_match_oracle_masks():
    dims = small_dims(keep=(7, 3), n_q=2)
    lengths = [0, 1, 9, 4, 7]
    inp = make_inputs(_wl(dims), lengths=lengths)
    _, probs = oracle.forward(inp, return_probs=True)
    work = cost.layer_work(lengths, dims)
    for l in range(dims.n_layers):
        for u in range(len(lengths)):
            nz = int(np.count_nonzero(probs[u][l][0]))
            assert work[l].pairs[u] == nz


def test_flop_counter_reference_totals():
    """Hand-derivable totals: one user, T = 4, keep 4 then 2, n_q = 1."""
    dims = Dims(d=8, heads=2, d_head=4, rank=6, d_ctx=3, n_q=1, keep=(4, 2), dtype="fp32")
    by = cost.flops_by_step([4], dims)
    # layer 1: T=4, n=4, q=5, P = 1*4 + 10 = 14;  layer 2: T=4, n=2, q=3, P = 4 + (4+3) = 11
    assert by["kv"] == 2 * 8 * 6 * (4 + 4)
    assert by["attn"] == 4 * 2 * 6 * (14 + 11)
    assert by["q"] == 2 * 8 * 2 * 6 * (5 + 3) + 2 * 2 * 3 * 2 * 6
    assert by["ffn1"] == by["ffn2"] == 2 * 8 * 32 * (5 + 3)
