"""Pins of the fp64 action tokenizer (MLP_act over per-field embeddings).

LLaTTE notes (huaxiaozhuan.com), appendix A.2 item 1 "Action Embeddings":
x_t = MLP_act(E_type(type_t), E_item(item_t), E_surface(surface_t),
E_time(tau_t), E_meta(meta_t)).  The oracle reads MLP_act as
W_a2 SiLU(W_a1 [e_1; ...; e_F]) without biases.  These checks tie it to
things other than itself: torch's embedding / linear / SiLU modules, the
tanh form of SiLU, one-hot selections, and structural invariants.
"""
import numpy as np
import pytest
import torch

from oracle.tokenizer import action_tokens, embed
from workloads.tokens import TOKENIZERS, TokDims, make_token_inputs


def _torch_tokens(ti):
    """The same map built from torch modules in float64."""
    embs = [torch.nn.Embedding.from_pretrained(torch.from_numpy(t.astype(np.float64)))
            for t in ti.tables]
    ids = torch.from_numpy(ti.ids.astype(np.int64))
    e = torch.cat([m(ids[:, f]) for f, m in enumerate(embs)], dim=1)
    l1 = torch.nn.Linear(ti.dims.d_in, ti.dims.d_hid, bias=False, dtype=torch.float64)
    l2 = torch.nn.Linear(ti.dims.d_hid, ti.dims.d, bias=False, dtype=torch.float64)
    with torch.no_grad():
        l1.weight.copy_(torch.from_numpy(ti.W_a1.astype(np.float64)))
        l2.weight.copy_(torch.from_numpy(ti.W_a2.astype(np.float64)))
        return l2(torch.nn.SiLU()(l1(e))).numpy()


@pytest.mark.parametrize("name", ["tiny", "odd_bf16"])
def test_matches_torch_modules(name):
    ti = make_token_inputs(TOKENIZERS[name], 300, seed=11)
    got = action_tokens(ti.ids, ti.tables, ti.W_a1, ti.W_a2)
    np.testing.assert_allclose(got, _torch_tokens(ti), rtol=1e-12, atol=1e-12)


def test_identity_weights_give_silu_of_embeddings_tanh_form():
    # W_a1 = I, W_a2 = I: x = SiLU(e) = (e/2)(1 + tanh(e/2)) elementwise
    dims = TokDims(rows=(5, 7), width=(3, 5), d_hid=8, d=8, dtype="fp32")
    ti = make_token_inputs(dims, 40, seed=3)
    eye = np.eye(8, dtype=np.float32)
    got = action_tokens(ti.ids, ti.tables, eye, eye)
    e = np.concatenate([ti.tables[0][ti.ids[:, 0]], ti.tables[1][ti.ids[:, 1]]], axis=1)
    e = e.astype(np.float64)
    np.testing.assert_allclose(got, 0.5 * e * (1.0 + np.tanh(0.5 * e)), rtol=1e-13, atol=1e-15)


def test_one_hot_weights_select_one_table_entry():
    # W_a1 row k picks concatenated column c; W_a2 routes hidden unit k to
    # output j with gain 2: x[:, j] = 2 SiLU(table_f[id_f, c - start_f])
    ti = make_token_inputs(TOKENIZERS["tiny"], 64, seed=5)
    dims = ti.dims
    starts = np.concatenate([[0], np.cumsum(dims.width)])
    W1 = np.zeros((dims.d_hid, dims.d_in), np.float32)
    W2 = np.zeros((dims.d, dims.d_hid), np.float32)
    picks = [(0, 1, 3), (1, 20, 9), (2, 33, 0), (4, 47, 63)]      # (hidden k, column c, out j)
    for k, c, j in picks:
        W1[k, c] = 1.0
        W2[j, k] = 2.0
    got = action_tokens(ti.ids, ti.tables, W1, W2)
    for k, c, j in picks:
        f = int(np.searchsorted(starts, c, side="right") - 1)
        v = ti.tables[f][ti.ids[:, f], c - starts[f]].astype(np.float64)
        np.testing.assert_allclose(got[:, j], 2 * 0.5 * v * (1 + np.tanh(0.5 * v)),
                                   rtol=1e-13, atol=1e-15)
    untouched = sorted(set(range(dims.d)) - {j for _, _, j in picks})
    assert np.all(got[:, untouched] == 0.0)


def test_embedding_concatenates_fields_in_table_order():
    ti = make_token_inputs(TOKENIZERS["tiny"], 16, seed=2)
    e = embed(ti.ids, ti.tables)
    col = 0
    for f, t in enumerate(ti.tables):
        w = t.shape[1]
        assert np.array_equal(e[:, col:col + w], t[ti.ids[:, f]].astype(np.float64))
        col += w
    assert col == e.shape[1] == ti.dims.d_in


def test_tokens_are_per_event_equal_ids_equal_tokens_and_permutation():
    ti = make_token_inputs(TOKENIZERS["tiny"], 50, seed=9)
    ids = ti.ids.copy()
    ids[7] = ids[3]
    x = action_tokens(ids, ti.tables, ti.W_a1, ti.W_a2)
    assert np.array_equal(x[7], x[3])
    perm = np.random.default_rng(0).permutation(50)
    xp = action_tokens(ids[perm], ti.tables, ti.W_a1, ti.W_a2)
    assert np.array_equal(xp, x[perm])


def test_linear_in_output_projection():
    ti = make_token_inputs(TOKENIZERS["tiny"], 30, seed=4)
    A = ti.W_a2
    Bm = np.random.default_rng(1).standard_normal(A.shape).astype(np.float32)
    xa = action_tokens(ti.ids, ti.tables, ti.W_a1, A)
    xb = action_tokens(ti.ids, ti.tables, ti.W_a1, Bm)
    xab = action_tokens(ti.ids, ti.tables, ti.W_a1, A.astype(np.float64) + Bm)
    np.testing.assert_allclose(xab, xa + xb, rtol=1e-12, atol=1e-12)


def test_id_outside_table_is_rejected():
    ti = make_token_inputs(TOKENIZERS["tiny"], 10, seed=1)
    bad = ti.ids.copy()
    bad[4, 2] = ti.dims.rows[2]
    with pytest.raises(ValueError):
        action_tokens(bad, ti.tables, ti.W_a1, ti.W_a2)
    bad[4, 2] = -1
    with pytest.raises(ValueError):
        action_tokens(bad, ti.tables, ti.W_a1, ti.W_a2)


def test_generator_ids_stay_in_tables_and_item_ids_are_skewed():
    ti = make_token_inputs(TOKENIZERS["online"], 20000, seed=1)
    for f, rows in enumerate(ti.dims.rows):
        assert ti.ids[:, f].min() >= 0 and ti.ids[:, f].max() < rows
    counts = np.bincount(ti.ids[:, 1], minlength=ti.dims.rows[1])
    # Zipf popularity: the most popular item takes a sizeable share
    assert counts.max() > 0.05 * 20000
