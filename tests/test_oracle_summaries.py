"""Pins for the oracle's sequence summaries (LLaTTE notes, huaxiaozhuan.com,
appendix A.2 item 4: Z_seq^(k) = LoRAMLP_k(Flatten(Z_raw))).

The oracle reads LoRAMLP_k(v) as W_up,k SiLU(W_down,k v) over the row-major
flattened final query tokens.  What pins it here, each against something
other than its own code:
* SiLU against the library tanh: silu(x) - silu(-x) = x and
  silu(x) + silu(-x) = x tanh(x/2), which fix silu(x) = (x + x tanh(x/2)) / 2.
* Flatten order and layer order with one-hot weights: W_down row t picking
  flat element (i, c) and W_up = I give summary entry t = silu(Z_raw[i, c]).
* The bottleneck: summaries of many inputs span exactly sum_rank dimensions
  (a nonlinearity after W_up, or a missing bottleneck, gives full rank).
* Summaries are independent of one another's weights and keep their order.
* The same MLP built from torch.nn modules in float64.
* The forward's summaries are those of its own final query-token rows.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from workloads import make_inputs, workload


def test_silu_closed_form_against_tanh():
    x = np.linspace(-30.0, 30.0, 2001)
    s, sm = oracle.silu(x), oracle.silu(-x)
    np.testing.assert_allclose(s - sm, x, rtol=0, atol=1e-12)
    np.testing.assert_allclose(s + sm, x * np.tanh(x / 2), rtol=0, atol=1e-12)
    assert oracle.silu(np.array([0.0]))[0] == 0.0


def test_one_hot_weights_select_flattened_elements():
    rng = np.random.default_rng(11)
    n_q, d, r = 3, 5, 7
    z = rng.standard_normal((n_q, d))
    picks = [(0, 0), (0, 4), (1, 0), (1, 3), (2, 1), (2, 4), (1, 2)]
    W_down = np.zeros((r, n_q * d))
    for t, (i, c) in enumerate(picks):
        W_down[t, i * d + c] = 1.0            # row-major: token i, coordinate c
    out = oracle.summaries(z, [{"W_down": W_down, "W_up": np.eye(r)}])
    assert out.shape == (1, r)
    sel = np.array([z[i, c] for i, c in picks])
    np.testing.assert_allclose(out[0], (sel + sel * np.tanh(sel / 2)) / 2, rtol=1e-13, atol=1e-15)


def test_zero_down_projection_gives_zero():
    rng = np.random.default_rng(2)
    z = rng.standard_normal((4, 6))
    out = oracle.summaries(z, [{"W_down": np.zeros((3, 24)), "W_up": rng.standard_normal((9, 3))}])
    assert np.all(out == 0.0)


def test_bottleneck_rank():
    rng = np.random.default_rng(5)
    n_q, d, r, d_seq = 4, 8, 3, 10
    w = {"W_down": rng.standard_normal((r, n_q * d)), "W_up": rng.standard_normal((d_seq, r))}
    outs = np.stack([oracle.summaries(rng.standard_normal((n_q, d)), [w])[0] for _ in range(40)])
    sv = np.linalg.svd(outs, compute_uv=False)
    assert sv[r - 1] > 1e-6 * sv[0]            # the r directions are all used
    assert np.all(sv[r:] < 1e-10 * sv[0])      # and nothing beyond them


def test_summaries_are_independent_and_ordered():
    rng = np.random.default_rng(8)
    n_q, d = 2, 4
    z = rng.standard_normal((n_q, d))
    ws = [{"W_down": rng.standard_normal((3, n_q * d)), "W_up": rng.standard_normal((5, 3))}
          for _ in range(3)]
    base = oracle.summaries(z, ws)
    assert base.shape == (3, 5)
    for k in range(3):
        np.testing.assert_array_equal(oracle.summaries(z, [ws[k]])[0], base[k])
    ws2 = [ws[0], {"W_down": rng.standard_normal((3, n_q * d)), "W_up": ws[1]["W_up"]}, ws[2]]
    other = oracle.summaries(z, ws2)
    np.testing.assert_array_equal(other[[0, 2]], base[[0, 2]])
    assert not np.allclose(other[1], base[1])


def test_matches_torch_modules():
    rng = np.random.default_rng(13)
    n_q, d, r, d_seq = 5, 6, 4, 7
    W_down, W_up = rng.standard_normal((r, n_q * d)), rng.standard_normal((d_seq, r))
    mlp = torch.nn.Sequential(torch.nn.Flatten(0), torch.nn.Linear(n_q * d, r, bias=False),
                              torch.nn.SiLU(), torch.nn.Linear(r, d_seq, bias=False)).double()
    with torch.no_grad():
        mlp[1].weight.copy_(torch.from_numpy(W_down))
        mlp[3].weight.copy_(torch.from_numpy(W_up))
    for _ in range(5):
        z = rng.standard_normal((n_q, d)) * 3
        with torch.no_grad():
            ref = mlp(torch.from_numpy(z)).numpy()
        got = oracle.summaries(z, [{"W_down": W_down, "W_up": W_up}])[0]
        np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("name", ["tiny_sum"])
def test_forward_summarises_its_final_query_rows(name):
    wl = workload(name)
    inp = make_inputs(wl)
    out = oracle.forward(inp)
    d = inp.dims
    assert out.shape == (inp.batch, d.n_sum, d.d_seq)
    plain = dataclasses.replace(inp, dims=dataclasses.replace(d, n_sum=0, sum_rank=0, d_seq=0),
                                summaries=None)
    rows = oracle.forward(plain)                       # [B, n_q, d]
    assert rows.shape == (inp.batch, d.n_q, d.d)
    for u in range(inp.batch):
        np.testing.assert_array_equal(out[u], oracle.summaries(rows[u], inp.summaries))
