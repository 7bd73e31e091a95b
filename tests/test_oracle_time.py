"""Pins for the oracle's additive timestamp encoding (LLaTTE notes, appendix
A.2 item 1: timestamp codes added on a subset of the hidden dims of the
action tokens), read as the sinusoidal code of the event's age in hours on the
first d_time dims.

What pins it, each against something other than the oracle's own formula:
* the code of age 0 is (0, 1, 0, 1, ...) and of age pi/2 starts (1, 0): sine
  first, cosine second, the first pair at 1 rad per hour;
* every (sin, cos) pair has unit norm, and the inner product of two codes
  depends only on the age difference (sum of cos of the difference times each
  frequency): the pairing is sine/cosine of the same argument;
* the frequencies fall geometrically from 1 to 10000^(-(d_time-2)/d_time),
  read off the zero crossings of each pair;
* the forward with the encoding equals the forward without it on inputs whose
  first d_time history dims were shifted by the code (query tokens untouched);
* in cross mode the output is invariant to permuting history tokens together
  with their ages, but not to permuting the ages alone (the encoding breaks
  the permutation invariance of the plain layer);
* Form A (non-absorbed, whole fused sequence) equals Form B with the encoding.
"""
import dataclasses

import numpy as np
import pytest

import oracle
from workloads import Dims, Workload, make_inputs, workload


def test_code_at_zero_and_quarter_period():
    te = oracle.time_encoding(np.array([0.0, np.pi / 2]), 8)
    np.testing.assert_allclose(te[0], [0, 1, 0, 1, 0, 1, 0, 1], atol=1e-15)
    np.testing.assert_allclose(te[1, :2], [1.0, 0.0], atol=1e-15)


def test_pairs_unit_norm_and_shift_invariant_inner_product():
    rng = np.random.default_rng(2)
    d = 12
    a = rng.uniform(0, 500, size=20)
    te = oracle.time_encoding(a, d)
    np.testing.assert_allclose(te[:, 0::2] ** 2 + te[:, 1::2] ** 2, 1.0, atol=1e-12)
    G = te @ te.T
    shift = 37.25
    G2 = oracle.time_encoding(a + shift, d) @ oracle.time_encoding(a + shift, d).T
    np.testing.assert_allclose(G, G2, atol=1e-9)


def test_frequencies_from_zero_crossings():
    d = 8
    t = np.linspace(0, 20000, 2_000_001)
    te = oracle.time_encoding(t, d)
    for i in range(d // 2):
        s = te[:, 2 * i]
        crossings = np.count_nonzero(np.signbit(s[1:]) != np.signbit(s[:-1]))
        w_est = np.pi * crossings / t[-1]
        w = 10000.0 ** (-2.0 * i / d)
        assert abs(w_est - w) <= np.pi / t[-1] * 1.01, (i, w_est, w)


def _dims(**kw):
    base = dict(d=16, heads=2, d_head=8, rank=12, d_ctx=3, n_q=3, keep=(9, 4), dtype="fp32",
                d_time=6)
    base.update(kw)
    return Dims(**base)


def _inp(dims, lengths, seed=5):
    wl = Workload(name="t", dims=dims, batch=len(lengths), lengths=("fixed", 1), seed=seed)
    return make_inputs(wl, lengths=lengths, random_gains=True)


def test_encoding_is_additive_on_history_dims_only():
    inp = _inp(_dims(), [7, 0, 12, 3])
    a = oracle.forward(inp)
    shifted = inp.values.astype(np.float64).copy()
    shifted[:, :6] += oracle.time_encoding(inp.event_age, 6)
    plain = dataclasses.replace(inp, dims=dataclasses.replace(inp.dims, d_time=0),
                                values=shifted, event_age=None)
    np.testing.assert_allclose(oracle.forward(plain), a, atol=1e-12)


def test_cross_mode_permutation_needs_the_ages_to_move_too():
    inp = _inp(_dims(keep=(0,)), [9])
    a = oracle.forward(inp)
    perm = np.random.default_rng(1).permutation(9)
    both = dataclasses.replace(inp, values=inp.values[perm], event_age=inp.event_age[perm])
    np.testing.assert_allclose(oracle.forward(both), a, atol=1e-12)
    tokens_only = dataclasses.replace(inp, values=inp.values[perm])
    assert np.abs(oracle.forward(tokens_only) - a).max() > 1e-3


@pytest.mark.parametrize("lengths", [[0, 1, 5, 13], [20, 3]])
def test_form_a_equals_form_b_with_encoding(lengths):
    inp = _inp(_dims(keep=(9, 4, 0)), lengths)
    np.testing.assert_allclose(oracle.forward(inp), oracle.forward_brute(inp), atol=1e-11)


def test_tiny_time_workload_forms_agree():
    inp = make_inputs(workload("tiny_time"))
    assert inp.event_age.shape == (int(inp.offsets[-1]),)
    assert np.all(np.diff(inp.event_age[inp.offsets[0]:inp.offsets[1]]) < 0)   # earliest oldest
    np.testing.assert_allclose(oracle.forward(inp), oracle.forward_brute(inp), atol=1e-12)
