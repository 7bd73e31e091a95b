"""Pins for the oracle's attention statistics (LLaTTE notes, appendix A.4):
the cumulative attention on the k most recent keys, on the k largest
probabilities, and by hours before the request, per query token and head.

What pins them, each against something other than the oracle's own code:
* probability rows sum to one, so both cumulative curves reach 1 once k
  covers every key, and give zeros for a user with no key;
* the top-k mass is the largest sum over all k-subsets (brute force over
  itertools.combinations on short rows), so it bounds the recent-k mass;
  top-1 is the row maximum;
* identical history tokens give uniform rows: both curves are min(k, T) / T;
* hour bins: with event t of a user aged (T - 1 - t) + 0.5 hours, bin b holds
  the probability of the key b places from the most recent one (also after
  pyramid trimming, which keeps the most recent events), the last bin the rest.
"""
import itertools

import numpy as np
import pytest

import oracle
from oracle.analysis import attention_stats, row_stats
from workloads import Dims, Workload, make_inputs


def _inp(lengths, seed=5, **kw):
    base = dict(d=16, heads=2, d_head=8, rank=12, d_ctx=3, n_q=3, keep=(9, 4), dtype="fp32")
    base.update(kw)
    wl = Workload(name="t", dims=Dims(**base), batch=len(lengths), lengths=("fixed", 1), seed=seed)
    return make_inputs(wl, lengths=lengths, random_gains=True)


def test_curves_reach_one_and_empty_users_give_zero():
    inp = _inp([0, 1, 5, 9, 13])
    R, K, _ = attention_stats(inp, layer=0, n_k=5)
    T = np.asarray(inp.lengths)
    for u in range(inp.batch):
        for i in range(5):
            k = 1 << i
            want = 1.0 if (T[u] > 0 and k >= T[u]) else None
            if T[u] == 0:
                assert np.all(R[u, :, :, i] == 0) and np.all(K[u, :, :, i] == 0)
            elif want is not None:
                np.testing.assert_allclose(R[u, :, :, i], 1.0, atol=1e-12)
                np.testing.assert_allclose(K[u, :, :, i], 1.0, atol=1e-12)


def test_topk_is_the_best_k_subset_and_bounds_recent():
    rng = np.random.default_rng(3)
    for T in (1, 2, 5, 7, 9):
        p = rng.random(T)
        p /= p.sum()
        rec, top, _ = row_stats(p, n_k=4)
        for i in range(4):
            k = min(1 << i, T)
            best = max(sum(c) for c in itertools.combinations(p, k))
            np.testing.assert_allclose(top[i], best, rtol=0, atol=1e-14)
            assert top[i] >= rec[i] - 1e-15
        assert top[0] == p.max()
        np.testing.assert_allclose(rec, [p[-(1 << i):].sum() for i in range(4)], atol=1e-15)


def test_model_rows_topk_bounds_recent_and_top1_is_max():
    inp = _inp([13, 6, 2], seed=9)
    R, K, _ = attention_stats(inp, layer=0, n_k=4)
    assert np.all(K >= R - 1e-12)
    assert np.all(np.diff(K, axis=-1) >= -1e-12)
    _, probs = oracle.forward(inp, return_probs=True)
    for u in range(inp.batch):
        for j in range(inp.dims.heads):
            P = probs[u][0][j]
            n = P.shape[0] - inp.dims.n_q
            np.testing.assert_allclose(K[u, :, j, 0], P[n:].max(axis=1), atol=1e-15)


def test_identical_keys_give_uniform_curves():
    inp = _inp([7, 4], seed=4, d_ctx=0)
    for u in range(inp.batch):
        a, b = inp.offsets[u], inp.offsets[u + 1]
        inp.values[a:b] = inp.values[a]                  # every history token the same
    R, K, _ = attention_stats(inp, layer=0, n_k=4)
    for u, T in enumerate(inp.lengths):
        want = np.minimum([1, 2, 4, 8], T) / T
        np.testing.assert_allclose(R[u], np.broadcast_to(want, R[u].shape), atol=1e-12)
        np.testing.assert_allclose(K[u], np.broadcast_to(want, K[u].shape), atol=1e-12)


@pytest.mark.parametrize("layer", [0, 1])
def test_hour_bins_follow_recency(layer):
    lengths = [13, 6, 0, 9]
    inp = _inp(lengths, seed=6)
    ages = np.concatenate([(L - 1 - np.arange(L)) + 0.5 for L in lengths]).astype(np.float32)
    n_hours = 5
    _, _, H = attention_stats(inp, layer=layer, n_k=1, ages=ages, n_hours=n_hours)
    _, probs = oracle.forward(inp, return_probs=True)
    for u in range(inp.batch):
        for j in range(inp.dims.heads):
            P = probs[u][layer][j]
            T = P.shape[1]
            n = P.shape[0] - inp.dims.n_q
            for i in range(inp.dims.n_q):
                row = P[n + i]
                want = np.zeros(n_hours)
                for b in range(min(T, n_hours - 1)):
                    want[b] = row[T - 1 - b]                  # b places from the most recent
                want[n_hours - 1] = row[:max(0, T - (n_hours - 1))].sum()
                np.testing.assert_allclose(H[u, i, j], want, atol=1e-15)
