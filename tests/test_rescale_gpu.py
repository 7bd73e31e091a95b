"""GPU parity when the softmax's running maximum grows a lot inside an item.

Both attention kernels compute probabilities against a running maximum and
rescale O and the row sum only when a later key tile's scores exceed it by
more than 2^8 (log2 units); the per-head kernel also computes the
probabilities of every tile after an item's first against the old maximum
before it knows the tile's own.  With random inputs the scores of all tiles
are alike and that branch is rarely taken, so this test builds a batch where
it must be: the KV latent is not normalised and the last events of every
history are scaled up, so their keys (and the queries of those rows) grow and
their scores exceed the earlier tiles' by far.  The test first checks, with
the oracle's own layer-0 scores, that some row's maximum does grow by more
than 2^8 from one 128-key tile to a later one, then compares both MLA forms
with the fp64 oracle (LLaTTE notes, appendix A.3; softmax over the visible
keys of appendix A.2)."""
import dataclasses

import numpy as np
import pytest

import oracle
from oracle.model import _f64, absorb, history_tokens
from workloads import Dims, Workload, make_inputs

from gpu_harness import assert_close, run

pytestmark = pytest.mark.gpu

PER_HEAD, ABSORBED = 2, 1
SCALE, LAST = 2.0, 100          # the last LAST events of every history, times SCALE (bf16-exact)
GROW = 8.0 / np.log2(np.e)       # 2^8 growth in natural-log units


def _jump_batch(form):
    dims = Dims(d=128, heads=2, d_head=64, rank=128, d_ctx=16, n_q=5, keep=(400, 100), kv_norm=0,
                attn_form=form)
    inp = make_inputs(Workload(name="jumps", dims=dims, batch=6, lengths=("uniform", 290, 400),
                               seed=11))
    values = inp.values.copy()
    for u in range(inp.batch):
        a, b = int(inp.offsets[u]), int(inp.offsets[u + 1])
        values[max(a, b - LAST):b] *= SCALE
    return dataclasses.replace(inp, values=values)


def _largest_growth(inp):
    """Largest step of a row's running score maximum from one 128-key tile to
    the next, over the layer-0 rows and heads of the batch (oracle scores)."""
    dims = inp.dims
    w = inp.layers[0]
    ab = absorb(w, dims)
    best = 0.0
    for u in range(inp.batch):
        H = history_tokens(inp, u)
        T = H.shape[0]
        n = min(T, dims.keep[0])
        C = H @ _f64(w["W_dkv"]).T
        R = np.concatenate([H[T - n:], _f64(inp.cand[u])], axis=0)
        RC = np.concatenate([R, np.broadcast_to(_f64(inp.ctx[u]), (R.shape[0], dims.d_ctx))], axis=1)
        for j in range(dims.heads):
            S = (RC @ ab["W_QK"][j].T) @ C.T
            for i in range(R.shape[0]):
                vis = T - n + i + 1 if i < n else T
                m_prev = -np.inf
                for k0 in range(0, vis, 128):
                    mt = S[i, k0:min(vis, k0 + 128)].max()
                    if np.isfinite(m_prev):
                        best = max(best, mt - m_prev)
                    m_prev = max(m_prev, mt)
    return best


@pytest.mark.parametrize("form", [PER_HEAD, ABSORBED])
def test_growing_scores_take_the_rescale_path(form):
    inp = _jump_batch(form)
    assert _largest_growth(inp) > GROW          # the batch does reach the rescale branch
    h, out = run(inp)
    assert h.status() == 0
    assert np.all(np.isfinite(out))
    assert_close(out, oracle.forward(inp), "bf16", f"rescale {'per-head' if form == PER_HEAD else 'absorbed'}")
