"""GPU parity: the CUDA path, called through the C ABI, against the fp64 oracle
on the same seeded inputs.  Floating point within the target tolerances
(bf16: max-abs 3e-2 and relative L2 1e-2; fp32: 1e-4); the pyramid offsets
bit-exact."""
import numpy as np
import pytest
import torch

import oracle
from oracle.plan import plan_layers
from workloads import Dims, Workload, make_inputs, workload

from gpu_harness import assert_close, make_handle, run, sample_users, to_device

pytestmark = pytest.mark.gpu

FULL = ["online", "upstream", "sweep200", "sweep400", "sweep800", "sweep1600", "skewed"]
# users the oracle recomputes one by one at full size (the GPU runs the whole batch)
# (the first ones, plus the longest and the shortest user of the batch)
SAMPLE = {"online": 8, "upstream": 8, "sweep200": 8, "sweep400": 8, "sweep800": 8,
          "sweep1600": 8, "skewed": 8}


def check_plan(h, inp):
    got = h.plan_export().cpu().numpy()
    plans = plan_layers(inp.lengths, inp.dims.keep, inp.dims.n_q)
    for l, p in enumerate(plans):
        np.testing.assert_array_equal(got[l, 0], p.hist_off, err_msg=f"hist offsets layer {l}")
        np.testing.assert_array_equal(got[l, 1], p.query_off, err_msg=f"query offsets layer {l}")


def test_tiny_fp32_all_users():
    inp = make_inputs(workload("tiny"))
    h, out = run(inp)
    assert h.status() == 0
    check_plan(h, inp)
    ref = oracle.forward(inp)
    assert_close(out, ref, "fp32", "tiny")


@pytest.mark.parametrize("name", FULL)
def test_full_size_sampled_users(name):
    inp = make_inputs(workload(name))
    h, out = run(inp)
    assert h.status() == 0
    check_plan(h, inp)
    users = sample_users(inp.lengths, SAMPLE[name])
    ref = oracle.forward(inp, users=users)
    assert_close(out[users], ref, inp.dims.dtype, name)
    # every row of the batch is finite, and for the query-token outputs has
    # unit RMS (post-norm rows with unit gain)
    assert np.all(np.isfinite(out))
    if not inp.dims.d_out:
        rms = np.sqrt((out ** 2).mean(-1))
        assert np.abs(rms - 1).max() < 2e-2


def _edge_wl(dtype, **kw):
    base = dict(d=128, heads=2, d_head=64, rank=64, d_ctx=16, n_q=5, keep=(300, 130, 0),
                dtype=dtype)
    base.update(kw)
    return Workload(name="edge", dims=Dims(**base), batch=1, lengths=("fixed", 1), seed=21)


EDGE_LENGTHS = [[0, 1, 2, 127, 128, 129, 300, 0, 255, 3], [1], [0], [333, 0, 64]]


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
@pytest.mark.parametrize("lengths", EDGE_LENGTHS)
@pytest.mark.parametrize("variant", ["cross_last", "no_queries_readout", "full_keep", "kv_plain"])
def test_edge_cases_all_users(dtype, lengths, variant):
    kw = {"cross_last": {}, "no_queries_readout": dict(n_q=0, d_ctx=0, d_out=96, keep=(256, 64)),
          "full_keep": dict(keep=(400, 400)), "kv_plain": dict(kv_norm=0, keep=(200, 7))}[variant]
    wl = _edge_wl(dtype, **kw)
    inp = make_inputs(wl, lengths=lengths, random_gains=True)
    h, out = run(inp, max_len=max(max(lengths), 1))
    assert h.status() == 0
    check_plan(h, inp)
    ref = oracle.forward(inp)
    assert_close(out, ref, dtype, f"{variant} {lengths}")


def test_repeatable_and_stream_independent():
    inp = make_inputs(workload("online"), batch=32)
    h, a = run(inp)
    _, b = run(inp, handle=h)
    assert np.array_equal(a, b)
    s = torch.cuda.Stream()
    values, offsets, ctx, cand = to_device(inp)
    with torch.cuda.stream(s):
        c = h.forward(values, offsets, ctx, cand, stream=s)
    s.synchronize()
    assert np.array_equal(a, c.cpu().numpy().astype(np.float64))


def test_batch_smaller_than_capacity_and_empty_batch():
    inp = make_inputs(workload("online"), batch=64)
    h = make_handle(inp, max_batch=256, max_len=400)
    _, out = run(inp, handle=h)
    users = [0, 5, 63]
    assert_close(out[users], oracle.forward(inp, users=users), "bf16", "B < max_batch")
    values, offsets, ctx, cand = to_device(inp)
    empty = h.forward(values, offsets[:1], ctx[:0], cand[:0])
    assert empty.shape[0] == 0
    assert h.status() == 0


def test_device_status_reports_bad_offsets_without_fault():
    inp = make_inputs(workload("online"), batch=8)
    h, good = run(inp)
    values, offsets, ctx, cand = to_device(inp)
    bad = offsets.clone()
    bad[3] = bad[5] + 1                       # offsets no longer non-decreasing
    h.forward(values, bad, ctx, cand)
    assert h.status() & 1
    long_ = offsets.clone()
    long_[1:] += 1000                         # user 0 longer than max_len
    h.forward(values, long_, ctx, cand)
    assert h.status() & 2
    # the handle stays usable and the next valid call is exact
    _, again = run(inp, handle=h)
    assert h.status() == 0
    assert np.array_equal(good, again)


def test_cuda_graph_replay_matches_eager():
    """A whole forward captured once in a CUDA graph and replayed gives the
    same bits as launching it eagerly (no host work inside the forward)."""
    inp = make_inputs(workload("online"), batch=48)
    h, eager = run(inp)
    values, offsets, ctx, cand = to_device(inp)
    out = torch.empty(h.out_shape(inp.batch), dtype=torch.float32, device="cuda")
    h.forward(values, offsets, ctx, cand, out=out)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        h.forward(values, offsets, ctx, cand, out=out)
    out.zero_()
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert h.status() == 0
    assert np.array_equal(out.cpu().numpy().astype(np.float64), eager)
