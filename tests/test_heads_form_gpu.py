"""GPU parity of MLA in its per-head form (LLaTTE notes, appendix A.3 first
display: K, V = split(RMSNorm(X W_down^KV) W_up^KV), scores over d_k = d_h =
64, then W_out) against the fp64 oracle, through the C ABI.  The per-head and
the absorbed forms compute the same function, so both are held to the same
oracle; the tests force each form on the same inputs."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from oracle.analysis import attention_stats
from workloads import Dims, Workload, make_event_ages, make_inputs, workload

from gpu_harness import EXPORT_TOL, assert_close, make_handle, run, sample_users, to_device

pytestmark = pytest.mark.gpu

PER_HEAD, ABSORBED = 2, 1


def _force(inp, form):
    return dataclasses.replace(inp, dims=dataclasses.replace(inp.dims, attn_form=form))


@pytest.mark.parametrize("name,n", [("online", 8), ("upstream", 8), ("skewed", 8),
                                    ("sweep1600", 8), ("sweep200", 8)])
def test_full_size_per_head_sampled_users(name, n):
    inp = _force(make_inputs(workload(name)), PER_HEAD)
    h, out = run(inp)
    assert h.status() == 0
    users = sample_users(inp.lengths, n)
    assert_close(out[users], oracle.forward(inp, users=users), "bf16", f"{name} per-head")
    assert np.all(np.isfinite(out))


def test_forms_agree_on_the_same_batch():
    inp = make_inputs(workload("online"), batch=24)
    _, a = run(_force(inp, ABSORBED))
    _, b = run(_force(inp, PER_HEAD))
    ref = oracle.forward(inp)
    assert_close(a, ref, "bf16", "absorbed")
    assert_close(b, ref, "bf16", "per-head")


def _wl(**kw):
    base = dict(d=128, heads=2, d_head=64, rank=64, d_ctx=16, n_q=5, keep=(300, 130, 0),
                attn_form=PER_HEAD)
    base.update(kw)
    return Workload(name="heads_edge", dims=Dims(**base), batch=1, lengths=("fixed", 1), seed=37)


LENGTHS = [0, 1, 2, 127, 128, 129, 300, 0, 255, 3]


@pytest.mark.parametrize("kw", [{}, dict(rank=256, heads=4), dict(n_q=0, d_ctx=0, d_out=64, keep=(256, 64)),
                                dict(d=512, heads=8, rank=128, keep=(200, 40)),
                                dict(kv_norm=0, keep=(200, 7)), dict(n_q=130, keep=(256, 0))])
def test_edge_shapes_all_users(kw):
    inp = make_inputs(_wl(**kw), lengths=LENGTHS, random_gains=True)
    h, out = run(inp, max_len=max(LENGTHS))
    assert h.status() == 0
    assert_close(out, oracle.forward(inp), "bf16", f"per-head {kw}")


def test_export_in_a_per_head_layer():
    inp = _force(make_inputs(workload("online"), batch=6), PER_HEAD)
    ages = make_event_ages(inp.lengths, seed=5)
    h = make_handle(inp)
    values, offsets, ctx, cand = to_device(inp)
    out, rec, top, hrs = h.forward_export(values, offsets, ctx, cand, layer=1, n_k=9,
                                          event_age=torch.from_numpy(ages).cuda(), n_hours=48)
    torch.cuda.synchronize()
    assert h.status() == 0
    R, K, H = attention_stats(inp, 1, 9, ages, 48)
    tol = EXPORT_TOL["bf16"]
    assert_close(rec.cpu().numpy().astype(np.float64), R, "bf16", "recent", tol)
    assert_close(top.cpu().numpy().astype(np.float64), K, "bf16", "topk", tol)
    assert_close(hrs.cpu().numpy().astype(np.float64), H, "bf16", "hours", tol)


@pytest.mark.parametrize("form", [ABSORBED, PER_HEAD])
def test_profiled_steps_count_each_layer_once_and_handles_close(form):
    """Per-step timing records each step once per layer in both forms, and a
    profiled handle closes cleanly (its events are released exactly once)."""
    inp = _force(make_inputs(workload("online"), batch=16), form)
    L = inp.dims.n_layers
    for _ in range(2):
        h = make_handle(inp)
        values, offsets, ctx, cand = to_device(inp)
        h.set_profiling(True)
        for _ in range(3):
            h.forward(values, offsets, ctx, cand)
        prof = h.profile()
        assert h.status() == 0
        for step in ("kv", "q", "attn", "o"):
            assert prof[step]["calls"] == 3 * L, (step, prof[step])
        h.profile_reset()
        h.forward(values, offsets, ctx, cand)
        h.close()
