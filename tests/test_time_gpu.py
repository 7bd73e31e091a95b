"""GPU parity of the additive timestamp encoding (LLaTTE notes, appendix A.2
item 1; the sinusoidal code of the event age on the first d_time dims of the
history tokens, added in the jagged gather) against the fp64 oracle, through
the C ABI."""
import numpy as np
import pytest
import torch

from latent_attention_jagged_b200.binding import LlatteError
import oracle
from oracle.analysis import attention_stats
from workloads import Dims, Workload, make_inputs, workload

from gpu_harness import (EXPORT_TOL, ages_on_device, assert_close, make_handle, run, sample_users,
                         to_device)

pytestmark = pytest.mark.gpu


def test_tiny_fp32_all_users():
    inp = make_inputs(workload("tiny_time"))
    h, out = run(inp)
    assert h.status() == 0
    assert_close(out, oracle.forward(inp), "fp32", "tiny_time")


def test_online_sampled_users():
    inp = make_inputs(workload("online_time"))
    h, out = run(inp)
    assert h.status() == 0
    users = sample_users(inp.lengths, 6)
    assert_close(out[users], oracle.forward(inp, users=users), "bf16", "online_time")


def test_old_events_fp32():
    """Ages up to thousands of hours: the code's argument reduction."""
    inp = make_inputs(_wl("fp32", d_time=64), lengths=LENGTHS, random_gains=True)
    inp.event_age = (inp.event_age * 40.0).astype(np.float32)
    assert inp.event_age.max() > 3000
    h, out = run(inp, max_len=max(LENGTHS))
    assert h.status() == 0
    assert_close(out, oracle.forward(inp), "fp32", "old events")


def _wl(dtype, **kw):
    base = dict(d=128, heads=2, d_head=64, rank=64, d_ctx=16, n_q=5, keep=(300, 130, 0),
                dtype=dtype, d_time=32)
    base.update(kw)
    return Workload(name="time_edge", dims=Dims(**base), batch=1, lengths=("fixed", 1), seed=31)


LENGTHS = [0, 1, 2, 127, 128, 129, 300, 0, 255, 3]


@pytest.mark.parametrize("dtype,kw", [
    ("bf16", {}), ("bf16", dict(d_time=2)), ("bf16", dict(d_time=128, keep=(300, 64))),
    ("bf16", dict(n_q=0, d_ctx=0, d_out=64, keep=(256, 64))),
    ("fp32", dict(d_time=10)), ("fp32", dict(d_time=128))])
def test_edge_shapes_all_users(dtype, kw):
    inp = make_inputs(_wl(dtype, **kw), lengths=LENGTHS, random_gains=True)
    h, out = run(inp, max_len=max(LENGTHS))
    assert h.status() == 0
    assert_close(out, oracle.forward(inp), dtype, f"timestamp code {kw}")


def test_forward_without_ages_is_rejected_and_export_uses_them():
    inp = make_inputs(workload("online_time"), batch=6)
    h = make_handle(inp)
    values, offsets, ctx, cand = to_device(inp)
    with pytest.raises(ValueError):
        h.forward(values, offsets, ctx, cand)
    ag = ages_on_device(inp)
    out, rec, top, hrs = h.forward_export(values, offsets, ctx, cand, layer=1, n_k=9,
                                          event_age=ag, n_hours=72)
    torch.cuda.synchronize()
    assert h.status() == 0
    assert_close(out.cpu().numpy().astype(np.float64), oracle.forward(inp), "bf16", "out")
    R, K, H = attention_stats(inp, 1, 9, inp.event_age, 72)
    tol = EXPORT_TOL["bf16"]
    assert_close(rec.cpu().numpy().astype(np.float64), R, "bf16", "recent", tol)
    assert_close(top.cpu().numpy().astype(np.float64), K, "bf16", "topk", tol)
    assert_close(hrs.cpu().numpy().astype(np.float64), H, "bf16", "hours", tol)
