"""The allocation-free plan entry point (llatte_plan_static).

Callers that cannot allocate device memory where they need the plan (inside
another framework's memory pool or allocator hook, or with all device memory
reserved up front) use this call instead of a handle.  It must return exactly
what the handle's own plan export returns for the same batch, on consecutive
calls, and must not allocate.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

from latent_attention_jagged_b200 import binding
from workloads import make_inputs, workload

from gpu_harness import make_handle, run

pytestmark = pytest.mark.gpu


def _reference_plan(inp):
    h, _ = run(inp)
    ref = h.plan_export().cpu()
    assert h.status() == 0
    return h, ref


def test_plan_static_matches_handle_on_two_calls_in_a_row():
    a = make_inputs(workload("skewed"), batch=300)
    b = make_inputs(workload("online"), batch=77)
    ha, ref_a = _reference_plan(a)
    hb, ref_b = _reference_plan(b)
    oa = torch.from_numpy(a.offsets).cuda()
    ob = torch.from_numpy(b.offsets).cuda()
    # two calls in a row on different batches, then the first batch again:
    # every result must equal the handle's plan for that batch (integers, so
    # exactly equal)
    got_a, st_a = binding.plan_static(a.dims, oa, max_batch=300, max_len=1600)
    got_b, st_b = binding.plan_static(b.dims, ob, max_batch=77, max_len=400)
    torch.cuda.synchronize()
    assert int(st_a.item()) == 0 and int(st_b.item()) == 0
    assert torch.equal(got_a.cpu(), ref_a)
    assert torch.equal(got_b.cpu(), ref_b)
    again = torch.empty_like(got_a)
    st = torch.empty_like(st_a)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    binding.plan_static(a.dims, oa, max_batch=300, max_len=1600, out=again, status=st)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0      # nothing allocated by the call
    assert int(st.item()) == 0
    assert torch.equal(again.cpu(), ref_a)
    ha.close()
    hb.close()


def test_plan_static_rejects_oversized_batch_and_reports_bad_offsets():
    inp = make_inputs(workload("online"), batch=8)
    big = torch.zeros(binding.PLAN_STATIC_MAX_BATCH + 2, dtype=torch.int64, device="cuda")
    with pytest.raises(binding.LlatteError) as e:
        binding.plan_static(inp.dims, big, max_batch=binding.PLAN_STATIC_MAX_BATCH + 1,
                            max_len=400)
    assert e.value.code == binding.LLATTE_ERR_UNSUPPORTED
    bad = torch.from_numpy(inp.offsets).cuda()
    bad[3] = bad[5] + 1
    out, st = binding.plan_static(inp.dims, bad, max_batch=8, max_len=400)
    torch.cuda.synchronize()
    assert int(st.item()) & binding.DEV_BAD_OFFSETS
    assert int(out.abs().sum().item()) == 0
    # a valid batch right after a rejected one is exact again
    good = torch.from_numpy(inp.offsets).cuda()
    h, ref = _reference_plan(inp)
    out2, st2 = binding.plan_static(inp.dims, good, max_batch=8, max_len=400)
    torch.cuda.synchronize()
    assert int(st2.item()) == 0 and torch.equal(out2.cpu(), ref)
    h.close()


def test_plan_static_reports_long_users_and_row_totals():
    """The other rejections of the same plan kernel, through the dims this
    entry point builds: a user longer than max_len, and more rows than
    max_total.  A rejected batch leaves zeros; the next valid batch is exact."""
    inp = make_inputs(workload("online"), batch=8)
    offs = torch.from_numpy(inp.offsets).cuda()
    h, ref = _reference_plan(inp)
    longest = int(inp.lengths.max())
    out, st = binding.plan_static(inp.dims, offs, max_batch=8, max_len=longest - 1)
    torch.cuda.synchronize()
    assert int(st.item()) & binding.DEV_TOO_LONG
    assert int(out.abs().sum().item()) == 0
    total = int(inp.offsets[-1])
    out, st = binding.plan_static(inp.dims, offs, max_batch=8, max_len=longest,
                                  max_total=total - 1)
    torch.cuda.synchronize()
    assert int(st.item()) & binding.DEV_TOO_MANY_ROWS
    assert int(out.abs().sum().item()) == 0
    out, st = binding.plan_static(inp.dims, offs, max_batch=8, max_len=longest, max_total=total)
    torch.cuda.synchronize()
    assert int(st.item()) == 0 and torch.equal(out.cpu(), ref)
    h.close()


def test_plan_static_empty_batch_writes_zeros():
    """B = 0: every layer's offsets are the single entry 0, written over
    whatever the caller's buffer held."""
    inp = make_inputs(workload("online"), batch=8)
    offs = torch.from_numpy(inp.offsets[:1]).cuda()
    out = torch.full((len(inp.dims.keep), 2, 1), 77, dtype=torch.int64, device="cuda")
    st = torch.full((1,), 5, dtype=torch.int32, device="cuda")
    binding.plan_static(inp.dims, offs, max_batch=8, max_len=400, out=out, status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    assert int(out.abs().sum().item()) == 0
