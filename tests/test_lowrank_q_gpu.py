"""GPU parity of the low-rank RMSNorm'd query (LLaTTE notes, appendix A.3,
first display: Q = RMSNorm(X W_down^Q) W_up^Q, here on the target-aware input
[x ; c]) against the fp64 oracle, through the C ABI.  Covers the tensor-core
path (down-projection GEMM with the per-user context term and the RMSNorm in
its epilogue, then the absorbed projection), with and without context, at
d = 256 and d = 512, and the CUDA-core path (fp32, and bf16 with a query rank
the tensor-core norm tile does not take)."""
import numpy as np
import pytest

import oracle
from workloads import Dims, Workload, make_inputs, workload

from gpu_harness import assert_close, run, sample_users

pytestmark = pytest.mark.gpu


def test_tiny_fp32_all_users():
    inp = make_inputs(workload("tiny_lq"))
    h, out = run(inp)
    assert h.status() == 0
    assert_close(out, oracle.forward(inp), "fp32", "tiny_lq")


@pytest.mark.parametrize("name,n", [("online_lq", 6), ("upstream_lq", 2)])
def test_full_size_sampled_users(name, n):
    inp = make_inputs(workload(name))
    h, out = run(inp)
    assert h.status() == 0
    users = sample_users(inp.lengths, n)
    assert_close(out[users], oracle.forward(inp, users=users), "bf16", name)
    assert np.all(np.isfinite(out))


def _wl(dtype, **kw):
    base = dict(d=128, heads=2, d_head=64, rank=64, d_ctx=16, n_q=5, keep=(300, 130, 0),
                dtype=dtype, q_rank=64)
    base.update(kw)
    return Workload(name="lq_edge", dims=Dims(**base), batch=1, lengths=("fixed", 1), seed=29)


LENGTHS = [0, 1, 2, 127, 128, 129, 300, 0, 255, 3]


@pytest.mark.parametrize("dtype,kw", [
    ("bf16", {}),                                          # tensor cores, context term
    ("bf16", dict(d_ctx=0, q_rank=128, keep=(300, 64))),   # tensor cores, no context
    ("bf16", dict(q_rank=96)),                             # CUDA cores (rank 96)
    ("bf16", dict(d=512, heads=8, rank=256, q_rank=512, keep=(200, 40))),
    ("bf16", dict(n_q=0, d_ctx=0, d_out=64, keep=(256, 64))),
    ("fp32", dict(q_rank=7)),
])
def test_edge_shapes_all_users(dtype, kw):
    inp = make_inputs(_wl(dtype, **kw), lengths=LENGTHS, random_gains=True)
    h, out = run(inp, max_len=max(LENGTHS))
    assert h.status() == 0
    assert_close(out, oracle.forward(inp), dtype, f"low-rank query {kw}")
