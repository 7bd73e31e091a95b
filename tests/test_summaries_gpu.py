"""GPU parity of the sequence summaries (LLaTTE notes, appendix A.2 item 4:
Z_seq^(k) = LoRAMLP_k(Flatten(Z_raw))) against the fp64 oracle, through the
C ABI.  Covers the tensor-core split-K bottleneck GEMM with 128- and 64-wide
column tiles, its CUDA-core fallback, one and two 128-user row tiles with a
ragged tail, k-slices of one k-block, a bottleneck rank that is not a
multiple of four, and a cross-attention last layer."""
import numpy as np
import pytest
import torch

import oracle
from workloads import Dims, Workload, make_inputs, workload

from gpu_harness import assert_close, make_handle, run, sample_users, to_device

pytestmark = pytest.mark.gpu


def test_tiny_fp32_all_users():
    inp = make_inputs(workload("tiny_sum"))
    h, out = run(inp)
    assert h.status() == 0
    assert out.shape == (inp.batch, 3, 12)
    assert_close(out, oracle.forward(inp), "fp32", "tiny_sum")


@pytest.mark.parametrize("batch", [6, 130, 256])
def test_online_summaries_sampled_users(batch):
    inp = make_inputs(workload("online_sum"), batch=batch)
    h, out = run(inp)
    assert h.status() == 0
    users = sorted(set(sample_users(inp.lengths, 5)) | {batch - 1, max(0, batch - 2)} |
                   ({127, 128} if batch > 128 else set()))
    ref = oracle.forward(inp, users=users)
    assert_close(out[users], ref, "bf16", f"online_sum B={batch}")
    assert np.all(np.isfinite(out))


def _wl(dtype, **kw):
    base = dict(d=128, heads=2, d_head=64, rank=64, d_ctx=16, n_q=5, keep=(300, 130, 0),
                dtype=dtype, n_sum=3, sum_rank=64, d_seq=96)
    base.update(kw)
    return Workload(name="sum_edge", dims=Dims(**base), batch=1, lengths=("fixed", 1), seed=23)


LENGTHS = [0, 1, 2, 127, 128, 129, 300, 0, 255, 3, 17]


@pytest.mark.parametrize("dtype,kw", [
    ("bf16", {}),                                              # N = 192: 64-wide tiles
    ("bf16", dict(n_sum=2, sum_rank=64, d_seq=256)),           # N = 128: 128-wide tiles
    ("bf16", dict(n_sum=2, sum_rank=20, d_seq=34)),            # N = 40: CUDA-core GEMM
    ("bf16", dict(keep=(300, 64))),                            # last layer keeps history
    ("bf16", dict(d=512, heads=8, rank=256, d_ctx=0, n_q=3, keep=(200, 40), n_sum=2,
                  sum_rank=64, d_seq=64)),                     # d = 512: SM-pair GEMMs
    ("fp32", dict(n_sum=3, sum_rank=6, d_seq=10)),             # rank not a multiple of 4
    ("fp32", dict(keep=(50, 50, 9), n_sum=1, sum_rank=33, d_seq=2)),
])
def test_summary_shapes_all_users(dtype, kw):
    inp = make_inputs(_wl(dtype, **kw), lengths=LENGTHS, random_gains=True)
    h, out = run(inp, max_len=max(LENGTHS))
    assert h.status() == 0
    d = inp.dims
    assert out.shape == (len(LENGTHS), d.n_sum, d.d_seq)
    assert_close(out, oracle.forward(inp), dtype, f"summaries {kw}")


def test_summaries_repeatable_and_graph_replay():
    """The split-K partials are summed in slice order: results are bit-exact
    from run to run, eager or replayed from a CUDA graph."""
    inp = make_inputs(workload("online_sum"), batch=40)
    h = make_handle(inp)
    values, offsets, ctx, cand = to_device(inp)
    a = h.forward(values, offsets, ctx, cand).clone()
    b = h.forward(values, offsets, ctx, cand).clone()
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    out = torch.empty_like(a)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        h.forward(values, offsets, ctx, cand, out=out)
    out.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, a)
    assert h.status() == 0
    del g
