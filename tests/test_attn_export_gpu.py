"""GPU parity of the attention-probability statistics (LLaTTE notes, appendix
A.4: cumulative attention on the most recent / the top-k keys, attention by
hours before the request) against the fp64 oracle, through the C ABI; and the
forward output is unchanged by the export."""
import numpy as np
import pytest
import torch

from latent_attention_jagged_b200.binding import LlatteError
from oracle.analysis import attention_stats
from workloads import make_event_ages, make_inputs, workload

from gpu_harness import EXPORT_TOL, assert_close, make_handle, to_device

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,batch,layers,n_hours", [
    ("tiny", None, [0, 1], 48), ("online", 8, [0, 2], 96), ("skewed", 5, [0, 3], 0),
    ("sweep1600", 3, [1], 200)])
def test_export_matches_oracle(name, batch, layers, n_hours):
    inp = make_inputs(workload(name), batch=batch)
    dt = inp.dims.dtype
    ages = make_event_ages(inp.lengths, seed=77)
    h = make_handle(inp)
    values, offsets, ctx, cand = to_device(inp)
    ag = torch.from_numpy(ages).cuda() if n_hours else None
    plain = h.forward(values, offsets, ctx, cand).clone()
    n_k = 11
    for layer in layers:
        out, rec, top, hrs = h.forward_export(values, offsets, ctx, cand, layer=layer, n_k=n_k,
                                              event_age=ag, n_hours=n_hours)
        torch.cuda.synchronize()
        assert h.status() == 0
        assert torch.equal(out, plain)
        R, K, H = attention_stats(inp, layer, n_k, ages if n_hours else None, n_hours)
        tol = EXPORT_TOL[dt]
        assert_close(rec.cpu().numpy().astype(np.float64), R, dt, f"{name} recent l{layer}", tol)
        assert_close(top.cpu().numpy().astype(np.float64), K, dt, f"{name} topk l{layer}", tol)
        if n_hours:
            assert_close(hrs.cpu().numpy().astype(np.float64), H, dt, f"{name} hours l{layer}",
                         tol)
        else:
            assert hrs is None


def test_export_rejects_bad_arguments():
    inp = make_inputs(workload("tiny"))
    h = make_handle(inp)
    values, offsets, ctx, cand = to_device(inp)
    for kw in (dict(layer=2), dict(layer=-1), dict(n_k=0), dict(n_k=17)):
        with pytest.raises(LlatteError):
            h.forward_export(values, offsets, ctx, cand, **kw)
