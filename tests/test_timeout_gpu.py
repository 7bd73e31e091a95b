"""Failure detection on the GPU without a fault: every wait of the tensor-core
kernels is bounded, and a wait that runs out records LLATTE_DEV_TIMEOUT in the
status word and lets the kernel wind down instead of hanging.  Here the
per-head attention is told to wait, with products and tiles in flight, on an
event that never happens (20 us limit); the call must return, report the
timeout, and leave the handle usable: the next forward without the injection
gives the same bits as before."""
import numpy as np
import pytest

from latent_attention_jagged_b200 import binding
from workloads import Dims, Workload, make_inputs

from gpu_harness import run

pytestmark = pytest.mark.gpu


def _tiny_bf16():
    # MLA in its per-head form (the two-tile attention kernel), two layers
    return Workload(name="wait_limit", dims=Dims(d=128, heads=2, d_head=64, rank=64, d_ctx=16,
                                                n_q=5, keep=(300, 130), attn_form=2),
                    batch=1, lengths=("fixed", 1), seed=23)


def test_wait_that_runs_out_is_reported_and_the_handle_recovers():
    inp = make_inputs(_tiny_bf16(), lengths=[0, 1, 2, 127, 128, 129, 300, 0, 255, 3])
    h, good = run(inp, max_len=300)
    assert h.status() == 0
    h.inject_timeout(True)
    run(inp, handle=h)
    st = h.status()
    assert st & binding.DEV_TIMEOUT, st
    h.inject_timeout(False)
    _, again = run(inp, handle=h)
    assert h.status() == 0
    assert np.array_equal(good, again)
    h.close()


def test_injection_needs_a_per_head_layer():
    tiny = make_inputs(Workload(name="t", dims=Dims(d=64, heads=2, d_head=32, rank=32, d_ctx=16,
                                                    n_q=4, keep=(64, 32), dtype="fp32"),
                                batch=2, lengths=("fixed", 8), seed=1))
    h, _ = run(tiny)
    with pytest.raises(binding.LlatteError) as e:
        h.inject_timeout(True)
    assert e.value.code == binding.LLATTE_ERR_UNSUPPORTED
    h.close()
